// libsa.cu — single translation unit of libsa.so, so that the kernels and the
// C ABI share device symbols (the device status word) without relocatable
// device code.
#include "mask_kernels.cu"
#include "attn_kernel.cu"
#include "linear_kernels.cu"
#include "tile_kernels.cu"
#include "permute_kernels.cu"
#include "bwd_kernels.cu"
#include "lin_bwd_kernels.cu"
#include "fp8_kernels.cu"
#include "sa_api.cu"
#include "noalloc.cu"
#include "diag.cu"
