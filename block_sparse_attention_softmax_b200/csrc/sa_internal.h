// sa_internal.h — declarations shared by the translation units of libsa.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "sa_device.cuh"

namespace sa {

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ inline int ceil_div_dev(int a, int b) { return (a + b - 1) / b; }
__host__ __device__ inline long long ceil_div_ll(long long a, long long b) { return (a + b - 1) / b; }

// Block means as four signed 7-bit slices per element plus a per-row power-of-two
// exponent (written by the pooling kernel, read by the integer tensor-core scores).
struct SliceOut {
  int8_t* q_sl;   // [BH, nqb, 4 d]
  int8_t* k_sl;   // [BH, nkb, 4 d]
  int* q_ex;      // [BH, nqb]
  int* k_ex;      // [BH, nkb]
};
cudaError_t launch_pool(const void* q, const void* k, int BH, int N, int d, int bq, int bk,
                        float* q_pool, float* k_pool, cudaStream_t st, const SliceOut* sl = nullptr);
cudaError_t launch_scores_i8(const SliceOut& sl, int BH, int nqb, int nkb, int d, double scale,
                             float* s, long long s_ld, cudaStream_t st);
// Full-row selection over the fp32 score matrix; with `rows`, only the rows
// rows[0 .. *n_rows_dev) (a device-side count).
cudaError_t launch_select(const float* s, long long s_ld, int n_rows, int nkb, int k_sel,
                          double topp, int* kv_idx, int* kv_cnt, uint8_t* mask,
                          cudaStream_t st, const int* rows = nullptr, const int* n_rows_dev = nullptr);

// Candidate path of the mask builder. Its per-row buffers (the candidate
// lists share the score rows' memory, which the handed-back rows reuse after
// the lists are read):
struct CandWs {
  void* st1;        // [rows][16] float4 approximate row statistics per key range and half
  void* st2;        // [rows][16] 16-byte normaliser partials
  void* rowinfo;    // [rows] float2
  int* cand_cnt;    // [rows][2]
  int* fb_cnt;      // 1
  int* fb_rows;     // [rows]
  int* tile_flag;   // [BH * ceil(nqb / 128)]
};
// Bytes of one score row (s_ld floats) or one candidate list, whichever is larger.
inline long long cand_row_bytes(long long s_ld) { return s_ld * 4 > 1024 ? s_ld * 4 : 1024; }
struct CandPlan {
  int want;      // candidates aimed at per row in the first list
  int cap;       // entries of the register selection (128 .. 1024)
  int c_hi;      // capacity of the first list (scores >= t)
  int c_lo;      // capacity of the second list (t_lo <= score < t)
  int all_cand;  // nkb <= cap: every key block is in the first list
  float zq;      // standard normal quantile with upper tail want / nkb (t)
  float zq_lo;   // the same with upper tail (want + 0.9 c_lo) / nkb (t_lo)
};
CandPlan cand_plan(int k_sel, int nkb, long long s_ld);
cudaError_t launch_mask_cand(const SliceOut& sl, int BH, int nqb, int nkb, int d, double scale, int k_sel,
                             double topp, float* s, long long s_ld, const CandWs& cw, int* kv_idx, int* kv_cnt,
                             uint8_t* mask, cudaStream_t st);
cudaError_t launch_compact_mask(const uint8_t* mask, int n_rows, int nkb, int* kv_idx,
                                int* kv_cnt, cudaStream_t st);

// Block-sparse attention over compacted lists. dense != 0 ignores the lists
// and keeps every key block.
struct AttnArgs {
  const void* q;
  const void* k;
  const void* v;
  void* o;
  float* lse;
  const int* kv_idx;
  const int* kv_cnt;
  int BH, N, d, bq, bk, nqb, nkb;
  float scale_log2;
  int dense;
  // optional blend in the epilogue: O = alpha ⊙ O_s + (1 - alpha) ⊙ O_l with
  // O_s still in fp32; alpha [H, d] fp32, o_l [BH, N, d] bf16
  const void* o_l = nullptr;
  const float* alpha = nullptr;
  int H = 1;
  // low-bit form: q, k, v are E4M3 bytes with one fp32 scale per (batch, head)
  // each (d = 128 only)
  int fp8 = 0;
  const float* q_scale = nullptr;
  const float* k_scale = nullptr;
  const float* v_scale = nullptr;
};
cudaError_t launch_sparse_attn(const AttnArgs& a, cudaStream_t st);

// Launch with programmatic stream serialization: the kernel's CTAs may start
// (and run their set-up) while the previous kernel in the stream finishes;
// the kernel itself calls grid_dep_wait() before it touches memory that
// earlier work writes or reads.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
// Per-slice E4M3 quantisation of BH slices of per_slice bf16 values (a multiple
// of 8): x8 codes, scale[BH] = amax / 448 (1 for an all-zero slice).
cudaError_t launch_quantize_fp8(const void* x, long long BH, long long per_slice, uint8_t* x8, float* scale,
                                cudaStream_t st);

struct LinearArgs {
  const void* q;
  const void* k;
  const void* v;
  const void* o_s;      // blend input (may be null when only O_l is wanted)
  const float* alpha;   // [H, d] or null (then O = O_l)
  float* kv_state;
  float* ksum;
  void* o;
  int B, H, N, d;
  void* ws;
};
size_t linear_state_ws_bytes(int BH, int N, int d);
size_t linear_out_ws_bytes(int BH, int d);
cudaError_t launch_linear_state(const LinearArgs& a, cudaStream_t st);
cudaError_t launch_linear_out(const LinearArgs& a, cudaStream_t st);

// Tile scoring: TripPool descriptors and the two-pass max-pooled heatmap.
cudaError_t launch_trip_pool(const void* x, int BH, int N, int d, int b, float* out, cudaStream_t st);
cudaError_t launch_heat(const void* q, const void* k, int BH, int N, int d, int bq, const int* rows, int n_items,
                        double scale, float* heat, float* lse, cudaStream_t st);

// Permuted token layouts: per-head tile-major permutations of a (T, Hh, W)
// grid and the row gather / scatter.
constexpr int kMaxPermHeads = 256;
cudaError_t launch_tile_perm(int H, int T, int Hh, int W, const int* tiles, int* perm, cudaStream_t st);
cudaError_t launch_permute_rows(const void* x, const int* perm, int BH, int H, int N, int d, int inverse, void* y,
                                cudaStream_t st);

// Backward pass of the sparse attention (declared with its argument block in
// bwd_kernels.cu) and the linear branch and blend (linear_kernels.cu).
struct BwdArgs;
size_t bwd_ws_bytes(int BH, int N, int nqb, int nkb);
cudaError_t launch_sparse_attn_bwd(const BwdArgs& a, int d, const void* o, void* ws, cudaStream_t st);
size_t lin_bwd_ws_bytes(int BH, int N, int d);
size_t blend_bwd_ws_bytes(int BH, int N, int d);
cudaError_t launch_linear_bwd(const void* q, const void* k, const void* v, const float* S, const float* z,
                              const void* dol, int BH, int N, int d, float* dq, float* dk, float* dv, int accumulate,
                              void* ws, cudaStream_t st);
cudaError_t launch_blend_bwd(const void* o_s, const void* o_l, const float* alpha, const void* dout, int B, int H,
                             int N, int d, void* do_s, void* do_l, float* dalpha, void* ws, cudaStream_t st);

// Driver entry point for cuTensorMapEncodeTiled, resolved once. 3-D maps
// (inner, rows, planes), 128-byte swizzle, zero fill out of bounds.
CUresult encode_tensor_map_3d_bf16(CUtensorMap* map, const void* base, uint64_t inner,
                                   uint64_t rows, uint64_t planes, uint32_t box_inner,
                                   uint32_t box_rows);
CUresult encode_tensor_map_3d_u8(CUtensorMap* map, const void* base, uint64_t inner,
                                 uint64_t rows, uint64_t planes, uint32_t box_inner,
                                 uint32_t box_rows);

}  // namespace sa
