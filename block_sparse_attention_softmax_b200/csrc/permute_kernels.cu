// permute_kernels.cu — permuted token layouts for the block-sparse path (pages:
// "Veda" §2.2, a tiling (p_t, p_h, p_w) of the latent grid chosen per head;
// "SparsePR" §2C, tokens reordered into a contiguous group-major layout before
// the block-sparse call). The sparse path then runs unchanged on the permuted
// sequence, whose blocks are runs of consecutive permuted tokens, and the
// output is scattered back.
//
// tile_perm_kernel   perm[h, pos] = raster index of the token at position pos of
//                    head h's tile-major order. Each thread takes one token
//                    (t, y, x) and computes its position in closed form: the
//                    tokens of all earlier tiles (edge tiles may be partial)
//                    plus its raster rank inside its own tile.
// permute_rows_kernel one warp per pair of token rows, 16-byte copies:
//                    gather y[bh, i] = x[bh, perm[h, i]] or the inverse scatter
//                    y[bh, perm[h, i]] = x[bh, i].
#include "sa_internal.h"

namespace sa {

struct TileSet {
  int tiles[kMaxPermHeads][3];   // (p_t, p_h, p_w) per head
};

__global__ void tile_perm_kernel(int H, int T, int Hh, int W, TileSet ts, int* __restrict__ perm) {
  const long long N = static_cast<long long>(T) * Hh * W;
  const long long g = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (g >= N * H) return;
  const int h = static_cast<int>(g / N);
  const int r = static_cast<int>(g % N);          // raster index of the token
  const int t = r / (Hh * W), y = (r / W) % Hh, x = r % W;
  const int pt = ts.tiles[h][0], ph = ts.tiles[h][1], pw = ts.tiles[h][2];
  const int a = t / pt, b = y / ph, c = x / pw;   // tile coordinates
  const int ta = min(pt, T - a * pt);             // extent of this tile along t, y, x
  const int hb = min(ph, Hh - b * ph);
  const int wc = min(pw, W - c * pw);
  long long pos = static_cast<long long>(a * pt) * Hh * W           // earlier tile layers
                  + static_cast<long long>(ta) * (b * ph) * W        // earlier tile rows of this layer
                  + static_cast<long long>(ta) * hb * (c * pw)       // earlier tiles of this row
                  + (static_cast<long long>(t - a * pt) * hb + (y - b * ph)) * wc + (x - c * pw);
  perm[static_cast<long long>(h) * N + pos] = r;
}

template <int D>
__global__ void __launch_bounds__(256) permute_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                           const int* __restrict__ perm, int H, int N,
                                                           long long rows, int inverse,
                                                           __nv_bfloat16* __restrict__ y) {
  constexpr int LPR = D / 8;                     // lanes per row (16 B each)
  constexpr int RPW = 32 / LPR;                  // rows per warp
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long gr = warp * RPW + lane / LPR;  // (bh, i) row of the destination walk
  if (gr >= rows) return;
  const long long bh = gr / N;
  const int i = static_cast<int>(gr % N);
  const int p = __ldg(perm + static_cast<long long>(bh % H) * N + i);
  const long long src = inverse ? gr : bh * N + p;
  const long long dst = inverse ? bh * N + p : gr;
  const int c8 = (lane % LPR) * 8;
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(x + src * D + c8));
  *reinterpret_cast<uint4*>(y + dst * D + c8) = v;
}

cudaError_t launch_tile_perm(int H, int T, int Hh, int W, const int* tiles, int* perm, cudaStream_t st) {
  TileSet ts;
  for (int h = 0; h < H; ++h)
    for (int j = 0; j < 3; ++j) ts.tiles[h][j] = tiles[h * 3 + j];
  const long long total = static_cast<long long>(T) * Hh * W * H;
  const long long grid = (total + 255) / 256;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  tile_perm_kernel<<<static_cast<int>(grid), 256, 0, st>>>(H, T, Hh, W, ts, perm);
  return cudaGetLastError();
}

cudaError_t launch_permute_rows(const void* x, const int* perm, int BH, int H, int N, int d, int inverse, void* y,
                                cudaStream_t st) {
  const long long rows = static_cast<long long>(BH) * N;
  const int rpw = 32 / (d / 8);
  const long long warps = (rows + rpw - 1) / rpw;
  const long long grid = (warps * 32 + 255) / 256;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  if (d == 128)
    permute_rows_kernel<128><<<static_cast<int>(grid), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), perm, H, N, rows, inverse, static_cast<__nv_bfloat16*>(y));
  else
    permute_rows_kernel<64><<<static_cast<int>(grid), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), perm, H, N, rows, inverse, static_cast<__nv_bfloat16*>(y));
  return cudaGetLastError();
}

}  // namespace sa
