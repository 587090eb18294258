// Token reordering between raster and tile-major order.
//
// "NABLA: Neighborhood Adaptive Block-Level Attention" (review, Figure 4 and
// the patch-size parameter P) reorders the flattened video tokens so that a
// spatial neighbourhood becomes one contiguous run ("fractal flattening");
// Sparse VideoGen does the same with a frame-major layout transform.  Here the
// neighbourhood is the 4x4x4 tile that forms one 64-token attention block:
//   raster index      s_r = (t*H + h)*W + w            on the T x H x W grid
//   tile-major index  s_m = ((tt*Th + th)*Tw + tw)*64 + (ut*4 + uh)*4 + uw
// with t = 4tt + ut, h = 4th + uh, w = 4tw + uw.
//
// One CTA per (bh, tile): 64 rows of `row_bytes` each, moved with 16-byte
// vectors.  In raster order the four w-neighbours of a tile row are one
// contiguous run, so both sides of the copy stay coalesced.  HBM-bound:
// bytes = 2 x the tensor.
#include <cuda_runtime.h>
#include <cstdint>

namespace nabla {

__global__ void __launch_bounds__(256) reorder_kernel(const uint4* __restrict__ src,
                                                      uint4* __restrict__ dst, int Tt, int Th,
                                                      int Tw, int vec_per_row, int to_tile_major) {
  const int64_t ntiles = static_cast<int64_t>(Tt) * Th * Tw;
  const int64_t bh = blockIdx.x / ntiles;
  const int64_t tile = blockIdx.x % ntiles;
  const int tw = static_cast<int>(tile % Tw), th = static_cast<int>((tile / Tw) % Th);
  const int tt = static_cast<int>(tile / (static_cast<int64_t>(Tw) * Th));
  const int64_t H = 4ll * Th, W = 4ll * Tw, S = 64ll * ntiles;
  const int64_t head = bh * S;
  const int total = 64 * vec_per_row;
  for (int i = threadIdx.x; i < total; i += blockDim.x) {
    const int u = i / vec_per_row, c = i % vec_per_row;
    const int ut = u >> 4, uh = (u >> 2) & 3, uw = u & 3;
    const int64_t s_r = ((4ll * tt + ut) * H + 4ll * th + uh) * W + 4ll * tw + uw;
    const int64_t s_m = tile * 64 + u;
    const int64_t from = (to_tile_major ? s_r : s_m) + head;
    const int64_t to = (to_tile_major ? s_m : s_r) + head;
    dst[to * vec_per_row + c] = __ldg(src + from * vec_per_row + c);
  }
}

cudaError_t launch_reorder(const void* src, void* dst, int64_t BH, int Tt, int Th, int Tw,
                           int row_bytes, int to_tile_major, cudaStream_t st) {
  const int64_t grid = BH * Tt * Th * Tw;
  if (grid == 0) return cudaSuccess;
  reorder_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(
      static_cast<const uint4*>(src), static_cast<uint4*>(dst), Tt, Th, Tw, row_bytes / 16,
      to_tile_major);
  return cudaGetLastError();
}

}  // namespace nabla
