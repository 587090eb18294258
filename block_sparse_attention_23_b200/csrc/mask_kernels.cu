// NABLA block-mask builder on sm_100a.
//
// Algorithm 1 of "NABLA: Neighborhood Adaptive Block-Level Attention" (as the
// pith.science review reads it in "What carries the argument" and "Core
// claim"): mean-pool Q and K over 64-token blocks, reduced map
// Qbar Kbar^T / sqrt(d), row softmax, keep the smallest descending prefix of
// each row whose mass reaches 1 - thr, then OR in the sliding-tile window of
// "Sliding Tile Attention", and compact to block CSR.
//
// Kernels (all stream-ordered, no host synchronisation):
//   pool_kernel        Q, K bf16 [BH,S,d] -> Qbar, Kbar fp32 [BH,nb,d]     HBM-bound
//   logits_kernel      per head Qbar Kbar^T / sqrt(d) -> L fp32 [BH,nb,nb] fp32 FFMA
//   select_kernel      one warp per row: softmax, prefix selection, STA OR ->
//                      keep bitmap [BH*nb, nw] + counts (+ optional uint8 mask)
//   mask_bits_kernel   external uint8 mask -> keep bitmap + counts
//   scan_kernel        counts -> row_ptr (exclusive scan), nnz, capacity check
//   fill_kernel        keep bitmap -> ascending col_idx per row
//
// The selection step does not sort.  The kept set of the sorted-prefix rule is
// {p > v*} plus the first tied entries (by block index) of value v*, where v*
// is the largest probability whose "mass at or above" reaches 1 - thr; v* is
// found by bisection on the fp32 bit pattern (order-preserving for p >= 0).
// That is the same set a descending sort + cumulative sum selects, with the
// partial sums taken in block order instead of sorted order (fp32 rounding of
// those sums is the only difference).
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_primitives.cuh"

namespace nabla {

// ------------------------------------------------------------------ pooling
// One warp per (tensor, bh, block): 64 rows of d bf16.  A row is d/8 16-byte
// chunks; the warp covers 32/(d/8) rows per step with 128-bit loads.
template <int D>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k,
                                                   float* __restrict__ qbar,
                                                   float* __restrict__ kbar, int64_t nblocks) {
  constexpr int kLanesPerRow = D / 8;            // 16 (d=128) or 8 (d=64)
  constexpr int kRowsPerStep = 32 / kLanesPerRow;  // 2 or 4
  constexpr int kSteps = 64 / kRowsPerStep;        // 32 or 16
  const int lane = threadIdx.x & 31;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (wid >= 2 * nblocks) return;
  const bool is_k = wid >= nblocks;
  const int64_t blk = is_k ? wid - nblocks : wid;
  const __nv_bfloat16* src = (is_k ? k : q) + blk * 64 * D;
  float* dst = (is_k ? kbar : qbar) + blk * D;
  const int chunk = lane % kLanesPerRow;
  const int sub = lane / kLanesPerRow;
  float acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll 8
  for (int s = 0; s < kSteps; ++s) {
    const int row = s * kRowsPerStep + sub;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + row * D) + chunk);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += __uint_as_float(w[i] << 16);
      acc[2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  // combine the row groups (fixed order: deterministic)
#pragma unroll
  for (int off = kLanesPerRow; off < 32; off <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
  }
  if (sub == 0) {
    float4* out = reinterpret_cast<float4*>(dst + chunk * 8);
    out[0] = make_float4(acc[0] * (1.f / 64), acc[1] * (1.f / 64), acc[2] * (1.f / 64),
                         acc[3] * (1.f / 64));
    out[1] = make_float4(acc[4] * (1.f / 64), acc[5] * (1.f / 64), acc[6] * (1.f / 64),
                         acc[7] * (1.f / 64));
  }
}

// ------------------------------------------------------------------ reduced map
// Per head: L = Qbar Kbar^T * inv_sqrt_d, 64x64 output tile per CTA, 4x4 per
// thread, the whole d extent staged transposed in shared memory.  Every
// element is one fixed-order fp32 FMA chain over k (deterministic).
template <int D>
__global__ void __launch_bounds__(256) logits_kernel(const float* __restrict__ qbar,
                                                     const float* __restrict__ kbar,
                                                     float* __restrict__ L, int nb,
                                                     float inv_sqrt_d) {
  constexpr int T = 64, LD = T + 4;
  extern __shared__ float4 logits_smem4[];
  float* As = reinterpret_cast<float*>(logits_smem4);  // [D][LD]: As[k][m]
  float* Bs = As + D * LD;                             // [D][LD]: Bs[k][n]
  const int bh = blockIdx.z;
  const int m0 = blockIdx.y * T, n0 = blockIdx.x * T;
  const float* qa = qbar + static_cast<int64_t>(bh) * nb * D;
  const float* ka = kbar + static_cast<int64_t>(bh) * nb * D;
  const int tid = threadIdx.x;
  for (int i = tid; i < T * (D / 4); i += 256) {
    const int r = i % T, c4 = i / T;   // consecutive threads: consecutive smem columns
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (m0 + r < nb) a = *reinterpret_cast<const float4*>(qa + static_cast<int64_t>(m0 + r) * D + 4 * c4);
    if (n0 + r < nb) b = *reinterpret_cast<const float4*>(ka + static_cast<int64_t>(n0 + r) * D + 4 * c4);
    As[(4 * c4 + 0) * LD + r] = a.x; As[(4 * c4 + 1) * LD + r] = a.y;
    As[(4 * c4 + 2) * LD + r] = a.z; As[(4 * c4 + 3) * LD + r] = a.w;
    Bs[(4 * c4 + 0) * LD + r] = b.x; Bs[(4 * c4 + 1) * LD + r] = b.y;
    Bs[(4 * c4 + 2) * LD + r] = b.z; Bs[(4 * c4 + 3) * LD + r] = b.w;
  }
  __syncthreads();
  const int ty = tid / 16, tx = tid % 16;
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
#pragma unroll 8
  for (int kk = 0; kk < D; ++kk) {
    const float4 a = *reinterpret_cast<const float4*>(As + kk * LD + ty * 4);
    const float4 b = *reinterpret_cast<const float4*>(Bs + kk * LD + tx * 4);
    const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
  }
  float* out = L + static_cast<int64_t>(bh) * nb * nb;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= nb) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < nb) out[static_cast<int64_t>(m) * nb + n] = acc[i][j] * inv_sqrt_d;
    }
  }
}

// ------------------------------------------------------------------ selection

// Butterfly sum; lanes may differ in the last ulp (different association), so
// lane 0's value is broadcast: every lane takes the same branch on it.
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return __shfl_sync(0xffffffffu, v, 0);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// Mass of the row at or above bit pattern v (p >= 0, so bit order = value order).
__device__ __forceinline__ float mass_at_or_above(const float* p, int nb, int lane, uint32_t v) {
  float s = 0.f;
  for (int c = lane; c < nb; c += 32) {
    const float x = p[c];
    s += (__float_as_uint(x) >= v) ? x : 0.f;
  }
  return warp_sum(s);
}

struct SelectParams {
  float thr;
  int use_sta, wt, wh, ww;
  int Tt, Th, Tw;
};

// One warp per row g = bh*nb + r.  Dynamic shared memory: 8 rows x nb floats.
__global__ void __launch_bounds__(256) select_kernel(const float* __restrict__ L, int64_t nrows,
                                                     int nb, SelectParams prm,
                                                     uint32_t* __restrict__ bits,
                                                     int32_t* __restrict__ counts,
                                                     uint8_t* __restrict__ mask_u8) {
  extern __shared__ float sel_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  if (g >= nrows) return;
  const int r = static_cast<int>(g % nb);
  const int nw = (nb + 31) >> 5;
  float* p = sel_smem + warp * nb;
  const float* Lrow = L + g * nb;

  // softmax over the row (max subtracted), p = e / Z
  float mx = -INFINITY;
  for (int c = lane; c < nb; c += 32) {
    const float x = Lrow[c];
    p[c] = x;
    mx = fmaxf(mx, x);
  }
  mx = warp_max(mx);
  float z = 0.f;
  for (int c = lane; c < nb; c += 32) {
    const float e = expf(p[c] - mx);
    p[c] = e;
    z += e;
  }
  z = warp_sum(z);
  uint32_t pmax_bits = 0;
  for (int c = lane; c < nb; c += 32) {
    const float v = p[c] / z;
    p[c] = v;
    pmax_bits = max(pmax_bits, __float_as_uint(v));
  }
  pmax_bits = warp_max_u32(pmax_bits);
  __syncwarp();

  // threshold v*: largest bit pattern whose mass-at-or-above reaches 1 - thr
  const float target = 1.f - prm.thr;
  bool keep_all = prm.thr <= 0.f;
  uint32_t vstar = pmax_bits;
  int tied_keep = 1;
  if (!keep_all) {
    if (target > 0.f) {
      const float total = mass_at_or_above(p, nb, lane, 0u);
      if (total < target) {
        keep_all = true;   // every exclusive prefix stays below the target
      } else {
        uint32_t lo = 0u, hi = pmax_bits + 1u;   // mass(lo) >= target > mass(hi)
        while (hi - lo > 1u) {
          const uint32_t mid = lo + ((hi - lo) >> 1);
          if (mass_at_or_above(p, nb, lane, mid) >= target) lo = mid; else hi = mid;
        }
        vstar = lo;
        const float above = mass_at_or_above(p, nb, lane, vstar + 1u);   // < target
        const float pv = __uint_as_float(vstar);
        int ntied = 0;
        for (int c = lane; c < nb; c += 32) ntied += __float_as_uint(p[c]) == vstar;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) ntied += __shfl_xor_sync(0xffffffffu, ntied, off);
        // tied entries in block order: entry j (0-based) is kept iff above + j*pv < target
        int j = 1;
        while (j < ntied && above + static_cast<float>(j) * pv < target) ++j;
        tied_keep = j;
      }
    }
    // target <= 0 (thr >= 1): only the first entry of the top value (vstar = pmax)
  }

  // flags -> bitmap words, optional uint8 row, STA union, counts
  const int rt = r / (prm.Th * prm.Tw), rh = (r / prm.Tw) % prm.Th, rw = r % prm.Tw;
  int tied_seen = 0, count = 0;
  uint32_t* brow = bits + g * nw;
  uint8_t* mrow = mask_u8 ? mask_u8 + g * nb : nullptr;
  for (int w = 0; w < nw; ++w) {
    const int c = w * 32 + lane;
    const bool inrow = c < nb;
    const uint32_t b = inrow ? __float_as_uint(p[c]) : 0u;
    bool keep;
    if (keep_all) {   // warp-uniform branch
      keep = inrow;
    } else {
      const bool tied = inrow && b == vstar;
      const uint32_t tb = __ballot_sync(0xffffffffu, tied);
      const int rank = tied_seen + __popc(tb & ((1u << lane) - 1u));
      tied_seen += __popc(tb);
      keep = inrow && (b > vstar || (tied && rank < tied_keep));
    }
    if (inrow && prm.use_sta) {
      const int ct = c / (prm.Th * prm.Tw), ch = (c / prm.Tw) % prm.Th, cw = c % prm.Tw;
      keep |= abs(ct - rt) <= prm.wt && abs(ch - rh) <= prm.wh && abs(cw - rw) <= prm.ww;
    }
    if (mrow && inrow) mrow[c] = keep ? 1 : 0;
    const uint32_t word = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) brow[w] = word;
    count += __popc(word);
  }
  if (lane == 0) counts[g] = count;
}

// External uint8 mask row -> bitmap + count.  One warp per row.
__global__ void __launch_bounds__(256) mask_bits_kernel(const uint8_t* __restrict__ mask,
                                                        int64_t nrows, int nb, int vec_ok,
                                                        uint32_t* __restrict__ bits,
                                                        int32_t* __restrict__ counts) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  if (g >= nrows) return;
  const int nw = (nb + 31) >> 5;
  const uint8_t* row = mask + g * nb;
  int count = 0;
  for (int w0 = 0; w0 < nw; w0 += 32) {
    const int w = w0 + lane;           // this lane builds word w from 32 bytes
    uint32_t word = 0;
    if (w < nw) {
      const int c0 = w * 32;
      if (vec_ok && c0 + 32 <= nb) {
        const uint4* src = reinterpret_cast<const uint4*>(row + c0);
        const uint4 a = __ldg(src), b = __ldg(src + 1);
        const uint32_t v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j)
            word |= (((v[i] >> (8 * j)) & 0xFFu) != 0u ? 1u : 0u) << (4 * i + j);
      } else {
        for (int j = 0; j < 32 && c0 + j < nb; ++j) word |= (row[c0 + j] != 0 ? 1u : 0u) << j;
      }
      bits[g * nw + w] = word;
    }
    count += __popc(word);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) count += __shfl_xor_sync(0xffffffffu, count, off);
  if (lane == 0) counts[g] = count;
}

// ------------------------------------------------------------------ CSR
// Single CTA of 1024 threads: exclusive scan of counts into row_ptr.
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* __restrict__ counts,
                                                    int64_t n, int32_t* __restrict__ row_ptr,
                                                    int32_t* __restrict__ nnz_out,
                                                    int64_t capacity, int* status) {
  __shared__ int32_t warp_tot[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t chunk = (n + 1023) / 1024;
  const int64_t b = tid * chunk, e = min(n, b + chunk);
  int32_t local = 0;
  for (int64_t i = b; i < e; ++i) local += counts[i];
  int32_t incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int32_t t = warp_tot[lane];
    int32_t ti = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, ti, off);
      if (lane >= off) ti += y;
    }
    warp_tot[lane] = ti - t;   // exclusive prefix of warp totals
  }
  __syncthreads();
  int32_t run = warp_tot[warp] + incl - local;
  for (int64_t i = b; i < e; ++i) {
    row_ptr[i] = run;
    run += counts[i];
  }
  if (tid == 1023) {
    row_ptr[n] = run;   // last thread's running sum is the grand total
    if (nnz_out) *nnz_out = run;
    if (static_cast<int64_t>(run) > capacity) atomicOr(status, kStatusCapacity);
  }
}

// One warp per row: set bits -> ascending column indices at row_ptr[g].
__global__ void __launch_bounds__(256) fill_kernel(const uint32_t* __restrict__ bits,
                                                   const int32_t* __restrict__ row_ptr,
                                                   int64_t nrows, int nb, int64_t capacity,
                                                   int32_t* __restrict__ col_idx) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  if (g >= nrows) return;
  const int nw = (nb + 31) >> 5;
  int64_t base = row_ptr[g];
  const int64_t end = row_ptr[g + 1];
  if (end > capacity) return;   // capacity overflow is reported by scan_kernel
  const uint32_t* brow = bits + g * nw;
  for (int w = 0; w < nw; ++w) {
    const uint32_t word = brow[w];
    if ((word >> lane) & 1u) col_idx[base + __popc(word & ((1u << lane) - 1u))] = w * 32 + lane;
    base += __popc(word);
  }
}

// ------------------------------------------------------------------ launchers

cudaError_t launch_pool(const void* q, const void* k, float* qbar, float* kbar, int64_t nblocks,
                        int d, cudaStream_t st) {
  const int64_t warps = 2 * nblocks;
  const unsigned grid = static_cast<unsigned>((warps * 32 + 255) / 256);
  if (d == 128)
    pool_kernel<128><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q),
                                            static_cast<const __nv_bfloat16*>(k), qbar, kbar,
                                            nblocks);
  else
    pool_kernel<64><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q),
                                           static_cast<const __nv_bfloat16*>(k), qbar, kbar,
                                           nblocks);
  return cudaGetLastError();
}

cudaError_t launch_logits(const float* qbar, const float* kbar, float* L, int BH, int nb, int d,
                          cudaStream_t st) {
  const dim3 grid((nb + 63) / 64, (nb + 63) / 64, BH);
  const size_t smem = 2ull * d * 68 * sizeof(float);
  const float inv = 1.0f / sqrtf(static_cast<float>(d));
  cudaError_t e;
  if (d == 128) {
    e = cudaFuncSetAttribute(logits_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    logits_kernel<128><<<grid, 256, smem, st>>>(qbar, kbar, L, nb, inv);
  } else {
    e = cudaFuncSetAttribute(logits_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    logits_kernel<64><<<grid, 256, smem, st>>>(qbar, kbar, L, nb, inv);
  }
  return cudaGetLastError();
}

cudaError_t launch_select(const float* L, int64_t nrows, int nb, float thr, int use_sta, int wt,
                          int wh, int ww, int Tt, int Th, int Tw, uint32_t* bits, int32_t* counts,
                          uint8_t* mask_u8, cudaStream_t st) {
  SelectParams prm{thr, use_sta, wt, wh, ww, Tt, Th, Tw};
  const size_t smem = 8ull * nb * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>((nrows + 7) / 8);
  select_kernel<<<grid, 256, smem, st>>>(L, nrows, nb, prm, bits, counts, mask_u8);
  return cudaGetLastError();
}

cudaError_t launch_mask_bits(const uint8_t* mask, int64_t nrows, int nb, uint32_t* bits,
                             int32_t* counts, cudaStream_t st) {
  const int vec_ok = (nb % 16 == 0) && (reinterpret_cast<uintptr_t>(mask) % 16 == 0);
  const unsigned grid = static_cast<unsigned>((nrows + 7) / 8);
  mask_bits_kernel<<<grid, 256, 0, st>>>(mask, nrows, nb, vec_ok, bits, counts);
  return cudaGetLastError();
}

cudaError_t launch_scan_fill(const uint32_t* bits, const int32_t* counts, int64_t nrows, int nb,
                             int32_t* row_ptr, int32_t* col_idx, int64_t capacity,
                             int32_t* nnz_out, int* status, cudaStream_t st) {
  scan_kernel<<<1, 1024, 0, st>>>(counts, nrows, row_ptr, nnz_out, capacity, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>((nrows + 7) / 8);
  fill_kernel<<<grid, 256, 0, st>>>(bits, row_ptr, nrows, nb, capacity, col_idx);
  return cudaGetLastError();
}

}  // namespace nabla
