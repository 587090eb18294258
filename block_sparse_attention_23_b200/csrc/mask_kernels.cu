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
//   pool_kernel        Q, K bf16 [BH,S,d] -> Qbar, Kbar fp64 [BH,nb,d]     HBM-bound
//                      (tile-major or raster token order)
//   logits_kernel      per head Qbar Kbar^T / sqrt(d) -> L fp64 [BH,nb,nb] fp64 FMA
//   select_kernel      one CTA per row: fp64 softmax, prefix (or top-k) selection, STA OR ->
//                      keep bitmap [BH*nb, nw] + counts (+ optional uint8 mask)
//   mask_bits_kernel   external uint8 mask -> keep bitmap + counts
//   scan_kernel        counts -> row_ptr (exclusive scan), nnz, capacity check
//   fill_kernel        keep bitmap -> ascending col_idx per row
//
// The selection step does not sort the row.  Pooling, the reduced map and the
// row probabilities are fp64 (fp32 logits reorder blocks whose probabilities
// agree to a few 1e-6, which moved cuts); the masses are exact fixed-point
// integers of those probabilities, and the cut is located by value binning
// down to at most 32 candidates, which are then ordered exactly (see the
// selection section below).
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_primitives.cuh"

namespace nabla {

// ------------------------------------------------------------------ pooling
// One warp per (tensor, bh, block): 64 rows of d bf16.  A row is d/8 16-byte
// chunks; the warp covers 32/(d/8) rows per step with 128-bit loads.  Sums are
// fp64, so the mean of 64 bf16 values is exact.
// Raster token order (kRaster): block r of a head is tile r of the 4Tt x 4Th x
// 4Tw grid, its row u the token ((4tt + u/16)*H + 4th + (u/4)%4)*W + 4tw + u%4.
template <int D, bool kRaster>
__global__ void __launch_bounds__(256) pool_kernel(const __nv_bfloat16* __restrict__ q,
                                                   const __nv_bfloat16* __restrict__ k,
                                                   double* __restrict__ qbar,
                                                   double* __restrict__ kbar, int64_t nblocks,
                                                   int nb, int Th, int Tw) {
  constexpr int kLanesPerRow = D / 8;              // 16 (d=128) or 8 (d=64)
  constexpr int kRowsPerStep = 32 / kLanesPerRow;  // 2 or 4
  constexpr int kSteps = 64 / kRowsPerStep;        // 32 or 16
  const int lane = threadIdx.x & 31;
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (wid >= 2 * nblocks) return;
  const bool is_k = wid >= nblocks;
  const int64_t blk = is_k ? wid - nblocks : wid;
  const __nv_bfloat16* src = (is_k ? k : q) + blk * 64 * D;   // tile-major: block rows
  int64_t head = 0;
  int tt = 0, th = 0, tw = 0;
  if (kRaster) {   // row u of the block is at head + token offset (see above)
    const int64_t bh = blk / nb;
    const int r = static_cast<int>(blk % nb);
    tw = r % Tw; th = (r / Tw) % Th; tt = r / (Tw * Th);
    head = bh * static_cast<int64_t>(nb) * 64;
    src = (is_k ? k : q) + head * D;
  }
  double* dst = (is_k ? kbar : qbar) + blk * D;
  const int chunk = lane % kLanesPerRow;
  const int sub = lane / kLanesPerRow;
  double acc[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i] = 0.0;
#pragma unroll 8
  for (int s = 0; s < kSteps; ++s) {
    const int row = s * kRowsPerStep + sub;
    int64_t tok = row;
    if (kRaster)
      tok = ((4ll * tt + (row >> 4)) * (4ll * Th) + 4ll * th + ((row >> 2) & 3)) * (4ll * Tw) +
            4ll * tw + (row & 3);
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + tok * D) + chunk);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      acc[2 * i] += static_cast<double>(__uint_as_float(w[i] << 16));
      acc[2 * i + 1] += static_cast<double>(__uint_as_float(w[i] & 0xFFFF0000u));
    }
  }
  // combine the row groups (fixed order: deterministic)
#pragma unroll
  for (int off = kLanesPerRow; off < 32; off <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
  }
  if (sub == 0) {
    double2* out = reinterpret_cast<double2*>(dst + chunk * 8);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      out[i] = make_double2(acc[2 * i] * (1.0 / 64), acc[2 * i + 1] * (1.0 / 64));
  }
}

// ------------------------------------------------------------------ reduced map
// Per head: L = Qbar Kbar^T * inv_sqrt_d in fp64.  A 64 x 128 output tile per
// CTA of 128 threads (two CTAs share an SM, so one CTA's barrier waits and
// loads overlap the other's multiplies); each thread owns rows {2ty, 2ty+1} +
// 16i and columns {2tx, 2tx+1} + 32j (i, j < 4), so its shared-memory reads are
// 16-byte vectors that are broadcast (A) or contiguous across the half-warp
// (B).  k is staged in chunks of 16 through two shared-memory stages, the next
// chunk's global loads in flight while the current one is multiplied.  Every
// element is one fixed-order FMA chain.
constexpr int kLgTM = 64, kLgTN = 128, kLgK = 16, kLgThreads = 128;
constexpr int kLgLdA = kLgTM + 2, kLgLdB = kLgTN + 2;
constexpr int kLgBufA = kLgK * kLgLdA, kLgBufB = kLgK * kLgLdB;   // doubles per operand buffer
constexpr size_t kLgSmem = 2ull * (kLgBufA + kLgBufB) * sizeof(double);   // 2 stages x (A, B)
constexpr int kLgPerA = kLgTM * kLgK / kLgThreads, kLgPerB = kLgTN * kLgK / kLgThreads;

template <int D>
__global__ void __launch_bounds__(kLgThreads, 2) logits_kernel(const double* __restrict__ qbar,
                                                              const double* __restrict__ kbar,
                                                              double* __restrict__ L, int nb,
                                                              double inv_sqrt_d) {
  extern __shared__ double lg_smem[];   // [stage][A [kLgK][kLgLdA] | B [kLgK][kLgLdB]]
  const int bh = blockIdx.z;
  const int m0 = blockIdx.y * kLgTM, n0 = blockIdx.x * kLgTN;
  const double* qa = qbar + static_cast<int64_t>(bh) * nb * D;
  const double* ka = kbar + static_cast<int64_t>(bh) * nb * D;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  // the next chunk is copied straight into its shared-memory stage by 8-byte
  // asynchronous copies (consecutive threads take consecutive k of one row:
  // coalesced 128-byte rows); rows past nb are zero-filled
  auto fetch = [&](int kc, int st) {
    double* As = lg_smem + st * (kLgBufA + kLgBufB);
    double* Bs = As + kLgBufA;
#pragma unroll
    for (int j = 0; j < kLgPerA; ++j) {
      const int i = tid + j * kLgThreads, r = i / kLgK, kk = i % kLgK;
      const bool in = m0 + r < nb;
      const double* src = qa + static_cast<int64_t>(in ? m0 + r : 0) * D + kc + kk;
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_addr(&As[kk * kLgLdA + r])),
                   "l"(src), "r"(in ? 8 : 0) : "memory");
    }
#pragma unroll
    for (int j = 0; j < kLgPerB; ++j) {
      const int i = tid + j * kLgThreads, r = i / kLgK, kk = i % kLgK;
      const bool in = n0 + r < nb;
      const double* src = ka + static_cast<int64_t>(in ? n0 + r : 0) * D + kc + kk;
      asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_addr(&Bs[kk * kLgLdB + r])),
                   "l"(src), "r"(in ? 8 : 0) : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  double acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
  constexpr int kChunks = D / kLgK;
  fetch(0, 0);
#pragma unroll 1
  for (int ch = 0; ch < kChunks; ++ch) {
    const int st = ch & 1;
    // chunk ch landed (this thread's copies), then every thread's
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    if (ch + 1 < kChunks) fetch((ch + 1) * kLgK, st ^ 1);   // in flight during the FMAs below
    const double* As = lg_smem + st * (kLgBufA + kLgBufB);
    const double* Bs = As + kLgBufA;
#pragma unroll
    for (int kk = 0; kk < kLgK; ++kk) {
      double a[8], b[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const double2 va = *reinterpret_cast<const double2*>(&As[kk * kLgLdA + 2 * ty + 16 * i]);
        const double2 vb = *reinterpret_cast<const double2*>(&Bs[kk * kLgLdB + 2 * tx + 32 * i]);
        a[2 * i] = va.x; a[2 * i + 1] = va.y;
        b[2 * i] = vb.x; b[2 * i + 1] = vb.y;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
  }
  double* out = L + static_cast<int64_t>(bh) * nb * nb;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + 2 * ty + 16 * (i >> 1) + (i & 1);
    if (m >= nb) continue;
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      const int n = n0 + 2 * tx + 32 * (j >> 1);
      double* dst = out + static_cast<int64_t>(m) * nb + n;
      if (n + 1 < nb && (nb & 1) == 0) {
        *reinterpret_cast<double2*>(dst) = make_double2(acc[i][j] * inv_sqrt_d, acc[i][j + 1] * inv_sqrt_d);
      } else {
        if (n < nb) dst[0] = acc[i][j] * inv_sqrt_d;
        if (n + 1 < nb) dst[1] = acc[i][j + 1] * inv_sqrt_d;
      }
    }
  }
}

// ------------------------------------------------------------------ selection
//
// One CTA of 128 threads per row g = bh*nb + r.  The row's weights are formed
// in fp64 as the rule states them: v = exp(L - max) (the softmax numerators;
// p = v / z with z their sum), or given non-negative weights v (p = v / z).
// The kept set is the smallest prefix of the row sorted by p descending (equal
// p: lower block index first) whose exclusive prefix mass stays below 1 - thr,
// the first entry always kept.  It is found without sorting the row:
//   - masses are fixed-point integers F = round(v * 2^50 / vmax), so every
//     partial sum is exact and the same in any summation order, and the target
//     is F((1 - thr) * z); comparing sums of v with (1 - thr) * z is the rule
//     E_k < 1 - thr multiplied through by z;
//   - the value range [lo, hi] of the candidates (at first the whole row) is
//     split into 256 equal bins, a monotone map, so the bins are ordered
//     intervals of v; the candidates' masses and counts are histogrammed with
//     shared-memory integer atomics (in the same pass that forms v at the first
//     level); a scan from the top bin finds the bin in which the cumulative mass
//     reaches the target; entries of higher bins are kept, of lower bins
//     dropped, and the crossing bin's entries are the next candidates (their
//     range is the next level's [lo, hi]);
//   - once at most 32 candidates remain one warp orders them exactly on
//     (p = v / z desc, block index asc) by a bitonic network, and each one's
//     exclusive prefix mass decides it; candidates that all share one value are
//     taken in block order.
// Top-k mode does the same with a count of 1 per entry as the mass and k as
// the target.  The sliding-tile window is OR-ed in as one run of columns per
// (t, h) row of the window.

constexpr int kSelBins = 256;
constexpr double kSelFix = 1125899906842624.0;   // 2^50: mass of the row's largest entry
constexpr int kSelMaxLevels = 16;                // binning levels (8 always suffice for fp64)

struct SelectParams {
  float thr;
  int use_sta, wt, wh, ww;
  int Tt, Th, Tw;
  int topk;        // > 0: keep the topk most probable blocks instead of the mass rule
};

// Shared memory of one row: v [nb] fp64, keep and candidate bitmaps [nw] u32
// each, bin masses [256] u64, bin counts [256] u32, and a small exchange area
// for the CTA's reductions and the last candidates (8-byte aligned parts).
constexpr int kSelThreads = 128, kSelWarps = kSelThreads / 32;
constexpr size_t kSelXchBytes = 8 * 8 * kSelWarps + 64 + 4 * 32 + 4 * 132;
__host__ __device__ inline size_t select_row_bytes(int nb) {
  const size_t n = static_cast<size_t>(nb), nw2 = ((n + 31) / 32 + 1) & ~static_cast<size_t>(1);
  return 8 * n + 8 * nw2 + 12 * static_cast<size_t>(kSelBins) + kSelXchBytes;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return __shfl_sync(0xffffffffu, v, 0);
}

__device__ __forceinline__ double warp_max(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

__device__ __forceinline__ double warp_min(double v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmin(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Bin of v in [lo, hi] split into kSelBins equal parts (s = kSelBins / (hi - lo)).
__device__ __forceinline__ int sel_bin(double v, double lo, double s) {
  return static_cast<int>(fmin((v - lo) * s, static_cast<double>(kSelBins - 1)));
}

// Set bits [c0, c1] of a bitmap (shared memory, atomically).
__device__ __forceinline__ void sel_set_run(uint32_t* bm, int c0, int c1) {
  for (int w = c0 >> 5; w <= (c1 >> 5); ++w) {
    const int lo = max(c0, w * 32) - w * 32, hi = min(c1, w * 32 + 31) - w * 32;
    const uint32_t m = (hi == 31 ? 0xffffffffu : ((1u << (hi + 1)) - 1u)) & ~((1u << lo) - 1u);
    atomicOr(&bm[w], m);
  }
}

template <bool kWeights>
__global__ void __launch_bounds__(kSelThreads) select_kernel(const void* __restrict__ in,
                                                             int64_t nrows, int nb,
                                                             SelectParams prm,
                                                             uint32_t* __restrict__ bits,
                                                             int32_t* __restrict__ counts,
                                                             uint8_t* __restrict__ mask_u8,
                                                             int32_t* __restrict__ votes) {
  extern __shared__ __align__(16) unsigned char sel_smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t g = blockIdx.x;
  if (g >= nrows) return;
  const unsigned full = 0xffffffffu;
  const int r = static_cast<int>(g % nb);
  const int nw = (nb + 31) >> 5;
  const int nw2 = (nw + 1) & ~1;
  double* pv = reinterpret_cast<double*>(sel_smem);
  uint32_t* kbits = reinterpret_cast<uint32_t*>(sel_smem + 8ull * nb);   // kept entries
  uint32_t* cbits = kbits + nw2;                                          // candidates
  unsigned long long* hm = reinterpret_cast<unsigned long long*>(cbits + nw2);
  uint32_t* hc = reinterpret_cast<uint32_t*>(hm + kSelBins);
  double* xd = reinterpret_cast<double*>(hc + kSelBins);                  // [2 * kSelWarps]
  unsigned long long* xu = reinterpret_cast<unsigned long long*>(xd + 2 * kSelWarps);  // [kSelWarps]
  int* xi = reinterpret_cast<int*>(xu + kSelWarps);                       // [2 * kSelWarps]
  unsigned long long* xs = reinterpret_cast<unsigned long long*>(xi + 2 * kSelWarps);  // [4]
  int* slot = reinterpret_cast<int*>(xs + 4);                             // [32] last candidates
  int* wpre = slot + 32;                                                  // [nw + 1] word prefix

  const bool topk_mode = prm.topk > 0;
  const bool keep_all_rule = topk_mode ? prm.topk >= nb : prm.thr <= 0.f;
  for (int w = tid; w < nw2; w += kSelThreads) {
    kbits[w] = 0u;
    cbits[w] = 0u;
  }
  for (int i = tid; i < kSelBins; i += kSelThreads) {
    hm[i] = 0ull;
    hc[i] = 0u;
  }

  // ---- pass 1: range of the row (max and min of L, or of the weights)
  const double* Lrow = static_cast<const double*>(in) + g * nb;
  const float* Wrow = static_cast<const float*>(in) + g * nb;
  double a = -INFINITY, b = INFINITY;
  for (int c = tid; c < nb; c += kSelThreads) {
    double x;
    if (kWeights) {
      const float w = Wrow[c];
      x = w > 0.f ? static_cast<double>(w) : 0.0;   // negative or NaN weights count as zero
      pv[c] = x;
    } else {
      x = Lrow[c];
    }
    a = fmax(a, x);
    b = fmin(b, x);
  }
  a = warp_max(a);
  b = warp_min(b);
  if (lane == 0) {
    xd[warp] = a;
    xd[kSelWarps + warp] = b;
  }
  __syncthreads();
  double vmax = xd[0], vmin = xd[kSelWarps];
#pragma unroll
  for (int w = 1; w < kSelWarps; ++w) {
    vmax = fmax(vmax, xd[w]);
    vmin = fmin(vmin, xd[kSelWarps + w]);
  }
  // logits: v = exp(L - max) lies in [exp(min - max), 1]
  const double mx = vmax;
  double lo = kWeights ? vmin : exp(vmin - mx);
  double hi = kWeights ? vmax : 1.0;
  const double sigma = kWeights ? (vmax > 0.0 ? kSelFix / vmax : 0.0) : kSelFix;

  // ---- pass 2: v, its sum, the total mass, and the first level's histogram
  const bool bin0 = !keep_all_rule && hi > lo;
  const double s0 = bin0 ? fmin(kSelBins / (hi - lo), 1.7976931348623157e308) : 0.0;
  double zl = 0.0;
  unsigned long long tot = 0;
  for (int c = tid; c < nb; c += kSelThreads) {
    double v;
    if (kWeights) {
      v = pv[c];
    } else {
      v = exp(Lrow[c] - mx);
      pv[c] = v;
    }
    zl += v;
    const unsigned long long f = topk_mode ? 1ull : __double2ull_rn(v * sigma);
    tot += f;
    if (bin0) {
      const int bb = sel_bin(v, lo, s0);
      atomicAdd(&hm[bb], f);
      atomicAdd(&hc[bb], 1u);
    }
  }
  zl = warp_sum(zl);
  tot = warp_sum_u64(tot);
  __syncthreads();   // xd consumed
  if (lane == 0) {
    xd[warp] = zl;
    xu[warp] = tot;
  }
  __syncthreads();
  double z = xd[0];
  tot = xu[0];
#pragma unroll
  for (int w = 1; w < kSelWarps; ++w) {
    z += xd[w];
    tot += xu[w];
  }
  const bool empty_row = kWeights && !(z > 0.0);

  // ---- the kept set (every branch below is uniform across the CTA)
  bool keep_all = keep_all_rule;
  unsigned long long T = 0;   // target: fixed-point mass, or the count k
  if (topk_mode) {
    T = static_cast<unsigned long long>(prm.topk);
  } else {
    const double t = 1.0 - static_cast<double>(prm.thr);
    T = t > 0.0 ? __double2ull_rn(t * z * sigma) : 0ull;
    // every exclusive prefix stays below the target when the whole row does
    if (!keep_all && !empty_row) keep_all = tot < T;
  }
  if (!keep_all && !empty_row) {
    unsigned long long above = 0;   // mass (or count) of the entries ranked above the candidates
    uint32_t above_n = 0;           // number of those entries
    int n_c = nb;                   // candidates: every entry at level 0, then those of cbits
    bool all = true;
    // entry c = i0 + tid: warp w of a chunk owns bitmap word i0/32 + w
    for (int level = 0; level < kSelMaxLevels && n_c > 32 && hi > lo; ++level) {
      const double sl = level == 0 ? s0 : fmin(kSelBins / (hi - lo), 1.7976931348623157e308);
      if (level > 0) {
        for (int i = tid; i < kSelBins; i += kSelThreads) {
          hm[i] = 0ull;
          hc[i] = 0u;
        }
        __syncthreads();
        for (int c = tid; c < nb; c += kSelThreads) {
          if (!((cbits[c >> 5] >> (c & 31)) & 1u)) continue;
          const double v = pv[c];
          const int bb = sel_bin(v, lo, sl);
          atomicAdd(&hm[bb], topk_mode ? 1ull : __double2ull_rn(v * sigma));
          atomicAdd(&hc[bb], 1u);
        }
        __syncthreads();
      }
      if (warp == 0) {
        // lane l holds bins [8l, 8l+8); suffix sums over lanes >= l (inclusive)
        unsigned long long loc = 0;
        uint32_t locn = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          loc += hm[8 * lane + j];
          locn += hc[8 * lane + j];
        }
        unsigned long long suf = loc;
        uint32_t sufn = locn;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const unsigned long long y = __shfl_down_sync(full, suf, off);
          const uint32_t yn = __shfl_down_sync(full, sufn, off);
          if (lane + off < 32) {
            suf += y;
            sufn += yn;
          }
        }
        // the crossing bin lies in the highest lane whose suffix reaches the
        // target (lane 0's suffix is every candidate, which always does)
        const uint32_t bal = __ballot_sync(full, above + suf >= T);
        const int cl = 31 - __clz(bal | 1u);
        if (lane == cl) {
          unsigned long long run = above + (suf - loc);
          uint32_t runn = above_n + (sufn - locn);
          int bb = 8 * lane + 7;
          for (; bb > 8 * lane; --bb) {
            if (run + hm[bb] >= T) break;
            run += hm[bb];
            runn += hc[bb];
          }
          xi[0] = bb;
          xi[1] = static_cast<int>(hc[bb]);
          xs[0] = run;
          xs[1] = runn;
        }
      }
      __syncthreads();
      const int bstar = xi[0];
      above = xs[0];
      above_n = static_cast<uint32_t>(xs[1]);
      // keep the higher bins; the crossing bin's entries are the next candidates
      double nlo = INFINITY, nhi = -INFINITY;
      for (int i0 = 0; i0 < nb; i0 += kSelThreads) {
        const int c = i0 + tid;
        const int w = c >> 5;
        bool cand = false, keep = false;
        if (c < nb && (all || ((cbits[w] >> lane) & 1u))) {
          const double v = pv[c];
          const int bb = sel_bin(v, lo, sl);
          keep = bb > bstar;
          cand = bb == bstar;
          if (cand) {
            nlo = fmin(nlo, v);
            nhi = fmax(nhi, v);
          }
        }
        const uint32_t kb = __ballot_sync(full, keep), cb = __ballot_sync(full, cand);
        if (lane == 0 && w < nw) {
          kbits[w] |= kb;
          cbits[w] = cb;
        }
      }
      n_c = xi[1];
      all = false;
      nlo = warp_min(nlo);
      nhi = warp_max(nhi);
      __syncthreads();   // xi, xs consumed; cbits and kbits written
      if (lane == 0) {
        xd[warp] = nlo;
        xd[kSelWarps + warp] = nhi;
      }
      __syncthreads();
      lo = xd[0];
      hi = xd[kSelWarps];
#pragma unroll
      for (int w = 1; w < kSelWarps; ++w) {
        lo = fmin(lo, xd[w]);
        hi = fmax(hi, xd[kSelWarps + w]);
      }
    }
    if (n_c <= 32) {
      if (warp == 0) {
        // gather the candidates (ascending index) into slot[0 .. n_c)
        int base = 0;
        for (int w0 = 0; w0 < nw; w0 += 32) {
          const int w = w0 + lane;
          uint32_t bitsw = 0u;
          if (w < nw)
            bitsw = all ? ((w == nw - 1 && (nb & 31)) ? (1u << (nb & 31)) - 1u : full) : cbits[w];
          const int cnt = __popc(bitsw);
          int incl = cnt;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(full, incl, off);
            if (lane >= off) incl += y;
          }
          int pos = base + incl - cnt;
          while (bitsw) {
            const int bit = __ffs(bitsw) - 1;
            bitsw &= bitsw - 1;
            if (pos < 32) slot[pos] = w * 32 + bit;
            ++pos;
          }
          base += __shfl_sync(full, incl, 31);
        }
        __syncwarp();
        // exact order of the last candidates: bitonic network on
        // (p = v / z desc, index asc); masses from v
        const int c = lane < n_c ? slot[lane] : -1;
        const double v = c >= 0 ? pv[c] : 0.0;
        unsigned long long key =
            c >= 0 ? static_cast<unsigned long long>(__double_as_longlong(v / z)) : 0ull;
        unsigned long long f =
            c >= 0 ? (topk_mode ? 1ull : __double2ull_rn(v * sigma)) : 0ull;
        int idx = c >= 0 ? c : 0x7fffffff;
#pragma unroll
        for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
          for (int j = k >> 1; j > 0; j >>= 1) {
            const unsigned long long ok = __shfl_xor_sync(full, key, j);
            const unsigned long long of = __shfl_xor_sync(full, f, j);
            const int oi = __shfl_xor_sync(full, idx, j);
            const bool other_first = ok > key || (ok == key && oi < idx);
            const bool lower = (lane & j) == 0, up = (lane & k) == 0;
            if ((lower == up) ? other_first : !other_first) {
              key = ok;
              f = of;
              idx = oi;
            }
          }
        }
        const bool valid = idx != 0x7fffffff;
        unsigned long long incl = f;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const unsigned long long y = __shfl_up_sync(full, incl, off);
          if (lane >= off) incl += y;
        }
        const bool keep = valid && ((above_n == 0 && lane == 0) || above + (incl - f) < T);
        if (keep) atomicOr(&kbits[idx >> 5], 1u << (idx & 31));
      }
    } else {
      // the candidates share one value (or the level cap was reached): the
      // first nkeep of them in block order
      if (warp == 0) {
        // exclusive prefix of candidate counts over the words, and the first candidate
        int base = 0, first = 0x7fffffff;
        for (int w0 = 0; w0 < nw; w0 += 32) {
          const int w = w0 + lane;
          const uint32_t bitsw = w < nw ? cbits[w] : 0u;
          if (bitsw) first = min(first, w * 32 + __ffs(bitsw) - 1);
          const int cnt = __popc(bitsw);
          int incl = cnt;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(full, incl, off);
            if (lane >= off) incl += y;
          }
          if (w < nw) wpre[w] = base + incl - cnt;
          base += __shfl_sync(full, incl, 31);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) first = min(first, __shfl_xor_sync(full, first, off));
        if (lane == 0) xi[0] = all ? 0 : first;
      }
      __syncthreads();
      const int c0 = xi[0];
      const unsigned long long f = topk_mode ? 1ull : __double2ull_rn(pv[c0] * sigma);
      int nkeep = 0;
      if (above < T) {
        const unsigned long long need = (T - above + f - 1) / (f > 0 ? f : 1ull);
        nkeep = (f == 0 || need >= static_cast<unsigned long long>(n_c)) ? n_c : static_cast<int>(need);
      }
      if (above_n == 0 && nkeep == 0) nkeep = 1;
      for (int c = tid; c < nb; c += kSelThreads) {
        const int w = c >> 5;
        bool take;
        if (all) {
          take = c < nkeep;
        } else {
          const uint32_t bitsw = cbits[w];
          take = ((bitsw >> (c & 31)) & 1u) && wpre[w] + __popc(bitsw & ((1u << (c & 31)) - 1u)) < nkeep;
        }
        if (take) atomicOr(&kbits[w], 1u << (c & 31));
      }
    }
  } else if (keep_all && !empty_row) {
    for (int w = tid; w < nw; w += kSelThreads)
      kbits[w] = (w == nw - 1 && (nb & 31)) ? (1u << (nb & 31)) - 1u : full;
  }
  __syncthreads();

  // ---- the sliding-tile window: one run of columns per (t, h) of the window
  if (prm.use_sta) {
    const int thw = prm.Th * prm.Tw;
    const int rt = r / thw, rh = (r / prm.Tw) % prm.Th, rw = r % prm.Tw;
    const int nh = 2 * prm.wh + 1, nrun = (2 * prm.wt + 1) * nh;
    const int w0 = max(rw - prm.ww, 0), w1 = min(rw + prm.ww, prm.Tw - 1);
    for (int j = tid; j < nrun; j += kSelThreads) {
      const int t = rt - prm.wt + j / nh, h = rh - prm.wh + j % nh;
      if (t < 0 || t >= prm.Tt || h < 0 || h >= prm.Th) continue;
      const int base = (t * prm.Th + h) * prm.Tw;
      sel_set_run(kbits, base + w0, base + w1);
    }
    __syncthreads();
  }

  // ---- outputs: bitmap words, count, optional uint8 row and votes
  int count = 0;
  for (int w = tid; w < nw; w += kSelThreads) {
    const uint32_t word = kbits[w];
    if (bits) bits[g * nw + w] = word;
    count += __popc(word);
  }
  if (mask_u8 || votes) {
    for (int c = tid; c < nb; c += kSelThreads) {
      const bool keep = (kbits[c >> 5] >> (c & 31)) & 1u;
      if (mask_u8) mask_u8[g * nb + c] = keep ? 1 : 0;
      if (votes && keep) votes[g * nb + c] += 1;
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) count += __shfl_xor_sync(full, count, off);
  if (lane == 0) xi[2 + warp] = count;
  __syncthreads();
  if (counts && tid == 0) {
    int total = 0;
    for (int w = 0; w < kSelWarps; ++w) total += xi[2 + w];
    counts[g] = total;
  }
}

// Calibrated mask from accumulated votes: keep (r, c) iff votes >= min_votes.
__global__ void __launch_bounds__(256) vote_mask_kernel(const int32_t* __restrict__ votes,
                                                        int64_t n, int32_t min_votes,
                                                        uint8_t* __restrict__ mask) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    mask[i] = votes[i] >= min_votes ? 1 : 0;
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


cudaError_t launch_pool(const void* q, const void* k, double* qbar, double* kbar,
                        int64_t nblocks, int d, int nb, int raster, int Th, int Tw,
                        cudaStream_t st) {
  const int64_t warps = 2 * nblocks;
  const unsigned grid = static_cast<unsigned>((warps * 32 + 255) / 256);
  const __nv_bfloat16* qq = static_cast<const __nv_bfloat16*>(q);
  const __nv_bfloat16* kk = static_cast<const __nv_bfloat16*>(k);
  if (raster) {
    if (d == 128) pool_kernel<128, true><<<grid, 256, 0, st>>>(qq, kk, qbar, kbar, nblocks, nb, Th, Tw);
    else pool_kernel<64, true><<<grid, 256, 0, st>>>(qq, kk, qbar, kbar, nblocks, nb, Th, Tw);
  } else {
    if (d == 128) pool_kernel<128, false><<<grid, 256, 0, st>>>(qq, kk, qbar, kbar, nblocks, nb, Th, Tw);
    else pool_kernel<64, false><<<grid, 256, 0, st>>>(qq, kk, qbar, kbar, nblocks, nb, Th, Tw);
  }
  return cudaGetLastError();
}

cudaError_t launch_logits(const double* qbar, const double* kbar, double* L, int BH, int nb,
                          int d, cudaStream_t st) {
  const dim3 grid((nb + kLgTN - 1) / kLgTN, (nb + kLgTM - 1) / kLgTM, BH);
  const double inv = 1.0 / sqrt(static_cast<double>(d));
  cudaError_t e;
  if (d == 128) {
    e = cudaFuncSetAttribute(logits_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kLgSmem));
    if (e != cudaSuccess) return e;
    logits_kernel<128><<<grid, kLgThreads, kLgSmem, st>>>(qbar, kbar, L, nb, inv);
  } else {
    e = cudaFuncSetAttribute(logits_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kLgSmem));
    if (e != cudaSuccess) return e;
    logits_kernel<64><<<grid, kLgThreads, kLgSmem, st>>>(qbar, kbar, L, nb, inv);
  }
  return cudaGetLastError();
}

cudaError_t launch_select(const double* L, int64_t nrows, int nb, float thr, int topk,
                          int use_sta, int wt, int wh, int ww, int Tt, int Th, int Tw,
                          uint32_t* bits, int32_t* counts, uint8_t* mask_u8, cudaStream_t st) {
  SelectParams prm{thr, use_sta, wt, wh, ww, Tt, Th, Tw, topk};
  const size_t smem = select_row_bytes(nb);
  cudaError_t e = cudaFuncSetAttribute(select_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  select_kernel<false><<<static_cast<unsigned>(nrows), kSelThreads, smem, st>>>(
      L, nrows, nb, prm, bits, counts, mask_u8, nullptr);
  return cudaGetLastError();
}

// The selection (a4-a6) on given non-negative block weights instead of the
// softmax of the pooled map: each row normalised by its sum, then the mass
// rule at thr or the top-k rule, then the STA window.
cudaError_t launch_select_weights(const float* weights, int64_t nrows, int nb, float thr, int topk,
                                  int use_sta, int wt, int wh, int ww, int Tt, int Th, int Tw,
                                  uint32_t* bits, int32_t* counts, uint8_t* mask_u8,
                                  cudaStream_t st) {
  SelectParams prm{thr, use_sta, wt, wh, ww, Tt, Th, Tw, topk};
  const size_t smem = select_row_bytes(nb);
  cudaError_t e = cudaFuncSetAttribute(select_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  select_kernel<true><<<static_cast<unsigned>(nrows), kSelThreads, smem, st>>>(
      weights, nrows, nb, prm, bits, counts, mask_u8, nullptr);
  return cudaGetLastError();
}

cudaError_t launch_calib_select(const float* energy, int64_t nrows, int nb, float eps,
                                int32_t* votes, cudaStream_t st) {
  SelectParams prm{eps, 0, 0, 0, 0, 1, 1, 1, 0};
  const size_t smem = select_row_bytes(nb);
  cudaError_t e = cudaFuncSetAttribute(select_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  select_kernel<true><<<static_cast<unsigned>(nrows), kSelThreads, smem, st>>>(
      energy, nrows, nb, prm, nullptr, nullptr, nullptr, votes);
  return cudaGetLastError();
}

cudaError_t launch_vote_mask(const int32_t* votes, int64_t n, int32_t min_votes, uint8_t* mask,
                             cudaStream_t st) {
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  vote_mask_kernel<<<static_cast<unsigned>(blocks), 256, 0, st>>>(votes, n, min_votes, mask);
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
