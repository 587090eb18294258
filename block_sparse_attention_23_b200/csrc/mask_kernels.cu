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
//   select_kernel      one warp per row: softmax, prefix (or top-k) selection, STA OR ->
//                      keep bitmap [BH*nb, nw] + counts (+ optional uint8 mask)
//   mask_bits_kernel   external uint8 mask -> keep bitmap + counts
//   scan_kernel        counts -> row_ptr (exclusive scan), nnz, capacity check
//   fill_kernel        keep bitmap -> ascending col_idx per row
//
// The selection step does not sort.  The kept set of the sorted-prefix rule is
// {p > v*} plus the first tied entries (by block index) of value v*, where v*
// is the largest probability whose "mass at or above" reaches 1 - thr; v* is
// found by bisection on the fp32 bit pattern (order-preserving for p >= 0).
// That is the set a descending sort + cumulative sum selects, with the partial
// sums taken in block order instead of sorted order.  Pooling and the reduced
// map are fp64 (fp32 logits reorder blocks whose probabilities agree to a few
// 1e-6, which moved cuts); the row softmax and the masses are fp32 values
// from the fp64 map, summed in fp64 across each warp.
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
// Per head: L = Qbar Kbar^T * inv_sqrt_d in fp64.  128x128 output tile per CTA
// of 256 threads; each thread owns rows {2ty, 2ty+1} + 32i and columns
// {2tx, 2tx+1} + 32j (i, j < 4), so its shared-memory reads are 16-byte
// vectors that are broadcast (A) or contiguous across the half-warp (B).
// k is staged in chunks of 16 through two shared-memory stages, the next
// chunk's global loads in flight while the current one is multiplied.  Every
// element is one fixed-order FMA chain.
constexpr int kLgT = 128, kLgK = 16, kLgLD = kLgT + 2;
constexpr int kLgBuf = kLgK * kLgLD;                       // doubles per operand buffer
constexpr size_t kLgSmem = 2ull * 2 * kLgBuf * sizeof(double);   // 2 stages x (A, B)

template <int D>
__global__ void __launch_bounds__(256) logits_kernel(const double* __restrict__ qbar,
                                                     const double* __restrict__ kbar,
                                                     double* __restrict__ L, int nb,
                                                     double inv_sqrt_d) {
  extern __shared__ double lg_smem[];   // [stage][A | B][kLgK][kLgLD]; As[k][m], Bs[k][n]
  const int bh = blockIdx.z;
  const int m0 = blockIdx.y * kLgT, n0 = blockIdx.x * kLgT;
  const double* qa = qbar + static_cast<int64_t>(bh) * nb * D;
  const double* ka = kbar + static_cast<int64_t>(bh) * nb * D;
  const int tid = threadIdx.x, ty = tid / 16, tx = tid % 16;
  // each thread moves 8 elements of A and 8 of B per k-chunk; consecutive
  // threads take consecutive k of one row (coalesced 128-byte rows)
  double ra[8], rb[8];
  auto fetch = [&](int kc) {
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = tid + j * 256, r = i / kLgK, kk = i % kLgK;
      ra[j] = (m0 + r < nb) ? qa[static_cast<int64_t>(m0 + r) * D + kc + kk] : 0.0;
      rb[j] = (n0 + r < nb) ? ka[static_cast<int64_t>(n0 + r) * D + kc + kk] : 0.0;
    }
  };
  auto stash = [&](int st) {
    double* As = lg_smem + st * 2 * kLgBuf;
    double* Bs = As + kLgBuf;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = tid + j * 256, r = i / kLgK, kk = i % kLgK;
      As[kk * kLgLD + r] = ra[j];
      Bs[kk * kLgLD + r] = rb[j];
    }
  };
  double acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
  fetch(0);
  stash(0);
  __syncthreads();
  constexpr int kChunks = D / kLgK;
#pragma unroll 1
  for (int ch = 0; ch < kChunks; ++ch) {
    const int st = ch & 1;
    if (ch + 1 < kChunks) fetch((ch + 1) * kLgK);   // in flight during the FMAs below
    const double* As = lg_smem + st * 2 * kLgBuf;
    const double* Bs = As + kLgBuf;
#pragma unroll
    for (int kk = 0; kk < kLgK; ++kk) {
      double a[8], b[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const double2 va = *reinterpret_cast<const double2*>(&As[kk * kLgLD + 2 * ty + 32 * i]);
        const double2 vb = *reinterpret_cast<const double2*>(&Bs[kk * kLgLD + 2 * tx + 32 * i]);
        a[2 * i] = va.x; a[2 * i + 1] = va.y;
        b[2 * i] = vb.x; b[2 * i + 1] = vb.y;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    if (ch + 1 < kChunks) stash(st ^ 1);
    __syncthreads();
  }
  double* out = L + static_cast<int64_t>(bh) * nb * nb;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + 2 * ty + 32 * (i >> 1) + (i & 1);
    if (m >= nb) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + 2 * tx + 32 * (j >> 1) + (j & 1);
      if (n < nb) out[static_cast<int64_t>(m) * nb + n] = acc[i][j] * inv_sqrt_d;
    }
  }
}

// ------------------------------------------------------------------ selection

// Butterfly sums; lanes may differ in the last ulp (different association), so
// lane 0's value is broadcast: every lane takes the same branch on it.
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

__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// Mass of the entries whose ordering key (fp32 bit pattern of p) is at least
// v: fp32 sums per lane (at most 128 terms), fp64 across the warp.
__device__ __forceinline__ double mass_at_or_above(const uint32_t* key, int nb, int lane,
                                                   uint32_t v) {
  float s = 0.f;
  for (int c = lane; c < nb; c += 32) {
    const uint32_t k = key[c];
    s += (k >= v) ? __uint_as_float(k) : 0.f;
  }
  return warp_sum(static_cast<double>(s));
}

// Entries whose ordering key is at least v.
__device__ __forceinline__ int count_at_or_above(const uint32_t* key, int nb, int lane, uint32_t v) {
  int n = 0;
  for (int c = lane; c < nb; c += 32) n += key[c] >= v;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) n += __shfl_xor_sync(0xffffffffu, n, off);
  return n;
}

struct SelectParams {
  float thr;
  int use_sta, wt, wh, ww;
  int Tt, Th, Tw;
  int topk;        // > 0: keep the topk most probable blocks instead of the mass rule
};

// One warp per row g = bh*nb + r; `wpc` warps per CTA; shared memory: one
// 32-bit key per entry.  The reduced map arrives in fp64.  p = exp(L - max) / Z
// is formed in fp32 from the fp64 difference (a few ulp), and its fp32 bit
// pattern is the ordering key (order-preserving for p >= 0); equal keys go by
// block index.  Masses are summed from those fp32 values, fp64 across the warp.
// Relative to the fp64 rule this can move the cut only for rows whose cut
// mass is within a few 1e-6 of 1 - thr, or swap blocks whose probabilities
// agree to ~1e-7.
//
// kEnergy: the row holds non-negative fp32 weights (block energies) instead of
// logits; p = w / sum(w) replaces the softmax, and a row of zero total keeps
// nothing.  votes (optional, [nrows, nb] int32) gets +1 for every kept entry;
// bits and counts are optional too.
template <bool kEnergy>
__global__ void __launch_bounds__(256) select_kernel(const void* __restrict__ in, int64_t nrows,
                                                     int nb, int wpc, SelectParams prm,
                                                     uint32_t* __restrict__ bits,
                                                     int32_t* __restrict__ counts,
                                                     uint8_t* __restrict__ mask_u8,
                                                     int32_t* __restrict__ votes) {
  extern __shared__ uint32_t sel_keys[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * wpc + warp;
  if (g >= nrows) return;
  const int r = static_cast<int>(g % nb);
  const int nw = (nb + 31) >> 5;
  uint32_t* key = sel_keys + static_cast<int64_t>(warp) * nb;

  float zl = 0.f;
  bool empty_row = false;
  if (kEnergy) {
    const float* Erow = static_cast<const float*>(in) + g * nb;
    for (int c = lane; c < nb; c += 32) {
      const float e = Erow[c];
      const float w = e > 0.f ? e : 0.f;   // negative or NaN weights count as zero
      key[c] = __float_as_uint(w);
      zl += w;
    }
  } else {
    // softmax over the row (max subtracted in fp64)
    const double* Lrow = static_cast<const double*>(in) + g * nb;
    double mx = -INFINITY;
    for (int c = lane; c < nb; c += 32) mx = fmax(mx, Lrow[c]);
    mx = warp_max(mx);
    for (int c = lane; c < nb; c += 32) {
      const float e = expf(static_cast<float>(Lrow[c] - mx));
      key[c] = __float_as_uint(e);
      zl += e;
    }
  }
  const float z = static_cast<float>(warp_sum(static_cast<double>(zl)));
  if (kEnergy) empty_row = !(z > 0.f);   // uniform: z is lane 0's value
  uint32_t kmax = 0;
  for (int c = lane; c < nb; c += 32) {
    const uint32_t kv = empty_row ? 0u : __float_as_uint(__uint_as_float(key[c]) / z);
    key[c] = kv;
    kmax = max(kmax, kv);
  }
  kmax = warp_max_u32(kmax);
  __syncwarp();

  // v*: largest key whose mass-at-or-above reaches 1 - thr.  Entries with a
  // larger key are kept; entries with key v* are taken in block order while
  // the exclusive prefix mass stays below the target.  The first entry of the
  // sorted row is always kept.
  const double target = 1.0 - static_cast<double>(prm.thr);
  const bool topk_mode = prm.topk > 0;
  bool keep_all = topk_mode ? prm.topk >= nb : prm.thr <= 0.f;
  uint32_t vstar = kmax;
  double above = 0.0;
  int tied_quota = 0;          // top-k: tied entries kept, in block order
  if (topk_mode && !keep_all) {
    // v*: largest key with at least topk entries at or above it
    uint32_t lo = 0u, hi = kmax + 1u;   // count(lo) = nb >= topk > count(hi) = 0
    while (hi - lo > 1u) {
      const uint32_t mid = lo + ((hi - lo) >> 1);
      if (count_at_or_above(key, nb, lane, mid) >= prm.topk) lo = mid; else hi = mid;
    }
    vstar = lo;
    tied_quota = prm.topk - count_at_or_above(key, nb, lane, vstar + 1u);
  } else if (!keep_all && target > 0.0) {
    const double total = mass_at_or_above(key, nb, lane, 0u);
    if (total < target) {
      keep_all = true;   // every exclusive prefix stays below the target
    } else {
      uint32_t lo = 0u, hi = kmax + 1u;   // mass(lo) >= target > mass(hi)
      while (hi - lo > 1u) {
        const uint32_t mid = lo + ((hi - lo) >> 1);
        if (mass_at_or_above(key, nb, lane, mid) >= target) lo = mid; else hi = mid;
      }
      vstar = lo;
      above = mass_at_or_above(key, nb, lane, vstar + 1u);   // < target
    }
  }

  // flags -> bitmap words, optional uint8 row, STA union, counts
  const int rt = r / (prm.Th * prm.Tw), rh = (r / prm.Tw) % prm.Th, rw = r % prm.Tw;
  const double pstar = static_cast<double>(__uint_as_float(vstar));
  double carry = above;        // exclusive prefix mass before the next tied entry
  bool first_tied = true;      // no tied entry seen yet
  int tied_seen = 0;
  int count = 0;
  uint32_t* brow = bits ? bits + g * nw : nullptr;
  uint8_t* mrow = mask_u8 ? mask_u8 + g * nb : nullptr;
  for (int w = 0; w < nw; ++w) {
    const int c = w * 32 + lane;
    const bool inrow = c < nb;
    bool keep;
    if (empty_row) {   // warp-uniform branch
      keep = false;
    } else if (keep_all) {   // warp-uniform branch
      keep = inrow;
    } else {
      const uint32_t kv = inrow ? key[c] : 0u;
      const bool tied = inrow && kv == vstar;
      const uint32_t tb = __ballot_sync(0xffffffffu, tied);
      const int rank = __popc(tb & ((1u << lane) - 1u));   // tied entries before this one
      const bool is_first = first_tied && tied && rank == 0;
      const double excl = carry + rank * pstar;
      if (topk_mode)
        keep = inrow && (kv > vstar || (tied && tied_seen + rank < tied_quota));
      else
        keep = inrow && (kv > vstar || (tied && (excl < target || (is_first && vstar == kmax))));
      carry += __popc(tb) * pstar;
      tied_seen += __popc(tb);
      if (tb) first_tied = false;
    }
    if (inrow && prm.use_sta) {
      const int ct = c / (prm.Th * prm.Tw), ch = (c / prm.Tw) % prm.Th, cw = c % prm.Tw;
      keep |= abs(ct - rt) <= prm.wt && abs(ch - rh) <= prm.wh && abs(cw - rw) <= prm.ww;
    }
    if (mrow && inrow) mrow[c] = keep ? 1 : 0;
    if (votes && keep) votes[g * nb + c] += 1;
    const uint32_t word = __ballot_sync(0xffffffffu, keep);
    if (brow && lane == 0) brow[w] = word;
    count += __popc(word);
  }
  if (counts && lane == 0) counts[g] = count;
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
  const dim3 grid((nb + kLgT - 1) / kLgT, (nb + kLgT - 1) / kLgT, BH);
  const double inv = 1.0 / sqrt(static_cast<double>(d));
  cudaError_t e;
  if (d == 128) {
    e = cudaFuncSetAttribute(logits_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kLgSmem));
    if (e != cudaSuccess) return e;
    logits_kernel<128><<<grid, 256, kLgSmem, st>>>(qbar, kbar, L, nb, inv);
  } else {
    e = cudaFuncSetAttribute(logits_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kLgSmem));
    if (e != cudaSuccess) return e;
    logits_kernel<64><<<grid, 256, kLgSmem, st>>>(qbar, kbar, L, nb, inv);
  }
  return cudaGetLastError();
}

cudaError_t launch_select(const double* L, int64_t nrows, int nb, float thr, int topk,
                          int use_sta, int wt, int wh, int ww, int Tt, int Th, int Tw,
                          uint32_t* bits, int32_t* counts, uint8_t* mask_u8, cudaStream_t st) {
  SelectParams prm{thr, use_sta, wt, wh, ww, Tt, Th, Tw, topk};
  const size_t per_warp = static_cast<size_t>(nb) * sizeof(uint32_t);
  int wpc = static_cast<int>((200u * 1024u) / per_warp);
  wpc = wpc < 1 ? 1 : (wpc > 8 ? 8 : wpc);
  const size_t smem = per_warp * wpc;
  cudaError_t e = cudaFuncSetAttribute(select_kernel<false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>((nrows + wpc - 1) / wpc);
  select_kernel<false><<<grid, 32 * wpc, smem, st>>>(L, nrows, nb, wpc, prm, bits, counts,
                                                     mask_u8, nullptr);
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
  const size_t per_warp = static_cast<size_t>(nb) * sizeof(uint32_t);
  int wpc = static_cast<int>((200u * 1024u) / per_warp);
  wpc = wpc < 1 ? 1 : (wpc > 8 ? 8 : wpc);
  const size_t smem = per_warp * wpc;
  cudaError_t e = cudaFuncSetAttribute(select_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>((nrows + wpc - 1) / wpc);
  select_kernel<true><<<grid, 32 * wpc, smem, st>>>(weights, nrows, nb, wpc, prm, bits, counts,
                                                    mask_u8, nullptr);
  return cudaGetLastError();
}

cudaError_t launch_calib_select(const float* energy, int64_t nrows, int nb, float eps,
                                int32_t* votes, cudaStream_t st) {
  SelectParams prm{eps, 0, 0, 0, 0, 1, 1, 1, 0};
  const size_t per_warp = static_cast<size_t>(nb) * sizeof(uint32_t);
  int wpc = static_cast<int>((200u * 1024u) / per_warp);
  wpc = wpc < 1 ? 1 : (wpc > 8 ? 8 : wpc);
  const size_t smem = per_warp * wpc;
  cudaError_t e = cudaFuncSetAttribute(select_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>((nrows + wpc - 1) / wpc);
  select_kernel<true><<<grid, 32 * wpc, smem, st>>>(energy, nrows, nb, wpc, prm, nullptr, nullptr,
                                                    nullptr, votes);
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
