// Block-sparse attention backward on sm_100a.
//
// Gradient of O = softmax(scale * Q K^T restricted to the kept blocks) V
// (FlashAttention abstract: exact attention by tiles, recomputing the
// probabilities from the saved log-sum-exp instead of storing them; NABLA
// trains with the same block mask in the backward pass, "NABLA:
// Neighborhood Adaptive Block-Level Attention", review summary: the 1.46x
// pretraining speed-up).  For every kept (query block r, key block c):
//   P  = exp(scale * Q_r K_c^T - LSE_r)          (64 x 64, recomputed)
//   dV_c += P^T dO_r        dP = dO_r V_c^T
//   dS = P o (dP - D_r),    D_i = sum_k dO_ik O_ik
//   dQ_r += scale dS K_c    dK_c += scale dS^T Q_r
//
// Two tcgen05 kernels, no atomics (results do not depend on scheduling):
//   key-stationary (dK, dV): one CTA per (b, h, key blocks 2p, 2p+1).  The
//     query blocks visited are those whose CSR row lists c0 or c1 (read from a
//     column bitmap built by bwd_colbits_kernel), two per 128-query tile.
//       S^T  = K Q^T,  dP^T = V dO^T                  (SS MMAs, 128 x 128)
//       P^T, dS^T in tensor memory (bf16, in place)    (elementwise warps)
//       dV  += P^T dO, dK += dS^T Q                    (TS MMAs, N = d)
//   query-stationary (dQ): one CTA per (b, h, query blocks 2p, 2p+1), key
//     blocks from the union of the two CSR rows, two per 128-key tile.
//       S = Q K^T, dP = dO V^T;  dS in tensor memory;  dQ += dS K
// The stationary pair of blocks sits in shared memory for the CTA's life; the
// streaming tiles arrive by TMA through a two-stage ring.  Both kernels share
// one template: X1, X2 are the stationary tiles (K, V or Q, dO) and Y1, Y2 the
// streaming ones (Q, dO or K, V), so that MMA1 = X1 Y1^T and MMA2 = X2 Y2^T.
//
// Roles (384 threads): warps 0-7 elementwise (warp w owns tensor-memory lanes
// 32(w%4).. and the 64 columns of union entry w/4; the two warps sharing a
// row both load their halves, meeting on an mbarrier, before either writes
// the packed bf16 results in place), warp 8 issues TMA loads, warp 9 owns tensor memory and issues MMAs,
// warps 10-11 idle (they complete the warpgroup that lowers its registers).
// Tensor memory: S(^T) [0,128), dP(^T) [128,256), accumulators from 256.
// Every mbarrier wait is time-bounded (kStatusTimeout, abort flag, drain).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_primitives.cuh"

namespace nabla {

constexpr int kBT = 128;              // rows of a stationary / streaming tile (two blocks)
constexpr int kBStages = 2;           // streaming ring depth
constexpr int kBEwWarps = 8;
constexpr int kBThreads = (kBEwWarps + 4) * 32;   // warps 10, 11 complete warpgroup 2
constexpr int kBProducerWarp = 8, kBMmaWarp = 9;
// Register split after set-up (per warpgroup): 8*216 + 4*72 = 12*168, the
// launch allocation (checked on the host before launch).
constexpr int kBRegsEw = 216, kBRegsOther = 72, kBRegsLaunch = 168;
constexpr int kBMaxNb = 4096;
constexpr uint32_t kBTmemCols = 512;
constexpr uint64_t kBDrainNs = 1000000000ull;
constexpr uint32_t kColS = 0, kColDP = 128, kColAcc = 256;

template <int D>
struct BwdSmem {
  static constexpr int kDH = D / 64;
  static constexpr uint32_t kTile = kBT * D * 2;                   // one 128 x d bf16 tile
  static constexpr uint32_t kOffX = 0;                             // X1, X2
  static constexpr uint32_t kOffY = 2 * kTile;                     // [stage][Y1, Y2]
  static constexpr uint32_t kOffVec = kOffY + kBStages * 2 * kTile;   // [stage][lse | D][128] fp32
  static constexpr uint32_t kVecBytes = 2 * kBT * 4;
  static constexpr uint32_t kOffBar = kOffVec + kBStages * kVecBytes;  // 32 mbarriers
  static constexpr uint32_t kOffMisc = kOffBar + 256;
  static constexpr uint32_t kOffBitmap = kOffMisc + 64;            // [2][kBMaxNb/32]
  static constexpr uint32_t kOffList = kOffBitmap + 2 * (kBMaxNb / 32) * 4;
  static constexpr uint32_t kBytes = kOffList + kBMaxNb * 4;
  static constexpr uint32_t kAlloc = kBytes + 1024;
};

enum : int {
  kBBarXFull = 0,
  kBBarYFull = 1,                          // + stage
  kBBarYEmpty = kBBarYFull + kBStages,     // + stage
  kBBarSFull = kBBarYEmpty + kBStages,     // MMA1 (S or S^T) done
  kBBarDPFull = kBBarSFull + 1,            // MMA2 (dP or dP^T) done
  kBBarSDone = kBBarDPFull + 1,            // key-stationary: P^T written; query-stationary: S read
  kBBarDSReady = kBBarSDone + 1,           // dS (dS^T) written
  kBBarAccFull = kBBarDSReady + 1,         // every accumulating MMA done
  kBBarDrain = kBBarAccFull + 1,
  kBBarPairS = kBBarDrain + 1,             // + lane quarter: both S halves loaded
  kBBarPairDP = kBBarPairS + 4,            // + lane quarter: both dP halves loaded
  kBNumBars = kBBarPairDP + 4
};
static_assert(kBNumBars * 8 <= 256, "barrier area");

struct BwdParams {
  const int32_t* row_ptr;      // CSR (query-stationary) or unused
  const int32_t* col_idx;
  const uint32_t* colbits;     // [BH*nb][nw] column bitmaps (key-stationary)
  const float* lse2;           // [BH*S] LSE * log2(e)
  const float* dvec;           // [BH*S] rowsum(dO o O)
  __nv_bfloat16* out1;         // dV or dQ
  __nv_bfloat16* out2;         // dK or null
  int* status;
  int S, nb, npairs;
  float scale;
  float scale_log2;
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ bool b_warp_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                            const volatile int* abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, limit_ns, abort));
}

__device__ __forceinline__ void b_abort(volatile int* abort, int* status) {
  *abort = 1;
  atomicOr(status, kStatusTimeout);
}

// ---------------------------------------------------------------- helpers

// D_i = sum_k dO_ik O_ik in fp32 from the bf16 tensors.  d/8 lanes per row
// (16-byte loads), rows packed into warps.  HBM-bound: reads O and dO once.
// It also writes lse2 = LSE * log2(e), the form the exponentials take.
template <int D>
__global__ void __launch_bounds__(256) bwd_dvec_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ dout,
                                                       const float* __restrict__ lse,
                                                       float* __restrict__ dvec,
                                                       float* __restrict__ lse2, int64_t rows) {
  constexpr int kLanes = D / 8;
  const int64_t gt = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t row = gt / kLanes;
  const int chunk = static_cast<int>(gt % kLanes);
  float s = 0.f;
  if (row < rows) {
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(o + row * D) + chunk);
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(dout + row * D) + chunk);
    const uint32_t av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      s = fmaf(__uint_as_float(av[i] << 16), __uint_as_float(bv[i] << 16), s);
      s = fmaf(__uint_as_float(av[i] & 0xFFFF0000u), __uint_as_float(bv[i] & 0xFFFF0000u), s);
    }
  }
#pragma unroll
  for (int off = kLanes / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (row < rows && chunk == 0) {
    dvec[row] = s;
    lse2[row] = lse[row] * 1.4426950408889634f;
  }
}

// Column bitmaps of the block CSR: bit r of colbits[bh*nb + c] is set iff row
// (bh, r) lists block c.  One warp per CSR row; atomicOr is order-free.
__global__ void __launch_bounds__(256) bwd_colbits_kernel(const int32_t* __restrict__ row_ptr,
                                                          const int32_t* __restrict__ col_idx,
                                                          int64_t nrows, int nb,
                                                          uint32_t* __restrict__ colbits,
                                                          int* status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * 8 + warp;
  if (g >= nrows) return;
  const int64_t bh = g / nb;
  const int r = static_cast<int>(g % nb);
  const int nw = (nb + 31) >> 5;
  const int b = row_ptr[g], e = row_ptr[g + 1];
  for (int i = b + lane; i < e; i += 32) {
    const int c = col_idx[i];
    if (static_cast<unsigned>(c) < static_cast<unsigned>(nb))
      atomicOr(&colbits[(bh * nb + c) * nw + (r >> 5)], 1u << (r & 31));
    else
      atomicOr(status, kStatusBadIndex);
  }
}

// ---------------------------------------------------------------- main kernel
// kKV = true: key-stationary (X = K, V; Y = Q, dO; writes dV, dK).
// kKV = false: query-stationary (X = Q, dO; Y = K, V; writes dQ).
template <int D, bool kKV>
__global__ void __launch_bounds__(kBThreads, 1)
    bsa_bwd_kernel(const __grid_constant__ CUtensorMap tmX1, const __grid_constant__ CUtensorMap tmX2,
                   const __grid_constant__ CUtensorMap tmY1, const __grid_constant__ CUtensorMap tmY2,
                   const BwdParams prm) {
  using L = BwdSmem<D>;
  extern __shared__ uint8_t bwd_smem_raw[];
  const uint32_t raw = smem_addr(bwd_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = bwd_smem_raw + (base - raw);
  const uint32_t sX = base + L::kOffX;
  const uint32_t sY = base + L::kOffY;
  const uint32_t sVec = base + L::kOffVec;
  const uint32_t bar0 = base + L::kOffBar;
  uint32_t* misc = reinterpret_cast<uint32_t*>(gbase + L::kOffMisc);
  volatile uint32_t* tmem_holder = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* n_union_s = reinterpret_cast<volatile int*>(misc + 2);
  uint32_t* bm = reinterpret_cast<uint32_t*>(gbase + L::kOffBitmap);
  int32_t* ulist = reinterpret_cast<int32_t*>(gbase + L::kOffList);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / prm.npairs;
  const int r0 = 2 * (blockIdx.x % prm.npairs);   // first stationary block
  const int nb = prm.nb;
  const int nx = min(2, nb - r0);                  // stationary blocks present
  const int nw = (nb + 31) >> 5;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  // ---------------------------------------------------------------- setup
  if (tid == 0) {
    mbar_init(bar(kBBarXFull), 1);
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(bar(kBBarYFull + s), 1);
      mbar_init(bar(kBBarYEmpty + s), 1);
    }
    mbar_init(bar(kBBarSFull), 1);
    mbar_init(bar(kBBarDPFull), 1);
    mbar_init(bar(kBBarSDone), kBEwWarps * 32);
    mbar_init(bar(kBBarDSReady), kBEwWarps * 32);
    mbar_init(bar(kBBarAccFull), 1);
    mbar_init(bar(kBBarDrain), 1);
    for (int qd = 0; qd < 4; ++qd) {
      mbar_init(bar(kBBarPairS + qd), 64);
      mbar_init(bar(kBBarPairDP + qd), 64);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kBMmaWarp) {
    tmem_alloc(smem_addr(misc), kBTmemCols);
    tmem_relinquish();
  }
  if (warp == kBProducerWarp && lane == 0) {
    tma_prefetch_desc(&tmX1);
    tma_prefetch_desc(&tmX2);
    tma_prefetch_desc(&tmY1);
    tma_prefetch_desc(&tmY2);
  }
  for (int i = tid; i < 2 * (kBMaxNb / 32); i += kBThreads) bm[i] = 0u;
  __syncthreads();
  for (int x = 0; x < nx; ++x) {
    const int64_t g = static_cast<int64_t>(bh) * nb + r0 + x;
    uint32_t* bmx = bm + x * (kBMaxNb / 32);
    if (kKV) {   // the query blocks that list key block r0 + x
      const uint32_t* src = prm.colbits + g * nw;
      for (int w = tid; w < nw; w += kBThreads) bmx[w] = src[w];
    } else {     // the key blocks listed by query block r0 + x
      const int b = prm.row_ptr[g], e = prm.row_ptr[g + 1];
      for (int i = b + tid; i < e; i += kBThreads) {
        const int c = prm.col_idx[i];
        if (static_cast<unsigned>(c) < static_cast<unsigned>(nb)) atomicOr(&bmx[c >> 5], 1u << (c & 31));
        else atomicOr(prm.status, kStatusBadIndex);
      }
    }
  }
  __syncthreads();
  if (warp == kBProducerWarp) {   // union, ascending, 2-bit membership at bit 16
    int run = 0;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t u0 = w < nw ? bm[w] : 0u;
      const uint32_t u1 = w < nw ? bm[kBMaxNb / 32 + w] : 0u;
      uint32_t any = u0 | u1;
      const int cnt = __popc(any);
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      int pos = run + incl - cnt;
      while (any) {
        const int b = __ffs(any) - 1;
        any &= any - 1;
        const int mem = static_cast<int>((u0 >> b) & 1u) | (static_cast<int>((u1 >> b) & 1u) << 1);
        ulist[pos++] = (w * 32 + b) | (mem << 16);
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) *n_union_s = run;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int n_u = *n_union_s;
  const int n_t = (n_u + 1) >> 1;
  const uint64_t lim = prm.wait_limit_ns;
  auto tile_entry = [&](int t, int i) { return (2 * t + i < n_u) ? ulist[2 * t + i] : 0; };

  if (warp >= kBEwWarps) {
  setmaxnreg_dec<kBRegsOther>();
  if (warp == kBProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_t > 0) {
      const int64_t row0 = static_cast<int64_t>(bh) * prm.S;
      int armed[kBStages] = {0, 0};
      mbar_arrive_expect_tx(bar(kBBarXFull), 2 * L::kTile);
      for (int x = 0; x < 2; ++x) {
        const int rb = r0 + (x < nx ? x : 0);   // a missing second block repeats the first
        for (int h = 0; h < L::kDH; ++h) {
          const uint32_t off = h * kBT * 128 + x * 64 * 128;
          const int32_t y = static_cast<int32_t>(row0 + static_cast<int64_t>(rb) * 64);
          tma_load_2d(sX + off, &tmX1, bar(kBBarXFull), h * 64, y);
          tma_load_2d(sX + L::kTile + off, &tmX2, bar(kBBarXFull), h * 64, y);
        }
      }
      constexpr uint32_t kStageTx = 2 * L::kTile + (kKV ? L::kVecBytes : 0u);
      for (int t = 0; t < n_t; ++t) {
        const int s = t % kBStages, n = t / kBStages;
        const int j0 = ulist[2 * t] & 0xFFFF;
        const int j1 = (2 * t + 1 < n_u) ? (ulist[2 * t + 1] & 0xFFFF) : j0;
        if (t >= kBStages && !mbar_wait(bar(kBBarYEmpty + s), (n - 1) & 1, lim, abort_flag)) {
          b_abort(abort_flag, prm.status);
          break;
        }
        const uint32_t fb = bar(kBBarYFull + s);
        mbar_arrive_expect_tx(fb, kStageTx);
        ++armed[s];
        const uint32_t y1 = sY + s * 2 * L::kTile, y2 = y1 + L::kTile;
        for (int e = 0; e < 2; ++e) {
          const int j = e ? j1 : j0;
          const int32_t y = static_cast<int32_t>(row0 + static_cast<int64_t>(j) * 64);
          for (int h = 0; h < L::kDH; ++h) {
            const uint32_t off = h * kBT * 128 + e * 64 * 128;
            tma_load_2d(y1 + off, &tmY1, fb, h * 64, y);
            tma_load_2d(y2 + off, &tmY2, fb, h * 64, y);
          }
          if (kKV) {   // LSE and D of the 64 query rows of entry e
            const uint32_t vs = sVec + s * L::kVecBytes;
            bulk_load(vs + e * 256, prm.lse2 + row0 + static_cast<int64_t>(j) * 64, 256, fb);
            bulk_load(vs + kBT * 4 + e * 256, prm.dvec + row0 + static_cast<int64_t>(j) * 64, 256, fb);
          }
        }
      }
      mbar_wait(bar(kBBarXFull), 0, kBDrainNs, nullptr);
      for (int s = 0; s < kBStages; ++s)
        if (armed[s]) mbar_wait(bar(kBBarYFull + s), (armed[s] - 1) & 1, kBDrainNs, nullptr);
    }
  } else if (warp == kBMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    // key-stationary, per tile: wait P^T -> dV += P^T dO, S^T(t+1) | wait dS^T
    //   -> dK += dS^T Q, dP^T(t+1).  dP^T runs under the exponentials, dV and
    //   the next S^T under the dS^T pass; each product that overwrites a
    //   tensor-memory operand is issued after the product that reads it.
    // query-stationary: S(t+1) is issued once the elementwise warps have read
    //   S(t), so it runs under the dS(t) pass; dS goes over dP, which dP(t+1)
    //   overwrites only after dQ(t) (issued first) has read it.
    if (lane == 0 && n_t > 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(kBT, kBT, false);
      constexpr uint32_t idesc_acc = idesc_bf16_f32(kBT, D, true);
      auto stage_y1 = [&](int t) { return sY + (t % kBStages) * 2 * L::kTile; };
      auto issue_ss = [&](uint32_t dcol, uint32_t xa, uint32_t yb) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBT * 128) + (kk & 3) * 32;
          tc_mma_ss(tmem + dcol, sdesc_sw128(xa + off, 16, 1024), sdesc_sw128(yb + off, 16, 1024),
                    idesc_s, kk > 0 ? 1u : 0u);
        }
      };
      // acc += (tensor-memory operand at acol) x (streaming tile yb, MN-major):
      // 16 streaming rows per step, packed bf16 columns [8kk, 8kk+8)
      auto issue_ts = [&](uint32_t dcol, uint32_t acol, uint32_t yb, bool first) {
#pragma unroll
        for (int kk = 0; kk < kBT / 16; ++kk)
          tc_mma_ts(tmem + dcol, tmem + acol + kk * 8, sdesc_sw128(yb + kk * 16 * 128, kBT * 128, 1024),
                    idesc_acc, (!first || kk > 0) ? 1u : 0u);
      };
      auto wait_y = [&](int t) {
        return mbar_wait(bar(kBBarYFull + t % kBStages), (t / kBStages) & 1, lim, abort_flag);
      };
      bool ok = mbar_wait(bar(kBBarXFull), 0, lim, abort_flag);
      if (kKV) {
        if (ok && !wait_y(0)) ok = false;
        if (ok) {
          tc_fence_after();
          issue_ss(kColS, sX, stage_y1(0));                         // S^T(0) = K Q^T
          tc_commit(bar(kBBarSFull));
          issue_ss(kColDP, sX + L::kTile, stage_y1(0) + L::kTile);  // dP^T(0) = V dO^T
          tc_commit(bar(kBBarDPFull));
        }
        for (int t = 0; ok && t < n_t; ++t) {
          const bool more = t + 1 < n_t;
          const uint32_t y1 = stage_y1(t), y2 = y1 + L::kTile;
          if (!mbar_wait(bar(kBBarSDone), t & 1, lim, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_ts(kColAcc, kColS, y2, t == 0);                     // dV += P^T dO
          if (more) {   // S^T(t+1) overwrites P^T(t) after dV(t) has read it (issue order)
            if (!wait_y(t + 1)) { ok = false; break; }
            tc_fence_after();
            issue_ss(kColS, sX, stage_y1(t + 1));
            tc_commit(bar(kBBarSFull));
          }
          if (!mbar_wait(bar(kBBarDSReady), t & 1, lim, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_ts(kColAcc + D, kColDP, y1, t == 0);                // dK += dS^T Q
          tc_commit(bar(kBBarYEmpty + t % kBStages));
          if (more) {   // dP^T(t+1) overwrites dS^T(t) after dK(t) has read it
            issue_ss(kColDP, sX + L::kTile, stage_y1(t + 1) + L::kTile);
            tc_commit(bar(kBBarDPFull));
          }
        }
      } else {
        if (ok && !wait_y(0)) ok = false;
        if (ok) {
          tc_fence_after();
          issue_ss(kColS, sX, stage_y1(0));                       // S(0) = Q K^T
          tc_commit(bar(kBBarSFull));
          issue_ss(kColDP, sX + L::kTile, stage_y1(0) + L::kTile);  // dP(0) = dO V^T
          tc_commit(bar(kBBarDPFull));
        }
        for (int t = 0; ok && t < n_t; ++t) {
          const bool more = t + 1 < n_t;
          if (more) {
            if (!wait_y(t + 1) || !mbar_wait(bar(kBBarSDone), t & 1, lim, abort_flag)) { ok = false; break; }
            tc_fence_after();
            issue_ss(kColS, sX, stage_y1(t + 1));                 // S(t+1)
            tc_commit(bar(kBBarSFull));
          }
          if (!mbar_wait(bar(kBBarDSReady), t & 1, lim, abort_flag)) { ok = false; break; }
          tc_fence_after();
          issue_ts(kColAcc, kColDP, stage_y1(t), t == 0);         // dQ += dS K
          tc_commit(bar(kBBarYEmpty + t % kBStages));
          if (more) {
            issue_ss(kColDP, sX + L::kTile, stage_y1(t + 1) + L::kTile);   // dP(t+1)
            tc_commit(bar(kBBarDPFull));
          }
        }
      }
      if (ok) tc_commit(bar(kBBarAccFull));
      else b_abort(abort_flag, prm.status);
      tc_commit(bar(kBBarDrain));
      mbar_wait(bar(kBBarDrain), 0, kBDrainNs, nullptr);
    }
  }
  } else {
    setmaxnreg_inc<kBRegsEw>();
    // ------------------------------------------------------------ elementwise (warps 0-7)
    const int quarter = warp & 3, half = warp >> 2;
    const int row = quarter * 32 + lane;          // tensor-memory lane = stationary row
    const int x = row >> 6;                       // stationary block (uniform per warp)
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tb = tmem + lane_off;
    const float sl2 = prm.scale_log2;
    float row_nlse2 = 0.f, row_d = 0.f;
    if (!kKV && x < nx) {
      const int64_t gr = static_cast<int64_t>(bh) * prm.S + static_cast<int64_t>(r0 + x) * 64 + (row & 63);
      row_nlse2 = -prm.lse2[gr];
      row_d = prm.dvec[gr];
    }
    bool ok = true;
    for (int t = 0; t < n_t; ++t) {
      const int s = t % kBStages;
      const int e = tile_entry(t, half);
      const bool member = ((e >> (16 + x)) & 1) != 0;   // uniform per warp
      // LSE and D of this entry's 64 queries (key-stationary), read as 16-byte vectors
      const uint32_t vl_addr = sVec + s * L::kVecBytes + 64 * half * 4;
      const uint32_t vd_addr = vl_addr + kBT * 4;
      auto load32 = [&](uint32_t addr, float (&r)[32]) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float4 f = lds_f4(addr + 16 * j);
          r[4 * j] = f.x; r[4 * j + 1] = f.y; r[4 * j + 2] = f.z; r[4 * j + 3] = f.w;
        }
      };
      // ---- S (S^T): probabilities, kept in registers
      if (!b_warp_wait(bar(kBBarSFull), t & 1, lim, abort_flag)) { ok = false; break; }
      tc_fence_after();
      // query-stationary: P in fp32; key-stationary: P^T packed to bf16 (the
      // values the dV product uses), which also feeds dS^T and keeps the
      // thread's live registers below the split (a spill would go to L2:
      // shared memory leaves almost no L1)
      float p[kKV ? 1 : 64];
      uint32_t pk[2][16];
      {
        uint32_t sv[2][32];
        if (member) {
          tmem_ld32(tb + kColS + 64 * half, sv[0]);
          tmem_ld32(tb + kColS + 64 * half + 32, sv[1]);
          tmem_ld_wait();
        }
        if (kKV) {
          // P^T goes over S^T in place: both column halves of these rows
          // must be in registers first (a bounded wait: the partner may have aborted)
          tc_fence_before();
          mbar_arrive(bar(kBBarPairS + quarter));
          if (!b_warp_wait(bar(kBBarPairS + quarter), t & 1, lim, abort_flag)) { ok = false; break; }
          tc_fence_after();
        } else {
          tc_fence_before();
          mbar_arrive(bar(kBBarSDone));            // S(t) read: S(t+1) may be computed
        }
        if (kKV) {
#pragma unroll
          for (int ch = 0; ch < 2; ++ch) {
            float lv[32];
            load32(vl_addr + 128 * ch, lv);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              float e[2];
#pragma unroll
              for (int u = 0; u < 2; ++u)
                e[u] = member ? fast_exp2(fmaf(__uint_as_float(sv[ch][2 * i + u]), sl2,
                                               -lv[2 * i + u]))
                              : 0.f;
              pk[ch][i] = pack_bf16x2(e[0], e[1]);
            }
          }
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            p[c & (kKV ? 0 : 63)] =
                member ? fast_exp2(fmaf(__uint_as_float(sv[c >> 5][c & 31]), sl2, row_nlse2)) : 0.f;
        }
      }
      if (kKV) {
        tmem_st16(tb + kColS + 32 * half, pk[0]);
        tmem_st16(tb + kColS + 32 * half + 16, pk[1]);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bar(kBBarSDone));              // P^T written: dV += P^T dO may run
      }
      // ---- dP (dP^T): dS = P o (dP - D), written over dP in place
      if (!b_warp_wait(bar(kBBarDPFull), t & 1, lim, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t dv[2][32];
      if (member) {
        tmem_ld32(tb + kColDP + 64 * half, dv[0]);
        tmem_ld32(tb + kColDP + 64 * half + 32, dv[1]);
        tmem_ld_wait();
      }
      tc_fence_before();
      mbar_arrive(bar(kBBarPairDP + quarter));
      if (!b_warp_wait(bar(kBBarPairDP + quarter), t & 1, lim, abort_flag)) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < 2; ++ch) {
        uint32_t dk[16];
        float dvv[32];
        if (kKV) load32(vd_addr + 128 * ch, dvv);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          // dS = P o (dP - D), two lanes of work per packed instruction
          const int c = 32 * ch + 2 * i;
          float2 pc, dd;
          if (kKV) {
            pc = make_float2(__uint_as_float(pk[ch][i] << 16), __uint_as_float(pk[ch][i] & 0xFFFF0000u));
            dd = make_float2(dvv[2 * i], dvv[2 * i + 1]);
          } else {
            pc = make_float2(p[c & (kKV ? 0 : 63)], p[(c + 1) & (kKV ? 0 : 63)]);
            dd = make_float2(row_d, row_d);
          }
          const float2 ds = fsubmul2(make_float2(__uint_as_float(dv[ch][2 * i]),
                                                 __uint_as_float(dv[ch][2 * i + 1])), dd, pc);
          dk[i] = member ? pack_bf16x2(ds.x, ds.y) : 0u;
        }
        tmem_st16(tb + kColDP + 32 * half + 16 * ch, dk);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(kBBarDSReady));
    }
    if (!ok) b_abort(abort_flag, prm.status);
    // ------------------------------------------------------------ epilogue
    bool have = false;
    if (ok && n_t > 0) {
      have = b_warp_wait(bar(kBBarAccFull), 0, lim, abort_flag);
      if (!have) b_abort(abort_flag, prm.status);
      tc_fence_after();
    }
    const bool write = x < nx && ok && (n_t == 0 || have);
    const int64_t grow = static_cast<int64_t>(bh) * prm.S + static_cast<int64_t>(r0 + x) * 64 + (row & 63);
    // key-stationary: half 0 writes dV (unscaled), half 1 dK (x scale) over all
    // d columns; query-stationary: half h writes dQ columns [h d/2, (h+1) d/2)
    constexpr int kCols = kKV ? D : D / 2;
    const uint32_t acc_col = kColAcc + (kKV ? half * D : half * (D / 2));
    const float mul = (kKV && half == 0) ? 1.f : prm.scale;
    __nv_bfloat16* dst = (kKV && half == 1) ? prm.out2 : prm.out1;
    __nv_bfloat16* drow = dst + grow * D + (kKV ? 0 : half * (D / 2));
#pragma unroll
    for (int cc = 0; cc < kCols / 32; ++cc) {
      uint32_t a[32];
      if (have) {
        tmem_ld32(tb + acc_col + cc * 32, a);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) a[i] = 0u;
      }
      if (write) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16x2(__uint_as_float(a[2 * i]) * mul, __uint_as_float(a[2 * i + 1]) * mul);
        uint4* o4 = reinterpret_cast<uint4*>(drow + cc * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) o4[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kBMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kBTmemCols);
  }
}

// ---------------------------------------------------------------- launchers

template <int D, bool kKV>
static cudaError_t launch_bwd_t(const CUtensorMap* maps, const BwdParams& prm, int64_t nitems,
                                cudaStream_t st) {
  constexpr uint32_t smem = BwdSmem<D>::kAlloc;
  static_assert(smem <= 227 * 1024, "shared memory");
  static_assert(8 * kBRegsEw + 4 * kBRegsOther <= 12 * kBRegsLaunch, "register split");
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, bsa_bwd_kernel<D, kKV>);
  if (e != cudaSuccess) return e;
  // setmaxnreg.inc below assumes the launch allocation of kBRegsLaunch registers
  if (attr.numRegs < kBRegsLaunch) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(bsa_bwd_kernel<D, kKV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  bsa_bwd_kernel<D, kKV><<<static_cast<unsigned>(nitems), kBThreads, smem, st>>>(
      maps[0], maps[1], maps[2], maps[3], prm);
  return cudaGetLastError();
}

// maps: Q, K, V, dO tensor maps (64 x 64 boxes, 128-byte swizzle).
cudaError_t launch_bsa_bwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                           const CUtensorMap& mdo, const void* o, const void* dout,
                           const float* lse, const int32_t* row_ptr, const int32_t* col_idx,
                           float* dvec, float* lse2, uint32_t* colbits, void* dq, void* dk, void* dv,
                           int* status, int BH, int S, int d, float scale, uint64_t wait_limit_ns,
                           cudaStream_t st) {
  const int nb = S / 64;
  const int64_t rows = static_cast<int64_t>(BH) * S;
  if (rows == 0) return cudaSuccess;
  // D = rowsum(dO o O)
  {
    const int64_t threads = rows * (d / 8);
    const unsigned grid = static_cast<unsigned>((threads + 255) / 256);
    if (d == 128)
      bwd_dvec_kernel<128><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(o),
                                                 static_cast<const __nv_bfloat16*>(dout), lse, dvec,
                                                 lse2, rows);
    else
      bwd_dvec_kernel<64><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(o),
                                                static_cast<const __nv_bfloat16*>(dout), lse, dvec,
                                                lse2, rows);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // column bitmaps of the block CSR
  const int nw = (nb + 31) / 32;
  const int64_t nrows = static_cast<int64_t>(BH) * nb;
  cudaError_t e = cudaMemsetAsync(colbits, 0, static_cast<size_t>(nrows) * nw * 4, st);
  if (e != cudaSuccess) return e;
  bwd_colbits_kernel<<<static_cast<unsigned>((nrows + 7) / 8), 256, 0, st>>>(row_ptr, col_idx, nrows,
                                                                             nb, colbits, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;

  BwdParams prm;
  prm.row_ptr = row_ptr;
  prm.col_idx = col_idx;
  prm.colbits = colbits;
  prm.lse2 = lse2;
  prm.dvec = dvec;
  prm.status = status;
  prm.S = S;
  prm.nb = nb;
  prm.npairs = (nb + 1) / 2;
  prm.scale = scale;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.wait_limit_ns = wait_limit_ns;
  const int64_t nitems = static_cast<int64_t>(BH) * prm.npairs;
  // key-stationary: X = K, V; Y = Q, dO
  BwdParams pkv = prm;
  pkv.out1 = static_cast<__nv_bfloat16*>(dv);
  pkv.out2 = static_cast<__nv_bfloat16*>(dk);
  const CUtensorMap kv_maps[4] = {mk, mv, mq, mdo};
  e = d == 128 ? launch_bwd_t<128, true>(kv_maps, pkv, nitems, st)
               : launch_bwd_t<64, true>(kv_maps, pkv, nitems, st);
  if (e != cudaSuccess) return e;
  // query-stationary: X = Q, dO; Y = K, V
  BwdParams pq = prm;
  pq.out1 = static_cast<__nv_bfloat16*>(dq);
  pq.out2 = nullptr;
  const CUtensorMap q_maps[4] = {mq, mdo, mk, mv};
  return d == 128 ? launch_bwd_t<128, false>(q_maps, pq, nitems, st)
                  : launch_bwd_t<64, false>(q_maps, pq, nitems, st);
}

}  // namespace nabla
