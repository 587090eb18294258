// Products over a pair of CTAs (tcgen05 cta_group::2, M = 256) on sm_100a.
//
// A cluster of two CTAs computes one M = 256 product: each CTA holds its 128
// rows of A and half of B's N columns in its own shared memory at the same
// offsets (or its 128 rows of A in its own tensor memory), and receives its 128
// rows of D in its own tensor memory; one thread of the even CTA issues the
// products for both.  Every load stays local to the CTA that issues it: the
// odd CTA waits for its own loads and then tells the even CTA, with an arrive
// on the even CTA's barrier, that its half is in place.  Products signal both
// CTAs' barriers through a multicast commit.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_primitives.cuh"

namespace nabla {

constexpr uint64_t kPairDrainLimitNs = 1000000000ull;

// Every lane waits (cluster scope, phase 0); the warp proceeds only if all
// lanes saw the phase complete.
__device__ __forceinline__ bool warp_wait_any(uint32_t bar, uint64_t limit_ns) {
  return __all_sync(0xffffffffu, mbar_wait_cluster(bar, 0, limit_ns, nullptr));
}

// ---------------------------------------------------------------- self-test
// variant 0: C[256][256] = A[256][128] B[256][128]^T (both K-major: CTA c holds
//            rows [128c, 128c+128) of A and of B, i.e. half of N)
// variant 1: C[256][128] = P[256][256] V[256][128] (P in tensor memory, V N-major:
//            CTA c holds columns [64c, 64c+64) of V for all 256 rows)
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(160, 1)
    mma_pair_selftest_kernel(const __grid_constant__ CUtensorMap tmA,
                             const __grid_constant__ CUtensorMap tmB,
                             const __nv_bfloat16* __restrict__ p_glob, float* __restrict__ c,
                             int variant, int* status, uint64_t lim) {
  extern __shared__ uint8_t pst_smem_raw[];
  const uint32_t raw = smem_addr(pst_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = pst_smem_raw + (base - raw);
  const uint32_t sA = base, sB = base + 32768, bars = base + 65536;
  uint32_t* holder = reinterpret_cast<uint32_t*>(gbase + 65536 + 64);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gbase + 65536 + 68);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t bar_tma = bars, bar_mma = bars + 8, bar_a = bars + 16, bar_peer = bars + 24;
  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_a, 128);
    mbar_init(bar_peer, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc_pair(smem_addr(holder), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // barriers of both CTAs initialised, both allocations made
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(holder);
  // the two CTAs must hold the same tensor-memory columns
  const uint32_t peer_tmem = ld_shared_cluster_u32(mapa_shared(smem_addr(holder), rank ^ 1u));
  const bool same = peer_tmem == tmem;
  if (!same && tid == 0) atomicOr(status, kStatusBadIndex);
  if (warp == 4 && lane == 0 && same) {
    // this CTA's halves
    if (variant == 0) {
      mbar_arrive_expect_tx(bar_tma, 65536);
      for (int rh = 0; rh < 2; ++rh)
        for (int h = 0; h < 2; ++h) {
          tma_load_2d(sA + h * 16384 + rh * 8192, &tmA, bar_tma, h * 64, 128 * rank + rh * 64);
          tma_load_2d(sB + h * 16384 + rh * 8192, &tmB, bar_tma, h * 64, 128 * rank + rh * 64);
        }
    } else {
      mbar_arrive_expect_tx(bar_tma, 32768);
      for (int e = 0; e < 4; ++e) tma_load_2d(sB + e * 8192, &tmB, bar_tma, 64 * rank, e * 64);
    }
    bool ok = mbar_wait(bar_tma, 0, lim, nullptr);
    if (ok && variant == 1) ok = mbar_wait(bar_a, 0, lim, nullptr);
    if (rank == 1) {
      // tell the even CTA that this CTA's operands are in place
      if (ok) {
        tc_fence_before();
        mbar_arrive_cluster(mapa_shared(bar_peer, 0));
      } else {
        atomicOr(status, kStatusTimeout);
      }
    } else {
      ok = ok && mbar_wait_cluster(bar_peer, 0, lim, nullptr);
      tc_fence_after();
      if (ok) {
        if (variant == 0) {
          for (int kk = 0; kk < 8; ++kk)
            tc_mma_ss_pair(tmem, sdesc_sw128(sA + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                           sdesc_sw128(sB + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                           idesc_bf16_f32(256, 256, false), kk > 0);
        } else {
          for (int kk = 0; kk < 16; ++kk)
            tc_mma_ts_pair(tmem, tmem + 256 + kk * 8, sdesc_sw128(sB + kk * 2048, 32768, 1024),
                           idesc_bf16_f32(256, 128, true), kk > 0);
        }
        tc_commit_pair(bar_mma, 0x3);
      } else {
        atomicOr(status, kStatusTimeout);
      }
    }
  }
  if (warp < 4) {
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const int row = 128 * rank + tid;
    if (variant == 1 && same) {   // row `row` of P into tensor memory as packed bf16 pairs
      const uint32_t* prow = reinterpret_cast<const uint32_t*>(p_glob + row * 256);
      for (int h = 0; h < 4; ++h) {
        uint32_t r[32];
        for (int i = 0; i < 32; ++i) r[i] = prow[h * 32 + i];
        tmem_st32(tmem + lane_off + 256 + h * 32, r);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_a);
    }
    const bool done = same && warp_wait_any(bar_mma, lim);
    tc_fence_after();
    const int ncols = variant == 0 ? 256 : 128;
    if (done) {
      for (int cc = 0; cc < ncols / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + cc * 32, r);
        tmem_ld_wait();
        for (int i = 0; i < 32; ++i) c[row * ncols + cc * 32 + i] = __uint_as_float(r[i]);
      }
    } else if (same) {
      atomicOr(status, kStatusTimeout);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // no product of the pair may still read either CTA's memory
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

cudaError_t launch_mma_pair_selftest(const CUtensorMap& a, const CUtensorMap& b,
                                     const void* p_glob, float* c, int variant, int* status,
                                     uint64_t lim, cudaStream_t st) {
  const uint32_t smem = 65536 + 1024 + 1024;
  cudaError_t e = cudaFuncSetAttribute(mma_pair_selftest_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  mma_pair_selftest_kernel<<<2, 160, smem, st>>>(a, b, static_cast<const __nv_bfloat16*>(p_glob),
                                                 c, variant, status, lim);
  return cudaGetLastError();
}


// ---------------------------------------------------------------- pair forward

constexpr int kPBM = 128;       // rows per CTA (two 64-token query blocks)
constexpr int kPBN = 256;       // keys per tile (four union entries)
constexpr int kPEntries = 4;
constexpr int kPThreads = 384;
constexpr int kPRegsSoftmax = 216, kPRegsOther = 72, kPRegsLaunch = 168;
constexpr int kPMaxNb = 4096;
constexpr uint32_t kPTmemCols = 512, kPColS = 0, kPColP = 256, kPColO = 384;
constexpr float kPFixedRefSumLimit = 65536.0f;

struct PairSmem {
  static constexpr uint32_t kQBytes = kPBM * 128 * 2;        // the CTA's query tile (d = 128)
  static constexpr uint32_t kKBytes = 128 * 128 * 2;         // its 128 keys of a K tile
  static constexpr uint32_t kVBytes = kPBN * 64 * 2;         // its 64 columns of a V tile
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + kQBytes;         // 2 stages
  static constexpr uint32_t kOffV = kOffK + 2 * kKBytes;     // 2 stages
  static constexpr uint32_t kOffBar = kOffV + 2 * kVBytes;   // 32 mbarriers
  static constexpr uint32_t kOffMisc = kOffBar + 256;        // tmem base, abort, n_u
  static constexpr uint32_t kOffXch = kOffMisc + 64;         // [2 parities][2 halves][128 rows] fp32
  static constexpr uint32_t kOffBitmap = kOffXch + 2 * 2 * kPBM * 4;   // 4 x kPMaxNb/32 words
  static constexpr uint32_t kOffList = kOffBitmap + 4 * (kPMaxNb / 32) * 4;
  static constexpr uint32_t kBytes = kOffList + kPMaxNb * 4;
  static constexpr uint32_t kAlloc = kBytes + 1024;
};

enum : int {
  kPQFull = 0,      // this CTA's Q landed
  kPKFull,          // + stage: this CTA's K half landed (2)
  kPVFull = 3,      // + stage: this CTA's V half landed (2)
  kPKEmpty = 5,     // + stage: S over the stage done (2), both CTAs
  kPVEmpty = 7,     // + stage: PV over the stage done (2), both CTAs
  kPSFull = 9,      // S(t) in both CTAs' tensor memory
  kPOFull,          // PV(t) done
  kPQPeer,          // even CTA: the odd CTA's Q landed
  kPKPeer,          // + stage (2): the odd CTA's K half landed
  kPVPeer = 14,     // + stage (2): the odd CTA's V half landed
  kPSFree = 16,     // even CTA: all 16 softmax warps copied S(t)
  kPPFull,          // even CTA: all 16 softmax warps wrote P(t)
  kPDrain,
  kPPair,           // + lane quarter (4)
  kPNumBars = kPPair + 4
};

struct PairParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  __nv_bfloat16* o;
  float* lse;
  int* status;
  int S, nb, ngroups;       // ngroups = query-block quadruples per head
  float scale_log2;
  uint64_t wait_limit_ns;
  int* redo;
};

__device__ __forceinline__ void pair_abort(volatile int* abort, int* status, int bit) {
  *abort = 1;
  atomicOr(status, bit);
}

__device__ __forceinline__ bool warp_wait_cl(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                             const volatile int* abort) {
  return __all_sync(0xffffffffu, mbar_wait_cluster(bar, parity, limit_ns, abort));
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPThreads, 1)
    bsa_fwd_pair_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const PairParams prm) {
  using L = PairSmem;
  constexpr int D = 128;
  extern __shared__ uint8_t pair_smem_raw[];
  const uint32_t raw = smem_addr(pair_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = pair_smem_raw + (base - raw);
  const uint32_t sQ = base + L::kOffQ, sK = base + L::kOffK, sV = base + L::kOffV;
  const uint32_t bar0 = base + L::kOffBar;
  uint32_t* misc = reinterpret_cast<uint32_t*>(gbase + L::kOffMisc);
  volatile uint32_t* tmem_holder = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* n_union_s = reinterpret_cast<volatile int*>(misc + 2);
  float* xch = reinterpret_cast<float*>(gbase + L::kOffXch);
  uint32_t* bm = reinterpret_cast<uint32_t*>(gbase + L::kOffBitmap);   // [4][kPMaxNb/32]
  int32_t* ulist = reinterpret_cast<int32_t*>(gbase + L::kOffList);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int item = blockIdx.x >> 1;
  const int bh = item / prm.ngroups;
  const int grp = item % prm.ngroups;
  const int nb = prm.nb;
  const int r4 = 4 * grp;                        // first query block of the quadruple
  const int r0 = r4 + 2 * static_cast<int>(rank);   // this CTA's first query block
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
  // the even CTA's copy of barrier i
  auto lead_bar = [&](int i) { return mapa_shared(bar(i), 0); };

  // ---------------------------------------------------------------- setup
  if (tid == 0) {
    for (int i = 0; i < kPNumBars; ++i) {
      uint32_t cnt = 1;
      if (i == kPSFree || i == kPPFull) cnt = 16;
      if (i >= kPPair) cnt = 64;
      mbar_init(bar(i), cnt);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc_pair(smem_addr(misc), kPTmemCols);
    tmem_relinquish_pair();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  const int nw = (nb + 31) >> 5;
  for (int i = tid; i < 4 * (kPMaxNb / 32); i += kPThreads) bm[i] = 0u;
  __syncthreads();
  for (int qb = 0; qb < 4; ++qb) {
    if (r4 + qb >= nb) break;
    const int64_t g = static_cast<int64_t>(bh) * nb + r4 + qb;
    const int b = prm.row_ptr[g], e = prm.row_ptr[g + 1];
    uint32_t* bmq = bm + qb * (kPMaxNb / 32);
    for (int i = b + tid; i < e; i += kPThreads) {
      const int c = prm.col_idx[i];
      if (static_cast<unsigned>(c) < static_cast<unsigned>(nb)) atomicOr(&bmq[c >> 5], 1u << (c & 31));
      else atomicOr(prm.status, kStatusBadIndex);
    }
  }
  __syncthreads();
  if (warp == 8) {   // the union of the four lists in ascending block order, 4-bit memberships
    int run = 0;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      const int w = w0 + lane;
      uint32_t u[4];
#pragma unroll
      for (int qb = 0; qb < 4; ++qb) u[qb] = w < nw ? bm[qb * (kPMaxNb / 32) + w] : 0u;
      uint32_t any = u[0] | u[1] | u[2] | u[3];
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
        int mem = 0;
#pragma unroll
        for (int qb = 0; qb < 4; ++qb) mem |= static_cast<int>((u[qb] >> b) & 1u) << qb;
        ulist[pos++] = (w * 32 + b) | (mem << 16);
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) *n_union_s = run;
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // both CTAs: barriers initialised, tensor memory allocated
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  // the two CTAs must hold the same tensor-memory columns and the same union
  {
    const uint32_t peer_tmem = ld_shared_cluster_u32(mapa_shared(smem_addr(misc), rank ^ 1u));
    const uint32_t peer_nu =
        ld_shared_cluster_u32(mapa_shared(smem_addr(const_cast<int*>(n_union_s)), rank ^ 1u));
    if (peer_tmem != tmem || static_cast<int>(peer_nu) != *n_union_s) {
      if (tid == 0) pair_abort(abort_flag, prm.status, kStatusBadIndex);
    }
  }
  __syncthreads();
  const bool consistent = *abort_flag == 0;
  const int n_u = consistent ? *n_union_s : 0;
  const int n_t = (n_u + kPEntries - 1) / kPEntries;
  const uint64_t lim = prm.wait_limit_ns;
  const int t_off =
      n_t > 0 ? static_cast<int>((static_cast<int64_t>(grp) * n_t) / prm.ngroups) : 0;
  auto tile_of = [&](int t) {
    const int u = t + t_off;
    return u >= n_t ? u - n_t : u;
  };
  auto tile_entry = [&](int t, int e) {
    const int u = tile_of(t);
    return (kPEntries * u + e < n_u) ? ulist[kPEntries * u + e] : 0;
  };

  if (warp >= 8) {
  setmaxnreg_dec<kPRegsOther>();
  if ((warp == 8 || warp == 10) && lane == 0 && n_t > 0) {
    // ------------------------------------------------------------ TMA producers
    const bool is_k = warp == 8;
    const CUtensorMap* map = is_k ? &tmK : &tmV;
    const int full0 = is_k ? kPKFull : kPVFull, empty0 = is_k ? kPKEmpty : kPVEmpty;
    const uint32_t stage_bytes = is_k ? L::kKBytes : L::kVBytes;
    const uint32_t buf0 = is_k ? sK : sV;
    int armed = 0;
    if (is_k) {
      mbar_arrive_expect_tx(bar(kPQFull), L::kQBytes);
      for (int qb = 0; qb < 2; ++qb)   // a block past the end repeats the last (rows unused)
        for (int h = 0; h < 2; ++h)
          tma_load_2d(sQ + h * kPBM * 128 + qb * 64 * 128, &tmQ, bar(kPQFull), h * 64,
                      static_cast<int32_t>(static_cast<int64_t>(bh) * prm.S +
                                           static_cast<int64_t>(min(r0 + qb, nb - 1)) * 64));
    }
    const int last = ulist[n_u - 1] & 0xFFFF;
    for (int t = 0; t < n_t; ++t) {
      const int st = t & 1;
      if (t >= 2 && !mbar_wait_cluster(bar(empty0 + st), ((t - 2) >> 1) & 1, lim, abort_flag)) {
        pair_abort(abort_flag, prm.status, kStatusTimeout);
        break;
      }
      mbar_arrive_expect_tx(bar(full0 + st), stage_bytes);
      ++armed;
      const uint32_t buf = buf0 + st * stage_bytes;
      const int u = tile_of(t);
      if (is_k) {
        // this CTA's keys: entries 2*rank, 2*rank+1 of the tile, both d halves
        for (int e = 0; e < 2; ++e) {
          const int ei = 2 * static_cast<int>(rank) + e;
          const int j = (kPEntries * u + ei < n_u) ? (ulist[kPEntries * u + ei] & 0xFFFF) : last;
          const int32_t y = static_cast<int32_t>(static_cast<int64_t>(bh) * prm.S +
                                                 static_cast<int64_t>(j) * 64);
          for (int h = 0; h < 2; ++h) tma_load_2d(buf + h * 128 * 128 + e * 64 * 128, map, bar(full0 + st), h * 64, y);
        }
      } else {
        // this CTA's 64 columns of d for all four entries
        for (int e = 0; e < kPEntries; ++e) {
          const int j = (kPEntries * u + e < n_u) ? (ulist[kPEntries * u + e] & 0xFFFF) : last;
          const int32_t y = static_cast<int32_t>(static_cast<int64_t>(bh) * prm.S +
                                                 static_cast<int64_t>(j) * 64);
          tma_load_2d(buf + e * 64 * 128, map, bar(full0 + st), 64 * static_cast<int>(rank), y);
        }
      }
    }
    // drain: every armed phase must complete before shared memory is released
    if (is_k) mbar_wait(bar(kPQFull), 0, kPairDrainLimitNs, nullptr);
    for (int st = 0; st < 2; ++st) {
      const int n_s = (armed + 1 - st) / 2;   // tiles t < armed with t & 1 == st
      if (n_s > 0) mbar_wait(bar(full0 + st), (n_s - 1) & 1, kPairDrainLimitNs, nullptr);
    }
  } else if (warp == 9 && lane == 0 && n_t > 0 && leader) {
    // ------------------------------------------------------------ pair MMA issuer
    constexpr uint32_t idesc_qk = idesc_bf16_f32(2 * kPBM, kPBN, false);
    constexpr uint32_t idesc_pv = idesc_bf16_f32(2 * kPBM, D, true);
    auto issue_s = [&](int t) {
      const uint32_t kb = sK + (t & 1) * L::kKBytes;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t offq = (kk >> 2) * (kPBM * 128) + (kk & 3) * 32;
        const uint32_t offk = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
        tc_mma_ss_pair(tmem + kPColS, sdesc_sw128(sQ + offq, 16, 1024),
                       sdesc_sw128(kb + offk, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
      }
      tc_commit_pair(bar(kPSFull), 0x3);
      tc_commit_pair(bar(kPKEmpty + (t & 1)), 0x3);
    };
    auto issue_pv = [&](int t) {
      const uint32_t vb = sV + (t & 1) * L::kVBytes;
#pragma unroll
      for (int kk = 0; kk < kPBN / 16; ++kk)
        tc_mma_ts_pair(tmem + kPColO, tmem + kPColP + kk * 8,
                       sdesc_sw128(vb + kk * 16 * 128, L::kVBytes, 1024), idesc_pv,
                       (t > 0 || kk > 0) ? 1u : 0u);
      tc_commit_pair(bar(kPOFull), 0x3);
      tc_commit_pair(bar(kPVEmpty + (t & 1)), 0x3);
    };
    auto kv_ready = [&](int full0, int peer0, int t) {
      const uint32_t ph = (t >> 1) & 1;
      return mbar_wait(bar(full0 + (t & 1)), ph, lim, abort_flag) &&
             mbar_wait_cluster(bar(peer0 + (t & 1)), ph, lim, abort_flag);
    };
    bool ok = mbar_wait(bar(kPQFull), 0, lim, abort_flag) &&
              mbar_wait_cluster(bar(kPQPeer), 0, lim, abort_flag) && kv_ready(kPKFull, kPKPeer, 0);
    if (ok) {
      tc_fence_after();
      issue_s(0);
    }
    for (int t = 0; ok && t < n_t; ++t) {
      if (t + 1 < n_t) {
        // S(t+1) overwrites S(t): every softmax warp of both CTAs must hold S(t)
        if (!mbar_wait_cluster(bar(kPSFree), t & 1, lim, abort_flag) ||
            !kv_ready(kPKFull, kPKPeer, t + 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_s(t + 1);
      }
      if (!mbar_wait_cluster(bar(kPPFull), t & 1, lim, abort_flag) ||
          !kv_ready(kPVFull, kPVPeer, t)) {
        ok = false;
        break;
      }
      tc_fence_after();
      issue_pv(t);
    }
    if (!ok) pair_abort(abort_flag, prm.status, kStatusTimeout);
    // drain: every product issued must finish before either CTA's memory is released
    tc_commit_pair(bar(kPDrain), 0x1);
    mbar_wait(bar(kPDrain), 0, kPairDrainLimitNs, nullptr);
  } else if ((warp == 9 || warp == 11) && lane == 0 && n_t > 0 && !leader) {
    // ------------------------------------------------------------ forwarders (odd CTA)
    // warp 9: K halves; warp 11: Q, then V halves
    const bool fwd_k = warp == 9;
    bool ok = true;
    if (!fwd_k) {
      ok = mbar_wait(bar(kPQFull), 0, lim, abort_flag);
      if (ok) mbar_arrive_cluster(lead_bar(kPQPeer));
    }
    const int full0 = fwd_k ? kPKFull : kPVFull, peer0 = fwd_k ? kPKPeer : kPVPeer;
    for (int t = 0; ok && t < n_t; ++t) {
      ok = mbar_wait(bar(full0 + (t & 1)), (t >> 1) & 1, lim, abort_flag);
      if (ok) mbar_arrive_cluster(lead_bar(peer0 + (t & 1)));
    }
    if (!ok) pair_abort(abort_flag, prm.status, kStatusTimeout);
  }
  } else {
    setmaxnreg_inc<kPRegsSoftmax>();
    // ------------------------------------------------------------ softmax (warps 0-7)
    const int quarter = warp & 3;
    const int half = warp >> 2;
    const int row = quarter * 32 + lane;
    const int qh = row >> 6;
    const int qblock = r0 + qh;
    const bool row_valid = qblock < nb;
    const int bit = 1 << (16 + 2 * static_cast<int>(rank) + qh);
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_base = tmem + lane_off + kPColS + 128u * half;
    const uint32_t p_base = tmem + lane_off + kPColP + 64u * half;
    const uint32_t o_base = tmem + lane_off + kPColO + static_cast<uint32_t>(D / 2) * half;
    const uint32_t pair_bar = bar(kPPair + quarter);
    const uint32_t sfree_bar = lead_bar(kPSFree), pfull_bar = lead_bar(kPPFull);
    const float sl2 = prm.scale_log2;
    float m = -INFINITY;
    float l = 0.f;
    int pair_n = 0;
    bool ok = true;
    for (int t = 0; t < n_t; ++t) {
      const bool v0 = (tile_entry(t, 2 * half) & bit) != 0;
      const bool v1 = (tile_entry(t, 2 * half + 1) & bit) != 0;
      if (!warp_wait_cl(bar(kPSFull), t & 1, lim, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[4][32];
      if (v0 && v1) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) tmem_ld32(s_base + 32 * ch, sv[ch]);
      } else {
        if (v0) { tmem_ld32(s_base, sv[0]); tmem_ld32(s_base + 32, sv[1]); }
        if (v1) { tmem_ld32(s_base + 64, sv[2]); tmem_ld32(s_base + 96, sv[3]); }
      }
      tmem_ld_wait();
      // S(t) is in registers: the pair may overwrite it with S(t+1)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(sfree_bar);
      // the row's reference: the max of the first key tile its block lists,
      // agreed with the other warp of the lane quarter, then kept
      const bool agree = __any_sync(0xffffffffu, m == -INFINITY);
      bool pv_done = t == 0;
      if (agree) {
        float mx[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          if ((ch < 2) ? v0 : v1) {
#pragma unroll
            for (int i = 0; i < 32; ++i) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(sv[ch][i]));
          }
        }
        const float m_part = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * sl2;
        xch[((pair_n & 1) * 2 + half) * kPBM + row] = m_part;
        mbar_arrive(pair_bar);
        if (!warp_wait_cl(pair_bar, pair_n & 1, lim, abort_flag)) { ok = false; break; }
        const float m_tile = fmaxf(m_part, xch[((pair_n & 1) * 2 + (half ^ 1)) * kPBM + row]);
        ++pair_n;
        if (m_tile > -INFINITY && m == -INFINITY) m = m_tile;
      }
      const bool live = m > -INFINITY;
      const float mneg = live ? -m : 0.f;
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[4][16];
      if (v0 && v1 && __all_sync(0xffffffffu, live)) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(sv[ch][2 * i]), sl2, mneg));
            const float p1 = fast_exp2(fmaf(__uint_as_float(sv[ch][2 * i + 1]), sl2, mneg));
            rs[i & 3] += p0 + p1;
            pk[ch][i] = pack_bf16x2(p0, p1);
          }
        }
      } else {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          if (((ch < 2) ? v0 : v1) && live) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float p0 = fast_exp2(fmaf(__uint_as_float(sv[ch][2 * i]), sl2, mneg));
              const float p1 = fast_exp2(fmaf(__uint_as_float(sv[ch][2 * i + 1]), sl2, mneg));
              rs[i & 3] += p0 + p1;
              pk[ch][i] = pack_bf16x2(p0, p1);
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[ch][i] = 0u;
          }
        }
      }
      const float l_tile = (rs[0] + rs[1]) + (rs[2] + rs[3]);
      l += l_tile;
      // a row whose later keys outgrow the fixed reference asks for the exact pass
      if (!agree && __any_sync(0xffffffffu, !(l_tile <= kPFixedRefSumLimit)) && lane == 0)
        atomicExch(prm.redo, 1);
      if (!pv_done && !warp_wait_cl(bar(kPOFull), (t - 1) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_st16(p_base + ch * 16, pk[ch]);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(pfull_bar);
    }
    if (!ok) pair_abort(abort_flag, prm.status, kStatusTimeout);
    // ------------------------------------------------------------ epilogue
    bool have_o = false;
    if (ok && n_t > 0) {
      have_o = warp_wait_cl(bar(kPOFull), (n_t - 1) & 1, lim, abort_flag);
      if (!have_o) pair_abort(abort_flag, prm.status, kStatusTimeout);
      tc_fence_after();
    }
    bool have_l = ok;
    float l_row = l;
    if (ok) {
      xch[((pair_n & 1) * 2 + half) * kPBM + row] = l;
      mbar_arrive(pair_bar);
      have_l = warp_wait_cl(pair_bar, pair_n & 1, lim, abort_flag);
      if (!have_l) pair_abort(abort_flag, prm.status, kStatusTimeout);
      else l_row = l + xch[((pair_n & 1) * 2 + (half ^ 1)) * kPBM + row];
    }
    const bool write = consistent && row_valid && have_l && (n_t == 0 || have_o);
    const int64_t grow = static_cast<int64_t>(bh) * prm.S +
                         (row_valid ? static_cast<int64_t>(qblock) * 64 + (row & 63) : 0);
    const float inv_l = l_row > 0.f ? 1.f / l_row : 0.f;
    __nv_bfloat16* orow = prm.o + grow * D + (D / 2) * half;
#pragma unroll
    for (int cc = 0; cc < D / 64; ++cc) {
      uint32_t o[32];
      if (have_o) {
        tmem_ld32(o_base + cc * 32, o);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) o[i] = 0u;
      }
      if (write) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
          w[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
        uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
    }
    if (write && half == 0 && prm.lse != nullptr)
      prm.lse[grow] = l_row > 0.f ? (m + __log2f(l_row)) * 0.69314718055994530942f : -INFINITY;
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();   // no product of the pair may still read or write either CTA's memory
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kPTmemCols);
  }
}

// Number of launches: one cluster of two CTAs per (b, h, quadruple of query
// blocks).
cudaError_t launch_bsa_fwd_pair(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                                const int32_t* row_ptr, const int32_t* col_idx, void* o,
                                float* lse, int* status, int* redo, int BH, int S, float scale,
                                uint64_t wait_limit_ns, cudaStream_t st) {
  PairParams prm;
  prm.row_ptr = row_ptr;
  prm.col_idx = col_idx;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.status = status;
  prm.S = S;
  prm.nb = S / 64;
  prm.ngroups = (prm.nb + 3) / 4;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.wait_limit_ns = wait_limit_ns;
  prm.redo = redo;
  const int64_t nitems = static_cast<int64_t>(BH) * prm.ngroups;
  if (nitems == 0) return cudaSuccess;
  constexpr uint32_t smem = PairSmem::kAlloc;
  static_assert(8 * kPRegsSoftmax + 4 * kPRegsOther <= 12 * kPRegsLaunch, "register split");
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, bsa_fwd_pair_kernel);
  if (e != cudaSuccess) return e;
  if (attr.numRegs < kPRegsLaunch) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(bsa_fwd_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  bsa_fwd_pair_kernel<<<static_cast<unsigned>(2 * nitems), kPThreads, smem, st>>>(q, k, v, prm);
  return cudaGetLastError();
}

}  // namespace nabla
