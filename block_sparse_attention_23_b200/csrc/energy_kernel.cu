// Block attention energy on sm_100a: for every listed (query block r, key
// block c) pair, the softmax probability mass that the 64 queries of block r
// place on the 64 keys of block c, averaged over the queries:
//
//   E[r][c] = (1/64) * sum_{i in r} sum_{j in c} exp(scale * q_i.k_j - LSE_i)
//
// With LSE from a dense forward pass, E is the true block-level attention map
// (each row of E sums to 1).  It is the quantity two of the pages rank blocks
// by: the "energy" (summed attention scores) per block that CalibAtt's offline
// calibration thresholds ("Accelerating Text-to-Video Generation with Calibrated
// Sparse Attention", section 2 "Methodologie: CalibAtt", A "Offline Kalibratie"), and the per-block true attention mass of the
// referee's fidelity check on NABLA's pooled proxy ("NABLA: Neighborhood
// Adaptive Block-Level Attention", review, major comment 1).  block_mass[r],
// the sum of E[r][c] over the listed c, is the fraction of the true mass that
// a block list retains.
//
// Work decomposition: one CTA per (b, h, pair of query blocks 2p, 2p+1) = one
// 128-row query tile; the key blocks visited are the union of the two CSR
// rows (2-bit membership), four union entries per 256-key tile, each entry a
// contiguous 64 x d slab loaded by one 2D TMA box per 64 columns.  S = Q K^T
// (N = 256: the full tensor rate) goes to tensor memory (two 256-column
// buffers, so the next tile's MMA runs while the current one is
// exponentiated); a thread owns one query row, reads its 256 columns in two
// halves of 128, exponentiates against its LSE and sums each 64-key entry;
// the two warps of a query block add their warp sums into a shared-memory row
// of E (exactly two addends onto zero: the result does not depend on their
// order).
//
// Roles (384 threads): warps 0-7 exponentiate and sum in two groups of four
// (group g takes the tiles t = g mod 2 and the S buffer g, so two warps per
// SM sub-partition keep the exponential unit busy), warp 8 compacts the union
// list and issues the TMA loads, warp 9 owns tensor memory and issues the MMAs,
// warps 10-11 idle.  Every mbarrier wait is time-bounded; a wait that runs out records
// kStatusTimeout, raises the CTA's abort flag and the CTA drains its own work
// before freeing tensor memory; an aborted CTA writes no output.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_primitives.cuh"

namespace nabla {

constexpr int kEM = 128;            // query rows per CTA (two blocks)
constexpr int kEN = 256;            // keys per tile (four list entries)
constexpr int kEStages = 2;         // K ring depth
constexpr int kEThreads = 384;
constexpr int kESumWarps = 8;                     // two groups of four, one per S buffer
constexpr int kEProducerWarp = 8, kEMmaWarp = 9;
constexpr int kEMaxNb = 4096;
constexpr uint32_t kETmemCols = 512;
constexpr uint64_t kEDrainNs = 1000000000ull;

template <int D>
struct EnergySmem {
  static constexpr int kDH = D / 64;
  static constexpr uint32_t kQBytes = kEM * D * 2;
  static constexpr uint32_t kKBytes = kEN * D * 2;
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + kQBytes;
  static constexpr uint32_t kOffBar = kOffK + kEStages * kKBytes;   // 16 mbarriers
  static constexpr uint32_t kOffMisc = kOffBar + 128;               // tmem base, abort, n_u
  static constexpr uint32_t kOffBitmap = kOffMisc + 64;             // [2][kEMaxNb/32]
  static constexpr uint32_t kOffList = kOffBitmap + 2 * (kEMaxNb / 32) * 4;
  static constexpr uint32_t kOffRowE = kOffList + kEMaxNb * 4;      // [2][kEMaxNb] fp32
  static constexpr uint32_t kBytes = kOffRowE + 2 * kEMaxNb * 4;
  static constexpr uint32_t kAlloc = kBytes + 1024;                 // 1024-byte alignment slack
};

enum : int {
  kEBarQFull = 0,
  kEBarKFull = 1,                        // + stage
  kEBarKEmpty = kEBarKFull + kEStages,   // + stage
  kEBarSFull = kEBarKEmpty + kEStages,   // + S buffer
  kEBarSFree = kEBarSFull + 2,           // + S buffer
  kEBarDrain = kEBarSFree + 2,
  kENumBars = kEBarDrain + 1
};
static_assert(kENumBars * 8 <= 128, "barrier area");

struct EnergyParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  const float* lse;        // [B*H*S] natural-log LSE of each query row
  float* energy;           // [B*H*nb*nb]
  float* block_mass;       // [B*H*nb] or null
  int* status;
  int S, nb, npairs;
  float scale_log2;        // softmax scale * log2(e)
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ bool e_warp_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                            const volatile int* abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, limit_ns, abort));
}

__device__ __forceinline__ void e_abort(volatile int* abort, int* status) {
  *abort = 1;
  atomicOr(status, kStatusTimeout);
}

__device__ __forceinline__ float e_warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

template <int D>
__global__ void __launch_bounds__(kEThreads, 1)
    block_energy_kernel(const __grid_constant__ CUtensorMap tmQ,
                        const __grid_constant__ CUtensorMap tmK, const EnergyParams prm) {
  using L = EnergySmem<D>;
  extern __shared__ uint8_t en_smem_raw[];
  const uint32_t raw = smem_addr(en_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = en_smem_raw + (base - raw);
  const uint32_t sQ = base + L::kOffQ;
  const uint32_t sK = base + L::kOffK;
  const uint32_t bar0 = base + L::kOffBar;
  uint32_t* misc = reinterpret_cast<uint32_t*>(gbase + L::kOffMisc);
  volatile uint32_t* tmem_holder = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* n_union_s = reinterpret_cast<volatile int*>(misc + 2);
  uint32_t* bm = reinterpret_cast<uint32_t*>(gbase + L::kOffBitmap);
  int32_t* ulist = reinterpret_cast<int32_t*>(gbase + L::kOffList);
  float* rowE = reinterpret_cast<float*>(gbase + L::kOffRowE);   // [2][kEMaxNb]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / prm.npairs;
  const int r0 = 2 * (blockIdx.x % prm.npairs);
  const int nb = prm.nb;
  const int nq = min(2, nb - r0);                 // query blocks present (1 or 2)
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  // ---------------------------------------------------------------- setup
  if (tid == 0) {
    mbar_init(bar(kEBarQFull), 1);
    for (int s = 0; s < kEStages; ++s) {
      mbar_init(bar(kEBarKFull + s), 1);
      mbar_init(bar(kEBarKEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(kEBarSFull + b), 1);
      mbar_init(bar(kEBarSFree + b), (kESumWarps / 2) * 32);
    }
    mbar_init(bar(kEBarDrain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kEMmaWarp) {
    tmem_alloc(smem_addr(misc), kETmemCols);
    tmem_relinquish();
  }
  if (warp == kEProducerWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  const int nw = (nb + 31) >> 5;
  for (int i = tid; i < 2 * (kEMaxNb / 32); i += kEThreads) bm[i] = 0u;
  for (int i = tid; i < nb; i += kEThreads) {
    rowE[i] = 0.f;
    rowE[kEMaxNb + i] = 0.f;
  }
  __syncthreads();
  for (int qb = 0; qb < nq; ++qb) {
    const int64_t g = static_cast<int64_t>(bh) * nb + r0 + qb;
    const int b = prm.row_ptr[g], e = prm.row_ptr[g + 1];
    uint32_t* bmq = bm + qb * (kEMaxNb / 32);
    for (int i = b + tid; i < e; i += kEThreads) {
      const int c = prm.col_idx[i];
      if (static_cast<unsigned>(c) < static_cast<unsigned>(nb)) atomicOr(&bmq[c >> 5], 1u << (c & 31));
      else atomicOr(prm.status, kStatusBadIndex);
    }
  }
  __syncthreads();
  if (warp == kEProducerWarp) {   // union of the two rows, ascending, 2-bit membership at bit 16
    int run = 0;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t u0 = w < nw ? bm[w] : 0u;
      const uint32_t u1 = w < nw ? bm[kEMaxNb / 32 + w] : 0u;
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
  const int n_t = (n_u + 3) >> 2;
  const uint64_t lim = prm.wait_limit_ns;
  auto tile_entry = [&](int t, int i) { return (4 * t + i < n_u) ? ulist[4 * t + i] : 0; };

  if (warp == kEProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && n_t > 0) {
      const int64_t row0 = static_cast<int64_t>(bh) * prm.S;
      int armed[kEStages] = {0, 0};
      mbar_arrive_expect_tx(bar(kEBarQFull), L::kQBytes);
      for (int qb = 0; qb < 2; ++qb) {
        const int rb = r0 + (qb < nq ? qb : 0);   // a missing second block repeats the first
        for (int h = 0; h < L::kDH; ++h)
          tma_load_2d(sQ + h * kEM * 128 + qb * 64 * 128, &tmQ, bar(kEBarQFull), h * 64,
                      static_cast<int32_t>(row0 + static_cast<int64_t>(rb) * 64));
      }
      const int last = ulist[n_u - 1] & 0xFFFF;   // padding entries repeat it (no row lists them)
      for (int t = 0; t < n_t; ++t) {
        const int s = t % kEStages, n = t / kEStages;
        if (t >= kEStages && !mbar_wait(bar(kEBarKEmpty + s), (n - 1) & 1, lim, abort_flag)) {
          e_abort(abort_flag, prm.status);
          break;
        }
        mbar_arrive_expect_tx(bar(kEBarKFull + s), L::kKBytes);
        ++armed[s];
        for (int kb = 0; kb < 4; ++kb) {
          const int j = (4 * t + kb < n_u) ? (ulist[4 * t + kb] & 0xFFFF) : last;
          for (int h = 0; h < L::kDH; ++h)
            tma_load_2d(sK + s * L::kKBytes + h * kEN * 128 + kb * 64 * 128, &tmK,
                        bar(kEBarKFull + s), h * 64,
                        static_cast<int32_t>(row0 + static_cast<int64_t>(j) * 64));
        }
      }
      // drain: every armed phase completes before shared memory is released
      mbar_wait(bar(kEBarQFull), 0, kEDrainNs, nullptr);
      for (int s = 0; s < kEStages; ++s)
        if (armed[s]) mbar_wait(bar(kEBarKFull + s), (armed[s] - 1) & 1, kEDrainNs, nullptr);
    }
  } else if (warp == kEMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_t > 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kEM, kEN, false);
      bool ok = mbar_wait(bar(kEBarQFull), 0, lim, abort_flag);
      for (int t = 0; ok && t < n_t; ++t) {
        const int b = t & 1, s = t % kEStages;
        if (!mbar_wait(bar(kEBarKFull + s), (t / kEStages) & 1, lim, abort_flag)) { ok = false; break; }
        // the S buffer is free once its group of four warps has loaded tile t-2
        if (t >= 2 && !mbar_wait(bar(kEBarSFree + b), ((t >> 1) - 1) & 1, lim, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kt = sK + s * L::kKBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offq = (kk >> 2) * (kEM * 128) + (kk & 3) * 32;
          const uint32_t offk = (kk >> 2) * (kEN * 128) + (kk & 3) * 32;
          tc_mma_ss(tmem + b * static_cast<uint32_t>(kEN), sdesc_sw128(sQ + offq, 16, 1024),
                    sdesc_sw128(kt + offk, 16, 1024), idesc, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(kEBarSFull + b));
        tc_commit(bar(kEBarKEmpty + s));
      }
      if (!ok) e_abort(abort_flag, prm.status);
      tc_commit(bar(kEBarDrain));
      mbar_wait(bar(kEBarDrain), 0, kEDrainNs, nullptr);
    }
  } else if (warp < kESumWarps) {
    // ------------------------------------------------------------ exponentiate and sum
    const int grp = warp >> 2;                 // tiles t = grp mod 2, S buffer grp
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;       // tile row == tensor-memory lane
    const int qh = row >> 6;                   // query block r0 + qh (uniform per warp)
    const int bit = 1 << (16 + qh);
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = prm.scale_log2;
    float neg_lse2 = 0.f;
    bool live = false;
    if (qh < nq) {
      const float v = prm.lse[static_cast<int64_t>(bh) * prm.S + static_cast<int64_t>(r0 + qh) * 64 +
                              (row & 63)];
      live = v > -INFINITY && v < INFINITY;    // an empty row (LSE = -inf) contributes nothing
      neg_lse2 = live ? -v * 1.4426950408889634f : 0.f;
    }
    float* myE = rowE + qh * kEMaxNb;
    bool ok = true;
    for (int t = grp; t < n_t; t += 2) {
      const int b = grp;
      if (!e_warp_wait(bar(kEBarSFull + b), (t >> 1) & 1, lim, abort_flag)) { ok = false; break; }
      tc_fence_after();
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {           // entries 4t + 2hf, 4t + 2hf + 1
        const int e0 = tile_entry(t, 2 * hf), e1 = tile_entry(t, 2 * hf + 1);
        const bool v0 = (e0 & bit) != 0, v1 = (e1 & bit) != 0;   // uniform per warp
        const uint32_t sb = tmem + lane_off + b * static_cast<uint32_t>(kEN) + 128u * hf;
        uint32_t sv[4][32];
        // both entries listed (and every row live): the first 32 columns, then
        // the other 96 while the first are exponentiated
        const bool split = v0 && v1 && __all_sync(0xffffffffu, live);
        if (split) {
          tmem_ld32(sb, sv[0]);
          tmem_ld_wait();
          reg_fence32(sv[0]);
          tmem_ld32(sb + 32, sv[1]);
          tmem_ld32(sb + 64, sv[2]);
          tmem_ld32(sb + 96, sv[3]);
        } else {
          if (v0) { tmem_ld32(sb, sv[0]); tmem_ld32(sb + 32, sv[1]); }
          if (v1) { tmem_ld32(sb + 64, sv[2]); tmem_ld32(sb + 96, sv[3]); }
          tmem_ld_wait();
          if (hf == 1) {   // both halves read: the tensor cores may refill the buffer
            tc_fence_before();
            mbar_arrive(bar(kEBarSFree + b));
          }
        }
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        if (split) {
          // one straight-line block without per-chunk branches
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
#pragma unroll
            for (int i = 0; i < 32; ++i)
              acc[ch >> 1][i & 3] += fast_exp2(fmaf(__uint_as_float(sv[ch][i]), sl2, neg_lse2));
            if (ch == 0) {
              tmem_ld_wait();
              reg_fence32(sv[1]);
              reg_fence32(sv[2]);
              reg_fence32(sv[3]);
              if (hf == 1) {   // both halves read: the tensor cores may refill the buffer
                tc_fence_before();
                mbar_arrive(bar(kEBarSFree + b));
              }
            }
          }
        } else {
#pragma unroll
          for (int ch = 0; ch < 4; ++ch) {
            if (((ch < 2) ? v0 : v1) && live) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                acc[ch >> 1][i & 3] += fast_exp2(fmaf(__uint_as_float(sv[ch][i]), sl2, neg_lse2));
            }
          }
        }
        if (v0) {
          const float w = e_warp_sum((acc[0][0] + acc[0][1]) + (acc[0][2] + acc[0][3]));
          if (lane == 0) atomicAdd(&myE[e0 & 0xFFFF], w);
        }
        if (v1) {
          const float w = e_warp_sum((acc[1][0] + acc[1][1]) + (acc[1][2] + acc[1][3]));
          if (lane == 0) atomicAdd(&myE[e1 & 0xFFFF], w);
        }
      }
    }
    if (!ok) e_abort(abort_flag, prm.status);
  }

  // ---------------------------------------------------------------- write-out
  tc_fence_before();
  __syncthreads();
  const bool aborted = *abort_flag != 0;
  if (!aborted) {
    constexpr float kInv = 1.0f / 64.0f;
    for (int qb = 0; qb < nq; ++qb) {
      float* dst = prm.energy + (static_cast<int64_t>(bh) * nb + r0 + qb) * nb;
      const float* src = rowE + qb * kEMaxNb;
      for (int c = tid; c < nb; c += kEThreads) dst[c] = src[c] * kInv;
    }
    if (prm.block_mass != nullptr && warp < nq) {   // warp qb sums row qb in a fixed order
      const float* src = rowE + warp * kEMaxNb;
      float s = 0.f;
      for (int c = lane; c < nb; c += 32) s += src[c] * kInv;
      s = e_warp_sum(s);
      if (lane == 0) prm.block_mass[static_cast<int64_t>(bh) * nb + r0 + warp] = s;
    }
  }
  if (warp == kEMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kETmemCols);
  }
}

template <int D>
static cudaError_t launch_energy_t(const CUtensorMap& q, const CUtensorMap& k,
                                   const EnergyParams& prm, int64_t nitems, cudaStream_t st) {
  constexpr uint32_t smem = EnergySmem<D>::kAlloc;
  static_assert(smem <= 227 * 1024, "shared memory");
  cudaError_t e = cudaFuncSetAttribute(block_energy_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  block_energy_kernel<D><<<static_cast<unsigned>(nitems), kEThreads, smem, st>>>(q, k, prm);
  return cudaGetLastError();
}

cudaError_t launch_block_energy(const CUtensorMap& q, const CUtensorMap& k, const int32_t* row_ptr,
                                const int32_t* col_idx, const float* lse, float* energy,
                                float* block_mass, int* status, int BH, int S, int d, float scale,
                                uint64_t wait_limit_ns, cudaStream_t st) {
  EnergyParams prm;
  prm.row_ptr = row_ptr;
  prm.col_idx = col_idx;
  prm.lse = lse;
  prm.energy = energy;
  prm.block_mass = block_mass;
  prm.status = status;
  prm.S = S;
  prm.nb = S / 64;
  prm.npairs = (prm.nb + 1) / 2;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.wait_limit_ns = wait_limit_ns;
  const int64_t nitems = static_cast<int64_t>(BH) * prm.npairs;
  if (nitems == 0) return cudaSuccess;
  if (d == 128) return launch_energy_t<128>(q, k, prm, nitems, st);
  return launch_energy_t<64>(q, k, prm, nitems, st);
}

}  // namespace nabla
