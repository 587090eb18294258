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

}  // namespace nabla
