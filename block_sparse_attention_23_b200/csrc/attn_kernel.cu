// Block-sparse attention forward on sm_100a: tcgen05 MMAs with tensor-memory
// accumulators, TMA-fed K/V tiles gathered by block index, warp-specialised
// load / MMA / softmax roles.
//
// The arithmetic is FlashAttention's (FlashAttention abstract: exact attention
// by tiles with an online softmax; its block-sparse extension skips zero
// blocks), driven by the NABLA block mask ("NABLA: Neighborhood Adaptive
// Block-Level Attention": the binary block mask decides which N x N blocks
// are computed).
//
// Work decomposition
//   One CTA per (b, h, pair of query blocks): 128 query rows = query blocks
//   2p and 2p+1.  The key blocks visited are the union of the two CSR rows;
//   each union entry carries a 2-bit membership flag, and a query row whose
//   block did not list the key block treats it as masked (probability 0, no
//   exponentials evaluated).  Key tiles are 128 keys = two union entries (the
//   second may be a repeat that both rows mask).  Every 64-key block is one
//   contiguous slab of the [B,H,S,d] tensor, so each is a plain 2D TMA box at
//   row (bh*S + 64*j).
//
// Two independent softmax streams per row
//   Key half h of every tile (the tile's h-th 64-key block) feeds its own
//   accumulator O_h with its own running max m_h and sum l_h, so the two
//   threads that serve a row never wait for each other inside the key loop.
//   The epilogue merges them exactly:
//     M = max(m_0, m_1),  f_h = 2^(m_h - M),
//     O = (f_0 O_0 + f_1 O_1) / (f_0 l_0 + f_1 l_1),  LSE = ln2 (M + log2 L).
//   Each stream keeps a lazy maximum: m_h is raised (and O_h, l_h rescaled by
//   2^(m_old - m_new)) only when a tile exceeds it by more than 2^8, so p <= 256.
//
// Roles (352 threads)
//   warps 0-7  softmax.  Warp w serves tensor-memory lanes 32*(w%4).. (query
//              rows) and key half w/4: tcgen05.ld of its 64 S columns,
//              max, exp2, P (bf16) written over the first 32 of those
//              columns, lazy rescale of its O_h row, epilogue.
//   warp 8     TMA producer of Q and K (and the union-list compaction).
//   warp 10    TMA producer of V.
//   warp 9     tensor-memory allocation and the single MMA-issuing thread:
//              S_t = Q K_t^T into buffer t&1, then O_h += P_t,h V_t,h for
//              h = 0, 1 as soon as that half of P is in place (A operand read
//              from tensor memory).
//
// Tensor memory (512 columns): S/P buffers [0,128) and [128,256), O_0 at 256,
// O_1 at 384 (d columns each).  Ordering of the in-place P: S_{t+2} reuses
// buffer t&1 and is issued after PV_t by the same thread, and MMAs of one
// thread execute in issue order; the completion of S_t (which the softmax
// waits for) also implies the completion of PV_{t-2}, which read P_{t-2}.
//
// Every mbarrier wait is time-bounded; a wait that runs out records
// kStatusTimeout, raises a CTA-wide abort flag, and the CTA drains its own TMA
// loads and MMAs (bounded again) before freeing tensor memory and returning.
// The softmax warps share one named barrier, in the epilogue, and agree on
// aborts there through bar.red.and.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_primitives.cuh"

namespace nabla {

constexpr int kBM = 128;        // query rows per CTA (two 64-token blocks)
constexpr int kBN = 128;        // keys per tile (two 64-token blocks)
constexpr int kKStages = 3;     // K ring depth (K is needed one S-MMA after its slot frees)
constexpr int kVStages = 2;     // V ring depth
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = kSoftmaxThreads + 96;
constexpr int kProducerWarp = 8, kMmaWarp = 9, kVProducerWarp = 10;
constexpr int kMaxNb = 4096;    // blocks per head supported
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColS1 = 128, kColO0 = 256, kColO1 = 384;
constexpr float kRescaleThreshold = 8.0f;            // log2 units
constexpr uint64_t kDrainLimitNs = 1000000000ull;   // 1 s for draining in-flight work
constexpr int kSoftmaxBarrier = 1;                   // named barrier id of warps 0-7

template <int D>
struct AttnSmem {
  static constexpr int kDH = D / 64;                       // 64-column halves of d
  static constexpr uint32_t kQBytes = kBM * D * 2;
  static constexpr uint32_t kKVBytes = kBN * D * 2;        // one K or V stage
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + kQBytes;
  static constexpr uint32_t kOffV = kOffK + kKStages * kKVBytes;
  static constexpr uint32_t kOffBar = kOffV + kVStages * kKVBytes;  // 32 mbarriers
  static constexpr uint32_t kOffMisc = kOffBar + 256;      // tmem base, abort, n_u
  static constexpr uint32_t kOffRed = kOffMisc + 64;       // [2 quantity][2 half][128] floats
  static constexpr uint32_t kOffBitmap = kOffRed + 2 * 2 * kBM * 4;   // 2 x kMaxNb/32 words
  static constexpr uint32_t kOffList = kOffBitmap + 2 * (kMaxNb / 32) * 4;
  static constexpr uint32_t kBytes = kOffList + kMaxNb * 4;
  static constexpr uint32_t kAlloc = kBytes + 1024;        // slack for 1024-byte alignment
};

// Barrier slots inside the barrier area.
enum : int {
  kBarQFull = 0,
  kBarKFull = 1,                      // + stage
  kBarKEmpty = kBarKFull + kKStages,
  kBarVFull = kBarKEmpty + kKStages,
  kBarVEmpty = kBarVFull + kVStages,
  kBarSFull = kBarVEmpty + kVStages,  // + (t & 1): S_t ready
  kBarPFull = kBarSFull + 2,          // + 2*half + (t & 1): P_t,h written
  kBarOFull = kBarPFull + 4,          // + 2*half + (t & 1): PV_t,h done
  kBarDrain = kBarOFull + 4,
  kNumBars = kBarDrain + 1
};

struct AttnParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  __nv_bfloat16* o;
  float* lse;
  int* status;
  int H, S, nb, npairs;
  float scale_log2;        // softmax scale * log2(e)
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ void record_abort(volatile int* abort, int* status, int bit) {
  *abort = 1;
  atomicOr(status, bit);
}

// Every lane waits; the warp proceeds only if all lanes saw the phase complete,
// so the warp-collective tcgen05.ld/st that follow are never divergent.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                          const volatile int* abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, limit_ns, abort));
}

// Named barrier over `n` threads that also ANDs a predicate across them.
__device__ __forceinline__ bool bar_red_and(int id, int n, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    bsa_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const AttnParams prm) {
  using L = AttnSmem<D>;
  extern __shared__ uint8_t attn_smem_raw[];
  const uint32_t raw = smem_addr(attn_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = attn_smem_raw + (base - raw);

  const uint32_t sQ = base + L::kOffQ;
  const uint32_t sK = base + L::kOffK;
  const uint32_t sV = base + L::kOffV;
  const uint32_t bar0 = base + L::kOffBar;
  uint32_t* misc = reinterpret_cast<uint32_t*>(gbase + L::kOffMisc);
  volatile uint32_t* tmem_holder = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  volatile int* n_union_s = reinterpret_cast<volatile int*>(misc + 2);
  float* red = reinterpret_cast<float*>(gbase + L::kOffRed);
  uint32_t* bm1 = reinterpret_cast<uint32_t*>(gbase + L::kOffBitmap);
  uint32_t* bm2 = bm1 + kMaxNb / 32;
  int32_t* ulist = reinterpret_cast<int32_t*>(gbase + L::kOffList);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item = blockIdx.x;
  const int bh = item / prm.npairs;
  const int pair = item % prm.npairs;
  const int nb = prm.nb;
  const int r1 = 2 * pair, r2 = 2 * pair + 1;
  const bool has2 = r2 < nb;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  // ---------------------------------------------------------------- setup
  if (tid == 0) {
    mbar_init(bar(kBarQFull), 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(bar(kBarKFull + s), 1);
      mbar_init(bar(kBarKEmpty + s), 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(bar(kBarVFull + s), 1);
      mbar_init(bar(kBarVEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) mbar_init(bar(kBarSFull + b), 1);
    // P and O barriers alternate with the tile parity: a half's softmax can run
    // one tile ahead of the MMA thread, never two, so no barrier is ever two
    // phases ahead of its waiter
    for (int b = 0; b < 4; ++b) {
      mbar_init(bar(kBarPFull + b), kSoftmaxThreads / 2);
      mbar_init(bar(kBarOFull + b), 1);
    }
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_addr(misc), kTmemCols);
    tmem_relinquish();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  const int nw = (nb + 31) >> 5;
  for (int i = tid; i < 2 * nw; i += kThreads) (i < nw ? bm1[i] : bm2[i - nw]) = 0u;
  __syncthreads();
  {
    const int64_t g1 = static_cast<int64_t>(bh) * nb + r1;
    const int b1 = prm.row_ptr[g1], e1 = prm.row_ptr[g1 + 1];
    for (int i = b1 + tid; i < e1; i += kThreads) {
      const int c = prm.col_idx[i];
      if (static_cast<unsigned>(c) < static_cast<unsigned>(nb)) atomicOr(&bm1[c >> 5], 1u << (c & 31));
      else atomicOr(prm.status, kStatusBadIndex);
    }
    if (has2) {
      const int b2 = prm.row_ptr[g1 + 1], e2 = prm.row_ptr[g1 + 2];
      for (int i = b2 + tid; i < e2; i += kThreads) {
        const int c = prm.col_idx[i];
        if (static_cast<unsigned>(c) < static_cast<unsigned>(nb)) atomicOr(&bm2[c >> 5], 1u << (c & 31));
        else atomicOr(prm.status, kStatusBadIndex);
      }
    }
  }
  __syncthreads();
  if (warp == kProducerWarp) {   // compact the union in ascending block order
    int run = 0;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      const int w = w0 + lane;
      const uint32_t u1 = w < nw ? bm1[w] : 0u, u2 = w < nw ? bm2[w] : 0u;
      uint32_t u = u1 | u2;
      const int cnt = __popc(u);
      int incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
      }
      int pos = run + incl - cnt;
      while (u) {
        const int b = __ffs(u) - 1;
        u &= u - 1;
        ulist[pos++] = (w * 32 + b) | (static_cast<int>((u1 >> b) & 1u) << 16) |
                       (static_cast<int>((u2 >> b) & 1u) << 17);
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

  if (warp == kProducerWarp || warp == kVProducerWarp) {
    // ------------------------------------------------------------ TMA producers
    // warp 8 streams Q and K, warp 10 streams V: a V slot frees only after the
    // softmax of its tile, and must not hold back the K prefetch
    if (lane == 0 && n_t > 0) {
      const int64_t row0 = static_cast<int64_t>(bh) * prm.S;
      const bool is_k = warp == kProducerWarp;
      const int nst = is_k ? kKStages : kVStages;
      const uint32_t ring = is_k ? sK : sV;
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      const int full0 = is_k ? kBarKFull : kBarVFull, empty0 = is_k ? kBarKEmpty : kBarVEmpty;
      int armed[kKStages] = {0, 0, 0};
      if (is_k) {
        mbar_arrive_expect_tx(bar(kBarQFull), L::kQBytes);
        for (int qb = 0; qb < 2; ++qb)
          for (int h = 0; h < L::kDH; ++h)
            tma_load_2d(sQ + h * kBM * 128 + qb * 64 * 128, &tmQ, bar(kBarQFull), h * 64,
                        static_cast<int32_t>(row0 + (r1 + qb) * 64));
      }
      for (int t = 0; t < n_t; ++t) {
        const int s = t % nst, n = t / nst;
        const int j0 = ulist[2 * t] & 0xFFFF;
        const int j1 = (2 * t + 1 < n_u) ? (ulist[2 * t + 1] & 0xFFFF) : j0;
        if (t >= nst && !mbar_wait(bar(empty0 + s), (n - 1) & 1, lim, abort_flag)) {
          record_abort(abort_flag, prm.status, kStatusTimeout);
          break;
        }
        mbar_arrive_expect_tx(bar(full0 + s), L::kKVBytes);
        ++armed[s];
        for (int kb = 0; kb < 2; ++kb)
          for (int h = 0; h < L::kDH; ++h)
            tma_load_2d(ring + s * L::kKVBytes + h * kBN * 128 + kb * 64 * 128, map, bar(full0 + s),
                        h * 64, static_cast<int32_t>(row0 + (kb ? j1 : j0) * 64));
      }
      // drain: every armed phase must complete before shared memory is released
      if (is_k) mbar_wait(bar(kBarQFull), 0, kDrainLimitNs, nullptr);
      for (int s = 0; s < nst; ++s)
        if (armed[s]) mbar_wait(bar(full0 + s), (armed[s] - 1) & 1, kDrainLimitNs, nullptr);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_t > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, true);
      bool ok = mbar_wait(bar(kBarQFull), 0, lim, abort_flag);
      tc_fence_after();
      auto issue_s = [&](int u) -> bool {
        const int s = u % kKStages;
        if (!mbar_wait(bar(kBarKFull + s), (u / kKStages) & 1, lim, abort_flag)) return false;
        tc_fence_after();
        const uint32_t kt = sK + s * L::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBM * 128) + (kk & 3) * 32;
          const uint32_t offk = (kk >> 2) * (kBN * 128) + (kk & 3) * 32;
          tc_mma_ss(tmem + ((u & 1) ? kColS1 : kColS0), sdesc_sw128(sQ + off, 16, 1024),
                    sdesc_sw128(kt + offk, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(kBarKEmpty + s));
        tc_commit(bar(kBarSFull + (u & 1)));
        return true;
      };
      if (ok) ok = issue_s(0);
      for (int t = 0; ok && t < n_t; ++t) {
        // S_{t+1} goes ahead of PV_t so the softmax of tile t+1 can start while PV_t runs
        if (t + 1 < n_t && !issue_s(t + 1)) { ok = false; break; }
        const int s = t % kVStages;
        if (!mbar_wait(bar(kBarVFull + s), (t / kVStages) & 1, lim, abort_flag)) { ok = false; break; }
        const uint32_t vt = sV + s * L::kKVBytes;
        const uint32_t pbuf = tmem + ((t & 1) ? kColS1 : kColS0);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (!mbar_wait(bar(kBarPFull + 2 * h + (t & 1)), (t >> 1) & 1, lim, abort_flag)) { ok = false; break; }
          tc_fence_after();
          // keys [64h, 64h+64) of the tile: P columns pbuf + 64h + [0,32) (bf16 pairs),
          // V rows [64h, 64h+64); the two 64-column halves of d are kBN*128 bytes apart
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_ts(tmem + (h ? kColO1 : kColO0), pbuf + h * 64 + kk * 8,
                      sdesc_sw128(vt + (h * 4 + kk) * 16 * 128, kBN * 128, 1024), idesc_pv,
                      (t > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar(kBarOFull + 2 * h + (t & 1)));
        }
        if (!ok) break;
        tc_commit(bar(kBarVEmpty + s));
      }
      if (!ok) record_abort(abort_flag, prm.status, kStatusTimeout);
      // drain: all MMAs this thread issued must finish before tensor memory is freed
      tc_commit(bar(kBarDrain));
      mbar_wait(bar(kBarDrain), 0, kDrainLimitNs, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax (warps 0-7)
    const int quarter = warp & 3;
    const int half = warp >> 2;                // key half of every tile this warp handles
    const int row = quarter * 32 + lane;       // query row == tensor-memory lane
    const int qh = row >> 6;                   // 0: block r1, 1: block r2
    const bool row_valid = qh == 0 || has2;
    const int bitsel = 1 << (16 + qh);
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t o_col = half ? kColO1 : kColO0;
    const float sl2 = prm.scale_log2;
    float m = -INFINITY;        // lazy running max of this stream, log2 units
    float l = 0.f;              // running sum of this stream
    bool ok = true;
    for (int t = 0; t < n_t; ++t) {
      const int b = t & 1;
      const int e = (2 * t + half < n_u) ? ulist[2 * t + half] : 0;
      const bool valid = (e & bitsel) != 0;    // uniform per warp
      if (!warp_wait(bar(kBarSFull + b), (t >> 1) & 1, lim, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const uint32_t scol = tmem + lane_off + (b ? kColS1 : kColS0) + half * 64;
      uint32_t pk[32];
      if (valid) {
        uint32_t s0[32], s1[32];
        tmem_ld32(scol, s0);
        tmem_ld_wait();
        tmem_ld32(scol + 32, s1);   // in flight while the first 32 columns are processed
        float mx[8];
        float rs[4] = {0.f, 0.f, 0.f, 0.f};
        // Speculative exponentials against the lazy max m: the tile max is formed
        // alongside them and only a rise of more than 2^8 (or no max yet) sends
        // the warp through the slow path below.
        const bool spec = __all_sync(0xffffffffu, m > -INFINITY);
        const float mneg = spec ? -m : 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) mx[i] = __uint_as_float(s0[i]);
#pragma unroll
        for (int i = 8; i < 32; ++i) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(s0[i]));
        if (spec) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(s0[2 * i]), sl2, mneg));
            const float p1 = fast_exp2(fmaf(__uint_as_float(s0[2 * i + 1]), sl2, mneg));
            rs[i & 3] += p0 + p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
        }
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(s1[i]));
        if (spec) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(s1[2 * i]), sl2, mneg));
            const float p1 = fast_exp2(fmaf(__uint_as_float(s1[2 * i + 1]), sl2, mneg));
            rs[i & 3] += p0 + p1;
            pk[16 + i] = pack_bf16x2(p0, p1);
          }
        }
        const float m_tile = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                   fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * sl2;
        const bool first = m == -INFINITY;
        const bool need = !first && (m_tile > m + kRescaleThreshold);   // rescale O_h, l
        const bool redo = first || need || !spec;                         // recompute p
        const float m_old = m;
        if (__any_sync(0xffffffffu, redo)) {
          if (first || need) m = m_tile;
          const float mn = -m;
          if (redo) {
            rs[0] = rs[1] = rs[2] = rs[3] = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float p0 = fast_exp2(fmaf(__uint_as_float(s0[2 * i]), sl2, mn));
              const float p1 = fast_exp2(fmaf(__uint_as_float(s0[2 * i + 1]), sl2, mn));
              const float p2 = fast_exp2(fmaf(__uint_as_float(s1[2 * i]), sl2, mn));
              const float p3 = fast_exp2(fmaf(__uint_as_float(s1[2 * i + 1]), sl2, mn));
              rs[i & 3] += (p0 + p1) + (p2 + p3);
              pk[i] = pack_bf16x2(p0, p1);
              pk[16 + i] = pack_bf16x2(p2, p3);
            }
          }
        }
        // P_t,h over the first 32 of this thread's S columns (S is already in registers)
        tmem_st32(scol, pk);
        // O_h must hold PV_{t-1},h before it is rescaled by 2^(m_old - m)
        bool rescale = __any_sync(0xffffffffu, need);
        if (rescale && t > 0 &&
            !warp_wait(bar(kBarOFull + 2 * half + ((t - 1) & 1)), ((t - 1) >> 1) & 1, lim,
                       abort_flag)) {
          ok = false;
          rescale = false;
        }
        if (rescale) {
          tc_fence_after();
          const float alpha = need ? fast_exp2(m_old - m) : 1.f;
          l *= alpha;
#pragma unroll
          for (int c = 0; c < D / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + o_col + c * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tmem + lane_off + o_col + c * 32, o);
          }
        }
        l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) pk[i] = 0u;
        tmem_st32(scol, pk);
      }
      tmem_st_wait();
      if (!ok) break;
      tc_fence_before();
      mbar_arrive(bar(kBarPFull + 2 * half + (t & 1)));
    }
    if (!ok) record_abort(abort_flag, prm.status, kStatusTimeout);
    // ------------------------------------------------------------ epilogue
    bool have_o = false;
    if (ok && n_t > 0) {
      have_o = warp_wait(bar(kBarOFull + 2 * half + ((n_t - 1) & 1)), ((n_t - 1) >> 1) & 1, lim,
                         abort_flag);
      tc_fence_after();
    }
    red[half * kBM + row] = m;
    red[2 * kBM + half * kBM + row] = l;
    // each half waited for its own last PV; after this barrier both O_0 and O_1 are final
    tc_fence_before();
    const bool all_ok = bar_red_and(kSoftmaxBarrier, kSoftmaxThreads, ok && (n_t == 0 || have_o));
    tc_fence_after();
    if (!all_ok) record_abort(abort_flag, prm.status, kStatusTimeout);
    const float m0 = red[row], m1 = red[kBM + row];
    const float l0 = red[2 * kBM + row], l1 = red[3 * kBM + row];
    const float M = fmaxf(m0, m1);
    const float f0 = l0 > 0.f ? fast_exp2(m0 - M) : 0.f;
    const float f1 = l1 > 0.f ? fast_exp2(m1 - M) : 0.f;
    const float lt = f0 * l0 + f1 * l1;
    const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
    const float g0 = f0 * inv_l, g1 = f1 * inv_l;
    const bool write = row_valid && all_ok;
    const int qrow = (qh ? r2 : r1) * 64 + (row & 63);
    const int64_t grow = static_cast<int64_t>(bh) * prm.S + qrow;
    // this thread writes d columns [half*D/2, half*D/2 + D/2) of its row
    __nv_bfloat16* orow = prm.o + grow * D + half * (D / 2);
    const bool read = all_ok && n_t > 0;
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      const uint32_t col = half * (D / 2) + c * 32;
      uint32_t a[32], b2[32];
      if (read) {
        tmem_ld32(tmem + lane_off + kColO0 + col, a);
        tmem_ld32(tmem + lane_off + kColO1 + col, b2);
        tmem_ld_wait();
      }
      if (write) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          // a stream with l == 0 contributed nothing (its O may never have been written)
          const float x0 = (g0 > 0.f ? __uint_as_float(a[2 * i]) * g0 : 0.f) +
                           (g1 > 0.f ? __uint_as_float(b2[2 * i]) * g1 : 0.f);
          const float x1 = (g0 > 0.f ? __uint_as_float(a[2 * i + 1]) * g0 : 0.f) +
                           (g1 > 0.f ? __uint_as_float(b2[2 * i + 1]) * g1 : 0.f);
          w[i] = pack_bf16x2(x0, x1);
        }
        uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = make_uint4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
    }
    if (write && half == 0 && prm.lse != nullptr)
      prm.lse[grow] = lt > 0.f ? (M + __log2f(lt)) * 0.69314718055994530942f : -INFINITY;
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------- self-test
// One 128 x 128 x 128 product through the same building blocks (see
// nabla_selftest_mma in the public header for the variants).
__global__ void __launch_bounds__(160, 1)
    mma_selftest_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __nv_bfloat16* __restrict__ a_glob, float* __restrict__ c,
                        int variant, int* status, uint64_t lim) {
  extern __shared__ uint8_t st_smem_raw[];
  const uint32_t raw = smem_addr(st_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = st_smem_raw + (base - raw);
  const uint32_t sA = base, sB = base + 32768, bars = base + 65536;
  uint32_t* holder = reinterpret_cast<uint32_t*>(gbase + 65536 + 64);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t bar_tma = bars, bar_mma = bars + 8, bar_a = bars + 16;
  if (tid == 0) {
    mbar_init(bar_tma, 1);
    mbar_init(bar_mma, 1);
    mbar_init(bar_a, 128);
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(smem_addr(holder), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(holder);
  bool ok = true;
  if (warp == 4 && lane == 0) {
    mbar_arrive_expect_tx(bar_tma, 65536);
    for (int rh = 0; rh < 2; ++rh)
      for (int h = 0; h < 2; ++h) {
        tma_load_2d(sA + h * 16384 + rh * 8192, &tmA, bar_tma, h * 64, rh * 64);
        tma_load_2d(sB + h * 16384 + rh * 8192, &tmB, bar_tma, h * 64, rh * 64);
      }
    ok = mbar_wait(bar_tma, 0, lim, nullptr);
    if (ok && variant == 3) ok = mbar_wait(bar_a, 0, lim, nullptr);
    tc_fence_after();
    if (ok) {
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t acc = kk > 0;
        const uint64_t ad = sdesc_sw128(sA + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
        if (variant == 0) {
          tc_mma_ss(tmem, ad, sdesc_sw128(sB + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                    idesc_bf16_f32(128, 128, false), acc);
        } else if (variant == 1) {
          tc_mma_ss(tmem, ad, sdesc_sw128(sB + kk * 2048, 16384, 1024),
                    idesc_bf16_f32(128, 128, true), acc);
        } else if (variant == 2) {
          for (int h = 0; h < 2; ++h)
            tc_mma_ss(tmem + h * 64, ad, sdesc_sw128(sB + h * 16384 + kk * 2048, 1024, 1024),
                      idesc_bf16_f32(128, 64, true), acc);
        } else {
          tc_mma_ts(tmem, tmem + 256 + kk * 8, sdesc_sw128(sB + kk * 2048, 16384, 1024),
                    idesc_bf16_f32(128, 128, true), acc);
        }
      }
      tc_commit(bar_mma);
    } else {
      atomicOr(status, kStatusTimeout);
    }
  }
  if (warp < 4) {
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    if (variant == 3) {   // A row `tid` into tensor memory as packed bf16 pairs
      const uint32_t* arow = reinterpret_cast<const uint32_t*>(a_glob + tid * 128);
      for (int h = 0; h < 2; ++h) {
        uint32_t r[32];
        for (int i = 0; i < 32; ++i) r[i] = arow[h * 32 + i];
        tmem_st32(tmem + lane_off + 256 + h * 32, r);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar_a);
    }
    const bool done = warp_wait(bar_mma, 0, lim, nullptr);
    tc_fence_after();
    if (done) {
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + cc * 32, r);
        tmem_ld_wait();
        for (int i = 0; i < 32; ++i) c[tid * 128 + cc * 32 + i] = __uint_as_float(r[i]);
      }
    } else {
      atomicOr(status, kStatusTimeout);
    }
  }
  if (warp == 4 && lane == 0 && ok) mbar_wait(bar_mma, 0, kDrainLimitNs, nullptr);
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- launchers

template <int D>
static cudaError_t launch_fwd_t(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                                const AttnParams& prm, int64_t nitems, cudaStream_t st) {
  constexpr uint32_t smem = AttnSmem<D>::kAlloc;
  cudaError_t e = cudaFuncSetAttribute(bsa_fwd_kernel<D>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  bsa_fwd_kernel<D><<<static_cast<unsigned>(nitems), kThreads, smem, st>>>(q, k, v, prm);
  return cudaGetLastError();
}

cudaError_t launch_bsa_fwd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                           const int32_t* row_ptr, const int32_t* col_idx, void* o, float* lse,
                           int* status, int BH, int H, int S, int d, float scale,
                           uint64_t wait_limit_ns, cudaStream_t st) {
  AttnParams prm;
  prm.row_ptr = row_ptr;
  prm.col_idx = col_idx;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.status = status;
  prm.H = H;
  prm.S = S;
  prm.nb = S / 64;
  prm.npairs = (prm.nb + 1) / 2;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.wait_limit_ns = wait_limit_ns;
  const int64_t nitems = static_cast<int64_t>(BH) * prm.npairs;
  if (nitems == 0) return cudaSuccess;
  if (d == 128) return launch_fwd_t<128>(q, k, v, prm, nitems, st);
  return launch_fwd_t<64>(q, k, v, prm, nitems, st);
}

cudaError_t launch_mma_selftest(const CUtensorMap& a, const CUtensorMap& b, const void* a_glob,
                                float* c, int variant, int* status, uint64_t lim,
                                cudaStream_t st) {
  const uint32_t smem = 65536 + 1024 + 1024;
  cudaError_t e = cudaFuncSetAttribute(mma_selftest_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  mma_selftest_kernel<<<1, 160, smem, st>>>(a, b, static_cast<const __nv_bfloat16*>(a_glob), c,
                                            variant, status, lim);
  return cudaGetLastError();
}

}  // namespace nabla
