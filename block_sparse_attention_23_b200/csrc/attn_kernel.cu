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
//   One CTA per (b, h, group of four query blocks 4g..4g+3) = two query
//   tiles of 128 rows: tile 0 = blocks 4g, 4g+1; tile 1 = blocks 4g+2, 4g+3.
//   The key blocks visited are the union of the four CSR rows, each entry with
//   a 4-bit membership mask.  Key tiles are 128 keys = two union entries (the
//   second may be a repeat that every row masks); each entry is one contiguous
//   64 x d slab of the [B,H,S,d] tensor, loaded as a plain 2D TMA box, so both
//   query tiles share every K/V tile that is loaded.  A query tile computes a
//   key tile only if one of its two blocks lists one of the tile's entries; a
//   row whose block did not list an entry gives it probability 0 (no
//   exponentials evaluated).
//
// Roles (384 threads)
//   warps 0-3   softmax of query tile 0, warps 4-7 of query tile 1: thread i of
//               the group owns row i (= tensor-memory lane i) for all 128 keys
//               of a tile: tcgen05.ld of S, lazy running max, exp2, P (bf16)
//               written over the first 64 S columns, O rescale, epilogue.
//   warp 8      TMA producer of Q and K (and the union-list compaction).
//   warp 9      tensor-memory allocation and the single MMA-issuing thread.
//   warp 10     TMA producer of V; warp 11 idles (completes warpgroup 2).
//
// MMA order (ping-pong between the two query tiles)
//   S_0(0), S_1(0), then for every key tile t: PV_0(t), S_0(t+1), PV_1(t),
//   S_1(t+1).  While softmax 0 works on S_0(t) the tensor cores run PV_1(t-1)
//   and S_1(t), and the other way round, so each softmax group has about two
//   MMA tile-products of time.  S_x(t+1) overwrites the S/P buffer of tile x
//   only after PV_x(t), which read P_x(t), was issued by the same thread (MMAs
//   of one thread execute in issue order).
//
// Token order: tile-major tensors are read as 2D boxes; raster-ordered ones
// (token (t,h,w) at (t*H + h)*W + w) as 5D boxes that gather one 4x4x4 tile,
// so the reorder to tile-major happens inside the TMA loads, and O / LSE rows
// are stored back at their raster positions.
//
// Online softmax with a lazy maximum: the running max m of a row is raised
// (and O, l rescaled by 2^(m_old - m_new)) only when a tile's max exceeds it by
// more than 2^8; otherwise p <= 256 and O / l, LSE = ln2 (m + log2 l) are
// unchanged in exact arithmetic.  The tile max is formed from the S row in
// registers, then the exponentials; a tile whose two key blocks the row both
// lists (the common case) runs that as one straight-line block without
// per-chunk branches, which lets the compiler interleave the whole row.
//
// Tensor memory (512 columns): tile 0 S/P [0,128), O [128,256);
// tile 1 S/P [256,384), O [384,512).
//
// Every mbarrier wait is time-bounded; a wait that runs out records
// kStatusTimeout, raises a CTA-wide abort flag, and the CTA drains its own TMA
// loads and MMAs (bounded again) before freeing tensor memory and returning.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_primitives.cuh"

namespace nabla {

constexpr int kBM = 128;        // rows per query tile (two 64-token blocks)
constexpr int kQTiles = 2;      // query tiles per CTA
constexpr int kBN = 128;        // keys per tile (two 64-token blocks)
constexpr int kKStages = 2;     // K ring depth
constexpr int kVStages = 2;     // V ring depth
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = kSoftmaxThreads + 128;   // warpgroups 0, 1 softmax; 2 load/MMA
constexpr int kProducerWarp = 8, kMmaWarp = 9, kVProducerWarp = 10;   // warp 11 idles
// Register budgets after set-up: a softmax thread holds a whole S row (128
// values); the load/MMA warpgroup needs few.  8*216 + 4*72 = 12*168, the
// launch allocation (checked on the host before launch).
constexpr int kRegsSoftmax = 216, kRegsOther = 72, kRegsLaunch = 168;
constexpr int kMaxNb = 4096;    // blocks per head supported
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleThreshold = 8.0f;            // log2 units
constexpr uint64_t kDrainLimitNs = 1000000000ull;   // 1 s for draining in-flight work

__host__ __device__ constexpr uint32_t col_s(int x) { return x ? 256u : 0u; }
__host__ __device__ constexpr uint32_t col_o(int x) { return x ? 384u : 128u; }

template <int D>
struct AttnSmem {
  static constexpr int kDH = D / 64;                       // 64-column halves of d
  static constexpr uint32_t kQBytes = kBM * D * 2;         // one query tile
  static constexpr uint32_t kKVBytes = kBN * D * 2;        // one K or V stage
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + kQTiles * kQBytes;
  static constexpr uint32_t kOffV = kOffK + kKStages * kKVBytes;
  static constexpr uint32_t kOffBar = kOffV + kVStages * kKVBytes;  // 32 mbarriers
  static constexpr uint32_t kOffMisc = kOffBar + 256;      // tmem base, abort, n_u
  static constexpr uint32_t kOffBitmap = kOffMisc + 64;    // 4 x kMaxNb/32 words
  static constexpr uint32_t kOffList = kOffBitmap + 4 * (kMaxNb / 32) * 4;
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
  kBarSFull = kBarVEmpty + kVStages,  // + query tile: S ready
  kBarPFull = kBarSFull + kQTiles,    // + query tile: P written
  kBarOFull = kBarPFull + kQTiles,    // + query tile: PV done
  kBarDrain = kBarOFull + kQTiles,
  kNumBars = kBarDrain + 1
};

struct AttnParams {
  const int32_t* row_ptr;
  const int32_t* col_idx;
  __nv_bfloat16* o;
  float* lse;
  int* status;
  int H, S, nb, ngroups;
  int Th, Tw;              // tile grid (raster token order only)
  float scale_log2;        // softmax scale * log2(e)
  uint64_t wait_limit_ns;
};

// One 64-token block of a [B,H,S,d] tensor as a 64 x 64 shared-memory box
// (columns [64h, 64h+64) of d).  Tile-major order: rows 64*blk.. of head bh,
// a 2D box.  Raster order: the block is tile blk of the 4Tt x 4Th x 4Tw token
// grid, read by one 5D box (d, w, h, t, bh) of 64 x 4 x 4 x 4 x 1, which lands
// its tokens in the same (t, h, w)-major row order.
template <bool kRaster>
__device__ __forceinline__ void load_block(uint32_t dst, const CUtensorMap* map, uint32_t bar,
                                           int h, int bh, int blk, int64_t S, int Th, int Tw) {
  if (kRaster) {
    const int tw = blk % Tw, th = (blk / Tw) % Th, tt = blk / (Tw * Th);
    tma_load_5d(dst, map, bar, h * 64, 4 * tw, 4 * th, 4 * tt, bh);
  } else {
    tma_load_2d(dst, map, bar, h * 64, static_cast<int32_t>(static_cast<int64_t>(bh) * S + static_cast<int64_t>(blk) * 64));
  }
}

// Position along S of row u of block blk.
template <bool kRaster>
__device__ __forceinline__ int64_t token_of(int blk, int u, int Th, int Tw) {
  if (!kRaster) return static_cast<int64_t>(blk) * 64 + u;
  const int tw = blk % Tw, th = (blk / Tw) % Th, tt = blk / (Tw * Th);
  const int64_t H = 4ll * Th, W = 4ll * Tw;
  return ((4ll * tt + (u >> 4)) * H + 4ll * th + ((u >> 2) & 3)) * W + 4ll * tw + (u & 3);
}

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

// Membership mask of query tile x (bits of its two blocks) in union entry e.
__device__ __forceinline__ int tile_bits(int e, int x) { return (e >> (16 + 2 * x)) & 3; }

template <int D, bool kRaster>
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
  uint32_t* bm = reinterpret_cast<uint32_t*>(gbase + L::kOffBitmap);   // [4][kMaxNb/32]
  int32_t* ulist = reinterpret_cast<int32_t*>(gbase + L::kOffList);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item = blockIdx.x;
  const int bh = item / prm.ngroups;
  const int grp = item % prm.ngroups;
  const int nb = prm.nb;
  const int r0 = 4 * grp;                       // first query block of the group
  const int nq = min(4, nb - r0);               // query blocks present (1..4)
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
    for (int x = 0; x < kQTiles; ++x) {
      mbar_init(bar(kBarSFull + x), 1);
      mbar_init(bar(kBarPFull + x), kSoftmaxThreads / kQTiles);
      mbar_init(bar(kBarOFull + x), 1);
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
  for (int i = tid; i < 4 * (kMaxNb / 32); i += kThreads) bm[i] = 0u;
  __syncthreads();
  for (int qb = 0; qb < nq; ++qb) {
    const int64_t g = static_cast<int64_t>(bh) * nb + r0 + qb;
    const int b = prm.row_ptr[g], e = prm.row_ptr[g + 1];
    uint32_t* bmq = bm + qb * (kMaxNb / 32);
    for (int i = b + tid; i < e; i += kThreads) {
      const int c = prm.col_idx[i];
      if (static_cast<unsigned>(c) < static_cast<unsigned>(nb)) atomicOr(&bmq[c >> 5], 1u << (c & 31));
      else atomicOr(prm.status, kStatusBadIndex);
    }
  }
  __syncthreads();
  if (warp == kProducerWarp) {   // compact the union in ascending block order
    int run = 0;
    for (int w0 = 0; w0 < nw; w0 += 32) {
      const int w = w0 + lane;
      uint32_t u[4];
#pragma unroll
      for (int qb = 0; qb < 4; ++qb) u[qb] = w < nw ? bm[qb * (kMaxNb / 32) + w] : 0u;
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
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const int n_u = *n_union_s;
  const int n_t = (n_u + 1) >> 1;
  const uint64_t lim = prm.wait_limit_ns;
  // membership of key tile t: OR of its two entries
  auto tile_entry = [&](int t, int i) { return (2 * t + i < n_u) ? ulist[2 * t + i] : 0; };
  auto tile_active = [&](int t, int x) {
    return tile_bits(tile_entry(t, 0) | tile_entry(t, 1), x) != 0;
  };

  if (warp >= 8) {
  setmaxnreg_dec<kRegsOther>();
  if (warp == kProducerWarp || warp == kVProducerWarp) {
    // ------------------------------------------------------------ TMA producers
    // warp 8 streams Q and K, warp 10 streams V: a V slot frees only after the
    // softmax of its tile, and must not hold back the K prefetch
    if (lane == 0 && n_t > 0) {
      const bool is_k = warp == kProducerWarp;
      const int nst = is_k ? kKStages : kVStages;
      const uint32_t ring = is_k ? sK : sV;
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      const int full0 = is_k ? kBarKFull : kBarVFull, empty0 = is_k ? kBarKEmpty : kBarVEmpty;
      int armed0 = 0, armed1 = 0;
      if (is_k) {
        mbar_arrive_expect_tx(bar(kBarQFull), kQTiles * L::kQBytes);
        for (int qb = 0; qb < 4; ++qb)   // blocks past the end repeat the last (rows unused)
          for (int h = 0; h < L::kDH; ++h)
            load_block<kRaster>(sQ + (qb >> 1) * L::kQBytes + h * kBM * 128 + (qb & 1) * 64 * 128,
                                &tmQ, bar(kBarQFull), h, bh, min(r0 + qb, nb - 1), prm.S, prm.Th,
                                prm.Tw);
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
        (s ? armed1 : armed0) += 1;
        for (int kb = 0; kb < 2; ++kb)
          for (int h = 0; h < L::kDH; ++h)
            load_block<kRaster>(ring + s * L::kKVBytes + h * kBN * 128 + kb * 64 * 128, map,
                                bar(full0 + s), h, bh, kb ? j1 : j0, prm.S, prm.Th, prm.Tw);
      }
      // drain: every armed phase must complete before shared memory is released
      if (is_k) mbar_wait(bar(kBarQFull), 0, kDrainLimitNs, nullptr);
      if (armed0) mbar_wait(bar(full0 + 0), (armed0 - 1) & 1, kDrainLimitNs, nullptr);
      if (armed1) mbar_wait(bar(full0 + 1), (armed1 - 1) & 1, kDrainLimitNs, nullptr);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_t > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, true);
      int n_pv[kQTiles] = {0, 0};   // PV products issued per query tile
      bool ok = mbar_wait(bar(kBarQFull), 0, lim, abort_flag);
      tc_fence_after();
      auto issue_s = [&](int x, int t) {
        const uint32_t kt = sK + (t % kKStages) * L::kKVBytes;
        const uint32_t qt = sQ + x * L::kQBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * (kBM * 128) + (kk & 3) * 32;
          const uint32_t offk = (kk >> 2) * (kBN * 128) + (kk & 3) * 32;
          tc_mma_ss(tmem + col_s(x), sdesc_sw128(qt + off, 16, 1024),
                    sdesc_sw128(kt + offk, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(kBarSFull + x));
      };
      auto issue_pv = [&](int x, int t) -> bool {
        if (!mbar_wait(bar(kBarPFull + x), n_pv[x] & 1, lim, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vt = sV + (t % kVStages) * L::kKVBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          // 16 keys per step: P columns [8kk, 8kk+8) of the S/P buffer, V rows
          // [16kk, 16kk+16); the 64-column halves of d are kBN*128 bytes apart
          tc_mma_ts(tmem + col_o(x), tmem + col_s(x) + kk * 8,
                    sdesc_sw128(vt + kk * 16 * 128, kBN * 128, 1024), idesc_pv,
                    (n_pv[x] > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(kBarOFull + x));
        ++n_pv[x];
        return true;
      };
      if (ok) ok = mbar_wait(bar(kBarKFull + 0), 0, lim, abort_flag);
      if (ok) {
        tc_fence_after();
        for (int x = 0; x < kQTiles; ++x)
          if (tile_active(0, x)) issue_s(x, 0);
        tc_commit(bar(kBarKEmpty + 0));
      }
      for (int t = 0; ok && t < n_t; ++t) {
        const bool more = t + 1 < n_t;
        if (!mbar_wait(bar(kBarVFull + t % kVStages), (t / kVStages) & 1, lim, abort_flag)) { ok = false; break; }
        if (more && !mbar_wait(bar(kBarKFull + (t + 1) % kKStages), ((t + 1) / kKStages) & 1, lim,
                               abort_flag)) { ok = false; break; }
        tc_fence_after();
        for (int x = 0; x < kQTiles; ++x) {
          if (tile_active(t, x) && !issue_pv(x, t)) { ok = false; break; }
          if (more && tile_active(t + 1, x)) issue_s(x, t + 1);
        }
        if (!ok) break;
        if (more) tc_commit(bar(kBarKEmpty + (t + 1) % kKStages));
        tc_commit(bar(kBarVEmpty + t % kVStages));
      }
      if (!ok) record_abort(abort_flag, prm.status, kStatusTimeout);
      // drain: all MMAs this thread issued must finish before tensor memory is freed
      tc_commit(bar(kBarDrain));
      mbar_wait(bar(kBarDrain), 0, kDrainLimitNs, nullptr);
    }
  }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax (warps 0-7)
    const int x = warp >> 2;                   // query tile of this warp group
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;       // row of the tile == tensor-memory lane
    const int qh = row >> 6;                   // block 4g + 2x + qh
    const int qblock = r0 + 2 * x + qh;
    const bool row_valid = qblock < nb;
    const int bit = 1 << (16 + 2 * x + qh);
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_base = tmem + lane_off + col_s(x);
    const uint32_t o_base = tmem + lane_off + col_o(x);
    const float sl2 = prm.scale_log2;
    float m = -INFINITY;        // lazy running max of the row, log2 units
    float l = 0.f;              // running sum of the row
    int c = 0;                  // key tiles this query tile has processed
    bool ok = true;
    for (int t = 0; t < n_t; ++t) {
      if (!tile_active(t, x)) continue;        // same decision as the MMA issuer
      const bool v0 = (tile_entry(t, 0) & bit) != 0;   // uniform per warp
      const bool v1 = (tile_entry(t, 1) & bit) != 0;
      if (!warp_wait(bar(kBarSFull + x), c & 1, lim, abort_flag)) { ok = false; break; }
      tc_fence_after();
      // the whole S row in one batch of loads (one load latency per tile)
      uint32_t sv[4][32];
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
      if (v0 && v1) {   // both entries listed: loads and max without per-chunk branches
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) tmem_ld32(s_base + 32 * ch, sv[ch]);
        tmem_ld_wait();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch)
#pragma unroll
          for (int i = 0; i < 32; ++i) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(sv[ch][i]));
      } else {
        if (v0) { tmem_ld32(s_base, sv[0]); tmem_ld32(s_base + 32, sv[1]); }
        if (v1) { tmem_ld32(s_base + 64, sv[2]); tmem_ld32(s_base + 96, sv[3]); }
        tmem_ld_wait();
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          if ((ch < 2) ? v0 : v1) {
#pragma unroll
            for (int i = 0; i < 32; ++i) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(sv[ch][i]));
          }
        }
      }
      const float m_tile = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                 fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) * sl2;
      const bool has = m_tile > -INFINITY;
      const bool first = m == -INFINITY;
      const bool need = has && !first && (m_tile > m + kRescaleThreshold);   // rescale O, l
      const float m_old = m;
      if (has && (first || need)) m = m_tile;
      // O must hold the previous PV of this tile before it is rescaled by 2^(m_old - m)
      bool rescale = __any_sync(0xffffffffu, need);
      if (rescale && c > 0 && !warp_wait(bar(kBarOFull + x), (c - 1) & 1, lim, abort_flag)) {
        ok = false;
        rescale = false;
      }
      if (rescale) {
        tc_fence_after();
        const float alpha = need ? fast_exp2(m_old - m) : 1.f;
        l *= alpha;
#pragma unroll 1
        for (int cc = 0; cc < D / 16; ++cc) {
          uint32_t o[16];
          tmem_ld16(o_base + cc * 16, o);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st16(o_base + cc * 16, o);
          tmem_st_wait();
        }
      }
      // p = 2^(s*scale*log2e - m); P chunk ch (keys [32ch, 32ch+32)) goes to
      // columns [16ch, 16ch+16), whose S values are already in registers
      const bool live = m > -INFINITY;
      const float mneg = live ? -m : 0.f;
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
      if (v0 && v1 && __all_sync(0xffffffffu, live)) {
        // common case, one straight-line block: every column of the row is listed
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(sv[ch][2 * i]), sl2, mneg));
            const float p1 = fast_exp2(fmaf(__uint_as_float(sv[ch][2 * i + 1]), sl2, mneg));
            rs[i & 3] += p0 + p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
          tmem_st16(s_base + ch * 16, pk);
        }
      } else
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t pk[16];
        if (((ch < 2) ? v0 : v1) && live) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(sv[ch][2 * i]), sl2, mneg));
            const float p1 = fast_exp2(fmaf(__uint_as_float(sv[ch][2 * i + 1]), sl2, mneg));
            rs[i & 3] += p0 + p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = 0u;
        }
        tmem_st16(s_base + ch * 16, pk);
      }
      l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
      tmem_st_wait();
      if (!ok) break;
      tc_fence_before();
      mbar_arrive(bar(kBarPFull + x));
      ++c;
    }
    if (!ok) record_abort(abort_flag, prm.status, kStatusTimeout);
    // ------------------------------------------------------------ epilogue
    bool have_o = false;
    if (ok && c > 0) {
      have_o = warp_wait(bar(kBarOFull + x), (c - 1) & 1, lim, abort_flag);
      if (!have_o) record_abort(abort_flag, prm.status, kStatusTimeout);
      tc_fence_after();
    }
    const bool write = row_valid && ok && (c == 0 || have_o);
    const int64_t grow = static_cast<int64_t>(bh) * prm.S +
                         (row_valid ? token_of<kRaster>(qblock, row & 63, prm.Th, prm.Tw) : 0);
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    __nv_bfloat16* orow = prm.o + grow * D;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
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
    if (write && prm.lse != nullptr)
      prm.lse[grow] = l > 0.f ? (m + __log2f(l)) * 0.69314718055994530942f : -INFINITY;
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

template <int D, bool kRaster>
static cudaError_t launch_fwd_t(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                                const AttnParams& prm, int64_t nitems, cudaStream_t st) {
  constexpr uint32_t smem = AttnSmem<D>::kAlloc;
  static_assert(8 * kRegsSoftmax + 4 * kRegsOther <= 12 * kRegsLaunch, "register split");
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, bsa_fwd_kernel<D, kRaster>);
  if (e != cudaSuccess) return e;
  // the in-kernel register split assumes the launch allocation of kRegsLaunch
  // registers per thread; anything less would make setmaxnreg.inc wait forever
  if (attr.numRegs < kRegsLaunch) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(bsa_fwd_kernel<D, kRaster>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem);
  if (e != cudaSuccess) return e;
  bsa_fwd_kernel<D, kRaster><<<static_cast<unsigned>(nitems), kThreads, smem, st>>>(q, k, v, prm);
  return cudaGetLastError();
}

cudaError_t launch_bsa_fwd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                           const int32_t* row_ptr, const int32_t* col_idx, void* o, float* lse,
                           int* status, int BH, int H, int S, int d, float scale, int raster,
                           int Th, int Tw, uint64_t wait_limit_ns, cudaStream_t st) {
  AttnParams prm;
  prm.row_ptr = row_ptr;
  prm.col_idx = col_idx;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.status = status;
  prm.H = H;
  prm.S = S;
  prm.nb = S / 64;
  prm.ngroups = (prm.nb + 3) / 4;
  prm.Th = Th;
  prm.Tw = Tw;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.wait_limit_ns = wait_limit_ns;
  const int64_t nitems = static_cast<int64_t>(BH) * prm.ngroups;
  if (nitems == 0) return cudaSuccess;
  if (raster) {
    if (d == 128) return launch_fwd_t<128, true>(q, k, v, prm, nitems, st);
    return launch_fwd_t<64, true>(q, k, v, prm, nitems, st);
  }
  if (d == 128) return launch_fwd_t<128, false>(q, k, v, prm, nitems, st);
  return launch_fwd_t<64, false>(q, k, v, prm, nitems, st);
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
