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
//   One CTA per (b, h, pair of query blocks 2g, 2g+1) = one query tile of 128
//   rows.  The key blocks visited are the union of the two CSR rows, each entry
//   with a 2-bit membership mask, taken four at a time: a key tile is 256 keys
//   (the last one repeats its final entry, masked for every row).  Each entry
//   is one contiguous 64 x d slab of the [B,H,S,d] tensor, loaded as a plain 2D
//   TMA box.  A row whose block did not list an entry gives it probability 0
//   (no exponentials evaluated).  Query tile g of a head starts at key tile
//   floor(g * n_t / groups) of its n_t and wraps around, so that neighbouring
//   CTAs in flight spread their K/V requests over the head.
//
// Roles (384 threads)
//   warps 0-7   softmax: warp w owns tensor-memory lane quarter q = w % 4 (rows
//               32q..32q+31 of the tile) and column half c = w / 4 (keys
//               [128c, 128c+128) of each key tile, its entries 2c and 2c+1).
//               The two warps of a lane quarter trade partial row maxima
//               when they agree on a reference (and, at the end, partial row
//               sums) through shared memory, meeting on an mbarrier with a
//               bounded wait.
//   warp 8      TMA producer of Q and K (and the union-list compaction).
//   warp 9      tensor-memory allocation and the single MMA-issuing thread.
//   warp 10     TMA producer of V; warp 11 idles (completes warpgroup 2).
//
// Tensor memory (512 columns): S [0,256) fp32, P [256,384) (bf16 pairs), O
// [384, 384+d).  P has its own columns, so the tensor cores do not wait for a
// softmax to finish before computing the next S:
//   S(0); then for every key tile t: S(t+1) as soon as the softmax has copied
//   S(t) to registers (and K(t+1) is in), PV(t) once P(t) is written.
// While the softmax works on tile t the tensor cores run S(t+1) and PV(t-1);
// the softmax stores P(t) only after PV(t-1), which read P(t-1), completed,
// and keeps P(t) in registers until then.  S at N = 256 runs at the full
// tensor rate (an N = 128 product with both operands in shared memory does
// not), and the per-tile softmax overhead is spread over 256 keys.  On a tile
// with a fixed reference and both of its entries listed, a softmax warp loads
// its first 32 columns, then the other 96 while it exponentiates the first,
// and releases S(t) once those are in.
//
// Token order: tile-major tensors are read as 2D boxes; a raster-ordered Q
// (token (t,h,w) at (t*H + h)*W + w) as 5D boxes that gather one 4x4x4 tile,
// so its reorder to tile-major happens inside the TMA loads, and O / LSE rows
// are stored back at their raster positions.  Raster K and V, streamed once
// per query tile, are read from tile-major copies when the caller's
// workspace holds them (made by the token reorder before the launch), else
// by 5D boxes as well (kv_raster).
//
// Online softmax with a reference maximum per row, in up to two passes over
// the CTA's query tile.  The fixed-reference pass: the two warps of a lane
// quarter agree on the row max of the first key tile the row's block lists,
// and that reference m stays for the rest of the row (no further max or
// exchange per tile; p = 2^(s*scale*log2e - m) may exceed 1).  A warp whose
// partial row sum of a tile (128 columns) exceeds 2^16 sets a flag in shared
// memory, and the CTA then runs the exact-reference pass over the same tile
// (the union list and Q stay in place, the barriers start afresh): there the
// warps agree on every tile's max and raise m (with O and l rescaled by
// 2^(m_old - m_new)) whenever it grows by more than 2^8, so p <= 256.  The
// first CTA of a call that needs the second pass sets a word in the caller's
// workspace and counts the call.  O / l and LSE = ln2 (m + log2 l) do not
// depend on the reference in exact arithmetic.
// A warp whose two entries the row both lists (the common case) runs its
// loads and exponentials as straight-line code without per-chunk branches.
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
constexpr int kBN = 256;        // keys per tile (four 64-token blocks)
constexpr int kEntries = 4;     // union entries per key tile
constexpr int kSoftmaxThreads = 256;
constexpr int kThreads = kSoftmaxThreads + 128;   // warpgroups 0, 1 softmax; 2 load/MMA
constexpr int kProducerWarp = 8, kMmaWarp = 9, kVProducerWarp = 10;   // warp 11 idles
// Register budgets after set-up: a softmax thread holds 128 S values of its
// row and the packed P; the load/MMA warpgroup needs few.  8*216 + 4*72 =
// 12*168, the launch allocation (checked on the host before launch).
constexpr int kRegsSoftmax = 216, kRegsOther = 72, kRegsLaunch = 168;
constexpr int kMaxNb = 4096;    // blocks per head supported
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColP = 256, kColO = 384;
constexpr float kRescaleThreshold = 8.0f;            // log2 units
// Largest partial row sum (one warp's 128 columns of a key tile, relative to
// the row's fixed reference) the fixed-reference pass accepts: every p stays
// below 2^16, so O and l keep the fp32 range the exact pass has for them.
constexpr float kFixedRefSumLimit = 65536.0f;
constexpr uint64_t kDrainLimitNs = 1000000000ull;   // 1 s for draining in-flight work

template <int D>
struct AttnSmem {
  static constexpr int kDH = D / 64;                       // 64-column halves of d
  static constexpr uint32_t kQBytes = kBM * D * 2;         // the query tile
  static constexpr uint32_t kKVBytes = kBN * D * 2;        // one K or V tile
  static constexpr uint32_t kOffQ = 0;
  static constexpr uint32_t kOffK = kOffQ + kQBytes;
  static constexpr uint32_t kOffV = kOffK + kKVBytes;
  static constexpr uint32_t kOffBar = kOffV + kKVBytes;    // 16 mbarriers
  static constexpr uint32_t kOffMisc = kOffBar + 128;      // tmem base, abort, n_u
  static constexpr uint32_t kOffXch = kOffMisc + 64;       // [2 parities][2 halves][128 rows] fp32
  static constexpr uint32_t kOffBitmap = kOffXch + 2 * 2 * kBM * 4;   // 2 x kMaxNb/32 words
  static constexpr uint32_t kOffList = kOffBitmap + 2 * (kMaxNb / 32) * 4;
  static constexpr uint32_t kBytes = kOffList + kMaxNb * 4;
  static constexpr uint32_t kAlloc = kBytes + 1024;        // slack for 1024-byte alignment
};

// Barrier slots inside the barrier area.
enum : int {
  kBarQFull = 0,
  kBarKFull,     // K(t) landed
  kBarKEmpty,    // S(t) done: the K buffer is free
  kBarVFull,     // V(t) landed
  kBarVEmpty,    // PV(t) done: the V buffer is free
  kBarSFull,     // S(t) in tensor memory
  kBarSFree,     // every softmax thread copied S(t) to registers
  kBarPFull,     // every softmax thread wrote P(t) (and rescaled its O half)
  kBarOFull,     // PV(t) done
  kBarDrain,
  kBarPair,      // + lane quarter: the two warps of a quarter met (4 slots)
  kNumBars = kBarPair + 4
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
  int* redo;               // set when a tile of the call needed the exact-reference pass
  int* exact_passes;       // counts the forwards that needed it
  int exact;               // 0: fixed reference, exact pass per tile when needed;
                           // 1: exact pass alone; 2: exact pass alone if *redo is set
  int kv_raster;           // raster token order: K and V read by 5D boxes too (else 2D)
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
  volatile int* cta_redo = reinterpret_cast<volatile int*>(misc + 3);   // a row outgrew the reference
  volatile int* pass_s = reinterpret_cast<volatile int*>(misc + 4);     // 0 fixed, 1 exact reference
  float* xch = reinterpret_cast<float*>(gbase + L::kOffXch);           // [2][2][kBM]
  uint32_t* bm = reinterpret_cast<uint32_t*>(gbase + L::kOffBitmap);   // [2][kMaxNb/32]
  int32_t* ulist = reinterpret_cast<int32_t*>(gbase + L::kOffList);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int item = blockIdx.x;
  // exact 2: an exact-reference launch after another kernel's fixed-reference
  // pass, which runs only if that pass asked for it
  if (prm.exact == 2 && *prm.redo == 0) return;
  if (prm.exact != 0 && item == 0 && tid == 0) atomicAdd(prm.exact_passes, 1);

  const int bh = item / prm.ngroups;
  const int grp = item % prm.ngroups;
  const int nb = prm.nb;
  const int r0 = 2 * grp;                       // first query block of the tile
  const int nq = min(2, nb - r0);               // query blocks present (1 or 2)
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  auto init_bars = [&]() {
    mbar_init(bar(kBarQFull), 1);
    mbar_init(bar(kBarKFull), 1);
    mbar_init(bar(kBarKEmpty), 1);
    mbar_init(bar(kBarVFull), 1);
    mbar_init(bar(kBarVEmpty), 1);
    mbar_init(bar(kBarSFull), 1);
    mbar_init(bar(kBarSFree), kSoftmaxThreads);
    mbar_init(bar(kBarPFull), kSoftmaxThreads);
    mbar_init(bar(kBarOFull), 1);
    mbar_init(bar(kBarDrain), 1);
    for (int q = 0; q < 4; ++q) mbar_init(bar(kBarPair + q), 64);
    fence_barrier_init();
  };

  // ---------------------------------------------------------------- setup
  if (tid == 0) {
    init_bars();
    *abort_flag = 0;
    *cta_redo = 0;
    *pass_s = prm.exact != 0 ? 1 : 0;
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
  for (int i = tid; i < 2 * (kMaxNb / 32); i += kThreads) bm[i] = 0u;
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
      const uint32_t u0 = w < nw ? bm[w] : 0u;
      const uint32_t u1 = w < nw ? bm[(kMaxNb / 32) + w] : 0u;
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
  const int n_t = (n_u + kEntries - 1) / kEntries;
  const uint64_t lim = prm.wait_limit_ns;
  // The key tiles are visited from a start that moves with the query tile's
  // place in the head (tile t is union tile (t + t_off) mod n_t), so the CTAs
  // in flight, neighbours in the head, do not all request the same K/V blocks
  // at the same moment; the online softmax does not depend on the order.
  const int t_off =
      n_t > 0 ? static_cast<int>((static_cast<int64_t>(grp) * n_t) / prm.ngroups) : 0;
  auto tile_of = [&](int t) {
    const int u = t + t_off;
    return u >= n_t ? u - n_t : u;
  };
  // entry e of key tile t (0 past the end of the union: no row lists it)
  auto tile_entry = [&](int t, int e) {
    const int u = tile_of(t);
    return (kEntries * u + e < n_u) ? ulist[kEntries * u + e] : 0;
  };

  // After a pass every thread meets here.  A second, exact-reference pass over
  // the same tile follows when a row of the tile outgrew its fixed reference
  // (the union list and Q stay in place; barriers start afresh).
  auto next_pass = [&]() {
    tc_fence_before();
    __syncthreads();
    const bool again = *pass_s == 0 && *cta_redo != 0 && *abort_flag == 0;
    if (again) {
      if (tid == 0) {
        init_bars();
        *pass_s = 1;
        // count the forward once, at its first recomputed tile
        if (atomicExch(prm.redo, 1) == 0) atomicAdd(prm.exact_passes, 1);
      }
      __syncthreads();
    }
    tc_fence_after();
    return again;
  };

  if (warp >= 8) {
  setmaxnreg_dec<kRegsOther>();
  while (true) {
  if (warp == kProducerWarp || warp == kVProducerWarp) {
    // ------------------------------------------------------------ TMA producers
    // warp 8 streams Q and K, warp 10 streams V (one buffer each: K(t+1) may
    // land once S(t) is done, V(t+1) once PV(t) is done)
    if (lane == 0 && n_t > 0) {
      const bool is_k = warp == kProducerWarp;
      const uint32_t buf = is_k ? sK : sV;
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      const int full = is_k ? kBarKFull : kBarVFull, empty = is_k ? kBarKEmpty : kBarVEmpty;
      int armed = 0;
      if (is_k && !(*cta_redo)) {   // the first pass of this tile loads Q
        mbar_arrive_expect_tx(bar(kBarQFull), L::kQBytes);
        for (int qb = 0; qb < 2; ++qb)   // a block past the end repeats the last (rows unused)
          for (int h = 0; h < L::kDH; ++h)
            load_block<kRaster>(sQ + h * kBM * 128 + qb * 64 * 128, &tmQ, bar(kBarQFull), h, bh,
                                min(r0 + qb, nb - 1), prm.S, prm.Th, prm.Tw);
      } else if (is_k) {
        mbar_arrive(bar(kBarQFull));   // Q is still in place from the first pass
      }
      const int last = ulist[n_u - 1] & 0xFFFF;
      const bool kv_raster = kRaster && prm.kv_raster;
      for (int t = 0; t < n_t; ++t) {
        if (t > 0 && !mbar_wait(bar(empty), (t - 1) & 1, lim, abort_flag)) {
          record_abort(abort_flag, prm.status, kStatusTimeout);
          break;
        }
        mbar_arrive_expect_tx(bar(full), L::kKVBytes);
        ++armed;
        for (int e = 0; e < kEntries; ++e) {
          const int u = tile_of(t);
          const int j = (kEntries * u + e < n_u) ? (ulist[kEntries * u + e] & 0xFFFF) : last;
          for (int h = 0; h < L::kDH; ++h)
            if (kv_raster)
              load_block<true>(buf + h * kBN * 128 + e * 64 * 128, map, bar(full), h, bh, j,
                               prm.S, prm.Th, prm.Tw);
            else
              load_block<false>(buf + h * kBN * 128 + e * 64 * 128, map, bar(full), h, bh, j,
                                prm.S, prm.Th, prm.Tw);
        }
      }
      // drain: every armed phase must complete before shared memory is released
      if (is_k) mbar_wait(bar(kBarQFull), 0, kDrainLimitNs, nullptr);
      if (armed) mbar_wait(bar(full), (armed - 1) & 1, kDrainLimitNs, nullptr);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_t > 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, D, true);
      // S = Q K^T over the 256 keys of the tile in K buffer, 16-deep steps of d
      auto issue_s = [&]() {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offq = (kk >> 2) * (kBM * 128) + (kk & 3) * 32;
          const uint32_t offk = (kk >> 2) * (kBN * 128) + (kk & 3) * 32;
          tc_mma_ss(tmem + kColS, sdesc_sw128(sQ + offq, 16, 1024), sdesc_sw128(sK + offk, 16, 1024),
                    idesc_qk, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar(kBarSFull));
        tc_commit(bar(kBarKEmpty));
      };
      // O += P V: 16 keys per step, P columns [8kk, 8kk+8) of the P buffer, V
      // rows [16kk, 16kk+16); the 64-column halves of d are kBN*128 bytes apart
      auto issue_pv = [&](int t) {
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          tc_mma_ts(tmem + kColO, tmem + kColP + kk * 8,
                    sdesc_sw128(sV + kk * 16 * 128, kBN * 128, 1024), idesc_pv,
                    (t > 0 || kk > 0) ? 1u : 0u);
        tc_commit(bar(kBarOFull));
        tc_commit(bar(kBarVEmpty));
      };
      bool ok = mbar_wait(bar(kBarQFull), 0, lim, abort_flag) &&
                mbar_wait(bar(kBarKFull), 0, lim, abort_flag);
      if (ok) {
        tc_fence_after();
        issue_s();
      }
      for (int t = 0; ok && t < n_t; ++t) {
        if (t + 1 < n_t) {
          // S(t+1) overwrites S(t): every softmax thread must hold S(t) in registers
          if (!mbar_wait(bar(kBarSFree), t & 1, lim, abort_flag) ||
              !mbar_wait(bar(kBarKFull), (t + 1) & 1, lim, abort_flag)) {
            ok = false;
            break;
          }
          tc_fence_after();
          issue_s();
        }
        if (!mbar_wait(bar(kBarPFull), t & 1, lim, abort_flag) ||
            !mbar_wait(bar(kBarVFull), t & 1, lim, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        issue_pv(t);
      }
      if (!ok) record_abort(abort_flag, prm.status, kStatusTimeout);
      // drain: all MMAs this thread issued must finish before tensor memory is freed
      tc_commit(bar(kBarDrain));
      mbar_wait(bar(kBarDrain), 0, kDrainLimitNs, nullptr);
    }
  }
  if (!next_pass()) break;
  }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // ------------------------------------------------------------ softmax (warps 0-7)
    const int quarter = warp & 3;
    const int half = warp >> 2;                  // column half of the key tile
    const int row = quarter * 32 + lane;         // row of the tile == tensor-memory lane
    const int qh = row >> 6;                     // block r0 + qh
    const int qblock = r0 + qh;
    const bool row_valid = qblock < nb;
    const int bit = 1 << (16 + qh);
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_base = tmem + lane_off + kColS + 128u * half;
    const uint32_t p_base = tmem + lane_off + kColP + 64u * half;
    const uint32_t o_base = tmem + lane_off + kColO + static_cast<uint32_t>(D / 2) * half;
    const uint32_t pair_bar = bar(kBarPair + quarter);
    const float sl2 = prm.scale_log2;
    while (true) {
    float m = -INFINITY;        // reference max of the row, log2 units (same in both warps)
    float l = 0.f;              // running sum over this warp's columns of the row
    int pair_n = 0;             // phases of the pair barrier used so far
    bool ok = true;
    const bool exact_pass = *pass_s != 0;
    // list entries of the tile this warp's columns cover, read one tile ahead
    int e_next0 = tile_entry(0, 2 * half), e_next1 = tile_entry(0, 2 * half + 1);
    for (int t = 0; t < n_t; ++t) {
      const bool v0 = (e_next0 & bit) != 0;       // uniform per warp
      const bool v1 = (e_next1 & bit) != 0;
      if (!warp_wait(bar(kBarSFull), t & 1, lim, abort_flag)) { ok = false; break; }
      tc_fence_after();
      const bool agree = exact_pass || __any_sync(0xffffffffu, m == -INFINITY);
      // Split loads when the reference is fixed and both entries are listed:
      // the first 32 columns, then the other 96 while the first are
      // exponentiated.  Otherwise this warp's columns in one batch.
      const bool split = !agree && v0 && v1;
      uint32_t sv[4][32];
      if (split) {
        tmem_ld32(s_base, sv[0]);
        tmem_ld_wait();
        reg_fence32(sv[0]);
        tmem_ld32(s_base + 32, sv[1]);
        tmem_ld32(s_base + 64, sv[2]);
        tmem_ld32(s_base + 96, sv[3]);
      } else {
        if (v0) { tmem_ld32(s_base, sv[0]); tmem_ld32(s_base + 32, sv[1]); }
        if (v1) { tmem_ld32(s_base + 64, sv[2]); tmem_ld32(s_base + 96, sv[3]); }
        tmem_ld_wait();
        // S(t) is in registers: the tensor cores may overwrite it with S(t+1)
        tc_fence_before();
        mbar_arrive(bar(kBarSFree));
      }
      // Reference of the exponentials.  Fixed-reference pass: the row's
      // reference is the max of the first key tile the row's block lists
      // (agreed with the other warp of the lane quarter), then kept.  Exact
      // pass: the two warps agree on every tile's max and raise the reference
      // lazily.  Both warps take the same branch (m is the same in both).
      bool pv_done = t == 0;                     // PV(t-1) completed (known so far)
      if (t + 1 < n_t) {
        e_next0 = tile_entry(t + 1, 2 * half);
        e_next1 = tile_entry(t + 1, 2 * half + 1);
      }
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
        // the row's max over all 256 keys: trade partial maxima with the other
        // warp of this lane quarter (slots alternate with the barrier's phase)
        xch[((pair_n & 1) * 2 + half) * kBM + row] = m_part;
        mbar_arrive(pair_bar);
        if (!warp_wait(pair_bar, pair_n & 1, lim, abort_flag)) { ok = false; break; }
        const float m_tile = fmaxf(m_part, xch[((pair_n & 1) * 2 + (half ^ 1)) * kBM + row]);
        ++pair_n;
        const bool has = m_tile > -INFINITY;
        const bool first = m == -INFINITY;
        const bool need = has && !first && (m_tile > m + kRescaleThreshold);   // rescale O, l
        const float m_old = m;
        if (has && (first || need)) m = m_tile;
        // O must hold PV(t-1) before it is rescaled by 2^(m_old - m)
        bool rescale = __any_sync(0xffffffffu, need);
        if (rescale && !pv_done) {
          if (!warp_wait(bar(kBarOFull), (t - 1) & 1, lim, abort_flag)) {
            ok = false;
            rescale = false;
          }
          pv_done = true;
        }
        if (rescale) {
          tc_fence_after();
          const float alpha = need ? fast_exp2(m_old - m) : 1.f;
          l *= alpha;
#pragma unroll 1
          for (int cc = 0; cc < D / 32; ++cc) {
            uint32_t o[16];
            tmem_ld16(o_base + cc * 16, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st16(o_base + cc * 16, o);
            tmem_st_wait();
          }
        }
      }
      // p = 2^(s*scale*log2e - m), packed to bf16 pairs and kept in registers
      // until PV(t-1) has read the P buffer
      const bool live = m > -INFINITY;
      const float mneg = live ? -m : 0.f;
      float rs[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t pk[4][16];
      if (v0 && v1 && __all_sync(0xffffffffu, live)) {
        // common case, one straight-line block: every column of the row is listed
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = fast_exp2(fmaf(__uint_as_float(sv[ch][2 * i]), sl2, mneg));
            const float p1 = fast_exp2(fmaf(__uint_as_float(sv[ch][2 * i + 1]), sl2, mneg));
            rs[i & 3] += p0 + p1;
            pk[ch][i] = pack_bf16x2(p0, p1);
          }
          if (ch == 0 && split) {
            tmem_ld_wait();
            reg_fence32(sv[1]);
            reg_fence32(sv[2]);
            reg_fence32(sv[3]);
            tc_fence_before();
            mbar_arrive(bar(kBarSFree));
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
      if (!ok) break;
      if (!pv_done && !warp_wait(bar(kBarOFull), (t - 1) & 1, lim, abort_flag)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) tmem_st16(p_base + ch * 16, pk[ch]);
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(kBarPFull));
      // a row whose later keys outgrow the fixed reference asks for the exact pass
      if (!agree && __any_sync(0xffffffffu, !(l_tile <= kFixedRefSumLimit)) && lane == 0)
        *cta_redo = 1;
    }
    if (!ok) record_abort(abort_flag, prm.status, kStatusTimeout);
    // ------------------------------------------------------------ epilogue
    bool have_o = false;
    if (ok && n_t > 0) {
      have_o = warp_wait(bar(kBarOFull), (n_t - 1) & 1, lim, abort_flag);
      if (!have_o) record_abort(abort_flag, prm.status, kStatusTimeout);
      tc_fence_after();
    }
    // the row sum over all keys: trade partial sums with the other warp
    bool have_l = ok;
    float l_row = l;
    if (ok) {
      xch[((pair_n & 1) * 2 + half) * kBM + row] = l;
      mbar_arrive(pair_bar);
      have_l = warp_wait(pair_bar, pair_n & 1, lim, abort_flag);
      if (!have_l) record_abort(abort_flag, prm.status, kStatusTimeout);
      else l_row = l + xch[((pair_n & 1) * 2 + (half ^ 1)) * kBM + row];
    }
    const bool write = row_valid && have_l && (n_t == 0 || have_o);
    const int64_t grow = static_cast<int64_t>(bh) * prm.S +
                         (row_valid ? token_of<kRaster>(qblock, row & 63, prm.Th, prm.Tw) : 0);
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
    if (!next_pass()) break;
    }
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
                           int* status, int* redo, int* exact_passes, int exact_only, int BH,
                           int H, int S, int d, float scale, int raster, int kv_raster, int Th,
                           int Tw, uint64_t wait_limit_ns, cudaStream_t st) {
  AttnParams prm;
  prm.row_ptr = row_ptr;
  prm.col_idx = col_idx;
  prm.o = static_cast<__nv_bfloat16*>(o);
  prm.lse = lse;
  prm.status = status;
  prm.H = H;
  prm.S = S;
  prm.nb = S / 64;
  prm.ngroups = (prm.nb + 1) / 2;
  prm.Th = Th;
  prm.Tw = Tw;
  prm.scale_log2 = scale * 1.4426950408889634f;
  prm.wait_limit_ns = wait_limit_ns;
  prm.redo = redo;
  prm.exact_passes = exact_passes;
  prm.kv_raster = kv_raster;
  const int64_t nitems = static_cast<int64_t>(BH) * prm.ngroups;
  if (nitems == 0) return cudaSuccess;
  // One launch.  exact_only 0: each CTA runs the fixed-reference pass and, if
  // a row of its tile outgrew the reference, the exact-reference pass over the
  // same tile (the first such CTA sets *redo and counts the forward); 1: the
  // exact-reference pass alone; 2: the exact-reference pass alone, only if a
  // fixed-reference pass that another kernel ran left *redo set.
  cudaError_t e = exact_only == 2 ? cudaSuccess : cudaMemsetAsync(redo, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  prm.exact = exact_only;
  if (raster) {
    e = d == 128 ? launch_fwd_t<128, true>(q, k, v, prm, nitems, st)
                 : launch_fwd_t<64, true>(q, k, v, prm, nitems, st);
  } else {
    e = d == 128 ? launch_fwd_t<128, false>(q, k, v, prm, nitems, st)
                 : launch_fwd_t<64, false>(q, k, v, prm, nitems, st);
  }
  return e;
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
