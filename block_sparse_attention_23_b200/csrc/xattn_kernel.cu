// XAttention antidiagonal block scores on sm_100a (the alternative scorer of
// "XAttention: Block Sparse Attention with Antidiagonal Scoring": blocks are
// scored along antidiagonals and then selected by a threshold).
//
// With stride St (4, 8 or 16), strided query row i and strided key row j of a
// head stand for the St x St sub-block of Q K^T at rows i*St.., columns j*St..;
// their score is the mean of that sub-block's antidiagonal,
//   a_ij = (1/St) sum_{s<St} q_{i*St + St-1-s} . k_{j*St + s} / sqrt(d),
// i.e. a dot product of two St*d-feature rows: Q' row i = the St query rows of
// group i in reverse order, K' row j = the St key rows of group j in order.
// p_i = softmax_j(a_i) over all L = S/St strided keys of the head, and the
// score of (query block r, key block c) is the mean over r's 64/St strided
// rows of the mass p puts on c's 64/St strided keys (rows of the score matrix
// sum to 1).  The scores then go through the mask builder's selection.
//
// Two passes of one kernel: pass 1 forms the log2-domain LSE of every strided
// query row (online max and sum over the key tiles), pass 2 the block sums of
// p = 2^(a log2e - lse2).  One CTA per (b, h, 128 strided query rows); key
// tiles of 256 strided rows; S = Q' K'^T (N = 256: the full tensor rate)
// accumulates over St*d/64 chunks of 64 features, each chunk a pair of 3D TMA
// boxes (128 Q' rows and 256 K' rows x 64 columns, rows St apart in the token
// axis: the antidiagonal gather happens in the copy).  S is double-buffered in
// tensor memory (2 x 256 columns); two groups of four warps take alternate key
// tiles (so two warps share each SM sub-partition's exponential unit), each
// row's 256 columns in two halves of 128, pass 1 combining the groups' running
// maxima and sums at the end, pass 2 writing disjoint blocks.  The block sums over a query block's 64/St rows
// (consecutive lanes of a warp) are butterfly shuffles; each block score is
// written once, by the lane that leads its rows.
//
// Roles (384 threads): warps 0-7 exponentials, warp 8 TMA producer, warp 9
// tensor memory and the MMA-issuing thread, warps 10-11 idle.  Every mbarrier
// wait is time-bounded (kStatusTimeout, abort flag, drain before freeing
// tensor memory); an aborted CTA writes nothing.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

#include "sm100_primitives.cuh"

namespace nabla {

constexpr int kXM = 128;                        // strided query rows per CTA
constexpr int kXN = 256;                        // strided key rows per tile
constexpr int kXStages = 4;                     // ring of (Q' chunk, K' chunk) pairs
constexpr int kXThreads = 384;
constexpr int kXExpWarps = 8;
constexpr int kXProducerWarp = 8, kXMmaWarp = 9;
constexpr uint32_t kXChunkQBytes = kXM * 64 * 2;   // Q' chunk: 128 rows x 64 bf16
constexpr uint32_t kXChunkKBytes = kXN * 64 * 2;   // K' chunk: 256 rows x 64 bf16
constexpr uint32_t kXStageBytes = kXChunkQBytes + kXChunkKBytes;
constexpr uint32_t kXTmemCols = 512;
// Register split after set-up (per warpgroup): 8*216 + 4*72 = 12*168, the
// launch allocation (checked on the host before launch).
constexpr int kXRegsExp = 216, kXRegsOther = 72, kXRegsLaunch = 168;
constexpr uint64_t kXDrainNs = 1000000000ull;

struct XSmem {
  static constexpr uint32_t kOffRing = 0;
  static constexpr uint32_t kOffBar = kOffRing + kXStages * kXStageBytes;   // 16 mbarriers
  static constexpr uint32_t kOffMisc = kOffBar + 128;                       // tmem base, abort
  static constexpr uint32_t kOffComb = kOffMisc + 64;                       // [2][kXM] (m, l) of group 1
  static constexpr uint32_t kBytes = kOffComb + 2 * kXM * 4;
  static constexpr uint32_t kAlloc = kBytes + 1024;
};

enum : int {
  kXBarFull = 0,                       // + stage
  kXBarEmpty = kXBarFull + kXStages,   // + stage
  kXBarSFull = kXBarEmpty + kXStages,  // + S buffer
  kXBarSFree = kXBarSFull + 2,         // + S buffer
  kXBarDrain = kXBarSFree + 2,
  kXNumBars = kXBarDrain + 1
};
static_assert(kXNumBars * 8 <= 128, "barrier area");

struct XParams {
  float* lse2;        // [BH * L] log2-domain LSE of each strided query row (pass 1 out, pass 2 in)
  float* scores;      // [BH * nb * nb]
  int* status;
  int L;              // strided rows per head (S / St)
  int nb;             // 64-token blocks per head
  int per;            // strided rows per block (64 / St)
  int St;
  int dh;             // 64-feature halves of d
  int nqt, nkt;       // 128-row query / key tiles per head
  float sl2;          // log2(e) / (St * sqrt(d))
  uint64_t wait_limit_ns;
};

__device__ __forceinline__ bool x_warp_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                            const volatile int* abort) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, limit_ns, abort));
}

__device__ __forceinline__ void x_abort(volatile int* abort, int* status) {
  *abort = 1;
  atomicOr(status, kStatusTimeout);
}

// kPass 1: LSE of the strided query rows; kPass 2: block scores.  kPer = 64 / St.
template <int kPass, int kPer>
__global__ void __launch_bounds__(kXThreads, 1)
    xattn_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                 const XParams prm) {
  using L = XSmem;
  extern __shared__ uint8_t x_smem_raw[];
  const uint32_t raw = smem_addr(x_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = x_smem_raw + (base - raw);
  const uint32_t sRing = base + L::kOffRing;
  const uint32_t bar0 = base + L::kOffBar;
  uint32_t* misc = reinterpret_cast<uint32_t*>(gbase + L::kOffMisc);
  volatile uint32_t* tmem_holder = misc;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  float* comb = reinterpret_cast<float*>(gbase + L::kOffComb);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x / prm.nqt;
  const int qt = blockIdx.x % prm.nqt;
  const int n_t = prm.nkt;
  const int nchunks = prm.St * prm.dh;
  const uint64_t lim = prm.wait_limit_ns;
  auto bar = [&](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };

  if (tid == 0) {
    for (int s = 0; s < kXStages; ++s) {
      mbar_init(bar(kXBarFull + s), 1);
      mbar_init(bar(kXBarEmpty + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(kXBarSFull + b), 1);
      mbar_init(bar(kXBarSFree + b), (kXExpWarps / 2) * 32);
    }
    mbar_init(bar(kXBarDrain), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kXMmaWarp) {
    tmem_alloc(smem_addr(misc), kXTmemCols);
    tmem_relinquish();
  }
  if (warp == kXProducerWarp && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;

  // per-thread results carried past the role branches (exponent warps only)
  float res_m = -INFINITY, res_l = 0.f;

  if (warp >= kXExpWarps) {
  setmaxnreg_dec<kXRegsOther>();
  if (warp == kXProducerWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const int32_t qrow = static_cast<int32_t>(static_cast<int64_t>(bh) * prm.L + qt * kXM);
      int armed[kXStages] = {0, 0, 0, 0};
      int u = 0;   // chunk counter over all tiles
      for (int t = 0; t < n_t; ++t) {
        const int32_t krow = static_cast<int32_t>(static_cast<int64_t>(bh) * prm.L + t * kXN);
        bool stop = false;
        for (int c = 0; c < nchunks; ++c, ++u) {
          const int st = u % kXStages, n = u / kXStages;
          if (u >= kXStages && !mbar_wait(bar(kXBarEmpty + st), (n - 1) & 1, lim, abort_flag)) {
            x_abort(abort_flag, prm.status);
            stop = true;
            break;
          }
          const int s = c / prm.dh, h = c % prm.dh;
          const uint32_t dst = sRing + st * kXStageBytes;
          mbar_arrive_expect_tx(bar(kXBarFull + st), kXStageBytes);
          ++armed[st];
          // Q' chunk: query rows i*St + (St-1-s); K' chunk: key rows j*St + s
          tma_load_3d(dst, &tmQ, bar(kXBarFull + st), h * 64, prm.St - 1 - s, qrow);
          tma_load_3d(dst + kXChunkQBytes, &tmK, bar(kXBarFull + st), h * 64, s, krow);
        }
        if (stop) break;
      }
      for (int st = 0; st < kXStages; ++st)
        if (armed[st]) mbar_wait(bar(kXBarFull + st), (armed[st] - 1) & 1, kXDrainNs, nullptr);
    }
  } else if (warp == kXMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kXM, kXN, false);
      bool ok = true;
      int u = 0;
      for (int t = 0; ok && t < n_t; ++t) {
        const int b = t & 1;
        // the S buffer is free once its group has loaded tile t-2
        if (t >= 2 && !mbar_wait(bar(kXBarSFree + b), ((t >> 1) - 1) & 1, lim, abort_flag)) {
          ok = false;
          break;
        }
        for (int c = 0; c < nchunks; ++c, ++u) {
          const int st = u % kXStages;
          if (!mbar_wait(bar(kXBarFull + st), (u / kXStages) & 1, lim, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a = sRing + st * kXStageBytes, bk = a + kXChunkQBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_ss(tmem + b * static_cast<uint32_t>(kXN), sdesc_sw128(a + kk * 32, 16, 1024),
                      sdesc_sw128(bk + kk * 32, 16, 1024), idesc, (c > 0 || kk > 0) ? 1u : 0u);
          tc_commit(bar(kXBarEmpty + st));
        }
        if (!ok) break;
        tc_commit(bar(kXBarSFull + b));
      }
      if (!ok) x_abort(abort_flag, prm.status);
      tc_commit(bar(kXBarDrain));
      mbar_wait(bar(kXBarDrain), 0, kXDrainNs, nullptr);
    }
  }
  } else {
    setmaxnreg_inc<kXRegsExp>();
    // ------------------------------------------------------------ exponentials
    const int grp = warp >> 2;                  // key tiles t = grp mod 2, S buffer grp
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;        // strided query row in the tile == lane
    const int qrow = qt * kXM + row;            // strided query row in the head
    const bool row_valid = qrow < prm.L;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sl2 = prm.sl2;
    float lse2 = 0.f;
    if (kPass == 2 && row_valid) lse2 = prm.lse2[static_cast<int64_t>(bh) * prm.L + qrow];
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int t = grp; t < n_t; t += 2) {
      const int nvalid_t = min(kXN, prm.L - t * kXN);   // a multiple of kPer
      if (!x_warp_wait(bar(kXBarSFull + grp), (t >> 1) & 1, lim, abort_flag)) { ok = false; break; }
      tc_fence_after();
#pragma unroll 1
      for (int hf = 0; hf < 2; ++hf) {     // 128 columns at a time
        const int nvalid = nvalid_t - 128 * hf;
        if (nvalid <= 0) {
          if (hf == 1) {   // the buffer is read (nothing in this half)
            tc_fence_before();
            mbar_arrive(bar(kXBarSFree + grp));
          }
          continue;
        }
        const uint32_t sb = tmem + lane_off + grp * static_cast<uint32_t>(kXN) + 128u * hf;
        uint32_t sv[4][32];
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) tmem_ld32(sb + ch * 32, sv[ch]);
        tmem_ld_wait();
        if (hf == 1) {   // both halves read: the tensor cores may refill the buffer
          tc_fence_before();
          mbar_arrive(bar(kXBarSFree + grp));
        }
        if (kPass == 1) {
          float mx = -INFINITY;
#pragma unroll
          for (int ch = 0; ch < 4; ++ch)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (ch * 32 + i < nvalid) mx = fmaxf(mx, __uint_as_float(sv[ch][i]));
          const float m_new = fmaxf(m, mx * sl2);
          float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int ch = 0; ch < 4; ++ch)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (ch * 32 + i < nvalid)
                acc[i & 3] += fast_exp2(fmaf(__uint_as_float(sv[ch][i]), sl2, -m_new));
          l = l * fast_exp2(m - m_new) + ((acc[0] + acc[1]) + (acc[2] + acc[3]));
          m = m_new;
        } else {
          // block sums of p over this half's 128 / kPer key blocks, then over
          // the kPer rows of the query block (consecutive lanes)
          constexpr int kNkb = 128 / kPer;
          float bs[kNkb];
#pragma unroll
          for (int j = 0; j < kNkb; ++j) {
            float a = 0.f;
#pragma unroll
            for (int e = 0; e < kPer; ++e) {
              const int c = j * kPer + e;
              if (c < nvalid) a += fast_exp2(fmaf(__uint_as_float(sv[c >> 5][c & 31]), sl2, -lse2));
            }
            bs[j] = row_valid ? a : 0.f;
          }
#pragma unroll
          for (int o = 1; o < kPer; o <<= 1)
#pragma unroll
            for (int j = 0; j < kNkb; ++j) bs[j] += __shfl_xor_sync(0xffffffffu, bs[j], o);
          if ((lane % kPer) == 0 && row_valid && *abort_flag == 0) {
            const int rb = qrow / kPer;                      // query block in the head
            float* dst = prm.scores + (static_cast<int64_t>(bh) * prm.nb + rb) * prm.nb +
                         (t * kXN + 128 * hf) / kPer;
            const float inv = 1.0f / kPer;
#pragma unroll
            for (int j = 0; j < kNkb; ++j)
              if (j * kPer < nvalid) dst[j] = bs[j] * inv;
          }
        }
      }
    }
    if (!ok) x_abort(abort_flag, prm.status);
    res_m = m;
    res_l = l;
  }

  // ---------------------------------------------------------------- combine (pass 1)
  tc_fence_before();
  __syncthreads();
  if (kPass == 1) {
    if (warp >= 4 && warp < kXExpWarps) {       // group 1 hands its (m, l) to group 0
      const int row = (warp & 3) * 32 + lane;
      comb[row] = res_m;
      comb[kXM + row] = res_l;
    }
    __syncthreads();
    if (warp < 4 && *abort_flag == 0) {
      const int row = warp * 32 + lane;
      const int qrow = qt * kXM + row;
      if (qrow < prm.L) {
        const float m1 = comb[row], l1 = comb[kXM + row];
        const float mm = fmaxf(res_m, m1);
        const float ll = (res_l > 0.f ? res_l * fast_exp2(res_m - mm) : 0.f) +
                         (l1 > 0.f ? l1 * fast_exp2(m1 - mm) : 0.f);
        prm.lse2[static_cast<int64_t>(bh) * prm.L + qrow] = mm + __log2f(ll);
      }
    }
  }
  if (warp == kXMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kXTmemCols);
  }
}

template <int kPass, int kPer>
static cudaError_t launch_x_t(const CUtensorMap& q, const CUtensorMap& k, const XParams& prm,
                              int64_t nitems, cudaStream_t st) {
  constexpr uint32_t smem = XSmem::kAlloc;
  static_assert(8 * kXRegsExp + 4 * kXRegsOther <= 12 * kXRegsLaunch, "register split");
  cudaFuncAttributes attr;
  cudaError_t e = cudaFuncGetAttributes(&attr, xattn_kernel<kPass, kPer>);
  if (e != cudaSuccess) return e;
  if (attr.numRegs < kXRegsLaunch) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(xattn_kernel<kPass, kPer>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem);
  if (e != cudaSuccess) return e;
  xattn_kernel<kPass, kPer><<<static_cast<unsigned>(nitems), kXThreads, smem, st>>>(q, k, prm);
  return cudaGetLastError();
}

template <int kPer>
static cudaError_t launch_x_both(const CUtensorMap& q, const CUtensorMap& k, const XParams& prm,
                                 int64_t nitems, cudaStream_t st) {
  cudaError_t e = launch_x_t<1, kPer>(q, k, prm, nitems, st);
  if (e != cudaSuccess) return e;
  return launch_x_t<2, kPer>(q, k, prm, nitems, st);
}

// q, k: 3D tensor maps over [BH * L][St][d] (boxes 64 x 1 x 128, 128-byte swizzle).
cudaError_t launch_xattn_scores(const CUtensorMap& q, const CUtensorMap& k, float* lse2,
                                float* scores, int* status, int BH, int S, int d, int St,
                                uint64_t wait_limit_ns, cudaStream_t st) {
  XParams prm;
  prm.lse2 = lse2;
  prm.scores = scores;
  prm.status = status;
  prm.St = St;
  prm.L = S / St;
  prm.nb = S / 64;
  prm.per = 64 / St;
  prm.dh = d / 64;
  prm.nqt = (prm.L + kXM - 1) / kXM;
  prm.nkt = (prm.L + kXN - 1) / kXN;
  prm.sl2 = 1.4426950408889634f / (static_cast<float>(St) * sqrtf(static_cast<float>(d)));
  prm.wait_limit_ns = wait_limit_ns;
  const int64_t nitems = static_cast<int64_t>(BH) * prm.nqt;
  if (nitems == 0) return cudaSuccess;
  switch (prm.per) {
    case 16: return launch_x_both<16>(q, k, prm, nitems, st);
    case 8: return launch_x_both<8>(q, k, prm, nitems, st);
    case 4: return launch_x_both<4>(q, k, prm, nitems, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace nabla
