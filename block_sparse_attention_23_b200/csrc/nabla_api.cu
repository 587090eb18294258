// libnabla C ABI: argument checks, workspace layout, TMA descriptors and
// kernel launches.  No entry point allocates device memory or synchronises,
// except nabla_query_status (which must read the device status word).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "../../include/nabla.h"
#include "sm100_primitives.cuh"

namespace nabla {
cudaError_t launch_pool(const void* q, const void* k, double* qbar, double* kbar,
                        int64_t nblocks, int d, int nb, int raster, int Th, int Tw,
                        cudaStream_t st);
cudaError_t launch_logits(const double* qbar, const double* kbar, double* L, int BH, int nb,
                          int d, cudaStream_t st);
cudaError_t launch_select(const double* L, int64_t nrows, int nb, float thr, int topk,
                          int use_sta, int wt, int wh, int ww, int Tt, int Th, int Tw,
                          uint32_t* bits, int32_t* counts, uint8_t* mask_u8, cudaStream_t st);
cudaError_t launch_mask_bits(const uint8_t* mask, int64_t nrows, int nb, uint32_t* bits,
                             int32_t* counts, cudaStream_t st);
cudaError_t launch_scan_fill(const uint32_t* bits, const int32_t* counts, int64_t nrows, int nb,
                             int32_t* row_ptr, int32_t* col_idx, int64_t capacity,
                             int32_t* nnz_out, int* status, cudaStream_t st);
cudaError_t launch_bsa_fwd(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                           const int32_t* row_ptr, const int32_t* col_idx, void* o, float* lse,
                           int* status, int* redo, int* exact_passes, int exact_only, int BH,
                           int H, int S, int d, float scale, int raster, int kv_raster, int Th,
                           int Tw, uint64_t wait_limit_ns, cudaStream_t st);
cudaError_t launch_reorder(const void* src, void* dst, int64_t BH, int Tt, int Th, int Tw,
                           int row_bytes, int to_tile_major, cudaStream_t st);
cudaError_t launch_block_energy(const CUtensorMap& q, const CUtensorMap& k, const int32_t* row_ptr,
                                const int32_t* col_idx, const float* lse, float* energy,
                                float* block_mass, int* status, int BH, int S, int d, float scale,
                                uint64_t wait_limit_ns, cudaStream_t st);
cudaError_t launch_calib_select(const float* energy, int64_t nrows, int nb, float eps,
                                int32_t* votes, cudaStream_t st);
cudaError_t launch_vote_mask(const int32_t* votes, int64_t n, int32_t min_votes, uint8_t* mask,
                             cudaStream_t st);
cudaError_t launch_bsa_bwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                           const CUtensorMap& mdo, const void* o, const void* dout,
                           const float* lse, const int32_t* row_ptr, const int32_t* col_idx,
                           float* dvec, float* lse2, uint32_t* colbits, void* dq, void* dk,
                           void* dv, int* status, int BH, int S, int d, float scale,
                           uint64_t wait_limit_ns, cudaStream_t st);
cudaError_t launch_select_weights(const float* weights, int64_t nrows, int nb, float thr, int topk,
                                  int use_sta, int wt, int wh, int ww, int Tt, int Th, int Tw,
                                  uint32_t* bits, int32_t* counts, uint8_t* mask_u8,
                                  cudaStream_t st);
cudaError_t launch_xattn_scores(const CUtensorMap& q, const CUtensorMap& k, float* lse2,
                                float* scores, int* status, int BH, int S, int d, int St,
                                uint64_t wait_limit_ns, cudaStream_t st);
cudaError_t launch_bsa_fwd_pair(const CUtensorMap& q, const CUtensorMap& k, const CUtensorMap& v,
                                const int32_t* row_ptr, const int32_t* col_idx, void* o,
                                float* lse, int* status, int* redo, int BH, int S, float scale,
                                uint64_t wait_limit_ns, cudaStream_t st);
cudaError_t launch_mma_pair_selftest(const CUtensorMap& a, const CUtensorMap& b,
                                     const void* p_glob, float* c, int variant, int* status,
                                     uint64_t lim, cudaStream_t st);
cudaError_t launch_mma_selftest(const CUtensorMap& a, const CUtensorMap& b, const void* a_glob,
                                float* c, int variant, int* status, uint64_t lim,
                                cudaStream_t st);
}  // namespace nabla

namespace {

// NVTX range over one library call (a no-op unless a profiler is attached), so
// timelines and `ncu --nvtx` filters show which entry point launched what.
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
};

// Workspace header (256 bytes, zeroed by nabla_workspace_init): int32 words
// [0] status bits, [1] the forward's exact-pass request, [2] exact passes run
// (a counter), [4 + slot] the exact-pass requests of the host-buffer layer's
// two slots.
constexpr size_t kHeaderBytes = 256;
constexpr int kHdrRedo = 1, kHdrExactPasses = 2;
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;   // 2 s
constexpr int kMaxNbSupported = 4096;

thread_local std::string g_last_error;
std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitLimitNs};
std::atomic<int> g_exact_reference{0};
// Which kernel runs the fixed-reference pass of a d = 128 tile-major forward:
// 0 (default) one CTA per two query blocks; 1 CTA pairs for block lists from
// the mask builder (bsa_fwd and the host-buffer layer) only; 2 CTA pairs
// always.  The pair kernel halves each SM's K/V traffic but puts cross-SM
// arrivals on the softmax -> PV -> softmax chain of every tile; on the Wan
// 720p-shaped layer it ran 19.4 ms against 15.0 ms for 8 heads.
std::atomic<int> g_pair_mode{0};
bool pair_for(bool builder_list) {
  const int m = g_pair_mode.load();
  return m == 2 || (m == 1 && builder_list);
}

nabla_status fail(nabla_status s, const std::string& msg) {
  g_last_error = msg;
  return s;
}

nabla_status cuda_fail(cudaError_t e, const char* where) {
  g_last_error = std::string(where) + ": " + cudaGetErrorString(e);
  return NABLA_ERR_CUDA;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates the tensor shape shared by every call.
nabla_status check_shape(const nabla_shape* s) {
  if (s == nullptr) return fail(NABLA_ERR_INVALID_ARG, "shape is NULL");
  if (s->B <= 0 || s->H <= 0 || s->S <= 0 || s->d <= 0)
    return fail(NABLA_ERR_INVALID_ARG, "B, H, S and d must be positive");
  if (s->d != 64 && s->d != 128) return fail(NABLA_ERR_UNSUPPORTED, "d must be 64 or 128");
  if (s->S % 64 != 0) return fail(NABLA_ERR_UNSUPPORTED, "S must be a multiple of 64");
  const int64_t nb = s->S / 64;
  if (nb > kMaxNbSupported) return fail(NABLA_ERR_UNSUPPORTED, "S/64 must be at most 4096");
  const int64_t rows = static_cast<int64_t>(s->B) * s->H * nb;
  if (rows * nb >= (static_cast<int64_t>(1) << 31))
    return fail(NABLA_ERR_UNSUPPORTED, "B*H*nb*nb must stay below 2^31");
  if (static_cast<int64_t>(s->B) * s->H * s->S >= (static_cast<int64_t>(1) << 31))
    return fail(NABLA_ERR_UNSUPPORTED, "B*H*S must stay below 2^31");
  if (s->layout != NABLA_LAYOUT_TILE_MAJOR && s->layout != NABLA_LAYOUT_RASTER)
    return fail(NABLA_ERR_INVALID_ARG, "unknown token layout");
  if (s->layout == NABLA_LAYOUT_RASTER &&
      (s->Tt <= 0 || s->Th <= 0 || s->Tw <= 0 ||
       static_cast<int64_t>(s->Tt) * s->Th * s->Tw != nb))
    return fail(NABLA_ERR_INVALID_ARG, "raster layout needs a tile grid with Tt*Th*Tw = S/64");
  return NABLA_OK;
}

// For calls that take tile-major tokens only.
nabla_status require_tile_major(const nabla_shape* s) {
  if (s->layout != NABLA_LAYOUT_TILE_MAJOR)
    return fail(NABLA_ERR_UNSUPPORTED, "this call takes tile-major tokens; use nabla_reorder_tokens");
  return NABLA_OK;
}

struct BuildLayout {
  size_t qbar, kbar, logits, bits, counts, total;
};

BuildLayout build_layout(const nabla_shape* s) {
  const size_t nb = s->S / 64, BH = static_cast<size_t>(s->B) * s->H, nw = (nb + 31) / 32;
  BuildLayout l;
  size_t off = kHeaderBytes;
  l.qbar = off; off = align256(off + BH * nb * s->d * 8);
  l.kbar = off; off = align256(off + BH * nb * s->d * 8);
  l.logits = off; off = align256(off + BH * nb * nb * 8);
  l.bits = off; off = align256(off + BH * nb * nw * 4);
  l.counts = off; off = align256(off + BH * nb * 4);
  l.total = off;
  return l;
}

struct BwdLayout {
  size_t dvec, lse2, colbits, total;
};

BwdLayout bwd_layout(const nabla_shape* s) {
  const size_t nb = s->S / 64, BH = static_cast<size_t>(s->B) * s->H, nw = (nb + 31) / 32;
  BwdLayout l;
  size_t off = kHeaderBytes;
  l.dvec = off; off = align256(off + BH * s->S * 4);
  l.lse2 = off; off = align256(off + BH * s->S * 4);
  l.colbits = off; off = align256(off + BH * nb * nw * 4);
  l.total = off;
  return l;
}

struct XattnLayout {
  size_t lse2, scores, bits, counts, total;
};

// Sized for the smallest supported stride (4): S/4 strided rows per head.
XattnLayout xattn_layout(const nabla_shape* s) {
  const size_t nb = s->S / 64, BH = static_cast<size_t>(s->B) * s->H, nw = (nb + 31) / 32;
  XattnLayout l;
  size_t off = kHeaderBytes;
  l.lse2 = off; off = align256(off + BH * (s->S / 4) * 4);
  l.scores = off; off = align256(off + BH * nb * nb * 4);
  l.bits = off; off = align256(off + BH * nb * nw * 4);
  l.counts = off; off = align256(off + BH * nb * 4);
  l.total = off;
  return l;
}

// One tile-major copy of K or V for a raster-ordered forward (256-aligned).
size_t kv_copy_bytes(const nabla_shape* s) {
  return align256(static_cast<size_t>(s->B) * s->H * s->S * s->d * 2);
}

// Bytes a forward needs after its other workspace contents: the tile-major
// K and V copies for raster token order, nothing otherwise.
size_t kv_scratch_bytes(const nabla_shape* s) {
  return s->layout == NABLA_LAYOUT_RASTER ? 2 * kv_copy_bytes(s) : 0;
}

struct MaskLayout {
  size_t bits, counts, row_ptr, col_idx, total;
};

MaskLayout mask_layout(const nabla_shape* s) {
  const size_t nb = s->S / 64, BH = static_cast<size_t>(s->B) * s->H, nw = (nb + 31) / 32;
  MaskLayout l;
  size_t off = kHeaderBytes;
  l.bits = off; off = align256(off + BH * nb * nw * 4);
  l.counts = off; off = align256(off + BH * nb * 4);
  l.row_ptr = off; off = align256(off + (BH * nb + 1) * 4);
  l.col_idx = off; off = align256(off + BH * nb * nb * 4);
  l.total = off;
  return l;
}

// cuTensorMapEncodeTiled, fetched from the driver at run time so the library
// has no link-time dependency on libcuda.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// [rows, cols] bf16 row-major; 64 x 64 boxes with 128-byte swizzle.
nabla_status make_map(CUtensorMap* map, const void* ptr, uint64_t rows, uint64_t cols) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(NABLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NABLA_ERR_CUDA, "cuTensorMapEncodeTiled failed");
  return NABLA_OK;
}

// [BH][4Tt][4Th][4Tw][d] bf16 (raster token order); 5D boxes of 64 x 4 x 4 x 4 x 1 =
// one 4x4x4 tile, 128-byte swizzle, rows landing in (t, h, w)-major order.
nabla_status make_map_raster(CUtensorMap* map, const void* ptr, const nabla_shape* s) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(NABLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t d = s->d, W = 4ull * s->Tw, H = 4ull * s->Th, T = 4ull * s->Tt;
  const cuuint64_t BH = static_cast<cuuint64_t>(s->B) * s->H;
  cuuint64_t dims[5] = {d, W, H, T, BH};
  cuuint64_t strides[4] = {d * 2, W * d * 2, H * W * d * 2, T * H * W * d * 2};
  cuuint32_t box[5] = {64, 4, 4, 4, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NABLA_ERR_CUDA, "cuTensorMapEncodeTiled (5D) failed");
  return NABLA_OK;
}

// [rows][St][d] bf16 viewed as stride-St groups of token rows: 3D boxes of
// 64 x 1 x 128 pick one token of each of 128 consecutive groups (128-byte swizzle).
nabla_status make_map_strided(CUtensorMap* map, const void* ptr, uint64_t groups, int St, int d,
                              uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return fail(NABLA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(St), groups};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(St) * d * 2};
  cuuint32_t box[3] = {64, 1, box_rows};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(NABLA_ERR_CUDA, "cuTensorMapEncodeTiled (3D) failed");
  return NABLA_OK;
}

int* status_ptr(void* ws) { return static_cast<int*>(ws); }

// Raster token order: K and V are reordered into kv_scratch (2 tile-major
// tensors) when the caller provides it, else read by 5D boxes in the kernel.
nabla_status run_fwd(const nabla_shape* shape, const void* q, const void* k, const void* v,
                     const int32_t* row_ptr, const int32_t* col_idx, float scale, void* o,
                     float* lse, int* header, int* redo, void* kv_scratch, cudaStream_t st,
                     bool use_pair) {
  const uint64_t rows = static_cast<uint64_t>(shape->B) * shape->H * shape->S;
  const bool raster = shape->layout == NABLA_LAYOUT_RASTER;
  const bool kv_raster = raster && kv_scratch == nullptr;
  CUtensorMap mq, mk, mv;
  nabla_status s;
  if (raster) {
    if ((s = make_map_raster(&mq, q, shape)) != NABLA_OK) return s;
    if (kv_raster) {
      if ((s = make_map_raster(&mk, k, shape)) != NABLA_OK) return s;
      if ((s = make_map_raster(&mv, v, shape)) != NABLA_OK) return s;
    } else {
      uint8_t* kt = static_cast<uint8_t*>(kv_scratch);
      uint8_t* vt = kt + kv_copy_bytes(shape);
      const int64_t BH = static_cast<int64_t>(shape->B) * shape->H;
      cudaError_t e = nabla::launch_reorder(k, kt, BH, shape->Tt, shape->Th, shape->Tw,
                                            shape->d * 2, 1, st);
      if (e == cudaSuccess)
        e = nabla::launch_reorder(v, vt, BH, shape->Tt, shape->Th, shape->Tw, shape->d * 2, 1, st);
      if (e != cudaSuccess) return cuda_fail(e, "K/V reorder launch");
      if ((s = make_map(&mk, kt, rows, shape->d)) != NABLA_OK) return s;
      if ((s = make_map(&mv, vt, rows, shape->d)) != NABLA_OK) return s;
    }
  } else {
    if ((s = make_map(&mq, q, rows, shape->d)) != NABLA_OK) return s;
    if ((s = make_map(&mk, k, rows, shape->d)) != NABLA_OK) return s;
    if ((s = make_map(&mv, v, rows, shape->d)) != NABLA_OK) return s;
  }
  if (!(scale > 0.f)) scale = 1.0f / std::sqrt(static_cast<float>(shape->d));
  int exact_only = g_exact_reference.load();
  if (use_pair && exact_only == 0 && shape->d == 128 && !raster) {
    // the fixed-reference pass on CTA pairs; the exact-reference pass (one-CTA
    // kernel) follows and returns at once unless a row asked for it
    cudaError_t e = cudaMemsetAsync(redo, 0, sizeof(int), st);
    if (e == cudaSuccess)
      e = nabla::launch_bsa_fwd_pair(mq, mk, mv, row_ptr, col_idx, o, lse, header, redo,
                                     shape->B * shape->H, shape->S, scale, g_wait_limit_ns.load(),
                                     st);
    if (e != cudaSuccess) return cuda_fail(e, "bsa_fwd pair launch");
    exact_only = 2;
  }
  cudaError_t e = nabla::launch_bsa_fwd(mq, mk, mv, row_ptr, col_idx, o, lse, header, redo,
                                        header + kHdrExactPasses, exact_only,
                                        shape->B * shape->H, shape->H,
                                        shape->S, shape->d, scale, raster ? 1 : 0,
                                        kv_raster ? 1 : 0, shape->Th, shape->Tw,
                                        g_wait_limit_ns.load(), st);
  if (e != cudaSuccess) return cuda_fail(e, "bsa_fwd launch");
  return NABLA_OK;
}

}  // namespace

namespace nabla {
// Lets other translation units of the library report through nabla_last_error().
void set_last_error(const std::string& msg) { g_last_error = msg; }
// bsa_fwd with an explicit header (status word, exact-pass counter) and
// exact-pass request word, for callers that run several forwards at once on
// one header (arguments already checked).
nabla_status fwd_with_header(const nabla_shape* shape, const void* q, const void* k,
                             const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                             float scale, void* o, float* lse, int* header, int* redo,
                             void* kv_scratch, nabla_stream_t stream, bool builder_list) {
  nabla_status s = check_shape(shape);
  if (s != NABLA_OK) return s;
  if (!q || !k || !v || !row_ptr || !col_idx || !o || !header || !redo)
    return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (kv_scratch != nullptr && (reinterpret_cast<uintptr_t>(kv_scratch) & 255u)))
    return fail(NABLA_ERR_INVALID_ARG, "q, k, v, o need 16-byte and K/V scratch 256-byte alignment");
  if (!std::isfinite(scale)) return fail(NABLA_ERR_INVALID_ARG, "scale must be finite");
  return run_fwd(shape, q, k, v, row_ptr, col_idx, scale, o, lse, header, redo, kv_scratch,
                 reinterpret_cast<cudaStream_t>(stream), pair_for(builder_list));
}
// The argument checks of a forward call (shape, token layout and tile grid,
// null pointers, 16-byte alignment of q, k, v, o, a finite scale), for entry
// points that must reject a call before they enqueue any work.
nabla_status check_fwd_args(const nabla_shape* shape, const void* q, const void* k,
                            const void* v, const void* o, float scale) {
  nabla_status s = check_shape(shape);
  if (s != NABLA_OK) return s;
  if (!q || !k || !v || !o) return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(NABLA_ERR_INVALID_ARG, "q, k, v, o need 16-byte alignment");
  if (!std::isfinite(scale)) return fail(NABLA_ERR_INVALID_ARG, "scale must be finite");
  return NABLA_OK;
}
// nabla_build_mask with its device status bits OR-ed into `status` instead of
// the workspace header (the host-buffer layer shares one header between the
// chunks it runs on two streams).
nabla_status build_mask_with_status(const nabla_shape* shape, const nabla_mask_params* params,
                                    const void* q, const void* k, uint8_t* mask_u8,
                                    int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                    int32_t* nnz_out, void* workspace, int* status,
                                    nabla_stream_t stream);
nabla_status build_mask_staged(const nabla_shape* shape, const nabla_mask_params* params,
                               const void* q, const void* k, uint8_t* mask_u8, int32_t* row_ptr,
                               int32_t* col_idx, int64_t col_capacity, int32_t* nnz_out,
                               void* workspace, int* status, nabla_stream_t stream,
                               cudaEvent_t* stage_events);
}  // namespace nabla

extern "C" {

int nabla_version(void) { return 230; }

const char* nabla_last_error(void) { return g_last_error.c_str(); }

void nabla_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns.store(ns == 0 ? kDefaultWaitLimitNs : ns);
}

void nabla_set_exact_reference(int on) { g_exact_reference.store(on ? 1 : 0); }

void nabla_set_pair_mode(int mode) { g_pair_mode.store(mode >= 0 && mode <= 2 ? mode : 0); }

int nabla_query_exact_passes(const void* workspace, nabla_stream_t stream) {
  if (workspace == nullptr) {
    g_last_error = "workspace is NULL";
    return -1;
  }
  int n = 0;
  cudaError_t e = cudaMemcpyAsync(&n, static_cast<const int*>(workspace) + kHdrExactPasses,
                                  sizeof(int), cudaMemcpyDeviceToHost,
                                  reinterpret_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) {
    g_last_error = std::string("nabla_query_exact_passes: ") + cudaGetErrorString(e);
    return -1;
  }
  return n;
}

size_t nabla_workspace_size(const nabla_shape* shape, int op) {
  if (check_shape(shape) != NABLA_OK) return 0;
  switch (op) {
    case NABLA_OP_BUILD_MASK: return build_layout(shape).total;
    case NABLA_OP_FWD: return kHeaderBytes + kv_scratch_bytes(shape);
    case NABLA_OP_FWD_WITH_MASK: return mask_layout(shape).total + kv_scratch_bytes(shape);
    case NABLA_OP_BWD: return bwd_layout(shape).total;
    case NABLA_OP_BUILD_XATTN: return xattn_layout(shape).total;
    default: g_last_error = "unknown op"; return 0;
  }
}

nabla_status nabla_workspace_init(void* workspace, nabla_stream_t stream) {
  if (workspace == nullptr) return fail(NABLA_ERR_INVALID_ARG, "workspace is NULL");
  cudaError_t e = cudaMemsetAsync(workspace, 0, kHeaderBytes, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "nabla_workspace_init");
  return NABLA_OK;
}

nabla_status nabla_query_status(void* workspace, nabla_stream_t stream) {
  if (workspace == nullptr) return fail(NABLA_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int word = 0;
  cudaError_t e = cudaMemcpyAsync(&word, workspace, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "nabla_query_status");
  e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "nabla_query_status");
  if (word & nabla::kStatusTimeout) return fail(NABLA_ERR_TIMEOUT, "a device pipeline wait ran out");
  if (word & nabla::kStatusCapacity) return fail(NABLA_ERR_CAPACITY, "kept blocks exceed col_capacity");
  if (word & nabla::kStatusBadIndex) return fail(NABLA_ERR_BAD_INDEX, "a CSR column index was out of range");
  return NABLA_OK;
}

nabla_status nabla_build_mask(const nabla_shape* shape, const nabla_mask_params* params,
                              const void* q, const void* k, uint8_t* mask_u8, int32_t* row_ptr,
                              int32_t* col_idx, int64_t col_capacity, int32_t* nnz_out,
                              void* workspace, nabla_stream_t stream) {
  CallRange range("nabla_build_mask");
  return nabla::build_mask_with_status(shape, params, q, k, mask_u8, row_ptr, col_idx, col_capacity,
                                       nnz_out, workspace, static_cast<int*>(workspace), stream);
}

nabla_status nabla_build_mask_stage_ms(const nabla_shape* shape, const nabla_mask_params* params,
                                       const void* q, const void* k, int32_t* row_ptr,
                                       int32_t* col_idx, int64_t col_capacity, int32_t* nnz_out,
                                       void* workspace, nabla_stream_t stream, float* ms_out) {
  if (ms_out == nullptr) return fail(NABLA_ERR_INVALID_ARG, "ms_out is NULL");
  cudaEvent_t ev[5] = {};
  cudaError_t e = cudaSuccess;
  int made = 0;
  for (; made < 5 && e == cudaSuccess; ++made) e = cudaEventCreate(&ev[made]);
  nabla_status s = NABLA_OK;
  if (e != cudaSuccess) {
    s = cuda_fail(e, "cudaEventCreate");
    --made;
  } else {
    s = nabla::build_mask_staged(shape, params, q, k, nullptr, row_ptr, col_idx, col_capacity,
                                 nnz_out, workspace, static_cast<int*>(workspace), stream, ev);
    if (s == NABLA_OK) {
      e = cudaEventSynchronize(ev[4]);
      for (int i = 0; i < 4 && e == cudaSuccess; ++i) e = cudaEventElapsedTime(&ms_out[i], ev[i], ev[i + 1]);
      if (e != cudaSuccess) s = cuda_fail(e, "stage timing");
    }
  }
  for (int i = 0; i < made; ++i) cudaEventDestroy(ev[i]);
  return s;
}

}  // extern "C"

namespace nabla {

// The mask build; stage_events (may be NULL): five events recorded on the
// stream before pooling, the reduced map, the selection, the compaction, and
// after it.
nabla_status build_mask_staged(const nabla_shape* shape, const nabla_mask_params* params,
                               const void* q, const void* k, uint8_t* mask_u8, int32_t* row_ptr,
                               int32_t* col_idx, int64_t col_capacity, int32_t* nnz_out,
                               void* workspace, int* status, nabla_stream_t stream,
                               cudaEvent_t* stage_events) {
  nabla_status s = check_shape(shape);
  if (s != NABLA_OK) return s;
  if (params == nullptr) return fail(NABLA_ERR_INVALID_ARG, "params is NULL");
  if (!(params->thr >= 0.f && params->thr <= 1.f))
    return fail(NABLA_ERR_UNSUPPORTED, "thr must lie in [0, 1]");
  if (params->topk < 0) return fail(NABLA_ERR_INVALID_ARG, "topk must be >= 0");
  if (params->use_sta && (params->wt < 0 || params->wh < 0 || params->ww < 0))
    return fail(NABLA_ERR_INVALID_ARG, "STA half-windows must be non-negative");
  if (shape->Tt <= 0 || shape->Th <= 0 || shape->Tw <= 0 ||
      static_cast<int64_t>(shape->Tt) * shape->Th * shape->Tw != shape->S / 64)
    return fail(NABLA_ERR_INVALID_ARG, "tile grid Tt*Th*Tw must equal S/64");
  if (!q || !k || !row_ptr || !workspace || !status) return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  if (col_capacity > 0 && col_idx == nullptr) return fail(NABLA_ERR_INVALID_ARG, "col_idx is NULL");
  if (col_capacity < 0) return fail(NABLA_ERR_INVALID_ARG, "col_capacity is negative");
  if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(NABLA_ERR_INVALID_ARG, "q, k need 16-byte and workspace 256-byte alignment");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const BuildLayout lay = build_layout(shape);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  double* qbar = reinterpret_cast<double*>(ws + lay.qbar);
  double* kbar = reinterpret_cast<double*>(ws + lay.kbar);
  double* L = reinterpret_cast<double*>(ws + lay.logits);
  uint32_t* bits = reinterpret_cast<uint32_t*>(ws + lay.bits);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + lay.counts);
  const int nb = shape->S / 64, BH = shape->B * shape->H;
  const int64_t nrows = static_cast<int64_t>(BH) * nb;
  auto mark = [&](int i) {
    return stage_events ? cudaEventRecord(stage_events[i], st) : cudaSuccess;
  };
  cudaError_t e = mark(0);
  if (e == cudaSuccess)
    e = nabla::launch_pool(q, k, qbar, kbar, nrows, shape->d, nb,
                           shape->layout == NABLA_LAYOUT_RASTER ? 1 : 0, shape->Th, shape->Tw, st);
  if (e != cudaSuccess) return cuda_fail(e, "pool launch");
  e = mark(1);
  if (e == cudaSuccess) e = nabla::launch_logits(qbar, kbar, L, BH, nb, shape->d, st);
  if (e != cudaSuccess) return cuda_fail(e, "logits launch");
  e = mark(2);
  if (e == cudaSuccess)
    e = nabla::launch_select(L, nrows, nb, params->thr, params->topk, params->use_sta ? 1 : 0,
                             params->wt, params->wh, params->ww, shape->Tt, shape->Th, shape->Tw,
                             bits, counts, mask_u8, st);
  if (e != cudaSuccess) return cuda_fail(e, "select launch");
  e = mark(3);
  if (e == cudaSuccess)
    e = nabla::launch_scan_fill(bits, counts, nrows, nb, row_ptr, col_idx, col_capacity, nnz_out,
                                status, st);
  if (e == cudaSuccess) e = mark(4);
  if (e != cudaSuccess) return cuda_fail(e, "scan/fill launch");
  return NABLA_OK;
}

nabla_status build_mask_with_status(const nabla_shape* shape, const nabla_mask_params* params,
                                    const void* q, const void* k, uint8_t* mask_u8,
                                    int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                    int32_t* nnz_out, void* workspace, int* status,
                                    nabla_stream_t stream) {
  return build_mask_staged(shape, params, q, k, mask_u8, row_ptr, col_idx, col_capacity, nnz_out,
                           workspace, status, stream, nullptr);
}

}  // namespace nabla

extern "C" {


nabla_status bsa_fwd(const nabla_shape* shape, const void* q, const void* k, const void* v,
                     const int32_t* row_ptr, const int32_t* col_idx, float scale, void* o,
                     float* lse, void* workspace, nabla_stream_t stream) {
  CallRange range("bsa_fwd");
  nabla_status s = check_shape(shape);
  if (s != NABLA_OK) return s;
  if (!q || !k || !v || !row_ptr || !col_idx || !o || !workspace)
    return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o))
    return fail(NABLA_ERR_INVALID_ARG, "q, k, v, o must be 16-byte aligned");
  if (shape->layout == NABLA_LAYOUT_RASTER && (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(NABLA_ERR_INVALID_ARG, "a raster-order workspace needs 256-byte alignment");
  if (!std::isfinite(scale)) return fail(NABLA_ERR_INVALID_ARG, "scale must be finite");
  void* kv_scratch = shape->layout == NABLA_LAYOUT_RASTER
                         ? static_cast<uint8_t*>(workspace) + kHeaderBytes : nullptr;
  return run_fwd(shape, q, k, v, row_ptr, col_idx, scale, o, lse, status_ptr(workspace),
                 status_ptr(workspace) + kHdrRedo, kv_scratch,
                 reinterpret_cast<cudaStream_t>(stream), pair_for(true));
}

nabla_status bsa_fwd_with_mask(const nabla_shape* shape, const void* q, const void* k,
                               const void* v, const uint8_t* mask_u8, float scale, void* o,
                               float* lse, void* workspace, nabla_stream_t stream) {
  CallRange range("bsa_fwd_with_mask");
  nabla_status s = check_shape(shape);
  if (s != NABLA_OK) return s;
  if (!q || !k || !v || !mask_u8 || !o || !workspace)
    return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(NABLA_ERR_INVALID_ARG, "q, k, v, o need 16-byte and workspace 256-byte alignment");
  if (!std::isfinite(scale)) return fail(NABLA_ERR_INVALID_ARG, "scale must be finite");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const MaskLayout lay = mask_layout(shape);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint32_t* bits = reinterpret_cast<uint32_t*>(ws + lay.bits);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + lay.counts);
  int32_t* row_ptr = reinterpret_cast<int32_t*>(ws + lay.row_ptr);
  int32_t* col_idx = reinterpret_cast<int32_t*>(ws + lay.col_idx);
  const int nb = shape->S / 64;
  const int64_t nrows = static_cast<int64_t>(shape->B) * shape->H * nb;
  const int64_t cap = nrows * nb;
  cudaError_t e = nabla::launch_mask_bits(mask_u8, nrows, nb, bits, counts, st);
  if (e != cudaSuccess) return cuda_fail(e, "mask_bits launch");
  e = nabla::launch_scan_fill(bits, counts, nrows, nb, row_ptr, col_idx, cap, nullptr,
                              status_ptr(workspace), st);
  if (e != cudaSuccess) return cuda_fail(e, "scan/fill launch");
  void* kv_scratch = shape->layout == NABLA_LAYOUT_RASTER ? ws + lay.total : nullptr;
  return run_fwd(shape, q, k, v, row_ptr, col_idx, scale, o, lse, status_ptr(workspace),
                 status_ptr(workspace) + kHdrRedo, kv_scratch, st, pair_for(false));
}

nabla_status nabla_reorder_tokens(const nabla_shape* shape, int direction, const void* src,
                                  void* dst, nabla_stream_t stream) {
  CallRange range("nabla_reorder_tokens");
  if (shape == nullptr) return fail(NABLA_ERR_INVALID_ARG, "shape is NULL");
  if (shape->B <= 0 || shape->H <= 0 || shape->d <= 0 || shape->Tt <= 0 || shape->Th <= 0 ||
      shape->Tw <= 0)
    return fail(NABLA_ERR_INVALID_ARG, "B, H, d and the tile grid must be positive");
  if (static_cast<int64_t>(shape->Tt) * shape->Th * shape->Tw * 64 != shape->S)
    return fail(NABLA_ERR_INVALID_ARG, "S must equal 64*Tt*Th*Tw");
  if ((shape->d * 2) % 16 != 0) return fail(NABLA_ERR_UNSUPPORTED, "d must be a multiple of 8");
  if (direction != NABLA_TO_TILE_MAJOR && direction != NABLA_TO_RASTER)
    return fail(NABLA_ERR_INVALID_ARG, "unknown direction");
  if (!src || !dst) return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  if (src == dst) return fail(NABLA_ERR_INVALID_ARG, "src and dst must not alias");
  if (!aligned16(src) || !aligned16(dst)) return fail(NABLA_ERR_INVALID_ARG, "src, dst need 16-byte alignment");
  const int64_t BH = static_cast<int64_t>(shape->B) * shape->H;
  if (BH * shape->Tt * shape->Th * shape->Tw >= (static_cast<int64_t>(1) << 31))
    return fail(NABLA_ERR_UNSUPPORTED, "B*H*S/64 must stay below 2^31");
  cudaError_t e = nabla::launch_reorder(src, dst, BH, shape->Tt, shape->Th, shape->Tw,
                                        shape->d * 2, direction == NABLA_TO_TILE_MAJOR ? 1 : 0,
                                        reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "reorder launch");
  return NABLA_OK;
}

nabla_status nabla_block_energy(const nabla_shape* shape, const void* q, const void* k,
                                const float* lse, const int32_t* row_ptr, const int32_t* col_idx,
                                float scale, float* energy, float* block_mass, void* workspace,
                                nabla_stream_t stream) {
  CallRange range("nabla_block_energy");
  nabla_status s = check_shape(shape);
  if (s != NABLA_OK) return s;
  if ((s = require_tile_major(shape)) != NABLA_OK) return s;
  if (!q || !k || !lse || !row_ptr || !col_idx || !energy || !workspace)
    return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k)) return fail(NABLA_ERR_INVALID_ARG, "q, k must be 16-byte aligned");
  if (!std::isfinite(scale)) return fail(NABLA_ERR_INVALID_ARG, "scale must be finite");
  const uint64_t rows = static_cast<uint64_t>(shape->B) * shape->H * shape->S;
  CUtensorMap mq, mk;
  if ((s = make_map(&mq, q, rows, shape->d)) != NABLA_OK) return s;
  if ((s = make_map(&mk, k, rows, shape->d)) != NABLA_OK) return s;
  if (!(scale > 0.f)) scale = 1.0f / std::sqrt(static_cast<float>(shape->d));
  cudaError_t e = nabla::launch_block_energy(mq, mk, row_ptr, col_idx, lse, energy, block_mass,
                                             status_ptr(workspace), shape->B * shape->H, shape->S,
                                             shape->d, scale, g_wait_limit_ns.load(),
                                             reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "block_energy launch");
  return NABLA_OK;
}

nabla_status nabla_calib_accumulate(const nabla_shape* shape, const float* energy, float eps,
                                    int32_t* votes, nabla_stream_t stream) {
  nabla_status s = check_shape(shape);
  if (s != NABLA_OK) return s;
  if (!(eps >= 0.f && eps <= 1.f)) return fail(NABLA_ERR_UNSUPPORTED, "eps must lie in [0, 1]");
  if (!energy || !votes) return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  const int nb = shape->S / 64;
  const int64_t nrows = static_cast<int64_t>(shape->B) * shape->H * nb;
  cudaError_t e = nabla::launch_calib_select(energy, nrows, nb, eps, votes,
                                             reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "calib select launch");
  return NABLA_OK;
}

nabla_status nabla_calib_finalize(const nabla_shape* shape, const int32_t* votes,
                                  int32_t min_votes, uint8_t* mask_u8, nabla_stream_t stream) {
  nabla_status s = check_shape(shape);
  if (s != NABLA_OK) return s;
  if (!votes || !mask_u8) return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  if (min_votes < 1) return fail(NABLA_ERR_INVALID_ARG, "min_votes must be at least 1");
  const int64_t nb = shape->S / 64;
  const int64_t n = static_cast<int64_t>(shape->B) * shape->H * nb * nb;
  cudaError_t e = nabla::launch_vote_mask(votes, n, min_votes, mask_u8,
                                          reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "vote mask launch");
  return NABLA_OK;
}

nabla_status bsa_bwd(const nabla_shape* shape, const void* q, const void* k, const void* v,
                     const void* o, const void* dout, const float* lse, const int32_t* row_ptr,
                     const int32_t* col_idx, float scale, void* dq, void* dk, void* dv,
                     void* workspace, nabla_stream_t stream) {
  CallRange range("bsa_bwd");
  nabla_status s = check_shape(shape);
  if (s != NABLA_OK) return s;
  if ((s = require_tile_major(shape)) != NABLA_OK) return s;
  if (!q || !k || !v || !o || !dout || !lse || !row_ptr || !col_idx || !dq || !dk || !dv ||
      !workspace)
    return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dout) ||
      !aligned16(lse) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(NABLA_ERR_INVALID_ARG,
                "tensors and lse need 16-byte and workspace 256-byte alignment");
  if (!std::isfinite(scale)) return fail(NABLA_ERR_INVALID_ARG, "scale must be finite");
  const uint64_t rows = static_cast<uint64_t>(shape->B) * shape->H * shape->S;
  CUtensorMap mq, mk, mv, mdo;
  if ((s = make_map(&mq, q, rows, shape->d)) != NABLA_OK) return s;
  if ((s = make_map(&mk, k, rows, shape->d)) != NABLA_OK) return s;
  if ((s = make_map(&mv, v, rows, shape->d)) != NABLA_OK) return s;
  if ((s = make_map(&mdo, dout, rows, shape->d)) != NABLA_OK) return s;
  if (!(scale > 0.f)) scale = 1.0f / std::sqrt(static_cast<float>(shape->d));
  const BwdLayout lay = bwd_layout(shape);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t e = nabla::launch_bsa_bwd(
      mq, mk, mv, mdo, o, dout, lse, row_ptr, col_idx, reinterpret_cast<float*>(ws + lay.dvec),
      reinterpret_cast<float*>(ws + lay.lse2), reinterpret_cast<uint32_t*>(ws + lay.colbits), dq, dk, dv, status_ptr(workspace),
      shape->B * shape->H, shape->S, shape->d, scale, g_wait_limit_ns.load(),
      reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "bsa_bwd launch");
  return NABLA_OK;
}

nabla_status nabla_build_mask_xattn(const nabla_shape* shape, const nabla_mask_params* params,
                                    int32_t stride, const void* q, const void* k, float* scores,
                                    uint8_t* mask_u8, int32_t* row_ptr, int32_t* col_idx,
                                    int64_t col_capacity, int32_t* nnz_out, void* workspace,
                                    nabla_stream_t stream) {
  CallRange range("nabla_build_mask_xattn");
  nabla_status s = check_shape(shape);
  if (s != NABLA_OK) return s;
  if ((s = require_tile_major(shape)) != NABLA_OK) return s;
  if (params == nullptr) return fail(NABLA_ERR_INVALID_ARG, "params is NULL");
  if (stride != 4 && stride != 8 && stride != 16)
    return fail(NABLA_ERR_UNSUPPORTED, "stride must be 4, 8 or 16");
  if (!(params->thr >= 0.f && params->thr <= 1.f))
    return fail(NABLA_ERR_UNSUPPORTED, "thr must lie in [0, 1]");
  if (params->topk < 0) return fail(NABLA_ERR_INVALID_ARG, "topk must be >= 0");
  if (params->use_sta && (params->wt < 0 || params->wh < 0 || params->ww < 0))
    return fail(NABLA_ERR_INVALID_ARG, "STA half-windows must be non-negative");
  if (params->use_sta && (shape->Tt <= 0 || shape->Th <= 0 || shape->Tw <= 0 ||
                          static_cast<int64_t>(shape->Tt) * shape->Th * shape->Tw != shape->S / 64))
    return fail(NABLA_ERR_INVALID_ARG, "the STA window needs a tile grid with Tt*Th*Tw = S/64");
  if (!q || !k || !row_ptr || !workspace) return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  if (col_capacity > 0 && col_idx == nullptr) return fail(NABLA_ERR_INVALID_ARG, "col_idx is NULL");
  if (col_capacity < 0) return fail(NABLA_ERR_INVALID_ARG, "col_capacity is negative");
  if (!aligned16(q) || !aligned16(k) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return fail(NABLA_ERR_INVALID_ARG, "q, k need 16-byte and workspace 256-byte alignment");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const XattnLayout lay = xattn_layout(shape);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* lse2 = reinterpret_cast<float*>(ws + lay.lse2);
  float* X = scores ? scores : reinterpret_cast<float*>(ws + lay.scores);
  uint32_t* bits = reinterpret_cast<uint32_t*>(ws + lay.bits);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + lay.counts);
  const int nb = shape->S / 64, BH = shape->B * shape->H;
  const int64_t nrows = static_cast<int64_t>(BH) * nb;
  const uint64_t groups = static_cast<uint64_t>(BH) * (shape->S / stride);
  CUtensorMap mq, mk;
  // Q' boxes of 128 strided rows, K' boxes of 256 (the scorer's query and key tiles)
  if ((s = make_map_strided(&mq, q, groups, stride, shape->d, 128)) != NABLA_OK) return s;
  if ((s = make_map_strided(&mk, k, groups, stride, shape->d, 256)) != NABLA_OK) return s;
  cudaError_t e = nabla::launch_xattn_scores(mq, mk, lse2, X, status_ptr(workspace), BH, shape->S,
                                             shape->d, stride, g_wait_limit_ns.load(), st);
  if (e != cudaSuccess) return cuda_fail(e, "xattn scores launch");
  // without the STA window the tile grid is not used (a 1 x 1 x nb grid stands in)
  const bool sta = params->use_sta != 0;
  e = nabla::launch_select_weights(X, nrows, nb, params->thr, params->topk, sta ? 1 : 0,
                                   params->wt, params->wh, params->ww, sta ? shape->Tt : nb,
                                   sta ? shape->Th : 1, sta ? shape->Tw : 1, bits, counts,
                                   mask_u8, st);
  if (e != cudaSuccess) return cuda_fail(e, "select launch");
  e = nabla::launch_scan_fill(bits, counts, nrows, nb, row_ptr, col_idx, col_capacity, nnz_out,
                              status_ptr(workspace), st);
  if (e != cudaSuccess) return cuda_fail(e, "scan/fill launch");
  return NABLA_OK;
}

nabla_status nabla_selftest_mma(int variant, const void* a, const void* b, float* c,
                                void* workspace, nabla_stream_t stream) {
  if (variant < 0 || variant > 3) return fail(NABLA_ERR_INVALID_ARG, "variant must be 0..3");
  if (!a || !b || !c || !workspace) return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(a) || !aligned16(b)) return fail(NABLA_ERR_INVALID_ARG, "a, b need 16-byte alignment");
  CUtensorMap ma, mb;
  nabla_status s;
  if ((s = make_map(&ma, a, 128, 128)) != NABLA_OK) return s;
  if ((s = make_map(&mb, b, 128, 128)) != NABLA_OK) return s;
  cudaError_t e = nabla::launch_mma_selftest(ma, mb, a, c, variant, status_ptr(workspace),
                                             g_wait_limit_ns.load(),
                                             reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return NABLA_OK;
}

nabla_status nabla_selftest_mma_pair(int variant, const void* a, const void* b, float* c,
                                     void* workspace, nabla_stream_t stream) {
  if (variant < 0 || variant > 1) return fail(NABLA_ERR_INVALID_ARG, "variant must be 0 or 1");
  if (!a || !b || !c || !workspace) return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  if (!aligned16(a) || !aligned16(b)) return fail(NABLA_ERR_INVALID_ARG, "a, b need 16-byte alignment");
  CUtensorMap ma, mb;
  nabla_status s;
  // variant 0: A [256][128], B [256][128]; variant 1: P [256][256] (read by
  // threads, not by a map), V [256][128]
  if ((s = make_map(&ma, variant == 0 ? a : b, 256, 128)) != NABLA_OK) return s;
  if ((s = make_map(&mb, b, 256, 128)) != NABLA_OK) return s;
  cudaError_t e = nabla::launch_mma_pair_selftest(ma, mb, a, c, variant, status_ptr(workspace),
                                                  g_wait_limit_ns.load(),
                                                  reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "pair selftest launch");
  return NABLA_OK;
}

}  // extern "C"
