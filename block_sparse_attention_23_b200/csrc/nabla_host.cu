// Host-resident layer: one NABLA attention layer (mask build + block-sparse
// forward) whose inputs and outputs live in pinned host memory.  Heads are
// independent, so the layer runs in chunks of heads through a two-slot device
// pipeline: the host-to-device copies of chunk c+1 and the device-to-host
// copies of chunk c-1 run on their own streams while chunk c computes, and
// PCIe transfers hide behind the attention instead of adding to it.  The two
// slots compute on two streams (slot 0 on the caller's, slot 1 on a
// library-owned one), so that the next chunk's kernels take the SMs that the
// last wave of the current chunk's attention grid leaves idle; the forward is a
// single launch per chunk (a query tile that needs the exact-reference pass
// runs it inside the same kernel), so nothing of one chunk waits behind the
// other chunk's grid.  Plain cudaMemcpyAsync copies only; stream order is kept
// with events, and the caller's stream waits for the last output copies before
// the call's work is complete on it.
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/nabla.h"

namespace nabla {
void set_last_error(const std::string& msg);
nabla_status build_mask_with_status(const nabla_shape* shape, const nabla_mask_params* params,
                                    const void* q, const void* k, uint8_t* mask_u8,
                                    int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                    int32_t* nnz_out, void* workspace, int* status,
                                    nabla_stream_t stream);
nabla_status fwd_with_header(const nabla_shape* shape, const void* q, const void* k,
                             const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                             float scale, void* o, float* lse, int* header, int* redo,
                             void* kv_scratch, nabla_stream_t stream, bool builder_list);
}  // namespace nabla

namespace {

constexpr int kSlots = 2;

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

nabla_status fail(nabla_status s, const std::string& msg) {
  nabla::set_last_error(msg);
  return s;
}

nabla_status cuda_fail(cudaError_t e, const char* where) {
  nabla::set_last_error(std::string(where) + ": " + cudaGetErrorString(e));
  return NABLA_ERR_CUDA;
}

constexpr size_t kHeaderBytes = 256;   // the caller's status header

// Workspace: the status header, then per slot the chunk's mask-build
// workspace, its block CSR, Q, K, V, O (bf16) and LSE (fp32).
struct HostLayout {
  size_t build, row_ptr, col_idx, q, k, v, o, lse;   // offsets inside a slot
  size_t slot_bytes, total;
  int64_t cap;                                       // col_idx capacity
};

HostLayout host_layout(const nabla_shape* s, int hc) {
  nabla_shape cs = *s;
  cs.B = 1;
  cs.H = hc;
  HostLayout l;
  const size_t nb = s->S / 64;
  const size_t tensor = align256(static_cast<size_t>(hc) * s->S * s->d * 2);
  size_t off = 0;
  l.build = off; off = align256(off + nabla_workspace_size(&cs, NABLA_OP_BUILD_MASK));
  l.row_ptr = off; off = align256(off + (static_cast<size_t>(hc) * nb + 1) * 4);
  l.cap = static_cast<int64_t>(hc) * nb * nb;
  l.col_idx = off; off = align256(off + static_cast<size_t>(l.cap) * 4);
  l.q = off; off += tensor;
  l.k = off; off += tensor;
  l.v = off; off += tensor;
  l.o = off; off += tensor;
  l.lse = off; off = align256(off + static_cast<size_t>(hc) * s->S * 4);
  l.slot_bytes = off;
  l.total = kHeaderBytes + kSlots * off;
  return l;
}

// Chunk sizes (heads) of one call.  The first chunk's input copy and the last
// chunk's output copy overlap nothing, so the schedule ramps up (1, 2, 4, ...
// heads: each copy takes about half the next chunk's compute at the PCIe and
// attention rates of one layer) and ends on a chunk of a quarter of the
// largest; the chunks between share the rest evenly, none above max_heads.
std::vector<int> chunk_schedule(int64_t heads, int max_heads) {
  std::vector<int> sizes;
  int64_t rem = heads;
  for (int64_t s = 1; s < max_heads && rem > 0; s *= 2) {
    const int64_t t = std::min(s, rem);
    sizes.push_back(static_cast<int>(t));
    rem -= t;
  }
  const int64_t last = std::max(1, max_heads / 4);
  const int64_t tail = rem > last ? last : 0;
  const int64_t mid = rem - tail;
  if (mid > 0) {
    const int64_t n = (mid + max_heads - 1) / max_heads;
    for (int64_t i = 0; i < n; ++i) sizes.push_back(static_cast<int>(mid / n + (i < mid % n ? 1 : 0)));
  }
  if (tail > 0) sizes.push_back(static_cast<int>(tail));
  return sizes;
}

// Streams and events reused across calls (one set per device, created once).
struct PipeRes {
  cudaStream_t h2d = nullptr, d2h = nullptr, comp1 = nullptr;   // comp1: slot 1's compute
  cudaEvent_t qk_ready[kSlots] = {}, in_ready[kSlots] = {}, in_free[kSlots] = {},
              out_ready[kSlots] = {}, out_free[kSlots] = {};
  cudaEvent_t join[3] = {};   // a failed call: the caller's stream waits for the other streams
  bool ok = false;
};

void release(PipeRes& r) {
  for (cudaStream_t* p : {&r.h2d, &r.d2h, &r.comp1})
    if (*p) { cudaStreamDestroy(*p); *p = nullptr; }
  for (int i = 0; i < kSlots; ++i)
    for (cudaEvent_t* p : {&r.qk_ready[i], &r.in_ready[i], &r.in_free[i], &r.out_ready[i],
                           &r.out_free[i]})
      if (*p) { cudaEventDestroy(*p); *p = nullptr; }
  for (cudaEvent_t& ev : r.join)
    if (ev) { cudaEventDestroy(ev); ev = nullptr; }
}
constexpr int kMaxDevices = 64;
std::mutex g_mutex;
PipeRes g_res[kMaxDevices];

nabla_status resources(PipeRes** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(NABLA_ERR_UNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lock(g_mutex);
  PipeRes& r = g_res[dev];
  if (!r.ok) {
    e = cudaStreamCreateWithFlags(&r.h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&r.d2h, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&r.comp1, cudaStreamNonBlocking);
    for (int i = 0; i < kSlots && e == cudaSuccess; ++i) {
      e = cudaEventCreateWithFlags(&r.qk_ready[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r.in_ready[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r.in_free[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r.out_ready[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r.out_free[i], cudaEventDisableTiming);
    }
    for (int i = 0; i < 3 && e == cudaSuccess; ++i)
      e = cudaEventCreateWithFlags(&r.join[i], cudaEventDisableTiming);
    if (e != cudaSuccess) {
      release(r);
      return cuda_fail(e, "pipeline streams/events");
    }
    r.ok = true;
  }
  *out = &r;
  return NABLA_OK;
}

}  // namespace

extern "C" {

NABLA_API int64_t nabla_layer_host_chunks(int64_t heads, int heads_per_chunk, int32_t* sizes,
                                          int64_t capacity) {
  if (heads <= 0 || heads_per_chunk <= 0) return 0;
  const std::vector<int> v = chunk_schedule(heads, heads_per_chunk);
  if (sizes != nullptr)
    for (size_t i = 0; i < v.size() && static_cast<int64_t>(i) < capacity; ++i) sizes[i] = v[i];
  return static_cast<int64_t>(v.size());
}

NABLA_API size_t nabla_layer_host_workspace_size(const nabla_shape* shape, int heads_per_chunk) {
  if (shape == nullptr || heads_per_chunk <= 0) return 0;
  if (nabla_workspace_size(shape, NABLA_OP_BUILD_MASK) == 0) return 0;   // shape rejected
  return host_layout(shape, heads_per_chunk).total;
}

NABLA_API nabla_status nabla_layer_host(const nabla_shape* shape, const nabla_mask_params* params,
                                        const void* q_host, const void* k_host,
                                        const void* v_host, void* o_host, float* lse_host,
                                        int heads_per_chunk, void* workspace,
                                        nabla_stream_t stream) {
  if (shape == nullptr || params == nullptr) return fail(NABLA_ERR_INVALID_ARG, "null shape or params");
  if (heads_per_chunk <= 0) return fail(NABLA_ERR_INVALID_ARG, "heads_per_chunk must be positive");
  if (!q_host || !k_host || !v_host || !o_host || !lse_host || !workspace)
    return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  if (nabla_workspace_size(shape, NABLA_OP_BUILD_MASK) == 0)
    return fail(NABLA_ERR_INVALID_ARG, std::string("shape rejected: ") + nabla_last_error());
  if (shape->layout != NABLA_LAYOUT_TILE_MAJOR)
    return fail(NABLA_ERR_UNSUPPORTED, "nabla_layer_host takes tile-major tokens");
  if (reinterpret_cast<uintptr_t>(workspace) & 255u)
    return fail(NABLA_ERR_INVALID_ARG, "workspace needs 256-byte alignment");
  // every check the chunks' calls make, before any copy is queued: a call that
  // fails later must not leave copies of the caller's buffers in flight
  if (!(params->thr >= 0.f && params->thr <= 1.f))
    return fail(NABLA_ERR_UNSUPPORTED, "thr must lie in [0, 1]");
  if (params->topk < 0) return fail(NABLA_ERR_INVALID_ARG, "topk must be >= 0");
  if (params->use_sta && (params->wt < 0 || params->wh < 0 || params->ww < 0))
    return fail(NABLA_ERR_INVALID_ARG, "STA half-windows must be non-negative");
  if (shape->Tt <= 0 || shape->Th <= 0 || shape->Tw <= 0 ||
      static_cast<int64_t>(shape->Tt) * shape->Th * shape->Tw != shape->S / 64)
    return fail(NABLA_ERR_INVALID_ARG, "tile grid Tt*Th*Tw must equal S/64");
  PipeRes* r = nullptr;
  nabla_status s = resources(&r);
  if (s != NABLA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t BH = static_cast<int64_t>(shape->B) * shape->H;
  const int hc = static_cast<int>(heads_per_chunk < BH ? heads_per_chunk : BH);
  const HostLayout lay = host_layout(shape, hc);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws);
  const std::vector<int> sizes = chunk_schedule(BH, hc);
  const int64_t nchunks = static_cast<int64_t>(sizes.size());
  // the other streams start after the work already queued on the caller's stream
  cudaEvent_t start = r->out_free[0];
  cudaError_t e;
  if ((e = cudaEventRecord(start, st)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(r->h2d, start, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(r->d2h, start, 0)) != cudaSuccess ||
      (e = cudaStreamWaitEvent(r->comp1, start, 0)) != cudaSuccess)
    return cuda_fail(e, "pipeline start");
  const nabla_status result = [&]() -> nabla_status {
  int64_t h0 = 0;
  for (int64_t c = 0; c < nchunks; h0 += sizes[c], ++c) {
    const int slot = static_cast<int>(c % kSlots);
    const int h = sizes[c];
    cudaStream_t cs = slot == 0 ? st : r->comp1;
    const size_t tbytes = static_cast<size_t>(h) * shape->S * shape->d * 2;
    const size_t lbytes = static_cast<size_t>(h) * shape->S * 4;
    const size_t toff = static_cast<size_t>(h0) * shape->S * shape->d * 2;
    const size_t loff = static_cast<size_t>(h0) * shape->S * 4;
    uint8_t* sb = ws + kHeaderBytes + slot * lay.slot_bytes;
    void* dq = sb + lay.q;
    void* dk = sb + lay.k;
    void* dv = sb + lay.v;
    void* dout = sb + lay.o;
    float* dlse = reinterpret_cast<float*>(sb + lay.lse);
    int32_t* row_ptr = reinterpret_cast<int32_t*>(sb + lay.row_ptr);
    int32_t* col_idx = reinterpret_cast<int32_t*>(sb + lay.col_idx);
    // inputs of chunk c into the slot, once chunk c-2 has finished reading it
    if (c >= kSlots && (e = cudaStreamWaitEvent(r->h2d, r->in_free[slot], 0)) != cudaSuccess)
      return cuda_fail(e, "h2d wait");
    if ((e = cudaMemcpyAsync(dq, static_cast<const uint8_t*>(q_host) + toff, tbytes,
                             cudaMemcpyHostToDevice, r->h2d)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dk, static_cast<const uint8_t*>(k_host) + toff, tbytes,
                             cudaMemcpyHostToDevice, r->h2d)) != cudaSuccess ||
        (e = cudaEventRecord(r->qk_ready[slot], r->h2d)) != cudaSuccess ||
        (e = cudaMemcpyAsync(dv, static_cast<const uint8_t*>(v_host) + toff, tbytes,
                             cudaMemcpyHostToDevice, r->h2d)) != cudaSuccess ||
        (e = cudaEventRecord(r->in_ready[slot], r->h2d)) != cudaSuccess)
      return cuda_fail(e, "h2d copy");
    // the mask of chunk c once its Q and K are in and chunk c-2's outputs have
    // left the slot; its attention once V is in as well
    if ((e = cudaStreamWaitEvent(cs, r->qk_ready[slot], 0)) != cudaSuccess)
      return cuda_fail(e, "compute wait");
    if (c >= kSlots && (e = cudaStreamWaitEvent(cs, r->out_free[slot], 0)) != cudaSuccess)
      return cuda_fail(e, "compute wait");
    nabla_shape chunk = *shape;
    chunk.B = 1;
    chunk.H = h;
    nabla_stream_t ns = reinterpret_cast<nabla_stream_t>(cs);
    s = nabla::build_mask_with_status(&chunk, params, dq, dk, nullptr, row_ptr, col_idx, lay.cap,
                                      nullptr, sb + lay.build, status, ns);
    if (s != NABLA_OK) return s;
    if ((e = cudaStreamWaitEvent(cs, r->in_ready[slot], 0)) != cudaSuccess)
      return cuda_fail(e, "compute wait");
    // the forward reports into the shared header, with the slot's own
    // exact-pass request word (header word 4 + slot)
    s = nabla::fwd_with_header(&chunk, dq, dk, dv, row_ptr, col_idx, 0.f, dout, dlse, status,
                               status + 4 + slot, nullptr, ns, true);
    if (s != NABLA_OK) return s;
    if ((e = cudaEventRecord(r->in_free[slot], cs)) != cudaSuccess ||
        (e = cudaEventRecord(r->out_ready[slot], cs)) != cudaSuccess)
      return cuda_fail(e, "compute record");
    // outputs of chunk c back to the host
    if ((e = cudaStreamWaitEvent(r->d2h, r->out_ready[slot], 0)) != cudaSuccess ||
        (e = cudaMemcpyAsync(static_cast<uint8_t*>(o_host) + toff, dout, tbytes,
                             cudaMemcpyDeviceToHost, r->d2h)) != cudaSuccess ||
        (e = cudaMemcpyAsync(reinterpret_cast<uint8_t*>(lse_host) + loff, dlse, lbytes,
                             cudaMemcpyDeviceToHost, r->d2h)) != cudaSuccess ||
        (e = cudaEventRecord(r->out_free[slot], r->d2h)) != cudaSuccess)
      return cuda_fail(e, "d2h copy");
  }
  // the call is complete on the caller's stream once the last outputs landed
  // (each output copy follows its chunk's compute)
  for (int i = 0; i < kSlots && i < nchunks; ++i)
    if ((e = cudaStreamWaitEvent(st, r->out_free[i], 0)) != cudaSuccess)
      return cuda_fail(e, "final wait");
  return NABLA_OK;
  }();
  if (result != NABLA_OK) {
    // whatever was queued before the failure is ordered before later work on
    // the caller's stream, so the caller's buffers are not in use once it syncs
    const cudaStream_t others[3] = {r->h2d, r->d2h, r->comp1};
    for (int i = 0; i < 3; ++i)
      if (cudaEventRecord(r->join[i], others[i]) == cudaSuccess)
        cudaStreamWaitEvent(st, r->join[i], 0);
  }
  return result;
}

}  // extern "C"
