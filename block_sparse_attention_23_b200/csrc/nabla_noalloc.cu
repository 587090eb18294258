// bsa_fwd_with_mask_static: the static-mask attention forward for callers
// that cannot allocate device memory.
//
// Some hosts of this library run where cudaMalloc is off limits: a serving
// runtime that owns every byte of device memory through its own pool and
// forbids allocation on its hot path, a plugin invoked from inside another
// framework's CUDA-graph capture, or an embedded caller with a fixed memory
// budget decided at start-up.  Such callers cannot provide the workspace
// that bsa_fwd_with_mask needs for the block CSR it builds from the mask.
// This entry point takes its scratch from a fixed array in device memory
// that belongs to the library instead, so the caller passes only inputs and
// outputs.
//
// The array (kStaticScratchBytes, 32 MiB) lives on every device on which this
// entry point has run, until the process exits.  Shapes whose block CSR does
// not fit are rejected with NABLA_ERR_UNSUPPORTED.  All calls share the one
// array, so two calls whose work overlaps on the GPU (different streams, no
// ordering between them) race and corrupt each other; calls in one stream, or
// otherwise ordered, are fine.  The first call on a device looks up the
// array's device address (cudaGetSymbolAddress, once per device, with that
// device current); make that first call before any stream capture begins.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <string>

#include "../../include/nabla.h"

namespace nabla {
void set_last_error(const std::string& msg);
cudaError_t launch_mask_bits(const uint8_t* mask, int64_t nrows, int nb, uint32_t* bits,
                             int32_t* counts, cudaStream_t st);
cudaError_t launch_scan_fill(const uint32_t* bits, const int32_t* counts, int64_t nrows, int nb,
                             int32_t* row_ptr, int32_t* col_idx, int64_t capacity,
                             int32_t* nnz_out, int* status, cudaStream_t st);
nabla_status fwd_with_header(const nabla_shape* shape, const void* q, const void* k,
                             const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                             float scale, void* o, float* lse, int* header, int* redo,
                             void* kv_scratch, nabla_stream_t stream, bool builder_list);
nabla_status check_fwd_args(const nabla_shape* shape, const void* q, const void* k,
                            const void* v, const void* o, float scale);
}  // namespace nabla

namespace {

constexpr size_t kStaticScratchBytes = NABLA_STATIC_SCRATCH_BYTES;
constexpr size_t kHeader = 256;      // status word at offset 0, as in a caller workspace
constexpr int kMaxDevices = 64;

// The library-owned scratch.  Host code must not use this name as an address:
// on the host it is only a stand-in; the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

nabla_status fail(nabla_status s, const std::string& msg) {
  nabla::set_last_error(msg);   // reported by nabla_last_error()
  return s;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Device address of the scratch on the current device (looked up once per device).
nabla_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(NABLA_ERR_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(NABLA_ERR_UNSUPPORTED, "device ordinal above 63");
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(NABLA_ERR_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return NABLA_OK;
}

}  // namespace

extern "C" {

NABLA_API nabla_status bsa_fwd_with_mask_static(const nabla_shape* shape, const void* q,
                                                const void* k, const void* v,
                                                const uint8_t* mask_u8, float scale, void* o,
                                                float* lse, int32_t* status_out,
                                                nabla_stream_t stream) {
  // every argument check of the forward runs before anything is enqueued, so
  // a rejected call leaves the shared scratch untouched
  nabla_status s = nabla::check_fwd_args(shape, q, k, v, o, scale);
  if (s != NABLA_OK) return s;
  if (mask_u8 == nullptr) return fail(NABLA_ERR_INVALID_ARG, "null pointer");
  // block CSR of the mask, laid out as in a bsa_fwd_with_mask workspace
  const size_t nb = static_cast<size_t>(shape->S) / 64;
  const size_t rows = static_cast<size_t>(shape->B) * shape->H * nb, nw = (nb + 31) / 32;
  size_t off = kHeader;
  const size_t off_bits = off; off = align256(off + rows * nw * 4);
  const size_t off_counts = off; off = align256(off + rows * 4);
  const size_t off_row_ptr = off; off = align256(off + (rows + 1) * 4);
  const size_t off_col_idx = off; off = align256(off + rows * nb * 4);
  if (nb > 4096 || off > kStaticScratchBytes)
    return fail(NABLA_ERR_UNSUPPORTED,
                "shape needs " + std::to_string(off) + " bytes of scratch; the static scratch "
                "holds " + std::to_string(kStaticScratchBytes) + " (B*H*(S/64)^2 must stay "
                "below about 8.3 million blocks)");
  void* base = nullptr;
  s = scratch_address(&base);
  if (s != NABLA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  unsigned char* ws = static_cast<unsigned char*>(base);
  // the status word must start at zero; everything else is overwritten below
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int), st);
  if (e != cudaSuccess) return fail(NABLA_ERR_CUDA, std::string("cudaMemsetAsync: ") + cudaGetErrorString(e));
  uint32_t* bits = reinterpret_cast<uint32_t*>(ws + off_bits);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + off_counts);
  int32_t* row_ptr = reinterpret_cast<int32_t*>(ws + off_row_ptr);
  int32_t* col_idx = reinterpret_cast<int32_t*>(ws + off_col_idx);
  e = nabla::launch_mask_bits(mask_u8, static_cast<int64_t>(rows), static_cast<int>(nb), bits,
                              counts, st);
  if (e == cudaSuccess)
    e = nabla::launch_scan_fill(bits, counts, static_cast<int64_t>(rows), static_cast<int>(nb),
                                row_ptr, col_idx, static_cast<int64_t>(rows * nb), nullptr,
                                reinterpret_cast<int*>(ws), st);
  if (e != cudaSuccess) return fail(NABLA_ERR_CUDA, std::string("mask compaction: ") + cudaGetErrorString(e));
  // no room for tile-major K/V copies here: raster K and V are read by 5D boxes
  s = nabla::fwd_with_header(shape, q, k, v, row_ptr, col_idx, scale, o, lse,
                             reinterpret_cast<int*>(ws), reinterpret_cast<int*>(ws) + 1, nullptr,
                             stream, false);
  if (s != NABLA_OK) return s;   // the forward has set the message
  if (status_out != nullptr) {
    e = cudaMemcpyAsync(status_out, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return fail(NABLA_ERR_CUDA, std::string("status copy: ") + cudaGetErrorString(e));
  }
  return NABLA_OK;
}

}  // extern "C"
