// Measured fp64 FMA rate of the device: the denominator of the reduced map's
// roofline (the map is an fp64 product Qbar Kbar^T).  A grid of a few CTAs per
// SM runs independent fma chains; the rate is timed with CUDA events on the
// caller's stream.  No device memory is allocated: the result that keeps the
// chains alive goes to a file-scope device word, written only if the chains end
// on a value they cannot reach.
#include <cuda_runtime.h>

#include <string>

#include "../../include/nabla.h"

namespace nabla {
void set_last_error(const std::string& msg);
}

namespace {

constexpr int kChains = 8;
__device__ double g_fp64_sink;

__global__ void __launch_bounds__(256) fp64_fma_kernel(double a, double b, int iters) {
  double acc[kChains];
#pragma unroll
  for (int i = 0; i < kChains; ++i) acc[i] = threadIdx.x * 1e-3 + i;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kChains; ++i) acc[i] = fma(acc[i], a, b);
  }
  double s = 0.0;
#pragma unroll
  for (int i = 0; i < kChains; ++i) s += acc[i];
  if (s == -1.25e300) g_fp64_sink = s;
}

}  // namespace

extern "C" {

nabla_status nabla_selftest_fp64_tflops(nabla_stream_t stream, double* tflops_out) {
  if (tflops_out == nullptr) {
    nabla::set_last_error("tflops_out is NULL");
    return NABLA_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaEvent_t t0 = nullptr, t1 = nullptr;
  if (e == cudaSuccess) e = cudaEventCreate(&t0);
  if (e == cudaSuccess) e = cudaEventCreate(&t1);
  const int blocks = 8 * sms, threads = 256, iters = 1 << 14;
  float ms = 0.f;
  if (e == cudaSuccess) {
    // a multiplier just below 1 keeps the chains finite
    fp64_fma_kernel<<<blocks, threads, 0, st>>>(0.999999, 1e-9, iters / 8);   // warm-up
    e = cudaEventRecord(t0, st);
    if (e == cudaSuccess) fp64_fma_kernel<<<blocks, threads, 0, st>>>(0.999999, 1e-9, iters);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaEventRecord(t1, st);
    if (e == cudaSuccess) e = cudaEventSynchronize(t1);
    if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, t0, t1);
  }
  if (t0) cudaEventDestroy(t0);
  if (t1) cudaEventDestroy(t1);
  if (e != cudaSuccess) {
    nabla::set_last_error(std::string("nabla_selftest_fp64_tflops: ") + cudaGetErrorString(e));
    return NABLA_ERR_CUDA;
  }
  const double flops = 2.0 * kChains * static_cast<double>(iters) * blocks * threads;
  *tflops_out = flops / (static_cast<double>(ms) * 1e-3) / 1e12;
  return NABLA_OK;
}

}  // extern "C"
