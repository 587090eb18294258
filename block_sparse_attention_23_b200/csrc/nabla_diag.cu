// Measured arithmetic rates of the device, the denominators of the mask
// build's compute-bound rooflines:
//   - fp64 FMA rate: the reduced map is an fp64 product Qbar Kbar^T;
//   - fp64 exponential rate: the selection forms one fp64 exp(L - max) per
//     entry of the map, its one transcendental step per entry, so entries per
//     second over this rate bounds how close it runs to its arithmetic;
//   - fp32 ex2.approx rate (the exponential unit): the block-energy kernel
//     takes one exponential per score of a kept block, 4,096 per block against
//     2*d*64*64 tensor FLOPs, so the exponential unit, not the tensor cores,
//     sets its floor.
// A grid of eight CTAs per SM runs independent chains; the rate is timed with
// CUDA events on the caller's stream after a shorter warm-up launch.  No
// device memory is allocated: the result that keeps the chains alive goes to a
// file-scope device word, written only if the chains end on a value they
// cannot reach.
#include <cuda_runtime.h>

#include <string>

#include "../../include/nabla.h"

namespace nabla {
void set_last_error(const std::string& msg);
}

namespace {

constexpr int kChains = 8;
constexpr int kDiagThreads = 256;
__device__ double g_fp64_sink;

__global__ void __launch_bounds__(kDiagThreads) fp64_fma_kernel(double a, double b, int iters) {
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

// x <- exp(-x) stays in [exp(-1), 1] from any start in [0, 1]
__global__ void __launch_bounds__(kDiagThreads) fp64_exp_kernel(int iters) {
  double x[kChains];
#pragma unroll
  for (int i = 0; i < kChains; ++i) x[i] = (threadIdx.x & 63) * (1.0 / 64) + i * (1.0 / 128);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kChains; ++i) x[i] = exp(-x[i]);
  }
  double s = 0.0;
#pragma unroll
  for (int i = 0; i < kChains; ++i) s += x[i];
  if (s == -1.25e300) g_fp64_sink = s;
}

// x <- 2^(-x) stays in [1/2, 1] from any start in [0, 1]
__global__ void __launch_bounds__(kDiagThreads) ex2_kernel(int iters) {
  float x[kChains];
#pragma unroll
  for (int i = 0; i < kChains; ++i) x[i] = (threadIdx.x & 63) * (1.f / 64) + i * (1.f / 128);
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < kChains; ++i) asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(x[i]) : "f"(-x[i]));
  }
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < kChains; ++i) s += x[i];
  if (s == -1.25e30f) g_fp64_sink = s;
}

// launch(iters) on the caller's stream: a warm-up with iters / 8, then the
// timed launch; returns the grid size and the elapsed milliseconds.
template <typename Launch>
cudaError_t time_chains(cudaStream_t st, int iters, Launch launch, int* blocks, float* ms) {
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaEvent_t t0 = nullptr, t1 = nullptr;
  if (e == cudaSuccess) e = cudaEventCreate(&t0);
  if (e == cudaSuccess) e = cudaEventCreate(&t1);
  *blocks = 8 * sms;
  if (e == cudaSuccess) {
    launch(*blocks, iters / 8);
    e = cudaEventRecord(t0, st);
    if (e == cudaSuccess) launch(*blocks, iters);
    if (e == cudaSuccess) e = cudaGetLastError();
    if (e == cudaSuccess) e = cudaEventRecord(t1, st);
    if (e == cudaSuccess) e = cudaEventSynchronize(t1);
    if (e == cudaSuccess) e = cudaEventElapsedTime(ms, t0, t1);
  }
  if (t0) cudaEventDestroy(t0);
  if (t1) cudaEventDestroy(t1);
  return e;
}

}  // namespace

extern "C" {

nabla_status nabla_selftest_fp64_tflops(nabla_stream_t stream, double* tflops_out) {
  if (tflops_out == nullptr) {
    nabla::set_last_error("tflops_out is NULL");
    return NABLA_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int iters = 1 << 14;
  int blocks = 0;
  float ms = 0.f;
  // a multiplier just below 1 keeps the chains finite
  const cudaError_t e = time_chains(st, iters, [&](int g, int n) {
    fp64_fma_kernel<<<g, kDiagThreads, 0, st>>>(0.999999, 1e-9, n);
  }, &blocks, &ms);
  if (e != cudaSuccess) {
    nabla::set_last_error(std::string("nabla_selftest_fp64_tflops: ") + cudaGetErrorString(e));
    return NABLA_ERR_CUDA;
  }
  const double flops = 2.0 * kChains * static_cast<double>(iters) * blocks * kDiagThreads;
  *tflops_out = flops / (static_cast<double>(ms) * 1e-3) / 1e12;
  return NABLA_OK;
}

nabla_status nabla_selftest_fp64_exp_rate(nabla_stream_t stream, double* gexp_out) {
  if (gexp_out == nullptr) {
    nabla::set_last_error("gexp_out is NULL");
    return NABLA_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int iters = 1 << 11;
  int blocks = 0;
  float ms = 0.f;
  const cudaError_t e = time_chains(st, iters, [&](int g, int n) {
    fp64_exp_kernel<<<g, kDiagThreads, 0, st>>>(n);
  }, &blocks, &ms);
  if (e != cudaSuccess) {
    nabla::set_last_error(std::string("nabla_selftest_fp64_exp_rate: ") + cudaGetErrorString(e));
    return NABLA_ERR_CUDA;
  }
  const double exps = static_cast<double>(kChains) * iters * blocks * kDiagThreads;
  *gexp_out = exps / (static_cast<double>(ms) * 1e-3) / 1e9;
  return NABLA_OK;
}

nabla_status nabla_selftest_ex2_rate(nabla_stream_t stream, double* gexp_out) {
  if (gexp_out == nullptr) {
    nabla::set_last_error("gexp_out is NULL");
    return NABLA_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int iters = 1 << 14;
  int blocks = 0;
  float ms = 0.f;
  const cudaError_t e = time_chains(st, iters, [&](int g, int n) {
    ex2_kernel<<<g, kDiagThreads, 0, st>>>(n);
  }, &blocks, &ms);
  if (e != cudaSuccess) {
    nabla::set_last_error(std::string("nabla_selftest_ex2_rate: ") + cudaGetErrorString(e));
    return NABLA_ERR_CUDA;
  }
  const double exps = static_cast<double>(kChains) * iters * blocks * kDiagThreads;
  *gexp_out = exps / (static_cast<double>(ms) * 1e-3) / 1e9;
  return NABLA_OK;
}

}  // extern "C"
