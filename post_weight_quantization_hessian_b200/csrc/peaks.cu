// Measured fp64 rates of the current device, the roofline denominators of the
// fp64 stages (the inverse-Hessian factorization and the GPTQ update on the
// fp64 tensor cores; the SQC calibration on the fp64 FMA pipe). Each kernel
// keeps 8 independent accumulation chains per thread busy on every SM; the
// results go to a file-scope device variable so the work is not removed.
#include <cstdint>
#include <cuda_runtime.h>
#include "common.cuh"
#include "../../include/slim.h"

namespace slim {

static __device__ double g_peak_sink;

__global__ void __launch_bounds__(256) peak_dfma_kernel(int iters) {
  double a[8];
  const double b = 1.0000001, c = 0.999999;
#pragma unroll
  for (int i = 0; i < 8; ++i) a[i] = threadIdx.x * 1e-3 + i;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = fma(a[i], b, c);
  }
  double s = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += a[i];
  if (s == 12345.0) g_peak_sink = s;
}

__global__ void __launch_bounds__(256) peak_dmma_kernel(int iters) {
  double acc[8][2];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = 0.0;
  const double a = threadIdx.x * 1e-3, b = 1.0 + threadIdx.x * 1e-4;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
                   : "+d"(acc[i][0]), "+d"(acc[i][1])
                   : "d"(a), "d"(b));
  }
  double s = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) s += acc[i][0] + acc[i][1];
  if (s == 12345.0) g_peak_sink = s;
}

}  // namespace slim

using namespace slim;

extern "C" int slim_peak_fp64(double* dmma_tflops, double* dfma_tflops, void* stream) {
  if (!dmma_tflops || !dfma_tflops) return SLIM_EINVAL;
  int dev = 0, sms = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SLIM_ENODEV;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (major != 10) return SLIM_ENODEV;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaEvent_t e[2];
  if (cudaEventCreate(&e[0]) != cudaSuccess || cudaEventCreate(&e[1]) != cudaSuccess) return SLIM_ECUDA;
  const int grid = sms * 4, threads = 256;
  double best[2] = {0.0, 0.0};
  // 8 chains x iters per thread; a DFMA is 2 flops, an m8n8k4 MMA 2 * 8 * 8 * 4 per warp
  const int it_fma = 20000, it_mma = 4000;
  for (int rep = 0; rep < 3; ++rep) {
    for (int kind = 0; kind < 2; ++kind) {
      cudaEventRecord(e[0], s);
      if (kind == 0)
        peak_dmma_kernel<<<grid, threads, 0, s>>>(it_mma);
      else
        peak_dfma_kernel<<<grid, threads, 0, s>>>(it_fma);
      cudaEventRecord(e[1], s);
      if (cudaEventSynchronize(e[1]) != cudaSuccess) {
        cudaEventDestroy(e[0]);
        cudaEventDestroy(e[1]);
        return SLIM_ECUDA;
      }
      float ms = 0.f;
      cudaEventElapsedTime(&ms, e[0], e[1]);
      const double flops = kind == 0 ? (double)grid * (threads / 32) * it_mma * 8 * 2.0 * 8 * 8 * 4
                                     : (double)grid * threads * it_fma * 8 * 2.0;
      const double tf = flops / (ms * 1e-3) / 1e12;
      if (tf > best[kind]) best[kind] = tf;
    }
  }
  count_launches(12);
  cudaEventDestroy(e[0]);
  cudaEventDestroy(e[1]);
  *dmma_tflops = best[0];
  *dfma_tflops = best[1];
  return cudaGetLastError() == cudaSuccess ? SLIM_OK : SLIM_ECUDA;
}
