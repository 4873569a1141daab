// sqc_calibrate: salience-weighted quantizer calibration and code packing
// (SliM-LLM write-up, rkmt.cn, section 核心设计 / 组件二 SQC; the arXiv abstract
// on the briefgpt.xyz page: the error weighs element-wise salience).
//
// One warp owns one (row, group): the calibration itself (3-sigma mask, tau
// search, all fp64 with the definition's rounding steps) is sqc_choose in
// sqc_core.cuh; then lanes over elements form the codes at the chosen tau,
// bytes go to shared memory and the group's g*b/32 little-endian words out.
//
// Cost: about 12 fp64 operations per (weight, tau); ALU-bound (the HBM traffic
// is ~4.3 bytes per weight).
#include <cstdint>
#include "common.cuh"
#include "sqc_core.cuh"

namespace slim {

constexpr int kSqcWarps = 8;
// Three blocks per SM (24 warps, up to 85 registers a thread): with the
// thread count alone as the bound the compiler settled at 64 registers and
// spilled the two candidates' chains at groups of 64 and 128; with this bound
// they stay in registers (6 to 8% faster there, 1% at group 32; same results).
constexpr int kSqcBlocksPerSm = 3;

template <int G>
__global__ void __launch_bounds__(kSqcWarps * 32, kSqcBlocksPerSm)
sqc_kernel(const float* __restrict__ W, int64_t m, int64_t n, const double* __restrict__ h,
           const uint8_t* __restrict__ bits, int avg_bits, double lam, int n_tau,
           uint32_t* __restrict__ codes, float* __restrict__ scale, float* __restrict__ zero,
           uint8_t* __restrict__ tau_idx) {
  constexpr int E = G / 32;  // elements per lane
  __shared__ double s_w[kSqcWarps][G];
  __shared__ double s_d[kSqcWarps][G];
  __shared__ uint8_t s_q[kSqcWarps][G];

  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int64_t k = n / G;
  const int64_t pairs = m * k;
  const int64_t row_words = n * avg_bits / 32;

  for (int64_t pr = (int64_t)blockIdx.x * kSqcWarps + wib; pr < pairs; pr += (int64_t)gridDim.x * kSqcWarps) {
    const int64_t i = pr / k;
    const int c = (int)(pr - i * k);
    const int b = bits[c];
    const float* wp = W + i * n + (int64_t)c * G;
    double w[E];
#pragma unroll
    for (int r = 0; r < E; ++r) w[r] = (double)wp[lane + 32 * r];
    const SqcChoice ch = sqc_choose<G>(w, h + (int64_t)c * G, b, lam, n_tau, s_w[wib], s_d[wib], lane);
#pragma unroll
    for (int r = 0; r < E; ++r) s_q[wib][lane + 32 * r] = (uint8_t)sqc_code(w[r], ch.s, ch.z0, (1 << b) - 1);
    __syncwarp();
    sqc_pack<G>(s_q[wib], bits, c, b, codes + i * row_words, row_words, lane);
    if (lane == 0) {
      scale[i * k + c] = (float)ch.s;
      zero[i * k + c] = (float)ch.z0;
      if (tau_idx) tau_idx[i * k + c] = (uint8_t)ch.t;
    }
    __syncwarp();
  }
}

cudaError_t launch_sqc(const float* W, int64_t m, int64_t n, const double* h, const uint8_t* bits, int group,
                       int avg_bits, double lam, int n_tau, uint32_t* codes, float* scale, float* zero,
                       uint8_t* tau_idx, int num_sms, cudaStream_t st) {
  const int64_t pairs = m * (n / group);
  const int64_t need = (pairs + kSqcWarps - 1) / kSqcWarps;
  const int grid = (int)(need < (int64_t)num_sms * 8 ? need : (int64_t)num_sms * 8);
  if (grid <= 0) return cudaSuccess;
  switch (group) {
    case 32: sqc_kernel<32><<<grid, kSqcWarps * 32, 0, st>>>(W, m, n, h, bits, avg_bits, lam, n_tau, codes, scale, zero, tau_idx); break;
    case 64: sqc_kernel<64><<<grid, kSqcWarps * 32, 0, st>>>(W, m, n, h, bits, avg_bits, lam, n_tau, codes, scale, zero, tau_idx); break;
    case 128: sqc_kernel<128><<<grid, kSqcWarps * 32, 0, st>>>(W, m, n, h, bits, avg_bits, lam, n_tau, codes, scale, zero, tau_idx); break;
    default: return cudaErrorInvalidValue;
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace slim
