// sqc_calibrate: salience-weighted quantizer calibration and code packing.
//
// SliM-LLM write-up (rkmt.cn), section 核心设计 / 组件二 SQC: inside each group a
// 3-sigma mask marks the scattered high-salience weights; salient and
// non-salient weights share one quantizer whose scale/zero are searched over
// n = 50 linear candidates tau in [1 - lambda, 1 + lambda], keeping the least
// l2 reconstruction error. The arXiv abstract (briefgpt.xyz page) adds that the
// error weighs element-wise salience.
//
// One warp owns one (row, group). Phase 1 (lanes over elements): load the
// group, moments, 3-sigma mask, min/max, element salience; stage w and delta
// in shared memory, the masked elements first (a stable partition, so each
// class is summed in column order without a per-element test). Phase 2
// (lanes over tau): lane l scores tau_l, tau_{l+32}, ... over all g elements;
// the code clamp runs on a 32-bit integer (round half to even, as rint). Every score is fp64 with the operation order of the
// definition (IEEE division and rint), so the chosen tau matches a float64
// evaluation except where two candidates' errors tie to rounding. Phase 3
// (lanes over elements): codes at the chosen tau, bytes to shared memory, then
// the group's g*b/32 little-endian words.
//
// The quotient w / s must be the correctly rounded one (the codes are
// rint(w / s + z0)). Per candidate, the lane takes y = 1/s with the IEEE
// division once, then per element Markstein's final division step (P.
// Markstein, IBM J. Res. Dev. 34(1), 1990): q0 = w*y, r = fma(-q0, s, w),
// q = fma(r, y, q0), which is the correctly rounded w/s when y = RN(1/s) and
// nothing overflows or underflows (weights and scales come from fp32 values).
//
// Cost: about 12 fp64 operations per (weight, tau); ALU-bound (the HBM traffic
// is ~4.3 bytes per weight).
#include <cstdint>
#include "common.cuh"

namespace slim {

constexpr int kSqcWarps = 8;

template <int G>
__global__ void __launch_bounds__(kSqcWarps * 32)
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
    const double qmax = (double)((1 << b) - 1);
    const int qmaxi = (1 << b) - 1;
    const float* wp = W + i * n + (int64_t)c * G;

    // ---- phase 1: moments, mask, range, salience
    double w[E];
    double sum = 0.0;
    double lo = 0.0, hi = 0.0;
#pragma unroll
    for (int r = 0; r < E; ++r) {
      w[r] = (double)wp[lane + 32 * r];
      sum += w[r];
      lo = r ? fmin(lo, w[r]) : w[r];
      hi = r ? fmax(hi, w[r]) : w[r];
    }
    sum = warp_sum(sum);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    const double mu = sum / (double)G;
    double var = 0.0;
#pragma unroll
    for (int r = 0; r < E; ++r) var += (w[r] - mu) * (w[r] - mu);
    var = warp_sum(var) / (double)G;
    const double sd = sqrt(var);
    const double tlo = mu - 3.0 * sd, thi = mu + 3.0 * sd;
    // stable partition in shared memory: the masked (salient) elements first,
    // each class in column order, so the tau loop sums each class without a
    // per-element test, in the same order as before
    bool mk[E];
    int ns = 0;
#pragma unroll
    for (int r = 0; r < E; ++r) {
      mk[r] = (w[r] < tlo) || (w[r] > thi);
      ns += __popc(__ballot_sync(0xffffffffu, mk[r]));
    }
    const int nu = G - ns;
    {
      const uint32_t lt = (1u << lane) - 1u;
      int before_m = 0;
#pragma unroll
      for (int r = 0; r < E; ++r) {
        const int j = lane + 32 * r;
        const uint32_t bm = __ballot_sync(0xffffffffu, mk[r]);
        const int pm = before_m + __popc(bm & lt);              // masked elements before j
        const int pos = mk[r] ? pm : ns + (j - pm);             // unmasked: after all masked
        const double hj = h[(int64_t)c * G + j];
        s_w[wib][pos] = w[r];
        s_d[wib][pos] = (w[r] * w[r]) / (hj * hj);
        before_m += __popc(bm);
      }
    }
    __syncwarp();

    const bool deg = (hi == lo);
    const double s0 = deg ? 1.0 : (hi - lo) / qmax;
    const double z0 = deg ? -lo : -lo / s0;

    // ---- phase 2: tau search, lanes over candidates
    double best_e = 0.0;
    int best_t = 0;
    if (!deg) {
      best_e = __longlong_as_double(0x7ff0000000000000ll);  // +inf
      best_t = n_tau;
      for (int t = lane; t < n_tau; t += 32) {
        const double tau = (n_tau == 1) ? 1.0 : (1.0 - lam) + ((2.0 * lam) * (double)t) / (double)(n_tau - 1);
        const double s = tau * s0;
        const double y = 1.0 / s;
        double es = 0.0, eu = 0.0;
        auto term = [&](int j) {
          const double wj = s_w[wib][j];
          const double q0 = wj * y;
          const double quot = fma(fma(-q0, s, wj), y, q0);   // = RN(wj / s)
          int qi = __double2int_rn(quot + z0);   // round half to even, as rint
          qi = qi < 0 ? 0 : (qi > qmaxi ? qmaxi : qi);
          const double q = (double)qi;
          const double e = wj - s * (q - z0);
          return s_d[wib][j] * (e * e);
        };
        for (int j = 0; j < ns; ++j) es += term(j);
#pragma unroll 4
        for (int j = ns; j < G; ++j) eu += term(j);
        double err = (nu > 0 ? eu / (double)nu : 0.0);
        if (ns > 0) err = err + es / (double)ns;
        if (err < best_e) { best_e = err; best_t = t; }
      }
      // warp argmin, ties to the smaller index
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double oe = __shfl_xor_sync(0xffffffffu, best_e, o);
        const int ot = __shfl_xor_sync(0xffffffffu, best_t, o);
        if (oe < best_e || (oe == best_e && ot < best_t)) { best_e = oe; best_t = ot; }
      }
    }
    const double tau_b = deg ? 1.0
                             : ((n_tau == 1) ? 1.0
                                             : (1.0 - lam) + ((2.0 * lam) * (double)best_t) / (double)(n_tau - 1));
    const double s_b = deg ? 1.0 : tau_b * s0;

    // ---- phase 3: codes and packing
#pragma unroll
    for (int r = 0; r < E; ++r) {
      const int j = lane + 32 * r;
      double q = 0.0;
      if (!deg) {
        q = rint(w[r] / s_b + z0);
        q = fmin(fmax(q, 0.0), qmax);
      }
      s_q[wib][j] = (uint8_t)q;
    }
    // word offset of this group inside its row: (G/32) * sum of earlier groups' bits
    int before = 0;
    for (int cc = lane; cc < c; cc += 32) before += bits[cc];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
    __syncwarp();
    const int nwords = G * b / 32;
    uint32_t* out = codes + i * row_words + (int64_t)(G / 32) * before;
    // an allocation that does not sum to k * avg_bits would overrun the row: write nothing past it
    if (lane < nwords && (int64_t)(G / 32) * before + nwords <= row_words) {
      const int pos0 = 32 * lane;
      const int j0 = pos0 / b, j1 = (pos0 + 31) / b;
      uint32_t word = 0;
      for (int j = j0; j <= j1 && j < G; ++j) {
        const int off = j * b - pos0;
        const uint64_t v = s_q[wib][j];
        word |= (off >= 0) ? (uint32_t)(v << off) : (uint32_t)(v >> (-off));
      }
      out[lane] = word;
    }
    if (lane == 0) {
      scale[i * k + c] = (float)s_b;
      zero[i * k + c] = (float)z0;
      if (tau_idx) tau_idx[i * k + c] = (uint8_t)best_t;
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
