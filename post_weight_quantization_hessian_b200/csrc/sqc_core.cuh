// One warp's salience-weighted quantizer calibration of one (row, group), and
// the packing of the group's codes: shared by the SQC kernel (the group's
// weights as they are) and the GPTQ kernel (the group's weights as the earlier
// columns' compensation has left them).
//
// SliM-LLM write-up (rkmt.cn), section 核心设计 / 组件二 SQC: inside each group a
// 3-sigma mask marks the scattered high-salience weights; salient and
// non-salient weights share one quantizer whose scale/zero are searched over
// n = 50 linear candidates tau in [1 - lambda, 1 + lambda], keeping the least
// l2 reconstruction error. The arXiv abstract (briefgpt.xyz page) adds that the
// error weighs element-wise salience.
//
// Lanes over elements (lane l holds elements l, l + 32, ... of the group):
// moments, 3-sigma mask, min/max, element salience; w and delta are staged in
// the warp's shared arrays, the masked elements first (a stable partition, so
// each class is summed in column order without a per-element test). Lanes over
// tau: lane l scores tau_l, tau_{l+32}, ... over all g elements; the code clamp
// runs on a 32-bit integer (round half to even, as rint). Every per-element
// step of a score is fp64 and rounded as the definition's expression is
// (correctly rounded quotient, separate products and sums, no fused
// multiply-add); the sums over elements run in column order within the masked
// and the unmasked class, which can differ from another evaluation's summation
// order in the last bits, so the chosen tau matches a float64 evaluation
// except where two candidates' errors tie to that level.
//
// The quotient w / s must be the correctly rounded one (the codes are
// rint(w / s + z0)). Per candidate, the lane takes y = 1/s with the IEEE
// division once, then per element Markstein's final division step (P.
// Markstein, IBM J. Res. Dev. 34(1), 1990): q0 = w*y, r = fma(-q0, s, w),
// q = fma(r, y, q0), which is the correctly rounded w/s when y = RN(1/s) and
// nothing overflows or underflows (weights and scales come from fp32 values).
#pragma once
#include <cstdint>
#include "common.cuh"

namespace slim {

struct SqcChoice {
  double s, z0;  // scale tau* s0 and zero-point z0 (s = 1, z0 = -lo for a group of equal values)
  int t;         // chosen tau index
};

// w: this lane's E = G / 32 elements (element lane + 32 r in w[r]); hg: h of the
// group's G columns; s_w, s_d: the warp's G-double shared arrays.
template <int G>
__device__ __forceinline__ SqcChoice sqc_choose(const double (&w)[G / 32], const double* __restrict__ hg, int b,
                                                double lam, int n_tau, double* s_w, double* s_d, int lane) {
  constexpr int E = G / 32;
  const double qmax = (double)((1 << b) - 1);
  const int qmaxi = (1 << b) - 1;
  double sum = 0.0, lo = 0.0, hi = 0.0;
#pragma unroll
  for (int r = 0; r < E; ++r) {
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
  // stable partition: the masked (salient) elements first, each class in column order
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
      const int pm = before_m + __popc(bm & lt);   // masked elements before j
      const int pos = mk[r] ? pm : ns + (j - pm);  // unmasked: after all masked
      const double hj = hg[j];
      s_w[pos] = w[r];
      s_d[pos] = (w[r] * w[r]) / (hj * hj);
      before_m += __popc(bm);
    }
  }
  __syncwarp();

  const bool deg = (hi == lo);
  const double s0 = deg ? 1.0 : (hi - lo) / qmax;
  const double z0 = deg ? -lo : -lo / s0;

  double best_e = 0.0;
  int best_t = 0;
  if (!deg) {
    best_e = __longlong_as_double(0x7ff0000000000000ll);  // +inf
    best_t = n_tau;
    // Two candidates per lane per pass (t0 = tb + lane, t1 = t0 + 32): their
    // error sums are independent chains over the same elements, so the fp64
    // add latency of one hides behind the other; each candidate's sum still
    // runs in column order within the masked and the unmasked class. A lane
    // without a second candidate (t1 >= n_tau) computes a discarded copy of
    // its first.
    const double step = (n_tau == 1) ? 0.0 : (2.0 * lam);
    for (int tb = 0; tb < n_tau; tb += 64) {
      const int t0 = tb + lane, t1 = t0 + 32;
      if (t0 >= n_tau) break;  // (n_tau <= 256: whole passes of the warp stay uniform until here)
      const bool two = t1 < n_tau;
      const double tau0 = (n_tau == 1) ? 1.0 : (1.0 - lam) + (step * (double)t0) / (double)(n_tau - 1);
      const double tau1 = two ? (1.0 - lam) + (step * (double)t1) / (double)(n_tau - 1) : tau0;
      const double sa = tau0 * s0, sb = tau1 * s0;
      const double ya = 1.0 / sa, yb = 1.0 / sb;
      double esa = 0.0, eua = 0.0, esb = 0.0, eub = 0.0;
      // each rounding step of the definition separately (the _rn intrinsics
      // keep the compiler from contracting a product and a sum into an fma,
      // which would round once where the definition rounds twice)
      auto term = [&](double wj, double dj, double s, double y) {
        const double q0 = __dmul_rn(wj, y);
        const double quot = fma(fma(-q0, s, wj), y, q0);   // = RN(wj / s)
        int qi = __double2int_rn(__dadd_rn(quot, z0));     // round half to even, as rint
        qi = qi < 0 ? 0 : (qi > qmaxi ? qmaxi : qi);
        const double q = (double)qi;
        const double e = __dsub_rn(wj, __dmul_rn(s, __dsub_rn(q, z0)));
        return __dmul_rn(dj, __dmul_rn(e, e));
      };
      for (int j = 0; j < ns; ++j) {
        const double wj = s_w[j], dj = s_d[j];
        esa = __dadd_rn(esa, term(wj, dj, sa, ya));
        esb = __dadd_rn(esb, term(wj, dj, sb, yb));
      }
#pragma unroll 2
      for (int j = ns; j < G; ++j) {
        const double wj = s_w[j], dj = s_d[j];
        eua = __dadd_rn(eua, term(wj, dj, sa, ya));
        eub = __dadd_rn(eub, term(wj, dj, sb, yb));
      }
      double erra = (nu > 0 ? eua / (double)nu : 0.0);
      if (ns > 0) erra = __dadd_rn(erra, esa / (double)ns);
      if (erra < best_e) { best_e = erra; best_t = t0; }
      if (two) {
        double errb = (nu > 0 ? eub / (double)nu : 0.0);
        if (ns > 0) errb = __dadd_rn(errb, esb / (double)ns);
        if (errb < best_e) { best_e = errb; best_t = t1; }
      }
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
  __syncwarp();
  return SqcChoice{deg ? 1.0 : tau_b * s0, z0, best_t};
}

// Code of one weight with a group's quantizer: clamp(rint(w / s + z0), 0, qmax),
// the quotient correctly rounded (IEEE division) and the sum rounded apart.
__device__ __forceinline__ int sqc_code(double w, double s, double z0, int qmaxi) {
  double q = rint(__dadd_rn(w / s, z0));
  q = fmin(fmax(q, 0.0), (double)qmaxi);
  return (int)q;
}

// The group's G codes (s_q, bytes in column order) packed little-endian into
// G * b / 32 words at word offset (G / 32) * (sum of the earlier groups' bits)
// of the row; a row whose allocation would overrun row_words gets nothing.
template <int G>
__device__ __forceinline__ void sqc_pack(const uint8_t* s_q, const uint8_t* __restrict__ bits, int c, int b,
                                         uint32_t* row_out, int64_t row_words, int lane) {
  int before = 0;
  for (int cc = lane; cc < c; cc += 32) before += bits[cc];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
  __syncwarp();
  const int nwords = G * b / 32;
  uint32_t* out = row_out + (int64_t)(G / 32) * before;
  if (lane < nwords && (int64_t)(G / 32) * before + nwords <= row_words) {
    const int pos0 = 32 * lane;
    const int j0 = pos0 / b, j1 = (pos0 + 31) / b;
    uint32_t word = 0;
    for (int j = j0; j <= j1 && j < G; ++j) {
      const int off = j * b - pos0;
      const uint64_t v = s_q[j];
      word |= (off >= 0) ? (uint32_t)(v << off) : (uint32_t)(v >> (-off));
    }
    out[lane] = word;
  }
  __syncwarp();
}

}  // namespace slim
