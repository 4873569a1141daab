// sba_search: salience-determined bit allocation (SliM-LLM write-up, rkmt.cn,
// section 组件一 SBA; atlas.scime.ai summary, section Approach).
//
// Candidate p promotes the p most salient groups to b+1 bits and demotes the p
// least salient to b-1 bits, p = 0 .. k/2, and is scored by
//   KL_p = mean_t KL(softmax(y_t) || softmax(yhat_t)),  y = X W^T, yhat = X W_p^T,
// W_p the per-group min-max round-to-nearest dequantization under that
// allocation. p* = the smallest p with the least KL.
//
// How all candidates are scored in one pass
// -----------------------------------------
// Write yhat_p = y + d_p with d_p = X (W_p - W)^T. Candidate p differs from p-1
// in two groups only (the p-th most salient goes b -> b+1, the p-th least
// salient b -> b-1), so
//   d_0 = X E0^T,                        E0 = W^(b) - W
//   d_p = d_{p-1} + X_{c+} Dp_{c+}^T + X_{c-} Dm_{c-}^T,
//                                        Dp = W^(b+1) - W^(b), Dm = W^(b-1) - W^(b)
// (the same sum, regrouped). Per token tile (128 tokens) and output tile (128
// outputs), the tensor cores build y and d_0 in tensor memory (TMEM) from the
// full K = n contraction, then add the two changed groups' K = 2g slices for
// every further p. After each step the epilogue reads d_p from TMEM and
// accumulates the softmax statistics. d carries the quantization error
// directly (not as a difference of two large products).
//
// Operands. X is fp16: converted exactly from bf16, or split into a high and a
// low fp16 part when it is fp32. Each weight-side array (W, E0, Dp, Dm) is
// scaled by 2^8 (exact; keeps small entries out of fp16 subnormals) and stored
// as an fp16 pair, v 2^8 = hi + lo with hi = RN16(v 2^8), lo = RN16(v 2^8 - hi):
// 22 significant bits instead of fp16's 11. A single fp16 copy of the weight
// side moves the output KL by up to several 1e-5 on layers with clustered
// activation outliers (its rounding error in y = X W^T is largest exactly
// where the outlier channels meet the salient weights); the pair removes that
// term. Every K box is therefore contracted as sub-chunks that share the X
// box: (X, hi) and (X, lo) for bf16 X; (X_hi, hi), (X_lo, hi), (X_hi, lo) for
// fp32 X (X_lo lo, about 2^-22 of the product, is left out). The fp32
// accumulators are scaled back by 2^-8. Executed tensor-core work:
// nsub (2Nnm (y) + 2Nnm (d_0) + (P-1) 4Ngm (updates)), nsub = 2 or 3, instead
// of P 2Nnm for one dequant-GEMM per candidate.
//
// KL from running sums, per token t and output range (with e_y = exp(y - M)):
//   S_y = sum e_y, S_q = sum e_y exp(d), A = sum e_y d
//   KL_t = log(S_q / S_y) - A / S_y        (= lse(y + d) - lse(y) - E_P[d])
// The epilogue keeps e_y in TMEM in place of y after the first step, so later
// steps need one exp per element.
//
// Kernels
//   sba_prep       warp per (row, group): RTN at b-1, b, b+1 in fp64 (the
//                  definition's operation order); writes the fp16 hi/lo pairs
//                  of 2^8 W, E0, Dp, Dm
//   x_to_f16       bf16 X -> fp16 (exact in fp16's normal range)
//   x_split        fp32 X: X ~ X_hi + X_lo as two fp16 halves of X_cat
//   sba_score      persistent tcgen05 kernel (below)
//   sba_merge      per token: merges the output-tile partials in fp64 -> KL_t,
//                  sums per token tile
//   sba_final      KL_p = sum / N, p* = first argmin, bits
#include <cstdint>
#include <cstdlib>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include "common.cuh"
#include "tmap.h"

namespace slim {

// ---------------------------------------------------------------- prep
constexpr float kOpScale = 256.0f;          // weight-side operands are stored x 2^8
constexpr float kOpUnscale = 1.0f / 256.0f;
constexpr float kHalfMax = 65504.0f;
constexpr int kStatusRange = kStatusRangeCode;

__device__ __forceinline__ __half to_half_checked(float v, DevStatus* st, int where) {
  if (!(fabsf(v) <= kHalfMax)) record_failure(st, kStatusRange, where);
  return __float2half_rn(v);
}

// v = hi + lo as two fp16 values (hi = RN16(v), lo = RN16(v - hi); v - hi is
// exact in fp64), hi range-checked.
__device__ __forceinline__ void split_half(double v, DevStatus* st, int where, __half& hi, __half& lo) {
  if (!(fabs(v) <= (double)kHalfMax)) record_failure(st, kStatusRange, where);
  hi = __double2half(v);
  lo = __double2half(v - (double)__half2float(hi));
}

// Weight-side operands. W is read as float4: a lane holds 4 consecutive
// weights, a group of G spans G/4 adjacent lanes (G divides 128 and n, so a
// group never leaves its lanes or its row). Per group: fp32 min/max, then per
// level b-1, b, b+1 the fp64 min-max RTN value. Each output array is row-major
// with rows of 2 npad fp16 values: the hi parts in columns [0, npad), the lo
// parts in [npad, 2 npad); a lane writes one 8-byte word to each half
// (rs2 = 2 npad / 4 and lo2 = npad / 4 in those words).
template <int G>
__global__ void __launch_bounds__(256) sba_prep_kernel(const float4* __restrict__ W, int64_t total4, int64_t n4,
                                                       int64_t rs2, int64_t lo2, int avg_bits,
                                                       uint2* __restrict__ Wb, uint2* __restrict__ E0,
                                                       uint2* __restrict__ Dp, uint2* __restrict__ Dm,
                                                       DevStatus* st) {
  constexpr int LPG = G / 4;  // lanes per group
  const int lane = threadIdx.x & 31;
  const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5) * 32;
  for (int64_t base = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * 32; base < total4;
       base += wstride) {
    const int64_t e = base + lane;
    const bool on = e < total4;  // whole groups are on or off together (the total is a multiple of G)
    const float4 v4 = on ? W[e] : make_float4(0.f, 0.f, 0.f, 0.f);
    const float w[4] = {v4.x, v4.y, v4.z, v4.w};
    float lo = fminf(fminf(w[0], w[1]), fminf(w[2], w[3]));
    float hi = fmaxf(fmaxf(w[0], w[1]), fmaxf(w[2], w[3]));
#pragma unroll
    for (int o = LPG / 2; o > 0; o >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    }
    if (!on) continue;
    const double dlo = lo, dhi = hi;
    const bool deg = (dhi == dlo);
    double wh[3][4];
#pragma unroll
    for (int l = 0; l < 3; ++l) {
      const int b = avg_bits - 1 + l;
      const double qmax = (double)((1 << b) - 1);
      const double s0 = deg ? 1.0 : (dhi - dlo) / qmax;
      const double z0 = deg ? -dlo : -dlo / s0;
      // w / s0 correctly rounded from one IEEE reciprocal and Markstein's final
      // division step (P. Markstein, IBM J. Res. Dev. 34(1), 1990): exact while
      // nothing overflows or underflows, which fp32 weights and scales ensure
      const double y = 1.0 / s0;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const double wd = w[r];
        const double q0 = wd * y;
        double q = rint(fma(fma(-q0, s0, wd), y, q0) + z0);
        q = fmin(fmax(q, 0.0), qmax);
        wh[l][r] = deg ? wd : s0 * (q - z0);
      }
    }
    __half h0[4], h1[4], h2[4], h3[4], l0[4], l1[4], l2[4], l3[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const double wd = w[r];
      split_half(wd * (double)kOpScale, st, 300, h0[r], l0[r]);
      split_half((wh[1][r] - wd) * (double)kOpScale, st, 301, h1[r], l1[r]);
      split_half((wh[2][r] - wh[1][r]) * (double)kOpScale, st, 302, h2[r], l2[r]);
      split_half((wh[0][r] - wh[1][r]) * (double)kOpScale, st, 303, h3[r], l3[r]);
    }
    const int64_t row = e / n4;
    const int64_t o = row * rs2 + (e - row * n4);
    Wb[o] = *reinterpret_cast<const uint2*>(h0);
    E0[o] = *reinterpret_cast<const uint2*>(h1);
    Dp[o] = *reinterpret_cast<const uint2*>(h2);
    Dm[o] = *reinterpret_cast<const uint2*>(h3);
    Wb[o + lo2] = *reinterpret_cast<const uint2*>(l0);
    E0[o + lo2] = *reinterpret_cast<const uint2*>(l1);
    Dp[o + lo2] = *reinterpret_cast<const uint2*>(l2);
    Dm[o + lo2] = *reinterpret_cast<const uint2*>(l3);
  }
}

// bf16 -> fp16, 8 elements per 16-byte load and store; XU loads in flight
// per thread, so that a grid of a few blocks per SM still keeps enough bytes
// in flight to stream at HBM rate.
constexpr int XU = 8;
__device__ __forceinline__ uint4 bf16x8_to_f16x8(const uint4 v, bool& bad) {
  const uint32_t in[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float a = __uint_as_float(in[q] << 16), b = __uint_as_float(in[q] & 0xFFFF0000u);
    bad |= !(fabsf(a) <= kHalfMax) || !(fabsf(b) <= kHalfMax);
    const __half2 h = __floats2half2_rn(a, b);
    out[q] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(out[0], out[1], out[2], out[3]);
}
__global__ void x_to_f16_kernel(const uint4* __restrict__ X, int64_t n8, uint4* __restrict__ Y, DevStatus* st) {
  const int64_t T = (int64_t)gridDim.x * blockDim.x;
  bool bad = false;
  int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (; e + (XU - 1) * T < n8; e += XU * T) {
    uint4 v[XU];
#pragma unroll
    for (int u = 0; u < XU; ++u) v[u] = X[e + u * T];
#pragma unroll
    for (int u = 0; u < XU; ++u) Y[e + u * T] = bf16x8_to_f16x8(v[u], bad);
  }
  for (; e < n8; e += T) Y[e] = bf16x8_to_f16x8(X[e], bad);
  if (bad) record_failure(st, kStatusRange, 310);
}

__global__ void x_split_kernel(const float* __restrict__ X, int64_t N, int64_t n, __half* __restrict__ Xc,
                               DevStatus* st) {
  const int64_t total = N * n;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = e / n, j = e - t * n;
    const float x = X[e];
    const __half hi = to_half_checked(x, st, 311);
    const __half lo = __float2half_rn(x - __half2float(hi));
    Xc[t * 2 * n + j] = hi;
    Xc[t * 2 * n + n + j] = lo;
  }
}

// ---------------------------------------------------------------- scoring kernel
constexpr int SB_BM = 128;        // tokens per tile (TMEM lanes)
constexpr int SB_BN = 128;        // outputs per tile (one TMEM slot: y and d, 128 columns each)
constexpr int SB_BK = 64;         // K elements per box (128 bytes of fp16)
constexpr int SB_BOX = SB_BM * SB_BK * 2;  // 16 KB
constexpr int SB_STAGE = 4 * SB_BOX;       // X(token tile 0), X(token tile 1), B1, B2
constexpr int kNarrowBox = SB_BM * 32 * 2;  // 128 rows x 32 fp16 columns: 8 KB (a group-32 step's boxes)
constexpr int SB_BAND = 16;                // token-tile pairs per raster band
constexpr int SB_MAX_K = 1024;
constexpr int SB_EPI_WARPS = 16;           // warps 2..9 read slot 0, warps 10..17 slot 1 (two per row)
constexpr int SB_THREADS = 64 + 32 * SB_EPI_WARPS;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kC1 = kLog2e * kOpUnscale;  // exponent scale for accumulator (x 2^8) units

struct SbaTmaps {
  CUtensorMap x, wb, e0, dp, dm;  // 64-column boxes, 128-byte swizzle
  CUtensorMap x32, dp32, dm32;     // 32-column boxes, 64-byte swizzle (candidate steps at group 32)
};

struct SbaParams {
  int64_t N, m, n;
  int npad;                      // weight-side row half: n rounded up to whole 64-column boxes
  int g, k, P, ksplit, nsub;     // nsub: 3 for fp32 X (every box); 2 for bf16 X (split boxes only)
  int nbox;                      // 64-wide K boxes, (n + 63) / 64
  const uint8_t* split;          // [nbox] 1: the box's weight side is taken as hi and lo (bf16 X)
  int n_tt, n_tp, n_ot, stages;  // token tiles, token-tile pairs, output tiles
  const int32_t* order;
  float* part;                   // [n_tt][n_ot][F][128], F = 2 + 2P
  float* yd;                     // split runs: [n_tt][n_ot][e^(y-M), d][128 outputs][128 tokens]
  int tp0;                       // first token-tile pair of this launch (n_tp pairs from there)
  DevStatus* st;
  uint64_t acc_wait_ns;          // limit of the epilogue's wait for an accumulator (normally kWaitLimitNs)
};

struct Chunk {
  int xcol, bcol, k16_lo, k16_hi;
  int which;  // 0: phase A (Wb, E0); 1: Dp; 2: Dm
};

// Sub-chunks. Every 64-wide K box is contracted as 1, 2 or 3 consecutive
// sub-chunks that share the box's X and weight columns:
//   bf16 X, box not split: (X, hi)
//   bf16 X, box split:     (X, hi), (X, lo)
//   fp32 X (every box):    (X_hi, hi), (X_lo, hi), (X_hi, lo)
// X_lo sits n columns after X_hi, a weight lo part npad columns after its hi
// part. s_split[b] (shared memory) marks the split boxes; sub_count(b) is the
// number of sub-chunks of box b.
__device__ __forceinline__ int sub_count(const SbaParams& p, const uint8_t* s_split, int b) {
  return p.nsub == 3 ? 3 : 1 + s_split[b];
}

// Per-item chunk geometry. Step 0 is phase A (y = X Wb^T, d = X E0^T over
// K = n), its chunks listed in s_tab (box << 2 | sub). Step p >= 1 adds the
// promoted group order[p-1] (Dp) and the demoted group order[k-p] (Dm),
// promoted chunks first; a group covers one box (g <= 64) or two (g = 128).
struct ItemGeom {
  int step, nch, n_up, box_up, box_dn, k16_lo_up, k16_lo_dn, k16_n, up0, dn0;  // up0/dn0: sub-chunks of a group's first box
};
__device__ __forceinline__ ItemGeom item_geom(const SbaParams& p, const int32_t* order, const uint8_t* s_split,
                                              int nA, int step) {
  ItemGeom g;
  g.step = step;
  g.k16_n = p.g >= 64 ? 4 : p.g / 16;
  g.box_up = g.box_dn = 0;
  g.k16_lo_up = g.k16_lo_dn = 0;
  g.up0 = g.dn0 = 0;
  if (step == 0) {
    g.nch = nA;
    g.n_up = nA;
    return g;
  }
  const int cu = order[step - 1] * p.g, cd = order[p.k - step] * p.g;
  g.box_up = cu >> 6;
  g.box_dn = cd >> 6;
  g.k16_lo_up = p.g >= 64 ? 0 : (cu & 63) >> 4;
  g.k16_lo_dn = p.g >= 64 ? 0 : (cd & 63) >> 4;
  g.up0 = sub_count(p, s_split, g.box_up);
  g.dn0 = sub_count(p, s_split, g.box_dn);
  g.n_up = g.up0 + (p.g == 128 ? sub_count(p, s_split, g.box_up + 1) : 0);
  g.nch = g.n_up + g.dn0 + (p.g == 128 ? sub_count(p, s_split, g.box_dn + 1) : 0);
  return g;
}
__device__ __forceinline__ void chunk_at(const SbaParams& p, const ItemGeom& g, const uint16_t* s_tab, int c,
                                         Chunk& ch) {
  int box, sub;
  if (g.step == 0) {
    box = s_tab[c] >> 2;
    sub = s_tab[c] & 3;
    ch.k16_lo = 0;
    ch.k16_hi = 4;
    ch.which = 0;
  } else {
    const bool up = c < g.n_up;
    const int l = up ? c : c - g.n_up;
    const int first = up ? g.up0 : g.dn0;
    box = (up ? g.box_up : g.box_dn) + (l >= first ? 1 : 0);
    sub = l >= first ? l - first : l;
    ch.k16_lo = up ? g.k16_lo_up : g.k16_lo_dn;
    ch.k16_hi = ch.k16_lo + g.k16_n;
    ch.which = up ? 1 : 2;
  }
  const int xs = (p.nsub == 3 && sub == 1) ? 1 : 0;      // X_lo
  const int bs = (sub == (p.nsub == 3 ? 2 : 1)) ? 1 : 0;  // weight lo part
  const int col = box * SB_BK;
  ch.xcol = col + (xs ? (int)p.n : 0);
  ch.bcol = col + (bs ? p.npad : 0);
}

// Work unit u -> (token-tile pair, output tile); raster bands of SB_BAND pairs.
__device__ __forceinline__ void unit_decode(const SbaParams& p, int u, int& tp, int& ot) {
  const int band_start = (u / (SB_BAND * p.n_ot)) * SB_BAND;
  const int bc = (p.n_tp - band_start < SB_BAND) ? p.n_tp - band_start : SB_BAND;
  const int r = u - band_start * p.n_ot;
  ot = r / bc;
  tp = p.tp0 + band_start + (r - ot * bc);
}

// What one launch of the scoring kernel covers.
enum SbaMode : int {
  kSbaAll = 0,     // phase A and every candidate step
  kSbaPhaseA = 1,  // phase A only (it needs no order), e^(y - M) and d kept in yd
  kSbaSteps = 2,   // candidate steps 1..P-1, starting from yd
};

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^k for an integral k <= 0 (exact; 0 below the normal range).
__device__ __forceinline__ float pow2i(float k) {
  return k >= -126.f ? __int_as_float((127 + (int)k) << 23) : 0.f;
}

// Packed fp32 pairs (sm_100 f32x2 arithmetic): the epilogue handles two output
// columns per instruction, which leaves more issue slots to the MMA thread on
// the same SM sub-partition.
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// max(a, b, c) in one instruction (sm_100 three-input max).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// One work unit is two token tiles (TMEM slots 0 and 1) against one output tile:
// every weight-side box feeds both slots' MMAs, so per output tile the kernel
// moves about a third fewer bytes than with one token tile.
//   warp 0      TMA producer (4 boxes per phase-A chunk, 3 per delta chunk)
//   warp 1      TMEM owner (512 columns) and MMA issuer: phase A as N = 256 MMAs
//               (Wb and E0 boxes adjacent; y and d adjacent in TMEM), delta steps
//               as N = 128 MMAs into d, in place
//   warps 2..17 epilogue, eight per slot: two threads per token row, 64 columns
//               each. A thread copies its d columns to registers and releases
//               the accumulator before computing, so the next candidate's MMA
//               overlaps the epilogue's exponentials; the two halves of a row
//               combine their row maximum and sums through shared memory.
// MODE splits the work in two launches (phase A does not depend on the
// salience order, so it can run before the order exists): kSbaPhaseA also
// stores each tile's e^(y - M) and d, exactly as they sit in TMEM after phase
// A; kSbaSteps loads them back into TMEM and continues with step 1, so the
// two launches together compute bit for bit what one kSbaAll launch does.
template <int MODE, int OBJ>
__global__ void __launch_bounds__(SB_THREADS, 1) sba_score_kernel(const __grid_constant__ SbaTmaps tm, SbaParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * SB_STAGE);
  uint64_t* empty = full + S;
  uint64_t* afull = empty + S;   // [2] step accumulated in TMEM slot s
  uint64_t* afree = afull + 2;   // [2] epilogue done reading slot s
  uint64_t* done = afree + 2;
  uint64_t* xbar = done + 1;     // [8 row groups (slot, quadrant)][4]: max of half 0, max of half 1, sums x2
  uint32_t* tslot = reinterpret_cast<uint32_t*>(xbar + 32);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);
  int32_t* s_order = reinterpret_cast<int32_t*>(tslot + 2);
  float* s_x = reinterpret_cast<float*>(s_order + ((p.k + 3) & ~3));  // [2 slots][128 rows][12]
  uint16_t* s_tab = reinterpret_cast<uint16_t*>(s_x + 2 * 128 * 12);    // phase-A chunks: box << 2 | sub
  uint8_t* s_split = reinterpret_cast<uint8_t*>(s_tab + 3 * p.nbox);   // [nbox]
  int* s_na = reinterpret_cast<int*>(s_split + ((p.nbox + 15) & ~15));  // chunks of phase A

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int s_lo = MODE == kSbaSteps ? 1 : 0;  // the launch's steps: [s_lo, s_hi)
  const int s_hi = MODE == kSbaPhaseA ? 1 : p.P;
  if (MODE != kSbaPhaseA)
    for (int c = threadIdx.x; c < p.k; c += blockDim.x) s_order[c] = p.order[c];
  for (int b = threadIdx.x; b < p.nbox; b += blockDim.x) s_split[b] = p.nsub == 3 ? 0 : (p.split[b] ? 1 : 0);
  __syncthreads();
  if (threadIdx.x == 0) {
    int c = 0;
    for (int b = 0; b < p.nbox; ++b)
      for (int u = 0; u < sub_count(p, s_split, b); ++u) s_tab[c++] = (uint16_t)(b << 2 | u);
    *s_na = c;
    for (int s = 0; s < S; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int s = 0; s < 2; ++s) { mbar_init(&afull[s], 1); mbar_init(&afree[s], SB_EPI_WARPS / 2); }
    mbar_init(done, 1);
    for (int b = 0; b < 32; ++b) mbar_init(&xbar[b], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  const int units = p.n_tp * p.n_ot;
  const int nA = *s_na;
  // candidate steps at group 32 with bf16 X: one stage per step of 32-column boxes
  const bool narrow = p.g == 32 && p.nsub == 2;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      uint32_t it = 0;
      int st = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        int tp, ot;
        unit_decode(p, u, tp, ot);
        const int xrow0 = 2 * tp * SB_BM, xrow1 = xrow0 + SB_BM, brow = ot * SB_BN;
        for (int step = s_lo; step < s_hi && ok; ++step) {
          if (narrow && step > 0) {
            // the whole step in one stage: X of both groups for both token tiles,
            // then the Dp / Dm boxes (hi, and lo for a split box), 8 KB each
            const int cu = s_order[step - 1] * 32, cd = s_order[p.k - step] * 32;
            const int su = s_split[cu >> 6], sd = s_split[cd >> 6];
            if (!mbar_wait(&empty[st], ph ^ 1, abort_flag, p.st, 200 + st)) { ok = false; break; }
            uint8_t* sb = smem + st * SB_STAGE;
            mbar_arrive_expect_tx(&full[st], (6 + su + sd) * kNarrowBox);
            tma_load_2d(sb, &tm.x32, &full[st], cu, xrow0);
            tma_load_2d(sb + kNarrowBox, &tm.x32, &full[st], cu, xrow1);
            tma_load_2d(sb + 2 * kNarrowBox, &tm.x32, &full[st], cd, xrow0);
            tma_load_2d(sb + 3 * kNarrowBox, &tm.x32, &full[st], cd, xrow1);
            tma_load_2d(sb + 4 * kNarrowBox, &tm.dp32, &full[st], cu, brow);
            tma_load_2d(sb + 5 * kNarrowBox, &tm.dm32, &full[st], cd, brow);
            if (su) tma_load_2d(sb + 6 * kNarrowBox, &tm.dp32, &full[st], p.npad + cu, brow);
            if (sd) tma_load_2d(sb + 7 * kNarrowBox, &tm.dm32, &full[st], p.npad + cd, brow);
            ++it;
            if (++st == S) { st = 0; ph ^= 1; }
            continue;
          }
          const ItemGeom geo = item_geom(p, s_order, s_split, nA, step);
          const int nch = geo.nch;
          for (int c = 0; c < nch; ++c) {
            Chunk ch;
            chunk_at(p, geo, s_tab, c, ch);
            if (!mbar_wait(&empty[st], ph ^ 1, abort_flag, p.st, 200 + st)) { ok = false; break; }
            uint8_t* sb = smem + st * SB_STAGE;
            mbar_arrive_expect_tx(&full[st], (ch.which == 0 ? 4 : 3) * SB_BOX);
            tma_load_2d(sb, &tm.x, &full[st], ch.xcol, xrow0);
            tma_load_2d(sb + SB_BOX, &tm.x, &full[st], ch.xcol, xrow1);
            if (ch.which == 0) {
              tma_load_2d(sb + 2 * SB_BOX, &tm.wb, &full[st], ch.bcol, brow);
              tma_load_2d(sb + 3 * SB_BOX, &tm.e0, &full[st], ch.bcol, brow);
            } else {
              tma_load_2d(sb + 2 * SB_BOX, ch.which == 1 ? (const void*)&tm.dp : (const void*)&tm.dm, &full[st],
                          ch.bcol, brow);
            }
            ++it;
            if (++st == S) { st = 0; ph ^= 1; }
          }
        }
      }
      // let every issued copy land before the CTA can exit
      for (uint32_t j = (it > (uint32_t)S ? it - S : 0); j < it; ++j) mbar_drain(&full[j % S], (j / S) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    // The issuing thread shares its SM sub-partition with four busy epilogue
    // warps, so its instruction stream per MMA is kept short: stage descriptors
    // come from one base by adding whole stages in 16-byte units, and the
    // 64-wide boxes' four K steps are unrolled.
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_f16_f32(SB_BM, SB_BN, false, false);
      constexpr uint32_t idesc2 = idesc_f16_f32(SB_BM, 2 * SB_BN, false, false);
      constexpr uint64_t kStage16 = SB_STAGE / 16, kBox16 = SB_BOX / 16;
      const uint64_t d_first = sdesc_sw128(smem_u32(smem), 16, 1024);  // start-address field never carries (< 256 KB)
      uint64_t dcur = d_first;
      int st = 0;
      uint32_t ph = 0, cnt = 0;
      bool ok = true;
      const uint32_t ty0 = tbase, ty1 = tbase + 256;
      const bool dfull = p.g >= 64;  // delta chunks are whole 64-wide boxes
      // The wait before a step's MMAs is for the epilogue's previous release of
      // the slot; a unit's first step in kSbaSteps waits for the load of the
      // unit's phase-A state instead, which is also the first completion of
      // afree (in the other modes the first wait passes on the initial phase).
      const uint32_t fpar = MODE == kSbaSteps ? 0u : 1u;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        for (int step = s_lo; step < s_hi && ok; ++step) {
          if (!mbar_wait(&afree[0], (cnt & 1) ^ fpar, abort_flag, p.st, 220) ||
              !mbar_wait(&afree[1], (cnt & 1) ^ fpar, abort_flag, p.st, 221)) { ok = false; break; }
          tc_fence_after();
          if (narrow && step > 0) {
            // one stage: both groups' 32-column boxes (64-byte swizzle), the
            // promoted group first, each as hi then lo, from a zero accumulator
            const int su = s_split[(s_order[step - 1] * 32) >> 6], sd = s_split[(s_order[p.k - step] * 32) >> 6];
            if (!mbar_wait(&full[st], ph, abort_flag, p.st, 230 + st)) { ok = false; break; }
            tc_fence_after();
            // box i of the stage at start address + i * 8 KB (= 512 in 16-byte units)
            const uint64_t d0 = sdesc_sw64(smem_u32(smem) + (uint32_t)st * SB_STAGE);
            constexpr uint64_t kNb16 = kNarrowBox / 16;
#pragma unroll
            for (int k16 = 0; k16 < 2; ++k16) {
              tc_mma_f16(ty0 + 128, d0 + 2 * k16, d0 + 4 * kNb16 + 2 * k16, idesc, k16 > 0 ? 1u : 0u);
              tc_mma_f16(ty1 + 128, d0 + kNb16 + 2 * k16, d0 + 4 * kNb16 + 2 * k16, idesc, k16 > 0 ? 1u : 0u);
            }
            if (su)
#pragma unroll
              for (int k16 = 0; k16 < 2; ++k16) {
                tc_mma_f16(ty0 + 128, d0 + 2 * k16, d0 + 6 * kNb16 + 2 * k16, idesc, 1u);
                tc_mma_f16(ty1 + 128, d0 + kNb16 + 2 * k16, d0 + 6 * kNb16 + 2 * k16, idesc, 1u);
              }
#pragma unroll
            for (int k16 = 0; k16 < 2; ++k16) {
              tc_mma_f16(ty0 + 128, d0 + 2 * kNb16 + 2 * k16, d0 + 5 * kNb16 + 2 * k16, idesc, 1u);
              tc_mma_f16(ty1 + 128, d0 + 3 * kNb16 + 2 * k16, d0 + 5 * kNb16 + 2 * k16, idesc, 1u);
            }
            if (sd)
#pragma unroll
              for (int k16 = 0; k16 < 2; ++k16) {
                tc_mma_f16(ty0 + 128, d0 + 2 * kNb16 + 2 * k16, d0 + 7 * kNb16 + 2 * k16, idesc, 1u);
                tc_mma_f16(ty1 + 128, d0 + 3 * kNb16 + 2 * k16, d0 + 7 * kNb16 + 2 * k16, idesc, 1u);
              }
            tc_commit(&empty[st]);
            if (++st == S) { st = 0; ph ^= 1; dcur = d_first; } else { dcur += kStage16; }
            tc_commit(&afull[0]);
            tc_commit(&afull[1]);
            ++cnt;
            continue;
          }
          const ItemGeom geo = item_geom(p, s_order, s_split, nA, step);
          const int nch = geo.nch;
          // A shared-memory access by this thread while its MMAs are in flight
          // waits for them to drain (about 380 cycles: the queue holds only a few
          // MMAs), so each wait is made to cover two chunks where it can: right
          // after the blocking wait on a chunk's stage, the next chunk of the
          // same step is tested (cheap, nothing new in flight) and, if its stage
          // is full too, both chunks go out behind the one wait. (Taking all
          // three stages at once is slower: no stage is then being refilled
          // while the MMAs run.)
          for (int c = 0; c < nch;) {
            if (!mbar_wait(&full[st], ph, abort_flag, p.st, 230 + st)) { ok = false; break; }
            int st2 = st + 1;
            uint32_t ph2 = ph;
            if (st2 == S) { st2 = 0; ph2 ^= 1; }
            const int take = (c + 1 < nch && mbar_test(&full[st2], ph2)) ? 2 : 1;
            tc_fence_after();
            for (int t = 0; t < take; ++t, ++c) {
              const uint64_t a0 = dcur, a1 = dcur + kBox16, b0 = dcur + 2 * kBox16;
              // advancing 32 bytes along K = +2 in the descriptor's 16-byte start-address field
              if (step == 0) {
#pragma unroll
                for (int k16 = 0; k16 < 4; ++k16) {
                  const uint32_t acc = (c > 0 || k16 > 0) ? 1u : 0u;
                  tc_mma_f16(ty0, a0 + 2 * k16, b0 + 2 * k16, idesc2, acc);
                  tc_mma_f16(ty1, a1 + 2 * k16, b0 + 2 * k16, idesc2, acc);
                }
              } else if (dfull) {
                // a step's update accumulates from zero (its own short chain); the
                // epilogue adds it to d in registers
#pragma unroll
                for (int k16 = 0; k16 < 4; ++k16) {
                  const uint32_t acc = (c > 0 || k16 > 0) ? 1u : 0u;
                  tc_mma_f16(ty0 + 128, a0 + 2 * k16, b0 + 2 * k16, idesc, acc);
                  tc_mma_f16(ty1 + 128, a1 + 2 * k16, b0 + 2 * k16, idesc, acc);
                }
              } else {
                Chunk ch;
                chunk_at(p, geo, s_tab, c, ch);
                for (int k16 = ch.k16_lo; k16 < ch.k16_hi; ++k16) {
                  const uint32_t acc = (c > 0 || k16 > ch.k16_lo) ? 1u : 0u;
                  tc_mma_f16(ty0 + 128, a0 + 2 * k16, b0 + 2 * k16, idesc, acc);
                  tc_mma_f16(ty1 + 128, a1 + 2 * k16, b0 + 2 * k16, idesc, acc);
                }
              }
              tc_commit(&empty[st]);
              if (++st == S) { st = 0; ph ^= 1; dcur = d_first; } else { dcur += kStage16; }
            }
          }
          if (!ok) break;
          tc_commit(&afull[0]);
          tc_commit(&afull[1]);
          ++cnt;
        }
      }
      tc_commit(done);
      mbar_drain(done, 0);
    }
  } else {
    // ------------------------------------------------ epilogue
    // warp e = warp - 2: slot e >> 3, column half h = (e >> 2) & 1, TMEM lane
    // quadrant q = warp & 3 (the quadrant a warp may access); row r = 32 q + lane.
    const int e = warp - 2;
    const int slot = e >> 3, h = (e >> 2) & 1, q = warp & 3;
    const int r = q * 32 + lane;
    const int F = 2 + 2 * p.P;
    const uint32_t ty = tbase + ((uint32_t)(q * 32) << 16) + slot * 256 + h * 64, td = ty + 128;
    float* xs = s_x + (slot * 128 + r) * 12;  // [0..3] even steps, [4..7] odd steps, [8..9] shifts
    uint64_t* xb = xbar + (slot * 4 + q) * 4;  // max h0, max h1, sums (even), sums (odd)
    uint32_t cnt = 0, nunit = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++nunit) {
      int tp, ot;
      unit_decode(p, u, tp, ot);
      const int tt = 2 * tp + slot;
      const bool have = tt < p.n_tt;        // the second tile of an odd pair is padding
      const int64_t col0 = (int64_t)ot * SB_BN + h * 64;
      const int nvalid = (int)((p.m - col0) > 64 ? 64 : ((p.m - col0) > 0 ? (p.m - col0) : 0));
      float* outp = p.part + ((size_t)(have ? tt : 0) * p.n_ot + ot) * F * SB_BM + r;
      // this thread's 64 outputs of its token row in yd (e^(y - M); d at + 128 rows)
      float* ydp = p.yd + ((size_t)(have ? tt : 0) * p.n_ot + ot) * 2 * SB_BN * SB_BM + (size_t)(h * 64) * SB_BM + r;
      float Mt = 0.f;
      // d of this thread's 64 outputs, kept in registers for the whole unit: phase A
      // leaves d_0 in tensor memory, every later step its update alone, added here
      // with round-to-nearest fp32 adds (the tensor core's accumulator truncates,
      // which over the long chain of all steps would shrink |d| systematically)
      uint32_t v[64];
      if (MODE == kSbaSteps) {
        // phase A's e^(y - M) back in tensor memory and its d_0 into registers; the
        // arrival on afree hands the slot to the first candidate step's MMAs (a
        // unit's last step does not release the slot in this mode: this load does)
#pragma unroll
        for (int j = 0; j < 64; ++j) v[j] = have ? __float_as_uint(ydp[(size_t)j * SB_BM]) : 0u;
        tmem_st32(ty, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_st32(ty + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tc_wait_st();
#pragma unroll
        for (int j = 0; j < 64; ++j) v[j] = have ? __float_as_uint(ydp[(size_t)(SB_BN + j) * SB_BM]) : 0u;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&afree[slot]);
      }
      // The tail of every step: the sums of this step's d over the thread's 64
      // outputs, the accumulator's release after the unit's last step, and the
      // halves' exchange and partial stores. false: a wait gave up.
      auto finish_step = [&](int step, float sy) -> bool {
        const bool last = step == s_hi - 1;
        // Per-token sums over this thread's 64 outputs. KL: S_q = sum e^(y-M) e^d
        // and A = sum e^(y-M) d. MSE: the sum of d^2 (accumulator units, x 2^16).
        uint64_t sqp = 0, ap = 0;  // packed (even, odd column) sums
        float csh = 0.f;           // S_q carries a factor 2^-csh (0 unless it could overflow)
        if (OBJ == 1) {
#pragma unroll
          for (int j = 0; j < 64; j += 2) {
            const uint64_t dd = f2_pack(__uint_as_float(v[j]), __uint_as_float(v[j + 1]));
            sqp = f2_fma(dd, dd, sqp);
          }
        } else {
          float dm = fmax3(__uint_as_float(v[0]), __uint_as_float(v[1]), __uint_as_float(v[2]));
#pragma unroll
          for (int j = 3; j < 63; j += 2) dm = fmax3(dm, __uint_as_float(v[j]), __uint_as_float(v[j + 1]));
          dm = fmaxf(dm, __uint_as_float(v[63]));
          // A quantized output far above its full-precision value (d above about
          // 44 in output units) would overflow e^d in fp32. The thread's largest
          // exponent decides a shift csh, a multiple of 32 that keeps every term
          // at most 2^64; it is 0 for ordinary layers, where e^(d log2(e) - 0)
          // is exactly the unshifted term.
          const float c = dm * kC1 - 64.f;
          csh = c > 0.f ? 32.f * ceilf(c * (1.f / 32.f)) : 0.f;
          const uint64_t kc2 = f2_pack(kC1, kC1), nc = f2_pack(-csh, -csh);
          // e^(y - M) in 8-column pieces. In the split launches the pieces are
          // double-buffered (the load of the next one is in flight while this one
          // is consumed); the one-pass launch loads them one at a time. Same
          // arithmetic either way.
          constexpr int NB = 2;
          uint32_t ev[NB][8];
          if (NB == 2) {
            tmem_ld8(ty, ev[0]);
            tc_wait_ld8(ev[0]);
          }
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            uint32_t (&cur)[8] = ev[cc % NB];
            if (NB == 1) {
              tmem_ld8(ty + cc * 8, cur);
              tc_wait_ld8(cur);
            } else if (cc + 1 < 8) {
              tmem_ld8(ty + (cc + 1) * 8, ev[(cc + 1) % NB]);
            }
#pragma unroll
            for (int j = 0; j < 8; j += 2) {
              const uint64_t ey = f2_pack(__uint_as_float(cur[j]), __uint_as_float(cur[j + 1]));
              const uint64_t dd = f2_pack(__uint_as_float(v[cc * 8 + j]), __uint_as_float(v[cc * 8 + j + 1]));
              float x0, x1;
              f2_unpack(f2_fma(dd, kc2, nc), x0, x1);
              sqp = f2_fma(ey, f2_pack(ex2(x0), ex2(x1)), sqp);
              ap = f2_fma(ey, dd, ap);
            }
            if (NB == 2 && cc + 1 < 8) tc_wait_ld8(ev[(cc + 1) % NB]);
          }
        }
        float sq0, sq1, a0, a1;
        f2_unpack(sqp, sq0, sq1);
        f2_unpack(ap, a0, a1);
        if (last && MODE != kSbaSteps) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&afree[slot]);
        }
        // half 1 hands its sums to half 0, which writes the row's partials
        const int par = cnt & 1;
        float* xo = xs + 4 * par;
        if (h == 1) {
          xo[1] = sy;
          xo[2] = sq0 + sq1;
          xo[3] = a0 + a1;
          xs[8 + par] = csh;
          __syncwarp();
          if (lane == 0) mbar_arrive(&xb[2 + par]);
        } else {
          if (!mbar_wait(&xb[2 + par], (cnt >> 1) & 1, abort_flag, p.st, 252 + slot)) return false;
          if (have) {
            if (step == 0) {
              outp[0] = Mt * kOpUnscale;
              outp[SB_BM] = sy + xo[1];
            }
            // S_q of the row: the plain sum when neither half is shifted (the
            // usual case); else the halves at a common shift, stored as the
            // value if it fits below 2^120 and otherwise as minus its log2
            // (S_q > 0, so a negative entry is unambiguous)
            const float c1 = xs[8 + par];
            float sq = (sq0 + sq1) + xo[2];
            if (csh != 0.f || c1 != 0.f) {
              const float ct = fmaxf(csh, c1);
              const float s2 = pow2i(csh - ct) * (sq0 + sq1) + pow2i(c1 - ct) * xo[2];
              const float l2 = log2f(s2) + ct;
              sq = l2 < 120.f ? exp2f(l2) : -l2;
            }
            outp[(size_t)(2 + 2 * step) * SB_BM] = sq;
            outp[(size_t)(3 + 2 * step) * SB_BM] = ((a0 + a1) + xo[3]) * kOpUnscale;
          }
        }
        ++cnt;
        return true;
      };
      // the accumulator's release once its contents are in registers (not after
      // the unit's last step: the next unit's first MMA overwrites e^(y - M))
      auto release_early = [&](int step) {
        if (step != s_hi - 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&afree[slot]);
        }
      };
      if (MODE != kSbaSteps) {
        // step 0 (phase A): y -> row maximum (both halves) -> e^(y - M) stored back
        // in place of y; then d_0 into registers
        if (!mbar_wait(&afull[slot], cnt & 1, abort_flag, p.st, 240 + slot, p.acc_wait_ns)) { ok = false; break; }
        tc_fence_after();
        // y in 8-column pieces (the maximum, then e^(y - M) written back in
        // place), so that no 64 registers besides d are needed
        float sy = 0.f;
        float mx = -3.0e38f;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t yv[8];
          tmem_ld8(ty + cc * 8, yv);
          tc_wait_ld8(yv);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            if (cc * 8 + j < nvalid) mx = fmaxf(mx, __uint_as_float(yv[j]));
        }
        xs[h ? 0 : 4] = mx;
        __syncwarp();
        if (lane == 0) mbar_arrive(&xb[h]);
        if (!mbar_wait(&xb[h ^ 1], nunit & 1, abort_flag, p.st, 250 + slot)) { ok = false; break; }
        mx = fmaxf(mx, xs[h ? 4 : 0]);
        const float mb = -mx * kC1;
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t yv[8];
          tmem_ld8(ty + cc * 8, yv);
          tc_wait_ld8(yv);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float ey = (cc * 8 + j < nvalid) ? ex2(fmaf(__uint_as_float(yv[j]), kC1, mb)) : 0.f;
            sy += ey;
            yv[j] = __float_as_uint(ey);
            if (MODE == kSbaPhaseA && have) ydp[(size_t)(cc * 8 + j) * SB_BM] = ey;
          }
          tmem_st8(ty + cc * 8, yv);
        }
        tc_wait_st();
        Mt = mx;
        tmem_ld32(td, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
        tmem_ld32(td + 32, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
        tc_wait_ld();
        if (MODE == kSbaPhaseA && have) {
#pragma unroll
          for (int j = 0; j < 64; ++j) ydp[(size_t)(SB_BN + j) * SB_BM] = __uint_as_float(v[j]);
        }
        release_early(0);
        if (!finish_step(0, sy)) { ok = false; break; }
      }
      for (int step = 1; step < s_hi; ++step) {
        // candidate step: d += this step's update (round to nearest)
        if (!mbar_wait(&afull[slot], cnt & 1, abort_flag, p.st, 240 + slot, p.acc_wait_ns)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t u[16];
          tmem_ld16(td + 16 * q, u);
          tc_wait_ld16(u);
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            float x0, x1;
            f2_unpack(f2_add(f2_pack(__uint_as_float(v[16 * q + j]), __uint_as_float(v[16 * q + j + 1])),
                             f2_pack(__uint_as_float(u[j]), __uint_as_float(u[j + 1]))),
                      x0, x1);
            v[16 * q + j] = __float_as_uint(x0);
            v[16 * q + j + 1] = __float_as_uint(x1);
          }
        }
        release_early(step);
        if (!finish_step(step, 0.f)) { ok = false; break; }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ---------------------------------------------------------------- merge and final
// Per token: KL_t = log(S_q / S_y) - A / S_y from the output tiles' partials,
// each tile's sums rescaled to the token's overall maximum M (fp64); an S_q
// partial stored as minus its log2 (it would not fit fp32) is 2^-v. MSE
// (objective 1): the tiles' sums of d^2, x 2^-16 / m.
__global__ void __launch_bounds__(128) sba_merge_kernel(const float* __restrict__ part, int n_ot, int P, int64_t N,
                                                        int n_tt, int objective, int64_t m,
                                                        double* __restrict__ kl_part) {
  constexpr int QB = 8;  // candidates per pass
  __shared__ double red[4][QB];
  const int tt = blockIdx.x, r = threadIdx.x;
  const int F = 2 + 2 * P;
  const bool valid = (int64_t)tt * SB_BM + r < N;
  const float* base = part + (size_t)tt * n_ot * F * SB_BM + r;
  const bool mse = objective == 1;
  // a tile's rescale factor to the token's overall maximum M, recomputed where
  // it is used (the same value every time) rather than kept per tile
  float M = -3.0e38f;
  double Sy = 0.0;
  if (!mse) {
    for (int og = 0; og < n_ot; ++og) M = fmaxf(M, base[(size_t)og * F * SB_BM]);
    for (int og = 0; og < n_ot; ++og) {
      const float f = exp2f((base[(size_t)og * F * SB_BM] - M) * kLog2e);
      Sy += (double)base[(size_t)og * F * SB_BM + SB_BM] * (double)f;
    }
  }
  // candidates in blocks of QB: one pass over the output tiles loads 2 QB
  // independent values per tile (the sums run over the tiles in order, as
  // one candidate at a time would)
  for (int q0 = 0; q0 < P; q0 += QB) {
    const int nq = (P - q0 < QB) ? P - q0 : QB;
    double sq[QB], a[QB];
#pragma unroll
    for (int j = 0; j < QB; ++j) sq[j] = a[j] = 0.0;
    bool shifted = false;
    for (int og = 0; og < n_ot; ++og) {
      const float* bt = base + (size_t)og * F * SB_BM;
      const double f = mse ? 1.0 : (double)exp2f((bt[0] - M) * kLog2e);
      const float* bq = bt + (size_t)(2 + 2 * q0) * SB_BM;
#pragma unroll
      for (int j = 0; j < QB; ++j)
        if (j < nq) {
          const float v = bq[(size_t)(2 * j) * SB_BM];
          shifted |= v < 0.f;
          sq[j] += (double)v * f;
          a[j] += (double)bq[(size_t)(2 * j + 1) * SB_BM] * f;
        }
    }
    if (shifted) {
      // rare: a partial stored as minus its log2 (see the scoring epilogue); the
      // S_q sums of this pass again, decoding those entries
#pragma unroll
      for (int j = 0; j < QB; ++j) sq[j] = 0.0;
      for (int og = 0; og < n_ot; ++og) {
        const float* bt = base + (size_t)og * F * SB_BM;
        const double f = mse ? 1.0 : (double)exp2f((bt[0] - M) * kLog2e);
        const float* bq = bt + (size_t)(2 + 2 * q0) * SB_BM;
        for (int j = 0; j < QB; ++j)
          if (j < nq) {
            const float v = bq[(size_t)(2 * j) * SB_BM];
            sq[j] += (v >= 0.f ? (double)v : exp2(-(double)v)) * f;
          }
      }
    }
#pragma unroll
    for (int j = 0; j < QB; ++j)
      if (j < nq) {
        double kl = 0.0;
        if (valid) kl = mse ? sq[j] * (1.0 / 65536.0) / (double)m : (log(sq[j] / Sy) - a[j] / Sy);
        kl = warp_sum(kl);
        if ((r & 31) == 0) red[r >> 5][j] = kl;
      }
    __syncthreads();
    if (r < nq) kl_part[(size_t)(q0 + r) * n_tt + tt] = (red[0][r] + red[1][r]) + (red[2][r] + red[3][r]);
    __syncthreads();
  }
}

__global__ void sba_final_kernel(const double* __restrict__ kl_part, int n_tt, int P, int64_t N,
                                 const int32_t* __restrict__ order, int k, int avg_bits, double* __restrict__ kl_out,
                                 int32_t* __restrict__ pstar_out, uint8_t* __restrict__ bits) {
  __shared__ double s_kl[SB_MAX_K / 2 + 1];
  __shared__ int s_p;
  // one warp per candidate: lane l adds token tiles l, l + 32, ... in order,
  // then a fixed shuffle tree (the same order every run)
  const int lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  for (int q = threadIdx.x >> 5; q < P; q += nw) {
    double acc = 0.0;
    for (int t = lane; t < n_tt; t += 32) acc += kl_part[(size_t)q * n_tt + t];
    acc = warp_sum(acc);
    if (lane == 0) {
      s_kl[q] = acc / (double)N;
      if (kl_out) kl_out[q] = s_kl[q];
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int best = 0;
    for (int q = 1; q < P; ++q)
      if (s_kl[q] < s_kl[best]) best = q;
    s_p = best;
    if (pstar_out) *pstar_out = best;
  }
  __syncthreads();
  const int ps = s_p;
  for (int c = threadIdx.x; c < k; c += blockDim.x) bits[c] = (uint8_t)avg_bits;
  __syncthreads();
  for (int q = threadIdx.x; q < ps; q += blockDim.x) {
    bits[order[q]] = (uint8_t)(avg_bits + 1);
    bits[order[k - 1 - q]] = (uint8_t)(avg_bits - 1);
  }
}

// ---------------------------------------------------------------- host side
// Workspace: [prepared operands: Wb, E0, Dp, Dm, X as fp16][search: partials, KL parts].
// The prepared region depends only on W and X, so it can be filled early.
struct SbaPlan {
  int k, P, ksplit, nsub, npad, nbox, n_tt, n_tp, n_ot, stages;
  size_t off_wb, off_e0, off_dp, off_dm, off_xc, off_split, off_part, off_klp, total;
  size_t smem;
};

// Box selection (bf16 X): column energies of W (all rows) and of X (its first
// kSelTokens tokens), then per 64-column box the score sum_j |x_j|^2 |w_j|^2, an
// estimate of the variance that fp16 rounding of the box's weight-side operands
// adds to the outputs. Boxes are taken in descending score until what is left
// is at most kSelRemainder of the total; those boxes are split into hi and lo.
constexpr int64_t kSelTokens = 16384;
constexpr int kSelRowsX = 128;
constexpr double kSelRemainder = 1.0 / 32.0;
// rows of W per block: 32, more for very tall W so the grid stays within 32768 row blocks
static int64_t sel_rows_w(int64_t m) {
  const int64_t r = (m + 32767) / 32768;
  return r > 32 ? r : 32;
}
static int sel_row_blocks_w(int64_t m) { return (int)((m + sel_rows_w(m) - 1) / sel_rows_w(m)); }
static int sel_row_blocks_x(int64_t N) {
  const int64_t t = N < kSelTokens ? N : kSelTokens;
  return (int)((t + kSelRowsX - 1) / kSelRowsX);
}
static size_t sel_bytes(int64_t m, int64_t n, int64_t N) {
  return ((size_t)(sel_row_blocks_w(m) + sel_row_blocks_x(N)) * n + n) * sizeof(double);
}

static size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

SbaPlan sba_plan(int64_t m, int64_t n, int64_t N, int xdtype, int group) {
  SbaPlan pl{};
  pl.k = (int)(n / group);
  pl.P = pl.k / 2 + 1;
  pl.ksplit = xdtype == 1 ? 1 : 2;
  pl.nsub = xdtype == 1 ? 2 : 3;
  pl.npad = (int)((n + SB_BK - 1) / SB_BK * SB_BK);
  pl.nbox = pl.npad / SB_BK;
  pl.n_tt = (int)((N + SB_BM - 1) / SB_BM);
  pl.n_ot = (int)((m + SB_BN - 1) / SB_BN);
  pl.n_tp = (pl.n_tt + 1) / 2;
  const size_t wbytes = (size_t)m * 2 * pl.npad * 2;  // hi and lo halves of npad columns each
  size_t off = 0;
  pl.off_wb = off; off = align256(off + wbytes);
  pl.off_e0 = off; off = align256(off + wbytes);
  pl.off_dp = off; off = align256(off + wbytes);
  pl.off_dm = off; off = align256(off + wbytes);
  pl.off_xc = off; off = align256(off + (size_t)N * pl.ksplit * n * 2);
  pl.off_split = off; off = align256(off + (size_t)pl.nbox);
  pl.off_part = off;
  {
    const size_t partials = (size_t)pl.n_tt * pl.n_ot * (2 + 2 * pl.P) * SB_BM * sizeof(float);
    const size_t sel = sel_bytes(m, n, N);  // the selection's scratch, before the partials exist
    off = align256(off + (partials > sel ? partials : sel));
  }
  pl.off_klp = off; off = align256(off + (size_t)pl.P * pl.n_tt * sizeof(double));
  pl.total = off;
  const size_t fixed = 1024 + 512 + 256 + (size_t)(pl.k + 4) * 4 + 64 + 2 * 128 * 12 * sizeof(float) +
                       (size_t)3 * pl.nbox * 2 + (size_t)((pl.nbox + 15) & ~15) + 16;
  int st = 3;
  while (st > 2 && fixed + (size_t)st * SB_STAGE > 227 * 1024) --st;
  pl.stages = st;
  pl.smem = fixed + (size_t)st * SB_STAGE;
  // more than half of the SM's shared memory: one CTA per SM, so the 512-column
  // TMEM allocation never waits on a second resident CTA
  if (pl.smem < 120 * 1024) pl.smem = 120 * 1024;
  return pl;
}

size_t sba_ws_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group) {
  return sba_plan(m, n, N, xdtype, group).total;
}
size_t sba_prep_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group) {
  return sba_plan(m, n, N, xdtype, group).off_part;
}
size_t sba_search_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group) {
  const SbaPlan pl = sba_plan(m, n, N, xdtype, group);
  return pl.total - pl.off_part;
}

// The weight-side fp16 hi/lo operands (RTN at b-1, b, b+1) into the prepared region
// (pw: sba_prep_bytes). bps caps the resident blocks per SM: a small cap
// leaves room on every SM for kernels that run beside these grid-stride loops
// on other streams.
cudaError_t launch_sba_prep_w(const float* W, int64_t m, int64_t n, int64_t N, int xdtype, int group, int avg_bits,
                              uint8_t* pw, DevStatus* st, int num_sms, int bps, cudaStream_t s) {
  const SbaPlan pl = sba_plan(m, n, N, xdtype, group);
  if (pl.k > SB_MAX_K) return cudaErrorInvalidValue;
  __half* Wb = reinterpret_cast<__half*>(pw + pl.off_wb);
  __half* E0 = reinterpret_cast<__half*>(pw + pl.off_e0);
  __half* Dp = reinterpret_cast<__half*>(pw + pl.off_dp);
  __half* Dm = reinterpret_cast<__half*>(pw + pl.off_dm);
  if (pl.npad != n) {  // the columns between n and npad of both halves must read as zero
    cudaError_t e = cudaMemsetAsync(pw + pl.off_wb, 0, pl.off_xc - pl.off_wb, s);
    if (e != cudaSuccess) return e;
  }
  const int64_t total4 = m * n / 4;              // n is a multiple of 32
  const int64_t n4 = n / 4, rs2 = 2 * (int64_t)pl.npad / 4, lo2 = pl.npad / 4;
  int pgrid = (int)((total4 + 255) / 256);        // 8 warps x 32 float4 per block and pass
  if (pgrid > num_sms * bps) pgrid = num_sms * bps;
  const float4* W4 = reinterpret_cast<const float4*>(W);
  uint2 *b0 = reinterpret_cast<uint2*>(Wb), *b1 = reinterpret_cast<uint2*>(E0), *b2 = reinterpret_cast<uint2*>(Dp),
        *b3 = reinterpret_cast<uint2*>(Dm);
  switch (group) {
    case 32: sba_prep_kernel<32><<<pgrid, 256, 0, s>>>(W4, total4, n4, rs2, lo2, avg_bits, b0, b1, b2, b3, st); break;
    case 64: sba_prep_kernel<64><<<pgrid, 256, 0, s>>>(W4, total4, n4, rs2, lo2, avg_bits, b0, b1, b2, b3, st); break;
    case 128: sba_prep_kernel<128><<<pgrid, 256, 0, s>>>(W4, total4, n4, rs2, lo2, avg_bits, b0, b1, b2, b3, st); break;
    default: return cudaErrorInvalidValue;
  }
  count_launches(1);
  return cudaGetLastError();
}

// Rows [t0, t1) of X as fp16 operands (bf16: converted; fp32: split into a
// high and a low fp16 part) into the prepared region.
cudaError_t launch_sba_prep_x(const void* X, int64_t m, int64_t n, int64_t N, int xdtype, int group, int64_t t0,
                              int64_t t1, uint8_t* pw, DevStatus* st, int num_sms, int bps, cudaStream_t s) {
  const SbaPlan pl = sba_plan(m, n, N, xdtype, group);
  if (t0 < 0 || t1 > N || t1 < t0) return cudaErrorInvalidValue;
  if (t1 == t0) return cudaSuccess;
  __half* Xc = reinterpret_cast<__half*>(pw + pl.off_xc);
  if (pl.ksplit == 2) {
    x_split_kernel<<<num_sms * bps, 256, 0, s>>>(static_cast<const float*>(X) + t0 * n, t1 - t0, n,
                                                 Xc + t0 * 2 * n, st);
  } else {
    x_to_f16_kernel<<<num_sms * bps, 256, 0, s>>>(static_cast<const uint4*>(X) + t0 * n / 8, (t1 - t0) * n / 8,
                                                  reinterpret_cast<uint4*>(Xc + t0 * n), st);
  }
  count_launches(1);
  return cudaGetLastError();
}

// Column sums of squares: blockIdx.y < rbw covers rows_w rows of W, the rest
// kSelRowsX tokens of X (bf16); each thread 4 adjacent columns. Fixed-order
// partials [row block][column], summed in order by sel_score_kernel.
__global__ void sel_colsq_kernel(const float* __restrict__ W, int64_t m, int64_t n, int64_t rows_w,
                                 const uint16_t* __restrict__ X, int64_t T0, int rbw, double* __restrict__ part) {
  const int64_t col = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (col >= n) return;
  const int rb = blockIdx.y;
  double a[4] = {0.0, 0.0, 0.0, 0.0};
  if (rb < rbw) {
    const int64_t r0 = (int64_t)rb * rows_w, r1 = (r0 + rows_w < m) ? r0 + rows_w : m;
    for (int64_t r = r0; r < r1; ++r) {
      const float4 v = *reinterpret_cast<const float4*>(W + r * n + col);
      a[0] += (double)v.x * v.x; a[1] += (double)v.y * v.y; a[2] += (double)v.z * v.z; a[3] += (double)v.w * v.w;
    }
  } else {
    const int64_t r0 = (int64_t)(rb - rbw) * kSelRowsX, r1 = (r0 + kSelRowsX < T0) ? r0 + kSelRowsX : T0;
    for (int64_t r = r0; r < r1; ++r) {
      const uint2 v = *reinterpret_cast<const uint2*>(X + r * n + col);
      const float x0 = __uint_as_float(v.x << 16), x1 = __uint_as_float(v.x & 0xFFFF0000u);
      const float x2 = __uint_as_float(v.y << 16), x3 = __uint_as_float(v.y & 0xFFFF0000u);
      a[0] += (double)x0 * x0; a[1] += (double)x1 * x1; a[2] += (double)x2 * x2; a[3] += (double)x3 * x3;
    }
  }
  double* o = part + (int64_t)rb * n + col;
  o[0] = a[0]; o[1] = a[1]; o[2] = a[2]; o[3] = a[3];
}

__global__ void sel_score_kernel(const double* __restrict__ part, int rbw, int rbx, int64_t n,
                                 double* __restrict__ score) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  double w = 0.0, x = 0.0;
  for (int r = 0; r < rbw; ++r) w += part[(int64_t)r * n + j];
  for (int r = 0; r < rbx; ++r) x += part[(int64_t)(rbw + r) * n + j];
  score[j] = w * x;
}

// One block of 1024 threads, nbox <= 1024: box scores, their stable descending
// rank, the shortest prefix of the ranking that leaves at most `rem` of the
// total, flags for the boxes in it.
__global__ void sel_pick_kernel(const double* __restrict__ score, int64_t n, int nbox, double rem,
                                uint8_t* __restrict__ split) {
  __shared__ double s_box[1024], s_sorted[1024];
  __shared__ int s_keep;
  const int b = threadIdx.x;
  double v = 0.0;
  if (b < nbox)
    for (int64_t j = (int64_t)b * 64; j < (int64_t)b * 64 + 64 && j < n; ++j) v += score[j];
  if (b < nbox) s_box[b] = v;
  __syncthreads();
  int rank = 0;
  if (b < nbox) {
    for (int o = 0; o < nbox; ++o) rank += (s_box[o] > v || (s_box[o] == v && o < b)) ? 1 : 0;
    s_sorted[rank] = v;
  }
  __syncthreads();
  if (b == 0) {
    double total = 0.0;
    for (int i = 0; i < nbox; ++i) total += s_sorted[i];
    double left = total;
    int keep = 0;
    while (keep < nbox && left > rem * total) left -= s_sorted[keep++];
    s_keep = keep;
  }
  __syncthreads();
  if (b < nbox) split[b] = rank < s_keep ? 1 : 0;
}

// The split flags into the prepared region (pw), from W and X (bf16: the first
// kSelTokens tokens), with the search region (sw) as scratch. precision 1: every
// box split. fp32 X needs no flags (every box is taken in three parts).
cudaError_t launch_sba_select(const float* W, const void* X, int64_t m, int64_t n, int64_t N, int xdtype, int group,
                              int precision, uint8_t* pw, uint8_t* sw, cudaStream_t s) {
  const SbaPlan pl = sba_plan(m, n, N, xdtype, group);
  uint8_t* flags = pw + pl.off_split;
  if (xdtype != 1) return cudaSuccess;
  if (pl.nbox > 1024) return cudaErrorInvalidValue;
  if (precision == 1) {
    count_launches(0);
    return cudaMemsetAsync(flags, 1, (size_t)pl.nbox, s);
  }
  const int rbw = sel_row_blocks_w(m), rbx = sel_row_blocks_x(N);
  const int64_t T0 = N < kSelTokens ? N : kSelTokens;
  double* part = reinterpret_cast<double*>(sw);
  double* score = part + (size_t)(rbw + rbx) * n;
  sel_colsq_kernel<<<dim3((unsigned)((n / 4 + 255) / 256), (unsigned)(rbw + rbx)), 256, 0, s>>>(
      W, m, n, sel_rows_w(m), static_cast<const uint16_t*>(X), T0, rbw, part);
  sel_score_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(part, rbw, rbx, n, score);
  sel_pick_kernel<<<1, 1024, 0, s>>>(score, n, pl.nbox, kSelRemainder, flags);
  count_launches(3);
  return cudaGetLastError();
}

// Where the split flags sit in the prepared region, and how many there are.
size_t sba_split_offset(int64_t m, int64_t n, int64_t N, int xdtype, int group, int* nbox) {
  const SbaPlan pl = sba_plan(m, n, N, xdtype, group);
  *nbox = pl.nbox;
  return pl.off_split;
}

size_t sba_yd_bytes(int64_t m, int64_t n, int64_t N, int xdtype, int group) {
  const SbaPlan pl = sba_plan(m, n, N, xdtype, group);
  return (size_t)pl.n_tt * pl.n_ot * 2 * SB_BN * SB_BM * sizeof(float);
}

// One scoring launch over token-tile pairs [tp0, tp1) on the prepared operands
// (pw) and the search region (sw).
template <int MODE>
static cudaError_t launch_score(const SbaPlan& pl, int64_t m, int64_t n, int64_t N, int group, const int32_t* order,
                                int objective, const uint8_t* pw, uint8_t* sw, float* yd, int tp0, int tp1,
                                DevStatus* st, int num_sms, cudaStream_t s, cudaEvent_t* kev) {
  if (pl.k > SB_MAX_K || tp0 < 0 || tp1 > pl.n_tp || tp1 < tp0) return cudaErrorInvalidValue;
  if (tp1 == tp0) return cudaSuccess;
  SbaTmaps tm;
  bool ok = make_tmap_f16(&tm.x, pw + pl.off_xc, (uint64_t)(n * pl.ksplit), (uint64_t)N, SB_BK, SB_BM);
  const uint64_t wcols = 2 * (uint64_t)pl.npad;  // hi | lo
  ok = ok && make_tmap_f16(&tm.wb, pw + pl.off_wb, wcols, (uint64_t)m, SB_BK, SB_BN);
  ok = ok && make_tmap_f16(&tm.e0, pw + pl.off_e0, wcols, (uint64_t)m, SB_BK, SB_BN);
  ok = ok && make_tmap_f16(&tm.dp, pw + pl.off_dp, wcols, (uint64_t)m, SB_BK, SB_BN);
  ok = ok && make_tmap_f16(&tm.dm, pw + pl.off_dm, wcols, (uint64_t)m, SB_BK, SB_BN);
  ok = ok && make_tmap_f16_sw64(&tm.x32, pw + pl.off_xc, (uint64_t)(n * pl.ksplit), (uint64_t)N, 32, SB_BM);
  ok = ok && make_tmap_f16_sw64(&tm.dp32, pw + pl.off_dp, wcols, (uint64_t)m, 32, SB_BN);
  ok = ok && make_tmap_f16_sw64(&tm.dm32, pw + pl.off_dm, wcols, (uint64_t)m, 32, SB_BN);
  if (!ok) return cudaErrorInvalidValue;
  SbaParams p;
  p.N = N; p.m = m; p.n = n; p.npad = pl.npad; p.g = group; p.k = pl.k; p.P = pl.P; p.ksplit = pl.ksplit;
  p.nsub = pl.nsub; p.nbox = pl.nbox; p.split = pw + pl.off_split;
  p.n_tt = pl.n_tt; p.n_tp = tp1 - tp0; p.n_ot = pl.n_ot; p.stages = pl.stages;
  p.order = order; p.part = reinterpret_cast<float*>(sw); p.yd = yd; p.tp0 = tp0; p.st = st;
  // A test can shorten one wait (the epilogue's wait for its accumulator) with
  // SLIM_TEST_ACC_WAIT_NS, to check that a wait that runs out returns
  // SLIM_ETIMEOUT and leaves the device usable. Nothing else reads it.
  p.acc_wait_ns = kWaitLimitNs;
  if (const char* t = std::getenv("SLIM_TEST_ACC_WAIT_NS")) {
    const unsigned long long v = std::strtoull(t, nullptr, 10);
    if (v > 0 && v < kWaitLimitNs) p.acc_wait_ns = v;
  }
  static std::atomic<uint64_t> attr{0};
  uint64_t bit = 0;
  if (attr_pending(attr, bit)) {  // the plan's shared memory never exceeds this bound
    cudaError_t e = cudaFuncSetAttribute(sba_score_kernel<MODE, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         227 * 1024);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(sba_score_kernel<MODE, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    attr.fetch_or(bit);
  }
  const int units = p.n_tp * pl.n_ot;
  const int grid = units < num_sms ? units : num_sms;
  if (kev) cudaEventRecord(kev[0], s);
  if (objective == 1)
    sba_score_kernel<MODE, 1><<<grid, SB_THREADS, pl.smem, s>>>(tm, p);
  else
    sba_score_kernel<MODE, 0><<<grid, SB_THREADS, pl.smem, s>>>(tm, p);
  if (kev) cudaEventRecord(kev[1], s);
  count_launches(1);
  return cudaGetLastError();
}

// Per-token KL from the partials, its means over tokens, p* and the bits.
static cudaError_t launch_merge_final(const SbaPlan& pl, int64_t m, int64_t N, int avg_bits, const int32_t* order,
                                      int objective, double* kl, int32_t* p_star, uint8_t* bits, uint8_t* sw,
                                      cudaStream_t s) {
  float* part = reinterpret_cast<float*>(sw);
  double* klp = reinterpret_cast<double*>(sw + (pl.off_klp - pl.off_part));
  sba_merge_kernel<<<pl.n_tt, SB_BM, 0, s>>>(part, pl.n_ot, pl.P, N, pl.n_tt, objective, m, klp);
  sba_final_kernel<<<1, 256, 0, s>>>(klp, pl.n_tt, pl.P, N, order, pl.k, avg_bits, kl, p_star, bits);
  count_launches(2);
  return cudaGetLastError();
}

// Scoring, merge and final selection on the prepared operands (pw) with the
// search region (sw: sba_search_bytes) for the partial sums.
cudaError_t launch_sba_search(int64_t m, int64_t n, int xdtype, int64_t N, int group, int avg_bits,
                              const int32_t* order, int objective, double* kl, int32_t* p_star, uint8_t* bits,
                              const uint8_t* pw, uint8_t* sw, DevStatus* st, int num_sms, cudaStream_t s,
                              cudaEvent_t* kev) {
  const SbaPlan pl = sba_plan(m, n, N, xdtype, group);
  cudaError_t e = launch_score<kSbaAll>(pl, m, n, N, group, order, objective, pw, sw, nullptr, 0, pl.n_tp, st,
                                        num_sms, s, kev);
  if (e != cudaSuccess) return e;
  return launch_merge_final(pl, m, N, avg_bits, order, objective, kl, p_star, bits, sw, s);
}

// Split search, first part: phase A for token-tile pairs [tp0, tp1) (pairs of
// 128-token tiles); it needs only the prepared operands of those tokens.
// Writes the pairs' phase-A partials into sw and their TMEM state into yd
// (sba_yd_bytes).
cudaError_t launch_sba_phase_a(int64_t m, int64_t n, int xdtype, int64_t N, int group, int objective, int tp0,
                               int tp1, const uint8_t* pw, uint8_t* sw, float* yd, DevStatus* st, int num_sms,
                               cudaStream_t s) {
  const SbaPlan pl = sba_plan(m, n, N, xdtype, group);
  return launch_score<kSbaPhaseA>(pl, m, n, N, group, nullptr, objective, pw, sw, yd, tp0, tp1, st, num_sms, s,
                                  nullptr);
}

// Split search, second part, once every pair's phase A is in sw and yd: the
// candidate steps, merge and final selection.
cudaError_t launch_sba_steps(int64_t m, int64_t n, int xdtype, int64_t N, int group, int avg_bits,
                             const int32_t* order, int objective, double* kl, int32_t* p_star, uint8_t* bits,
                             const uint8_t* pw, uint8_t* sw, float* yd, DevStatus* st, int num_sms, cudaStream_t s) {
  const SbaPlan pl = sba_plan(m, n, N, xdtype, group);
  if (pl.P > 1) {
    cudaError_t e = launch_score<kSbaSteps>(pl, m, n, N, group, order, objective, pw, sw, yd, 0, pl.n_tp, st,
                                            num_sms, s, nullptr);
    if (e != cudaSuccess) return e;
  }
  return launch_merge_final(pl, m, N, avg_bits, order, objective, kl, p_star, bits, sw, s);
}

cudaError_t launch_sba(const float* W, int64_t m, int64_t n, const void* X, int xdtype, int64_t N, int group,
                       int avg_bits, const int32_t* order, int objective, int precision, double* kl, int32_t* p_star,
                       uint8_t* bits, uint8_t* ws, DevStatus* st, int num_sms, cudaStream_t s, cudaEvent_t* kev) {
  const SbaPlan pl = sba_plan(m, n, N, xdtype, group);
  cudaError_t e = launch_sba_prep_w(W, m, n, N, xdtype, group, avg_bits, ws, st, num_sms, 8, s);
  if (e == cudaSuccess) e = launch_sba_prep_x(X, m, n, N, xdtype, group, 0, N, ws, st, num_sms, 8, s);
  if (e == cudaSuccess) e = launch_sba_select(W, X, m, n, N, xdtype, group, precision, ws, ws + pl.off_part, s);
  if (e != cudaSuccess) return e;
  return launch_sba_search(m, n, xdtype, N, group, avg_bits, order, objective, kl, p_star, bits, ws,
                           ws + pl.off_part, st, num_sms, s, kev);
}

}  // namespace slim
