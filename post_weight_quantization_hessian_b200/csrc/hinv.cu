// hinv_diag: h_j = [H_d^-1]_jj, the inverse-Hessian diagonal of the salience
// formula (SliM-LLM write-up, rkmt.cn, section 组件一 SBA).
//
// H_d = H with zero diagonal entries set to 1, plus alpha * mean(diag) on the
// diagonal. With H_d = L L^T, H_d^-1 = L^-T L^-1, so h_j is the squared norm of
// column j of M = L^-1. All arithmetic is fp64. The matrix is padded to a
// multiple of 32 with an identity block (which leaves the first n entries of
// the inverse's diagonal unchanged) and cut into 64 x 64 blocks, T of them per
// side, the last one 32 or 64 wide.
//
//   Cholesky, right-looking, per diagonal block K:
//     pp(K)     every CTA applies step K-1's update to block K and factors it
//               (L_KK, M_KK = L_KK^-1); CTA 0 stores M_KK, CTA b > 0 updates
//               its block row I = K + b of column K and stores L_IK = A_IK M_KK^T
//               (A_KK itself is never overwritten: every CTA reads it)
//     trail(K)  A_IJ -= L_IK L_JK^T for K + 2 <= J <= I
//   Inverse, forward substitution of L M = I, right-looking, per block row I:
//     rowmult(I)    M_IJ = M_II R_IJ for J < I (R accumulates -sum L_IK M_KJ)
//     inv_update(I) R_I'J -= L_I'I M_IJ for I' > I, J <= I
//   Column norms    h_j = sum_i M_ij^2 (partials, then a fixed-order sum)
//
// pp, trail and the inverse run on three streams of decreasing priority:
// pp(K) needs only trail(K-2) (which brought column K up to step K-2), so the
// factorization chain overlaps the trailing updates, and the inverse fills
// the rest. Tile products use the fp64 tensor-core MMA (m8n8k4) on tiles
// staged in shared memory by cp.async.
//
// Flops are n^3/3 for each half. A non-positive pivot records SLIM_ENOTPD with
// its index; the remaining kernels run to completion on the bad values.
#include <cstdint>
#include <vector>
#include "common.cuh"
#include "f64_tiles.cuh"

namespace slim {



__host__ __device__ inline int64_t pad32(int64_t n) { return (n + 31) / 32 * 32; }

__host__ __device__ inline int blk_size(int64_t n, int b) {
  const int64_t s = n - (int64_t)b * NB;
  return (int)(s < NB ? s : NB);
}

// ---------------------------------------------------------------- damping
__global__ void diag_sum_kernel(const double* __restrict__ H, int64_t n, double alpha, double* __restrict__ out) {
  __shared__ double red[32];
  double acc = 0.0;
  for (int64_t j = threadIdx.x; j < n; j += blockDim.x) {
    const double d = H[j * n + j];
    acc += (d == 0.0) ? 1.0 : d;
  }
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0;
    v = warp_sum(v);
    if (threadIdx.x == 0) out[0] = alpha * (v / (double)n);
  }
}

// A (np x np) = lower triangle of H with the dead-column fix and damping, an
// identity block on the padding, zeros elsewhere. A thread writes two adjacent
// entries (np is even) with one 16-byte store, grid-stride over the matrix so
// that a few waves of blocks keep many stores in flight.
__global__ void damp_copy_kernel(const double* __restrict__ H, int64_t n, int64_t np, const double* __restrict__ damp,
                                 double* __restrict__ A) {
  const double dv = damp[0];
  const int64_t half = np / 2, total = np * half;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / half, j0 = 2 * (e - i * half);
    double v[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int64_t j = j0 + u;
      double x = 0.0;
      if (i < n && j < n) {
        if (j < i) x = H[i * n + j];
        else if (j == i) {
          const double d = H[i * n + i];
          x = ((d == 0.0) ? 1.0 : d) + dv;
        }
      } else if (i == j) {
        x = 1.0;
      }
      v[u] = x;
    }
    *reinterpret_cast<double2*>(A + i * np + j0) = make_double2(v[0], v[1]);
  }
}

// ---------------------------------------------------------------- diagonal block
// Shared scratch of factor_block: two 48-double broadcast buffers, then the
// reciprocal pivots 1/L_pp of the block.
constexpr int kFacScratch = 2 * 48 + 64;

// Warp 0: unblocked Cholesky of the 16 x 16 sub-block at (kb, kb) of D, L into
// D (rows >= p of column p), irdv[kb + p] = 1 / L_pp.
// Lane i (< 16) keeps row i of the columns not yet factored, shifted so that
// x[0] is always the current pivot column. Per pivot p the new column of L is
// broadcast through a shared buffer, written at an offset that lines row
// p+1+c up with slot c; lane p+1 forms the next pivot from its own values, and
// the next reciprocal square root is issued before the rank-1 update so that
// its latency overlaps the update. The pivot loop is unrolled and branch-free
// (a non-positive pivot is replaced by 1 and reported after the loop), so the
// compiler can overlap consecutive pivots. Lanes 16..31 mirror 0..15 and
// store nothing.
__device__ __forceinline__ void factor16(double* D, double* bc, double* irdv, int kb, DevStatus* st, int where0) {
  const int lane = threadIdx.x & 31, i = lane & 15;
  const bool own = lane < 16;
  double x[16];
  const double* drow = D + (kb + i) * LD + kb;
#pragma unroll
  for (int c = 0; c < 16; ++c) x[c] = drow[c];
  double piv = __shfl_sync(0xffffffffu, x[0], 0);
  int bad = (piv > 0.0) ? 16 : 0;  // first non-positive pivot, 16 = none
  piv = (piv > 0.0) ? piv : 1.0;
  double ird = rsqrt(piv);
#pragma unroll
  for (int p = 0; p < 16; ++p) {
    const double lv = (i == p) ? piv * ird : x[0] * ird;  // L_ip for rows i >= p
    double pn = __shfl_sync(0xffffffffu, fma(-lv, lv, x[1]), (p + 1) & 15);
    bad = (bad == 16 && p < 15 && !(pn > 0.0)) ? p + 1 : bad;
    pn = (pn > 0.0) ? pn : 1.0;
    const double irn = rsqrt(pn);
    double* b = bc + (p & 1) * 48;
    if (own && i >= p) D[(kb + i) * LD + kb + p] = lv;
    if (own && i > p) b[15 + i - p] = lv;  // slot c = i - p - 1 at b[16 + c]
    if (lane == 0) irdv[kb + p] = ird;
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 14; c += 2) {
      const double2 v = *reinterpret_cast<const double2*>(b + 16 + c);
      x[c] = fma(-lv, v.x, x[c + 1]);
      x[c + 1] = fma(-lv, v.y, x[c + 2]);
    }
    x[14] = fma(-lv, b[30], x[15]);
    x[15] = 0.0;
    piv = pn;
    ird = irn;
  }
  if (bad < 16 && lane == 0) record_failure(st, kStatusNotPD, where0 + bad);
}

// Warp 1: M_DD = L_DD^-1 of the 16 x 16 sub-block at kb, into Mi (zeros above
// the diagonal). Lane j < 16 forms column j by forward substitution,
// M_ij = -(1 / L_ii) sum_{k < i} L_ik M_kj.
__device__ __forceinline__ void invert16(const double* D, double* Mi, const double* irdv, int kb) {
  const int j = threadIdx.x & 15;
  double m[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    double a0 = 0.0, a1 = 0.0;
#pragma unroll
    for (int k = 0; k < i; ++k) {
      const double l = D[(kb + i) * LD + kb + k];
      if (k & 1) a1 = fma(l, m[k], a1);
      else a0 = fma(l, m[k], a0);
    }
    const double r = irdv[kb + i];
    m[i] = (i == j) ? r : ((i > j) ? -r * (a0 + a1) : 0.0);
  }
  if ((threadIdx.x & 31) < 16) {
#pragma unroll
    for (int i = 0; i < 16; ++i) Mi[(kb + i) * LD + kb + j] = m[i];
  }
}

// One thread per row r of the sub-panel below the sub-block at kb: the row
// becomes L, P = A L_DD^-T, by forward substitution along the 16 columns.
__device__ __forceinline__ void trsm16_row(double* D, const double* irdv, int kb, int r) {
  double a[16];
#pragma unroll
  for (int c = 0; c < 16; c += 2) {
    const double2 v = *reinterpret_cast<const double2*>(D + r * LD + kb + c);
    a[c] = v.x;
    a[c + 1] = v.y;
  }
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    a[c] *= irdv[kb + c];
#pragma unroll
    for (int c2 = c + 1; c2 < 16; ++c2) a[c2] = fma(-a[c], D[(kb + c2) * LD + kb + c], a[c2]);
  }
#pragma unroll
  for (int c = 0; c < 16; c += 2) *reinterpret_cast<double2*>(D + r * LD + kb + c) = make_double2(a[c], a[c + 1]);
}

// All 256 threads: factor the nb x nb block in D (lower triangle) in 16-wide
// steps; D receives L, Mi (zero above its diagonal 16 x 16 blocks on entry)
// receives L^-1. scr: kFacScratch doubles of shared memory.
//   per step: warp 0 factors the 16 x 16 diagonal piece (factor16); then warp 1
//   inverts it while warps 2..7 turn the rows below into L (one row each); the
//   trailing lower triangle takes the rank-16 update (tensor-core pieces).
//   The off-diagonal blocks of L^-1 then follow from
//   [[A, 0], [B, C]]^-1 = [[A^-1, 0], [-C^-1 B A^-1, C^-1]] at 16 and 32.
__device__ void factor_block(double* D, double* Mi, double* scr, int nb, DevStatus* st, int where0) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, kq = lane & 3;
  double* bc = scr;
  double* irdv = scr + 96;
  for (int kb = 0; kb < nb; kb += 16) {
    if (w == 0) factor16(D, bc, irdv, kb, st, where0 + kb);
    __syncthreads();
    const int r0 = kb + 16, R = nb - r0;
    if (w == 1) invert16(D, Mi, irdv, kb);
    else if (w >= 2 && (int)threadIdx.x - 64 < R) trsm16_row(D, irdv, kb, r0 + (int)threadIdx.x - 64);
    __syncthreads();
    if (R <= 0) break;
    // trailing lower triangle, 8 x 8 pieces (tr, ts), ts <= tr
    const int tn = R / 8, ntri = tn * (tn + 1) / 2;
    for (int t = w; t < ntri; t += 8) {
      int tr = 0;
      while ((tr + 1) * (tr + 2) / 2 <= t) ++tr;
      const int ts = t - tr * (tr + 1) / 2;
      double* cp = D + (r0 + 8 * tr + g) * LD + r0 + 8 * ts + 2 * kq;
      const double2 v = *reinterpret_cast<const double2*>(cp);
      double c[2] = {v.x, v.y};
      const double* ar = D + (r0 + 8 * tr + g) * LD + kb + kq;
      const double* br = D + (r0 + 8 * ts + g) * LD + kb + kq;
#pragma unroll
      for (int k = 0; k < 16; k += 4) dmma(c, -ar[k], br[k]);
      *reinterpret_cast<double2*>(cp) = make_double2(c[0], c[1]);
    }
    __syncthreads();
  }
  // inverse, 16-level: pairs of 16-blocks at q = 0 and (nb = 64) q = 32
  {
    const int npair = nb / 32, q = 32 * (w >> 2), mt = (w >> 1) & 1, nt = w & 1;
    const bool act = w < 4 * npair;
    double t1[2] = {0.0, 0.0};
    if (act) {  // T = L_{hi,lo} M_lo, stored where M_{hi,lo} goes
      const double* ar = D + (q + 16 + 8 * mt + g) * LD + q + kq;
#pragma unroll
      for (int k = 0; k < 16; k += 4) dmma(t1, ar[k], Mi[(q + k + kq) * LD + q + 8 * nt + g]);
      *reinterpret_cast<double2*>(Mi + (q + 16 + 8 * mt + g) * LD + q + 8 * nt + 2 * kq) = make_double2(t1[0], t1[1]);
    }
    __syncthreads();
    double t2[2] = {0.0, 0.0};
    if (act) {  // M_{hi,lo} = -M_hi T
      const double* ar = Mi + (q + 16 + 8 * mt + g) * LD + q + 16 + kq;
#pragma unroll
      for (int k = 0; k < 16; k += 4) dmma(t2, -ar[k], Mi[(q + 16 + k + kq) * LD + q + 8 * nt + g]);
    }
    __syncthreads();
    if (act)
      *reinterpret_cast<double2*>(Mi + (q + 16 + 8 * mt + g) * LD + q + 8 * nt + 2 * kq) = make_double2(t2[0], t2[1]);
    __syncthreads();
  }
  if (nb == 64) {  // 32-level: M_BA = -M_B (L_BA M_A), 16 pieces of 8 x 8, two per warp
    double u[2][2];
#pragma unroll
    for (int q2 = 0; q2 < 2; ++q2) {
      const int t = w + 8 * q2, mt = t >> 2, nt = t & 3;
      u[q2][0] = u[q2][1] = 0.0;
      const double* ar = D + (32 + 8 * mt + g) * LD + kq;
#pragma unroll
      for (int k = 0; k < 32; k += 4) dmma(u[q2], ar[k], Mi[(k + kq) * LD + 8 * nt + g]);
      *reinterpret_cast<double2*>(Mi + (32 + 8 * mt + g) * LD + 8 * nt + 2 * kq) = make_double2(u[q2][0], u[q2][1]);
    }
    __syncthreads();
#pragma unroll
    for (int q2 = 0; q2 < 2; ++q2) {
      const int t = w + 8 * q2, mt = t >> 2, nt = t & 3;
      u[q2][0] = u[q2][1] = 0.0;
      const double* ar = Mi + (32 + 8 * mt + g) * LD + 32 + kq;
#pragma unroll
      for (int k = 0; k < 32; k += 4) dmma(u[q2], -ar[k], Mi[(32 + k + kq) * LD + 8 * nt + g]);
    }
    __syncthreads();
#pragma unroll
    for (int q2 = 0; q2 < 2; ++q2) {
      const int t = w + 8 * q2, mt = t >> 2, nt = t & 3;
      *reinterpret_cast<double2*>(Mi + (32 + 8 * mt + g) * LD + 8 * nt + 2 * kq) = make_double2(u[q2][0], u[q2][1]);
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- Cholesky kernels
constexpr size_t kPpSmem = 2 * kTileBytes + kFacScratch * sizeof(double);

// D's 36 lower 8 x 8 pieces -= U U^T over k < 64. Warp w takes pieces w, w + 8,
// ... (five at most, updated together), so the two warps of each SM
// sub-partition (w and w + 4) hold nine pieces between them.
__device__ __forceinline__ void lower_update(double* D, const double* U) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, kq = lane & 3;
  double c[5][2];
  int ao[5], bo[5], co[5];
#pragma unroll
  for (int q = 0; q < 5; ++q) {
    const int t0 = w + 8 * q, t = (t0 < 36) ? t0 : 0;
    int tr = 0;
    while ((tr + 1) * (tr + 2) / 2 <= t) ++tr;
    const int ts = t - tr * (tr + 1) / 2;
    co[q] = (8 * tr + g) * LD + 8 * ts + 2 * kq;
    ao[q] = (8 * tr + g) * LD + kq;
    bo[q] = (8 * ts + g) * LD + kq;
    const double2 v = *reinterpret_cast<const double2*>(D + co[q]);
    c[q][0] = v.x;
    c[q][1] = v.y;
  }
  const bool five = w + 32 < 36;
#pragma unroll 2
  for (int k = 0; k < NB; k += 4) {
#pragma unroll
    for (int q = 0; q < 4; ++q) dmma(c[q], -U[ao[q] + k], U[bo[q] + k]);
    if (five) dmma(c[4], -U[ao[4] + k], U[bo[4] + k]);
  }
#pragma unroll
  for (int q = 0; q < 4; ++q) *reinterpret_cast<double2*>(D + co[q]) = make_double2(c[q][0], c[q][1]);
  if (five) *reinterpret_cast<double2*>(D + co[4]) = make_double2(c[4][0], c[4][1]);
}

// L_IK = X Mi^T with Mi lower triangular (column j needs k <= j only), stored to
// G (rows < rows, columns < cols). Warp w owns rows 32 (w >> 2) .. + 31 and the
// 8-column pieces c0 = w & 3 and c1 = 7 - c0, so every warp does 18 k-steps
// per row piece.
__device__ __forceinline__ void panel_tri(const double* X, const double* Mi, int kn, double* G, int64_t ld, int rows,
                                          int cols) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, kq = lane & 3;
  const int rb = 32 * (w >> 2), c0 = w & 3, c1 = 7 - c0;
  const int k0end = min(8 * (c0 + 1), kn), k1end = min(8 * (c1 + 1), kn);
  double acc[4][2][2];
#pragma unroll
  for (int mi = 0; mi < 4; ++mi) acc[mi][0][0] = acc[mi][0][1] = acc[mi][1][0] = acc[mi][1][1] = 0.0;
  const double* xa = X + (rb + g) * LD + kq;
  const double* m0 = Mi + (8 * c0 + g) * LD + kq;
  const double* m1 = Mi + (8 * c1 + g) * LD + kq;
  for (int k = 0; k < k1end; k += 4) {
    double a[4];
#pragma unroll
    for (int mi = 0; mi < 4; ++mi) a[mi] = xa[8 * mi * LD + k];
    const double b1 = m1[k];
#pragma unroll
    for (int mi = 0; mi < 4; ++mi) dmma(acc[mi][1], a[mi], b1);
    if (k < k0end) {
      const double b0 = m0[k];
#pragma unroll
      for (int mi = 0; mi < 4; ++mi) dmma(acc[mi][0], a[mi], b0);
    }
  }
#pragma unroll
  for (int mi = 0; mi < 4; ++mi)
#pragma unroll
    for (int ci = 0; ci < 2; ++ci) {
      const int r = rb + 8 * mi + g, c = 8 * (ci ? c1 : c0) + 2 * kq;
      if (r < rows && c < cols)
        *reinterpret_cast<double2*>(G + (int64_t)r * ld + c) = make_double2(acc[mi][ci][0], acc[mi][ci][1]);
    }
}

// pp(K): grid T - K. Shared: D (block K), Mi (holds L_{K,K-1} until the
// update is applied, then L_KK^-1) and the factorization scratch, about 70 KB,
// so a pp CTA fits beside two trailing-update CTAs and starts as soon as one
// CTA of a full SM finishes. The block row I = K + b of column K and its
// L_{I,K-1} go straight from global memory (L2) into MMA fragments; the updated
// block stays in registers during the factorization and is staged in D's
// space for the panel product.
__global__ void __launch_bounds__(HT, 1) pp_kernel(double* __restrict__ A, double* __restrict__ M, int64_t n, int K,
                                                   DevStatus* st) {
  extern __shared__ __align__(16) double sm[];
  double* D = sm;
  double* Mi = sm + TILE;
  double* scr = sm + 2 * TILE;
  const int b = blockIdx.x, I = K + b;
  const int nbk = blk_size(n, K), nbi = blk_size(n, I);
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, kq = lane & 3;
  double* aKK = A + (int64_t)K * NB * n + (int64_t)K * NB;
  double* aIK = A + (int64_t)I * NB * n + (int64_t)K * NB;
  tile_load_async(D, aKK, n, nbk, nbk);
  if (K > 0) tile_load_async(Mi, aKK - NB, n, nbk, NB);
  cp_commit();
  Acc acc2;  // block row I of column K (b > 0)
  double ua[16][2];
  if (b > 0) {
    acc_from_global(acc2, aIK, n, nbi, nbk);
    if (K > 0) {  // A fragments of L_{I,K-1}: rows 16 (w >> 1) + g and + 8
      const int r0 = 16 * (w >> 1) + g;
      const double* u0 = aIK - NB + (int64_t)r0 * n + kq;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        ua[j][0] = (r0 < nbi) ? u0[4 * j] : 0.0;
        ua[j][1] = (r0 + 8 < nbi) ? u0[8 * n + 4 * j] : 0.0;
      }
    }
  }
  cp_wait_all();
  __syncthreads();
  // step K-1's update of column K: A_KK -= L L^T (lower pieces), A_IK -= L_{I,K-1} L_{K,K-1}^T
  if (K > 0) {
    lower_update(D, Mi);
    if (b > 0) {
      const int cb = 32 * (w & 1) + g;
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        double bb[4];
#pragma unroll
        for (int ni = 0; ni < 4; ++ni) bb[ni] = Mi[(cb + 8 * ni) * LD + 4 * j + kq];
#pragma unroll
        for (int mi = 0; mi < 2; ++mi)
#pragma unroll
          for (int ni = 0; ni < 4; ++ni) dmma(acc2[mi][ni], -ua[j][mi], bb[ni]);
      }
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < 6 * 16 * 8; e += HT) {  // zero the six 16 x 16 blocks above the diagonal ones
    const int blk = e >> 7, r = (e >> 3) & 15, c = (e & 7) * 2;
    const int bi = (blk < 3) ? 0 : ((blk < 5) ? 1 : 2);
    const int bj = (blk < 3) ? blk + 1 : ((blk < 5) ? blk - 1 : 3);
    *reinterpret_cast<double2*>(Mi + (16 * bi + r) * LD + 16 * bj + c) = make_double2(0.0, 0.0);
  }
  if (threadIdx.x < 96) scr[threadIdx.x] = 0.0;
  __syncthreads();
  factor_block(D, Mi, scr, nbk, st, K * NB);
  if (b > 0) {
    acc_to_smem(acc2, D);  // L_KK is stored by CTA 0; this CTA reuses D's space
    __syncthreads();
    panel_tri(D, Mi, nbk, aIK, n, nbi, nbk);
  } else {
    // Only M_KK goes out. L_KK stays in shared memory: no later kernel reads
    // a diagonal block of L, and writing it over A_KK here would race with
    // the CTAs of this launch that have not yet loaded A_KK (nothing makes
    // them resident at once).
    double* mKK = M + (int64_t)K * NB * n + (int64_t)K * NB;
    for (int e = threadIdx.x; e < nbk * nbk; e += HT) {
      const int r = e / nbk, c = e - r * nbk;
      mKK[(int64_t)r * n + c] = (c <= r) ? Mi[r * LD + c] : 0.0;
    }
  }
}

// lower-triangle tile index x -> (ti, tj), tj <= ti
__device__ __forceinline__ void tri_index(int x, int& ti, int& tj) {
  int t = (int)((sqrt(8.0 * (double)x + 1.0) - 1.0) * 0.5);
  while ((t + 1) * (t + 2) / 2 <= x) ++t;
  while (t * (t + 1) / 2 > x) --t;
  ti = t;
  tj = x - t * (t + 1) / 2;
}

// trail(K): A_IJ -= L_IK L_JK^T for K + 2 <= J <= I (one CTA per block).
__global__ void __launch_bounds__(HT, 3) trail_kernel(double* __restrict__ A, int64_t n, int K) {
  extern __shared__ __align__(16) double sm[];
  double* Ls = sm;
  double* Rs = sm + TILE;
  int ti, tj;
  tri_index(blockIdx.x, ti, tj);
  const int I = K + 2 + ti, J = K + 2 + tj;
  const int nbi = blk_size(n, I), nbj = blk_size(n, J);
  tile_load_async(Ls, A + (int64_t)I * NB * n + (int64_t)K * NB, n, nbi, NB);
  if (I != J) tile_load_async(Rs, A + (int64_t)J * NB * n + (int64_t)K * NB, n, nbj, NB);
  cp_commit();
  double* C = A + (int64_t)I * NB * n + (int64_t)J * NB;
  Acc acc;
  acc_from_global(acc, C, n, nbi, nbj);
  cp_wait_all();
  __syncthreads();
  warp_mma64<true, true>(acc, Ls, (I == J) ? Ls : Rs, NB);
  acc_to_global(acc, C, n, nbi, nbj);
}

// ---------------------------------------------------------------- inverse kernels
// rowmult(I): M_IJ = M_II R_IJ for J < I (one CTA per J), R_IJ stored in place.
__global__ void __launch_bounds__(HT, 3) rowmult_kernel(double* __restrict__ M, int64_t n, int I) {
  extern __shared__ __align__(16) double sm[];
  double* Ls = sm;
  double* Rs = sm + TILE;
  const int J = blockIdx.x;
  const int nbi = blk_size(n, I);
  double* r = M + (int64_t)I * NB * n + (int64_t)J * NB;
  tile_load_async(Ls, M + (int64_t)I * NB * n + (int64_t)I * NB, n, nbi, nbi);
  tile_load_async(Rs, r, n, nbi, NB);
  cp_commit();
  cp_wait_all();
  __syncthreads();
  Acc acc;
  acc_zero(acc);
  warp_mma64<false, false>(acc, Ls, Rs, nbi);
  acc_to_global(acc, r, n, nbi, NB);
}

// inv_update(I): R_I'J -= L_I'I M_IJ for I' > I, J <= I. Grid (T - 1 - I) x (I + 1).
__global__ void __launch_bounds__(HT, 3) inv_update_kernel(const double* __restrict__ L, double* __restrict__ M,
                                                           int64_t n, int I) {
  extern __shared__ __align__(16) double sm[];
  double* Ls = sm;
  double* Rs = sm + TILE;
  const int Ip = I + 1 + blockIdx.x, J = blockIdx.y;
  const int nbp = blk_size(n, Ip);
  tile_load_async(Ls, L + (int64_t)Ip * NB * n + (int64_t)I * NB, n, nbp, NB);
  tile_load_async(Rs, M + (int64_t)I * NB * n + (int64_t)J * NB, n, NB, NB);
  cp_commit();
  double* C = M + (int64_t)Ip * NB * n + (int64_t)J * NB;
  Acc acc;
  acc_from_global(acc, C, n, nbp, NB);
  cp_wait_all();
  __syncthreads();
  warp_mma64<false, true>(acc, Ls, Rs, NB);
  acc_to_global(acc, C, n, nbp, NB);
}

// ---------------------------------------------------------------- column norms
constexpr int kNormRows = 64;
constexpr int kSmsHint = 148;  // grid size hint of the streaming copy (a few blocks per SM)
// Partial column sums of squares of the lower triangle of M over runs of
// kNormRows rows; four independent chains per thread keep four loads in flight.
__global__ void colsumsq_partial_kernel(const double* __restrict__ M, int64_t ld, int64_t n,
                                        double* __restrict__ part) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  const int64_t r0 = (int64_t)blockIdx.y * kNormRows;
  const int64_t i1 = r0 + kNormRows < ld ? r0 + kNormRows : ld;
  const int64_t i0 = r0 < j ? j : r0;
  double a[4] = {0.0, 0.0, 0.0, 0.0};
  int64_t i = i0;
  for (; i + 3 < i1; i += 4) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const double v = M[(i + u) * ld + j];
      a[u] = fma(v, v, a[u]);
    }
  }
  for (; i < i1; ++i) {
    const double v = M[i * ld + j];
    a[0] = fma(v, v, a[0]);
  }
  part[(int64_t)blockIdx.y * n + j] = (a[0] + a[1]) + (a[2] + a[3]);
}
__global__ void colsumsq_final_kernel(const double* __restrict__ part, int nparts, int64_t n, double* __restrict__ h) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  double acc = 0.0;
  for (int p = 0; p < nparts; ++p) acc += part[(int64_t)p * n + j];
  h[j] = acc;
}

// ---------------------------------------------------------------- host side
// Per host thread and device: an origin stream, the three working streams
// (highest priority for the factorization chain, then the trailing updates,
// lowest for the inverse) and their events.
struct HinvStreams {
  int dev = -1;
  bool ok = false;
  cudaStream_t o = nullptr, p = nullptr, t = nullptr, s = nullptr;
  std::vector<cudaEvent_t> ev;
};
static HinvStreams& hinv_streams(int events) {
  thread_local HinvStreams hs[16];
  int dev = 0;
  cudaGetDevice(&dev);
  HinvStreams& x = hs[dev & 15];
  if (x.dev != dev) {
    int least = 0, greatest = 0;
    cudaDeviceGetStreamPriorityRange(&least, &greatest);
    x.ok = cudaStreamCreateWithFlags(&x.o, cudaStreamNonBlocking) == cudaSuccess &&
           cudaStreamCreateWithPriority(&x.p, cudaStreamNonBlocking, greatest) == cudaSuccess &&
           cudaStreamCreateWithPriority(&x.t, cudaStreamNonBlocking, (least + greatest) / 2) == cudaSuccess &&
           cudaStreamCreateWithPriority(&x.s, cudaStreamNonBlocking, least) == cudaSuccess;
    x.dev = dev;
  }
  while (x.ok && (int)x.ev.size() < events) {
    cudaEvent_t e;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) {
      x.ok = false;
      break;
    }
    x.ev.push_back(e);
  }
  return x;
}

size_t hinv_workspace_doubles(int64_t n) {
  const int64_t np = pad32(n);
  const int64_t parts = (np + kNormRows - 1) / kNormRows;
  return (size_t)(2 * np * np + parts * n + 64);
}

// Enqueue the whole computation on origin stream o (the working streams fork
// from it and join back). Returns the number of kernels.
static int enqueue_hinv(const double* H, int64_t n, double alpha, double* h, double* ws, DevStatus* st,
                        cudaStream_t o, HinvStreams& hs) {
  const int64_t np = pad32(n);
  double* A = ws;
  double* M = ws + np * np;
  const int64_t parts = (np + kNormRows - 1) / kNormRows;
  double* part = M + np * np;
  double* damp = part + parts * n;
  const int T = (int)((np + NB - 1) / NB);
  diag_sum_kernel<<<1, 1024, 0, o>>>(H, n, alpha, damp);
  damp_copy_kernel<<<kSmsHint * 8, 256, 0, o>>>(H, n, np, damp, A);
  cudaMemsetAsync(M, 0, (size_t)np * np * sizeof(double), o);
  cudaEvent_t* ePP = hs.ev.data();
  cudaEvent_t* eTr = ePP + T;
  cudaEvent_t* eX = eTr + T;  // fork, and one join per working stream
  cudaEventRecord(eX[0], o);
  cudaStreamWaitEvent(hs.p, eX[0], 0);
  cudaStreamWaitEvent(hs.t, eX[0], 0);
  cudaStreamWaitEvent(hs.s, eX[0], 0);
  int launches = 4;
  for (int K = 0; K < T; ++K) {
    if (K >= 2) cudaStreamWaitEvent(hs.p, eTr[K - 2], 0);
    pp_kernel<<<T - K, HT, kPpSmem, hs.p>>>(A, M, np, K, st);
    cudaEventRecord(ePP[K], hs.p);
    ++launches;
    const int rem = T - K - 2;
    if (rem > 0) {
      cudaStreamWaitEvent(hs.t, ePP[K], 0);
      trail_kernel<<<rem * (rem + 1) / 2, HT, 2 * kTileBytes, hs.t>>>(A, np, K);
      ++launches;
    }
    cudaEventRecord(eTr[K], hs.t);
    cudaStreamWaitEvent(hs.s, ePP[K], 0);
    if (K > 0) {
      rowmult_kernel<<<K, HT, 2 * kTileBytes, hs.s>>>(M, np, K);
      ++launches;
    }
    if (K < T - 1) {
      inv_update_kernel<<<dim3((unsigned)(T - 1 - K), (unsigned)(K + 1)), HT, 2 * kTileBytes, hs.s>>>(A, M, np, K);
      ++launches;
    }
  }
  cudaEventRecord(eX[1], hs.p);
  cudaEventRecord(eX[2], hs.t);
  cudaEventRecord(eX[3], hs.s);
  cudaStreamWaitEvent(o, eX[1], 0);
  cudaStreamWaitEvent(o, eX[2], 0);
  cudaStreamWaitEvent(o, eX[3], 0);
  colsumsq_partial_kernel<<<dim3((unsigned)((n + 255) / 256), (unsigned)parts), 256, 0, o>>>(M, np, n, part);
  colsumsq_final_kernel<<<(unsigned)((n + 255) / 256), 256, 0, o>>>(part, (int)parts, n, h);
  return launches;
}

// Per host thread and device: the executable graph of the last call's launch
// sequence and the arguments it was captured with. A call with other
// arguments re-captures (same n: the executable graph is updated in place).
// Graph launches cut the gaps between the several hundred dependent kernels
// that event waits across streams leave on a busy GPU; node priorities keep
// the factorization chain ahead.
struct HinvGraph {
  bool valid = false;
  int64_t n = 0;
  const double* H = nullptr;
  double alpha = 0.0;
  double* h = nullptr;
  double* ws = nullptr;
  DevStatus* st = nullptr;
  cudaGraphExec_t exec = nullptr;
  int launches = 0;
};

cudaError_t launch_hinv(const double* H, int64_t n, double alpha, double* h, double* ws, DevStatus* st,
                        cudaStream_t s) {
  static std::atomic<uint64_t> attr{0};
  uint64_t bit = 0;
  if (attr_pending(attr, bit)) {
    cudaError_t e = cudaFuncSetAttribute(pp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPpSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(trail_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(2 * kTileBytes));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(rowmult_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(2 * kTileBytes));
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(inv_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(2 * kTileBytes));
    if (e != cudaSuccess) return e;
    attr.fetch_or(bit);
  }
  const int T = (int)((pad32(n) + NB - 1) / NB);
  HinvStreams& hs = hinv_streams(2 * T + 6);
  if (!hs.ok) return cudaErrorMemoryAllocation;
  thread_local HinvGraph graphs[16];
  int dev = 0;
  cudaGetDevice(&dev);
  HinvGraph& g = graphs[dev & 15];
  const bool hit = g.valid && g.n == n && g.H == H && g.alpha == alpha && g.h == h && g.ws == ws && g.st == st;
  if (!hit) {
    g.valid = false;
    cudaGraph_t graph = nullptr;
    int launches = 0;
    cudaError_t e = cudaStreamBeginCapture(hs.o, cudaStreamCaptureModeThreadLocal);
    if (e == cudaSuccess) {
      launches = enqueue_hinv(H, n, alpha, h, ws, st, hs.o, hs);
      e = cudaStreamEndCapture(hs.o, &graph);
    }
    if (e == cudaSuccess && g.exec) {
      cudaGraphExecUpdateResultInfo info;
      if (cudaGraphExecUpdate(g.exec, graph, &info) != cudaSuccess) {
        cudaGetLastError();
        cudaGraphExecDestroy(g.exec);
        g.exec = nullptr;
      }
    }
    if (e == cudaSuccess && !g.exec) e = cudaGraphInstantiateWithFlags(&g.exec, graph, cudaGraphInstantiateFlagUseNodePriority);
    if (graph) cudaGraphDestroy(graph);
    if (e != cudaSuccess) return e;
    g.valid = true;
    g.n = n;
    g.H = H;
    g.alpha = alpha;
    g.h = h;
    g.ws = ws;
    g.st = st;
    g.launches = launches;
  }
  cudaEvent_t* eIO = hs.ev.data() + 2 * T + 4;
  cudaEventRecord(eIO[0], s);
  cudaStreamWaitEvent(hs.o, eIO[0], 0);
  cudaGraphLaunch(g.exec, hs.o);
  cudaEventRecord(eIO[1], hs.o);
  cudaStreamWaitEvent(s, eIO[1], 0);
  count_launches(g.launches);
  return cudaGetLastError();
}

}  // namespace slim
