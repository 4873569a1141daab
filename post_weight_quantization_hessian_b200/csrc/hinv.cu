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
//               (L_KK, M_KK = L_KK^-1); CTA 0 stores them, CTA b > 0 updates
//               its block row I = K + b of column K and stores L_IK = A_IK M_KK^T
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

namespace slim {

constexpr int NB = 64;         // block size
constexpr int LD = 68;         // shared row stride in doubles: 16-byte rows, conflict-free fragment loads
constexpr int TILE = NB * LD;  // doubles per shared tile
constexpr int HT = 256;        // threads per CTA of every blocked kernel
constexpr size_t kTileBytes = TILE * sizeof(double);

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
// identity block on the padding, zeros elsewhere.
__global__ void damp_copy_kernel(const double* __restrict__ H, int64_t n, int64_t np, const double* __restrict__ damp,
                                 double* __restrict__ A) {
  const double dv = damp[0];
  for (int64_t i = blockIdx.y; i < np; i += gridDim.y)
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < np; j += (int64_t)gridDim.x * blockDim.x) {
      double v = 0.0;
      if (i < n && j < n) {
        if (j < i) v = H[i * n + j];
        else if (j == i) {
          const double d = H[i * n + i];
          v = ((d == 0.0) ? 1.0 : d) + dv;
        }
      } else if (i == j) {
        v = 1.0;
      }
      A[i * np + j] = v;
    }
}

// ---------------------------------------------------------------- tiles and fp64 MMA
__device__ __forceinline__ void cp16(double* sdst, const double* gsrc, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(smem_u32(sdst)), "l"(gsrc),
               "r"(valid ? 16 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
__device__ __forceinline__ void cp_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::: "memory"); }

// Queue the copy of a rows x cols block of G (leading dimension ld) into the
// shared tile S; zeros outside the block. cols is even.
__device__ __forceinline__ void tile_load_async(double* S, const double* G, int64_t ld, int rows, int cols) {
#pragma unroll
  for (int q = 0; q < NB * NB / 2 / HT; ++q) {
    const int e = threadIdx.x + HT * q;
    const int r = e >> 5, c = (e & 31) * 2;
    const bool v = (r < rows) && (c < cols);
    cp16(S + r * LD + c, v ? G + (int64_t)r * ld + c : G, v);
  }
}

// d (8 x 8, two per lane) += a (8 x 4) * b (4 x 8)
__device__ __forceinline__ void dmma(double (&d)[2], double a, double b) {
  asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
      : "+d"(d[0]), "+d"(d[1])
      : "d"(a), "d"(b));
}

// Warp w of 8 owns rows 16 (w >> 1) .. + 15 and columns 32 (w & 1) .. + 31 of a
// 64 x 64 result: acc[mi][ni] is the 8 x 8 piece at row 16 (w >> 1) + 8 mi,
// column 32 (w & 1) + 8 ni; a lane holds row (lane >> 2), columns 2 (lane & 3)
// and 2 (lane & 3) + 1 of each piece.
using Acc = double[2][4][2];

__device__ __forceinline__ void acc_zero(Acc& acc) {
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int ni = 0; ni < 4; ++ni) acc[mi][ni][0] = acc[mi][ni][1] = 0.0;
}

__device__ __forceinline__ int acc_row(int mi) { return 16 * (threadIdx.x >> 6) + 8 * mi + ((threadIdx.x & 31) >> 2); }
__device__ __forceinline__ int acc_col(int ni) { return 32 * ((threadIdx.x >> 5) & 1) + 8 * ni + 2 * (threadIdx.x & 3); }

__device__ __forceinline__ void acc_from_smem(Acc& acc, const double* S) {
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int ni = 0; ni < 4; ++ni) {
      const double2 v = *reinterpret_cast<const double2*>(S + acc_row(mi) * LD + acc_col(ni));
      acc[mi][ni][0] = v.x;
      acc[mi][ni][1] = v.y;
    }
}
__device__ __forceinline__ void acc_to_smem(const Acc& acc, double* S) {
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int ni = 0; ni < 4; ++ni)
      *reinterpret_cast<double2*>(S + acc_row(mi) * LD + acc_col(ni)) = make_double2(acc[mi][ni][0], acc[mi][ni][1]);
}
__device__ __forceinline__ void acc_from_global(Acc& acc, const double* G, int64_t ld, int rows, int cols) {
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int ni = 0; ni < 4; ++ni) {
      const int r = acc_row(mi), c = acc_col(ni);
      double2 v = make_double2(0.0, 0.0);
      if (r < rows && c < cols) v = *reinterpret_cast<const double2*>(G + (int64_t)r * ld + c);
      acc[mi][ni][0] = v.x;
      acc[mi][ni][1] = v.y;
    }
}
__device__ __forceinline__ void acc_to_global(const Acc& acc, double* G, int64_t ld, int rows, int cols) {
#pragma unroll
  for (int mi = 0; mi < 2; ++mi)
#pragma unroll
    for (int ni = 0; ni < 4; ++ni) {
      const int r = acc_row(mi), c = acc_col(ni);
      if (r < rows && c < cols)
        *reinterpret_cast<double2*>(G + (int64_t)r * ld + c) = make_double2(acc[mi][ni][0], acc[mi][ni][1]);
    }
}

// acc += (NEG ? -1 : 1) * sum_{k < kn} As[row][k] * B(k, col), kn a multiple of 4.
// BT: Bs holds B transposed (Bs[col][k], the product is As Bs^T); else Bs[k][col].
template <bool BT, bool NEG>
__device__ __forceinline__ void warp_mma64(Acc& acc, const double* As, const double* Bs, int kn) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, kq = lane & 3;
  const double* a0 = As + (16 * (w >> 1) + g) * LD + kq;
  const int cb = 32 * (w & 1) + g;
#pragma unroll 4
  for (int k = 0; k < kn; k += 4) {
    double a[2], b[4];
    a[0] = a0[k];
    a[1] = a0[8 * LD + k];
    if (NEG) {
      a[0] = -a[0];
      a[1] = -a[1];
    }
#pragma unroll
    for (int ni = 0; ni < 4; ++ni) b[ni] = BT ? Bs[(cb + 8 * ni) * LD + k + kq] : Bs[(k + kq) * LD + cb + 8 * ni];
#pragma unroll
    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
      for (int ni = 0; ni < 4; ++ni) dmma(acc[mi][ni], a[mi], b[ni]);
  }
}

// ---------------------------------------------------------------- diagonal block
// Warp 0: unblocked Cholesky of the 16 x 16 sub-block at (kb, kb) of D and its
// inverse, in registers. Lanes 0..15 own the rows of L: lane i keeps row i of
// the not yet factored columns, shifted so that x[0] is always the current
// pivot column (so every register index is static while the pivot loop stays
// a compact loop). Lanes 16..31 own the rows of the inverse, built right-
// looking: at pivot p, row p becomes final (scaled by 1/L_pp) and is removed
// from the rows below. Each pivot broadcasts, in one shuffle per column, the
// new L column to the L lanes and row p of the inverse to the inverse lanes.
// L is written into D (rows >= p of column p); the inverse into Mi.
__device__ __forceinline__ void factor16(double* D, double* Mi, int kb, DevStatus* st, int where0) {
  const int lane = threadIdx.x & 31, i = lane & 15;
  const bool lo = lane < 16;
  double x[16];
  const double* drow = D + (kb + i) * LD + kb;
#pragma unroll
  for (int c = 0; c < 16; ++c) x[c] = lo ? drow[c] : ((c == i) ? 1.0 : 0.0);
  double piv = __shfl_sync(0xffffffffu, x[0], 0);
#pragma unroll 1
  for (int p = 0; p < 16; ++p) {
    if (!(piv > 0.0)) {
      if (lane == 0) record_failure(st, kStatusNotPD, where0 + p);
      piv = 1.0;
    }
    const double ird = rsqrt(piv);
    const double lv = (i == p) ? piv * ird : x[0] * ird;  // L lanes, rows i >= p: L_ip
    const double lg = __shfl_sync(0xffffffffu, lv, i);     // inverse lanes: L_ip of their row
    const double tn = fma(-lv, lv, x[1]);                  // lane p + 1: the next pivot
    if (lo && i >= p) D[(kb + i) * LD + kb + p] = lv;
    // L lanes: x[c] <- x[c + 1] - L_ip L_{p+1+c, p}; inverse lanes: x[c] <- x[c] - L_ip M_pc
    // (row i > p), M_pc = R_pc / L_pp (row p), unchanged (rows i < p).
    const double alpha = lo ? -lv : ((i > p) ? -lg * ird : ((i == p) ? ird : 0.0));
    const double beta = (lo || i != p) ? 1.0 : 0.0;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
      const double y = lo ? lv : x[c];
      const double gv = __shfl_sync(0xffffffffu, y, lo ? ((p + 1 + c) & 31) : (16 + p));
      const double base = lo ? ((c < 15) ? x[c + 1] : 0.0) : x[c];
      x[c] = fma(alpha, gv, beta * base);
    }
    piv = __shfl_sync(0xffffffffu, tn, (p + 1) & 31);
  }
  if (!lo) {
#pragma unroll
    for (int c = 0; c < 16; ++c) Mi[(kb + i) * LD + kb + c] = (c <= i) ? x[c] : 0.0;
  }
}

// All 256 threads: factor the nb x nb block in D (lower triangle) in 16-wide
// steps; D receives L, Mi (zero on entry) receives L^-1.
//   per step: warp 0 factors the 16 x 16 diagonal piece (factor16); the piece
//   below it becomes L (P = A M_DD^T); the trailing lower triangle takes the
//   rank-16 update. The off-diagonal blocks of L^-1 then follow from
//   [[A, 0], [B, C]]^-1 = [[A^-1, 0], [-C^-1 B A^-1, C^-1]] at 16 and 32.
__device__ void factor_block(double* D, double* Mi, int nb, DevStatus* st, int where0) {
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, kq = lane & 3;
  for (int kb = 0; kb < nb; kb += 16) {
    if (w == 0) factor16(D, Mi, kb, st, where0 + kb);
    __syncthreads();
    const int r0 = kb + 16, R = nb - r0;
    if (R <= 0) break;
    // sub-panel: R x 16 pieces of 8 x 8 (R / 4 of them, at most 12), two per warp at most
    const int npc = R / 4;
    double pv[2][2];
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int t = w + 8 * q;
      pv[q][0] = pv[q][1] = 0.0;
      if (t < npc) {
        const int mt = t >> 1, nt = t & 1;
        const double* ar = D + (r0 + 8 * mt + g) * LD + kb + kq;
        const double* br = Mi + (kb + 8 * nt + g) * LD + kb + kq;
#pragma unroll
        for (int k = 0; k < 16; k += 4) dmma(pv[q], ar[k], br[k]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int t = w + 8 * q;
      if (t < npc) {
        const int mt = t >> 1, nt = t & 1;
        *reinterpret_cast<double2*>(D + (r0 + 8 * mt + g) * LD + kb + 8 * nt + 2 * kq) = make_double2(pv[q][0], pv[q][1]);
      }
    }
    __syncthreads();
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
// pp(K): grid T - K. Shared: D (block K), Mi (holds L_{K,K-1} until the update
// is applied, then L_KK^-1), X (block row I of column K), U (L_{I,K-1}).
__global__ void __launch_bounds__(HT, 1) pp_kernel(double* __restrict__ A, double* __restrict__ M, int64_t n, int K,
                                                   DevStatus* st) {
  extern __shared__ __align__(16) double sm[];
  double* D = sm;
  double* Mi = sm + TILE;
  double* X = sm + 2 * TILE;
  double* U = sm + 3 * TILE;
  const int b = blockIdx.x, I = K + b;
  const int nbk = blk_size(n, K), nbi = blk_size(n, I);
  double* aKK = A + (int64_t)K * NB * n + (int64_t)K * NB;
  double* aIK = A + (int64_t)I * NB * n + (int64_t)K * NB;
  tile_load_async(D, aKK, n, nbk, nbk);
  if (K > 0) tile_load_async(Mi, aKK - NB, n, nbk, NB);
  if (b > 0) {
    tile_load_async(X, aIK, n, nbi, nbk);
    if (K > 0) tile_load_async(U, aIK - NB, n, nbi, NB);
  }
  cp_commit();
  cp_wait_all();
  __syncthreads();
  if (K > 0) {  // step K-1's update of column K: A_KK -= L L^T, A_IK -= L_{I,K-1} L_{K,K-1}^T
    Acc acc, acc2;
    acc_from_smem(acc, D);
    warp_mma64<true, true>(acc, Mi, Mi, NB);
    if (b > 0) {
      acc_from_smem(acc2, X);
      warp_mma64<true, true>(acc2, U, Mi, NB);
    }
    __syncthreads();
    acc_to_smem(acc, D);
    if (b > 0) acc_to_smem(acc2, X);
  }
  for (int e = threadIdx.x; e < TILE; e += HT) Mi[e] = 0.0;
  __syncthreads();
  factor_block(D, Mi, nbk, st, K * NB);
  if (b > 0) {
    Acc acc;
    acc_zero(acc);
    warp_mma64<true, false>(acc, X, Mi, nbk);
    acc_to_global(acc, aIK, n, nbi, nbk);
  } else {
    double* mKK = M + (int64_t)K * NB * n + (int64_t)K * NB;
    for (int e = threadIdx.x; e < nbk * nbk; e += HT) {
      const int r = e / nbk, c = e - r * nbk;
      aKK[(int64_t)r * n + c] = (c <= r) ? D[r * LD + c] : 0.0;
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
constexpr int kNormRows = 128;
__global__ void colsumsq_partial_kernel(const double* __restrict__ M, int64_t ld, int64_t n,
                                        double* __restrict__ part) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  int64_t i0 = (int64_t)blockIdx.y * kNormRows;
  int64_t i1 = i0 + kNormRows < ld ? i0 + kNormRows : ld;
  if (i0 < j) i0 = j;
  double acc = 0.0;
  for (int64_t i = i0; i < i1; ++i) {
    const double v = M[i * ld + j];
    acc = fma(v, v, acc);
  }
  part[(int64_t)blockIdx.y * n + j] = acc;
}
__global__ void colsumsq_final_kernel(const double* __restrict__ part, int nparts, int64_t n, double* __restrict__ h) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  double acc = 0.0;
  for (int p = 0; p < nparts; ++p) acc += part[(int64_t)p * n + j];
  h[j] = acc;
}

// ---------------------------------------------------------------- host side
// Per host thread and device: the three streams (highest priority for the
// factorization chain, then the trailing updates, lowest for the inverse) and
// their events.
struct HinvStreams {
  int dev = -1;
  bool ok = false;
  cudaStream_t p = nullptr, t = nullptr, s = nullptr;
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
    x.ok = cudaStreamCreateWithPriority(&x.p, cudaStreamNonBlocking, greatest) == cudaSuccess &&
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

cudaError_t launch_hinv(const double* H, int64_t n, double alpha, double* h, double* ws, DevStatus* st,
                        cudaStream_t s) {
  const int64_t np = pad32(n);
  double* A = ws;
  double* M = ws + np * np;
  const int64_t parts = (np + kNormRows - 1) / kNormRows;
  double* part = M + np * np;
  double* damp = part + parts * n;
  static bool attr_done = false;
  if (!attr_done) {
    cudaFuncSetAttribute(pp_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(4 * kTileBytes));
    cudaFuncSetAttribute(trail_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(2 * kTileBytes));
    cudaFuncSetAttribute(rowmult_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(2 * kTileBytes));
    cudaFuncSetAttribute(inv_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(2 * kTileBytes));
    attr_done = true;
  }
  diag_sum_kernel<<<1, 1024, 0, s>>>(H, n, alpha, damp);
  damp_copy_kernel<<<dim3((unsigned)((np + 255) / 256), (unsigned)(np < 65535 ? np : 65535)), 256, 0, s>>>(H, n, np, damp,
                                                                                                      A);
  cudaMemsetAsync(M, 0, (size_t)np * np * sizeof(double), s);
  const int T = (int)((np + NB - 1) / NB);
  HinvStreams& hs = hinv_streams(2 * T + 4);
  if (!hs.ok) return cudaErrorMemoryAllocation;
  cudaEvent_t* ePP = hs.ev.data();
  cudaEvent_t* eTr = ePP + T;
  cudaEvent_t* eX = eTr + T;  // fork, and one join per stream
  cudaEventRecord(eX[0], s);
  cudaStreamWaitEvent(hs.p, eX[0], 0);
  cudaStreamWaitEvent(hs.t, eX[0], 0);
  cudaStreamWaitEvent(hs.s, eX[0], 0);
  int launches = 0;
  for (int K = 0; K < T; ++K) {
    if (K >= 2) cudaStreamWaitEvent(hs.p, eTr[K - 2], 0);
    pp_kernel<<<T - K, HT, 4 * kTileBytes, hs.p>>>(A, M, np, K, st);
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
  cudaStreamWaitEvent(s, eX[1], 0);
  cudaStreamWaitEvent(s, eX[2], 0);
  cudaStreamWaitEvent(s, eX[3], 0);
  colsumsq_partial_kernel<<<dim3((unsigned)((n + 255) / 256), (unsigned)parts), 256, 0, s>>>(M, np, n, part);
  colsumsq_final_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(part, (int)parts, n, h);
  count_launches(2 + launches + 2);
  return cudaGetLastError();
}

}  // namespace slim
