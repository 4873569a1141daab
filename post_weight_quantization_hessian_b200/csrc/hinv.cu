// hinv_diag: h_j = [H_d^-1]_jj, the inverse-Hessian diagonal of the salience
// formula (SliM-LLM write-up, rkmt.cn, section 组件一 SBA).
//
// H_d = H with zero diagonal entries set to 1, plus alpha * mean(diag) on the
// diagonal. With H_d = L L^T, H_d^-1 = L^-T L^-1, so h_j is the squared norm of
// column j of M = L^-1. All arithmetic is fp64 on the CUDA cores, in 64 x 64
// blocks (T = ceil(n / 64) block rows, the last one possibly 32 wide):
//
//   Cholesky, right-looking, per diagonal block K:
//     potrf_diag   one CTA: L_KK = chol(A_KK) in shared memory, M_KK = L_KK^-1
//     panel        L_IK = A_IK M_KK^T for every block row I > K
//     syrk         A_IJ -= L_IK L_JK^T for K < J <= I (lower tiles only)
//   Inverse, forward substitution of L M = I, right-looking, per block row I:
//     rowmult      M_IJ = M_II R_IJ for J < I (R accumulates -sum L_IK M_KJ)
//     update       R_I'J -= L_I'I M_IJ for I' > I, J <= I
//   Column norms   h_j = sum_{i >= j} M_ij^2 (partials, then a fixed-order sum)
// The inverse steps run on a side stream, overlapping the Cholesky chain.
//
// Flops are n^3/3 for each half. A non-positive pivot records SLIM_ENOTPD with
// its index; the remaining kernels run to completion on the bad values.
#include <cstdint>
#include <vector>
#include "common.cuh"

namespace slim {

constexpr int NB = 64;
constexpr int LDS = NB + 1;  // padded shared-memory row (doubles)

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

// A = lower triangle of H with the dead-column fix and damping; upper part 0.
__global__ void damp_copy_kernel(const double* __restrict__ H, int64_t n, const double* __restrict__ damp,
                                 double* __restrict__ A) {
  const int64_t i = blockIdx.y;
  const double dv = damp[0];
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n; j += (int64_t)gridDim.x * blockDim.x) {
    double v = 0.0;
    if (j < i) v = H[i * n + j];
    else if (j == i) {
      const double d = H[i * n + i];
      v = ((d == 0.0) ? 1.0 : d) + dv;
    }
    A[i * n + j] = v;
  }
}

// ---------------------------------------------------------------- tile helpers
// Load a (rows x cols) block at G (row-major, leading dim ld) into S[64][LDS],
// either as is (S[r][c] = G[r][c]) or transposed (S[c][r] = G[r][c]); zero fill.
// 256 threads, 16 elements each, all loads issued before the first store.
__device__ __forceinline__ void load_tile(double (*S)[LDS], const double* G, int64_t ld, int rows, int cols,
                                          bool transpose) {
  double v[16];
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int e = threadIdx.x + 256 * k, r = e / NB, c = e % NB;
    v[k] = (r < rows && c < cols) ? G[(int64_t)r * ld + c] : 0.0;
  }
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const int e = threadIdx.x + 256 * k, r = e / NB, c = e % NB;
    if (transpose) S[c][r] = v[k]; else S[r][c] = v[k];
  }
}

// acc[r][c] = sum_l At[l][ty + 16 r] * B[l][tx + 16 c]   (256 threads)
__device__ __forceinline__ void tile_mma(const double (*At)[LDS], const double (*B)[LDS], double (&acc)[4][4], int kdim) {
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.0;
  for (int l = 0; l < kdim; ++l) {
    double a[4], b[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) a[r] = At[l][ty + 16 * r];
#pragma unroll
    for (int c = 0; c < 4; ++c) b[c] = B[l][tx + 16 * c];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = fma(a[r], b[c], acc[r][c]);
  }
}

__host__ __device__ inline int blk_size(int64_t n, int b) {
  const int64_t s = n - (int64_t)b * NB;
  return (int)(s < NB ? s : NB);
}

// ---------------------------------------------------------------- Cholesky pieces
// Factor diagonal block K of A in place; write M_KK = L_KK^-1 into M.
//
// The pivots of a Cholesky factorization form a sequential chain (n of them
// over the whole matrix), so each pivot step must be cheap. The 64 x 64 block
// is processed in 16-wide sub-blocks:
//   (1) warp 0 factors the 16 x 16 diagonal sub-block in shared memory (one
//       rsqrt per pivot, warp-level synchronization only) and, in the same
//       pivot loop, inverts it (right-looking: row p of M is row p of R
//       scaled by 1/L_pp, then R_ic -= L_ip M_pc for i > p, c <= p);
//   (2) all warps compute the sub-panel below it, P = A_panel M_DD^T;
//   (3) all warps apply the rank-16 update to the trailing lower triangle.
// After the last sub-block, the off-diagonal 16 x 16 blocks of M = L^-1 come
// from block forward substitution, M_IJ = -M_II sum_{K=J}^{I-1} L_IK M_KJ.
constexpr int SB16 = 16;
__global__ void __launch_bounds__(256) potrf_diag_kernel(double* __restrict__ A, double* __restrict__ M, int64_t n,
                                                         int K, DevStatus* st) {
  extern __shared__ double smem[];
  double (*s)[LDS] = reinterpret_cast<double (*)[LDS]>(smem);
  double (*mi)[LDS] = reinterpret_cast<double (*)[LDS]>(smem + NB * LDS);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nb = blk_size(n, K);
  const int64_t off = (int64_t)K * NB * n + (int64_t)K * NB;
  {
    double v[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int e = tid + 256 * k, r = e / NB, c = e % NB;
      v[k] = (r < nb && c < nb && c <= r) ? A[off + (int64_t)r * n + c] : 0.0;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const int e = tid + 256 * k, r = e / NB, c = e % NB;
      s[r][c] = v[k];
      mi[r][c] = (r == c) ? 1.0 : 0.0;
    }
  }
  __syncthreads();
  for (int kb = 0; kb < nb; kb += SB16) {
    const int w = (nb - kb < SB16) ? nb - kb : SB16;
    if (warp == 0) {
      // (1) unblocked Cholesky of the 16 x 16 diagonal sub-block, and its inverse, in
      // registers: lane = row i (lane & 15), columns 8h .. 8h+7 (h = lane >> 4). Each
      // pivot's column and row travel by shuffles; the loop is unrolled so register
      // slots are static. (n is a multiple of 32, so sub-blocks are always 16 wide.)
      const int i = lane & 15, h = lane >> 4;
      double a[8], r[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        a[c] = s[kb + i][kb + 8 * h + c];
        r[c] = (i == 8 * h + c) ? 1.0 : 0.0;
      }
#pragma unroll
      for (int p = 0; p < SB16; ++p) {
        const int ph = p >> 3, pc = p & 7;
        double d = __shfl_sync(0xffffffffu, a[pc], p + 16 * ph);
        if (!(d > 0.0)) {
          if (lane == 0) record_failure(st, kStatusNotPD, K * NB + kb + p);
          d = 1.0;
        }
        const double ird = rsqrt(d);
        const double ci = __shfl_sync(0xffffffffu, a[pc], i + 16 * ph);   // unscaled a_ip
        const double fi = ci * ird;                                        // L_ip
        double cl[8], rp[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          cl[c] = __shfl_sync(0xffffffffu, a[pc], 8 * h + c + 16 * ph) * ird;   // L_lp
          rp[c] = __shfl_sync(0xffffffffu, r[c], p + 16 * h) * ird;             // M_pl
        }
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int l = 8 * h + c;
          if (l == p) a[c] = (i == p) ? d * ird : ((i > p) ? fi : a[c]);
          else if (l > p && l <= i) a[c] = fma(-fi, cl[c], a[c]);
          if (l <= p) {
            if (i == p) r[c] *= ird;
            else if (i > p) r[c] = fma(-fi, rp[c], r[c]);
          }
        }
      }
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        s[kb + i][kb + 8 * h + c] = a[c];
        mi[kb + i][kb + 8 * h + c] = r[c];
      }
    }
    __syncthreads();
    const int r0 = kb + w;
    if (r0 < nb) {
      // (2) sub-panel P[i][c] = sum_{l <= c} A[i][kb + l] M_DD[c][l], rows r0 .. nb-1
      const int rows = nb - r0;
      double pv[3];
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const int e = tid + 256 * q;
        pv[q] = 0.0;
        if (e < rows * w) {
          const int i = r0 + e / w, c = e % w;
          double a0 = 0.0, a1 = 0.0;
          int l = 0;
          for (; l + 1 <= c; l += 2) {
            a0 = fma(s[i][kb + l], mi[kb + c][kb + l], a0);
            a1 = fma(s[i][kb + l + 1], mi[kb + c][kb + l + 1], a1);
          }
          if (l <= c) a0 = fma(s[i][kb + l], mi[kb + c][kb + l], a0);
          pv[q] = a0 + a1;
        }
      }
      __syncthreads();
#pragma unroll
      for (int q = 0; q < 3; ++q) {
        const int e = tid + 256 * q;
        if (e < rows * w) s[r0 + e / w][kb + e % w] = pv[q];
      }
      __syncthreads();
      // (3) trailing update of the lower triangle, rank w
      for (int e = tid; e < rows * rows; e += blockDim.x) {
        const int i = r0 + e / rows, l = r0 + e % rows;
        if (l <= i) {
          double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
          int p = 0;
          for (; p + 3 < w; p += 4) {
            a0 = fma(s[i][kb + p], s[l][kb + p], a0);
            a1 = fma(s[i][kb + p + 1], s[l][kb + p + 1], a1);
            a2 = fma(s[i][kb + p + 2], s[l][kb + p + 2], a2);
            a3 = fma(s[i][kb + p + 3], s[l][kb + p + 3], a3);
          }
          for (; p < w; ++p) a0 = fma(s[i][kb + p], s[l][kb + p], a0);
          s[i][l] -= (a0 + a1) + (a2 + a3);
        }
      }
      __syncthreads();
    }
  }
  // off-diagonal blocks of M by block forward substitution
  const int nbl = (nb + SB16 - 1) / SB16;
  for (int I = 1; I < nbl; ++I) {
    const int i0 = I * SB16, wi = (nb - i0 < SB16) ? nb - i0 : SB16;
    // T = sum_{K=J}^{I-1} L_IK M_KJ for every column block J < I, parked in mi[block I][0 .. i0)
    for (int e = tid; e < wi * i0; e += blockDim.x) {
      const int ii = e / i0, col = e % i0;
      const int k0 = (col / SB16) * SB16;
      double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
      for (int k = k0; k < i0; k += 4) {        // i0 - k0 is a multiple of 16
        a0 = fma(s[i0 + ii][k], mi[k][col], a0);
        a1 = fma(s[i0 + ii][k + 1], mi[k + 1][col], a1);
        a2 = fma(s[i0 + ii][k + 2], mi[k + 2][col], a2);
        a3 = fma(s[i0 + ii][k + 3], mi[k + 3][col], a3);
      }
      mi[i0 + ii][col] = (a0 + a1) + (a2 + a3);
    }
    __syncthreads();
    double tv[3];
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      const int e = tid + 256 * q;
      tv[q] = 0.0;
      if (e < wi * i0) {
        const int ii = e / i0, col = e % i0;
        double acc = 0.0;
        for (int t = 0; t <= ii; ++t) acc = fma(mi[i0 + ii][i0 + t], mi[i0 + t][col], acc);
        tv[q] = -acc;
      }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 3; ++q) {
      const int e = tid + 256 * q;
      if (e < wi * i0) mi[i0 + e / i0][e % i0] = tv[q];
    }
    __syncthreads();
  }
  for (int e = tid; e < nb * nb; e += blockDim.x) {
    const int r = e / nb, c = e % nb;
    A[off + (int64_t)r * n + c] = (c <= r) ? s[r][c] : 0.0;
    M[off + (int64_t)r * n + c] = (c <= r) ? mi[r][c] : 0.0;
  }
}

// L_IK = A_IK * M_KK^T for block rows I > K (one CTA per block row).
__global__ void __launch_bounds__(256) panel_kernel(double* __restrict__ A, const double* __restrict__ M, int64_t n,
                                                    int K) {
  extern __shared__ double smem[];
  double (*At)[LDS] = reinterpret_cast<double (*)[LDS]>(smem);
  double (*Bs)[LDS] = reinterpret_cast<double (*)[LDS]>(smem + NB * LDS);
  const int I = K + 1 + blockIdx.x;
  const int nbk = blk_size(n, K), nbi = blk_size(n, I);
  double* a = A + (int64_t)I * NB * n + (int64_t)K * NB;
  const double* mk = M + (int64_t)K * NB * n + (int64_t)K * NB;
  load_tile(At, a, n, nbi, nbk, true);   // At[l][r] = A_IK[r][l]
  load_tile(Bs, mk, n, nbk, nbk, true);  // Bs[l][j] = M_KK[j][l]
  __syncthreads();
  double acc[4][4];
  tile_mma(At, Bs, acc, nbk);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int rr = ty + 16 * r, cc = tx + 16 * c;
      if (rr < nbi && cc < nbk) a[(int64_t)rr * n + cc] = acc[r][c];
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

// A_IJ -= L_IK L_JK^T for K < J <= I.
__global__ void __launch_bounds__(256) syrk_kernel(double* __restrict__ A, int64_t n, int K) {
  extern __shared__ double smem[];
  double (*At)[LDS] = reinterpret_cast<double (*)[LDS]>(smem);
  double (*Bs)[LDS] = reinterpret_cast<double (*)[LDS]>(smem + NB * LDS);
  int ti, tj;
  tri_index(blockIdx.x, ti, tj);
  const int I = K + 1 + ti, J = K + 1 + tj;
  const int nbk = blk_size(n, K), nbi = blk_size(n, I), nbj = blk_size(n, J);
  load_tile(At, A + (int64_t)I * NB * n + (int64_t)K * NB, n, nbi, nbk, true);  // At[l][i] = L_IK[i][l]
  load_tile(Bs, A + (int64_t)J * NB * n + (int64_t)K * NB, n, nbj, nbk, true);  // Bs[l][j] = L_JK[j][l]
  __syncthreads();
  double acc[4][4];
  tile_mma(At, Bs, acc, nbk);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  double* c0 = A + (int64_t)I * NB * n + (int64_t)J * NB;
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int rr = ty + 16 * r, cc = tx + 16 * c;
      if (rr < nbi && cc < nbj && (I != J || cc <= rr)) c0[(int64_t)rr * n + cc] -= acc[r][c];
    }
}

// ---------------------------------------------------------------- inverse pieces
// M_IJ = M_II * R_IJ for J < I (one CTA per J), R_IJ stored in place.
__global__ void __launch_bounds__(256) rowmult_kernel(double* __restrict__ M, int64_t n, int I) {
  extern __shared__ double smem[];
  double (*At)[LDS] = reinterpret_cast<double (*)[LDS]>(smem);
  double (*Bs)[LDS] = reinterpret_cast<double (*)[LDS]>(smem + NB * LDS);
  const int J = blockIdx.x;
  const int nbi = blk_size(n, I), nbj = blk_size(n, J);
  double* r = M + (int64_t)I * NB * n + (int64_t)J * NB;
  load_tile(At, M + (int64_t)I * NB * n + (int64_t)I * NB, n, nbi, nbi, true);  // At[l][i] = M_II[i][l]
  load_tile(Bs, r, n, nbi, nbj, false);                                            // Bs[l][j] = R_IJ[l][j]
  __syncthreads();
  double acc[4][4];
  tile_mma(At, Bs, acc, nbi);
  __syncthreads();
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
  for (int rr = 0; rr < 4; ++rr)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = ty + 16 * rr, j = tx + 16 * c;
      if (i < nbi && j < nbj) r[(int64_t)i * n + j] = acc[rr][c];
    }
}

// R_I'J -= L_I'I M_IJ for I' > I, J <= I. Grid: (T - 1 - I) x (I + 1).
__global__ void __launch_bounds__(256) inv_update_kernel(const double* __restrict__ L, double* __restrict__ M,
                                                         int64_t n, int I) {
  extern __shared__ double smem[];
  double (*At)[LDS] = reinterpret_cast<double (*)[LDS]>(smem);
  double (*Bs)[LDS] = reinterpret_cast<double (*)[LDS]>(smem + NB * LDS);
  const int Ip = I + 1 + blockIdx.x, J = blockIdx.y;
  const int nbi = blk_size(n, I), nbp = blk_size(n, Ip), nbj = blk_size(n, J);
  load_tile(At, L + (int64_t)Ip * NB * n + (int64_t)I * NB, n, nbp, nbi, true);  // At[l][i'] = L_I'I[i'][l]
  load_tile(Bs, M + (int64_t)I * NB * n + (int64_t)J * NB, n, nbi, nbj, false);  // Bs[l][j] = M_IJ[l][j]
  __syncthreads();
  double acc[4][4];
  tile_mma(At, Bs, acc, nbi);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  double* c0 = M + (int64_t)Ip * NB * n + (int64_t)J * NB;
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = ty + 16 * r, j = tx + 16 * c;
      if (i < nbp && j < nbj) c0[(int64_t)i * n + j] -= acc[r][c];
    }
}

// ---------------------------------------------------------------- column norms
constexpr int kNormRows = 128;
__global__ void colsumsq_partial_kernel(const double* __restrict__ M, int64_t n, double* __restrict__ part) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= n) return;
  int64_t i0 = (int64_t)blockIdx.y * kNormRows;
  int64_t i1 = i0 + kNormRows < n ? i0 + kNormRows : n;
  if (i0 < j) i0 = j;
  double acc = 0.0;
  for (int64_t i = i0; i < i1; ++i) {
    const double v = M[i * n + j];
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

// Per host thread and device: a low-priority stream and events for the
// inverse half of hinv_diag.
struct SideStream {
  int dev = -1;
  bool ok = false;
  cudaStream_t stream = nullptr;
  std::vector<cudaEvent_t> ev;
};
static SideStream& side_stream(int events) {
  thread_local SideStream ss[16];
  int dev = 0;
  cudaGetDevice(&dev);
  SideStream& x = ss[dev & 15];
  if (x.dev != dev) {
    int lo = 0, hi = 0;
    cudaDeviceGetStreamPriorityRange(&lo, &hi);
    x.ok = cudaStreamCreateWithPriority(&x.stream, cudaStreamNonBlocking, lo) == cudaSuccess;
    x.dev = dev;
  }
  while (x.ok && (int)x.ev.size() < events) {
    cudaEvent_t e;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) { x.ok = false; break; }
    x.ev.push_back(e);
  }
  return x;
}

size_t hinv_workspace_doubles(int64_t n) {
  const int64_t parts = (n + kNormRows - 1) / kNormRows;
  return (size_t)(2 * n * n + parts * n + 64);
}

cudaError_t launch_hinv(const double* H, int64_t n, double alpha, double* h, double* ws, DevStatus* st,
                        cudaStream_t s) {
  double* A = ws;
  double* M = ws + n * n;
  const int64_t parts = (n + kNormRows - 1) / kNormRows;
  double* part = M + n * n;
  double* damp = part + parts * n;
  const size_t tile_smem = 2 * NB * LDS * sizeof(double);
  static bool attr_done = false;
  if (!attr_done) {
    cudaFuncSetAttribute(potrf_diag_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tile_smem);
    cudaFuncSetAttribute(panel_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tile_smem);
    cudaFuncSetAttribute(syrk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tile_smem);
    cudaFuncSetAttribute(rowmult_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tile_smem);
    cudaFuncSetAttribute(inv_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)tile_smem);
    attr_done = true;
  }
  diag_sum_kernel<<<1, 1024, 0, s>>>(H, n, alpha, damp);
  damp_copy_kernel<<<dim3((unsigned)((n + 255) / 256), (unsigned)n), 256, 0, s>>>(H, n, damp, A);
  cudaMemsetAsync(M, 0, (size_t)n * n * sizeof(double), s);
  const int T = (int)((n + NB - 1) / NB);
  // The inverse steps run on a lower-priority side stream: step I needs only
  // panel I (column block I of L is final then; later trailing updates touch
  // column blocks > K) and the diagonal inverse M_II, so they fill the SMs the
  // one-CTA diagonal factorizations leave idle. Joined back before the norms.
  SideStream& ss = side_stream(T + 1);
  if (!ss.ok) return cudaErrorMemoryAllocation;
  cudaEventRecord(ss.ev[T], s);
  cudaStreamWaitEvent(ss.stream, ss.ev[T], 0);
  for (int K = 0; K < T; ++K) {
    potrf_diag_kernel<<<1, 256, tile_smem, s>>>(A, M, n, K, st);
    const int below = T - 1 - K;
    if (below > 0) panel_kernel<<<below, 256, tile_smem, s>>>(A, M, n, K);
    cudaEventRecord(ss.ev[K], s);
    if (below > 0) syrk_kernel<<<below * (below + 1) / 2, 256, tile_smem, s>>>(A, n, K);
    cudaStreamWaitEvent(ss.stream, ss.ev[K], 0);
    if (K > 0) rowmult_kernel<<<K, 256, tile_smem, ss.stream>>>(M, n, K);
    if (K < T - 1)
      inv_update_kernel<<<dim3((unsigned)(T - 1 - K), (unsigned)(K + 1)), 256, tile_smem, ss.stream>>>(A, M, n, K);
  }
  cudaEventRecord(ss.ev[T], ss.stream);
  cudaStreamWaitEvent(s, ss.ev[T], 0);
  colsumsq_partial_kernel<<<dim3((unsigned)((n + 255) / 256), (unsigned)parts), 256, 0, s>>>(M, n, part);
  colsumsq_final_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(part, (int)parts, n, h);
  count_launches(2 + T + 2 * (T - 1) + 2 * (T - 1) + 2);
  return cudaGetLastError();
}

}  // namespace slim
