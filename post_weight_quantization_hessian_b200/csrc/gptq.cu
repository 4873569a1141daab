// gptq: SliM-LLM inside the GPTQ layer loop (SliM-LLM write-up, rkmt.cn,
// section 核心设计: the GPTQ layer-wise quantization skeleton with the two
// salience-driven components inserted; section FAQ). SBA's bits fix each
// group's width; when the column loop reaches a group's first column, SQC
// calibrates the group's quantizer on the weights as the earlier columns'
// compensation has left them; every column is rounded with its group's
// quantizer and its error, over U_jj, is spread along row j of U, the upper
// Cholesky factor of the damped inverse Hessian (H_d^-1 = U^T U).
//
// U without forming H_d^-1: with J the reversal permutation, J H_d J = L~ L~^T
// gives H_d = (J L~ J)(J L~ J)^T with J L~ J upper triangular, so
// U = (J L~ J)^-1 = J L~^-1 J, i.e. U_jk = [L~^-1]_{n-1-j, n-1-k}. The
// inverse-Hessian stage's blocked fp64 Cholesky and inverse, run on the
// reversed matrix, give L~^-1, and its column norms give diag(H_d^-1) reversed.
//
// Column loop, in blocks of 128 columns (all fp64):
//   gptq_block   warp per row; the block's U (128 x 128) in shared memory.
//                Per group of the block: sqc_choose (the SQC kernel's own
//                calibration) on the row's current group values; then per
//                column j: code, w_hat = s (q - z0), err = (w - w_hat) / U_jj,
//                w_k -= err U_jk for the later columns k of the block (each
//                product and difference rounded apart, as the definition's
//                outer-product update); err to Err[row][j - j0]; codes packed
//                per group.
//   gptq_update  the later blocks' columns take the block's errors at once:
//                W[:, e:] -= Err U[j0:e, e:] (the same sums regrouped), 64 x 64
//                tiles on the fp64 tensor cores (mma.sync m8n8k4).
#include <cstdint>
#include "common.cuh"
#include "f64_tiles.cuh"
#include "sqc_core.cuh"

namespace slim {

constexpr int GQ_BS = 128;    // columns per block
constexpr int GQ_WARPS = 16;  // rows of a CTA in flight
constexpr size_t kGqSmem = (size_t)GQ_BS * GQ_BS * sizeof(double);

cudaError_t launch_hinv(const double* H, int64_t n, double alpha, double* h, double* ws, DevStatus* st,
                        cudaStream_t s);
size_t hinv_workspace_doubles(int64_t n);

// R[i][j] = H[n-1-i][n-1-j]
__global__ void reverse_matrix_kernel(const double* __restrict__ H, int64_t n, double* __restrict__ R) {
  const int64_t total = n * n;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / n, j = e - i * n;
    R[e] = H[(n - 1 - i) * n + (n - 1 - j)];
  }
}

// U[j][k] = Minv[n-1-j][n-1-k] for k >= j, 0 below (Minv: np x np, lower);
// h[j] = hr[n-1-j].
__global__ void gptq_u_kernel(const double* __restrict__ Minv, int64_t np, int64_t n, const double* __restrict__ hr,
                              double* __restrict__ U, double* __restrict__ h) {
  const int64_t total = n * n;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = e / n, k = e - j * n;
    U[e] = k >= j ? Minv[(n - 1 - j) * np + (n - 1 - k)] : 0.0;
    if (e < n) h[e] = hr[n - 1 - e];
  }
}

__global__ void to_f64_kernel(const float* __restrict__ W, int64_t total, double* __restrict__ Wk) {
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x)
    Wk[e] = (double)W[e];
}

// One block of bw (<= 128, a multiple of G) columns starting at j0. Lane l
// holds the row's block columns l, l + 32, l + 64, l + 96 in w[0..3].
template <int G>
__global__ void __launch_bounds__(GQ_WARPS * 32, 1)
gptq_block_kernel(const double* __restrict__ Wk, int64_t m, int64_t n, const double* __restrict__ U,
                  const double* __restrict__ h, const uint8_t* __restrict__ bits, int avg_bits, double lam, int n_tau,
                  int j0, int bw, uint32_t* __restrict__ codes, float* __restrict__ scale, float* __restrict__ zero,
                  uint8_t* __restrict__ tau_idx, double* __restrict__ Err) {
  constexpr int E = G / 32;
  extern __shared__ double s_u[];  // [128][128]: U[j0 + r][j0 + c] for c >= r, else 0
  __shared__ double s_w[GQ_WARPS][G];
  __shared__ double s_d[GQ_WARPS][G];
  __shared__ uint8_t s_q[GQ_WARPS][G];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  for (int e = threadIdx.x; e < GQ_BS * GQ_BS; e += blockDim.x) {
    const int r = e >> 7, c = e & 127;
    s_u[e] = (r < bw && c < bw && c >= r) ? U[(int64_t)(j0 + r) * n + j0 + c] : 0.0;
  }
  __syncthreads();
  const int64_t k = n / G;
  const int64_t row_words = n * avg_bits / 32;
  for (int64_t i = (int64_t)blockIdx.x * GQ_WARPS + wib; i < m; i += (int64_t)gridDim.x * GQ_WARPS) {
    double w[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int col = lane + 32 * r;
      w[r] = col < bw ? Wk[i * n + j0 + col] : 0.0;
    }
#pragma unroll
    for (int gi = 0; gi < GQ_BS / G; ++gi) {
      if (gi * G >= bw) break;
      const int64_t c = j0 / G + gi;
      const int b = bits[c];
      const int qmaxi = (1 << b) - 1;
      double wg[E];
#pragma unroll
      for (int e = 0; e < E; ++e) wg[e] = w[gi * E + e];
      const SqcChoice ch = sqc_choose<G>(wg, h + c * G, b, lam, n_tau, s_w[wib], s_d[wib], lane);
      if (lane == 0) {
        scale[i * k + c] = (float)ch.s;
        zero[i * k + c] = (float)ch.z0;
        if (tau_idx) tau_idx[i * k + c] = (uint8_t)ch.t;
      }
#pragma unroll
      for (int sr = 0; sr < E; ++sr) {
        const int slot = gi * E + sr;
        for (int l = 0; l < 32; ++l) {
          const int jl = slot * 32 + l;  // column within the block
          const double wj = __shfl_sync(0xffffffffu, w[slot], l);
          const int q = sqc_code(wj, ch.s, ch.z0, qmaxi);
          const double wq = __dmul_rn(ch.s, __dsub_rn((double)q, ch.z0));
          const double err = __dsub_rn(wj, wq) / s_u[jl * GQ_BS + jl];
          if (lane == l) {
            s_q[wib][sr * 32 + l] = (uint8_t)q;
            Err[i * GQ_BS + jl] = err;
          }
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int col = lane + 32 * r;
            if (col > jl) w[r] = __dsub_rn(w[r], __dmul_rn(err, s_u[jl * GQ_BS + col]));
          }
        }
      }
      __syncwarp();
      sqc_pack<G>(s_q[wib], bits, (int)c, b, codes + i * row_words, row_words, lane);
    }
  }
}

// W[:, e:] -= Err[:, 0:bw] U[j0:j0 + bw, e:], e = j0 + bw. CTA (x, y): the 64 x 64
// tile of rows 64 y, columns e + 64 x.
__global__ void __launch_bounds__(HT) gptq_update_kernel(double* __restrict__ Wk, int64_t m, int64_t n,
                                                         const double* __restrict__ Err, const double* __restrict__ U,
                                                         int j0, int bw) {
  extern __shared__ double smem_t[];
  double* As = smem_t;
  double* Bs = smem_t + TILE;
  const int64_t e = j0 + bw;
  const int64_t r0 = (int64_t)blockIdx.y * NB, c0 = e + (int64_t)blockIdx.x * NB;
  const int rows = (int)((m - r0) < NB ? m - r0 : NB), cols = (int)((n - c0) < NB ? n - c0 : NB);
  Acc acc;
  acc_from_global(acc, Wk + r0 * n + c0, n, rows, cols);
  for (int k0 = 0; k0 < bw; k0 += NB) {
    const int kn = (bw - k0) < NB ? bw - k0 : NB;
    __syncthreads();
    tile_load_async(As, Err + r0 * GQ_BS + k0, GQ_BS, rows, kn);
    tile_load_async(Bs, U + (int64_t)(j0 + k0) * n + c0, n, kn, cols);
    cp_commit();
    cp_wait_all();
    __syncthreads();
    warp_mma64<false, true>(acc, As, Bs, kn);
  }
  acc_to_global(acc, Wk + r0 * n + c0, n, rows, cols);
}

// Workspace of launch_gptq, in doubles: the reversed H, the inverse stage's
// scratch, U, the working weights, the block errors, the reversed diagonal.
size_t gptq_workspace_doubles(int64_t m, int64_t n) {
  return (size_t)(n * n) + hinv_workspace_doubles(n) + (size_t)(n * n) + (size_t)(m * n) + (size_t)(m * GQ_BS) +
         (size_t)n + 64;
}

cudaError_t launch_gptq(const float* W, int64_t m, int64_t n, const double* H, double alpha, const uint8_t* bits,
                        int group, int avg_bits, double lam, int n_tau, uint32_t* codes, float* scale, float* zero,
                        uint8_t* tau_idx, double* h, double* ws, DevStatus* st, int num_sms, cudaStream_t s) {
  if (group != 32 && group != 64 && group != 128) return cudaErrorInvalidValue;
  double* Hr = ws;
  double* hws = Hr + n * n;
  double* U = hws + hinv_workspace_doubles(n);
  double* Wk = U + n * n;
  double* Err = Wk + m * n;
  double* hr = Err + m * GQ_BS;
  const int64_t np = (n + 31) / 32 * 32;
  const int eg = num_sms * 8;
  reverse_matrix_kernel<<<eg, 256, 0, s>>>(H, n, Hr);
  count_launches(1);
  cudaError_t e = launch_hinv(Hr, n, alpha, hr, hws, st, s);
  if (e != cudaSuccess) return e;
  gptq_u_kernel<<<eg, 256, 0, s>>>(hws + np * np, np, n, hr, U, h);
  to_f64_kernel<<<eg, 256, 0, s>>>(W, m * n, Wk);
  count_launches(2);
  static std::atomic<uint64_t> attr{0};
  uint64_t bit = 0;
  if (attr_pending(attr, bit)) {
    e = cudaFuncSetAttribute(gptq_block_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGqSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gptq_block_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGqSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gptq_block_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGqSmem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(gptq_update_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)(2 * kTileBytes));
    if (e != cudaSuccess) return e;
    attr.fetch_or(bit);
  }
  const int64_t need = (m + GQ_WARPS - 1) / GQ_WARPS;
  const int bgrid = (int)(need < num_sms ? need : num_sms);
  for (int64_t j0 = 0; j0 < n; j0 += GQ_BS) {
    const int bw = (int)((n - j0) < GQ_BS ? n - j0 : GQ_BS);
    switch (group) {
      case 32: gptq_block_kernel<32><<<bgrid, GQ_WARPS * 32, kGqSmem, s>>>(Wk, m, n, U, h, bits, avg_bits, lam, n_tau, (int)j0, bw, codes, scale, zero, tau_idx, Err); break;
      case 64: gptq_block_kernel<64><<<bgrid, GQ_WARPS * 32, kGqSmem, s>>>(Wk, m, n, U, h, bits, avg_bits, lam, n_tau, (int)j0, bw, codes, scale, zero, tau_idx, Err); break;
      default: gptq_block_kernel<128><<<bgrid, GQ_WARPS * 32, kGqSmem, s>>>(Wk, m, n, U, h, bits, avg_bits, lam, n_tau, (int)j0, bw, codes, scale, zero, tau_idx, Err); break;
    }
    count_launches(1);
    const int64_t rest = n - (j0 + bw);
    if (rest > 0) {
      const dim3 grid((unsigned)((rest + NB - 1) / NB), (unsigned)((m + NB - 1) / NB));
      gptq_update_kernel<<<grid, HT, 2 * kTileBytes, s>>>(Wk, m, n, Err, U, (int)j0, bw);
      count_launches(1);
    }
  }
  return cudaGetLastError();
}

}  // namespace slim
