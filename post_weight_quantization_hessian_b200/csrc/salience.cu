// salience: element salience delta_ij = w_ij^2 / [H^-1]_jj^2 (SliM-LLM write-up,
// rkmt.cn, section 组件一 SBA, the SparseGPT-style elimination error with the
// denominator squared as printed), reduced to the mean of each group of
// columns (atlas.scime.ai summary, section Approach: allocation by average
// group salience), then the groups ordered by descending mean.
//
// sum_{i, j in G_c} w_ij^2 / h_j^2 = sum_{j in G_c} (sum_i w_ij^2) / h_j^2, so the
// streaming pass only needs column sums of squares of W (fp64), one read of W:
//   colsq_partial  grid (column blocks x row blocks): float4 loads, each thread
//                  4 adjacent columns over a run of rows, fp64 partials;
//   group_reduce   one block per group: sums the partials, divides by h_j^2,
//                  writes S_c;
//   rank_sort      one block: rank_c = #{c' : S_c' > S_c or (S_c' == S_c and
//                  c' < c)}, a stable descending order.
#include <cstdint>
#include <mutex>
#include "common.cuh"
#include "../../include/slim.h"

namespace slim {

constexpr int kColThreads = 256;   // x 4 columns = 1024 columns per block
constexpr int kRowsPerBlock = 32;

__global__ void __launch_bounds__(kColThreads)
colsq_partial_kernel(const float* __restrict__ W, int64_t m, int64_t n, double* __restrict__ part) {
  const int64_t col = ((int64_t)blockIdx.x * kColThreads + threadIdx.x) * 4;
  const int64_t r0 = (int64_t)blockIdx.y * kRowsPerBlock;
  if (col >= n) return;
  const int64_t r1 = (r0 + kRowsPerBlock < m) ? r0 + kRowsPerBlock : m;
  double a0 = 0, a1 = 0, a2 = 0, a3 = 0;
  const float4* p = reinterpret_cast<const float4*>(W + r0 * n + col);
  const int64_t stride = n / 4;
  for (int64_t r = r0; r < r1; ++r, p += stride) {
    const float4 v = __ldcs(p);
    a0 += (double)v.x * (double)v.x;
    a1 += (double)v.y * (double)v.y;
    a2 += (double)v.z * (double)v.z;
    a3 += (double)v.w * (double)v.w;
  }
  double* o = part + (int64_t)blockIdx.y * n + col;
  o[0] = a0; o[1] = a1; o[2] = a2; o[3] = a3;
}

__global__ void group_reduce_kernel(const double* __restrict__ part, int rblocks, int64_t m, int64_t n,
                                    const double* __restrict__ h, int group, double* __restrict__ S) {
  __shared__ double red[32];
  const int c = blockIdx.x;
  double acc = 0.0;
  // threads stride over (row block, column) pairs of this group
  const int64_t total = (int64_t)rblocks * group;
  for (int64_t e = threadIdx.x; e < total; e += blockDim.x) {
    const int rb = (int)(e / group);
    const int64_t j = (int64_t)c * group + (e - (int64_t)rb * group);
    const double hj = h[j];
    acc += part[(int64_t)rb * n + j] / (hj * hj);
  }
  acc = warp_sum(acc);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x < 32) {
    double v = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.0;
    v = warp_sum(v);
    if (threadIdx.x == 0) S[c] = v / ((double)m * (double)group);
  }
}

__global__ void rank_sort_kernel(const double* __restrict__ S, int k, int32_t* __restrict__ order) {
  for (int c = threadIdx.x; c < k; c += blockDim.x) {
    const double v = S[c];
    int rank = 0;
    for (int o = 0; o < k; ++o) {
      const double u = S[o];
      rank += (u > v || (u == v && o < c)) ? 1 : 0;
    }
    order[rank] = c;
  }
}

int salience_row_blocks(int64_t m) { return (int)((m + kRowsPerBlock - 1) / kRowsPerBlock); }

cudaError_t launch_salience(const float* W, int64_t m, int64_t n, const double* h, int group, double* S,
                            int32_t* order, double* part, cudaStream_t st) {
  const int rb = salience_row_blocks(m);
  dim3 g1((unsigned)((n / 4 + kColThreads - 1) / kColThreads), (unsigned)rb);
  colsq_partial_kernel<<<g1, kColThreads, 0, st>>>(W, m, n, part);
  const int k = (int)(n / group);
  group_reduce_kernel<<<k, 256, 0, st>>>(part, rb, m, n, h, group, S);
  rank_sort_kernel<<<1, 1024, 0, st>>>(S, k, order);
  count_launches(3);
  return cudaGetLastError();
}

// A caller's order of the k groups (device), checked to be a permutation of
// 0..k-1 and copied to `out`; if it is not, the identity is written instead
// (so later kernels never index outside the groups) and SLIM_EINVAL recorded.
// One block of 1024 threads; k <= 1024.
__global__ void order_check_kernel(const int32_t* __restrict__ order, int k, int32_t* __restrict__ out,
                                   DevStatus* st) {
  __shared__ int seen[1024];
  __shared__ int bad;
  for (int c = threadIdx.x; c < k; c += blockDim.x) seen[c] = 0;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int c = threadIdx.x; c < k; c += blockDim.x) {
    const int v = order[c];
    if (v < 0 || v >= k || atomicAdd(&seen[v], 1) != 0) atomicExch(&bad, 1);
  }
  __syncthreads();
  const bool ok = bad == 0;
  for (int c = threadIdx.x; c < k; c += blockDim.x) out[c] = ok ? order[c] : c;
  if (!ok && threadIdx.x == 0) record_failure(st, kStatusInvalid, 0);
}

cudaError_t launch_order_check(const int32_t* order, int k, int32_t* out, DevStatus* st, cudaStream_t s) {
  if (k < 1 || k > 1024) return cudaErrorInvalidValue;
  order_check_kernel<<<1, 1024, 0, s>>>(order, k, out, st);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace slim

namespace slim {

// ---------------------------------------------------------------------------
// Allocation-free variant (slim_salience_noalloc).
//
// Its scratch, the per-row-block column sums of squares, lives in one fixed
// file-scope device array instead of caller or library allocations. Every GPU
// that loads the library holds these 256 KiB until the process exits, and all
// calls on a device share them: calls that overlap on the GPU race. The array
// is fully rewritten by each call before it is read, so nothing carries over.
// ---------------------------------------------------------------------------
constexpr int64_t kNoAllocScratchDoubles = 32768;  // 256 KiB: row blocks x n <= 32768
static __device__ __align__(256) double g_salience_scratch[kNoAllocScratchDoubles];

// Column sums of squares over runs of `rows_per_block` rows (runtime), the
// same per-thread arithmetic as colsq_partial_kernel.
__global__ void __launch_bounds__(kColThreads)
colsq_partial_rows_kernel(const float* __restrict__ W, int64_t m, int64_t n, int64_t rows_per_block,
                          double* __restrict__ part) {
  const int64_t col = ((int64_t)blockIdx.x * kColThreads + threadIdx.x) * 4;
  const int64_t r0 = (int64_t)blockIdx.y * rows_per_block;
  if (col >= n) return;
  const int64_t r1 = (r0 + rows_per_block < m) ? r0 + rows_per_block : m;
  double a0 = 0, a1 = 0, a2 = 0, a3 = 0;
  const float4* p = reinterpret_cast<const float4*>(W + r0 * n + col);
  const int64_t stride = n / 4;
  for (int64_t r = r0; r < r1; ++r, p += stride) {
    const float4 v = *p;
    a0 += (double)v.x * (double)v.x;
    a1 += (double)v.y * (double)v.y;
    a2 += (double)v.z * (double)v.z;
    a3 += (double)v.w * (double)v.w;
  }
  double* o = part + (int64_t)blockIdx.y * n + col;
  o[0] = a0; o[1] = a1; o[2] = a2; o[3] = a3;
}

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
double* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_salience_scratch on the current device, looked up once
// per device (host code cannot use the array's name as a device pointer).
cudaError_t noalloc_scratch(double** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_salience_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = static_cast<double*>(p);
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}
}  // namespace

}  // namespace slim

extern "C" int slim_salience_noalloc(const float* W, int64_t m, int64_t n, const double* h, int group, double* S,
                                     int32_t* order, void* stream) {
  using namespace slim;
  if (!W || !h || !S || !order || (reinterpret_cast<uintptr_t>(W) & 15)) return SLIM_EINVAL;
  if (m < 1 || n < 1 || (group != 32 && group != 64 && group != 128) || n % group || n / group > 1024)
    return SLIM_EINVAL;
  if (n > kNoAllocScratchDoubles) return SLIM_EINVAL;  // beyond the fixed scratch: at most 32768 input columns
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SLIM_ENODEV;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (major != 10) return SLIM_ENODEV;
  double* part = nullptr;
  if (noalloc_scratch(&part) != cudaSuccess) return SLIM_ECUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int64_t rb = (m + kRowsPerBlock - 1) / kRowsPerBlock;
  if (rb > kNoAllocScratchDoubles / n) rb = kNoAllocScratchDoubles / n;
  const int64_t rows_per_block = (m + rb - 1) / rb;
  rb = (m + rows_per_block - 1) / rows_per_block;
  dim3 g1((unsigned)((n / 4 + kColThreads - 1) / kColThreads), (unsigned)rb);
  colsq_partial_rows_kernel<<<g1, kColThreads, 0, st>>>(W, m, n, rows_per_block, part);
  const int k = (int)(n / group);
  group_reduce_kernel<<<k, 256, 0, st>>>(part, (int)rb, m, n, h, group, S);
  rank_sort_kernel<<<1, 1024, 0, st>>>(S, k, order);
  count_launches(3);
  if (cudaGetLastError() != cudaSuccess) return SLIM_ECUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return SLIM_ECUDA;
  return SLIM_OK;
}
