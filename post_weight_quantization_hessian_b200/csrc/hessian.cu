// hessian_accum: H = 2 X^T X over the calibration tokens (SliM-LLM write-up,
// rkmt.cn, section 组件一 SBA: the Hessian comes from calibration activations,
// without backpropagation).
//
// bf16 X: a tcgen05 tensor-core SYRK. H is cut into 256 x 256 feature blocks;
// only blocks (ba <= bb) are computed and the fp64 reduction mirrors them. The
// tokens are cut into slices of `slice_tokens`; a work unit is (block pair,
// slice) and writes an fp32 partial, so each fp32 accumulation chain is one
// slice long and the slices are summed in fp64 (deterministic order).
//
//   persistent CTA, 192 threads, one per SM:
//     warp 0      TMA producer: per 64-token stage, four 64-feature boxes of
//                 block ba and four of block bb (one set on diagonal blocks),
//                 128-byte swizzle, no multicast
//     warp 1      TMEM owner (512 columns) and single-thread MMA issuer:
//                 two M=128 x N=256 x K=16 bf16 MMAs per 16 tokens into two
//                 fp32 accumulators (rows ba*256 + [0,128) and [128,256))
//     warps 2..5  epilogue: tcgen05.ld of both accumulators, fp32 partial store
//   Both operands are MN-major (features contiguous, tokens along K), exactly
//   how X sits in memory, so no transpose pass is needed.
//
// fp32 X: tiled CUDA-core kernel with fp64 accumulation (the products of fp32
// values are exact in fp64), token-split partials, same fp64 reduction.
#include <cstdint>
#include "common.cuh"
#include "tmap.h"

namespace slim {

constexpr int HS_BK = 64;
constexpr int HS_TILE = 256;
constexpr int HS_STAGES = 3;
constexpr int HS_BOX = 64 * 64 * 2;       // 64 tokens x 64 features, bf16
constexpr int HS_HALF = 4 * HS_BOX;       // 256 features
constexpr int HS_STAGE = 2 * HS_HALF;
constexpr int HS_SMEM = HS_STAGES * HS_STAGE + 1024 /*align*/ + 256 /*barriers*/;

struct SyrkParams {
  int64_t N, n;
  int nblk, npairs, nslices;
  int slice0, launch_slices;  // this launch covers slices [slice0, slice0 + launch_slices)
  int64_t slice_tokens;  // multiple of 64
  float* part;           // [nslices][npairs][256][256]
  DevStatus* st;
};

__device__ __forceinline__ void tri_decode(int x, int& hi, int& lo) {
  int t = (int)((sqrt(8.0 * (double)x + 1.0) - 1.0) * 0.5);
  while ((t + 1) * (t + 2) / 2 <= x) ++t;
  while (t * (t + 1) / 2 > x) --t;
  hi = t;
  lo = x - t * (t + 1) / 2;
}

__global__ void __launch_bounds__(192, 1) syrk_tc_kernel(const __grid_constant__ CUtensorMap tmX, SyrkParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + HS_STAGES * HS_STAGE);
  uint64_t* empty = full + HS_STAGES;
  uint64_t* tfull = empty + HS_STAGES;
  uint64_t* tempty = tfull + 1;
  uint64_t* done = tempty + 1;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tslot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < HS_STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(tfull, 1);
    mbar_init(tempty, 4);
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmX);
  }
  if (warp == 1) tmem_alloc(tslot, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tslot;
  const int units = p.npairs * p.launch_slices;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      for (int u = blockIdx.x; u < units && !*abort_flag; u += gridDim.x) {
        const int sl = u / p.npairs, pair = u - sl * p.npairs, slice = p.slice0 + sl;
        int bb, ba;
        tri_decode(pair, bb, ba);
        const int64_t t0 = (int64_t)slice * p.slice_tokens;
        const int64_t t1 = (t0 + p.slice_tokens < p.N) ? t0 + p.slice_tokens : p.N;
        const int nk = (int)((t1 - t0 + HS_BK - 1) / HS_BK);
        const bool diag = (ba == bb);
        for (int kk = 0; kk < nk; ++kk, ++it) {
          const int s = it % HS_STAGES;
          const uint32_t ph = (it / HS_STAGES) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, p.st, 100 + s)) break;
          mbar_arrive_expect_tx(&full[s], diag ? HS_HALF : HS_STAGE);
          uint8_t* sa = smem + s * HS_STAGE;
          const int y = (int)(t0 + (int64_t)kk * HS_BK);
#pragma unroll
          for (int q = 0; q < 4; ++q) tma_load_2d(sa + q * HS_BOX, &tmX, &full[s], ba * HS_TILE + q * 64, y);
          if (!diag) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              tma_load_2d(sa + HS_HALF + q * HS_BOX, &tmX, &full[s], bb * HS_TILE + q * 64, y);
          }
        }
      }
      // let every issued copy land before the CTA can exit, also after an
      // abort (bounded, but not cut short by the abort flag)
      for (uint32_t j = (it > HS_STAGES ? it - HS_STAGES : 0); j < it; ++j) mbar_drain(&full[j % HS_STAGES], (j / HS_STAGES) & 1);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, 256, true, true);
      uint32_t it = 0, ui = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++ui) {
        const int sl = u / p.npairs, pair = u - sl * p.npairs, slice = p.slice0 + sl;
        int bb, ba;
        tri_decode(pair, bb, ba);
        const int64_t t0 = (int64_t)slice * p.slice_tokens;
        const int64_t t1 = (t0 + p.slice_tokens < p.N) ? t0 + p.slice_tokens : p.N;
        const int nk = (int)((t1 - t0 + HS_BK - 1) / HS_BK);
        const bool diag = (ba == bb);
        if (!mbar_wait(tempty, (ui & 1) ^ 1, abort_flag, p.st, 120)) { ok = false; break; }
        tc_fence_after();
        for (int kk = 0; kk < nk; ++kk, ++it) {
          const int s = it % HS_STAGES;
          const uint32_t ph = (it / HS_STAGES) & 1;
          if (!mbar_wait(&full[s], ph, abort_flag, p.st, 130 + s)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + s * HS_STAGE);
          const uint32_t b_base = diag ? a_base : a_base + HS_HALF;
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const uint32_t acc = (kk > 0 || k16 > 0) ? 1u : 0u;
            const uint64_t bd = sdesc_sw128(b_base + k16 * 2048, HS_BOX, 1024);
            const uint64_t a0 = sdesc_sw128(a_base + k16 * 2048, HS_BOX, 1024);
            const uint64_t a1 = sdesc_sw128(a_base + 2 * HS_BOX + k16 * 2048, HS_BOX, 1024);
            tc_mma_bf16(tbase + 0, a0, bd, idesc, acc);
            tc_mma_bf16(tbase + 256, a1, bd, idesc, acc);
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(tfull);
      }
      // every issued MMA completes before TMEM can be freed, also after an abort
      tc_commit(done);
      mbar_drain(done, 0);
    }
  } else {
    const int wq = warp & 3;
    uint32_t ui = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++ui) {
      if (!mbar_wait(tfull, ui & 1, abort_flag, p.st, 150)) break;
      tc_fence_after();
      float* dst = p.part + ((size_t)p.slice0 * p.npairs + u) * HS_TILE * HS_TILE;
#pragma unroll 1
      for (int q = 0; q < 2; ++q) {
        const int row = q * 128 + wq * 32 + lane;
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t r[32];
          tmem_ld32(tbase + ((uint32_t)(wq * 32) << 16) + q * 256 + cc * 32, r);
          tc_wait_ld();
          float4* o = reinterpret_cast<float4*>(dst + (size_t)row * HS_TILE + cc * 32);
#pragma unroll
          for (int v = 0; v < 8; ++v)
            o[v] = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                               __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty);
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// H[a][b] = H[b][a] = 2 * sum over slices of the fp32 partials (fp64 sum).
__global__ void syrk_reduce_kernel(const float* __restrict__ part, int npairs, int nslices, int64_t n,
                                   double* __restrict__ H) {
  const int pair = blockIdx.y;
  int bb, ba;
  tri_decode(pair, bb, ba);
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= HS_TILE * HS_TILE) return;
  const int r = e / HS_TILE, c = e % HS_TILE;
  if (ba == bb && c < r) return;
  const int64_t a = (int64_t)ba * HS_TILE + r, b = (int64_t)bb * HS_TILE + c;
  if (a >= n || b >= n) return;
  double acc = 0.0;
  for (int s = 0; s < nslices; ++s) acc += (double)part[((size_t)s * npairs + pair) * HS_TILE * HS_TILE + e];
  acc *= 2.0;
  H[a * n + b] = acc;
  H[b * n + a] = acc;
}

// ---------------------------------------------------------------- fp32 X
constexpr int HF_T = 64, HF_KT = 32;
__global__ void __launch_bounds__(256) syrk_f32_kernel(const float* __restrict__ X, int64_t N, int64_t n,
                                                       int64_t slice_tokens, double* __restrict__ part) {
  __shared__ double xa[HF_KT][HF_T + 1];
  __shared__ double xb[HF_KT][HF_T + 1];
  const int ta = blockIdx.x, tb = blockIdx.y, sl = blockIdx.z;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t t0 = (int64_t)sl * slice_tokens;
  const int64_t t1 = (t0 + slice_tokens < N) ? t0 + slice_tokens : N;
  double acc[4][4] = {};
  for (int64_t tk = t0; tk < t1; tk += HF_KT) {
    for (int e = threadIdx.x; e < HF_KT * HF_T; e += 256) {
      const int r = e / HF_T, c = e % HF_T;
      const int64_t t = tk + r;
      const int64_t fa = (int64_t)ta * HF_T + c, fb = (int64_t)tb * HF_T + c;
      xa[r][c] = (t < t1 && fa < n) ? (double)X[t * n + fa] : 0.0;
      xb[r][c] = (t < t1 && fb < n) ? (double)X[t * n + fb] : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int l = 0; l < HF_KT; ++l) {
      double a[4], b[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) a[r] = xa[l][ty + 16 * r];
#pragma unroll
      for (int c = 0; c < 4; ++c) b[c] = xb[l][tx + 16 * c];
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = fma(a[r], b[c], acc[r][c]);
    }
    __syncthreads();
  }
  double* o = part + (size_t)sl * n * n;
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int64_t a = (int64_t)ta * HF_T + ty + 16 * r, b = (int64_t)tb * HF_T + tx + 16 * c;
      if (a < n && b < n) o[a * n + b] = acc[r][c];
    }
}

__global__ void sum_slices_kernel(const double* __restrict__ part, int nslices, int64_t nn, double* __restrict__ H) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= nn) return;
  double acc = 0.0;
  for (int s = 0; s < nslices; ++s) acc += part[(size_t)s * nn + e];
  H[e] = 2.0 * acc;
}

// ---------------------------------------------------------------- host side
struct SyrkPlan {
  int nblk, npairs, nslices;
  int64_t slice_tokens;
  size_t part_bytes;
};

constexpr int64_t kSyrkSliceTokens = 16384;

SyrkPlan syrk_plan_bf16(int64_t N, int64_t n) {
  SyrkPlan pl;
  pl.nblk = (int)((n + HS_TILE - 1) / HS_TILE);
  pl.npairs = pl.nblk * (pl.nblk + 1) / 2;
  pl.slice_tokens = kSyrkSliceTokens;
  pl.nslices = (int)((N + pl.slice_tokens - 1) / pl.slice_tokens);
  pl.part_bytes = (size_t)pl.nslices * pl.npairs * HS_TILE * HS_TILE * sizeof(float);
  return pl;
}

SyrkPlan syrk_plan_f32(int64_t N, int64_t n) {
  SyrkPlan pl{};
  int64_t s = (N + 1023) / 1024;
  if (s > 16) s = 16;
  if (s < 1) s = 1;
  pl.nslices = (int)s;
  pl.slice_tokens = (N + s - 1) / s;
  pl.part_bytes = (size_t)s * n * n * sizeof(double);
  return pl;
}

size_t hessian_ws_bytes(int64_t N, int64_t n, int xdtype) {
  return xdtype == 1 ? syrk_plan_bf16(N, n).part_bytes : syrk_plan_f32(N, n).part_bytes;
}

// bf16 X, token slices [slice0, slice0 + nsl) only: their fp32 partials. The
// rows of those slices must be in X; other rows are not read.
cudaError_t launch_hessian_slices(const void* X, int64_t N, int64_t n, void* part, DevStatus* st, int num_sms,
                                  cudaStream_t s, int slice0, int nsl) {
  const SyrkPlan pl = syrk_plan_bf16(N, n);
  CUtensorMap tm;
  if (!make_tmap_bf16(&tm, X, (uint64_t)n, (uint64_t)N, 64, 64)) return cudaErrorInvalidValue;
  static std::atomic<uint64_t> attr{0};
  uint64_t bit = 0;
  if (attr_pending(attr, bit)) {
    cudaError_t e = cudaFuncSetAttribute(syrk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, HS_SMEM);
    if (e != cudaSuccess) return e;
    attr.fetch_or(bit);
  }
  SyrkParams p;
  p.N = N; p.n = n; p.nblk = pl.nblk; p.npairs = pl.npairs; p.nslices = pl.nslices;
  p.slice0 = slice0; p.launch_slices = nsl;
  p.slice_tokens = pl.slice_tokens; p.part = static_cast<float*>(part); p.st = st;
  const int units = pl.npairs * nsl;
  const int grid = units < num_sms ? units : num_sms;
  syrk_tc_kernel<<<grid, 192, HS_SMEM, s>>>(tm, p);
  count_launches(1);
  return cudaGetLastError();
}

// H from the fp32 partials of all slices (bf16 X).
cudaError_t launch_hessian_reduce(int64_t N, int64_t n, const void* part, double* H, cudaStream_t s) {
  const SyrkPlan pl = syrk_plan_bf16(N, n);
  syrk_reduce_kernel<<<dim3(HS_TILE * HS_TILE / 256, pl.npairs), 256, 0, s>>>(static_cast<const float*>(part),
                                                                              pl.npairs, pl.nslices, n, H);
  count_launches(1);
  return cudaGetLastError();
}

int hessian_slice_tokens() { return (int)kSyrkSliceTokens; }

cudaError_t launch_hessian(const void* X, int xdtype, int64_t N, int64_t n, double* H, void* part, DevStatus* st,
                           int num_sms, cudaStream_t s, cudaEvent_t* kev) {
  if (xdtype == 1) {
    const SyrkPlan pl = syrk_plan_bf16(N, n);
    CUtensorMap tm;
    if (!make_tmap_bf16(&tm, X, (uint64_t)n, (uint64_t)N, 64, 64)) return cudaErrorInvalidValue;
    static std::atomic<uint64_t> attr{0};
    uint64_t bit = 0;
    if (attr_pending(attr, bit)) {
      cudaError_t e = cudaFuncSetAttribute(syrk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, HS_SMEM);
      if (e != cudaSuccess) return e;
      attr.fetch_or(bit);
    }
    SyrkParams p;
    p.N = N; p.n = n; p.nblk = pl.nblk; p.npairs = pl.npairs; p.nslices = pl.nslices;
    p.slice0 = 0; p.launch_slices = pl.nslices;
    p.slice_tokens = pl.slice_tokens; p.part = static_cast<float*>(part); p.st = st;
    const int units = pl.npairs * pl.nslices;
    const int grid = units < num_sms ? units : num_sms;
    if (kev) cudaEventRecord(kev[0], s);
    syrk_tc_kernel<<<grid, 192, HS_SMEM, s>>>(tm, p);
    if (kev) cudaEventRecord(kev[1], s);
    syrk_reduce_kernel<<<dim3(HS_TILE * HS_TILE / 256, pl.npairs), 256, 0, s>>>(
        static_cast<const float*>(part), pl.npairs, pl.nslices, n, H);
  } else {
    const SyrkPlan pl = syrk_plan_f32(N, n);
    const int T = (int)((n + HF_T - 1) / HF_T);
    syrk_f32_kernel<<<dim3(T, T, pl.nslices), 256, 0, s>>>(static_cast<const float*>(X), N, n, pl.slice_tokens,
                                                             static_cast<double*>(part));
    const int64_t nn = n * n;
    sum_slices_kernel<<<(unsigned)((nn + 255) / 256), 256, 0, s>>>(static_cast<const double*>(part), pl.nslices, nn, H);
  }
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace slim
