// dequant_gemv: y = x W_hat^T on the packed mixed-precision layout, the
// inference product of a SliM-LLM layer (its token rate on current GPU kernels
// is the method's stated limitation: rkmt.cn write-up, section 局限性;
// atlas.scime.ai summary, Limitations). w_hat = scale (q - zero) per (row,
// group); group c's codes take bits[c] bits each, packed little-endian after
// the earlier groups' codes (one row = n * avg_bits / 32 words).
//
// Decode without integer-to-float conversions: a b-bit code q placed in the
// top mantissa bits of 1.0f gives f = 1 + q 2^-b exactly, so
//   sum_j x_j q_j = 2^b (sum_j x_j f_j - sum_j x_j)
// and per (row, group) y += scale (2^b (A - xs) - zero xs), with
// A = sum_j x_j f_j (one fma per code) and xs = sum_j x_j (once per group and
// batch row, shared by all rows). Per code that is a funnel shift, one
// logical op and one fma.
//
// Layout of the work. A block takes 32 output rows and a range of groups
// (all of them unless a row's words would not fit in shared memory). It first
// copies the rows' packed words, scales and zeros into shared memory with
// coalesced asynchronous copies (consecutive threads take consecutive words of
// one row, all in flight at once; the rows are stored at an odd word stride),
// and sums x over each group of the range; then each of its 8 warps decodes every 8th group with lane = row, so
// that all lanes decode the same code positions (uniform control flow, one x
// address per warp) and read their own row's words from shared memory without
// bank conflicts. The warps' sums are added in a fixed order: one launch, no
// atomics, deterministic. Batch rows: up to 8, each code's f reused for all of
// them. HBM-bound on the codes, scales and zeros at batch 1.
#include <algorithm>
#include <cstdint>
#include "common.cuh"

namespace slim {

constexpr int DG_WARPS = 8;
constexpr int DG_ROWS = 32;
constexpr size_t DG_SMEM_MAX = 110 * 1024;  // two blocks per SM

// 4-byte asynchronous copy global -> shared (cp.async), and the wait for all of
// this thread's copies.
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Shared-memory plan of one block.
struct DgPlan {
  int ks, gps;   // group-range splits, groups per split
  int wstride;   // words per staged row (>= the range's words, odd)
  int sstride;   // scales / zeros per staged row (>= gps, odd)
  size_t smem;
};

static size_t dg_smem(int wstride, int sstride, int gps, int group, int B) {
  return (size_t)DG_ROWS * wstride * 4 + 2 * (size_t)DG_ROWS * sstride * 4 + (size_t)(gps + 1) * 4 +
         (size_t)B * gps * 4 + (size_t)DG_WARPS * B * DG_ROWS * 4 + (size_t)B * gps * group * 4;
}

// A range of groups holds at most its groups' full-row share of words when the
// allocation is the usual one (rw words per row in all); widths up to 8 bits
// bound it in any case.
static DgPlan dg_plan(int64_t n, int group, int avg_bits, int B) {
  const int k = (int)(n / group);
  const int64_t rw = n * avg_bits / 32;
  DgPlan pl{};
  for (int ks = 1;; ++ks) {
    const int gps = (k + ks - 1) / ks;
    const int64_t wmax = std::min<int64_t>((int64_t)gps * group / 4, rw);
    pl.ks = ks;
    pl.gps = gps;
    pl.wstride = (int)(wmax | 1);
    pl.sstride = gps | 1;
    pl.smem = dg_smem(pl.wstride, pl.sstride, gps, group, B);
    if (pl.smem <= DG_SMEM_MAX || gps == 1) break;
  }
  return pl;
}

// A[bb] += sum_j x[bb][j] f_j over 32 consecutive codes of BITS bits each: the
// BITS words at wp (32 codes of b bits are exactly b words), x (fp32) at xr +
// bb * xstride. Code j sits at bit j*BITS; one shift brings it to bit 23 - BITS
// and one three-input logic op keeps it and sets the exponent of 1.0f.
template <int BITS, int MB>
__device__ __forceinline__ void dg_unit(const uint32_t* __restrict__ wp, const float* __restrict__ xr, int xstride,
                                        int B, float (&A)[MB]) {
  uint32_t w[BITS];
#pragma unroll
  for (int u = 0; u < BITS; ++u) w[u] = wp[u];
  constexpr uint32_t kField = ((1u << BITS) - 1) << (23 - BITS);
#pragma unroll
  for (int j4 = 0; j4 < 32; j4 += 4) {
    float f[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int pos = (j4 + u) * BITS, wi = pos >> 5, off = pos & 31;
      uint32_t v;
      if (off + BITS <= 32) {
        constexpr int kTo = 23 - BITS;  // the field moves from bit off to bit kTo
        v = off <= kTo ? w[wi] << (kTo - off) : w[wi] >> (off - kTo);
      } else {
        v = __funnelshift_r(w[wi], w[wi + 1], off) << (23 - BITS);
      }
      f[u] = __uint_as_float((v & kField) | 0x3F800000u);
    }
#pragma unroll
    for (int bb = 0; bb < MB; ++bb)
      if (bb < B) {
        const float4 xv = *reinterpret_cast<const float4*>(xr + bb * xstride + j4);
        A[bb] = fmaf(xv.x, f[0], A[bb]);
        A[bb] = fmaf(xv.y, f[1], A[bb]);
        A[bb] = fmaf(xv.z, f[2], A[bb]);
        A[bb] = fmaf(xv.w, f[3], A[bb]);
      }
  }
}

template <int G, int MB>
__global__ void __launch_bounds__(DG_WARPS * 32)
dg_kernel(const uint32_t* __restrict__ codes, int64_t m, int64_t rw, const uint8_t* __restrict__ bits,
          const float* __restrict__ scale, const float* __restrict__ zero, int k, const void* __restrict__ x,
          int xdtype, int B, int64_t n, int gps, int wstride, int sstride, float* __restrict__ out) {
  constexpr int SU = G / 32;  // 32-code sub-units per group
  extern __shared__ uint32_t dsm[];
  // (the regions whose sizes are multiples of 4 words come first, so that the
  // 16-byte accesses to x stay aligned)
  uint32_t* wsm = dsm;                                             // [32 rows][wstride] words
  float* ssm = reinterpret_cast<float*>(wsm + DG_ROWS * wstride);  // [32][sstride] scales
  float* zsm = ssm + DG_ROWS * sstride;                            // [32][sstride] zeros
  float* xfs = zsm + DG_ROWS * sstride;                            // [B][gps * G] x of the range, fp32
  float* red = xfs + B * gps * G;                                  // [warps][B][32]
  float* xsm = red + DG_WARPS * B * DG_ROWS;                       // [B][gps] group sums of x
  int* woff = reinterpret_cast<int*>(xsm + B * gps);               // [gps + 1] word offsets in the range
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r0 = (int64_t)blockIdx.x * DG_ROWS;
  const int c0 = blockIdx.y * gps, c1 = (c0 + gps < k) ? c0 + gps : k, nc = c1 - c0;
  const bool xbf = xdtype == 1;
  // word offsets: the range's start (SU times the earlier groups' bits) and a
  // prefix sum over the range
  if (warp == 0) {
    int before = 0;
    for (int c = lane; c < c0; c += 32) before += bits[c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
    int run = SU * before;
    for (int cb = 0; cb < nc; cb += 32) {
      const int c = cb + lane;
      const int v = c < nc ? SU * (int)bits[c0 + c] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      if (c < nc) woff[c] = run + incl - v;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) woff[nc] = run;
  }
  // scales and zeros of the 32 rows, copied asynchronously (consecutive threads:
  // consecutive groups of a row); rows past m read as zero
  for (int r = warp; r < DG_ROWS; r += DG_WARPS)
    for (int c = lane; c < nc; c += 32) {
      if (r0 + r < m) {
        cp_async4(ssm + r * sstride + c, scale + (r0 + r) * k + c0 + c);
        cp_async4(zsm + r * sstride + c, zero + (r0 + r) * k + c0 + c);
      } else {
        ssm[r * sstride + c] = 0.f;
        zsm[r * sstride + c] = 0.f;
      }
    }
  // x of the range as fp32 (bf16 widened exactly), 16-byte loads
  const int xstride = gps * G, ncol = nc * G;
  for (int e = tid; e < B * (ncol / 8); e += DG_WARPS * 32) {
    const int bb = e / (ncol / 8), j = (e - bb * (ncol / 8)) * 8;
    const int64_t src = (int64_t)bb * n + (int64_t)c0 * G + j;
    float* d = xfs + bb * xstride + j;
    if (xbf) {
      const uint4 v = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + src);
      *reinterpret_cast<float4*>(d) = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                                                  __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
      *reinterpret_cast<float4*>(d + 4) = make_float4(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xFFFF0000u),
                                                      __uint_as_float(v.w << 16), __uint_as_float(v.w & 0xFFFF0000u));
    } else {
      const float4* xp = reinterpret_cast<const float4*>(static_cast<const float*>(x) + src);
      *reinterpret_cast<float4*>(d) = xp[0];
      *reinterpret_cast<float4*>(d + 4) = xp[1];
    }
  }
  __syncthreads();
  // group sums of x over the range: a thread per (batch row, group)
  for (int e = tid; e < B * nc; e += DG_WARPS * 32) {
    const int bb = e / nc, c = e - bb * nc;
    const float4* xp = reinterpret_cast<const float4*>(xfs + bb * xstride + c * G);
    float s0 = 0.f, s1 = 0.f;
#pragma unroll
    for (int j = 0; j < G / 4; j += 2) {
      const float4 v = xp[j], w2 = xp[j + 1];
      s0 += (v.x + v.y) + (v.z + v.w);
      s1 += (w2.x + w2.y) + (w2.z + w2.w);
    }
    xsm[bb * gps + c] = s0 + s1;
  }
  __syncthreads();
  // the rows' words of the range, copied asynchronously (consecutive threads:
  // consecutive words of a row); words past the staged stride (an allocation
  // that does not fill its rows the usual way) are not read
  const int w0 = woff[0];
  const int nw = min(woff[nc] - w0, wstride);
  for (int r = warp; r < DG_ROWS; r += DG_WARPS) {
    const bool row_ok = r0 + r < m;
    const uint32_t* src = codes + (row_ok ? r0 + r : 0) * rw + w0;
    for (int w = lane; w < nw; w += 32) {
      if (row_ok && (int64_t)w0 + w < rw)
        cp_async4(wsm + r * wstride + w, src + w);
      else
        wsm[r * wstride + w] = 0u;
    }
  }
  cp_async_wait_all();
  __syncthreads();
  // decode: warp w takes groups w, w + 8, ... of the range; lane = row
  float acc[MB];
#pragma unroll
  for (int bb = 0; bb < MB; ++bb) acc[bb] = 0.f;
  const uint32_t* myw = wsm + lane * wstride;
  for (int c = warp; c < nc; c += DG_WARPS) {
    const int b = bits[c0 + c];
    const int wl = woff[c] - w0;  // the group's first word in the staged row
    if (b < 1 || b > 8 || wl + SU * b > nw) continue;  // not a valid width or beyond the staged words: adds nothing
    float A[MB];
#pragma unroll
    for (int bb = 0; bb < MB; ++bb) A[bb] = 0.f;
    const float* xr = xfs + c * G;
#pragma unroll
    for (int j = 0; j < SU; ++j) {
      const uint32_t* wp = myw + wl + j * b;
      switch (b) {
        case 1: dg_unit<1, MB>(wp, xr + 32 * j, xstride, B, A); break;
        case 2: dg_unit<2, MB>(wp, xr + 32 * j, xstride, B, A); break;
        case 3: dg_unit<3, MB>(wp, xr + 32 * j, xstride, B, A); break;
        case 4: dg_unit<4, MB>(wp, xr + 32 * j, xstride, B, A); break;
        case 5: dg_unit<5, MB>(wp, xr + 32 * j, xstride, B, A); break;
        case 6: dg_unit<6, MB>(wp, xr + 32 * j, xstride, B, A); break;
        case 7: dg_unit<7, MB>(wp, xr + 32 * j, xstride, B, A); break;
        default: dg_unit<8, MB>(wp, xr + 32 * j, xstride, B, A); break;
      }
    }
    const float s = ssm[lane * sstride + c], z = zsm[lane * sstride + c];
    const float p2 = __int_as_float((127 + b) << 23);  // 2^b
#pragma unroll
    for (int bb = 0; bb < MB; ++bb)
      if (bb < B) {
        const float xsum = xsm[bb * gps + c];
        acc[bb] = fmaf(s, fmaf(p2, A[bb] - xsum, -z * xsum), acc[bb]);
      }
  }
#pragma unroll
  for (int bb = 0; bb < MB; ++bb)
    if (bb < B) red[(warp * B + bb) * 32 + lane] = acc[bb];
  __syncthreads();
  // the warps' sums in order; a single range writes y, several write partials [split][B][m]
  for (int e = tid; e < B * DG_ROWS; e += DG_WARPS * 32) {
    const int bb = e / DG_ROWS, r = e - bb * DG_ROWS;
    if (r0 + r >= m) continue;
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < DG_WARPS; ++w) s += red[(w * B + bb) * 32 + r];
    out[((int64_t)blockIdx.y * B + bb) * m + r0 + r] = s;
  }
}

__global__ void dg_reduce_kernel(const float* __restrict__ part, int ks, int B, int64_t m, float* __restrict__ y) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)B * m) return;
  float s = 0.f;
  for (int q = 0; q < ks; ++q) s += part[(int64_t)q * B * m + e];
  y[e] = s;
}

size_t dg_workspace_bytes(int64_t m, int64_t n, int group, int avg_bits, int64_t B) {
  const DgPlan pl = dg_plan(n, group, avg_bits, (int)B);
  return pl.ks > 1 ? (size_t)pl.ks * B * m * 4 : 0;
}

// The kernel instance's shared-memory limit raised to the plan's bound once per
// device (a flag per instance and device), not on every call.
template <int G, int MB>
static cudaError_t dg_allow_smem() {
  static std::atomic<uint64_t> done{0};
  uint64_t bit = 0;
  if (!attr_pending(done, bit)) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(dg_kernel<G, MB>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  if (e == cudaSuccess) done.fetch_or(bit);
  return e;
}

cudaError_t launch_dequant_gemv(const uint32_t* codes, const uint8_t* bits, const float* scale, const float* zero,
                                int64_t m, int64_t n, int group, int avg_bits, const void* x, int xdtype, int B,
                                float* y, uint8_t* ws, cudaStream_t s) {
  const int k = (int)(n / group);
  const int64_t rw = n * avg_bits / 32;
  const DgPlan pl = dg_plan(n, group, avg_bits, B);
  if (pl.smem > 227 * 1024) return cudaErrorInvalidValue;
  float* out = pl.ks > 1 ? reinterpret_cast<float*>(ws) : y;
  const int mb = B <= 1 ? 1 : (B <= 2 ? 2 : (B <= 4 ? 4 : 8));
  const dim3 grid((unsigned)((m + DG_ROWS - 1) / DG_ROWS), (unsigned)pl.ks);
  cudaError_t e = cudaSuccess;
#define SLIM_DG(G, MB)                                                                                           \
  do {                                                                                                           \
    if (pl.smem > 48 * 1024) e = dg_allow_smem<G, MB>();                                                         \
    if (e == cudaSuccess)                                                                                        \
      dg_kernel<G, MB><<<grid, DG_WARPS * 32, pl.smem, s>>>(codes, m, rw, bits, scale, zero, k, x, xdtype, B, n, \
                                                            pl.gps, pl.wstride, pl.sstride, out);                \
  } while (0)
#define SLIM_DG_B(G)               \
  switch (mb) {                    \
    case 1: SLIM_DG(G, 1); break;  \
    case 2: SLIM_DG(G, 2); break;  \
    case 4: SLIM_DG(G, 4); break;  \
    default: SLIM_DG(G, 8); break; \
  }
  switch (group) {
    case 32: SLIM_DG_B(32); break;
    case 64: SLIM_DG_B(64); break;
    case 128: SLIM_DG_B(128); break;
    default: return cudaErrorInvalidValue;
  }
#undef SLIM_DG_B
#undef SLIM_DG
  if (e != cudaSuccess) return e;
  int launches = 1;
  if (pl.ks > 1) {
    dg_reduce_kernel<<<(unsigned)((B * m + 255) / 256), 256, 0, s>>>(out, pl.ks, B, m, y);
    ++launches;
  }
  count_launches(launches);
  return cudaGetLastError();
}

}  // namespace slim
