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
// Layout of the work: lane = output row (32 rows per warp), so every lane of a
// warp decodes the same code positions (uniform control flow, x read by all
// lanes at one address); each lane reads its own row's words of a group
// (whole groups are whole words). The groups are split over gridDim.y warps
// per row block, so that enough loads are in flight; their partial sums go to
// a fixed-order reduction (deterministic). Batch rows: up to 8, each code's f
// reused for all of them. HBM-bound on the codes and the per-group scale and
// zero at batch 1.
#include <cstdint>
#include "common.cuh"

namespace slim {

constexpr int DG_WARPS = 4;
constexpr int DG_MAXB = 8;

// One warp per (batch row b, group c): x of the group's G columns as fp32
// (bf16 widened exactly) into xf, their sum into xs[b][c].
__global__ void dg_prep_kernel(int k, int G, const void* __restrict__ x, int xdtype, int B, int64_t n,
                               float* __restrict__ xf, float* __restrict__ xs) {
  const int lane = threadIdx.x & 31;
  const int e = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (e >= B * k) return;
  const int b = e / k, c = e - b * k;
  const int64_t base = (int64_t)b * n + (int64_t)c * G;
  float s = 0.f;
  for (int j = lane; j < G; j += 32) {
    float v;
    if (xdtype == 1)
      v = __uint_as_float((uint32_t)static_cast<const uint16_t*>(x)[base + j] << 16);
    else
      v = static_cast<const float*>(x)[base + j];
    xf[base + j] = v;
    s += v;
  }
  s = warp_sum(s);
  if (lane == 0) xs[e] = s;
}

// A[bb] += sum_j x[bb][j] f_j over the group's G codes (BITS each) in buf.
template <int G, int BITS>
__device__ __forceinline__ void dg_group(const uint32_t (&buf)[G / 4], const float* __restrict__ xg, int64_t n, int B,
                                         float (&A)[DG_MAXB]) {
#pragma unroll
  for (int j4 = 0; j4 < G; j4 += 4) {
    float f[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      constexpr int kMask = (1 << BITS) - 1;
      const int pos = (j4 + u) * BITS, wi = pos >> 5, off = pos & 31;
      uint32_t v;
      if (off + BITS <= 32)
        v = buf[wi] >> off;
      else
        v = __funnelshift_r(buf[wi], buf[wi + 1], off);
      f[u] = __uint_as_float(((v & kMask) << (23 - BITS)) | 0x3F800000u);
    }
#pragma unroll
    for (int bb = 0; bb < DG_MAXB; ++bb)
      if (bb < B) {
        const float4 xv = *reinterpret_cast<const float4*>(xg + (int64_t)bb * n + j4);
        A[bb] = fmaf(xv.x, f[0], A[bb]);
        A[bb] = fmaf(xv.y, f[1], A[bb]);
        A[bb] = fmaf(xv.z, f[2], A[bb]);
        A[bb] = fmaf(xv.w, f[3], A[bb]);
      }
  }
}

template <int G>
__global__ void __launch_bounds__(DG_WARPS * 32)
dg_kernel(const uint32_t* __restrict__ codes, int64_t m, int64_t rw, const uint8_t* __restrict__ bits,
          const float* __restrict__ scale, const float* __restrict__ zero, int k,
          const float* __restrict__ xf, const float* __restrict__ xs, int B, int64_t n, int gps,
          float* __restrict__ part) {
  constexpr int NW = G / 4;  // words of a group at 8 bits, the widest
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t rb = (int64_t)blockIdx.x * DG_WARPS + warp;
  const int64_t row = rb * 32 + lane;
  const bool valid = row < m;
  const int c0 = blockIdx.y * gps, c1 = (c0 + gps < k) ? c0 + gps : k;
  float acc[DG_MAXB];
#pragma unroll
  for (int bb = 0; bb < DG_MAXB; ++bb) acc[bb] = 0.f;
  const uint32_t* rowp = codes + (valid ? row : 0) * rw;
  // word offset of group c0 in a row: (G / 32) * sum of the earlier groups' bits,
  // summed by the warp's lanes (the same on every lane); later groups add theirs
  int before = 0;
  for (int c = lane; c < c0; c += 32) before += bits[c];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) before += __shfl_xor_sync(0xffffffffu, before, o);
  int ws = (G / 32) * before;
  for (int c = c0; c < c1; ws += (G / 32) * bits[c], ++c) {
    const int b = bits[c];
    const int nw = (G / 32) * b;
    uint32_t buf[NW];
#pragma unroll
    for (int u = 0; u < NW; ++u) buf[u] = (valid && u < nw && ws + u < rw) ? rowp[ws + u] : 0u;
    float A[DG_MAXB];
#pragma unroll
    for (int bb = 0; bb < DG_MAXB; ++bb) A[bb] = 0.f;
    const float* xg = xf + (int64_t)c * G;
    switch (b) {
      case 1: dg_group<G, 1>(buf, xg, n, B, A); break;
      case 2: dg_group<G, 2>(buf, xg, n, B, A); break;
      case 3: dg_group<G, 3>(buf, xg, n, B, A); break;
      case 4: dg_group<G, 4>(buf, xg, n, B, A); break;
      case 5: dg_group<G, 5>(buf, xg, n, B, A); break;
      case 6: dg_group<G, 6>(buf, xg, n, B, A); break;
      case 7: dg_group<G, 7>(buf, xg, n, B, A); break;
      case 8: dg_group<G, 8>(buf, xg, n, B, A); break;
      default: continue;  // not a valid width (the caller's precondition): the group adds nothing
    }
    const float s = valid ? scale[row * k + c] : 0.f, z = valid ? zero[row * k + c] : 0.f;
    const float p2 = (float)(1 << b);
#pragma unroll
    for (int bb = 0; bb < DG_MAXB; ++bb)
      if (bb < B) {
        const float xsum = xs[bb * k + c];
        acc[bb] = fmaf(s, fmaf(p2, A[bb] - xsum, -z * xsum), acc[bb]);
      }
  }
  if (valid)
#pragma unroll
    for (int bb = 0; bb < DG_MAXB; ++bb)
      if (bb < B) part[((int64_t)blockIdx.y * B + bb) * m + row] = acc[bb];
}

__global__ void dg_reduce_kernel(const float* __restrict__ part, int ks, int B, int64_t m, float* __restrict__ y) {
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= (int64_t)B * m) return;
  float s = 0.f;
  for (int q = 0; q < ks; ++q) s += part[(int64_t)q * B * m + e];
  y[e] = s;
}

// Splits of the groups per row block: enough warps for about 16 per SM.
static int dg_splits(int64_t m, int k, int num_sms) {
  const int64_t rbw = (m + 31) / 32;
  int64_t ks = ((int64_t)num_sms * 16 + rbw - 1) / rbw;
  if (ks > k) ks = k;
  if (ks < 1) ks = 1;
  return (int)ks;
}

size_t dg_workspace_bytes(int64_t m, int64_t n, int group, int64_t B, int num_sms) {
  const int k = (int)(n / group);
  const int ks = dg_splits(m, k, num_sms);
  auto al = [](size_t x) { return (x + 255) & ~size_t(255); };
  return al((size_t)B * n * 4) + al((size_t)B * k * 4) + al((size_t)ks * B * m * 4);
}

cudaError_t launch_dequant_gemv(const uint32_t* codes, const uint8_t* bits, const float* scale, const float* zero,
                                int64_t m, int64_t n, int group, int avg_bits, const void* x, int xdtype, int B,
                                float* y, uint8_t* ws, int num_sms, cudaStream_t s) {
  const int k = (int)(n / group);
  const int64_t rw = n * avg_bits / 32;
  const int ks = dg_splits(m, k, num_sms);
  const int gps = (k + ks - 1) / ks;
  const int ksr = (k + gps - 1) / gps;  // splits actually holding groups
  auto al = [](size_t v) { return (v + 255) & ~size_t(255); };
  float* xf = reinterpret_cast<float*>(ws);
  float* xs = reinterpret_cast<float*>(ws + al((size_t)B * n * 4));
  float* part = reinterpret_cast<float*>(ws + al((size_t)B * n * 4) + al((size_t)B * k * 4));
  dg_prep_kernel<<<(B * k + 7) / 8, 256, 0, s>>>(k, group, x, xdtype, B, n, xf, xs);
  const dim3 grid((unsigned)(((m + 31) / 32 + DG_WARPS - 1) / DG_WARPS), (unsigned)ksr);
  switch (group) {
    case 32: dg_kernel<32><<<grid, DG_WARPS * 32, 0, s>>>(codes, m, rw, bits, scale, zero, k, xf, xs, B, n, gps, part); break;
    case 64: dg_kernel<64><<<grid, DG_WARPS * 32, 0, s>>>(codes, m, rw, bits, scale, zero, k, xf, xs, B, n, gps, part); break;
    case 128: dg_kernel<128><<<grid, DG_WARPS * 32, 0, s>>>(codes, m, rw, bits, scale, zero, k, xf, xs, B, n, gps, part); break;
    default: return cudaErrorInvalidValue;
  }
  dg_reduce_kernel<<<(unsigned)((B * m + 255) / 256), 256, 0, s>>>(part, ksr, B, m, y);
  count_launches(3);
  return cudaGetLastError();
}

}  // namespace slim
