// 64 x 64 fp64 tiles in shared memory and the fp64 tensor-core product
// (mma.sync m8n8k4) over them, as used by the blocked Cholesky / inverse of
// the inverse-Hessian stage and by the GPTQ update: tiles are staged by
// cp.async with a padded row stride, and a CTA of 8 warps holds one 64 x 64
// result tile in registers.
#pragma once
#include <cstdint>
#include "common.cuh"

namespace slim {

constexpr int NB = 64;         // block size
constexpr int LD = 68;         // shared row stride in doubles: 16-byte rows, conflict-free fragment loads
constexpr int TILE = NB * LD;  // doubles per shared tile
constexpr int HT = 256;        // threads per CTA of every blocked kernel
constexpr size_t kTileBytes = TILE * sizeof(double);

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

}  // namespace slim
