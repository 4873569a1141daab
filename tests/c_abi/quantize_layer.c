/*
 * A plain C caller of libslim: quantizes one synthetic layer through the
 * host-buffer entry point and checks the outputs' invariants.
 *
 *   quantize_layer [m n N group avg_bits]      (defaults 256 512 4096 128 2)
 *
 * W ~ N(0, 0.02^2) with four input columns scaled x8; X ~ N(0, 1) as bf16 with
 * two outlier channels x20 (the shape of the small synthetic layer the tests
 * use). Checks: every group's bits are avg_bits - 1, avg_bits or avg_bits + 1
 * and they sum to k * avg_bits; scales are positive; every packed code fits
 * its group's width; the dequantized layer's relative error is finite.
 * Exit status 0 when all hold.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "slim.h"

static uint64_t rng_state = 0x9E3779B97F4A7C15ull;

static double uniform01(void) {
  /* xorshift64*; 53 random bits in (0, 1) */
  rng_state ^= rng_state >> 12;
  rng_state ^= rng_state << 25;
  rng_state ^= rng_state >> 27;
  return ((double)((rng_state * 0x2545F4914F6CDD1Dull) >> 11) + 0.5) / 9007199254740992.0;
}

static double normal(void) {
  const double u = uniform01(), v = uniform01();
  return sqrt(-2.0 * log(u)) * cos(6.283185307179586 * v);
}

static uint16_t to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u); /* round to nearest even */
  return (uint16_t)(u >> 16);
}

int main(int argc, char** argv) {
  int64_t m = 256, n = 512, N = 4096;
  int group = 128, avg_bits = 2;
  if (argc == 6) {
    m = atoll(argv[1]);
    n = atoll(argv[2]);
    N = atoll(argv[3]);
    group = atoi(argv[4]);
    avg_bits = atoi(argv[5]);
  } else if (argc != 1) {
    fprintf(stderr, "usage: %s [m n N group avg_bits]\n", argv[0]);
    return 2;
  }
  if (group <= 0 || n % group != 0) {
    fprintf(stderr, "group must divide n\n");
    return 2;
  }
  const int64_t k = n / group, words = slim_row_words(n, avg_bits);
  float* W = malloc(sizeof(float) * m * n);
  uint16_t* X = malloc(sizeof(uint16_t) * N * n);
  uint32_t* codes = malloc(sizeof(uint32_t) * m * words);
  float* scale = malloc(sizeof(float) * m * k);
  float* zero = malloc(sizeof(float) * m * k);
  uint8_t* bits = malloc((size_t)k);
  if (!W || !X || !codes || !scale || !zero || !bits) {
    fprintf(stderr, "out of host memory\n");
    return 1;
  }
  for (int64_t i = 0; i < m * n; ++i) W[i] = (float)(0.02 * normal());
  for (int c = 0; c < 4; ++c) {
    const int64_t col = (int64_t)(uniform01() * (double)n);
    for (int64_t i = 0; i < m; ++i) W[i * n + col] *= 8.0f;
  }
  int64_t outl[2];
  for (int c = 0; c < 2; ++c) outl[c] = (int64_t)(uniform01() * (double)n);
  for (int64_t t = 0; t < N; ++t)
    for (int64_t j = 0; j < n; ++j) {
      float x = (float)normal();
      if (j == outl[0] || j == outl[1]) x *= 20.0f;
      X[t * n + j] = to_bf16(x);
    }

  const int rc = slim_quantize_layer_host(W, m, n, X, SLIM_X_BF16, N, group, avg_bits, 0.1, 50, codes, scale, zero,
                                          bits, NULL);
  if (rc != SLIM_OK) {
    fprintf(stderr, "slim_quantize_layer_host: %s (%s; detail %d)\n", slim_status_string(rc), slim_last_cuda_error(),
            slim_last_status_detail());
    return 1;
  }

  int ok = 1;
  int64_t sum = 0;
  for (int64_t c = 0; c < k; ++c) {
    sum += bits[c];
    if (bits[c] < avg_bits - 1 || bits[c] > avg_bits + 1) ok = 0;
  }
  if (sum != k * avg_bits) ok = 0;
  for (int64_t i = 0; i < m * k; ++i)
    if (!(scale[i] > 0.0f)) ok = 0;
  /* unpack every row: group c's codes follow the groups before it, bits[c]
     bits each, least significant bit first */
  double err2 = 0.0, ref2 = 0.0;
  for (int64_t i = 0; i < m && ok; ++i) {
    const uint32_t* row = codes + i * words;
    int64_t pos = 0;
    for (int64_t c = 0; c < k; ++c) {
      const int b = bits[c];
      for (int j = 0; j < group; ++j, pos += b) {
        const uint64_t lo = row[pos >> 5], hi = ((pos >> 5) + 1 < words) ? row[(pos >> 5) + 1] : 0;
        const uint32_t q = (uint32_t)(((hi << 32 | lo) >> (pos & 31)) & ((1u << b) - 1u));
        const float w = W[i * n + c * group + j];
        const float wh = scale[i * k + c] * ((float)q - zero[i * k + c]);
        err2 += (double)(w - wh) * (double)(w - wh);
        ref2 += (double)w * (double)w;
      }
    }
    if (pos != words * 32) ok = 0;
  }
  const double rel = sqrt(err2 / ref2);
  if (!(rel < 1.0)) ok = 0;
  printf("%s: m=%lld n=%lld N=%lld group=%d avg_bits=%d bits[0..%lld)=", ok ? "ok" : "FAILED", (long long)m,
         (long long)n, (long long)N, group, avg_bits, (long long)k);
  for (int64_t c = 0; c < k; ++c) printf("%d", bits[c]);
  printf(" relative error %.4f\n", rel);
  free(W);
  free(X);
  free(codes);
  free(scale);
  free(zero);
  free(bits);
  return ok ? 0 : 1;
}
