/*
 * Host side of the seeded synthetic-input generator (see rng.h).  Fills
 * host buffers with weights ~ sigma * N(0,1) approximations in fp32, fp16 or
 * Q4_0, and exposes the scalar primitives for tests.  OpenMP over elements;
 * the result does not depend on the thread count.
 */
#include <stdint.h>
#include "rng.h"

uint64_t sy_key_of(uint64_t seed, uint64_t layer, uint64_t tensor) {
  return sy_key(seed, layer, tensor);
}

double sy_gauss_of(uint64_t key, uint64_t e) { return sy_gauss(key, e); }

uint16_t sy_half_bits_of(double v) { return sy_half_bits(v); }

void sy_fill_f32(uint64_t key, double sigma, int64_t n, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t e = 0; e < n; ++e) out[e] = (float)(sigma * sy_gauss(key, (uint64_t)e));
}

void sy_fill_f16(uint64_t key, double sigma, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
  for (int64_t e = 0; e < n; ++e) out[e] = sy_half_bits(sigma * sy_gauss(key, (uint64_t)e));
}

/* rows x cols weights (cols % 32 == 0), element (i, c) drawn as number
 * i*cols + c of the stream; qs: [rows][cols/32][16] bytes, scales:
 * [rows][cols/32] binary16 bits. */
void sy_fill_q4_0(uint64_t key, double sigma, int64_t rows, int64_t cols,
                  uint8_t* qs, uint16_t* scales) {
  int64_t nb = cols / 32;
#pragma omp parallel for schedule(static)
  for (int64_t blk = 0; blk < rows * nb; ++blk) {
    int64_t i = blk / nb, b = blk % nb;
    double w[32];
    for (int k = 0; k < 32; ++k)
      w[k] = sigma * sy_gauss(key, (uint64_t)(i * cols + b * 32 + k));
    sy_q4_0_encode(w, qs + blk * 16, scales + blk);
  }
}

/* Raw (unrounded) weights as doubles, for tests of the encoder. */
void sy_fill_f64(uint64_t key, double sigma, int64_t n, double* out) {
#pragma omp parallel for schedule(static)
  for (int64_t e = 0; e < n; ++e) out[e] = sigma * sy_gauss(key, (uint64_t)e);
}
