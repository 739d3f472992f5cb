/*
 * Seeded synthetic-input generator: counter-based random numbers, an
 * approximately normal variate, IEEE binary16 rounding and Q4_0 block
 * encoding of generated weights.
 *
 * This header is compiled twice, by gcc for the host generator and by nvcc
 * for the device generator, so that both produce the same bits for the same
 * (key, index).  It holds input preparation only: nothing here is a step of
 * the sparse-FFN method (the Q4_0 *encoder* prepares quantised weights; the
 * method's decode step lives elsewhere).
 *
 * Generator: SplitMix64 (G. Steele, D. Lea, C. Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014), used counter-style: draw i
 * of a stream with key k is the SplitMix64 output for state k + (i+1)*gamma.
 * Normal variate: Irwin-Hall sum of twelve uniforms minus six, the uniforms
 * being 16-bit fields of three consecutive draws; integer sum, one exact
 * power-of-two division, so host and device agree bit for bit.
 */
#ifndef PI_SYNTH_RNG_H
#define PI_SYNTH_RNG_H

#include <math.h>
#include <stdint.h>
#include <string.h>

#ifdef __CUDACC__
#define SY_FN static __host__ __device__ __forceinline__
#else
#define SY_FN static inline
#endif

#define SY_GAMMA 0x9E3779B97F4A7C15ULL

/* SplitMix64 output function (mix of the incremented state). */
SY_FN uint64_t sy_mix(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Stream key for one tensor of one layer of one seeded workload. */
SY_FN uint64_t sy_key(uint64_t seed, uint64_t layer, uint64_t tensor) {
  uint64_t k = sy_mix(seed * SY_GAMMA + 0x243F6A8885A308D3ULL);
  k = sy_mix(k ^ ((layer + 1) * 0xD1B54A32D192ED03ULL));
  k = sy_mix(k ^ ((tensor + 1) * 0x8CB92BA72F3D8DD7ULL));
  return k;
}

/* Draw i of the stream with key `key`. */
SY_FN uint64_t sy_u64(uint64_t key, uint64_t i) {
  return sy_mix(key + (i + 1) * SY_GAMMA);
}

/* Approximately standard normal variate number e of a stream:
 * (sum of 12 uniforms on (0,1)) - 6, each uniform = (u16 + 0.5) / 65536. */
SY_FN double sy_gauss(uint64_t key, uint64_t e) {
  int64_t n = 0;
  for (int t = 0; t < 3; ++t) {
    uint64_t v = sy_u64(key, 3 * e + (uint64_t)t);
    n += (int64_t)(v & 0xFFFFu) + (int64_t)((v >> 16) & 0xFFFFu) +
         (int64_t)((v >> 32) & 0xFFFFu) + (int64_t)((v >> 48) & 0xFFFFu);
  }
  /* sum_k (u_k + 0.5)/65536 - 6 = (n + 6 - 6*65536) / 65536, exact */
  return (double)(n + 6 - 393216) / 65536.0;
}

SY_FN uint64_t sy_double_bits(double v) {
#ifdef __CUDA_ARCH__
  return (uint64_t)__double_as_longlong(v);
#else
  uint64_t b;
  memcpy(&b, &v, sizeof b);
  return b;
#endif
}

SY_FN double sy_bits_double(uint64_t b) {
#ifdef __CUDA_ARCH__
  return __longlong_as_double((long long)b);
#else
  double v;
  memcpy(&v, &b, sizeof v);
  return v;
#endif
}

/* Round a finite double to IEEE binary16, round-to-nearest-even, returning
 * the 16 bit pattern.  Integer arithmetic only. */
SY_FN uint16_t sy_half_bits(double v) {
  uint64_t b = sy_double_bits(v);
  uint16_t sign = (uint16_t)((b >> 48) & 0x8000u);
  int e2 = (int)((b >> 52) & 0x7FF);
  if (e2 == 0x7FF) return (uint16_t)(sign | 0x7C00u); /* inf/nan -> inf */
  if (e2 == 0) return sign;                           /* zero or tiny */
  int e = e2 - 1023;
  if (e > 15) return (uint16_t)(sign | 0x7C00u);
  uint64_t m = (b & 0x000FFFFFFFFFFFFFULL) | 0x0010000000000000ULL;
  int eh = e < -14 ? -14 : e;
  int s = 42 + (eh - e); /* m >> s has 11 significant bits for normals */
  if (s >= 64) return sign;
  uint64_t q = m >> s;
  uint64_t rem = m & ((1ULL << s) - 1);
  uint64_t half = 1ULL << (s - 1);
  if (rem > half || (rem == half && (q & 1))) q += 1;
  uint64_t bits = ((uint64_t)(eh + 14) << 10) + q;
  if (bits >= 0x7C00u) bits = 0x7C00u;
  return (uint16_t)(sign | (uint16_t)bits);
}

/* Exact value of a binary16 bit pattern (used by the encoder to quantise
 * against the rounded scale). */
SY_FN double sy_half_value(uint16_t h) {
  int e = (h >> 10) & 0x1F;
  int f = h & 0x3FF;
  double mag;
  if (e == 0) {
    mag = (double)f * (1.0 / 16777216.0); /* f * 2^-24 */
  } else {
    /* (1024 + f) * 2^(e-25): build 2^(e-25) exactly from its bit pattern */
    mag = (double)(1024 + f) * sy_bits_double((uint64_t)(e - 25 + 1023) << 52);
  }
  return (h & 0x8000u) ? -mag : mag;
}

/* Encode one block of 32 weights as Q4_0: scale s = binary16(m / -8) with
 * m the element of largest magnitude (first on ties); code
 * q = clamp(floor(w/s + 8.5), 0, 15); all-zero block -> s = 0, q = 8.
 * Byte k (k < 16) holds element k in its low nibble and element k+16 in
 * its high nibble. */
SY_FN void sy_q4_0_encode(const double* w, uint8_t* qs, uint16_t* scale_bits) {
  int im = 0;
  double amax = w[0] < 0 ? -w[0] : w[0];
  for (int k = 1; k < 32; ++k) {
    double a = w[k] < 0 ? -w[k] : w[k];
    if (a > amax) { amax = a; im = k; }
  }
  uint16_t sb = sy_half_bits(w[im] / -8.0);
  double s = sy_half_value(sb);
  int q[32];
  for (int k = 0; k < 32; ++k) {
    if (s == 0.0) { q[k] = 8; continue; }
    double t = floor(w[k] / s + 8.5);
    q[k] = t < 0.0 ? 0 : (t > 15.0 ? 15 : (int)t);
  }
  for (int k = 0; k < 16; ++k) qs[k] = (uint8_t)(q[k] | (q[k + 16] << 4));
  *scale_bits = sb;
}

#endif /* PI_SYNTH_RNG_H */
