/*
 * synth.h - seeded, counter-based synthetic input generator.
 *
 * This module produces the inputs of the MoE layer (tokens x, router weights,
 * expert weights) for both sides of every comparison: the CPU oracle and the
 * CUDA library.  It holds none of the layer's arithmetic.  The same header is
 * compiled by g++ (host fill, synth_host.cpp) and by nvcc (device fill,
 * synth_cuda.cu); both fills must produce identical bits, which is why every
 * floating-point step below is an IEEE-754 basic operation (+, -, *, /, sqrt,
 * all correctly rounded on both processors) written so that no compiler may
 * fuse a multiply and an add:
 *   - on the device through the __dadd_rn / __dmul_rn / __ddiv_rn / __dsqrt_rn
 *     intrinsics, which are never contracted;
 *   - on the host by compiling with -ffp-contract=off and no -ffast-math.
 *
 * Definition of element i of tensor (seed, tensor_id):
 *   key    = mix64(mix64(seed) + tensor_id * GAMMA + GAMMA)
 *   b1, b2 = mix64(key + (2i+1)*GAMMA), mix64(key + (2i+2)*GAMMA)
 *            (two consecutive outputs of Steele, Lea & Flood's SplitMix64
 *             generator started at state `key`; mix64 is its output finaliser)
 *   u1     = ((b1 >> 11) + 1) * 2^-53          in (0, 1]
 *   u2     = (b2 >> 11) * 2^-53                 in [0, 1)
 *   z      = sqrt(-2 ln u1) * cos(2 pi u2)      (Box & Muller, 1958)
 *   value  = round_to_dtype(float(z * std))     (binary32 RNE, then bf16 RNE)
 *
 * ln and cos are evaluated with our own series (below) so that no libm or
 * CUDA math routine decides a bit:
 *   ln u  = e ln2 + 2 atanh(f),  f = (m-1)/(m+1),  u = m 2^e, m in (sqrt2/2, sqrt2]
 *           atanh(f) = f * sum_{j=0..10} f^(2j) / (2j+1)       (|f| <= 0.1716)
 *   cos   : quarter-turn reduction, then the Taylor series of sin and cos on
 *           [0, pi/4] in nested form, nine terms each.
 * The series are accurate to about 1e-16, far below what the bf16/fp32
 * rounding of the output keeps; bit-equality between host and device is what
 * matters and is tested.
 */
#ifndef SYNTH_H_
#define SYNTH_H_

#include <stdint.h>

#if defined(__CUDACC__)
#define SYNTH_FN __host__ __device__ __forceinline__
#else
#define SYNTH_FN static inline
#endif

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL

enum { SYNTH_BF16 = 0, SYNTH_F32 = 1 };

SYNTH_FN uint64_t synth_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

SYNTH_FN uint64_t synth_key(uint64_t seed, uint64_t tensor_id) {
  return synth_mix64(synth_mix64(seed) + tensor_id * SYNTH_GAMMA + SYNTH_GAMMA);
}

SYNTH_FN double synth_bits2d(uint64_t b) {
  union { uint64_t u; double d; } v;
  v.u = b;
  return v.d;
}
SYNTH_FN uint64_t synth_d2bits(double d) {
  union { uint64_t u; double d; } v;
  v.d = d;
  return v.u;
}

/* IEEE basic operations, never contracted into an FMA. */
SYNTH_FN double synth_add(double a, double b) {
#if defined(__CUDA_ARCH__)
  return __dadd_rn(a, b);
#else
  return a + b;
#endif
}
SYNTH_FN double synth_sub(double a, double b) {
#if defined(__CUDA_ARCH__)
  return __dsub_rn(a, b);
#else
  return a - b;
#endif
}
SYNTH_FN double synth_mul(double a, double b) {
#if defined(__CUDA_ARCH__)
  return __dmul_rn(a, b);
#else
  return a * b;
#endif
}
SYNTH_FN double synth_div(double a, double b) {
#if defined(__CUDA_ARCH__)
  return __ddiv_rn(a, b);
#else
  return a / b;
#endif
}
SYNTH_FN double synth_sqrt(double a) {
#if defined(__CUDA_ARCH__)
  return __dsqrt_rn(a);
#else
  return __builtin_sqrt(a);
#endif
}

/* Natural log of u in (0, 1], u a normal double (u >= 2^-53 here). */
SYNTH_FN double synth_log(double u) {
  const double kSqrt2 = synth_bits2d(0x3FF6A09E667F3BCDULL); /* sqrt(2) */
  const double kLn2 = synth_bits2d(0x3FE62E42FEFA39EFULL);   /* ln(2) */
  uint64_t bits = synth_d2bits(u);
  int e = (int)((bits >> 52) & 0x7FF) - 1023;
  double m = synth_bits2d((bits & 0x000FFFFFFFFFFFFFULL) | 0x3FF0000000000000ULL);
  if (m > kSqrt2) {
    m = synth_mul(m, 0.5);
    e += 1;
  }
  double f = synth_div(synth_sub(m, 1.0), synth_add(m, 1.0));
  double f2 = synth_mul(f, f);
  /* sum_{j=0..10} f2^j / (2j+1), Horner from the highest term. */
  double p = synth_div(1.0, 21.0);
  p = synth_add(synth_mul(p, f2), synth_div(1.0, 19.0));
  p = synth_add(synth_mul(p, f2), synth_div(1.0, 17.0));
  p = synth_add(synth_mul(p, f2), synth_div(1.0, 15.0));
  p = synth_add(synth_mul(p, f2), synth_div(1.0, 13.0));
  p = synth_add(synth_mul(p, f2), synth_div(1.0, 11.0));
  p = synth_add(synth_mul(p, f2), synth_div(1.0, 9.0));
  p = synth_add(synth_mul(p, f2), synth_div(1.0, 7.0));
  p = synth_add(synth_mul(p, f2), synth_div(1.0, 5.0));
  p = synth_add(synth_mul(p, f2), synth_div(1.0, 3.0));
  p = synth_add(synth_mul(p, f2), 1.0);
  double ln_m = synth_mul(synth_mul(2.0, f), p);
  return synth_add(synth_mul((double)e, kLn2), ln_m);
}

/* cos(x) and sin(x) for x in [0, pi/4], nested Taylor form (nine terms). */
SYNTH_FN double synth_cos_q(double x) {
  double x2 = synth_mul(x, x);
  double c = 1.0;
  for (int k = 9; k >= 1; --k) {
    double d = (double)((2 * k) * (2 * k - 1));
    c = synth_sub(1.0, synth_div(synth_mul(x2, c), d));
  }
  return c;
}
SYNTH_FN double synth_sin_q(double x) {
  double x2 = synth_mul(x, x);
  double s = 1.0;
  for (int k = 9; k >= 1; --k) {
    double d = (double)((2 * k) * (2 * k + 1));
    s = synth_sub(1.0, synth_div(synth_mul(x2, s), d));
  }
  return synth_mul(x, s);
}

/* cos(2 pi v) for v in [0, 1). */
SYNTH_FN double synth_cos2pi(double v) {
  const double kHalfPi = synth_bits2d(0x3FF921FB54442D18ULL); /* pi/2 */
  double w = synth_mul(v, 4.0);  /* exact */
  int q = (int)w;                /* quadrant 0..3 */
  double fr = synth_sub(w, (double)q); /* exact, in [0, 1) */
  double c, s;                   /* cos and sin of fr*pi/2 */
  if (fr > 0.5) {
    double th = synth_mul(synth_sub(1.0, fr), kHalfPi);
    c = synth_sin_q(th);
    s = synth_cos_q(th);
  } else {
    double th = synth_mul(fr, kHalfPi);
    c = synth_cos_q(th);
    s = synth_sin_q(th);
  }
  switch (q & 3) {
    case 0: return c;
    case 1: return -s;
    case 2: return -c;
    default: return s;
  }
}

/* Standard normal draw for element index i of the stream `key`. */
SYNTH_FN double synth_normal(uint64_t key, uint64_t i) {
  uint64_t b1 = synth_mix64(key + (2 * i + 1) * SYNTH_GAMMA);
  uint64_t b2 = synth_mix64(key + (2 * i + 2) * SYNTH_GAMMA);
  const double k2m53 = synth_bits2d(0x3CA0000000000000ULL); /* 2^-53 */
  double u1 = synth_mul((double)((b1 >> 11) + 1), k2m53);
  double u2 = synth_mul((double)(b2 >> 11), k2m53);
  double r = synth_sqrt(synth_mul(-2.0, synth_log(u1)));
  return synth_mul(r, synth_cos2pi(u2));
}

SYNTH_FN float synth_to_f32(double d) {
#if defined(__CUDA_ARCH__)
  return __double2float_rn(d);
#else
  return (float)d;
#endif
}

/* binary32 -> bf16 bit pattern, round to nearest even (values are finite). */
SYNTH_FN uint16_t synth_f32_to_bf16(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  uint32_t lsb = (v.u >> 16) & 1u;
  return (uint16_t)((v.u + 0x7FFFu + lsb) >> 16);
}

#endif /* SYNTH_H_ */
