/*
 * Seeded synthetic-input generator: the arithmetic shared by the host (C) and
 * device (CUDA) builds of the generator.  It holds none of the attention
 * method's arithmetic; it only draws the Q, K, V tensors that both the CPU
 * oracle and the GPU library consume.
 *
 * Random source: Philox-4x32-10, the counter-based generator of Salmon,
 * Moraes, Dror and Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3"
 * (SC'11), written from its published definition: ten rounds of two 32x32
 * multiply-high/low products with the multipliers 0xD2511F53 and 0xCD9E8D57,
 * and a Weyl key schedule with increments 0x9E3779B9 and 0xBB67AE85.
 *
 * Normal deviates: the four 32-bit words of one Philox output are summed as
 * integers (Irwin-Hall with n = 4), centred, and scaled to unit variance.
 * Everything up to the final scaling is exact integer arithmetic, and the
 * scaling is a single correctly rounded fp64 product, so the host and device
 * builds produce bit-identical values.  The distribution is symmetric,
 * unit-variance and bounded at +-2*sqrt(3); it stands in for N(0, 1).
 *
 * Rounding: values are formed in fp64, rounded to fp32 (round to nearest
 * even), and, for bf16 tensors, rounded from fp32 to bf16 (round to nearest
 * even) by integer bit manipulation.
 *
 * Both builds compile this file with floating-point contraction disabled
 * (gcc -ffp-contract=off, nvcc -fmad=false) so that no multiply-add is fused.
 */
#ifndef SYNTH_GEN_CORE_H
#define SYNTH_GEN_CORE_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SYN_HD __host__ __device__ __forceinline__
#else
#define SYN_HD static inline
#endif

/* Tensor ids used as the top counter word. */
#define SYN_T_Q 1u
#define SYN_T_K 2u
#define SYN_T_V 3u
#define SYN_T_SHARP 16u
#define SYN_T_PLANT 17u
/* Step word for the step-independent base draw. */
#define SYN_STEP_BASE 0xFFFFFFFFu

typedef struct {
  uint32_t v[4];
} syn_u32x4;

SYN_HD uint32_t syn_mulhilo(uint32_t a, uint32_t b, uint32_t* hi) {
  uint64_t p = (uint64_t)a * (uint64_t)b;
  *hi = (uint32_t)(p >> 32);
  return (uint32_t)p;
}

/* Philox-4x32 with 10 rounds: counter c, key (k0, k1). */
SYN_HD syn_u32x4 syn_philox4x32_10(syn_u32x4 c, uint32_t k0, uint32_t k1) {
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    uint32_t hi0, hi1;
    uint32_t lo0 = syn_mulhilo(0xD2511F53u, c.v[0], &hi0);
    uint32_t lo1 = syn_mulhilo(0xCD9E8D57u, c.v[2], &hi1);
    syn_u32x4 n;
    n.v[0] = hi1 ^ c.v[1] ^ k0;
    n.v[1] = lo1;
    n.v[2] = hi0 ^ c.v[3] ^ k1;
    n.v[3] = lo0;
    c = n;
  }
  return c;
}

/* Centred Irwin-Hall integer of one Philox output: sum of the four words
 * minus its mean 2*(2^32 - 1).  Range [-(2^33 - 2), 2^33 - 2]. */
SYN_HD int64_t syn_ih_int(uint64_t elem, uint32_t step, uint32_t tensor,
                          uint32_t k0, uint32_t k1) {
  syn_u32x4 c;
  c.v[0] = (uint32_t)elem;
  c.v[1] = (uint32_t)(elem >> 32);
  c.v[2] = step;
  c.v[3] = tensor;
  syn_u32x4 w = syn_philox4x32_10(c, k0, k1);
  int64_t s = (int64_t)w.v[0] + (int64_t)w.v[1] + (int64_t)w.v[2] + (int64_t)w.v[3];
  return s - (int64_t)8589934590LL; /* 2^33 - 2 */
}

/* Unit-variance scale: the variance of a uniform integer on [0, 2^32) is
 * (2^64 - 1)/12, so the sum of four has standard deviation 2^32/sqrt(3)
 * (to within 2^-64 relative).  Passed in by the caller as sqrt(3) * 2^-32,
 * computed once in fp64. */
SYN_HD double syn_normal(uint64_t elem, uint32_t step, uint32_t tensor,
                         uint32_t k0, uint32_t k1, double unit) {
  return (double)syn_ih_int(elem, step, tensor, k0, k1) * unit;
}

/* fp32 -> bf16 bits, round to nearest even (NaN is not produced here). */
SYN_HD uint16_t syn_f32_to_bf16(float f) {
  union {
    float f;
    uint32_t u;
  } x;
  x.f = f;
  uint32_t u = x.u;
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* One element of a step tensor, in fp64 before rounding.
 *   Q:  sharp * (z_base + noise * z_step)
 *   K:  z_base + shift (planted blocks only) + noise * z_step
 *   V:  z_base + noise * z_step
 * The products and sums are written out one operation at a time; with
 * contraction disabled each is a correctly rounded IEEE operation. */
SYN_HD double syn_value(uint64_t elem, uint32_t step, uint32_t tensor, uint32_t k0,
                        uint32_t k1, double unit, double noise, double sharp,
                        double shift) {
  double zb = syn_normal(elem, SYN_STEP_BASE, tensor, k0, k1, unit);
  double zs = syn_normal(elem, step, tensor, k0, k1, unit);
  double ns = noise * zs;
  double x = zb + shift;
  x = x + ns;
  x = sharp * x;
  return x;
}

#endif
