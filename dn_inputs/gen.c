/*
 * Seeded synthetic input generator for the gated delta-rule recurrence.
 *
 * This file holds no arithmetic of the recurrence itself: it only draws the
 * random tensors (q, k, v, gates, initial state) that both the CUDA path and
 * the fp64 oracle consume, so that the two sides see bit-identical inputs.
 *
 * Generator (counter-based, so every element is a pure function of
 * (seed, counter) and any slice can be regenerated independently):
 *   splitmix64: out(seed, c) = mix(seed + (c + 1) * 0x9E3779B97F4A7C15)
 *   uniform:    u = (out >> 11) * 2^-53                   in [0, 1)
 *   normal:     z_i = sqrt(-2 ln(1 - u_{2i})) * cos(2 pi u_{2i+1})   (Box-Muller)
 * Element i of a tensor uses counter pair (2(i+offset), 2(i+offset)+1) where i
 * is its flat row-major index.
 *
 * Transforms (all evaluated in fp64, then stored):
 *   DN_GEN_NORMAL        mean + std * z
 *   DN_GEN_UNIFORM       lo + (hi - lo) * u
 *   DN_GEN_SIGMOID       sigmoid(z)
 *   DN_GEN_EXP_NEG_SOFTPLUS  exp(-softplus(z) * scale),  softplus(x) = log(1 + e^x)
 *   DN_GEN_L2ROWS        rows of length `row` of N(0,1), each divided by its L2 norm
 * Storage: fp64, fp32 (round-to-nearest-even from fp64), or bf16 (fp64 -> fp32
 * RNE, then fp32 -> bf16 RNE on the bit pattern).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define DN_GEN_NORMAL 0
#define DN_GEN_UNIFORM 1
#define DN_GEN_SIGMOID 2
#define DN_GEN_EXP_NEG_SOFTPLUS 3
#define DN_GEN_L2ROWS 4

#define DN_OUT_F64 0
#define DN_OUT_F32 1
#define DN_OUT_BF16 2

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t splitmix_at(uint64_t seed, uint64_t ctr) {
  return mix64(seed + (ctr + 1ULL) * 0x9E3779B97F4A7C15ULL);
}

static inline double unit_at(uint64_t seed, uint64_t ctr) {
  return (double)(splitmix_at(seed, ctr) >> 11) * 0x1.0p-53;
}

static inline double normal_at(uint64_t seed, uint64_t i) {
  double u1 = 1.0 - unit_at(seed, 2 * i); /* (0, 1] keeps log finite */
  double u2 = unit_at(seed, 2 * i + 1);
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t x;
  memcpy(&x, &f, 4);
  if ((x & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((x >> 16) | 0x40u); /* NaN */
  uint32_t lsb = (x >> 16) & 1u;
  x += 0x7fffu + lsb;
  return (uint16_t)(x >> 16);
}

static inline void store(void* out, int out_kind, int64_t i, double v) {
  if (out_kind == DN_OUT_F64) {
    ((double*)out)[i] = v;
  } else if (out_kind == DN_OUT_F32) {
    ((float*)out)[i] = (float)v;
  } else {
    ((uint16_t*)out)[i] = f32_to_bf16_rne((float)v);
  }
}

static inline double transform(int kind, double p0, double p1, uint64_t seed, uint64_t i) {
  switch (kind) {
    case DN_GEN_NORMAL:
      return p0 + p1 * normal_at(seed, i);
    case DN_GEN_UNIFORM:
      return p0 + (p1 - p0) * unit_at(seed, i);
    case DN_GEN_SIGMOID: {
      double z = normal_at(seed, i);
      return 1.0 / (1.0 + exp(-z));
    }
    case DN_GEN_EXP_NEG_SOFTPLUS: {
      double z = normal_at(seed, i);
      double sp = (z > 30.0) ? z : log1p(exp(z));
      return exp(-sp * p0);
    }
    default:
      return 0.0;
  }
}

/*
 * Fill `n` elements of `out` (flat indices offset .. offset+n-1 of the stream).
 * For DN_GEN_L2ROWS, `row` is the row length and n must be a multiple of it.
 * Returns 0 on success, -1 on a bad argument.
 */
int dn_gen_fill(uint64_t seed, uint64_t offset, int64_t n, int kind, double p0, double p1,
                int64_t row, int out_kind, void* out) {
  if (n < 0 || !out) return -1;
  if (out_kind < DN_OUT_F64 || out_kind > DN_OUT_BF16) return -1;
  if (kind == DN_GEN_L2ROWS) {
    if (row <= 0 || n % row != 0) return -1;
    int64_t rows = n / row;
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
      double ss = 0.0;
      for (int64_t j = 0; j < row; ++j) {
        double z = normal_at(seed, offset + (uint64_t)(r * row + j));
        ss += z * z;
      }
      double inv = 1.0 / sqrt(ss);
      for (int64_t j = 0; j < row; ++j) {
        double z = normal_at(seed, offset + (uint64_t)(r * row + j));
        store(out, out_kind, r * row + j, z * inv);
      }
    }
    return 0;
  }
  if (kind < DN_GEN_NORMAL || kind > DN_GEN_EXP_NEG_SOFTPLUS) return -1;
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    store(out, out_kind, i, transform(kind, p0, p1, seed, offset + (uint64_t)i));
  }
  return 0;
}

/* Raw generator values, exposed so tests can pin the generator to its definition. */
uint64_t dn_gen_splitmix_at(uint64_t seed, uint64_t ctr) { return splitmix_at(seed, ctr); }
double dn_gen_normal_at(uint64_t seed, uint64_t i) { return normal_at(seed, i); }
