// Per-token decay factors of one chunk of C = 64 tokens whose gates are all scalars per token (GDN:
// alpha, beta^k, beta^v, d), shared by the fused per-token-gate kernel (dn_chunk_sc.cu) and the
// chunk-parallel transform kernel of the split path (dn_split_sc.cu).
//
// With gamma_t = prod_{s <= t} alpha_s (from the chunk start, token t included), kept as
// rho_t 2^{e_t} (rho in [0.5, 1)), and gamma_C / gamma_t = mu_t 2^{n_t}, the chunk's WY evaluation
// needs, per token:
//   A_ti  = (k_t . k_i) beta_i d_i rho_t / rho_i 2^{e_t - e_i}        (i < t)
//   P'_ti = (q_t . k_i) 2^{E_t - e_i} / (rho_i mu_i)                   (i <= t; i < t before the update)
//   T Diag(gamma) and T Diag(beta^v) (column factors gamma_i, beta^v_i)
//   c_t = beta_t d_t mu_t (scale of the residual row u_t), n_t (power of two on the key row k_t),
//   E_t and rho'_t (power of two on q_t and the o scale: those of gamma_t, or of gamma_{t-1} before
//   the update), gamma_C
// (see dn_chunk_sc.cu for the derivation). Every factor is a ratio of decay products of at most 1 in
// size for gates in [0, 1], so any gate strength is safe.
#pragma once

#include "dn_common.cuh"
#include "dn_tc_ptx.cuh"
#include "dn_ut_inverse.cuh"

namespace dn {
namespace scf {

constexpr int C = 64;

// Factors of one chunk, in shared memory.
struct Factors {
  float rho[C], rhoi[C];  // mantissa of gamma_t and its reciprocal
  float orho[C];          // o scale (mantissa of gamma_t, or of gamma_{t-1} before the update)
  float pinv[C];          // 1 / (rho_t mu_t)
  float c[C];             // beta^k_t d_t mu_t
  float ws[C];            // beta^k_t d_t
  float bv[C];            // beta^v_t
  float gam[C];           // gamma_t as a float (0 once it leaves the float range)
  int ex[C];              // exponent of gamma_t
  int oex[C];             // exponent of the read-out's decay (pairs with orho)
  int n[C];               // exponent of gamma_C / gamma_t
  float glast;            // gamma_C as a float
};

// The gates of token j of chunk cn (and the alpha of token j ^ 32, which the scan of the other half
// needs); absent gates read as 1, tokens past the end as alpha 1 and 0 for the others (no decay, no
// write).
struct Gates {
  float al, bk, d, bv, al_p;
};

// (Each value is preset and overwritten by a predicated load, so nothing waits for a load before
// the values are used.)
__device__ __forceinline__ Gates load_gates(const Args& a, int b, int h, int cn, int j) {
  Gates g;
  const int left = a.T - cn * C;
  const bool valid = j < left, valid_p = (j ^ 32) < left;
  const int64_t tok = ((int64_t)b * a.T + cn * C + j) * a.H + h;
  const int64_t tok_p = ((int64_t)b * a.T + cn * C + (j ^ 32)) * a.H + h;
  g.al = 1.f;
  g.bk = valid ? 1.f : 0.f;
  g.d = 1.f;
  g.bv = valid ? 1.f : 0.f;
  g.al_p = 1.f;
  if (valid && a.alpha == DN_GATE_SCALAR) g.al = __ldg(a.alpha_p + tok);
  if (valid && a.beta_k == DN_GATE_SCALAR) g.bk = __ldg(a.beta_k_p + tok);
  if (valid && a.key_scale == DN_GATE_SCALAR) g.d = __ldg(a.key_scale_p + tok);
  if (valid && a.beta_v == DN_GATE_SCALAR) g.bv = __ldg(a.beta_v_p + tok);
  if (valid_p && a.alpha == DN_GATE_SCALAR) g.al_p = __ldg(a.alpha_p + tok_p);
  return g;
}

// Factors of one chunk from the gates of its tokens. Called by the 64 threads j = 0..63 of two whole
// warps (lane = j % 32): each warp scans both halves of the chunk (lane l holds tokens l and 32 + l),
// so neither waits for the other; inclusive prefix products in mantissa-exponent form give gamma_t,
// gamma_{t-1} and gamma_C.
__device__ __forceinline__ void token_factors(const Gates& g, int j, int lane, int pre, Factors& f) {
  const bool hi = j >= 32;
  float m1, m2;
  int e1, e2;
  split_pow2(hi ? g.al_p : g.al, m1, e1);  // token lane
  split_pow2(hi ? g.al : g.al_p, m2, e2);  // token 32 + lane
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y1 = __shfl_up_sync(0xffffffffu, m1, off), y2 = __shfl_up_sync(0xffffffffu, m2, off);
    const int f1 = __shfl_up_sync(0xffffffffu, e1, off), f2 = __shfl_up_sync(0xffffffffu, e2, off);
    if (lane >= off) {
      mul_pow2(m1, e1, y1, f1);
      mul_pow2(m2, e2, y2, f2);
    }
  }
  const float t1m = __shfl_sync(0xffffffffu, m1, 31), t2m = __shfl_sync(0xffffffffu, m2, 31);
  const int t1e = __shfl_sync(0xffffffffu, e1, 31), t2e = __shfl_sync(0xffffffffu, e2, 31);
  float p1m = __shfl_up_sync(0xffffffffu, m1, 1), p2m = __shfl_up_sync(0xffffffffu, m2, 1);
  int p1e = __shfl_up_sync(0xffffffffu, e1, 1), p2e = __shfl_up_sync(0xffffffffu, e2, 1);
  float gm, pm;  // gamma_j and gamma_{j-1}
  int ge, pe;
  if (!hi) {
    gm = m1, ge = e1;
    if (lane == 0) p1m = 0.5f, p1e = 1;  // gamma_{-1} = 1
    pm = p1m, pe = p1e;
  } else {
    gm = t1m, ge = t1e;
    mul_pow2(gm, ge, m2, e2);
    pm = t1m, pe = t1e;
    if (lane > 0) mul_pow2(pm, pe, p2m, p2e);
  }
  float lm = t1m;  // gamma_C
  int le = t1e;
  mul_pow2(lm, le, t2m, t2e);
  float mu = __fdividef(lm, gm);  // gamma_C / gamma_j = mu 2^ne, mu in [0.5, 1)
  int ne = le - ge;
  if (mu >= 1.f) mu *= 0.5f, ne += 1;
  const float ws = g.bk * g.d;
  f.rho[j] = gm;
  f.rhoi[j] = __fdividef(1.f, gm);
  f.ex[j] = ge;
  f.orho[j] = pre ? pm : gm;
  f.oex[j] = pre ? pe : ge;
  f.pinv[j] = __fdividef(1.f, gm * mu);
  f.c[j] = ws * mu;
  f.n[j] = ne;
  f.gam[j] = gm * pow2f(ge);
  f.ws[j] = ws;
  f.bv[j] = g.bv;
  if (j == 63) f.glast = lm * pow2f(le);
}

// From the Gram [K; Q] K^T of the chunk in tensor memory (128 lanes x 64 columns at tmem_gram): A
// (strictly lower, scaled) into the fp32 64 x 64 array sL (ut::xi layout) from rows 0..63, and P'
// (lower incl., or strictly lower before the update) into the bf16 64 x 64 canonical tile pt from
// rows 64..127. Called by 256 threads of 8 warps; q4 = warp % 4 is the warp's lane quadrant, gch =
// warp / 4 the 32-column half it covers.
__device__ __forceinline__ void extract_ap(const Factors& f, uint32_t tmem_gram, int q4, int gch, int lane, int pre,
                                           float* sL, uint8_t* pt) {
  const uint32_t taddr = tmem_gram + ((uint32_t)(32 * q4) << 16) + 32 * gch;
  if (q4 < 2) {
    const int t = 32 * q4 + lane;
    const float rt = f.rho[t];
    const int et = f.ex[t];
    float x[32];
    tc::tmem_ld32(taddr, x);
#pragma unroll
    for (int e4 = 0; e4 < 8; ++e4) {
      float y[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i = 32 * gch + 4 * e4 + e;
        const float fa = f.ws[i] * (rt * f.rhoi[i]) * pow2f(et - f.ex[i]);  // (gamma_t / gamma_i) beta_i d_i
        y[e] = (i < t) ? x[4 * e4 + e] * fa : 0.f;
      }
      *reinterpret_cast<float4*>(sL + ut::xi(t, 32 * gch + 4 * e4)) = make_float4(y[0], y[1], y[2], y[3]);
    }
  } else {
    const int t = 32 * (q4 - 2) + lane;
    const int et = f.oex[t];
    float x[32];
    tc::tmem_ld32(taddr, x);
#pragma unroll
    for (int q8 = 0; q8 < 4; ++q8) {
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int i = 32 * gch + 8 * q8 + e;
        const float fp = f.pinv[i] * pow2f(et - f.ex[i]);  // 2^{E_t - e_i} / (rho_i mu_i)
        y[e] = (i <= t - pre) ? x[8 * q8 + e] * fp : 0.f;
      }
      *reinterpret_cast<uint4*>(pt + tc::canon_chunk(t, 4 * gch + q8, 64)) =
          make_uint4(tc::pack_bf16(y[0], y[1]), tc::pack_bf16(y[2], y[3]), tc::pack_bf16(y[4], y[5]),
                     tc::pack_bf16(y[6], y[7]));
    }
  }
}

// The same A and P' as extract_ap for a chunk whose decay exponents (ex and oex of every token) all
// lie in [-100, 100]: then gamma_t and 1 / gamma_i are plain normal floats and the factors split
// into a row part and a column part, (gamma_t / gamma_i) beta_i d_i = gamma_t * wg_i and
// 2^{E_t - e_i} / (rho_i mu_i) = 2^{E_t} * pw_i, with wg_i = beta_i d_i / gamma_i and
// pw_i = 1 / (gamma_i mu_i) precomputed per token (the powers of two are exact, so only the rounding
// order of the mantissa products differs from extract_ap).
__device__ __forceinline__ void extract_ap_fast(const Factors& f, const float* wg, const float* pw, uint32_t tmem_gram,
                                                int q4, int gch, int lane, int pre, float* sL, uint8_t* pt) {
  const uint32_t taddr = tmem_gram + ((uint32_t)(32 * q4) << 16) + 32 * gch;
  if (q4 < 2) {
    const int t = 32 * q4 + lane;
    const float gt = f.rho[t] * pow2f(f.ex[t]);
    float x[32];
    tc::tmem_ld32(taddr, x);
#pragma unroll
    for (int e4 = 0; e4 < 8; ++e4) {
      const int i0 = 32 * gch + 4 * e4;
      const float4 w = *reinterpret_cast<const float4*>(wg + i0);
      const float y0 = (i0 < t) ? x[4 * e4] * (gt * w.x) : 0.f;
      const float y1 = (i0 + 1 < t) ? x[4 * e4 + 1] * (gt * w.y) : 0.f;
      const float y2 = (i0 + 2 < t) ? x[4 * e4 + 2] * (gt * w.z) : 0.f;
      const float y3 = (i0 + 3 < t) ? x[4 * e4 + 3] * (gt * w.w) : 0.f;
      *reinterpret_cast<float4*>(sL + ut::xi(t, i0)) = make_float4(y0, y1, y2, y3);
    }
  } else {
    const int t = 32 * (q4 - 2) + lane;
    const float et = pow2f(f.oex[t]);
    float x[32];
    tc::tmem_ld32(taddr, x);
#pragma unroll
    for (int q8 = 0; q8 < 4; ++q8) {
      const int i0 = 32 * gch + 8 * q8;
      const float4 p0 = *reinterpret_cast<const float4*>(pw + i0), p1 = *reinterpret_cast<const float4*>(pw + i0 + 4);
      const float pp[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
      float y[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) y[e] = (i0 + e <= t - pre) ? x[8 * q8 + e] * (et * pp[e]) : 0.f;
      *reinterpret_cast<uint4*>(pt + tc::canon_chunk(t, 4 * gch + q8, 64)) =
          make_uint4(tc::pack_bf16(y[0], y[1]), tc::pack_bf16(y[2], y[3]), tc::pack_bf16(y[4], y[5]),
                     tc::pack_bf16(y[6], y[7]));
    }
  }
}

}  // namespace scf
}  // namespace dn
