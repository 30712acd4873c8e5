// Chunked backward (training pass) of the recurrence, either read-out: the gradients
// of sum <dO, o> + <dS_T, S_T> with respect to q, k, v, every gate and S0. The pages name
// chunk-parallel training (FG2-GDN page, section 3 item 2) but print no backward; the equations
// below are the chain rule through the chunk form of the forward.
//
// Chunk form (C = 64 tokens, local t = 0..C-1; g_t = sum_{s<=t} log alpha_s per key channel; r = g at
// token (n-1)/2 of the chunk's n valid tokens, a reference held fixed; h_t = g_t - r):
//   K+ = k e^h,  Q+ = q e^h,  W- = w e^-h (w = beta^k d k),  V~ = beta^v v,  S_m = Diag(e^r) S
//   T = (I + strictly-lower(K+ W-^T))^-1,  P = lower-incl(Q+ W-^T)
//   U = T (V~ - K+ S_m),  O = Q+ S_m + P U,  S' = Diag(lam) X,  X = S_m + W-^T U,  lam = e^{g_last - r}
// Reverse, given dO and the chunk-end adjoint dS':
//   dX = Diag(lam) dS',  dU = P^T dO + W- dX,  dV~ = T^T dU,  dS = Diag(e^r)(dX + Q+^T dO - K+^T dV~)
//   dP = lower-incl(dO U^T),  dL = -strictly-lower(dV~ U^T)
//   dQ+ = dO S_m^T + dP W-,  dK+ = -dV~ S_m^T + dL W-,  dW- = U dX^T + dP^T Q+ + dL^T K+
//   dh_t = Q+ dQ+ + K+ dK+ - W- dW- (per channel), plus rowsum(dX (.) X) at the last token;
//   d log alpha_s = sum_{t >= s in the chunk} dh_t; then the products back to q, k, w, gates.
// (The outputs do not depend on r, so its own adjoint terms cancel and r is held fixed.)
// Pre-update read-out (o_t = S_{t-1}^T q_t): Q+_t = q_t e^{h_t} / alpha_t and P is strictly lower, so
// dP is strictly lower, dq = e^h / alpha dQ+, and d log alpha_t also gets -Q+_t dQ+_t (not cumulated).
//
// Four kernels, all fp32 with the dense per-chunk products on warp tensor cores (mma.sync TF32 with
// a three-product hi/lo split, so each product keeps about fp32 accuracy):
//   bwd_prep   one CTA per chunk: the chunk's K+, Q+, W-, e^h, e^r, lam, T and P -> workspace
//   bwd_state  one CTA per (b, h, 32 columns of d_v), chunks in order:   S_m, U  -> workspace
//   bwd_dstate one CTA per (b, h, 64 columns of d_v), chunks in reverse: dX, dV~ -> workspace; dS0
//   bwd_local  one CTA per chunk: dq, dk, dv and the gate gradients (key channels in slices of 32)
// The two chains are sequential over chunks; all elementwise work (gates, logs, exponentials) is done
// once per chunk by bwd_prep, so a chain step only copies its operands in (cp.async) and multiplies.
#include <cstring>

#include "dn_bwd.cuh"
#include "dn_ut_inverse.cuh"

namespace dn {
namespace {

constexpr int kC = 64;     // chunk length
constexpr int kNT = 256;   // threads per CTA (8 warps)
constexpr int kDVS_STATE = 32;   // value columns per CTA of the state chain (two CTAs per SM)
constexpr int kDVS_DSTATE = 64;  // value columns per CTA of the adjoint chain (one CTA per SM, fewer waves)
constexpr int kDKS = 32;         // key channels per slice of the local-gradient kernel

struct BwdArgs {
  Args f;  // forward inputs and sizes
  const void* dO;
  const float* dS_T;
  void* gq;
  void* gk;
  void* gv;
  float* galpha;
  float* gbeta_k;
  float* gbeta_v;
  float* gkey_scale;
  float* gS0;
  float* wT;    // [BH][nc][C][C]
  float* wP;    // [BH][nc][C][C]
  float* wKp;   // [BH][nc][C][dk]: K+
  float* wQp;   // [BH][nc][C][dk]: Q+
  float* wWm;   // [BH][nc][C][dk]: W-
  float* wEh;   // [BH][nc][C][dk]: e^h
  float* wEr;   // [BH][nc][dk]:    e^r
  float* wLam;  // [BH][nc][dk]:    lam
  float* wSm;   // [BH][nc][dk][dv]
  float* wU;    // [BH][nc][C][dv]
  float* wdX;   // [BH][nc][dk][dv]
  float* wdVt;  // [BH][nc][C][dv]
  int* wFlag;   // [BH][nc]: the forward's chunks beyond the factorisation's range (null in the backward)
  int nc;
};

// ------------------------------------------------------------------ warp tensor-core products
// x = hi + lo: hi is x with the 13 low mantissa bits cleared (a TF32 value, taken with one logic op
// rather than a conversion) and lo = x - hi, exact in fp32. lo goes to the tensor core as it is: a
// TF32 operand's low 13 bits are not read, so lo enters truncated, off by less than 2^-10 |lo|, that
// is 2^-20 |x|, the size of the lo * lo product the split leaves out.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = __float_as_uint(x) & 0xffffe000u;
  lo = __float_as_uint(x - __uint_as_float(hi));
}

// acc[MI][NI] (16 x 8 fragments) += sum_{k < K} A(m, k) B(k, n) over the warp tile of 16 MI rows and
// 8 NI columns, with x = hi + lo split operands: a b ~ a_lo b_hi + a_hi b_lo + a_hi b_hi.
// BEXACT: every B(k, n) is a TF32 value (bf16 data, say), so its lo part is zero and the a_hi b_lo
// product is left out.
template <int MI, int NI, int K, bool BEXACT = false, class FA, class FB>
__device__ __forceinline__ void warp_gemm(float (&acc)[MI][NI][4], FA A, FB B, int lane) {
  const int g = lane >> 2, t = lane & 3;
  constexpr bool kSplit = MI * NI <= 4;
  constexpr int AM = kSplit ? MI : 1, AN = kSplit ? NI : 1;
  float acc_b[AM][AN][4] = {}, acc_c[AM][AN][4] = {};
#pragma unroll 2
  for (int k0 = 0; k0 < K; k0 += 8) {
    uint32_t ah[MI][4], al[MI][4];
#pragma unroll
    for (int mi = 0; mi < MI; ++mi) {
      split_tf32(A(16 * mi + g, k0 + t), ah[mi][0], al[mi][0]);
      split_tf32(A(16 * mi + g + 8, k0 + t), ah[mi][1], al[mi][1]);
      split_tf32(A(16 * mi + g, k0 + t + 4), ah[mi][2], al[mi][2]);
      split_tf32(A(16 * mi + g + 8, k0 + t + 4), ah[mi][3], al[mi][3]);
    }
    uint32_t bh[NI][2], bl[NI][2];
#pragma unroll
    for (int ni = 0; ni < NI; ++ni) {
      if constexpr (BEXACT) {
        bh[ni][0] = __float_as_uint(B(k0 + t, 8 * ni + g));
        bh[ni][1] = __float_as_uint(B(k0 + t + 4, 8 * ni + g));
      } else {
        split_tf32(B(k0 + t, 8 * ni + g), bh[ni][0], bl[ni][0]);
        split_tf32(B(k0 + t + 4, 8 * ni + g), bh[ni][1], bl[ni][1]);
      }
    }
    // issuing each round over all fragments keeps MI * NI independent products in flight; with
    // few fragments the three products also go to three accumulators, summed at the end
#pragma unroll
    for (int mi = 0; mi < MI; ++mi)
#pragma unroll
      for (int ni = 0; ni < NI; ++ni) ut::mma_tf32(acc[mi][ni], al[mi], bh[ni]);
    if constexpr (!BEXACT) {
#pragma unroll
      for (int mi = 0; mi < MI; ++mi)
#pragma unroll
        for (int ni = 0; ni < NI; ++ni) ut::mma_tf32(kSplit ? acc_b[mi % AM][ni % AN] : acc[mi][ni], ah[mi], bl[ni]);
    }
#pragma unroll
    for (int mi = 0; mi < MI; ++mi)
#pragma unroll
      for (int ni = 0; ni < NI; ++ni) ut::mma_tf32(kSplit ? acc_c[mi % AM][ni % AN] : acc[mi][ni], ah[mi], bh[ni]);
  }
  if constexpr (kSplit) {
#pragma unroll
    for (int mi = 0; mi < MI; ++mi)
#pragma unroll
      for (int ni = 0; ni < NI; ++ni)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[mi][ni][q] += acc_b[mi][ni][q] + acc_c[mi][ni][q];
  }
}

// Four 8 x 4 tiles of 32-bit words from shared memory, one register per tile and lane: lane l gives
// the address of row l % 8 of tile l / 8 and receives word l % 4 of row l / 4 of each tile (the b16
// matrix load moves every 32-bit word whole, as two adjacent 16-bit elements). For rows of fp32
// values with k contiguous this is the m16n8k8 TF32 fragment of A, or of B stored n by k.
__device__ __forceinline__ void ldm_x4(uint32_t (&r)[4], const float* row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(tc::smem_u32(row))
               : "memory");
}

__device__ __forceinline__ void split_bits(uint32_t w, uint32_t& hi, uint32_t& lo) {
  split_tf32(__uint_as_float(w), hi, lo);
}

// acc[a][MI][NI] += A_a B^T over K for NA operands A_a sharing B: each A_a is a warp tile of 16 MI
// rows, B one of 8 NI rows (NI even), both fp32 in shared memory with k contiguous (row strides lda,
// ldb: multiples of 4 floats, 16-byte aligned rows), fragments taken by matrix loads and split as
// in warp_gemm.
template <int NA, int MI, int NI, int K>
__device__ __forceinline__ void warp_gemm_ldm(float (&acc)[NA][MI][NI][4], const float* const (&A)[NA], int lda,
                                              const float* Bt, int ldb, int lane) {
  static_assert(NI % 2 == 0 && K % 8 == 0, "tiles");
  const int j = lane >> 3, r = lane & 7;
  constexpr bool kSplit = NA * MI * NI <= 4;  // three accumulators per fragment, as in warp_gemm
  constexpr int AA = kSplit ? NA : 1, AM = kSplit ? MI : 1, AN = kSplit ? NI : 1;
  float acc_b[AA][AM][AN][4] = {}, acc_c[AA][AM][AN][4] = {};
  const int aoff = ((j & 1) * 8 + r) * lda + (j >> 1) * 4;  // tiles: rows 0-7 / 8-15, k 0-3 / 4-7
  const int boff = ((j >> 1) * 8 + r) * ldb + (j & 1) * 4;  // tiles: n 0-7 / 8-15, k 0-3 / 4-7
#pragma unroll 4
  for (int k0 = 0; k0 < K; k0 += 8) {
    uint32_t bh[NI][2], bl[NI][2];
#pragma unroll
    for (int np = 0; np < NI / 2; ++np) {
      uint32_t w[4];
      ldm_x4(w, Bt + 16 * np * ldb + boff + k0);
#pragma unroll
      for (int q = 0; q < 4; ++q) split_bits(w[q], bh[2 * np + (q >> 1)][q & 1], bl[2 * np + (q >> 1)][q & 1]);
    }
#pragma unroll
    for (int a = 0; a < NA; ++a) {
      uint32_t ah[MI][4], al[MI][4];
#pragma unroll
      for (int mi = 0; mi < MI; ++mi) {
        uint32_t w[4];
        ldm_x4(w, A[a] + 16 * mi * lda + aoff + k0);
#pragma unroll
        for (int q = 0; q < 4; ++q) split_bits(w[q], ah[mi][q], al[mi][q]);
      }
#pragma unroll
      for (int mi = 0; mi < MI; ++mi)
#pragma unroll
        for (int ni = 0; ni < NI; ++ni) ut::mma_tf32(acc[a][mi][ni], al[mi], bh[ni]);
#pragma unroll
      for (int mi = 0; mi < MI; ++mi)
#pragma unroll
        for (int ni = 0; ni < NI; ++ni)
          ut::mma_tf32(kSplit ? acc_b[a % AA][mi % AM][ni % AN] : acc[a][mi][ni], ah[mi], bl[ni]);
#pragma unroll
      for (int mi = 0; mi < MI; ++mi)
#pragma unroll
        for (int ni = 0; ni < NI; ++ni)
          ut::mma_tf32(kSplit ? acc_c[a % AA][mi % AM][ni % AN] : acc[a][mi][ni], ah[mi], bh[ni]);
    }
  }
  if constexpr (kSplit) {
#pragma unroll
    for (int a = 0; a < NA; ++a)
#pragma unroll
      for (int mi = 0; mi < MI; ++mi)
#pragma unroll
        for (int ni = 0; ni < NI; ++ni)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[a][mi][ni][q] += acc_b[a][mi][ni][q] + acc_c[a][mi][ni][q];
  }
}

// E(m, n, value) for every element of the warp tile's accumulator.
template <int MI, int NI, class FE>
__device__ __forceinline__ void warp_epilogue(const float (&acc)[MI][NI][4], FE E, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int mi = 0; mi < MI; ++mi)
#pragma unroll
    for (int ni = 0; ni < NI; ++ni) {
      E(16 * mi + g, 8 * ni + 2 * t, acc[mi][ni][0]);
      E(16 * mi + g, 8 * ni + 2 * t + 1, acc[mi][ni][1]);
      E(16 * mi + g + 8, 8 * ni + 2 * t, acc[mi][ni][2]);
      E(16 * mi + g + 8, 8 * ni + 2 * t + 1, acc[mi][ni][3]);
    }
}

// ------------------------------------------------------------------ chunk quantities
__device__ __forceinline__ int64_t token(const Args& a, int b, int h, int t) {
  return ((int64_t)b * a.T + t) * a.H + h;
}

// Batched loads: N elements (token row tok0 + tt[u] H, channel / column ch[u]) of q, k or v and of a
// gate, every load issued before any value is used (the dtype and gate-mode branches are uniform and
// outside the element loop), so that they are all in flight at once. The caller clamps tt to a real
// token and masks the values of elements past the end.
template <int N>
__device__ __forceinline__ void io_load_n(float* out, const void* p, int64_t tok0, const int* tt, int H, const int* ch,
                                          int width, int bf16) {
  if (bf16) {
    const __nv_bfloat16* q = reinterpret_cast<const __nv_bfloat16*>(p);
#pragma unroll
    for (int u = 0; u < N; ++u) out[u] = __bfloat162float(q[(tok0 + (int64_t)tt[u] * H) * width + ch[u]]);
  } else {
    const float* q = reinterpret_cast<const float*>(p);
#pragma unroll
    for (int u = 0; u < N; ++u) out[u] = q[(tok0 + (int64_t)tt[u] * H) * width + ch[u]];
  }
}
template <int N>
__device__ __forceinline__ void gate_load_n(float* out, const float* g, int mode, int64_t tok0, const int* tt, int H,
                                            const int* ch, int width) {
  if (mode == DN_GATE_CHANNEL) {
#pragma unroll
    for (int u = 0; u < N; ++u) out[u] = g[(tok0 + (int64_t)tt[u] * H) * width + ch[u]];
  } else if (mode == DN_GATE_SCALAR) {
#pragma unroll
    for (int u = 0; u < N; ++u) out[u] = g[tok0 + (int64_t)tt[u] * H];
  } else {
#pragma unroll
    for (int u = 0; u < N; ++u) out[u] = 1.f;
  }
}

// Key channels [i0, i0 + NCH) of the chunk starting at token t0 (n valid tokens) of head (b, h), into
// [C][NCH + 4] arrays: hb = h_t, Kp = k e^h, Qp = q e^h, Wm = w e^-h (Kp, Qp may be null; hb may be
// Wm itself), er = e^r, lam = e^{g_last - r}; e^h also to global ehg ([C][NCH]) when not null.
// Tokens past the end have k = q = w = 0 and alpha = 1.
// Called by all kNT threads; returns after a barrier.
template <int NCH, int C = kC>
__device__ void prep_chunk(const Args& a, int b, int h, int t0, int n, int i0, float* hb, float* Kp, float* Qp,
                           float* Wm, float* er, float* lam, float* ehg, int tid, int* flag) {
  constexpr int LD = NCH + 4, PER = C * NCH / kNT, BAT = PER < 8 ? PER : 8;
  static_assert(PER * kNT == C * NCH && PER % BAT == 0, "work split");
  // Every loop below first loads a batch into registers and only then computes and stores to
  // shared memory, so a thread's global loads are all in flight at once.
  const int64_t tok0 = token(a, b, h, t0);
  constexpr int BA = PER < 16 ? PER : 16;
  static_assert(PER % BA == 0, "work split");
  for (int it0 = 0; it0 < PER; it0 += BA) {
    float al[BA];
    int tt[BA], ci[BA];
#pragma unroll
    for (int u = 0; u < BA; ++u) {
      const int e = tid + (it0 + u) * kNT, t = e / NCH, i = e % NCH;
      tt[u] = t < n ? t : 0;
      ci[u] = i0 + i;
    }
    gate_load_n<BA>(al, a.alpha_p, a.alpha, tok0, tt, a.H, ci, a.dk);
#pragma unroll
    for (int u = 0; u < BA; ++u) {
      const int e = tid + (it0 + u) * kNT, t = e / NCH, i = e % NCH;
      hb[t * LD + i] = logf(t < n ? al[u] : 1.f);
    }
  }
  __syncthreads();
  const int tr = (n - 1) / 2;
  for (int i = tid; i < NCH; i += kNT) {
    float run = 0.f, r = 0.f;
    for (int t = 0; t < C; ++t) {
      run += hb[t * LD + i];
      hb[t * LD + i] = run;
      if (t == tr) r = run;
    }
    // every exponent of the factorisation within +-80 (e^80 ~ 5.5e34), else the chunk's factors
    // would over- or underflow fp32: report it instead of returning non-finite gradients (the
    // forward marks the chunk instead, and evaluates it token by token)
    bool ok = fabsf(r) <= 80.f && fabsf(run - r) <= 80.f;
    for (int t = 0; t < C; ++t) {
      hb[t * LD + i] -= r;
      ok = ok && fabsf(hb[t * LD + i]) <= 80.f;
    }
    if (!ok) {
      if (flag)
        *flag = 1;
      else if (a.status)
        atomicExch(a.status, kDevGateRange);
    }
    er[i] = expf(r);
    lam[i] = expf(run - r);
  }
  __syncthreads();
  for (int it0 = 0; it0 < PER; it0 += BAT) {
    float kk[BAT], qq[BAT], ws[BAT], dd[BAT], al2[BAT];
    int tt[BAT], ci[BAT];
#pragma unroll
    for (int u = 0; u < BAT; ++u) {
      const int e = tid + (it0 + u) * kNT, t = e / NCH, i = e % NCH;
      tt[u] = t < n ? t : 0;
      ci[u] = i0 + i;
    }
    io_load_n<BAT>(kk, a.k, tok0, tt, a.H, ci, a.dk, a.io_bf16);
    if (Qp) io_load_n<BAT>(qq, a.q, tok0, tt, a.H, ci, a.dk, a.io_bf16);
    gate_load_n<BAT>(ws, a.beta_k_p, a.beta_k, tok0, tt, a.H, ci, a.dk);
    gate_load_n<BAT>(dd, a.key_scale_p, a.key_scale, tok0, tt, a.H, ci, a.dk);
    if (Qp && a.pre_read) gate_load_n<BAT>(al2, a.alpha_p, a.alpha, tok0, tt, a.H, ci, a.dk);
#pragma unroll
    for (int u = 0; u < BAT; ++u) {
      const int e = tid + (it0 + u) * kNT, t = e / NCH;
      if (t < n) {
        ws[u] *= dd[u];
        if (Qp && a.pre_read) qq[u] /= al2[u];  // read before the decay
      } else {
        kk[u] = qq[u] = ws[u] = 0.f;
      }
      if (!Qp) qq[u] = 0.f;
    }
#pragma unroll
    for (int u = 0; u < BAT; ++u) {
      const int e = tid + (it0 + u) * kNT, t = e / NCH, i = e % NCH;
      const float eh = expf(hb[t * LD + i]);
      if (ehg) ehg[t * NCH + i] = eh;
      if (Kp) Kp[t * LD + i] = kk[u] * eh;
      if (Qp) Qp[t * LD + i] = qq[u] * eh;
      Wm[t * LD + i] = ws[u] * kk[u] / eh;
    }
  }
  __syncthreads();
}

constexpr int kLDC = kC + 4;  // row stride of shared 64 x 64 arrays
template <int DVS>
constexpr int kLdsState = DVS + 4;
template <int DVS>
constexpr int kLdsDstate = DVS + 8;

// cp.async copy of a ROWS x COLS fp32 block (global row stride gs floats) into shared rows of ss
// floats; 16-byte granules, so COLS, gs, ss and both bases must be multiples of 4 floats. The caller
// commits and waits.
template <int ROWS, int COLS>
__device__ __forceinline__ void async_rows(float* sm, int ss, const float* g, int64_t gs, int tid) {
  constexpr int V = COLS / 4;
  static_assert(COLS % 4 == 0, "16-byte granules");
  for (int e = tid; e < ROWS * V; e += kNT) {
    const int r = e / V, c = (e % V) * 4;
    tc::cp_async_16_zfill(sm + r * ss + c, g + r * gs + c, 16);
  }
}

// T = (I + L)^-1 for the strictly lower C x C L in Lm (row stride C + 4) into Tm (same stride), fp32.
// The C / 16 diagonal blocks of 16 x 16 by forward substitution (one column per thread), then the
// blocks below the diagonal by block distance d: T_ij = -T_ii sum_{j <= k < i} L_ik T_kj.
// scr: 768 floats.
template <int C>
__device__ void inverse_blocked(const float* Lm, float* Tm, float* scr, int tid) {
  constexpr int LDC = C + 4, NB = C / 16;
  static_assert(C % 16 == 0 && NB <= 4, "16-row blocks, scratch for four");
  for (int e = tid; e < C * C; e += kNT) Tm[(e / C) * LDC + e % C] = 0.f;
  __syncthreads();
  if (tid < C) {
    const int o = (tid >> 4) * 16, j = tid & 15;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) x[i] = i == j ? 1.f : 0.f;
#pragma unroll
    for (int i = 1; i < 16; ++i) {
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < i; ++k) s = fmaf(Lm[(o + i) * LDC + o + k], x[k], s);
      if (i > j) x[i] = -s;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) Tm[(o + i) * LDC + o + j] = x[i];
  }
  __syncthreads();
  for (int d = 1; d < NB; ++d) {
    const int np = NB - d;
    for (int e = tid; e < np * 256; e += kNT) {
      const int bj = e >> 8, bi = bj + d, r = (e >> 4) & 15, col = e & 15;
      float s = 0.f;
      for (int k = bj * 16; k < bi * 16; ++k) s = fmaf(Lm[(bi * 16 + r) * LDC + k], Tm[k * LDC + bj * 16 + col], s);
      scr[e] = s;
    }
    __syncthreads();
    for (int e = tid; e < np * 256; e += kNT) {
      const int bj = e >> 8, bi = bj + d, r = (e >> 4) & 15, col = e & 15;
      float s = 0.f;
#pragma unroll
      for (int k = 0; k < 16; ++k) s = fmaf(Tm[(bi * 16 + r) * LDC + bi * 16 + k], scr[(bj << 8) + (k << 4) + col], s);
      Tm[(bi * 16 + r) * LDC + bj * 16 + col] = -s;
    }
    __syncthreads();
  }
}

// ------------------------------------------------------------------ kernel 1: per-chunk operands
// (C tokens per chunk: 64 for the backward; the forward takes 16, 32 or 64)
template <int DK, int C = kC>
__global__ void __launch_bounds__(kNT) bwd_prep_kernel(BwdArgs p) {
  extern __shared__ float4 smem4[];
  constexpr int LDK = DK + 4, LDC = C + 4;
  float* Kp = reinterpret_cast<float*>(smem4);
  float* Qp = Kp + C * LDK;
  float* Wm = Qp + C * LDK;
  float* scr = Wm + C * LDK;
  float* er = scr + 768;
  float* lam = er + DK;
  float* Lm = Kp;  // once K+ and Q+ are consumed, their space holds L and T
  float* Tm = Qp;
  const Args& a = p.f;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x % p.nc, bh = blockIdx.x / p.nc, b = bh / a.H, h = bh % a.H;
  const int t0 = c * C, n = min(C, a.T - t0);
  const int64_t cb = (int64_t)bh * p.nc + c;
  if (p.wFlag && tid == 0) p.wFlag[cb] = 0;  // (ordered before any mark by prep_chunk's first barrier)
  prep_chunk<DK, C>(a, b, h, t0, n, 0, Wm, Kp, Qp, Wm, er, lam, p.wEh ? p.wEh + cb * C * DK : nullptr, tid,
                    p.wFlag ? p.wFlag + cb : nullptr);

  // warps 0-3: L = strictly-lower(K+ W-^T) (kept in registers); warps 4-7: P = lower(Q+ W-^T), with the
  // diagonal for the post read-out and without it for the pre read-out. Warp tiles of WM x WN: 32 x 32
  // (C = 64), 16 x 16 (C = 32: four per product; C = 16: one, the other three warps of the four idle)
  constexpr int MI = C >= 64 ? 2 : 1, NI = C >= 64 ? 4 : 2, WM = 16 * MI, WN = 8 * NI;
  constexpr int NWN = C / WN, NW = (C / WM) * NWN;
  static_assert(NW <= 4, "four warps per product");
  const int wi = warp & 3;
  const bool gram = wi < NW;
  const int m0 = (wi / NWN) * WM, n0 = (wi % NWN) * WN;
  float acc[MI][NI][4] = {};
  if (gram) {
    const float* X = warp < 4 ? Kp : Qp;
    warp_gemm<MI, NI, DK>(
        acc, [&](int m, int k) { return X[(m0 + m) * LDK + k]; }, [&](int k, int nn) { return Wm[(n0 + nn) * LDK + k]; },
        lane);
  }
  if (warp >= 4 && gram) {
    float* P = p.wP + cb * C * C;
    const int diag = a.pre_read ? 0 : 1;  // the pre read-out excludes the token's own write
    warp_epilogue(acc, [&](int m, int nn, float v) { P[(m0 + m) * C + n0 + nn] = n0 + nn < m0 + m + diag ? v : 0.f; },
                  lane);
  }
  if (tid < DK) {
    p.wEr[cb * DK + tid] = er[tid];
    p.wLam[cb * DK + tid] = lam[tid];
  }
  {  // K+, Q+, W- to the workspace
    float* dst[3] = {p.wKp + cb * C * DK, p.wQp + cb * C * DK, p.wWm + cb * C * DK};
    const float* src[3] = {Kp, Qp, Wm};
#pragma unroll
    for (int q = 0; q < 3; ++q)
      for (int e = tid; e < C * DK / 4; e += kNT) {
        const int t = e / (DK / 4), i = (e % (DK / 4)) * 4;
        *reinterpret_cast<float4*>(dst[q] + t * DK + i) = *reinterpret_cast<const float4*>(src[q] + t * LDK + i);
      }
  }
  __syncthreads();  // K+ and Q+ are consumed
  if (warp < 4 && gram)
    warp_epilogue(acc, [&](int m, int nn, float v) { Lm[(m0 + m) * LDC + n0 + nn] = n0 + nn < m0 + m ? v : 0.f; }, lane);
  __syncthreads();
  inverse_blocked<C>(Lm, Tm, scr, tid);
  float* Tg = p.wT + cb * C * C;
  for (int e = tid; e < C * C; e += kNT) Tg[e] = Tm[(e / C) * LDC + e % C];
}

// ------------------------------------------------------------------ kernel 2: states, chunks in order
template <int DK, int DV, int DVS, int C = kC>
__global__ void __launch_bounds__(kNT) bwd_state_kernel(BwdArgs p) {
  extern __shared__ float4 smem4[];
  // row stride of the [.][DVS] arrays: = 4 (mod 32) banks, so the lanes of a B fragment (rows t, columns
  // g) fall on at most two of them, with two CTAs per SM still fitting
  // (W- is read only transposed, rows t and columns g of a fragment: its stride is = 8 (mod 32) banks)
  constexpr int LDK = DK + 4, LDW = DK + 8, LDS = kLdsState<DVS>, LDC = C + 4, NI = DVS / 16;
  // warp tiles of the C x DVS products: RT x CT tiles of 16 x TW (with C = 16 and 32 columns, four warps)
  constexpr int RT = C / 16, CT = (8 / RT < DVS / 8) ? 8 / RT : DVS / 8, TW = DVS / CT, NIT = TW / 8;
  static_assert(RT * CT <= 8 && TW % 8 == 0, "warp tiles");
  float* S = reinterpret_cast<float*>(smem4);  // [DK][LDS]
  float* Kp = S + DK * LDS;                     // [C][LDK]
  float* Wm = Kp + C * LDK;                     // [C][LDW]
  float* Tm = Wm + C * LDW;                     // [C][LDC]
  float* R = Tm + C * LDC;                      // [C][LDS]: V~ - K+ S_m, then U
  float* erb = R + C * LDS;                     // [2][DK] (chunk parity)
  float* lamb = erb + 2 * DK;                   // [2][DK]
  const Args& a = p.f;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int NS = DV / DVS;
  constexpr int PER = C * DVS / kNT;
  const int bh = blockIdx.x / NS, j0 = (blockIdx.x % NS) * DVS, b = bh / a.H, h = bh % a.H;
  // Each chunk's operands are copied in as soon as their buffers are free (K+ with e^r and lam after
  // the K+ S_m product, T after U = T R, W- after the state update) and V~ comes in through registers
  // during the state update, so that a step does not wait for its loads. cp.async groups per chunk, in
  // issue order: A1 = {K+, e^r, lam}, A2 = {T}, B = {W-} (empty past the last chunk).
  auto cbk = [&](int c) { return (int64_t)bh * p.nc + c; };
  auto issue_a1 = [&](int c) {
    if (c < p.nc) {
      async_rows<C, DK>(Kp, LDK, p.wKp + cbk(c) * C * DK, DK, tid);
      async_rows<1, DK>(erb + (c & 1) * DK, 0, p.wEr + cbk(c) * DK, 0, tid);
      async_rows<1, DK>(lamb + (c & 1) * DK, 0, p.wLam + cbk(c) * DK, 0, tid);
    }
    tc::cp_async_commit();
  };
  auto issue_a2 = [&](int c) {
    if (c < p.nc) async_rows<C, C>(Tm, LDC, p.wT + cbk(c) * C * C, C, tid);
    tc::cp_async_commit();
  };
  auto issue_b = [&](int c) {
    if (c < p.nc) async_rows<C, DK>(Wm, LDW, p.wWm + cbk(c) * C * DK, DK, tid);
    tc::cp_async_commit();
  };
  auto load_v = [&](int c, float* x) {  // V~ = beta^v v of chunk c, this thread's elements
    const int t0 = c * C, n = min(C, a.T - t0);
    const int64_t tok0 = token(a, b, h, t0);
    int tt[PER], cj[PER];
    float bv[PER];
#pragma unroll
    for (int it = 0; it < PER; ++it) {
      const int e = tid + it * kNT, t = e / DVS, j = e % DVS;
      tt[it] = t < n ? t : 0;
      cj[it] = j0 + j;
    }
    io_load_n<PER>(x, a.v, tok0, tt, a.H, cj, DV, a.io_bf16);
    gate_load_n<PER>(bv, a.beta_v_p, a.beta_v, tok0, tt, a.H, cj, DV);
#pragma unroll
    for (int it = 0; it < PER; ++it) {
      const int t = (tid + it * kNT) / DVS;
      x[it] = t < n ? x[it] * bv[it] : 0.f;
    }
  };
  for (int e = tid; e < DK * DVS; e += kNT) {
    const int i = e / DVS, j = e % DVS;
    S[i * LDS + j] = a.S0 ? a.S0[((int64_t)bh * DK + i) * DV + j0 + j] : 0.f;
  }
  const bool tiled = warp < RT * CT;
  const int m0 = (warp / CT) * 16, n0 = (warp % CT) * TW;  // this warp's tile of a C x DVS result
  float xv[PER];
  if (p.nc > 0) {
    issue_a1(0);
    issue_a2(0);
    issue_b(0);
    load_v(0, xv);
  }
  for (int c = 0; c < p.nc; ++c) {
    const int t0 = c * C, n = min(C, a.T - t0);
    const int64_t cb = (int64_t)bh * p.nc + c;
    const float* er = erb + (c & 1) * DK;
    const float* lam = lamb + (c & 1) * DK;
    __syncthreads();  // the previous chunk is done with every buffer
    if (p.wFlag && p.wFlag[cb]) {
      tc::cp_async_wait_all();  // (this chunk's copies are not used; none may still be in flight below)
      // (forward) a chunk beyond the factorisation's range: its tokens one by one, exactly, on this
      // CTA's columns; thread (j, part) owns column j and DK / TPC rows of it, so the sums over the
      // rows take TPC - 1 shuffles. S holds the true state before and after.
      constexpr int TPC = kNT / DVS, RW = DK / TPC;
      const int j = tid / TPC, part = tid % TPC, k0 = part * RW;
      float Sr[RW];
#pragma unroll
      for (int r = 0; r < RW; ++r) Sr[r] = S[(k0 + r) * LDS + j];
      for (int t = 0; t < n; ++t) {
        const int64_t tok = token(a, b, h, t0 + t);
        float al[RW], kk[RW], qq[RW], ws[RW];
#pragma unroll
        for (int r = 0; r < RW; ++r) {
          al[r] = gate_load(a.alpha_p, a.alpha, tok, DK, k0 + r);
          kk[r] = io_load(a.k, tok * DK + k0 + r, a.io_bf16);
          qq[r] = io_load(a.q, tok * DK + k0 + r, a.io_bf16);
          ws[r] = gate_load(a.beta_k_p, a.beta_k, tok, DK, k0 + r) * gate_load(a.key_scale_p, a.key_scale, tok, DK, k0 + r);
        }
        const float vt = gate_load(a.beta_v_p, a.beta_v, tok, DV, j0 + j) * io_load(a.v, tok * DV + j0 + j, a.io_bf16);
        float rr = 0.f, ss = 0.f, wq = 0.f;  // (alpha (.) S)^T k, the read-out's S^T q and w . q over these rows
#pragma unroll
        for (int r = 0; r < RW; ++r) {
          const float sb = al[r] * Sr[r];
          rr = fmaf(sb, kk[r], rr);
          ss = fmaf(a.pre_read ? Sr[r] : sb, qq[r], ss);
          wq = fmaf(ws[r] * kk[r], qq[r], wq);
          Sr[r] = sb;
        }
#pragma unroll
        for (int off = 1; off < TPC; off <<= 1) {
          rr += __shfl_xor_sync(0xffffffffu, rr, off);
          ss += __shfl_xor_sync(0xffffffffu, ss, off);
          wq += __shfl_xor_sync(0xffffffffu, wq, off);
        }
        const float u = vt - rr;  // u_t = beta^v v_t - S_bar^T k_t
#pragma unroll
        for (int r = 0; r < RW; ++r) Sr[r] = fmaf(ws[r] * kk[r], u, Sr[r]);
        // o_t = S_t^T q_t = S_bar^T q_t + (w . q) u_t; before the update: S_{t-1}^T q_t
        if (part == 0) io_store(a.o, tok * DV + j0 + j, a.pre_read ? ss : fmaf(wq, u, ss), a.io_bf16);
      }
#pragma unroll
      for (int r = 0; r < RW; ++r) S[(k0 + r) * LDS + j] = Sr[r];
      issue_a1(c + 1);
      issue_a2(c + 1);
      issue_b(c + 1);
      if (c + 1 < p.nc) load_v(c + 1, xv);
      continue;
    }
#pragma unroll
    for (int it = 0; it < PER; ++it) {
      const int e = tid + it * kNT;
      R[(e / DVS) * LDS + e % DVS] = xv[it];
    }
    tc::cp_async_wait_group<2>();  // A1(c) has landed (A2(c), B(c) may still be in flight)
    __syncthreads();
    float* Smg = p.wSm + cb * DK * DV;
    for (int e = tid; e < DK * DVS / 4; e += kNT) {  // four columns per thread: 16-byte stores
      const int i = e / (DVS / 4), j = (e % (DVS / 4)) * 4;
      float2* r = reinterpret_cast<float2*>(&S[i * LDS + j]);  // (rows are 8-byte aligned)
      const float f = er[i];
      const float2 x0 = r[0], x1 = r[1];
      const float4 y = make_float4(x0.x * f, x0.y * f, x1.x * f, x1.y * f);
      r[0] = make_float2(y.x, y.y);
      r[1] = make_float2(y.z, y.w);
      *reinterpret_cast<float4*>(&Smg[(int64_t)i * DV + j0 + j]) = y;
    }
    __syncthreads();
    if (tiled) {  // R = V~ - K+ S_m (each warp updates only its own tile)
      float acc[1][NIT][4] = {};
      warp_gemm<1, NIT, DK>(
          acc, [&](int m, int k) { return Kp[(m0 + m) * LDK + k]; }, [&](int k, int nn) { return S[k * LDS + n0 + nn]; },
          lane);
      warp_epilogue(acc, [&](int m, int nn, float v) { R[(m0 + m) * LDS + n0 + nn] -= v; }, lane);
    }
    tc::cp_async_wait_group<1>();  // A2(c) has landed (B(c) may still be in flight)
    __syncthreads();
    issue_a1(c + 1);  // K+ is free
    {  // U = T R
      float acc[1][NIT][4] = {};
      if (tiled)
        warp_gemm<1, NIT, C>(
            acc, [&](int m, int k) { return Tm[(m0 + m) * LDC + k]; }, [&](int k, int nn) { return R[k * LDS + n0 + nn]; },
            lane);
      __syncthreads();
      issue_a2(c + 1);  // T is free
      float* Ug = p.wU + cb * C * DV;
      if (tiled)
        warp_epilogue(acc,
                      [&](int m, int nn, float v) {
                        R[(m0 + m) * LDS + n0 + nn] = v;
                        Ug[(int64_t)(m0 + m) * DV + j0 + n0 + nn] = v;
                      },
                      lane);
    }
    if (c + 1 < p.nc) load_v(c + 1, xv);
    tc::cp_async_wait_group<2>();  // B(c) has landed (A1(c + 1), A2(c + 1) may still be in flight)
    __syncthreads();
    // S' = Diag(lam) (S_m + W-^T U): DK x DVS in 16 x DVS/2 tiles
    for (int tile = warp; tile < (DK / 16) * 2; tile += kNT / 32) {
      const int r0 = (tile >> 1) * 16, q0 = (tile & 1) * (DVS / 2);
      float acc[1][NI][4] = {};
      warp_gemm<1, NI, C>(
          acc, [&](int m, int k) { return Wm[k * LDW + r0 + m]; }, [&](int k, int nn) { return R[k * LDS + q0 + nn]; },
          lane);
      warp_epilogue(acc,
                    [&](int m, int nn, float v) {
                      float* s = &S[(r0 + m) * LDS + q0 + nn];
                      *s = lam[r0 + m] * (*s + v);
                    },
                    lane);
    }
    __syncthreads();  // W- is free
    issue_b(c + 1);
  }
  tc::cp_async_wait_all();
  if (p.wFlag) {  // (forward) S_T
    __syncthreads();
    for (int e = tid; e < DK * DVS; e += kNT) {
      const int i = e / DVS, j = e % DVS;
      a.S[((int64_t)bh * DK + i) * DV + j0 + j] = S[i * LDS + j];
    }
  }
}

// ------------------------------------------------------------------ kernel 3: state adjoints, chunks in reverse
// Each chunk's operands are copied in as soon as their buffers are free, so that a step of the chain
// does not wait for its loads: W- and P (with e^r and lam, double-buffered) after the dU product, T
// after the dV~ product, Q+ and K+ after the dS product, and dO (double-buffered) through registers
// during the dV~ and dS products. cp.async groups per step, in issue order: A1 = {W-, P, e^r, lam},
// A2 = {T}, B = {Q+, K+} (empty groups past the first chunk keep the count).
template <int DK, int DV, int DVS>
__global__ void __launch_bounds__(kNT) bwd_dstate_kernel(BwdArgs p) {
  extern __shared__ float4 smem4[];
  // row stride of the [.][DVS] arrays: = 8 (mod 32) banks, so the 32 lanes of a B fragment (rows t,
  // columns g) fall on 32 different banks
  // (Q+ and K+ are read only transposed: their stride is = 8 (mod 32) banks; W- is read by rows)
  constexpr int LDK = DK + 4, LDQ = DK + 8, LDS = kLdsDstate<DVS>, NI = DVS / 16;
  constexpr int PER = kC * DVS / kNT;
  float* dS = reinterpret_cast<float*>(smem4);  // [DK][LDS]: dS', then dX, then dS
  float* Qp = dS + DK * LDS;                     // [C][LDQ]
  float* Kp = Qp + kC * LDQ;                     // [C][LDQ]
  float* Wm = Kp + kC * LDQ;                     // [C][LDK]
  float* Tm = Wm + kC * LDK;  // [C][kLDC]
  float* Pm = Tm + kC * kLDC;
  float* dO0 = Pm + kC * kLDC;  // [C][LDS] x 2 (chunk parity)
  float* dO1 = dO0 + kC * LDS;
  float* dU = dO1 + kC * LDS;   // [C][LDS]: dU, then dV~
  float* erb = dU + kC * LDS;   // [2][DK]
  float* lamb = erb + 2 * DK;   // [2][DK]
  const Args& a = p.f;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  constexpr int NS = DV / DVS;
  const int bh = blockIdx.x / NS, j0 = (blockIdx.x % NS) * DVS, b = bh / a.H, h = bh % a.H;
  auto cbk = [&](int c) { return (int64_t)bh * p.nc + c; };
  auto issue_a1 = [&](int c) {
    if (c >= 0) {
      async_rows<kC, DK>(Wm, LDK, p.wWm + cbk(c) * kC * DK, DK, tid);
      async_rows<kC, kC>(Pm, kLDC, p.wP + cbk(c) * kC * kC, kC, tid);
      async_rows<1, DK>(erb + (c & 1) * DK, 0, p.wEr + cbk(c) * DK, 0, tid);
      async_rows<1, DK>(lamb + (c & 1) * DK, 0, p.wLam + cbk(c) * DK, 0, tid);
    }
    tc::cp_async_commit();
  };
  auto issue_a2 = [&](int c) {
    if (c >= 0) async_rows<kC, kC>(Tm, kLDC, p.wT + cbk(c) * kC * kC, kC, tid);
    tc::cp_async_commit();
  };
  auto issue_b = [&](int c) {
    if (c >= 0) {
      async_rows<kC, DK>(Qp, LDQ, p.wQp + cbk(c) * kC * DK, DK, tid);
      async_rows<kC, DK>(Kp, LDQ, p.wKp + cbk(c) * kC * DK, DK, tid);
    }
    tc::cp_async_commit();
  };
  auto load_dO = [&](int c, float* x) {
    const int t0 = c * kC, n = min(kC, a.T - t0);
    const int64_t tok0 = token(a, b, h, t0);
    int tt[PER], cj[PER];
#pragma unroll
    for (int it = 0; it < PER; ++it) {
      const int e = tid + it * kNT, t = e / DVS, j = e % DVS;
      tt[it] = t < n ? t : 0;
      cj[it] = j0 + j;
    }
    io_load_n<PER>(x, p.dO, tok0, tt, a.H, cj, DV, a.io_bf16);
#pragma unroll
    for (int it = 0; it < PER; ++it)
      if ((tid + it * kNT) / DVS >= n) x[it] = 0.f;
  };
  auto store_dO = [&](int c, const float* x) {
    float* d = (c & 1) ? dO1 : dO0;
#pragma unroll
    for (int it = 0; it < PER; ++it) {
      const int e = tid + it * kNT;
      d[(e / DVS) * LDS + e % DVS] = x[it];
    }
  };
  for (int e = tid; e < DK * DVS; e += kNT) {
    const int i = e / DVS, j = e % DVS;
    dS[i * LDS + j] = p.dS_T ? p.dS_T[((int64_t)bh * DK + i) * DV + j0 + j] : 0.f;
  }
  if (p.nc > 0) {
    issue_a1(p.nc - 1);
    issue_a2(p.nc - 1);
    issue_b(p.nc - 1);
    float x[PER];
    load_dO(p.nc - 1, x);
    store_dO(p.nc - 1, x);
  }
  const int m0 = (warp >> 1) * 16, n0 = (warp & 1) * (DVS / 2);
  for (int c = p.nc - 1; c >= 0; --c) {
    const int64_t cb = cbk(c);
    const float* dOs = (c & 1) ? dO1 : dO0;
    const float* er = erb + (c & 1) * DK;
    const float* lam = lamb + (c & 1) * DK;
    tc::cp_async_wait_group<1>();  // A1(c) and A2(c) have landed (B(c) may still be in flight)
    __syncthreads();               // and for every thread; dO(c) is stored; the previous step is done
    float* dXg = p.wdX + cb * DK * DV;
    for (int e = tid; e < DK * DVS / 4; e += kNT) {  // four columns per thread: 16-byte stores
      const int i = e / (DVS / 4), j = (e % (DVS / 4)) * 4;
      float2* r = reinterpret_cast<float2*>(&dS[i * LDS + j]);  // (rows are 8-byte aligned)
      const float f = lam[i];
      const float2 x0 = r[0], x1 = r[1];
      const float4 y = make_float4(x0.x * f, x0.y * f, x1.x * f, x1.y * f);
      r[0] = make_float2(y.x, y.y);
      r[1] = make_float2(y.z, y.w);
      *reinterpret_cast<float4*>(&dXg[(int64_t)i * DV + j0 + j]) = y;
    }
    __syncthreads();
    {  // dU = P^T dO + W- dX (dO from bf16 io is exact in TF32)
      float acc[1][NI][4] = {};
      const auto pT = [&](int m, int k) { return Pm[k * kLDC + m0 + m]; };
      const auto dOb = [&](int k, int nn) { return dOs[k * LDS + n0 + nn]; };
      if (a.io_bf16)
        warp_gemm<1, NI, kC, true>(acc, pT, dOb, lane);
      else
        warp_gemm<1, NI, kC>(acc, pT, dOb, lane);
      warp_gemm<1, NI, DK>(
          acc, [&](int m, int k) { return Wm[(m0 + m) * LDK + k]; }, [&](int k, int nn) { return dS[k * LDS + n0 + nn]; },
          lane);
      warp_epilogue(acc, [&](int m, int nn, float v) { dU[(m0 + m) * LDS + n0 + nn] = v; }, lane);
    }
    __syncthreads();
    issue_a1(c - 1);  // W- and P are free
    float xo[PER];
    if (c > 0) load_dO(c - 1, xo);
    {  // dV~ = T^T dU
      float acc[1][NI][4] = {};
      warp_gemm<1, NI, kC>(
          acc, [&](int m, int k) { return Tm[k * kLDC + m0 + m]; }, [&](int k, int nn) { return dU[k * LDS + n0 + nn]; },
          lane);
      __syncthreads();
      float* dVg = p.wdVt + cb * kC * DV;
      warp_epilogue(acc,
                    [&](int m, int nn, float v) {
                      dU[(m0 + m) * LDS + n0 + nn] = v;
                      dVg[(int64_t)(m0 + m) * DV + j0 + n0 + nn] = v;
                    },
                    lane);
    }
    issue_a2(c - 1);               // T is free (every warp passed the barrier inside the product above)
    tc::cp_async_wait_group<2>();  // B(c) has landed (A1(c - 1), A2(c - 1) may still be in flight)
    __syncthreads();
    // dS = Diag(e^r) (dX + Q+^T dO - K+^T dV~): DK x DVS in 16 x DVS/2 tiles
    for (int tile = warp; tile < (DK / 16) * 2; tile += kNT / 32) {
      const int r0 = (tile >> 1) * 16, q0 = (tile & 1) * (DVS / 2);
      float acc[1][NI][4] = {};
      const auto qT = [&](int m, int k) { return Qp[k * LDQ + r0 + m]; };
      const auto dOb = [&](int k, int nn) { return dOs[k * LDS + q0 + nn]; };
      if (a.io_bf16)
        warp_gemm<1, NI, kC, true>(acc, qT, dOb, lane);
      else
        warp_gemm<1, NI, kC>(acc, qT, dOb, lane);
      warp_gemm<1, NI, kC>(
          acc, [&](int m, int k) { return -Kp[k * LDQ + r0 + m]; }, [&](int k, int nn) { return dU[k * LDS + q0 + nn]; },
          lane);
      warp_epilogue(acc,
                    [&](int m, int nn, float v) {
                      float* s = &dS[(r0 + m) * LDS + q0 + nn];
                      *s = er[r0 + m] * (*s + v);
                    },
                    lane);
    }
    __syncthreads();  // Q+, K+ and dO(c + 1)'s buffer are free
    issue_b(c - 1);
    if (c > 0) store_dO(c - 1, xo);
  }
  tc::cp_async_wait_all();
  if (p.gS0) {
    __syncthreads();
    for (int e = tid; e < DK * DVS; e += kNT) {
      const int i = e / DVS, j = e % DVS;
      p.gS0[((int64_t)bh * DK + i) * DV + j0 + j] = dS[i * LDS + j];
    }
  }
}

// ------------------------------------------------------------------ kernel 4: per-token gradients
template <int DK, int DV>
__global__ void __launch_bounds__(kNT) bwd_local_kernel(BwdArgs p) {
  extern __shared__ float4 smem4[];
  // LDS: = 8 (mod 32) banks, for the [C][kDKS] tiles read as transposed fragments (rows t, columns g)
  constexpr int LDV = DV + 4, LDS = kDKS + 8;
  float* U = reinterpret_cast<float*>(smem4);  // [C][LDV]
  float* dVt = U + kC * LDV;
  float* dOs = dVt + kC * LDV;
  float* dP = dOs + kC * LDV;   // [C][kLDC]
  float* dL = dP + kC * kLDC;
  float* Sm = dL + kC * kLDC;   // [kDKS][LDV]: rows i0.. of S_m
  float* dX = Sm + kDKS * LDV;  // [kDKS][LDV]
  float* Eh = dX + kDKS * LDV;  // [C][LDS]: e^h
  float* Qp = Eh + kC * LDS;    // then the beta^k gradient terms
  float* Kp = Qp + kC * LDS;    // then the d gradient terms
  float* Wm = Kp + kC * LDS;    // then dh, then d log alpha
  float* Xq = Wm + kC * LDS;    // Q+ (.) dQ+, the pre read-out's own-token decay term
  float* red = Xq + kC * LDS;   // [4][kDKS]
  float* acc_a = red + 4 * kDKS;  // [C] per-token sums for gates of width 1
  float* acc_bk = acc_a + kC;
  float* acc_d = acc_bk + kC;
  const Args& a = p.f;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x % p.nc, bh = blockIdx.x / p.nc, b = bh / a.H, h = bh % a.H;
  const int t0 = c * kC, n = min(kC, a.T - t0);
  const int64_t cb = (int64_t)bh * p.nc + c;
  {
    constexpr int PER4 = kC * DV / 4 / kNT;  // float4 per thread of a C x DV array
    const float4* Ug = reinterpret_cast<const float4*>(p.wU + cb * kC * DV);
    const float4* dVg = reinterpret_cast<const float4*>(p.wdVt + cb * kC * DV);
    float4 xu[PER4], xv[PER4];
#pragma unroll
    for (int it = 0; it < PER4; ++it) {
      xu[it] = Ug[tid + it * kNT];
      xv[it] = dVg[tid + it * kNT];
    }
    // dO rows in 16-byte vectors (8 bf16 or 4 fp32 values), issued with the loads above; rows past the
    // end read the chunk's first row and are stored as zeros
    constexpr int VB = DV / 8, PB = kC * VB / kNT, VF = DV / 4, PF = kC * VF / kNT;
    const int64_t tok0 = token(a, b, h, t0);
    const uint4* dOg = reinterpret_cast<const uint4*>(p.dO);
    uint4 xo[PF];
    if (a.io_bf16) {
#pragma unroll
      for (int u = 0; u < PB; ++u) {
        const int e = tid + u * kNT, t = e / VB;
        xo[u] = dOg[(tok0 + (int64_t)(t < n ? t : 0) * a.H) * VB + e % VB];
      }
    } else {
#pragma unroll
      for (int u = 0; u < PF; ++u) {
        const int e = tid + u * kNT, t = e / VF;
        xo[u] = dOg[(tok0 + (int64_t)(t < n ? t : 0) * a.H) * VF + e % VF];
      }
    }
#pragma unroll
    for (int it = 0; it < PER4; ++it) {
      const int e = (tid + it * kNT) * 4, t = e / DV, j = e % DV;
      *reinterpret_cast<float4*>(&U[t * LDV + j]) = xu[it];
      *reinterpret_cast<float4*>(&dVt[t * LDV + j]) = xv[it];
    }
    if (a.io_bf16) {
#pragma unroll
      for (int u = 0; u < PB; ++u) {
        const int e = tid + u * kNT, t = e / VB, j = (e % VB) * 8;
        const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xo[u]);
        float f[8];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 y = __bfloat1622float2(x2[q]);
          f[2 * q] = t < n ? y.x : 0.f;
          f[2 * q + 1] = t < n ? y.y : 0.f;
        }
        *reinterpret_cast<float4*>(&dOs[t * LDV + j]) = make_float4(f[0], f[1], f[2], f[3]);
        *reinterpret_cast<float4*>(&dOs[t * LDV + j + 4]) = make_float4(f[4], f[5], f[6], f[7]);
      }
    } else {
#pragma unroll
      for (int u = 0; u < PF; ++u) {
        const int e = tid + u * kNT, t = e / VF, j = (e % VF) * 4;
        const float4 y = *reinterpret_cast<const float4*>(&xo[u]);
        *reinterpret_cast<float4*>(&dOs[t * LDV + j]) = t < n ? y : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    if (tid < kC) acc_a[tid] = acc_bk[tid] = acc_d[tid] = 0.f;
  }
  __syncthreads();
  // dv = beta^v dV~, and the beta^v gradient v dV~ (summed over channels for a per-token gate); eight
  // columns of a row per vector, every load of the thread issued before any is used
  {
    constexpr int V8 = DV / 8, P8 = kC * V8 / kNT;
    const int64_t tok0 = token(a, b, h, t0);
    float bv[P8][8], vv[P8][8];
#pragma unroll
    for (int u = 0; u < P8; ++u) {
      const int e = tid + u * kNT, t = e / V8, j = (e % V8) * 8;
      const int64_t r = tok0 + (int64_t)(t < n ? t : 0) * a.H;
      if (a.beta_v == DN_GATE_CHANNEL) {
        const float4 b0 = *reinterpret_cast<const float4*>(a.beta_v_p + r * DV + j);
        const float4 b1 = *reinterpret_cast<const float4*>(a.beta_v_p + r * DV + j + 4);
        bv[u][0] = b0.x, bv[u][1] = b0.y, bv[u][2] = b0.z, bv[u][3] = b0.w;
        bv[u][4] = b1.x, bv[u][5] = b1.y, bv[u][6] = b1.z, bv[u][7] = b1.w;
        if (a.io_bf16) {
          const uint4 x = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.v) + r * DV + j);
          const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&x);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 y = __bfloat1622float2(x2[q]);
            vv[u][2 * q] = y.x, vv[u][2 * q + 1] = y.y;
          }
        } else {
          const float4 v0 = *reinterpret_cast<const float4*>(static_cast<const float*>(a.v) + r * DV + j);
          const float4 v1 = *reinterpret_cast<const float4*>(static_cast<const float*>(a.v) + r * DV + j + 4);
          vv[u][0] = v0.x, vv[u][1] = v0.y, vv[u][2] = v0.z, vv[u][3] = v0.w;
          vv[u][4] = v1.x, vv[u][5] = v1.y, vv[u][6] = v1.z, vv[u][7] = v1.w;
        }
      } else {
        const float x = a.beta_v == DN_GATE_SCALAR ? a.beta_v_p[r] : 1.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) bv[u][q] = x, vv[u][q] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < P8; ++u) {
      const int e = tid + u * kNT, t = e / V8, j = (e % V8) * 8;
      if (t < n) {
        const int64_t r = tok0 + (int64_t)t * a.H;
        const float4 d0 = *reinterpret_cast<const float4*>(&dVt[t * LDV + j]);
        const float4 d1 = *reinterpret_cast<const float4*>(&dVt[t * LDV + j + 4]);
        const float dv8[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
        float g8[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) g8[q] = bv[u][q] * dv8[q];
        if (a.io_bf16) {
          uint4 o;
          __nv_bfloat162* o2 = reinterpret_cast<__nv_bfloat162*>(&o);
#pragma unroll
          for (int q = 0; q < 4; ++q) o2[q] = __floats2bfloat162_rn(g8[2 * q], g8[2 * q + 1]);
          *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.gv) + r * DV + j) = o;
        } else {
          float* o = static_cast<float*>(p.gv) + r * DV + j;
          *reinterpret_cast<float4*>(o) = make_float4(g8[0], g8[1], g8[2], g8[3]);
          *reinterpret_cast<float4*>(o + 4) = make_float4(g8[4], g8[5], g8[6], g8[7]);
        }
        if (a.beta_v == DN_GATE_CHANNEL) {  // (gate gradients need only fp32 alignment: scalar stores)
#pragma unroll
          for (int q = 0; q < 8; ++q) p.gbeta_v[r * DV + j + q] = vv[u][q] * dv8[q];
        }
      }
    }
  }
  if (a.beta_v == DN_GATE_SCALAR) {
    for (int t = warp; t < n; t += kNT / 32) {  // uniform per warp: every lane takes part in the shuffles
      const int64_t tok = token(a, b, h, t0 + t);
      float s = 0.f;
      for (int j = lane; j < DV; j += 32) s = fmaf(io_load(a.v, tok * DV + j, a.io_bf16), dVt[t * LDV + j], s);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) p.gbeta_v[tok] = s;
    }
  }
  {  // warps 0-3: dP = lower-incl(dO U^T); warps 4-7: dL = -strictly-lower(dV~ U^T); 32 x 32 tiles
    const int m0 = ((warp & 3) >> 1) * 32, n0 = (warp & 1) * 32;
    const float* const X[1] = {(warp < 4 ? dOs : dVt) + m0 * LDV};
    float acc[1][2][4][4] = {};
    warp_gemm_ldm<1, 2, 4, DV>(acc, X, LDV, U + n0 * LDV, LDV, lane);
    const int diag = a.pre_read ? 0 : 1;
    if (warp < 4)
      warp_epilogue(acc[0], [&](int m, int nn, float v) { dP[(m0 + m) * kLDC + n0 + nn] = n0 + nn < m0 + m + diag ? v : 0.f; },
                    lane);
    else
      warp_epilogue(acc[0], [&](int m, int nn, float v) { dL[(m0 + m) * kLDC + n0 + nn] = n0 + nn < m0 + m ? -v : 0.f; }, lane);
  }
  __syncthreads();

  const float* Smg = p.wSm + cb * DK * DV;
  const float* dXg = p.wdX + cb * DK * DV;
  const int m0 = (warp >> 1) * 16, n0 = (warp & 1) * 16;  // 16 x 16 tile of a 64 x 32 (token x channel) result
  constexpr int XN = DV / 4, NIX = XN / 8;                 // X (32 x DV, channel x column): 16 x XN warp tiles
  const int mx = (warp >> 2) * 16, nx = (warp & 3) * XN;
  for (int i0 = 0; i0 < DK; i0 += kDKS) {
    async_rows<kC, kDKS>(Eh, LDS, p.wEh + cb * kC * DK + i0, DK, tid);
    async_rows<kC, kDKS>(Qp, LDS, p.wQp + cb * kC * DK + i0, DK, tid);
    async_rows<kC, kDKS>(Kp, LDS, p.wKp + cb * kC * DK + i0, DK, tid);
    async_rows<kC, kDKS>(Wm, LDS, p.wWm + cb * kC * DK + i0, DK, tid);
    async_rows<kDKS, DV>(Sm, LDV, Smg + (int64_t)i0 * DV, DV, tid);
    async_rows<kDKS, DV>(dX, LDV, dXg + (int64_t)i0 * DV, DV, tid);
    tc::cp_async_commit();
    tc::cp_async_wait_all();
    __syncthreads();
    float aqk[2][1][2][4] = {}, aw1[1][1][2][4] = {}, ax[1][NIX][4] = {};
    float(&aq)[1][2][4] = aqk[0];
    float(&ak)[1][2][4] = aqk[1];
    float(&aw)[1][2][4] = aw1[0];
    {  // dO S_m^T and dV~ S_m^T in one pass over the shared S_m fragments
      const float* const X[2] = {dOs + m0 * LDV, dVt + m0 * LDV};
      warp_gemm_ldm<2, 1, 2, DV>(aqk, X, LDV, Sm + n0 * LDV, LDV, lane);
    }
#pragma unroll
    for (int ni = 0; ni < 2; ++ni)
#pragma unroll
      for (int q = 0; q < 4; ++q) ak[0][ni][q] = -ak[0][ni][q];
    // dQ+ = dO S_m^T + dP W-
    warp_gemm<1, 2, kC>(
        aq, [&](int m, int k) { return dP[(m0 + m) * kLDC + k]; }, [&](int k, int nn) { return Wm[k * LDS + n0 + nn]; },
        lane);
    // dK+ = -dV~ S_m^T + dL W-
    warp_gemm<1, 2, kC>(
        ak, [&](int m, int k) { return dL[(m0 + m) * kLDC + k]; }, [&](int k, int nn) { return Wm[k * LDS + n0 + nn]; },
        lane);
    // dW- = U dX^T + dP^T Q+ + dL^T K+
    {
      const float* const X[1] = {U + m0 * LDV};
      warp_gemm_ldm<1, 1, 2, DV>(aw1, X, LDV, dX + n0 * LDV, LDV, lane);
    }
    warp_gemm<1, 2, kC>(
        aw, [&](int m, int k) { return dP[k * kLDC + m0 + m]; }, [&](int k, int nn) { return Qp[k * LDS + n0 + nn]; },
        lane);
    warp_gemm<1, 2, kC>(
        aw, [&](int m, int k) { return dL[k * kLDC + m0 + m]; }, [&](int k, int nn) { return Kp[k * LDS + n0 + nn]; },
        lane);
    // X - S_m = W-^T U for these channels
    warp_gemm<1, NIX, kC>(
        ax, [&](int m, int k) { return Wm[k * LDS + mx + m]; }, [&](int k, int nn) { return U[k * LDV + nx + nn]; }, lane);
    {  // partial rowsum(dX (.) X) over this warp's columns
      const int g = lane >> 2, t4 = lane & 3;
      float s0 = 0.f, s1 = 0.f;
#pragma unroll
      for (int ni = 0; ni < NIX; ++ni) {
        const int j = nx + 8 * ni + 2 * t4;
        const int r0 = mx + g, r1 = mx + g + 8;
        s0 += dX[r0 * LDV + j] * (Sm[r0 * LDV + j] + ax[0][ni][0]) + dX[r0 * LDV + j + 1] * (Sm[r0 * LDV + j + 1] + ax[0][ni][1]);
        s1 += dX[r1 * LDV + j] * (Sm[r1 * LDV + j] + ax[0][ni][2]) + dX[r1 * LDV + j + 1] * (Sm[r1 * LDV + j + 1] + ax[0][ni][3]);
      }
      s0 += __shfl_xor_sync(0xffffffffu, s0, 1);
      s0 += __shfl_xor_sync(0xffffffffu, s0, 2);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 1);
      s1 += __shfl_xor_sync(0xffffffffu, s1, 2);
      if (t4 == 0) {
        red[(warp & 3) * kDKS + mx + g] = s0;
        red[(warp & 3) * kDKS + mx + g + 8] = s1;
      }
    }
    __syncthreads();  // every product has read Q+, K+, W- before they are overwritten below
    {
      // Per (token, channel) of this warp's tiles: dq, dk, the beta^k and d gradients, and dh. Each
      // thread then reads and writes only its own elements of hb, Qp, Kp, Wm.
      float gq[2][4], gk[2][4], lk[2][4], lb[2][4], ld[2][4], la[2][4];
      const int g = lane >> 2, t4 = lane & 3;
      {  // the inputs of this thread's elements, every load issued before any is used
        int tt[8], ci[8];
#pragma unroll
        for (int ni = 0; ni < 2; ++ni)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int t = m0 + g + (q >> 1) * 8;
            tt[4 * ni + q] = t < n ? t : 0;
            ci[4 * ni + q] = i0 + n0 + 8 * ni + 2 * t4 + (q & 1);
          }
        const int64_t tok0 = token(a, b, h, t0);
        io_load_n<8>(&lk[0][0], a.k, tok0, tt, a.H, ci, DK, a.io_bf16);
        gate_load_n<8>(&lb[0][0], a.beta_k_p, a.beta_k, tok0, tt, a.H, ci, DK);
        gate_load_n<8>(&ld[0][0], a.key_scale_p, a.key_scale, tok0, tt, a.H, ci, DK);
        if (a.pre_read) gate_load_n<8>(&la[0][0], a.alpha_p, a.alpha, tok0, tt, a.H, ci, DK);
#pragma unroll
        for (int ni = 0; ni < 2; ++ni)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            if (!a.pre_read) la[ni][q] = 1.f;
            if (m0 + g + (q >> 1) * 8 >= n) {
              lk[ni][q] = 0.f;
              lb[ni][q] = ld[ni][q] = la[ni][q] = 1.f;
            }
          }
      }
      auto elem = [&](int ni, int q, int m, int nn, float vq, float vk, float vw) {
        const int t = m0 + m, il = n0 + nn;
        const float eh = Eh[t * LDS + il];
        const float dw = vw / eh;
        const float kk = lk[ni][q], bk = lb[ni][q], dd = ld[ni][q];
        const float dk = vk * eh + bk * dd * dw;
        const float gbk = dd * kk * dw, gdd = bk * kk * dw;
        gq[ni][q] = vq * eh / la[ni][q];
        gk[ni][q] = dk;
        const float xq = Qp[t * LDS + il] * vq;
        Xq[t * LDS + il] = xq;
        const float dh = xq + Kp[t * LDS + il] * vk - Wm[t * LDS + il] * vw;
        Qp[t * LDS + il] = gbk;
        Kp[t * LDS + il] = gdd;
        Wm[t * LDS + il] = dh;
      };
#pragma unroll
      for (int ni = 0; ni < 2; ++ni) {
        elem(ni, 0, g, 8 * ni + 2 * t4, aq[0][ni][0], ak[0][ni][0], aw[0][ni][0]);
        elem(ni, 1, g, 8 * ni + 2 * t4 + 1, aq[0][ni][1], ak[0][ni][1], aw[0][ni][1]);
        elem(ni, 2, g + 8, 8 * ni + 2 * t4, aq[0][ni][2], ak[0][ni][2], aw[0][ni][2]);
        elem(ni, 3, g + 8, 8 * ni + 2 * t4 + 1, aq[0][ni][3], ak[0][ni][3], aw[0][ni][3]);
      }
#pragma unroll
      for (int ni = 0; ni < 2; ++ni)
#pragma unroll
        for (int q = 0; q < 4; q += 2) {  // elements q and q + 1: the same token, channels gi and gi + 1
          const int t = m0 + g + (q >> 1) * 8, gi = i0 + n0 + 8 * ni + 2 * t4;
          if (t < n) {
            const int64_t o = token(a, b, h, t0 + t) * DK + gi;
            if (a.io_bf16) {
              *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.gq) + o) =
                  __floats2bfloat162_rn(gq[ni][q], gq[ni][q + 1]);
              *reinterpret_cast<__nv_bfloat162*>(static_cast<__nv_bfloat16*>(p.gk) + o) =
                  __floats2bfloat162_rn(gk[ni][q], gk[ni][q + 1]);
            } else {
              *reinterpret_cast<float2*>(static_cast<float*>(p.gq) + o) = make_float2(gq[ni][q], gq[ni][q + 1]);
              *reinterpret_cast<float2*>(static_cast<float*>(p.gk) + o) = make_float2(gk[ni][q], gk[ni][q + 1]);
            }
            if (a.beta_k == DN_GATE_CHANNEL) {
              p.gbeta_k[o] = Qp[t * LDS + gi - i0];
              p.gbeta_k[o + 1] = Qp[t * LDS + gi + 1 - i0];
            }
            if (a.key_scale == DN_GATE_CHANNEL) {
              p.gkey_scale[o] = Kp[t * LDS + gi - i0];
              p.gkey_scale[o + 1] = Kp[t * LDS + gi + 1 - i0];
            }
          }
        }
    }
    __syncthreads();
    // d log alpha_s = sum_{t >= s} dh_t + rowsum(dX (.) X) (the last token's share), per channel: the
    // suffix sums in shared memory (a dependent chain over the tokens), then d alpha = d log alpha /
    // alpha for every (token, channel) of the slice at once
    {  // warp w sums tokens 8w .. 8w + 7 of channel (lane); the segments' totals go through S_m's
       // buffer, free until the next slice's loads
      static_assert(kNT == 8 * kDKS && kC == 64, "eight segments of eight tokens, one per warp");
      const int il = tid % kDKS, sg = tid / kDKS;
      float x[8], tot = 0.f;
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        x[q] = Wm[(8 * sg + q) * LDS + il];
        tot += x[q];
      }
      float* seg = Sm;
      seg[sg * kDKS + il] = tot;
      __syncthreads();
      float run = red[il] + red[kDKS + il] + red[2 * kDKS + il] + red[3 * kDKS + il];
      for (int s2 = sg + 1; s2 < 8; ++s2) run += seg[s2 * kDKS + il];
#pragma unroll
      for (int q = 7; q >= 0; --q) {
        const int t = 8 * sg + q;
        run += x[q];
        Wm[t * LDS + il] = a.pre_read ? run - Xq[t * LDS + il] : run;
      }
    }
    __syncthreads();
    if (a.alpha == DN_GATE_CHANNEL) {
      for (int e = tid; e < n * kDKS; e += kNT) {
        const int t = e / kDKS, il = e % kDKS;
        const int64_t tok = token(a, b, h, t0 + t);
        p.galpha[tok * DK + i0 + il] = Wm[t * LDS + il] / gate_load(a.alpha_p, a.alpha, tok, DK, i0 + il);
      }
    }
    {  // per-token sums over these channels, for gates of width 1: four threads per token
      static_assert(kNT == 4 * kC && kDKS % 4 == 0, "four threads per token");
      const int t = tid >> 2, part = tid & 3;
      float sa = 0.f, sb = 0.f, sd = 0.f;
#pragma unroll
      for (int q = 0; q < kDKS / 4; ++q) {
        const int il = 4 * q + part;
        sa += Wm[t * LDS + il];
        sb += Qp[t * LDS + il];
        sd += Kp[t * LDS + il];
      }
#pragma unroll
      for (int off = 1; off < 4; off <<= 1) {
        sa += __shfl_xor_sync(0xffffffffu, sa, off);
        sb += __shfl_xor_sync(0xffffffffu, sb, off);
        sd += __shfl_xor_sync(0xffffffffu, sd, off);
      }
      if (part == 0) {
        acc_a[t] += sa;
        acc_bk[t] += sb;
        acc_d[t] += sd;
      }
    }
    __syncthreads();
  }
  if (tid < n) {
    const int64_t tok = token(a, b, h, t0 + tid);
    if (a.alpha == DN_GATE_SCALAR) p.galpha[tok] = acc_a[tid] / a.alpha_p[tok];
    if (a.beta_k == DN_GATE_SCALAR) p.gbeta_k[tok] = acc_bk[tid];
    if (a.key_scale == DN_GATE_SCALAR) p.gkey_scale[tok] = acc_d[tid];
  }
}

// ------------------------------------------------------------------ forward outputs of the fp32 chunked forward
// O = Q+ S_m + P U for one chunk (all d_v columns), from the prep and state kernels' workspace; the
// chunks the state kernel evaluated exactly (marked) already have their o rows.
template <int DK, int DV, int C>
__global__ void __launch_bounds__(kNT) fwd_out_kernel(BwdArgs p) {
  extern __shared__ float4 smem4[];
  // warp w: rows 16 (w / CT) .. + 15, columns (w % CT) TW .. + TW
  constexpr int LDK = DK + 4, LDV = DV + 4, LDC = C + 4, RT = C / 16, CT = 8 / RT, TW = DV / CT, NI = TW / 8;
  static_assert(RT * CT == 8 && TW % 8 == 0, "warp tiles");
  float* Qp = reinterpret_cast<float*>(smem4);  // [C][LDK]
  float* Sm = Qp + C * LDK;                      // [DK][LDV]
  float* Pm = Sm + DK * LDV;                     // [C][LDC]
  float* U = Pm + C * LDC;                       // [C][LDV]
  const Args& a = p.f;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x % p.nc, bh = blockIdx.x / p.nc, b = bh / a.H, h = bh % a.H;
  const int t0 = c * C, n = min(C, a.T - t0);
  const int64_t cb = (int64_t)bh * p.nc + c;
  if (p.wFlag[cb]) return;
  async_rows<C, DK>(Qp, LDK, p.wQp + cb * C * DK, DK, tid);
  async_rows<DK, DV>(Sm, LDV, p.wSm + cb * DK * DV, DV, tid);
  async_rows<C, C>(Pm, LDC, p.wP + cb * C * C, C, tid);
  async_rows<C, DV>(U, LDV, p.wU + cb * C * DV, DV, tid);
  tc::cp_async_commit();
  tc::cp_async_wait_all();
  __syncthreads();
  const int m0 = (warp / CT) * 16, n0 = (warp % CT) * TW;
  float acc[1][NI][4] = {};
  warp_gemm<1, NI, DK>(
      acc, [&](int m, int k) { return Qp[(m0 + m) * LDK + k]; }, [&](int k, int nn) { return Sm[k * LDV + n0 + nn]; },
      lane);
  warp_gemm<1, NI, C>(
      acc, [&](int m, int k) { return Pm[(m0 + m) * LDC + k]; }, [&](int k, int nn) { return U[k * LDV + n0 + nn]; },
      lane);
  warp_epilogue(acc,
                [&](int m, int nn, float v) {
                  const int t = m0 + m;
                  if (t < n) io_store(a.o, token(a, b, h, t0 + t) * DV + n0 + nn, v, a.io_bf16);
                },
                lane);
}

// ------------------------------------------------------------------ host side
template <int DK, int C = kC>
constexpr size_t prep_smem() {
  return sizeof(float) * (3 * C * (DK + 4) + 768 + 2 * DK);
}
template <int DK, int DVS, int C = kC>
constexpr size_t state_smem() {
  return sizeof(float) * (DK * kLdsState<DVS> + C * (DK + 4) + C * (DK + 8) + C * (C + 4) + C * kLdsState<DVS> + 4 * DK);
}
template <int DK, int DVS>
constexpr size_t dstate_smem() {
  return sizeof(float) *
         (DK * kLdsDstate<DVS> + 2 * kC * (DK + 8) + kC * (DK + 4) + 2 * kC * kLDC + 3 * kC * kLdsDstate<DVS> + 4 * DK);
}
template <int DV>
constexpr size_t local_smem() {
  return sizeof(float) * (3 * kC * (DV + 4) + 2 * kC * kLDC + 2 * kDKS * (DV + 4) + 5 * kC * (kDKS + 8) + 4 * kDKS +
                          3 * kC);
}

template <int DK, int DV, int C>
constexpr size_t out_smem() {
  return sizeof(float) * (C * (DK + 4) + DK * (DV + 4) + C * (C + 4) + C * (DV + 4));
}

template <class K>
cudaError_t launch(K kernel, unsigned grid, size_t smem, cudaStream_t s, const BwdArgs& p) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  kernel<<<grid, kNT, smem, s>>>(p);
  return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_dims(const BwdArgs& p, cudaStream_t s) {
  constexpr int S1 = kDVS_STATE, S2 = kDVS_DSTATE < DV ? kDVS_DSTATE : DV;
  static_assert(DV % S1 == 0 && DV % S2 == 0, "d_v slices");
  static_assert(local_smem<DV>() <= 227 * 1024 && dstate_smem<DK, S2>() <= 227 * 1024, "shared memory");
  static_assert(state_smem<DK, S1>() <= 113 * 1024, "two state-chain CTAs per SM");
  const int64_t bh = (int64_t)p.f.B * p.f.H;
  const unsigned chunks = (unsigned)(bh * p.nc);
  cudaError_t e;
  if ((e = launch(bwd_prep_kernel<DK>, chunks, prep_smem<DK>(), s, p)) != cudaSuccess) return e;
  if ((e = launch(bwd_state_kernel<DK, DV, S1>, (unsigned)(bh * (DV / S1)), state_smem<DK, S1>(), s, p)) != cudaSuccess)
    return e;
  if ((e = launch(bwd_dstate_kernel<DK, DV, S2>, (unsigned)(bh * (DV / S2)), dstate_smem<DK, S2>(), s, p)) !=
      cudaSuccess)
    return e;
  return launch(bwd_local_kernel<DK, DV>, chunks, local_smem<DV>(), s, p);
}

template <int DK, int DV, int C>
cudaError_t launch_fwd32_dims(const BwdArgs& p, cudaStream_t s) {
  constexpr int S1 = kDVS_STATE;
  static_assert(out_smem<DK, DV, C>() <= 227 * 1024, "shared memory");
  const int64_t bh = (int64_t)p.f.B * p.f.H;
  const unsigned chunks = (unsigned)(bh * p.nc);
  cudaError_t e;
  if ((e = launch(bwd_prep_kernel<DK, C>, chunks, prep_smem<DK, C>(), s, p)) != cudaSuccess) return e;
  if ((e = launch(bwd_state_kernel<DK, DV, S1, C>, (unsigned)(bh * (DV / S1)), state_smem<DK, S1, C>(), s, p)) !=
      cudaSuccess)
    return e;
  return launch(fwd_out_kernel<DK, DV, C>, chunks, out_smem<DK, DV, C>(), s, p);
}

template <int C>
cudaError_t launch_fwd32_c(const BwdArgs& p, cudaStream_t s) {
  const Args& f = p.f;
  if (f.dk == 128 && f.dv == 128) return launch_fwd32_dims<128, 128, C>(p, s);
  if (f.dk == 128 && f.dv == 64) return launch_fwd32_dims<128, 64, C>(p, s);
  if (f.dk == 64 && f.dv == 128) return launch_fwd32_dims<64, 128, C>(p, s);
  return launch_fwd32_dims<64, 64, C>(p, s);
}

// The forward's workspace, per (b, h, chunk of C tokens): T and P (C x C), S_m (d_k x d_v), U
// (C x d_v), K+, Q+ and W- (C x d_k), e^r and lam (d_k), all fp32; then one int per chunk (the
// marks of the chunks evaluated token by token), the whole rounded up to 16 bytes.
int64_t fwd32_floats_per_chunk(int C, int dk, int dv) {
  return 2LL * C * C + (int64_t)dk * dv + (int64_t)C * dv + 3LL * C * dk + 2LL * dk;
}

void set_fwd_workspace(BwdArgs& p, const Args& f, float* ws) {
  const int C = f.chunk;
  p.nc = (f.T + C - 1) / C;
  const int64_t blocks = (int64_t)f.B * f.H * p.nc;
  p.wT = ws;
  p.wP = p.wT + blocks * C * C;
  p.wSm = p.wP + blocks * C * C;
  p.wU = p.wSm + blocks * f.dk * f.dv;
  p.wKp = p.wU + blocks * C * f.dv;
  p.wQp = p.wKp + blocks * C * f.dk;
  p.wWm = p.wQp + blocks * C * f.dk;
  p.wEr = p.wWm + blocks * C * f.dk;
  p.wLam = p.wEr + blocks * f.dk;
  p.wEh = nullptr;  // (the backward's e^h is not needed)
  p.wFlag = reinterpret_cast<int*>(p.wLam + blocks * f.dk);
}

// The backward's workspace layout, for its chunks of kC tokens.
void set_workspace(BwdArgs& p, const Args& f, float* ws) {
  p.nc = (f.T + kC - 1) / kC;
  const int64_t blocks = (int64_t)f.B * f.H * p.nc;
  p.wT = ws;
  p.wP = p.wT + blocks * kC * kC;
  p.wSm = p.wP + blocks * kC * kC;
  p.wU = p.wSm + blocks * f.dk * f.dv;
  p.wdX = p.wU + blocks * kC * f.dv;
  p.wdVt = p.wdX + blocks * f.dk * f.dv;
  p.wKp = p.wdVt + blocks * kC * f.dv;
  p.wQp = p.wKp + blocks * kC * f.dk;
  p.wWm = p.wQp + blocks * kC * f.dk;
  p.wEh = p.wWm + blocks * kC * f.dk;
  p.wEr = p.wEh + blocks * kC * f.dk;
  p.wLam = p.wEr + blocks * f.dk;
  p.wFlag = nullptr;
}

}  // namespace

bool chunk_fwd32_supported(const Args& a) {
  if (!((a.dk == 64 || a.dk == 128) && (a.dv == 64 || a.dv == 128) && a.T > 0)) return false;
  if (!(a.chunk == 16 || a.chunk == 32 || a.chunk == kC)) return false;
  if ((int64_t)a.B * a.H * ((a.T + a.chunk - 1) / a.chunk) >= ((int64_t)1 << 31)) return false;  // (one CTA per chunk)
  if (a.chunk == 16 || a.chunk == 32) return true;  // (the tcgen05 kernels' tiles are 64 tokens)
  return a.chunk == kC && !(a.io_bf16 && a.dk == 128);  // (bf16 with d_k = 128 has the tcgen05 kernels)
}

size_t chunk_fwd32_workspace_bytes(const Args& a) {
  const int64_t blocks = (int64_t)a.B * a.H * ((a.T + a.chunk - 1) / a.chunk);
  const size_t bytes = (size_t)(blocks * fwd32_floats_per_chunk(a.chunk, a.dk, a.dv)) * sizeof(float) +
                       (size_t)blocks * sizeof(int);
  return (bytes + 15) & ~size_t(15);
}

cudaError_t launch_chunk_fwd32(const Args& f, float* ws, cudaStream_t s) {
  BwdArgs p;
  memset(&p, 0, sizeof(p));
  p.f = f;
  set_fwd_workspace(p, f, ws);
  if (f.chunk == 16) return launch_fwd32_c<16>(p, s);
  if (f.chunk == 32) return launch_fwd32_c<32>(p, s);
  return launch_fwd32_c<kC>(p, s);
}

size_t chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
  const int64_t nc = (T + kC - 1) / kC;
  const int64_t per = 2LL * kC * kC + 2LL * dk * dv + 2LL * kC * dv + 4LL * kC * dk + 2LL * dk;
  return (size_t)((int64_t)B * H * nc * per) * sizeof(float);
}

cudaError_t launch_chunk_bwd(const Args& f, const void* dO, const float* dS_T, void* gq, void* gk, void* gv,
                             float* galpha, float* gbeta_k, float* gbeta_v, float* gkey_scale, float* gS0, float* ws,
                             cudaStream_t s) {
  BwdArgs p;
  p.f = f;
  p.dO = dO;
  p.dS_T = dS_T;
  p.gq = gq;
  p.gk = gk;
  p.gv = gv;
  p.galpha = galpha;
  p.gbeta_k = gbeta_k;
  p.gbeta_v = gbeta_v;
  p.gkey_scale = gkey_scale;
  p.gS0 = gS0;
  set_workspace(p, f, ws);
  if (f.dk == 128 && f.dv == 128) return launch_dims<128, 128>(p, s);
  if (f.dk == 128 && f.dv == 64) return launch_dims<128, 64>(p, s);
  if (f.dk == 64 && f.dv == 128) return launch_dims<64, 128>(p, s);
  return launch_dims<64, 64>(p, s);
}

}  // namespace dn
