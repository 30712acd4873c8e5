// Backward of the small-state recurrence (d_k, d_v in {8, 16}: the delta-mem page's 8 x 8 memory,
// section 2.A), both read-outs: the gradients of sum <dO, o> + <dS_T, S_T> with respect to q, k, v,
// every gate and S0, by the chain rule through the per-token steps (the pages print no backward).
//
// One warp per (b, h); lane j < d_v owns column j of the state, as in the forward small-state kernel.
// The forward pass stores the state entering every token in the workspace ([T][d_k][d_v] per head,
// 256 bytes per token at 8 x 8); the reverse pass walks the tokens backwards with the adjoint dS in
// registers. Per token, with S_bar = Diag(alpha) S_prev, u = beta^v v - S_bar^T k, w = beta^k d k,
// S_t = S_bar + w u^T:
//   post read-out: dS += q dO^T, dq = S_t dO          pre read-out: dq = S_prev dO
//   dw = dS u,  du = dS^T w,  dk = beta^k d dw - S_bar du,  dv = beta^v du,  dbeta^v = v du
//   dbeta^k = d k dw,  dd = beta^k k dw,  dS_bar = dS - k du^T,  dalpha_i = <row i of dS_bar, row i of S_prev>
//   dS_prev = Diag(alpha) dS_bar  (+ q dO^T for the pre read-out)
// Everything indexed by the column j is lane-local; the sums over j (dq, dw, S_bar du, dalpha) are
// warp butterflies over the d_v lanes. fp32 throughout.
#include "dn_common.cuh"

namespace dn {
namespace {

constexpr int kWarps = 4;  // heads per CTA

template <int DK, int DV>
__global__ void __launch_bounds__(32 * kWarps)
    small_bwd_kernel(Args a, const void* dO, const float* dS_T, void* gq, void* gk, void* gv, float* galpha,
                     float* gbeta_k, float* gbeta_v, float* gkey_scale, float* gS0, float* ws) {
  static_assert(DV <= 16 && DK <= 16, "small states");
  const int lane = threadIdx.x & 31;
  const int bh = blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (bh >= a.B * a.H) return;  // whole warps only
  const int T = a.T, H = a.H, b = bh / H, h = bh % H;
  const bool act = lane < DV;
  const int j = act ? lane : 0;
  const bool pre = a.pre_read != 0;
  float* st = ws + (int64_t)bh * T * DK * DV;

  // forward: keep the state entering every token
  float S[DK];
#pragma unroll
  for (int i = 0; i < DK; ++i) S[i] = (act && a.S0) ? a.S0[((int64_t)bh * DK + i) * DV + j] : 0.f;
  for (int t = 0; t < T; ++t) {
    const int64_t tok = ((int64_t)b * T + t) * H + h;
    if (act) {
#pragma unroll
      for (int i = 0; i < DK; ++i) st[((int64_t)t * DK + i) * DV + j] = S[i];
    }
    float u = act ? gate_load(a.beta_v_p, a.beta_v, tok, DV, j) * io_load(a.v, tok * DV + j, a.io_bf16) : 0.f;
#pragma unroll
    for (int i = 0; i < DK; ++i) {
      S[i] *= gate_load(a.alpha_p, a.alpha, tok, DK, i);
      u = fmaf(-S[i], io_load(a.k, tok * DK + i, a.io_bf16), u);
    }
#pragma unroll
    for (int i = 0; i < DK; ++i) {
      const float w = gate_load(a.beta_k_p, a.beta_k, tok, DK, i) * gate_load(a.key_scale_p, a.key_scale, tok, DK, i) *
                      io_load(a.k, tok * DK + i, a.io_bf16);
      S[i] = fmaf(w, act ? u : 0.f, S[i]);
    }
  }

  // reverse
  float dS[DK];
#pragma unroll
  for (int i = 0; i < DK; ++i) dS[i] = (act && dS_T) ? dS_T[((int64_t)bh * DK + i) * DV + j] : 0.f;
  for (int t = T - 1; t >= 0; --t) {
    const int64_t tok = ((int64_t)b * T + t) * H + h;
    float kk[DK], qq[DK], al[DK], bk[DK], dd[DK], Sp[DK], Sb[DK];
#pragma unroll
    for (int i = 0; i < DK; ++i) {
      kk[i] = io_load(a.k, tok * DK + i, a.io_bf16);
      qq[i] = io_load(a.q, tok * DK + i, a.io_bf16);
      al[i] = gate_load(a.alpha_p, a.alpha, tok, DK, i);
      bk[i] = gate_load(a.beta_k_p, a.beta_k, tok, DK, i);
      dd[i] = gate_load(a.key_scale_p, a.key_scale, tok, DK, i);
      Sp[i] = act ? st[((int64_t)t * DK + i) * DV + j] : 0.f;
    }
    const float vj = act ? io_load(a.v, tok * DV + j, a.io_bf16) : 0.f;
    const float bvj = gate_load(a.beta_v_p, a.beta_v, tok, DV, j);
    const float dOj = act ? io_load(dO, tok * DV + j, a.io_bf16) : 0.f;
    float u = bvj * vj;
#pragma unroll
    for (int i = 0; i < DK; ++i) {
      Sb[i] = al[i] * Sp[i];
      u = fmaf(-Sb[i], kk[i], u);
    }
    if (!act) u = 0.f;
    // per-lane partials of the sums over the columns j
    float pq[DK], pw[DK], pk[DK], pa[DK];
    float du = 0.f;
#pragma unroll
    for (int i = 0; i < DK; ++i) {
      const float w = bk[i] * dd[i] * kk[i];
      const float St = fmaf(w, u, Sb[i]);
      if (!pre) dS[i] = fmaf(qq[i], dOj, dS[i]);
      pq[i] = (pre ? Sp[i] : St) * dOj;
      pw[i] = dS[i] * u;
      du = fmaf(dS[i], w, du);
    }
#pragma unroll
    for (int i = 0; i < DK; ++i) {
      pk[i] = Sb[i] * du;
      const float dsb = fmaf(-kk[i], du, dS[i]);
      pa[i] = dsb * Sp[i];
      dS[i] = al[i] * dsb;
      if (pre) dS[i] = fmaf(qq[i], dOj, dS[i]);
    }
    // butterflies over the d_v lanes (lanes >= d_v hold zeros and only pass values along)
#pragma unroll
    for (int o = DV / 2; o > 0; o >>= 1) {
#pragma unroll
      for (int i = 0; i < DK; ++i) {
        pq[i] += __shfl_xor_sync(0xffffffffu, pq[i], o);
        pw[i] += __shfl_xor_sync(0xffffffffu, pw[i], o);
        pk[i] += __shfl_xor_sync(0xffffffffu, pk[i], o);
        pa[i] += __shfl_xor_sync(0xffffffffu, pa[i], o);
      }
    }
    // per-channel outputs, written by lane 0
    if (lane == 0) {
      float sbk = 0.f, sdd = 0.f, sal = 0.f;
#pragma unroll
      for (int i = 0; i < DK; ++i) {
        const float dw = pw[i];
        io_store(gq, tok * DK + i, pq[i], a.io_bf16);
        io_store(gk, tok * DK + i, bk[i] * dd[i] * dw - pk[i], a.io_bf16);
        const float gb = dd[i] * kk[i] * dw, gd = bk[i] * kk[i] * dw;
        if (a.beta_k == DN_GATE_CHANNEL) gbeta_k[tok * DK + i] = gb;
        if (a.key_scale == DN_GATE_CHANNEL) gkey_scale[tok * DK + i] = gd;
        if (a.alpha == DN_GATE_CHANNEL) galpha[tok * DK + i] = pa[i];
        sbk += gb;
        sdd += gd;
        sal += pa[i];
      }
      if (a.beta_k == DN_GATE_SCALAR) gbeta_k[tok] = sbk;
      if (a.key_scale == DN_GATE_SCALAR) gkey_scale[tok] = sdd;
      if (a.alpha == DN_GATE_SCALAR) galpha[tok] = sal;
    }
    // per-column outputs
    float pv = vj * du;
    if (act) {
      io_store(gv, tok * DV + j, bvj * du, a.io_bf16);
      if (a.beta_v == DN_GATE_CHANNEL) gbeta_v[tok * DV + j] = pv;
    }
    if (a.beta_v == DN_GATE_SCALAR) {
#pragma unroll
      for (int o = DV / 2; o > 0; o >>= 1) pv += __shfl_xor_sync(0xffffffffu, pv, o);
      if (lane == 0) gbeta_v[tok] = pv;
    }
  }
  if (gS0 && act) {
#pragma unroll
    for (int i = 0; i < DK; ++i) gS0[((int64_t)bh * DK + i) * DV + j] = dS[i];
  }
}

template <int DK>
cudaError_t launch_dk(const Args& a, const void* dO, const float* dS_T, void* gq, void* gk, void* gv, float* galpha,
                      float* gbeta_k, float* gbeta_v, float* gkey_scale, float* gS0, float* ws, cudaStream_t s) {
  const unsigned grid = (unsigned)((a.B * a.H + kWarps - 1) / kWarps);
  if (a.dv == 8)
    small_bwd_kernel<DK, 8><<<grid, 32 * kWarps, 0, s>>>(a, dO, dS_T, gq, gk, gv, galpha, gbeta_k, gbeta_v, gkey_scale,
                                                         gS0, ws);
  else
    small_bwd_kernel<DK, 16><<<grid, 32 * kWarps, 0, s>>>(a, dO, dS_T, gq, gk, gv, galpha, gbeta_k, gbeta_v,
                                                          gkey_scale, gS0, ws);
  return cudaGetLastError();
}

}  // namespace

size_t small_bwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
  return (size_t)B * H * T * dk * dv * sizeof(float);
}

cudaError_t launch_small_bwd(const Args& a, const void* dO, const float* dS_T, void* gq, void* gk, void* gv,
                             float* galpha, float* gbeta_k, float* gbeta_v, float* gkey_scale, float* gS0, float* ws,
                             cudaStream_t s) {
  return a.dk == 8 ? launch_dk<8>(a, dO, dS_T, gq, gk, gv, galpha, gbeta_k, gbeta_v, gkey_scale, gS0, ws, s)
                   : launch_dk<16>(a, dO, dS_T, gq, gk, gv, galpha, gbeta_k, gbeta_v, gkey_scale, gS0, ws, s);
}

}  // namespace dn
