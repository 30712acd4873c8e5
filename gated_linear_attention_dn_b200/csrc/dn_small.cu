// Small states (d_k, d_v in {8, 16}): the delta-mem page keeps an 8 x 8 memory per head (section
// 2.A). The recurrence is the same as everywhere else (see dn_decode.cu for its terms); at this
// size one warp per (b, h) runs it token by token with lane j owning column j of S (d_k values
// in registers), so the residual u_j = beta^v_j v_j - sum_i S_bar_ij k_i, the read-out
// s_j = sum_i S_ij q_i and the update S_ij += w_i u_j are all lane-local: no reduction crosses
// lanes. The token vectors (q, k, alpha, w = beta^k d k, beta^v v) are staged in shared memory
// 16 tokens at a time by the whole warp. fp32 arithmetic; serves dn_chunk_fwd (any T) and
// dn_decode_step (T = 1, S updated in place), with either read-out.
#include "dn_common.cuh"

namespace dn {
namespace {

constexpr int kTT = 16;  // tokens staged per batch

template <int DK, int DV>
__global__ void __launch_bounds__(32) small_state_kernel(Args a) {
  static_assert(DK <= 32 && DV <= 32, "small states");
  __shared__ float s_k[kTT][DK], s_q[kTT][DK], s_al[kTT][DK], s_w[kTT][DK], s_v[kTT][DV];
  const int T = a.T, H = a.H, lane = threadIdx.x;
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  const bool pre = a.pre_read != 0;
  float S[DK];
#pragma unroll
  for (int i = 0; i < DK; ++i)
    S[i] = (a.S0 && lane < DV) ? a.S0[((int64_t)bh * DK + i) * DV + lane] : 0.f;

  for (int t0 = 0; t0 < T; t0 += kTT) {
    const int nt = min(kTT, T - t0);
    __syncwarp();  // the previous batch is consumed
    for (int e = lane; e < nt * DK; e += 32) {
      const int t = e / DK, i = e % DK;
      const int64_t tok = ((int64_t)b * T + t0 + t) * H + h;
      const float kk = io_load(a.k, tok * DK + i, a.io_bf16);
      s_k[t][i] = kk;
      s_q[t][i] = io_load(a.q, tok * DK + i, a.io_bf16);
      s_al[t][i] = gate_load(a.alpha_p, a.alpha, tok, DK, i);
      s_w[t][i] = gate_load(a.beta_k_p, a.beta_k, tok, DK, i) * gate_load(a.key_scale_p, a.key_scale, tok, DK, i) * kk;
    }
    for (int e = lane; e < nt * DV; e += 32) {
      const int t = e / DV, j = e % DV;
      const int64_t tok = ((int64_t)b * T + t0 + t) * H + h;
      s_v[t][j] = gate_load(a.beta_v_p, a.beta_v, tok, DV, j) * io_load(a.v, tok * DV + j, a.io_bf16);
    }
    __syncwarp();
    if (lane < DV) {
      for (int t = 0; t < nt; ++t) {
        float s = 0.f, r = 0.f, wq = 0.f;
#pragma unroll
        for (int i = 0; i < DK; ++i) {
          const float al = s_al[t][i], qi = s_q[t][i];
          s = fmaf(S[i], pre ? qi : qi * al, s);  // read-out before or after the decay
          S[i] *= al;
          r = fmaf(S[i], s_k[t][i], r);
          wq = fmaf(s_w[t][i], qi, wq);
        }
        const float u = s_v[t][lane] - r;
#pragma unroll
        for (int i = 0; i < DK; ++i) S[i] = fmaf(s_w[t][i], u, S[i]);
        const int64_t tok = ((int64_t)b * T + t0 + t) * H + h;
        io_store(a.o, tok * DV + lane, pre ? s : fmaf(u, wq, s), a.io_bf16);
      }
    }
  }
  if (lane < DV) {
#pragma unroll
    for (int i = 0; i < DK; ++i) a.S[((int64_t)bh * DK + i) * DV + lane] = S[i];
  }
}

template <int DK>
cudaError_t launch_dk(const Args& a, cudaStream_t s) {
  const unsigned grid = (unsigned)(a.B * a.H);
  if (a.dv == 8) {
    small_state_kernel<DK, 8><<<grid, 32, 0, s>>>(a);
  } else {
    small_state_kernel<DK, 16><<<grid, 32, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace

bool small_state_supported(const Args& a) { return (a.dk == 8 || a.dk == 16) && (a.dv == 8 || a.dv == 16); }

cudaError_t launch_small_state(const Args& a, cudaStream_t s) {
  return a.dk == 8 ? launch_dk<8>(a, s) : launch_dk<16>(a, s);
}

}  // namespace dn
