// fp32 CUDA-core evaluation of a whole sequence, one token after another.
//
// Used for fp32 io, where the 1e-4 relative error budget rules out bf16 tensor
// core operands. The state lives in registers for the whole sequence; per
// token the kernel applies the decay, forms r = S_bar^T k and s = S_bar^T q with
// one block reduction, then u = beta^v (.) v - r, S += w u^T and o = s + u <w, q>
// (the same recurrence as the decode step; see dn_decode.cu for the sources).
//
// Layout: one CTA (256 threads) per (b, h) and 32-column slice of S. Thread
// (rg, c4) owns columns 4*c4..4*c4+3 of rows rg, rg+32, rg+64, rg+96. Token
// vectors are staged in shared memory 16 tokens at a time.
#include "dn_common.cuh"

namespace dn {
namespace {

constexpr int kThreads = 256;
constexpr int kCols = 32;
constexpr int kTT = 16;  // tokens staged per batch

template <int DK>
__global__ void __launch_bounds__(kThreads) seq_fwd_kernel(Args a) {
  constexpr int RPT = DK / 32;
  const int dv = a.dv, T = a.T, H = a.H;
  const int slices = dv / kCols;
  const int bh = blockIdx.x / slices;
  const int b = bh / H, h = bh % H;
  const int col0 = (blockIdx.x % slices) * kCols;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c4 = tid & 7, rg = tid >> 3;
  const bool pre = a.pre_read != 0;

  __shared__ float s_k[kTT][DK], s_q[kTT][DK], s_al[kTT][DK], s_w[kTT][DK];
  __shared__ float s_v[kTT][kCols];
  __shared__ float s_wq[kTT];
  __shared__ float s_red[8][kCols][2];
  __shared__ float s_u[kCols];

  float4 x[RPT];
  {
    const float* S0 = a.S0 ? a.S0 + (int64_t)bh * DK * dv + col0 + 4 * c4 : nullptr;
#pragma unroll
    for (int j = 0; j < RPT; ++j) {
      x[j] = S0 ? *reinterpret_cast<const float4*>(S0 + (int64_t)(rg + 32 * j) * dv)
                : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }

  for (int t0 = 0; t0 < T; t0 += kTT) {
    const int nt = min(kTT, T - t0);
    __syncthreads();  // previous batch fully consumed
    for (int e = tid; e < nt * DK; e += kThreads) {
      const int t = e / DK, i = e % DK;
      const int64_t tok = ((int64_t)b * T + t0 + t) * H + h;
      const float kk = io_load(a.k, tok * DK + i, a.io_bf16);
      s_k[t][i] = kk;
      s_q[t][i] = io_load(a.q, tok * DK + i, a.io_bf16);
      s_al[t][i] = gate_load(a.alpha_p, a.alpha, tok, DK, i);
      s_w[t][i] = gate_load(a.beta_k_p, a.beta_k, tok, DK, i) *
                  gate_load(a.key_scale_p, a.key_scale, tok, DK, i) * kk;
    }
    for (int e = tid; e < nt * kCols; e += kThreads) {
      const int t = e / kCols, j = e % kCols;
      const int64_t tok = ((int64_t)b * T + t0 + t) * H + h;
      s_v[t][j] = gate_load(a.beta_v_p, a.beta_v, tok, dv, col0 + j) *
                  io_load(a.v, tok * dv + col0 + j, a.io_bf16);
    }
    __syncthreads();
    for (int t = warp; t < nt; t += 8) {
      float p = 0.f;
      for (int i = lane; i < DK; i += 32) p = fmaf(s_w[t][i], s_q[t][i], p);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
      if (lane == 0) s_wq[t] = p;
    }
    __syncthreads();

    for (int t = 0; t < nt; ++t) {
      float r[4] = {0.f, 0.f, 0.f, 0.f}, s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        const int i = rg + 32 * j;
        const float al = s_al[t][i], kk = s_k[t][i], qq = s_q[t][i];
        // s = S^T q from the state before the decay (pre-update read-out) or after it
        const float sq = pre ? qq : qq * al;
        s[0] = fmaf(x[j].x, sq, s[0]);
        s[1] = fmaf(x[j].y, sq, s[1]);
        s[2] = fmaf(x[j].z, sq, s[2]);
        s[3] = fmaf(x[j].w, sq, s[3]);
        x[j].x *= al;
        x[j].y *= al;
        x[j].z *= al;
        x[j].w *= al;
        r[0] = fmaf(x[j].x, kk, r[0]);
        r[1] = fmaf(x[j].y, kk, r[1]);
        r[2] = fmaf(x[j].z, kk, r[2]);
        r[3] = fmaf(x[j].w, kk, r[3]);
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        r[c] += __shfl_xor_sync(0xffffffffu, r[c], 8);
        r[c] += __shfl_xor_sync(0xffffffffu, r[c], 16);
        s[c] += __shfl_xor_sync(0xffffffffu, s[c], 8);
        s[c] += __shfl_xor_sync(0xffffffffu, s[c], 16);
      }
      if ((lane & 24) == 0) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          s_red[warp][4 * c4 + c][0] = r[c];
          s_red[warp][4 * c4 + c][1] = s[c];
        }
      }
      __syncthreads();
      if (tid < kCols) {
        float rr = 0.f, ss = 0.f;
#pragma unroll
        for (int w8 = 0; w8 < 8; ++w8) {
          rr += s_red[w8][tid][0];
          ss += s_red[w8][tid][1];
        }
        const float u = s_v[t][tid] - rr;
        s_u[tid] = u;
        const int64_t tok = ((int64_t)b * T + t0 + t) * H + h;
        io_store(a.o, tok * dv + col0 + tid, pre ? ss : fmaf(u, s_wq[t], ss), a.io_bf16);
      }
      __syncthreads();
      const float u0 = s_u[4 * c4], u1 = s_u[4 * c4 + 1], u2 = s_u[4 * c4 + 2], u3 = s_u[4 * c4 + 3];
#pragma unroll
      for (int j = 0; j < RPT; ++j) {
        const float w = s_w[t][rg + 32 * j];
        x[j].x = fmaf(w, u0, x[j].x);
        x[j].y = fmaf(w, u1, x[j].y);
        x[j].z = fmaf(w, u2, x[j].z);
        x[j].w = fmaf(w, u3, x[j].w);
      }
    }
  }
  float* ST = a.S + (int64_t)bh * DK * dv + col0 + 4 * c4;
#pragma unroll
  for (int j = 0; j < RPT; ++j) *reinterpret_cast<float4*>(ST + (int64_t)(rg + 32 * j) * dv) = x[j];
}

}  // namespace

cudaError_t launch_seq_fwd(const Args& a, cudaStream_t s) {
  const int grid = a.B * a.H * (a.dv / kCols);
  if (a.dk == 128) {
    seq_fwd_kernel<128><<<grid, kThreads, 0, s>>>(a);
  } else {
    seq_fwd_kernel<64><<<grid, kThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace dn
