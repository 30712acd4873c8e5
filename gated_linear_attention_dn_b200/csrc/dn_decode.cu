// Single-token recurrent step, HBM-streaming.
//
// Per (b, h) the resident fp32 state S [d_k, d_v] is read once and written
// once; everything else (q, k, v, gates: a few hundred bytes) is noise. With
// alpha applied to the rows of S:
//   S_bar = Diag(alpha) S,  r = S_bar^T k,  s = S_bar^T q,  w = beta^k (.) d (.) k
//   u = beta^v (.) v - r,   S' = S_bar + w u^T,  o = S'^T q = s + u <w, q>
// (delta rule as an online-gradient step, OSDN page section 1; decay before the
// delta step, Sparse Delta Memory page "Gated Delta Updates"; channel decay and
// beta^k / beta^v, FG2-GDN page sections 1 and 2.B; write key d (.) k, OSDN page
// section 2.1). The read-out uses o = s + u <w, q> so that S' never has to be
// re-read.
//
// Layout: one CTA of 256 threads per (b, h) and 64-column slice of S. Thread
// (rg, c4) holds columns 4*c4 .. 4*c4+3 of rows rg, rg+16, rg+32, ... as float4
// registers, so each row slice of 256 bytes is read by 16 consecutive threads
// (fully coalesced 16-byte accesses), and all of a thread's loads are issued
// before any arithmetic to keep many bytes in flight per SM.
#include "dn_common.cuh"

namespace dn {
namespace {

constexpr int kThreads = 256;
constexpr int kCols = 64;  // columns of S per CTA

template <int DK>
__global__ void __launch_bounds__(kThreads) decode_kernel(Args a) {
  constexpr int RPT = DK / 16;  // rows per thread
  const int dv = a.dv;
  const int slices = dv / kCols;
  const int bh = blockIdx.x / slices;
  const int col0 = (blockIdx.x % slices) * kCols;
  const int tid = threadIdx.x;
  const int c4 = tid & 15;
  const bool pre = a.pre_read != 0;
  const int rg = tid >> 4;

  __shared__ float s_alpha[DK], s_k[DK], s_q[DK], s_w[DK];
  __shared__ float s_red[8][kCols][2];
  __shared__ float s_u[kCols];
  __shared__ float s_wq_part[DK / 32];

  float* Sbh = a.S + (int64_t)bh * DK * dv + col0 + 4 * c4;
  float4 x[RPT];
#pragma unroll
  for (int j = 0; j < RPT; ++j) x[j] = ld_stream_f4(Sbh + (int64_t)(rg + 16 * j) * dv);

  // per-head vectors (token index = bh because T == 1)
  if (tid < DK) {
    const int i = tid;
    const float kk = io_load(a.k, (int64_t)bh * DK + i, a.io_bf16);
    const float qq = io_load(a.q, (int64_t)bh * DK + i, a.io_bf16);
    const float al = gate_load(a.alpha_p, a.alpha, bh, DK, i);
    const float bk = gate_load(a.beta_k_p, a.beta_k, bh, DK, i);
    const float dd = gate_load(a.key_scale_p, a.key_scale, bh, DK, i);
    const float w = bk * dd * kk;
    s_alpha[i] = al;
    s_k[i] = kk;
    s_q[i] = qq;
    s_w[i] = w;
    float p = w * qq;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
    if ((i & 31) == 0) s_wq_part[i >> 5] = p;
  }
  __syncthreads();

  float r[4] = {0.f, 0.f, 0.f, 0.f}, s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < RPT; ++j) {
    const int i = rg + 16 * j;
    const float al = s_alpha[i], kk = s_k[i], qq = s_q[i];
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
  // reduce the two row groups that share a warp, then across the 8 warps
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    r[c] += __shfl_xor_sync(0xffffffffu, r[c], 16);
    s[c] += __shfl_xor_sync(0xffffffffu, s[c], 16);
  }
  const int warp = tid >> 5;
  if ((tid & 16) == 0) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      s_red[warp][4 * c4 + c][0] = r[c];
      s_red[warp][4 * c4 + c][1] = s[c];
    }
  }
  __syncthreads();
  if (tid < kCols) {
    const int j = tid;
    float rr = 0.f, ss = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < 8; ++w8) {
      rr += s_red[w8][j][0];
      ss += s_red[w8][j][1];
    }
    float wq = 0.f;
#pragma unroll
    for (int p = 0; p < DK / 32; ++p) wq += s_wq_part[p];
    const int col = col0 + j;
    const float vv = io_load(a.v, (int64_t)bh * dv + col, a.io_bf16);
    const float bv = gate_load(a.beta_v_p, a.beta_v, bh, dv, col);
    const float u = bv * vv - rr;
    s_u[j] = u;
    io_store(a.o, (int64_t)bh * dv + col, pre ? ss : fmaf(u, wq, ss), a.io_bf16);
  }
  __syncthreads();
  const float u0 = s_u[4 * c4 + 0], u1 = s_u[4 * c4 + 1], u2 = s_u[4 * c4 + 2], u3 = s_u[4 * c4 + 3];
#pragma unroll
  for (int j = 0; j < RPT; ++j) {
    const float w = s_w[rg + 16 * j];
    float4 y;
    y.x = fmaf(w, u0, x[j].x);
    y.y = fmaf(w, u1, x[j].y);
    y.z = fmaf(w, u2, x[j].z);
    y.w = fmaf(w, u3, x[j].w);
    st_stream_f4(Sbh + (int64_t)(rg + 16 * j) * dv, y);
  }
}

}  // namespace

cudaError_t launch_decode(const Args& a, cudaStream_t s) {
  const int grid = a.B * a.H * (a.dv / kCols);
  if (a.dk == 128) {
    decode_kernel<128><<<grid, kThreads, 0, s>>>(a);
  } else {
    decode_kernel<64><<<grid, kThreads, 0, s>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace dn
