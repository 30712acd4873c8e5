// Memory Caching read-out (Memory Caching page, sections 2 and 3): a token t of segment
// j = t / L adds to its output the gated read of the cached memories of the earlier segments,
//   o_t += sum_{s < j} g_{t,s} M_s^T q_t,
// with g = 1 for the residual memory (section 3, item 1) or caller-given gates for the gated
// residual memory (item 2). The memories are the segment-final states M_s [d_k, d_v] fp32 that
// dn_chunk_fwd returns as S_T when the sequence is viewed as B * N sequences of L tokens.
//
// One CTA (256 threads) per (b, h) and tile of 64 tokens: the tile's q rows sit in shared memory
// as fp32; each memory M_s streams through shared memory in slabs of 16 rows; thread (ty, tx)
// accumulates 4 tokens x (d_v / 16) columns in registers and weights each memory's contribution
// by its tokens' gates (0 for a memory of the token's own or a later segment). For the residual
// memory on a tile inside one segment, the memories are summed while they are loaded and one
// product serves them all. fp32 throughout.
#include "dn_common.cuh"

namespace dn {
namespace {

constexpr int kTok = 64;   // tokens per CTA
constexpr int kSlab = 16;  // rows of a memory per shared-memory slab

template <int DK, int DV, bool BF16>
__global__ void __launch_bounds__(256) mc_readout_kernel(const void* q, const float* M, const float* gates,
                                                         void* o, int T, int H, int L, int N) {
  constexpr int CPT = DV / 16;  // columns per thread
  __shared__ __align__(16) float s_q[kTok][DK + 4];
  __shared__ __align__(16) float s_m[kSlab][DV];
  __shared__ float s_g[kTok];
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int tiles = (T + kTok - 1) / kTok;
  const int bh = blockIdx.x / tiles, tile = blockIdx.x % tiles;
  const int b = bh / H, h = bh % H;
  const int t0 = tile * kTok, nt = min(kTok, T - t0);
  const int jmax = (t0 + nt - 1) / L;  // memories this tile reads: s < jmax
  if (jmax == 0) return;               // the whole tile is in the first segment

  for (int e = tid; e < kTok * DK; e += 256) {
    const int t = e / DK, c = e % DK;
    float x = 0.f;
    if (t < nt) {
      const int64_t i = (((int64_t)b * T + t0 + t) * H + h) * DK + c;
      x = BF16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q)[i]) : reinterpret_cast<const float*>(q)[i];
    }
    s_q[t][c] = x;
  }
  float acc[4][CPT];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < CPT; ++c) acc[r][c] = 0.f;

  // residual memory over a tile that lies in one segment: every token reads the same memories,
  // so their sum is formed while loading and one product serves them all
  const bool summed = gates == nullptr && t0 / L == jmax;
  const int passes = summed ? 1 : jmax;
  for (int s = 0; s < passes; ++s) {
    __syncthreads();  // every thread is done with the previous memory's gates
    if (tid < kTok) {
      const int t = t0 + tid;
      const bool reads = tid < nt && (summed || s < t / L);
      s_g[tid] = reads ? (gates ? gates[(((int64_t)b * T + t) * H + h) * N + s] : 1.f) : 0.f;
    }
    const float* Ms = M + (((int64_t)b * N + s) * H + h) * DK * DV;
    const int64_t mstride = (int64_t)H * DK * DV;  // from memory s to s + 1
    float tmp[4][CPT];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < CPT; ++c) tmp[r][c] = 0.f;
    for (int k0 = 0; k0 < DK; k0 += kSlab) {
      __syncthreads();  // the previous slab (and, at k0 = 0, the q tile and gates) is settled
      for (int e = tid; e < kSlab * DV / 4; e += 256) {
        float4 m4 = reinterpret_cast<const float4*>(Ms + (int64_t)k0 * DV)[e];
        if (summed) {
          for (int s2 = 1; s2 < jmax; ++s2) {
            const float4 y = reinterpret_cast<const float4*>(Ms + s2 * mstride + (int64_t)k0 * DV)[e];
            m4.x += y.x, m4.y += y.y, m4.z += y.z, m4.w += y.w;
          }
        }
        reinterpret_cast<float4*>(&s_m[0][0])[e] = m4;
      }
      __syncthreads();
#pragma unroll 4
      for (int kk = 0; kk < kSlab; ++kk) {
        float mv[CPT];
#pragma unroll
        for (int c = 0; c < CPT; c += 4) {
          const float4 m4 = *reinterpret_cast<const float4*>(&s_m[kk][tx * CPT + c]);
          mv[c] = m4.x, mv[c + 1] = m4.y, mv[c + 2] = m4.z, mv[c + 3] = m4.w;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float qv = s_q[4 * ty + r][k0 + kk];
#pragma unroll
          for (int c = 0; c < CPT; ++c) tmp[r][c] = fmaf(qv, mv[c], tmp[r][c]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const float g = s_g[4 * ty + r];
#pragma unroll
      for (int c = 0; c < CPT; ++c) acc[r][c] = fmaf(g, tmp[r][c], acc[r][c]);
    }
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int t = 4 * ty + r;
    if (t >= nt) continue;
    const int64_t base = (((int64_t)b * T + t0 + t) * H + h) * DV + tx * CPT;
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
      if (BF16) {
        __nv_bfloat16* p = reinterpret_cast<__nv_bfloat16*>(o) + base + c;
        *p = __float2bfloat16_rn(__bfloat162float(*p) + acc[r][c]);
      } else {
        float* p = reinterpret_cast<float*>(o) + base + c;
        *p += acc[r][c];
      }
    }
  }
}

template <int DK, int DV>
cudaError_t launch_dims(const void* q, const float* M, const float* gates, void* o, int B, int T, int H, int L,
                        int bf16, cudaStream_t s) {
  const int N = (T + L - 1) / L;
  const int64_t grid = (int64_t)B * H * ((T + kTok - 1) / kTok);
  if (bf16)
    mc_readout_kernel<DK, DV, true><<<(unsigned)grid, 256, 0, s>>>(q, M, gates, o, T, H, L, N);
  else
    mc_readout_kernel<DK, DV, false><<<(unsigned)grid, 256, 0, s>>>(q, M, gates, o, T, H, L, N);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_mc_readout(const void* q, const float* M, const float* gates, void* o, int B, int T, int H,
                              int dk, int dv, int L, int bf16, cudaStream_t s) {
  if ((int64_t)B * H * T == 0 || T <= L) return cudaSuccess;  // nothing reads a cached memory
  if (dk == 128 && dv == 128) return launch_dims<128, 128>(q, M, gates, o, B, T, H, L, bf16, s);
  if (dk == 128 && dv == 64) return launch_dims<128, 64>(q, M, gates, o, B, T, H, L, bf16, s);
  if (dk == 64 && dv == 128) return launch_dims<64, 128>(q, M, gates, o, B, T, H, L, bf16, s);
  return launch_dims<64, 64>(q, M, gates, o, B, T, H, L, bf16, s);
}

}  // namespace dn
