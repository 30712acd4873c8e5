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
// product serves them all. fp32 throughout (the kernel for fp32 io, and for bf16 q or o not 16-byte
// aligned).
//
// For bf16 io the read-out runs on the tensor cores (mc_readout_tc_kernel): one CTA of 256 threads
// per (b, h) and tile of 128 tokens; the q tile arrives by TMA; each memory (or, for the residual
// memory on a tile inside one segment, the sum of the memories it reads) is split into bf16 hi + lo
// MN-major operand tiles, so that a product carries about 16 bits of the fp32 memory; tcgen05
// accumulates q M_hi + q M_lo (one M 128 x N d_v x K d_k pass each) into tensor memory; with gates,
// or on a tile that straddles a segment boundary, the rows of q are scaled by each memory's gates
// (0 for a memory the token does not read) and split hi + lo too (hi M_hi + hi M_lo + lo M_hi). The
// accumulated rows are added to o at the end. Every mbarrier wait is bounded.
#include "dn_common.cuh"
#include "dn_tc_ptx.cuh"

namespace dn {
namespace {

using namespace tc;

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

// ------------------------------------------------------------------ tensor-core read-out (bf16 io)
constexpr int kTcTok = 128;                        // tokens per CTA (the MMA's M)
constexpr uint64_t kMcDrainNs = 2000000000ull;     // bound of the drain waits after a failure

__device__ __forceinline__ uint8_t* mc_align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

template <int DK, int DV, bool MASKED>
struct McLayout {
  static constexpr int QT = 0;                                     // q tile [128][DK] bf16 (TMA), K-major
  static constexpr int AH = QT + kTcTok * DK * 2;                  // masked: rows of q scaled by g, hi
  static constexpr int AL = AH + (MASKED ? kTcTok * DK * 2 : 0);   // masked: lo
  static constexpr int BH = AL + (MASKED ? kTcTok * DK * 2 : 0);   // memory hi [DK][DV], MN-major
  static constexpr int BL = BH + DK * DV * 2;                      // memory lo
  static constexpr int TOTAL = BL + DK * DV * 2;
};

template <int DK, int DV, bool MASKED>
__global__ void __launch_bounds__(256) mc_readout_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const float* M,
                                                            const float* gates, __nv_bfloat16* o, int T, int H,
                                                            int L, int N, int* status, uint64_t wait_ns) {
  using Ly = McLayout<DK, DV, MASKED>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = mc_align1024(smem_raw);
  __shared__ __align__(8) uint64_t bar_q, bar_mma;
  __shared__ uint32_t s_tmem;
  __shared__ float s_g[kTcTok];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q4 = warp & 3, ch = warp >> 2;
  const int tiles = (T + kTcTok - 1) / kTcTok;
  const int bh = blockIdx.x / tiles, tile = blockIdx.x % tiles, b = bh / H, h = bh % H;
  const int t0 = tile * kTcTok, nt = min(kTcTok, T - t0);
  const int jmax = (t0 + nt - 1) / L;  // memories this tile reads: s < jmax
  if (jmax == 0) return;               // the whole tile is in the first segment
  // without masking, every tile lies inside one segment (the launch checks L % 128 == 0 and no gates)
  const int passes = MASKED ? jmax : 1;
  const int64_t mstride = (int64_t)H * DK * DV;  // from memory s to s + 1
  const float* Mb = M + ((int64_t)b * N * H + h) * DK * DV;

  if (tid == 0) {
    mbar_init(&bar_q, 1);
    mbar_init(&bar_mma, 1);
    fence_mbar_init();
    mbar_expect_tx(&bar_q, (uint32_t)kTcTok * DK * 2);
#pragma unroll
    for (int x = 0; x < DK / 64; ++x)
#pragma unroll
      for (int r = 0; r < 2; ++r)
        tma_load_4d(sm + Ly::QT + x * kTcTok * 128 + r * 64 * 128, &tm_q, &bar_q, 64 * x, h, t0 + 64 * r, b);
  }
  if (warp == 0) tmem_alloc(&s_tmem, DV);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t id = idesc_bf16(128, DV, 0, 1);
  bool ok = true, issued = false, q_seen = false;
  for (int s = 0; s < passes && ok; ++s) {
    // the memory (or the sum of memories 0 .. jmax - 1) as bf16 hi + lo tiles, 16-byte chunks of
    // 8 columns: consecutive threads take consecutive chunks of a row; every load of a memory is in
    // flight before any of it is used
    {
      constexpr int PER = DK * DV / 8 / 256;  // chunks per thread
      static_assert(PER * 256 * 8 == DK * DV, "work split");
      float4 m0[PER], m1[PER];
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int e = tid + 256 * i, k = e / (DV / 8), x8 = e % (DV / 8);
        const float* src = Mb + (int64_t)s * mstride + (int64_t)k * DV + 8 * x8;
        m0[i] = *reinterpret_cast<const float4*>(src);
        m1[i] = *reinterpret_cast<const float4*>(src + 4);
      }
      if (!MASKED) {
        for (int s2 = 1; s2 < jmax; ++s2) {
          float4 y0[PER], y1[PER];
#pragma unroll
          for (int i = 0; i < PER; ++i) {
            const int e = tid + 256 * i, k = e / (DV / 8), x8 = e % (DV / 8);
            const float* src = Mb + s2 * mstride + (int64_t)k * DV + 8 * x8;
            y0[i] = *reinterpret_cast<const float4*>(src);
            y1[i] = *reinterpret_cast<const float4*>(src + 4);
          }
#pragma unroll
          for (int i = 0; i < PER; ++i) {
            m0[i].x += y0[i].x, m0[i].y += y0[i].y, m0[i].z += y0[i].z, m0[i].w += y0[i].w;
            m1[i].x += y1[i].x, m1[i].y += y1[i].y, m1[i].z += y1[i].z, m1[i].w += y1[i].w;
          }
        }
      }
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int e = tid + 256 * i, k = e / (DV / 8), x8 = e % (DV / 8);
        uint4 hi, lo;
        split_bf16(m0[i].x, m0[i].y, hi.x, lo.x);
        split_bf16(m0[i].z, m0[i].w, hi.y, lo.y);
        split_bf16(m1[i].x, m1[i].y, hi.z, lo.z);
        split_bf16(m1[i].z, m1[i].w, hi.w, lo.w);
        const uint32_t off = canon_chunk(k, x8, DK);
        *reinterpret_cast<uint4*>(sm + Ly::BH + off) = hi;
        *reinterpret_cast<uint4*>(sm + Ly::BL + off) = lo;
      }
    }
    if (MASKED) {
      // this memory's gate of every token of the tile (0 when the token does not read it)
      if (tid < kTcTok) {
        const int t = t0 + tid;
        const bool reads = tid < nt && s < t / L;
        s_g[tid] = reads ? (gates ? gates[(((int64_t)b * T + t) * H + h) * N + s] : 1.f) : 0.f;
      }
      if (!q_seen) {  // the q tile is read below
        ok = mbar_wait_bounded(&bar_q, 0, wait_ns);
        q_seen = true;
      }
      __syncthreads();
      if (ok) {
        // rows of q scaled by their gates, hi + lo
        for (int e = tid; e < kTcTok * DK / 8; e += 256) {
          const int t = e / (DK / 8), x8 = e % (DK / 8);
          const uint32_t off = canon_chunk(t, x8, kTcTok);
          const uint4 qv = *reinterpret_cast<const uint4*>(sm + Ly::QT + off);
          const float g = s_g[t];
          const float2 q0 = unpack_bf16(qv.x), q1 = unpack_bf16(qv.y), q2 = unpack_bf16(qv.z), q3 = unpack_bf16(qv.w);
          uint4 hi, lo;
          split_bf16(g * q0.x, g * q0.y, hi.x, lo.x);
          split_bf16(g * q1.x, g * q1.y, hi.y, lo.y);
          split_bf16(g * q2.x, g * q2.y, hi.z, lo.z);
          split_bf16(g * q3.x, g * q3.y, hi.w, lo.w);
          *reinterpret_cast<uint4*>(sm + Ly::AH + off) = hi;
          *reinterpret_cast<uint4*>(sm + Ly::AL + off) = lo;
        }
      }
    }
    fence_proxy_async();
    tc_fence_before();
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    tc_fence_after();
    // the products of this pass (thread 0)
    if (tid == 0) {
      if (!MASKED && !q_seen) {
        ok = mbar_wait_bounded(&bar_q, 0, wait_ns);
        q_seen = true;
      }
      if (ok) {
        tc_fence_after();
        const uint32_t a_hi = smem_u32(sm + (MASKED ? Ly::AH : Ly::QT)), a_lo = smem_u32(sm + Ly::AL);
        const uint32_t b_hi = smem_u32(sm + Ly::BH), b_lo = smem_u32(sm + Ly::BL);
#pragma unroll
        for (int kk = 0; kk < DK; kk += 16) {
          const uint32_t ao = (kk >> 6) * (kTcTok * 128) + (kk & 63) * 2;
          const uint64_t bh_ = sdesc(b_hi + kk * 128, DK * 128, 1024), bl_ = sdesc(b_lo + kk * 128, DK * 128, 1024);
          mma_bf16(tmem, sdesc(a_hi + ao, 16, 1024), bh_, id, (s > 0 || kk > 0) ? 1 : 0);
          mma_bf16(tmem, sdesc(a_hi + ao, 16, 1024), bl_, id, 1);
          if (MASKED) mma_bf16(tmem, sdesc(a_lo + ao, 16, 1024), bh_, id, 1);
        }
        mma_commit(&bar_mma);
        issued = true;
      }
    }
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    // the products are done before the tiles are rewritten (next pass) or the sums read (below)
    ok = mbar_wait_bounded(&bar_mma, s & 1, wait_ns);
    if (__syncthreads_or(!ok)) {
      ok = false;
      break;
    }
    tc_fence_after();
  }
  if (ok) {
    // o rows += the accumulated read: warp (q4, ch) takes rows 32 q4 .. +31 and columns ch DV / 2 ..
    const int t = 32 * q4 + lane;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
#pragma unroll
    for (int cb = 0; cb < DV / 64; ++cb) {
      const int col = ch * (DV / 2) + 32 * cb;
      float x[32];
      tmem_ld32(tmem + lane_base + col, x);
      if (t < nt) {
        uint4* p = reinterpret_cast<uint4*>(o + (((int64_t)b * T + t0 + t) * H + h) * DV + col);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const uint4 v = p[q8];
          const float2 v0 = unpack_bf16(v.x), v1 = unpack_bf16(v.y), v2 = unpack_bf16(v.z), v3 = unpack_bf16(v.w);
          const float* y = x + 8 * q8;
          p[q8] = make_uint4(pack_bf16(v0.x + y[0], v0.y + y[1]), pack_bf16(v1.x + y[2], v1.y + y[3]),
                             pack_bf16(v2.x + y[4], v2.y + y[5]), pack_bf16(v3.x + y[6], v3.y + y[7]));
        }
      }
    }
  } else if (tid == 0) {
    // a wait gave up: let what was issued finish (bounded), then report
    if (!q_seen) mbar_wait_bounded(&bar_q, 0, kMcDrainNs);
    if (issued) {
      mma_commit(&bar_mma);
      mbar_wait_bounded(&bar_mma, 0, kMcDrainNs);
      mbar_wait_bounded(&bar_mma, 1, kMcDrainNs);
    }
    atomicExch(status, kDevTimeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, DV);
}

template <int DK, int DV>
cudaError_t launch_tc_dims(const CUtensorMap& mq, const float* M, const float* gates, void* o, int B, int T, int H,
                           int L, int* status, uint64_t wait_ns, cudaStream_t s) {
  const int N = (T + L - 1) / L;
  const int64_t grid = (int64_t)B * H * ((T + kTcTok - 1) / kTcTok);
  auto* ob = static_cast<__nv_bfloat16*>(o);
  if (gates || L % kTcTok != 0) {
    using Ly = McLayout<DK, DV, true>;
    const int smem = Ly::TOTAL + 1024;
    cudaError_t e = cudaFuncSetAttribute(mc_readout_tc_kernel<DK, DV, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    mc_readout_tc_kernel<DK, DV, true><<<(unsigned)grid, 256, smem, s>>>(mq, M, gates, ob, T, H, L, N, status, wait_ns);
  } else {
    using Ly = McLayout<DK, DV, false>;
    const int smem = Ly::TOTAL + 1024;
    cudaError_t e = cudaFuncSetAttribute(mc_readout_tc_kernel<DK, DV, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    mc_readout_tc_kernel<DK, DV, false><<<(unsigned)grid, 256, smem, s>>>(mq, M, gates, ob, T, H, L, N, status,
                                                                          wait_ns);
  }
  return cudaGetLastError();
}

template <int DK, int DV>
cudaError_t launch_dims(const void* q, const float* M, const float* gates, void* o, int B, int T, int H, int L,
                        int bf16, int* status, uint64_t wait_ns, cudaStream_t s) {
  CUtensorMap mq;
  // (the tensor-core kernel reads q by TMA and o with 16-byte accesses)
  if (bf16 && ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(o)) & 15) == 0 &&
      make_bthd_map(&mq, q, DK, H, T, B, 64))
    return launch_tc_dims<DK, DV>(mq, M, gates, o, B, T, H, L, status, wait_ns, s);
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
                              int dk, int dv, int L, int bf16, int* status, uint64_t wait_ns, cudaStream_t s) {
  if ((int64_t)B * H * T == 0 || T <= L) return cudaSuccess;  // nothing reads a cached memory
  if (dk == 128 && dv == 128) return launch_dims<128, 128>(q, M, gates, o, B, T, H, L, bf16, status, wait_ns, s);
  if (dk == 128 && dv == 64) return launch_dims<128, 64>(q, M, gates, o, B, T, H, L, bf16, status, wait_ns, s);
  if (dk == 64 && dv == 128) return launch_dims<64, 128>(q, M, gates, o, B, T, H, L, bf16, status, wait_ns, s);
  return launch_dims<64, 64>(q, M, gates, o, B, T, H, L, bf16, status, wait_ns, s);
}

}  // namespace dn
