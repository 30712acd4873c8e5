// Tensor-core chunked prefill (bf16 io, d_k = 128, d_v in {64, 128}) for sm_100a.
//
// One CTA (256 threads) owns one (b, h) sequence and walks its chunks of C = 64
// tokens in order, keeping the fp32 state in tensor memory. Per chunk, with the
// decay referenced to the chunk midpoint m (after token 31), so that every
// decay factor spans at most half a chunk:
//
//   r_t = gamma_t / gamma_m  (per key channel; products of alpha, no exp/log)
//   K+ = k (.) r,  Q+ = q (.) r,  W- = beta^k (.) d (.) k / r,  V~ = beta^v (.) v
//   A  = K+ W-^T (strictly lower part), P = Q+ W-^T (lower incl. diagonal)
//   T  = (I + A)^{-1}                              (UT transform, fp32, CUDA cores)
//   Wk = T K+,  U0 = T V~                          (tensor cores)
//   S_m = Diag(gamma_m) S                          (state decayed to the midpoint)
//   U  = U0 - Wk S_m,  O = Q+ S_m + P U            (tensor cores + CUDA cores)
//   S' = Diag(gamma_C / gamma_m) (S_m + W-^T U)    (tensor cores, fp32 accumulate)
//
// This is the chunk-parallel (WY / UT transform) evaluation that the FG2-GDN page
// says the DPLR update keeps (sections 2.A and 3 item 2) and whose block Gram
// matrix and intra-block scores take the preconditioned key under OSDN (OSDN
// page, section 2.1); the algebra is derived from the recurrence in dn.h.
//
// Two gate classes share the kernel:
//  * per-token gates only (GDN: scalar alpha, beta^k, beta^v, d): every decay and
//    write factor is a scalar per token, so they move onto the 64x64 and 64xN
//    matrices (A_ti = (k_t.k_i) beta_i r_t / r_i, T K+ = (T Diag(r)) K,
//    W-^T U = K^T (Diag(beta / r) U), O_t = r_t (Q S_m + P_raw U')_t) and the raw
//    TMA tiles of q, k, v feed the tensor cores directly, with no elementwise pass;
//  * any per-channel gate (KDA decay, FG2-GDN+ vector beta, OSDN d): the CUDA
//    cores build K+, Q+, W- (hi/lo) and V~ (hi/lo) tiles per chunk, with all gate
//    loads of a chunk in flight at once.
//
// Precision plan (bf16 operands, fp32 accumulation everywhere): the state update
// W-^T U is the product whose rounding reaches S_T directly, so its operands are
// split hi + lo in bf16 (raw k is exact in bf16, so the per-token path splits
// only U); V~ is split the same way when beta^v is a vector. All other operands
// are single bf16.
//
// Shared-memory operand tiles use the 128-byte-swizzled canonical layout (see
// canon()); q/k/v tiles arrive by TMA (4-D tensor maps over [B, T, H, d], boxes of
// 64 channels x 64 tokens, zero fill past the end of the sequence).
//
// Tensor memory (512 columns): S_acc [0, NV) | D1 [NV, 2NV) | U0 [2NV, 3NV) | scratch (Gram, Wk).
// Every wait on an mbarrier is bounded in time; on expiry the CTA sets the status
// word, drains what it issued (again bounded), frees its tensor memory and exits.
#include <cudaTypedefs.h>

#include "dn_common.cuh"
#include "dn_tc_ptx.cuh"

namespace dn {
namespace {

using namespace tc;

constexpr int C = 64;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s per wait, far above any legitimate wait

template <int DK, int NV>
struct Layout {
  static constexpr int STK = 0;                       // raw k  [C][DK]   (TMA)
  static constexpr int STQ = STK + C * DK * 2;        // raw q  [C][DK]   (TMA); per-token path: T~ tile
  static constexpr int STV = STQ + C * DK * 2;        // raw v  [C][NV]   (TMA), V~ hi after prep
  static constexpr int VLO = STV + C * NV * 2;        // V~ lo  [C][NV]
  static constexpr int KQ = VLO + C * NV * 2;         // [K+ ; Q+] then [Wk ; Q+]   [128][DK]
  static constexpr int WHI = KQ + 128 * DK * 2;       // W- hi  [C][DK]
  static constexpr int WLO = WHI + C * DK * 2;        // W- lo  [C][DK]
  static constexpr int TP = WLO + C * DK * 2;         // [T ; P]  [128][C]
  static constexpr int UHI = TP + 128 * C * 2;        // U hi   [C][NV]
  static constexpr int ULO = UHI + C * NV * 2;        // U lo   [C][NV]
  static constexpr int SM = ULO + C * NV * 2;         // S_m bf16 [DK][NV]
  static constexpr int END = SM + DK * NV * 2;
  // fp32 scratch of the 64x64 inverse (L and T): aliases the U tiles when they are large enough
  static constexpr int INV = (2 * C * NV * 2 >= 2 * C * C * 4) ? UHI : END;
  static constexpr int TOTAL = (INV + 2 * C * C * 4 > END) ? INV + 2 * C * C * 4 : END;
  static constexpr int TM_S = 0, TM_D1 = NV, TM_U0 = 2 * NV, TM_SCR = 3 * NV;
  static_assert(TM_SCR + (DK > 64 ? DK : 64) <= (int)kTmemCols, "tensor memory budget");
};

// Index into a 64x64 fp32 array: rows of 64, columns XOR-permuted in groups of 4
// by (row mod 8), so float4 accesses stay aligned and column walks by
// consecutive rows spread over the banks.
__device__ __forceinline__ int xi(int r, int c) { return (r << 6) | (c ^ ((r & 7) << 2)); }

__device__ __forceinline__ float4 f4(float x) { return make_float4(x, x, x, x); }
__device__ __forceinline__ float4 mul4(float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); }
__device__ __forceinline__ float4 rcp4(float4 a) {
  return make_float4(__fdividef(1.f, a.x), __fdividef(1.f, a.y), __fdividef(1.f, a.z), __fdividef(1.f, a.w));
}

// gate values of four consecutive channels (mode ONE -> 1, SCALAR -> broadcast)
__device__ __forceinline__ float4 gate4(const float* g, int mode, int64_t tok, int width, int ch) {
  if (mode == DN_GATE_ONE) return f4(1.f);
  if (mode == DN_GATE_SCALAR) return f4(g[tok]);
  return *reinterpret_cast<const float4*>(g + tok * width + ch);
}

// Gate values of 8 tokens (rows tok0 + i * tstride, i < 8) for 4 consecutive channels, with every
// load issued before any is used: the mode branch is uniform and outside the loads, and tokens past
// the end (i >= nvalid) re-read row tok0 + (nvalid - 1) * tstride, or row tok0 when nvalid == 0
// (the caller points tok0 at a real token then); their values are replaced by `dflt`.
__device__ __forceinline__ void gate4x8(float4* out, const float* g, int mode, int64_t tok0, int64_t tstride,
                                        int width, int ch, int nvalid, float dflt) {
  if (mode == DN_GATE_CHANNEL) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ic = i < nvalid ? i : max(nvalid - 1, 0);
      out[i] = __ldg(reinterpret_cast<const float4*>(g + (tok0 + ic * tstride) * width + ch));
    }
  } else if (mode == DN_GATE_SCALAR) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ic = i < nvalid ? i : max(nvalid - 1, 0);
      out[i] = f4(__ldg(g + tok0 + ic * tstride));
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) out[i] = f4(1.f);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (i >= nvalid) out[i] = f4(dflt);
}

__device__ __forceinline__ float4 lds4(const float* p, int idx) { return *reinterpret_cast<const float4*>(p + idx); }
__device__ __forceinline__ void sts4(float* p, int idx, float4 v) { *reinterpret_cast<float4*>(p + idx) = v; }

__device__ __forceinline__ uint2 pack4(float4 v) { return make_uint2(pack_bf16(v.x, v.y), pack_bf16(v.z, v.w)); }
__device__ __forceinline__ float4 unpack4(uint2 u) {
  const float2 a = unpack_bf16(u.x), b = unpack_bf16(u.y);
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ void split4(float4 v, uint2& hi, uint2& lo) {
  split_bf16(v.x, v.y, hi.x, lo.x);
  split_bf16(v.z, v.w, hi.y, lo.y);
}

// Warp-level tensor-core product (mma.sync, TF32 inputs, fp32 accumulation), used only for the
// small block products inside the 64x64 triangular inverse; T is rounded to bf16 afterwards, so
// TF32 (10-bit mantissa) operands here add an error well below that rounding. Fragment layouts
// of m16n8k8 row.col (g = lane / 4, t = lane % 4): A 16x8: (g, t) (g+8, t) (g, t+4) (g+8, t+4);
// B 8x8: (t, g) (t+4, g); C 16x8: (g, 2t) (g, 2t+1) (g+8, 2t) (g+8, 2t+1).
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ void mma_tf32(float* d, const uint32_t* a, const uint32_t* b) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// d[16x8] += X[16 x K] * Y[K x 8] for one warp; X(i, k), Y(k, n) fetch elements.
template <int K, class FX, class FY>
__device__ __forceinline__ void warp_mm(float* d, FX X, FY Y, int lane) {
  const int g = lane >> 2, t = lane & 3;
#pragma unroll
  for (int k = 0; k < K; k += 8) {
    const uint32_t av[4] = {to_tf32(X(g, k + t)), to_tf32(X(g + 8, k + t)), to_tf32(X(g, k + t + 4)),
                            to_tf32(X(g + 8, k + t + 4))};
    const uint32_t bv[2] = {to_tf32(Y(k + t, g)), to_tf32(Y(k + t + 4, g))};
    mma_tf32(d, av, bv);
  }
}

// writes the 16x8 accumulator fragment as column pairs through W(i, n, v_n, v_n+1)
template <class FW>
__device__ __forceinline__ void warp_store2(const float* d, FW W, int lane) {
  const int g = lane >> 2, t = lane & 3;
  W(g, 2 * t, d[0], d[1]);
  W(g + 8, 2 * t, d[2], d[3]);
}

// writes the 16x8 accumulator fragment through W(i, n, value)
template <class FW>
__device__ __forceinline__ void warp_store(const float* d, FW W, int lane) {
  const int g = lane >> 2, t = lane & 3;
  W(g, 2 * t, d[0]);
  W(g, 2 * t + 1, d[1]);
  W(g + 8, 2 * t, d[2]);
  W(g + 8, 2 * t + 1, d[3]);
}

// T = (I + L)^{-1} for the 64x64 strictly lower L in sL (zeros on and above the diagonal).
// Blocking by doubling: the eight 8x8 diagonal blocks by forward substitution (one column per
// thread, chains of at most seven steps); then three merge levels with warp mma.sync, each using
// [[A, 0], [C, B]]^{-1} = [[A^-1, 0], [-B^-1 C A^-1, B^-1]]:
//   8 -> 16 (warps 0..3), 16 -> 32 (warps 0..1), 32 -> 64 (all 8 warps).
// fp32 blocks that later levels read are kept in sT; every element of the lower triangle is also
// written as bf16 straight into rows 0..63 of the 128-row tile tp (scaled by column factor
// cs_c[i] when SC) and, when SC, T Diag(cs_v) into tile tt. Elements above the 8x8 block diagonal
// are not written (their zeros are set once by the caller). scr: 2048 floats of scratch.
// Not inlined: it gets its own register budget. All 256 threads call it.
template <bool SC>
__device__ __noinline__ void unit_lower_inverse(const float* sL, float* sT, float* scr, uint8_t* tp, uint8_t* tt,
                                                const float* cs_c, const float* cs_v, int tid) {
  const int warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  auto emit1 = [&](int t, int i, float v) {
    const uint32_t off = canon(t, i, 128);
    *reinterpret_cast<__nv_bfloat16*>(tp + off) = __float2bfloat16_rn(SC ? v * cs_c[i] : v);
    if (SC) *reinterpret_cast<__nv_bfloat16*>(tt + off) = __float2bfloat16_rn(v * cs_v[i]);
  };
  auto emit2 = [&](int t, int i, float v0, float v1) {  // columns i, i + 1 (i even)
    const uint32_t off = canon(t, i, 128);
    *reinterpret_cast<uint32_t*>(tp + off) = pack_bf16(SC ? v0 * cs_c[i] : v0, SC ? v1 * cs_c[i + 1] : v1);
    if (SC) *reinterpret_cast<uint32_t*>(tt + off) = pack_bf16(v0 * cs_v[i], v1 * cs_v[i + 1]);
  };
  if (tid < 64) {
    const int base = 8 * (tid >> 3), j = tid & 7;
    float x[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      float s0 = (r == j) ? 1.f : 0.f, s1 = 0.f;
#pragma unroll
      for (int i = 0; i < r; ++i) {
        const float l = sL[xi(base + r, base + i)];
        if (i & 1)
          s1 = fmaf(-l, x[i], s1);
        else
          s0 = fmaf(-l, x[i], s0);
      }
      x[r] = s0 + s1;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      sT[xi(base + r, base + j)] = x[r];
      emit1(base + r, base + j, x[r]);
    }
  } else {
    // zero, inside each 32x32 diagonal block, the 8x8 and 16x16 blocks above the diagonal that the
    // merge levels read: rows 16p..+8 x cols 16p+8..+8 (p < 4); rows 32q..+16 x cols 32q+16..+16 (q < 2)
    for (int e = tid - 64; e < 768; e += 192) {
      if (e < 256) {
        const int p = e >> 6, r = (e >> 3) & 7, cc = e & 7;
        sT[xi(16 * p + r, 16 * p + 8 + cc)] = 0.f;
      } else {
        const int e2 = e - 256, q = e2 >> 8, r = (e2 >> 4) & 15, cc = e2 & 15;
        sT[xi(32 * q + r, 32 * q + 16 + cc)] = 0.f;
      }
    }
  }
  __syncthreads();
  // 8 -> 16: T_ba = -T_bb (L_ba T_aa) in each 16x16 diagonal block (rows 8..15 of the 16-row
  // mma operands repeat rows 0..7 and their results are ignored)
  if (warp < 4) {
    const int a0 = 16 * warp, b0 = a0 + 8;
    float* Y = scr + warp * 96;  // 8 x 12 (padded)
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    warp_mm<8>(d, [&](int i, int k) { return sL[xi(b0 + (i & 7), a0 + k)]; },
               [&](int k, int n) { return sT[xi(a0 + k, a0 + n)]; }, lane);
    Y[g * 12 + 2 * t4] = d[0];
    Y[g * 12 + 2 * t4 + 1] = d[1];
    __syncwarp();
    float e[4] = {0.f, 0.f, 0.f, 0.f};
    warp_mm<8>(e, [&](int i, int k) { return sT[xi(b0 + (i & 7), b0 + k)]; },
               [&](int k, int n) { return Y[k * 12 + n]; }, lane);
    sT[xi(b0 + g, a0 + 2 * t4)] = -e[0];
    sT[xi(b0 + g, a0 + 2 * t4 + 1)] = -e[1];
    emit2(b0 + g, a0 + 2 * t4, -e[0], -e[1]);
  }
  __syncthreads();
  // 16 -> 32: T_{i,i-1} = -T_ii (L_{i,i-1} T_{i-1,i-1}) for (i, i-1) = (1, 0), (3, 2); warp w < 4
  // owns pair w / 2 and the 8-column tile w % 2 (a column tile of the result needs only the
  // same column tile of L T)
  if (warp < 4) {
    const int bi = 1 + 2 * (warp >> 1), bk = bi - 1, nt = warp & 1;
    float* Y = scr + 1152 + warp * 192;  // 16 x 12 (padded) dense scratch of this warp
    {
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      warp_mm<16>(d, [&](int i, int k) { return sL[xi(16 * bi + i, 16 * bk + k)]; },
                  [&](int k, int n) { return sT[xi(16 * bk + k, 16 * bk + 8 * nt + n)]; }, lane);
      warp_store(d, [&](int i, int n, float v) { Y[i * 12 + n] = v; }, lane);
    }
    __syncwarp();
    {
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      warp_mm<16>(d, [&](int i, int k) { return sT[xi(16 * bi + i, 16 * bi + k)]; },
                  [&](int k, int n) { return Y[k * 12 + n]; }, lane);
      warp_store2(d, [&](int i, int n, float v0, float v1) {
        sT[xi(16 * bi + i, 16 * bk + 8 * nt + n)] = -v0;
        sT[xi(16 * bi + i, 16 * bk + 8 * nt + n + 1)] = -v1;
        emit2(16 * bi + i, 16 * bk + 8 * nt + n, -v0, -v1);
      }, lane);
    }
  }
  __syncthreads();
  // 32 -> 64: X = L21 T1, then T21 = -T2 X; warp w owns rows 16 (w / 4) .. +16, columns 8 (w % 4) .. +8
  float* X = scr;  // 32 x 36 (padded) dense
  const int mt = warp >> 2, nt = warp & 3;
  {
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    warp_mm<32>(d, [&](int i, int k) { return sL[xi(32 + 16 * mt + i, k)]; },
                [&](int k, int n) { return sT[xi(k, 8 * nt + n)]; }, lane);
    warp_store(d, [&](int i, int n, float v) { X[(16 * mt + i) * 36 + 8 * nt + n] = v; }, lane);
  }
  __syncthreads();
  {
    float d[4] = {0.f, 0.f, 0.f, 0.f};
    warp_mm<32>(d, [&](int i, int k) { return sT[xi(32 + 16 * mt + i, 32 + k)]; },
                [&](int k, int n) { return X[k * 36 + 8 * nt + n]; }, lane);
    warp_store2(d, [&](int i, int n, float v0, float v1) { emit2(32 + 16 * mt + i, 8 * nt + n, -v0, -v1); },
                lane);
  }
  __syncthreads();
}

template <int DK, int NV, bool SC>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Args a) {
  using Ly = Layout<DK, NV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_qk, bar_k, bar_v, bar_mma, bar_gram;
  __shared__ int s_gram_ready;  // per-token path: the next chunk's Gram MMA was issued early
  __shared__ uint32_t s_tmem;
  __shared__ __align__(16) float s_lam[2][DK];   // gamma_C / gamma_m per key channel (per-channel path)
  __shared__ __align__(16) float s_gm[DK];       // gamma_m per key channel
  __shared__ __align__(16) float s_grp[8][DK];   // per-8-token decay products (per-channel path)
  __shared__ __align__(16) float s_Y[2048];
  // per-token path, by chunk parity: r_t, 1/r_t, beta^k d, beta^v; gamma_C / gamma_m; gamma_m
  __shared__ float s_r[2][C], s_ri[2][C], s_ws[2][C], s_bv[2][C];
  __shared__ float s_lam1[2], s_gm1[2];
  __shared__ float s_nx[2][4][C];  // per-token path: gates of the next chunk (alpha, beta^k, d, beta^v)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, ch = warp >> 2;
  const int T = a.T, H = a.H, dv = a.dv;
  // one CTA per (b, h) and slice of NV value columns (columns of the state evolve independently)
  const int nslices = dv / NV;
  const int bh = blockIdx.x / nslices, b = bh / H, h = bh % H;
  const int col0 = (blockIdx.x % nslices) * NV;
  const int nchunks = (T + C - 1) / C;

  if (tid == 0) {
    mbar_init(&bar_qk, 1);
    mbar_init(&bar_k, 1);
    mbar_init(&bar_v, 1);
    mbar_init(&bar_mma, 1);
    mbar_init(&bar_gram, 1);
    s_gram_ready = 0;
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&s_tmem, kTmemCols);
  // rows 0..63 of the [T; P] tile (and of the T~ tile): the 8x8 blocks above the block diagonal
  // of T are zero and nothing else writes them; set them once
  for (int e = tid; e < 64 * 8; e += kThreads) {
    const int t = e >> 3, x8 = e & 7;
    if (x8 > (t >> 3)) {
      *reinterpret_cast<uint4*>(sm + Ly::TP + canon_chunk(t, x8, 128)) = make_uint4(0, 0, 0, 0);
      if (SC) *reinterpret_cast<uint4*>(sm + Ly::STQ + canon_chunk(t, x8, 128)) = make_uint4(0, 0, 0, 0);
    }
  }
  if (SC) {
    // rows 64..127 of the T~ tile are never meaningful; keep them finite
    for (int i = tid; i < 64 * 128 / 16; i += kThreads)
      reinterpret_cast<uint4*>(sm + Ly::STQ + 64 * 128)[i] = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t lane_base = (uint32_t)(32 * q4) << 16;

  // Operand buffers. Per-channel path: raw k, q staging (STK, STQ) feeds the prep,
  // which writes [K+; Q+] into KQ. Per-token path: the raw [K; Q] tile (Gram operand,
  // later [Wk; Q]) is double-buffered in KQ and in the W- region it does not use, so
  // the next chunk's tile loads during this chunk; a separate raw k tile (STK) serves
  // the state update at the end of the chunk and reloads after it.
  auto kq_buf = [&](int c) -> uint8_t* { return (SC && (c & 1)) ? sm + Ly::WHI : sm + Ly::KQ; };
  auto issue_qk = [&](int c) {
    mbar_expect_tx(&bar_qk, 2u * C * DK * 2);
#pragma unroll
    for (int x = 0; x < DK / 64; ++x) {
      if (SC) {
        uint8_t* kq = kq_buf(c);
        tma_load_4d(kq + x * 128 * 128, &tm_k, &bar_qk, 64 * x, h, c * C, b);
        tma_load_4d(kq + x * 128 * 128 + 64 * 128, &tm_q, &bar_qk, 64 * x, h, c * C, b);
      } else {
        tma_load_4d(sm + Ly::STK + x * C * 128, &tm_k, &bar_qk, 64 * x, h, c * C, b);
        tma_load_4d(sm + Ly::STQ + x * C * 128, &tm_q, &bar_qk, 64 * x, h, c * C, b);
      }
    }
  };
  auto issue_k = [&](int c) {  // per-token path only
    mbar_expect_tx(&bar_k, (uint32_t)C * DK * 2);
#pragma unroll
    for (int x = 0; x < DK / 64; ++x) tma_load_4d(sm + Ly::STK + x * C * 128, &tm_k, &bar_k, 64 * x, h, c * C, b);
  };
  auto issue_v = [&](int c) {
    mbar_expect_tx(&bar_v, (uint32_t)C * NV * 2);
#pragma unroll
    for (int x = 0; x < NV / 64; ++x)
      tma_load_4d(sm + Ly::STV + x * C * 128, &tm_v, &bar_v, col0 + 64 * x, h, c * C, b);
  };

  uint32_t ph_qk = 0, ph_k = 0, ph_v = 0, ph_mma = 0, ph_gram = 0;
  bool qk_pending = false, k_pending = false, v_pending = false, mma_pending = false, gram_pending = false;
  bool failed = false;
  if (tid == 0 && nchunks > 0) {
    issue_qk(0);
    if (SC) issue_k(0);
    issue_v(0);
  }
  if (nchunks > 0) qk_pending = v_pending = true;
  if (SC && nchunks > 0) k_pending = true;

  const uint32_t id_gram = idesc_bf16(128, 64, 0, 0);
  const uint32_t id_wk = idesc_bf16(128, DK, 0, 1);
  const uint32_t id_nv = idesc_bf16(128, NV, 0, 1);
  const uint32_t id_state = idesc_bf16(128, NV, 1, 1);
  const bool bv_split = !SC && a.beta_v != DN_GATE_ONE;
  float* sL = reinterpret_cast<float*>(sm + Ly::INV);
  float* sT = sL + C * C;

  // per-token path: thread j < 64 copies token j's gates of the next chunk into shared memory
  // one chunk ahead with cp.async (absent gates and tokens past the end are written directly)
  auto prefetch_token_gates = [&](int cn, int j) {
    const int t0n = cn * C;
    float* dst = &s_nx[cn & 1][0][j];
    const float* src[4] = {a.alpha_p, a.beta_k_p, a.key_scale_p, a.beta_v_p};
    const int mode[4] = {a.alpha, a.beta_k, a.key_scale, a.beta_v};
    const bool valid = j < T - t0n;
    const int64_t tok = ((int64_t)b * T + t0n + j) * H + h;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      if (valid && mode[g] == DN_GATE_SCALAR)
        cp_async_4(dst + g * C, src[g] + tok);
      else
        dst[g * C] = valid ? 1.f : (g == 0 ? 1.f : 0.f);
    }
    cp_async_commit();
  };
  // per-token path, threads 0..63 (token j): decay factors of chunk cn from its prefetched gates;
  // warp 1 (tokens 32..63) forms r_j = prod_{s=32..j} alpha_s by an inclusive product scan,
  // warp 0 (tokens 0..31) forms 1/r_j = prod_{s=j+1..31} alpha_s by an exclusive suffix scan
  auto token_prep = [&](int cn, int j, bool upper) {
    const int par = cn & 1;
    cp_async_wait_all();
    const float al = s_nx[par][0][j], ws = s_nx[par][1][j] * s_nx[par][2][j], bv = s_nx[par][3][j];
    if (cn + 1 < nchunks) prefetch_token_gates(cn + 1, j);
    float p = al;
    if (upper) {
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, p, off);
        if (lane >= off) p *= y;
      }
      s_r[par][j] = p;
      s_ri[par][j] = __fdividef(1.f, p);
      if (lane == 31) s_lam1[par] = p;
    } else {
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_down_sync(0xffffffffu, p, off);
        if (lane + off < 32) p *= y;
      }
      const float nxt = __shfl_down_sync(0xffffffffu, p, 1);
      const float ri = lane == 31 ? 1.f : nxt;
      s_ri[par][j] = ri;
      s_r[par][j] = __fdividef(1.f, ri);
      if (lane == 0) s_gm1[par] = p;
    }
    s_ws[par][j] = ws;
    s_bv[par][j] = bv;
  };
  if (SC && tid < 64 && nchunks > 0) {
    prefetch_token_gates(0, tid);
    token_prep(0, tid, warp == 1);
  }

  // S_m = Diag(lambda_prev * gamma_m) S for rows 32 q4 .. +32, columns of half ch: the state in
  // chunk c's frame, in TMEM (fp32) and as the bf16 operand tile
  auto state_to_frame = [&](int c) {
    const int cur = c & 1, prev = cur ^ 1;
    const int k = 32 * q4 + lane;
    const float mu = SC ? ((c == 0) ? s_gm1[cur] : s_lam1[prev] * s_gm1[cur])
                        : ((c == 0) ? s_gm[k] : s_lam[prev][k] * s_gm[k]);
#pragma unroll
    for (int cb = 0; cb < NV / 64; ++cb) {
      const int col = ch * (NV / 2) + 32 * cb;
      float x[32];
      if (c == 0) {
        if (a.S0) {
          const float* src = a.S0 + ((int64_t)bh * DK + k) * dv + col0 + col;
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 f = *reinterpret_cast<const float4*>(src + e);
            x[e] = f.x, x[e + 1] = f.y, x[e + 2] = f.z, x[e + 3] = f.w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = 0.f;
        }
      } else {
        tmem_ld32(tmem + lane_base + Ly::TM_S + col, x);
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] *= mu;
      tmem_st32(tmem + lane_base + Ly::TM_S + col, x);
#pragma unroll
      for (int q8 = 0; q8 < 4; ++q8) {
        uint4 pk = make_uint4(pack_bf16(x[8 * q8], x[8 * q8 + 1]), pack_bf16(x[8 * q8 + 2], x[8 * q8 + 3]),
                              pack_bf16(x[8 * q8 + 4], x[8 * q8 + 5]), pack_bf16(x[8 * q8 + 6], x[8 * q8 + 7]));
        *reinterpret_cast<uint4*>(sm + Ly::SM + canon_chunk(k, col / 8 + q8, DK)) = pk;
      }
    }
  };
  // o rows of chunk c from rows 64..127 of D1 (warps of quadrants 2 and 3, columns of half ch); the
  // TMEM load is warp-collective: every lane loads, only rows of real tokens store
  auto store_o = [&](int c) {
    const int t = 32 * (q4 - 2) + lane, t0c = c * C, nc = min(C, T - t0c);
    const float os = SC ? s_r[c & 1][t] : 1.f;
    __nv_bfloat16* orow =
        reinterpret_cast<__nv_bfloat16*>(a.o) + (((int64_t)b * T + t0c + t) * H + h) * dv + col0;
#pragma unroll
    for (int cb = 0; cb < NV / 64; ++cb) {
      const int col = ch * (NV / 2) + 32 * cb;
      float x[32];
      tmem_ld32(tmem + lane_base + Ly::TM_D1 + col, x);
      if (t < nc) {
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint4 pk = make_uint4(pack_bf16(os * x[8 * q8], os * x[8 * q8 + 1]),
                                pack_bf16(os * x[8 * q8 + 2], os * x[8 * q8 + 3]),
                                pack_bf16(os * x[8 * q8 + 4], os * x[8 * q8 + 5]),
                                pack_bf16(os * x[8 * q8 + 6], os * x[8 * q8 + 7]));
          *reinterpret_cast<uint4*>(orow + col + 8 * q8) = pk;
        }
      }
    }
  };

  // Gram [K+; Q+] W-^T (per-token path: [K; Q] K^T) of chunk c -> TMEM scratch; thread 0 only
  auto issue_gram = [&](int c) {
    uint8_t* kqc = kq_buf(c);
    const uint8_t* gb = SC ? kqc : sm + Ly::WHI;
    const uint32_t gb_blk = SC ? 128 * 128 : C * 128;
#pragma unroll
    for (int kk = 0; kk < DK; kk += 16) {
      const uint64_t ad = sdesc(smem_u32(kqc) + (kk >> 6) * (128 * 128) + (kk & 63) * 2, 16, 1024);
      const uint64_t bd = sdesc(smem_u32(gb) + (kk >> 6) * gb_blk + (kk & 63) * 2, 16, 1024);
      mma_bf16(tmem + Ly::TM_SCR, ad, bd, id_gram, kk > 0);
    }
  };

  for (int c = 0; c < nchunks; ++c) {
    const int t0 = c * C;
    const int n = min(C, T - t0);
    const int cur = c & 1, prev = cur ^ 1;

    // ---- P0: this chunk's q, k, v have landed
    {
      bool ok = mbar_wait_bounded(&bar_qk, ph_qk, kWaitNs) && mbar_wait_bounded(&bar_v, ph_v, kWaitNs);
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      ph_qk ^= 1;
      ph_v ^= 1;
      qk_pending = v_pending = false;
    }
    uint8_t* const kq = kq_buf(c);
    // per-token path: the other [K; Q] buffer was last read by the previous chunk's D1 MMA
    if (SC && tid == 0 && c + 1 < nchunks) issue_qk(c + 1);
    if (SC && c + 1 < nchunks) qk_pending = true;

    // ---- P1: decay factors (and, per-channel path, the operand tiles)
    if (SC) {
      // per-token factors of this chunk were computed during the previous chunk (token_prep)
    } else {
      // per-channel path: thread (g4, tg) owns channels 4g4..4g4+3 of tokens 8tg..8tg+7
      const int g4 = lane, tg = warp, cb0 = 4 * g4;
      float4 al[8], ws[8], dd[8];
      uint2 kr[8], qr[8];
      // tokens 8 tg .. 8 tg + 7 of this chunk; a group wholly past the end reads token 0 of the
      // chunk (always a real token) and discards it
      const int nvalid = max(0, min(8, n - 8 * tg));
      const int64_t tok0 = ((int64_t)b * T + t0 + (nvalid > 0 ? 8 * tg : 0)) * H + h;
      gate4x8(al, a.alpha_p, a.alpha, tok0, H, DK, cb0, nvalid, 1.f);
      gate4x8(ws, a.beta_k_p, a.beta_k, tok0, H, DK, cb0, nvalid, 0.f);
      gate4x8(dd, a.key_scale_p, a.key_scale, tok0, H, DK, cb0, nvalid, 0.f);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int j = 8 * tg + i;
        kr[i] = *reinterpret_cast<const uint2*>(sm + Ly::STK + canon(j, cb0, C));
        qr[i] = *reinterpret_cast<const uint2*>(sm + Ly::STQ + canon(j, cb0, C));
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) ws[i] = mul4(ws[i], dd[i]);
      // products inside the group: prefix (second half) or exclusive suffix (first half)
      float4 loc[8];
      float4 grp;
      if (tg >= 4) {
        float4 p = f4(1.f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          p = mul4(p, al[i]);
          loc[i] = p;
        }
        grp = p;
      } else {
        float4 p = f4(1.f);
#pragma unroll
        for (int i = 7; i >= 0; --i) {
          loc[i] = p;
          p = mul4(p, al[i]);
        }
        grp = p;
      }
      sts4(&s_grp[tg][0], cb0, grp);
      __syncthreads();
      float4 off = f4(1.f);
      if (tg >= 4) {
        for (int g = 4; g < tg; ++g) off = mul4(off, lds4(&s_grp[g][0], cb0));
      } else {
        for (int g = tg + 1; g < 4; ++g) off = mul4(off, lds4(&s_grp[g][0], cb0));
      }
      if (tg == 0) {
        float4 gm = f4(1.f), lm = f4(1.f);
#pragma unroll
        for (int g = 0; g < 4; ++g) gm = mul4(gm, lds4(&s_grp[g][0], cb0));
#pragma unroll
        for (int g = 4; g < 8; ++g) lm = mul4(lm, lds4(&s_grp[g][0], cb0));
        sts4(s_gm, cb0, gm);
        sts4(&s_lam[cur][0], cb0, lm);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int j = 8 * tg + i;
        float4 r, rinv;
        if (tg >= 4) {
          r = mul4(off, loc[i]);
          rinv = rcp4(r);
        } else {
          rinv = mul4(off, loc[i]);
          r = rcp4(rinv);
        }
        const float4 kk = unpack4(kr[i]), qq = unpack4(qr[i]);
        *reinterpret_cast<uint2*>(kq + canon(j, cb0, 128)) = pack4(mul4(kk, r));
        *reinterpret_cast<uint2*>(kq + canon(64 + j, cb0, 128)) = pack4(mul4(qq, r));
        uint2 hi, lo;
        split4(mul4(mul4(ws[i], kk), rinv), hi, lo);
        *reinterpret_cast<uint2*>(sm + Ly::WHI + canon(j, cb0, C)) = hi;
        *reinterpret_cast<uint2*>(sm + Ly::WLO + canon(j, cb0, C)) = lo;
      }
      if (bv_split && cb0 < NV) {
        // V~ = beta^v (.) v, split hi (in place) / lo
        float4 bvs[8];
        gate4x8(bvs, a.beta_v_p, a.beta_v, tok0, H, dv, col0 + cb0, nvalid, 0.f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int j = 8 * tg + i;
          const float4 bv = bvs[i];
          const uint32_t off2 = canon(j, cb0, C);
          const float4 vv = unpack4(*reinterpret_cast<const uint2*>(sm + Ly::STV + off2));
          uint2 hi, lo;
          split4(mul4(vv, bv), hi, lo);
          *reinterpret_cast<uint2*>(sm + Ly::STV + off2) = hi;
          *reinterpret_cast<uint2*>(sm + Ly::VLO + off2) = lo;
        }
      }
    }
    __syncthreads();

    // ---- P1.5: (the state is brought into this chunk's frame while the T MMAs run, below)
    fence_proxy_async();
    __syncthreads();

    // ---- P2: Gram [K+; Q+] W-^T (per-token path: [K; Q] K^T) -> scratch
    const bool gram_early = SC && s_gram_ready;  // uniform: written before the last barrier
    if (gram_early) {
      bool ok = mbar_wait_bounded(&bar_gram, ph_gram, kWaitNs);
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      ph_gram ^= 1;
      gram_pending = false;
      tc_fence_after();
    } else {
      if (tid == 0) {
        // per-channel path: the raw q, k staging was consumed by the prep; prefetch the next chunk
        if (!SC && c + 1 < nchunks) {
          fence_proxy_async();
          issue_qk(c + 1);
        }
        issue_gram(c);
        mma_commit(&bar_mma);
      }
      if (!SC && c + 1 < nchunks) qk_pending = true;
      mma_pending = true;
      bool ok = mbar_wait_bounded(&bar_mma, ph_mma, kWaitNs);
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      ph_mma ^= 1;
      mma_pending = false;
      tc_fence_after();
    }

    // ---- P3: A (strict lower) -> fp32 scratch; P (lower incl.) -> bf16 TP rows 64..127
    {
      float x[32];
      tmem_ld32(tmem + lane_base + Ly::TM_SCR + 32 * ch, x);
      const int i0 = 32 * ch;
      if (q4 < 2) {
        const int t = 32 * q4 + lane;
        const float rt = SC ? s_r[cur][t] : 1.f;
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          float y[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = i0 + 4 * e4 + e;
            float v = x[4 * e4 + e];
            if (SC) v *= s_ws[cur][i] * rt * s_ri[cur][i];
            y[e] = (i < t) ? v : 0.f;
          }
          sts4(sL, xi(t, i0 + 4 * e4), make_float4(y[0], y[1], y[2], y[3]));
        }
      } else {
        const int t = 32 * (q4 - 2) + lane;
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) y[e] = (i0 + 8 * q8 + e <= t) ? x[8 * q8 + e] : 0.f;
          uint4 pk = make_uint4(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]), pack_bf16(y[4], y[5]),
                                pack_bf16(y[6], y[7]));
          *reinterpret_cast<uint4*>(sm + Ly::TP + canon_chunk(64 + t, i0 / 8 + q8, 128)) = pk;
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    unit_lower_inverse<SC>(sL, sT, s_Y, sm + Ly::TP, sm + Ly::STQ, s_r[cur], s_bv[cur], tid);
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- P4: Wk = [T; P] K+ -> scratch;  U0 = [T; P] V~ (per-token path: T~ V) -> U0
    if (tid == 0) {
      const uint8_t* ta = SC ? sm + Ly::STQ : sm + Ly::TP;
#pragma unroll
      for (int kk = 0; kk < C; kk += 16) {
        const uint64_t ad = sdesc(smem_u32(sm + Ly::TP) + kk * 2, 16, 1024);
        const uint64_t bk = sdesc(smem_u32(kq) + kk * 128, 128 * 128, 1024);
        mma_bf16(tmem + Ly::TM_SCR, ad, bk, id_wk, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < C; kk += 16) {
        const uint64_t ad = sdesc(smem_u32(ta) + kk * 2, 16, 1024);
        const uint64_t bv = sdesc(smem_u32(sm + Ly::STV) + kk * 128, C * 128, 1024);
        mma_bf16(tmem + Ly::TM_U0, ad, bv, id_nv, kk > 0);
      }
      if (bv_split) {
#pragma unroll
        for (int kk = 0; kk < C; kk += 16) {
          const uint64_t ad = sdesc(smem_u32(sm + Ly::TP) + kk * 2, 16, 1024);
          const uint64_t bv = sdesc(smem_u32(sm + Ly::VLO) + kk * 128, C * 128, 1024);
          mma_bf16(tmem + Ly::TM_U0, ad, bv, id_nv, 1);
        }
      }
      mma_commit(&bar_mma);
    }
    mma_pending = true;
    // while those MMAs run: the previous chunk's outputs (D1 rows 64..127) and the state in this
    // chunk's frame (S_acc columns; no overlap with the TMEM the MMAs write)
    if (!SC && c > 0 && q4 >= 2) store_o(c - 1);
    state_to_frame(c);
    {
      bool ok = mbar_wait_bounded(&bar_mma, ph_mma, kWaitNs);
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      ph_mma ^= 1;
      mma_pending = false;
      tc_fence_after();
    }
    if (tid == 0 && c + 1 < nchunks) {
      fence_proxy_async();
      issue_v(c + 1);
    }
    if (c + 1 < nchunks) v_pending = true;

    // ---- P5: Wk -> bf16 into KQ rows 0..63 (K+ / raw K there is dead now)
    if (q4 < 2) {
      const int t = 32 * q4 + lane;
#pragma unroll
      for (int cb = 0; cb < DK / 64; ++cb) {
        const int col = ch * (DK / 2) + 32 * cb;
        float x[32];
        tmem_ld32(tmem + lane_base + Ly::TM_SCR + col, x);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint4 pk = make_uint4(pack_bf16(x[8 * q8], x[8 * q8 + 1]), pack_bf16(x[8 * q8 + 2], x[8 * q8 + 3]),
                                pack_bf16(x[8 * q8 + 4], x[8 * q8 + 5]), pack_bf16(x[8 * q8 + 6], x[8 * q8 + 7]));
          *reinterpret_cast<uint4*>(kq + canon_chunk(t, col / 8 + q8, 128)) = pk;
        }
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- P6: D1 = [Wk; Q+] S_m
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < DK; kk += 16) {
        const uint64_t ad = sdesc(smem_u32(kq) + (kk >> 6) * (128 * 128) + (kk & 63) * 2, 16, 1024);
        const uint64_t bd = sdesc(smem_u32(sm + Ly::SM) + kk * 128, DK * 128, 1024);
        mma_bf16(tmem + Ly::TM_D1, ad, bd, id_nv, kk > 0);
      }
      mma_commit(&bar_mma);
    }
    mma_pending = true;
    {
      bool ok = mbar_wait_bounded(&bar_mma, ph_mma, kWaitNs);
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      ph_mma ^= 1;
      mma_pending = false;
      tc_fence_after();
    }

    // ---- P7: U = U0 - Wk S_m (per-token path: U' = beta_t / r_t * U) -> hi / lo tiles
    // (per-token path: warps 2, 3 meanwhile compute the next chunk's decay factors)
    if (SC && (warp == 2 || warp == 3) && c + 1 < nchunks) token_prep(c + 1, tid - 64, warp == 3);
    if (q4 < 2) {
      const int t = 32 * q4 + lane;
      const float us = SC ? s_ws[cur][t] * s_ri[cur][t] : 1.f;
#pragma unroll
      for (int cb = 0; cb < NV / 64; ++cb) {
        const int col = ch * (NV / 2) + 32 * cb;
        float u0[32], d1[32];
        tmem_ld32(tmem + lane_base + Ly::TM_U0 + col, u0);
        tmem_ld32(tmem + lane_base + Ly::TM_D1 + col, d1);
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = 8 * q8 + 2 * e;
            split_bf16(us * (u0[i] - d1[i]), us * (u0[i + 1] - d1[i + 1]), hi[e], lo[e]);
          }
          const uint32_t off = canon_chunk(t, col / 8 + q8, C);
          *reinterpret_cast<uint4*>(sm + Ly::UHI + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(sm + Ly::ULO + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- P8: O = Q+ S_m + P U (rows 64..127 of D1); S_acc += W-^T U (split)
    if (SC) {
      bool ok = mbar_wait_bounded(&bar_k, ph_k, kWaitNs);
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      ph_k ^= 1;
      k_pending = false;
    }
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < C; kk += 16) {
        const uint64_t ad = sdesc(smem_u32(sm + Ly::TP) + kk * 2, 16, 1024);
        const uint64_t bd = sdesc(smem_u32(sm + Ly::UHI) + kk * 128, C * 128, 1024);
        mma_bf16(tmem + Ly::TM_D1, ad, bd, id_nv, 1);
      }
#pragma unroll
      for (int kk = 0; kk < C; kk += 16) {
        const uint64_t buh = sdesc(smem_u32(sm + Ly::UHI) + kk * 128, C * 128, 1024);
        const uint64_t bul = sdesc(smem_u32(sm + Ly::ULO) + kk * 128, C * 128, 1024);
        if (SC) {
          const uint64_t ak = sdesc(smem_u32(sm + Ly::STK) + kk * 128, C * 128, 1024);
          mma_bf16(tmem + Ly::TM_S, ak, buh, id_state, 1);
          mma_bf16(tmem + Ly::TM_S, ak, bul, id_state, 1);
        } else {
          const uint64_t awh = sdesc(smem_u32(sm + Ly::WHI) + kk * 128, C * 128, 1024);
          const uint64_t awl = sdesc(smem_u32(sm + Ly::WLO) + kk * 128, C * 128, 1024);
          mma_bf16(tmem + Ly::TM_S, awh, buh, id_state, 1);
          mma_bf16(tmem + Ly::TM_S, awh, bul, id_state, 1);
          mma_bf16(tmem + Ly::TM_S, awl, buh, id_state, 1);
        }
      }
      mma_commit(&bar_mma);
      // per-token path: the next chunk's [K; Q] tile has its own buffer; once it has landed, its
      // Gram can follow these MMAs on the tensor core right away
      int ready = 0;
      if (SC && c + 1 < nchunks && mbar_wait_bounded(&bar_qk, ph_qk, kWaitNs)) {
        issue_gram(c + 1);
        mma_commit(&bar_gram);
        ready = 1;
      }
      s_gram_ready = ready;
    }
    mma_pending = true;
    {
      bool ok = mbar_wait_bounded(&bar_mma, ph_mma, kWaitNs);
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      ph_mma ^= 1;
      mma_pending = false;
      tc_fence_after();
    }
    if (SC && s_gram_ready) gram_pending = true;
    // per-token path: the raw k tile of the state update is free now: load the next chunk's
    if (SC && tid == 0 && c + 1 < nchunks) {
      fence_proxy_async();
      issue_k(c + 1);
    }
    if (SC && c + 1 < nchunks) k_pending = true;
    // per-token path: this chunk's outputs, while the next chunk's Gram runs
    if (SC && q4 >= 2) store_o(c);

    // ---- P9: (this chunk's outputs are stored during the next chunk's inverse, or after the loop)
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  if (!failed && nchunks > 0) {
    if (!SC && q4 >= 2) store_o(nchunks - 1);
    // S_T = Diag(gamma_C / gamma_m) S_acc of the last chunk
    const int k = 32 * q4 + lane;
    const float lam = SC ? s_lam1[(nchunks - 1) & 1] : s_lam[(nchunks - 1) & 1][k];
#pragma unroll
    for (int cb = 0; cb < NV / 64; ++cb) {
      const int col = ch * (NV / 2) + 32 * cb;
      float x[32];
      tmem_ld32(tmem + lane_base + Ly::TM_S + col, x);
      float* dst = a.S + ((int64_t)bh * DK + k) * dv + col0 + col;
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(dst + e) = make_float4(lam * x[e], lam * x[e + 1], lam * x[e + 2], lam * x[e + 3]);
    }
  }
  if (failed) {
    // drain whatever this CTA still has in flight (bounded), then report
    if (qk_pending) mbar_wait_bounded(&bar_qk, ph_qk, kWaitNs);
    if (k_pending) mbar_wait_bounded(&bar_k, ph_k, kWaitNs);
    if (v_pending) mbar_wait_bounded(&bar_v, ph_v, kWaitNs);
    if (mma_pending) mbar_wait_bounded(&bar_mma, ph_mma, kWaitNs);
    if (gram_pending) mbar_wait_bounded(&bar_gram, ph_gram, kWaitNs);
    if (tid == 0) atomicExch(a.status, kDevTimeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool get_encode() {
  if (g_encode) return true;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return false;
  g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  return true;
}

// 4-D map over a [B, T, H, d] bf16 tensor; box = 64 channels x 1 head x 64 tokens x 1 batch.
bool make_map(CUtensorMap* m, const void* base, int d, int H, int T, int B) {
  cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
  cuuint32_t box[4] = {64, 1, (cuuint32_t)C, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int DK, int NV, bool SC>
cudaError_t launch_impl(const Args& a, cudaStream_t s) {
  using Ly = Layout<DK, NV>;
  const int smem = Ly::TOTAL + 1024;
  // per call: the attribute is per device, and the call is cheap next to the kernel
  cudaError_t e =
      cudaFuncSetAttribute(chunk_tc_kernel<DK, NV, SC>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  CUtensorMap mq, mk, mv;
  if (!get_encode()) return cudaErrorNotSupported;
  if (!make_map(&mq, a.q, DK, a.H, a.T, a.B) || !make_map(&mk, a.k, DK, a.H, a.T, a.B) ||
      !make_map(&mv, a.v, a.dv, a.H, a.T, a.B))
    return cudaErrorInvalidValue;
  chunk_tc_kernel<DK, NV, SC><<<a.B * a.H * (a.dv / NV), kThreads, smem, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace

bool chunk_tc_supported(const Args& a) {
  return a.io_bf16 && a.dk == 128 && (a.dv == 128 || a.dv == 64) && a.chunk == C && a.T > 0;
}

cudaError_t launch_chunk_tc(const Args& a, cudaStream_t s) {
  // per-token gates only -> the raw-tile path
  const bool sc = a.alpha != DN_GATE_CHANNEL && a.beta_k != DN_GATE_CHANNEL && a.beta_v != DN_GATE_CHANNEL &&
                  a.key_scale != DN_GATE_CHANNEL;
  // few sequences: split the 128 value columns into two 64-column CTAs when that still fits in one
  // wave (each CTA repeats the column-independent prep, Gram and inverse)
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const bool split = a.dv == 128 && (int64_t)a.B * a.H * 2 <= sms;
  if (a.dv == 128 && !split) return sc ? launch_impl<128, 128, true>(a, s) : launch_impl<128, 128, false>(a, s);
  return sc ? launch_impl<128, 64, true>(a, s) : launch_impl<128, 64, false>(a, s);
}

}  // namespace dn
