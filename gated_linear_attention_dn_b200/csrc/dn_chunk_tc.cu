// Tensor-core chunked prefill (bf16 io, d_k = 128, d_v in {64, 128}) for sm_100a.
//
// One CTA (256 threads) owns one (b, h) sequence and walks its chunks of C = 64
// tokens in order, keeping the fp32 state in tensor memory. Per chunk, with the
// log-decay prefix referenced to the chunk midpoint m (after token 31), so that
// every exponent spans at most half a chunk of decay:
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
// Precision plan (bf16 operands, fp32 accumulation everywhere): the state update
// W-^T U is the product whose rounding reaches S_T directly, so both operands
// are split hi + lo in bf16 (three MMAs: hi*hi + hi*lo + lo*hi); V~ is split the
// same way when beta^v is present. All other operands are single bf16.
//
// Shared-memory operand tiles use the 128-byte-swizzled canonical layout (see
// canon()); q/k/v tiles arrive by TMA (4-D tensor maps over [B, T, H, d], boxes of
// 64 channels x 64 tokens, zero fill past the end of the sequence).
//
// Tensor memory (512 columns): S_acc [0, NV) | D1 [NV, 2NV) | U0 [2NV, 3NV) | scratch (Gram, Wk).
// Every wait on an mbarrier is bounded; on expiry the CTA sets the status word,
// drains what it issued (again bounded), frees its tensor memory and exits.
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
  static constexpr int STQ = STK + C * DK * 2;        // raw q  [C][DK]   (TMA)
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

// rotated index into a 64x64 fp32 array: row r's columns start at bank r, so
// column-wise access by 32 consecutive rows is conflict-free
__device__ __forceinline__ int ri(int r, int c) { return (r << 6) | ((c + r) & 63); }

__device__ __forceinline__ float2 gate2(const float* g, int mode, int64_t tok, int width, int ch) {
  if (mode == DN_GATE_ONE) return make_float2(1.f, 1.f);
  if (mode == DN_GATE_SCALAR) {
    const float x = g[tok];
    return make_float2(x, x);
  }
  return *reinterpret_cast<const float2*>(g + tok * width + ch);
}

// X = sum_{k=j}^{i-1} L_ik T_kj for block (i, j) of the 16x16 blocking; element (r, cc).
__device__ __forceinline__ float block_lt(const float* sL, const float* sT, int i, int j, int r, int cc) {
  float s = 0.f;
  for (int k = j; k < i; ++k) {
#pragma unroll
    for (int m = 0; m < 16; ++m) s = fmaf(sL[ri(16 * i + r, 16 * k + m)], sT[ri(16 * k + m, 16 * j + cc)], s);
  }
  return s;
}

// T_ij = -T_ii X for block (i, j); element (r, cc); X is 16x16 row-major.
__device__ __forceinline__ float block_tx(const float* sT, const float* X, int i, int r, int cc) {
  float s = 0.f;
#pragma unroll
  for (int m = 0; m < 16; ++m) s = fmaf(sT[ri(16 * i + r, 16 * i + m)], X[m * 16 + cc], s);
  return -s;
}

template <int DK, int NV>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Args a) {
  using Ly = Layout<DK, NV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_qk, bar_v, bar_mma;
  __shared__ uint32_t s_tmem;
  __shared__ float s_lam[2][DK];
  __shared__ float s_gm[DK];
  __shared__ float s_X[3][256];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, ch = warp >> 2;
  const int T = a.T, H = a.H, dv = a.dv;
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  const int nchunks = (T + C - 1) / C;

  if (tid == 0) {
    mbar_init(&bar_qk, 1);
    mbar_init(&bar_v, 1);
    mbar_init(&bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&s_tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t lane_base = (uint32_t)(32 * q4) << 16;

  auto issue_qk = [&](int c) {
    mbar_expect_tx(&bar_qk, 2u * C * DK * 2);
#pragma unroll
    for (int x = 0; x < DK / 64; ++x) {
      tma_load_4d(sm + Ly::STK + x * C * 128, &tm_k, &bar_qk, 64 * x, h, c * C, b);
      tma_load_4d(sm + Ly::STQ + x * C * 128, &tm_q, &bar_qk, 64 * x, h, c * C, b);
    }
  };
  auto issue_v = [&](int c) {
    mbar_expect_tx(&bar_v, (uint32_t)C * NV * 2);
#pragma unroll
    for (int x = 0; x < NV / 64; ++x) tma_load_4d(sm + Ly::STV + x * C * 128, &tm_v, &bar_v, 64 * x, h, c * C, b);
  };

  uint32_t ph_qk = 0, ph_v = 0, ph_mma = 0;
  bool qk_pending = false, v_pending = false, mma_pending = false;
  bool failed = false;
  if (tid == 0 && nchunks > 0) {
    issue_qk(0);
    issue_v(0);
  }
  if (nchunks > 0) qk_pending = v_pending = true;

  const uint32_t id_gram = idesc_bf16(128, 64, 0, 0);
  const uint32_t id_wk = idesc_bf16(128, DK, 0, 1);
  const uint32_t id_nv = idesc_bf16(128, NV, 0, 1);
  const uint32_t id_state = idesc_bf16(128, NV, 1, 1);
  const bool bv_split = a.beta_v != DN_GATE_ONE;
  float* sL = reinterpret_cast<float*>(sm + Ly::INV);
  float* sT = sL + C * C;

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

    // ---- P1: gate prefix products and operand tiles
    if (tid < 128) {
      const int c0 = 2 * (tid & 63);
      const int half = tid >> 6;
      float2 r = make_float2(1.f, 1.f), rinv = make_float2(1.f, 1.f), rho = make_float2(1.f, 1.f);
      const int jbeg = half ? 32 : 31, jend = half ? 64 : -1, jstep = half ? 1 : -1;
      for (int j = jbeg; j != jend; j += jstep) {
        const bool valid = j < n;
        const int64_t tok = ((int64_t)b * T + t0 + j) * H + h;
        float2 al = make_float2(1.f, 1.f), ws = make_float2(0.f, 0.f);
        if (valid) {
          al = gate2(a.alpha_p, a.alpha, tok, DK, c0);
          const float2 bk = gate2(a.beta_k_p, a.beta_k, tok, DK, c0);
          const float2 dd = gate2(a.key_scale_p, a.key_scale, tok, DK, c0);
          ws = make_float2(bk.x * dd.x, bk.y * dd.y);
        }
        const float2 ial = make_float2(__fdividef(1.f, al.x), __fdividef(1.f, al.y));
        if (half) {  // forward from the midpoint: r_j = prod_{s=32..j} alpha_s
          r.x *= al.x;
          r.y *= al.y;
          rinv.x *= ial.x;
          rinv.y *= ial.y;
        }
        const float2 kk = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm + Ly::STK + canon(j, c0, C)));
        const float2 qq = unpack_bf16(*reinterpret_cast<const uint32_t*>(sm + Ly::STQ + canon(j, c0, C)));
        *reinterpret_cast<uint32_t*>(sm + Ly::KQ + canon(j, c0, 128)) = pack_bf16(kk.x * r.x, kk.y * r.y);
        *reinterpret_cast<uint32_t*>(sm + Ly::KQ + canon(64 + j, c0, 128)) = pack_bf16(qq.x * r.x, qq.y * r.y);
        uint32_t whi, wlo;
        split_bf16(ws.x * kk.x * rinv.x, ws.y * kk.y * rinv.y, whi, wlo);
        *reinterpret_cast<uint32_t*>(sm + Ly::WHI + canon(j, c0, C)) = whi;
        *reinterpret_cast<uint32_t*>(sm + Ly::WLO + canon(j, c0, C)) = wlo;
        if (!half) {  // backward from the midpoint: r_{j-1} = r_j / alpha_j
          r.x *= ial.x;
          r.y *= ial.y;
          rinv.x *= al.x;
          rinv.y *= al.y;
          rho.x *= al.x;
          rho.y *= al.y;
        }
      }
      if (half) {
        s_lam[cur][c0] = r.x;
        s_lam[cur][c0 + 1] = r.y;
      } else {
        s_gm[c0] = rho.x;
        s_gm[c0 + 1] = rho.y;
      }
    } else if (bv_split) {
      // V~ = beta^v (.) v, split hi (in place) / lo
      const int u = tid - 128;
      const int j = u >> 1;
      const bool valid = j < n;
      const int64_t tok = ((int64_t)b * T + t0 + j) * H + h;
      constexpr int CH8 = NV / 16;  // 16-byte chunks per thread (half a row)
#pragma unroll
      for (int i = 0; i < CH8; ++i) {
        const int x8 = (u & 1) * CH8 + i;
        const uint32_t off = canon_chunk(j, x8, C);
        uint4 raw = *reinterpret_cast<const uint4*>(sm + Ly::STV + off);
        float bv[8];
        if (!valid) {
#pragma unroll
          for (int e = 0; e < 8; ++e) bv[e] = 0.f;
        } else if (a.beta_v == DN_GATE_SCALAR) {
          const float x = a.beta_v_p[tok];
#pragma unroll
          for (int e = 0; e < 8; ++e) bv[e] = x;
        } else {
          const float4 lo4 = *reinterpret_cast<const float4*>(a.beta_v_p + tok * dv + 8 * x8);
          const float4 hi4 = *reinterpret_cast<const float4*>(a.beta_v_p + tok * dv + 8 * x8 + 4);
          bv[0] = lo4.x, bv[1] = lo4.y, bv[2] = lo4.z, bv[3] = lo4.w;
          bv[4] = hi4.x, bv[5] = hi4.y, bv[6] = hi4.z, bv[7] = hi4.w;
        }
        uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w}, hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 vv = unpack_bf16(w[e]);
          split_bf16(vv.x * bv[2 * e], vv.y * bv[2 * e + 1], hi[e], lo[e]);
        }
        *reinterpret_cast<uint4*>(sm + Ly::STV + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(sm + Ly::VLO + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    __syncthreads();

    // ---- P1.5: bring the state into this chunk's frame: S_m = Diag(lambda_prev * gamma_m) S
    {
      const int k = 32 * q4 + lane;
      const float mu = (c == 0) ? s_gm[k] : s_lam[prev][k] * s_gm[k];
#pragma unroll
      for (int cb = 0; cb < NV / 64; ++cb) {
        const int col = ch * (NV / 2) + 32 * cb;
        float x[32];
        if (c == 0) {
          if (a.S0) {
            const float* src = a.S0 + ((int64_t)bh * DK + k) * dv + col;
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
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- P2: prefetch next q/k; Gram [K+; Q+] W-^T -> scratch
    if (tid == 0) {
      if (c + 1 < nchunks) issue_qk(c + 1);
#pragma unroll
      for (int kk = 0; kk < DK; kk += 16) {
        const uint64_t ad = sdesc(smem_u32(sm + Ly::KQ) + (kk >> 6) * (128 * 128) + (kk & 63) * 2, 16, 1024);
        const uint64_t bd = sdesc(smem_u32(sm + Ly::WHI) + (kk >> 6) * (C * 128) + (kk & 63) * 2, 16, 1024);
        mma_bf16(tmem + Ly::TM_SCR, ad, bd, id_gram, kk > 0);
      }
      mma_commit(&bar_mma);
    }
    if (c + 1 < nchunks) qk_pending = true;
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

    // ---- P3: A (strict lower) -> fp32 scratch; P (lower incl.) -> bf16 TP rows 64..127
    {
      float x[32];
      tmem_ld32(tmem + lane_base + Ly::TM_SCR + 32 * ch, x);
      const int i0 = 32 * ch;
      if (q4 < 2) {
        const int t = 32 * q4 + lane;
#pragma unroll
        for (int e = 0; e < 32; ++e) sL[ri(t, i0 + e)] = (i0 + e < t) ? x[e] : 0.f;
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
    // inverse of the unit lower-triangular (I + A), 16x16 blocking
    if (tid < 64) {
      const int blk = tid >> 4, j = tid & 15;
      float xv[16];
#pragma unroll
      for (int r = 0; r < 16; ++r) {
        float s = (r == j) ? 1.f : 0.f;
#pragma unroll
        for (int i = 0; i < r; ++i) s = fmaf(-sL[ri(16 * blk + r, 16 * blk + i)], xv[i], s);
        xv[r] = s;
      }
#pragma unroll
      for (int r = 0; r < 16; ++r) sT[ri(16 * blk + r, 16 * blk + j)] = xv[r];
    }
    __syncthreads();
    {
      const int r = tid >> 4, cc = tid & 15;
      // level 1: (1,0) (2,1) (3,2)
#pragma unroll
      for (int bi = 1; bi < 4; ++bi) s_X[bi - 1][tid] = block_lt(sL, sT, bi, bi - 1, r, cc);
      __syncthreads();
#pragma unroll
      for (int bi = 1; bi < 4; ++bi) sT[ri(16 * bi + r, 16 * (bi - 1) + cc)] = block_tx(sT, s_X[bi - 1], bi, r, cc);
      __syncthreads();
      // level 2: (2,0) (3,1)
#pragma unroll
      for (int bi = 2; bi < 4; ++bi) s_X[bi - 2][tid] = block_lt(sL, sT, bi, bi - 2, r, cc);
      __syncthreads();
#pragma unroll
      for (int bi = 2; bi < 4; ++bi) sT[ri(16 * bi + r, 16 * (bi - 2) + cc)] = block_tx(sT, s_X[bi - 2], bi, r, cc);
      __syncthreads();
      // level 3: (3,0)
      s_X[0][tid] = block_lt(sL, sT, 3, 0, r, cc);
      __syncthreads();
      sT[ri(48 + r, cc)] = block_tx(sT, s_X[0], 3, r, cc);
      __syncthreads();
    }
    // T -> bf16 TP rows 0..63
    {
      const int t = tid >> 2;
      const int i0 = 16 * (tid & 3);
#pragma unroll
      for (int q8 = 0; q8 < 2; ++q8) {
        float y[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int i = i0 + 8 * q8 + e;
          y[e] = ((i >> 4) > (t >> 4)) ? 0.f : sT[ri(t, i)];
        }
        uint4 pk = make_uint4(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]), pack_bf16(y[4], y[5]),
                              pack_bf16(y[6], y[7]));
        *reinterpret_cast<uint4*>(sm + Ly::TP + canon_chunk(t, i0 / 8 + q8, 128)) = pk;
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- P4: Wk = [T; P] K+ -> scratch;  U0 = [T; P] V~ -> U0
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < C; kk += 16) {
        const uint64_t ad = sdesc(smem_u32(sm + Ly::TP) + kk * 2, 16, 1024);
        const uint64_t bk = sdesc(smem_u32(sm + Ly::KQ) + kk * 128, 128 * 128, 1024);
        mma_bf16(tmem + Ly::TM_SCR, ad, bk, id_wk, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < C; kk += 16) {
        const uint64_t ad = sdesc(smem_u32(sm + Ly::TP) + kk * 2, 16, 1024);
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

    // ---- P5: Wk -> bf16 into KQ rows 0..63 (K+ is dead now)
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
          *reinterpret_cast<uint4*>(sm + Ly::KQ + canon_chunk(t, col / 8 + q8, 128)) = pk;
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
        const uint64_t ad = sdesc(smem_u32(sm + Ly::KQ) + (kk >> 6) * (128 * 128) + (kk & 63) * 2, 16, 1024);
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

    // ---- P7: U = U0 - Wk S_m -> hi / lo tiles
    if (q4 < 2) {
      const int t = 32 * q4 + lane;
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
            split_bf16(u0[i] - d1[i], u0[i + 1] - d1[i + 1], hi[e], lo[e]);
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
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < C; kk += 16) {
        const uint64_t ad = sdesc(smem_u32(sm + Ly::TP) + kk * 2, 16, 1024);
        const uint64_t bd = sdesc(smem_u32(sm + Ly::UHI) + kk * 128, C * 128, 1024);
        mma_bf16(tmem + Ly::TM_D1, ad, bd, id_nv, 1);
      }
#pragma unroll
      for (int kk = 0; kk < C; kk += 16) {
        const uint64_t awh = sdesc(smem_u32(sm + Ly::WHI) + kk * 128, C * 128, 1024);
        const uint64_t awl = sdesc(smem_u32(sm + Ly::WLO) + kk * 128, C * 128, 1024);
        const uint64_t buh = sdesc(smem_u32(sm + Ly::UHI) + kk * 128, C * 128, 1024);
        const uint64_t bul = sdesc(smem_u32(sm + Ly::ULO) + kk * 128, C * 128, 1024);
        mma_bf16(tmem + Ly::TM_S, awh, buh, id_state, 1);
        mma_bf16(tmem + Ly::TM_S, awh, bul, id_state, 1);
        mma_bf16(tmem + Ly::TM_S, awl, buh, id_state, 1);
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

    // ---- P9: o rows of this chunk
    if (q4 >= 2) {
      // the TMEM load is warp-collective: every lane loads, only rows of real tokens store
      const int t = 32 * (q4 - 2) + lane;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) + (((int64_t)b * T + t0 + t) * H + h) * dv;
#pragma unroll
      for (int cb = 0; cb < NV / 64; ++cb) {
        const int col = ch * (NV / 2) + 32 * cb;
        float x[32];
        tmem_ld32(tmem + lane_base + Ly::TM_D1 + col, x);
        if (t < n) {
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            uint4 pk = make_uint4(pack_bf16(x[8 * q8], x[8 * q8 + 1]), pack_bf16(x[8 * q8 + 2], x[8 * q8 + 3]),
                                  pack_bf16(x[8 * q8 + 4], x[8 * q8 + 5]), pack_bf16(x[8 * q8 + 6], x[8 * q8 + 7]));
            *reinterpret_cast<uint4*>(orow + col + 8 * q8) = pk;
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  if (!failed && nchunks > 0) {
    // S_T = Diag(gamma_C / gamma_m) S_acc of the last chunk
    const int k = 32 * q4 + lane;
    const float lam = s_lam[(nchunks - 1) & 1][k];
#pragma unroll
    for (int cb = 0; cb < NV / 64; ++cb) {
      const int col = ch * (NV / 2) + 32 * cb;
      float x[32];
      tmem_ld32(tmem + lane_base + Ly::TM_S + col, x);
      float* dst = a.S + ((int64_t)bh * DK + k) * dv + col;
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(dst + e) = make_float4(lam * x[e], lam * x[e + 1], lam * x[e + 2], lam * x[e + 3]);
    }
  }
  if (failed) {
    // drain whatever this CTA still has in flight (bounded), then report
    if (qk_pending) mbar_wait_bounded(&bar_qk, ph_qk, kWaitNs);
    if (v_pending) mbar_wait_bounded(&bar_v, ph_v, kWaitNs);
    if (mma_pending) mbar_wait_bounded(&bar_mma, ph_mma, kWaitNs);
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

template <int DK, int NV>
cudaError_t launch_impl(const Args& a, cudaStream_t s) {
  using Ly = Layout<DK, NV>;
  const int smem = Ly::TOTAL + 1024;
  // per call: the attribute is per device, and the call is cheap next to the kernel
  cudaError_t e = cudaFuncSetAttribute(chunk_tc_kernel<DK, NV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  CUtensorMap mq, mk, mv;
  if (!get_encode()) return cudaErrorNotSupported;
  if (!make_map(&mq, a.q, DK, a.H, a.T, a.B) || !make_map(&mk, a.k, DK, a.H, a.T, a.B) ||
      !make_map(&mv, a.v, NV, a.H, a.T, a.B))
    return cudaErrorInvalidValue;
  chunk_tc_kernel<DK, NV><<<a.B * a.H, kThreads, smem, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace

bool chunk_tc_supported(const Args& a) {
  return a.io_bf16 && a.dk == 128 && (a.dv == 128 || a.dv == 64) && a.chunk == C && a.T > 0;
}

cudaError_t launch_chunk_tc(const Args& a, cudaStream_t s) {
  if (a.dv == 128) return launch_impl<128, 128>(a, s);
  return launch_impl<128, 64>(a, s);
}

}  // namespace dn
