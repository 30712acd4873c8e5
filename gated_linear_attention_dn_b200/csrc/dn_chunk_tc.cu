// Tensor-core chunked prefill for gates with a per-channel part (KDA channel decay, FG2-GDN+
// vector beta, OSDN key scale d), bf16 io, d_k = 128, d_v in {64, 128}, sm_100a. (Problems whose
// gates are all per-token scalars take the pipelined kernel in dn_chunk_sc.cu.)
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
// The CUDA cores build the K+, Q+, W- (hi/lo) and V~ (hi/lo) tiles per chunk from the raw
// TMA tiles and the gates, with all gate loads of a chunk in flight at once.
//
// Precision plan (bf16 operands, fp32 accumulation everywhere): the state update
// W-^T U is the product whose rounding reaches S_T directly, so its operands are
// split hi + lo in bf16; V~ is split the same way when beta^v is a vector. All
// other operands are single bf16.
//
// Shared-memory operand tiles use the 128-byte-swizzled canonical layout (see
// canon()); q/k/v tiles arrive by TMA (4-D tensor maps over [B, T, H, d], boxes of
// 64 channels x 64 tokens, zero fill past the end of the sequence).
//
// Strong decay: the midpoint-referenced factors stay within 2^-50 .. 2^50 only while the gates of
// each half chunk multiply to no less than that (mean alpha above ~0.34 per token). A chunk whose
// factors leave that range (any gate product of a half chunk below 2^-50, per channel) is evaluated
// exactly instead, token by token on the CUDA cores in fp32 (exact_chunk), from and back to the
// state in tensor memory; every other chunk keeps the tensor-core path.
//
// Tensor memory (512 columns): S_acc [0, NV) | D1 [NV, 2NV) | U0 [2NV, 3NV) | scratch (Gram, Wk).
// Every wait on an mbarrier is bounded in time; on expiry the CTA sets the status
// word, drains what it issued (again bounded), frees its tensor memory and exits.
#include "dn_common.cuh"
#include "dn_tc_ptx.cuh"
#include "dn_ut_inverse.cuh"

namespace dn {
namespace {

using namespace tc;
using namespace ut;

constexpr int C = 64;
constexpr int kThreads = 256;
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s: the bound of the drain waits after a failure

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
  // the exact path's fp32 state transpose (DK x (NV + 1)) overlays [T; P] and what follows it
  static_assert(TP + DK * (NV + 1) * 4 <= TOTAL, "transpose buffer of the exact path");
};

__device__ __forceinline__ float4 f4(float x) { return make_float4(x, x, x, x); }
__device__ __forceinline__ float4 mul4(float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); }
__device__ __forceinline__ float4 rcp4(float4 a) {
  return make_float4(__fdividef(1.f, a.x), __fdividef(1.f, a.y), __fdividef(1.f, a.z), __fdividef(1.f, a.w));
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

// shared -> global bulk copy (both addresses 16-byte aligned, bytes a multiple of 16), its group
// commit, and the wait until the committed copies have completed
__device__ __forceinline__ void bulk_store(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(ssrc)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ float4 lds4(const float* p, int idx) { return *reinterpret_cast<const float4*>(p + idx); }

// every component within [2^-50, 2^50] (false for NaN)
__device__ __forceinline__ bool in_range4(float4 v) {
  constexpr float lo = 8.8817842e-16f, hi = 1.1258999e15f;
  return v.x >= lo && v.x <= hi && v.y >= lo && v.y <= hi && v.z >= lo && v.z <= hi && v.w >= lo && v.w <= hi;
}
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

// Exact evaluation of one chunk, token by token on the CUDA cores in fp32, for a chunk whose decay is
// too strong for the midpoint-referenced factors of the tensor-core path. In: the chunk's raw k and q
// tiles, V~ (bf16 hi + lo when beta^v is given, else raw v), alpha and w = beta^k d k per token and
// key channel as fp32 rows (sAl, sWk, [C][DK]) and w_t . q_t per token (s_wq); the state entering
// the chunk comes from tensor memory times the previous chunk's pending end factor lam_prev (or from
// S0 at c == 0). Out: o of the chunk's n tokens straight to global memory, and the chunk-end state
// back into tensor memory (S_acc, no pending factor). Thread (j, part) owns value column j and DK / TPC
// key rows of it, so the per-token sums over the rows take TPC - 1 shuffles and no barrier; sX
// (DK x (NV + 1) fp32) transposes the state between the tensor-memory rows and these columns.
// Called by all 256 threads.
template <int DK, int NV>
__device__ __forceinline__ void exact_chunk(const Args& a, const uint8_t* sk, const uint8_t* sq, const uint8_t* svhi,
                                         const uint8_t* svlo, bool v_split, const float* sAl, const float* sWk,
                                         const float* s_wq, float* sX, const float* lam_prev, uint32_t tmem_s,
                                         int c, int n, int b, int h, int bh, int col0, int tid) {
  constexpr int TPC = kThreads / NV;  // threads per value column
  constexpr int R = DK / TPC;          // key rows per thread
  constexpr int LDX = NV + 1;
  const int warp = tid >> 5, lane = tid & 31, q4 = warp & 3, ch = warp >> 2;
  const int j = tid / TPC, part = tid % TPC, k0 = part * R;
  const int T = a.T, H = a.H, dv = a.dv, pre = a.pre_read;
  {
    // the state entering the chunk, tensor-memory rows -> sX
    const int k = 32 * q4 + lane;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
#pragma unroll
    for (int cb = 0; cb < NV / 64; ++cb) {
      const int col = ch * (NV / 2) + 32 * cb;
      float x[32];
      if (c == 0) {
        const float* src = a.S0 ? a.S0 + ((int64_t)bh * DK + k) * dv + col0 + col : nullptr;
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = src ? src[e] : 0.f;
      } else {
        tmem_ld32(tmem_s + lane_base + col, x);
        const float l = lam_prev[k];
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] *= l;
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) sX[k * LDX + col + e] = x[e];
    }
  }
  __syncthreads();
  float S[R];
#pragma unroll
  for (int r = 0; r < R; ++r) S[r] = sX[(k0 + r) * LDX + j];
  __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(a.o) + (((int64_t)b * T + c * C) * H + h) * dv + col0 + j;
  for (int t = 0; t < n; ++t) {
    const float* al = sAl + t * DK + k0;
    const float* wr = sWk + t * DK + k0;
    float rr = 0.f, ss = 0.f;  // (alpha (.) S)^T k and the read-out's S^T q over this thread's rows
#pragma unroll
    for (int r8 = 0; r8 < R; r8 += 8) {
      const uint4 kv = *reinterpret_cast<const uint4*>(sk + canon_chunk(t, (k0 + r8) >> 3, C));
      const uint4 qv = *reinterpret_cast<const uint4*>(sq + canon_chunk(t, (k0 + r8) >> 3, C));
      const float2 k01 = unpack_bf16(kv.x), k23 = unpack_bf16(kv.y), k45 = unpack_bf16(kv.z), k67 = unpack_bf16(kv.w);
      const float2 q01 = unpack_bf16(qv.x), q23 = unpack_bf16(qv.y), q45 = unpack_bf16(qv.z), q67 = unpack_bf16(qv.w);
      const float kf[8] = {k01.x, k01.y, k23.x, k23.y, k45.x, k45.y, k67.x, k67.y};
      const float qf[8] = {q01.x, q01.y, q23.x, q23.y, q45.x, q45.y, q67.x, q67.y};
      const float4 a0 = lds4(al, r8), a1 = lds4(al, r8 + 4);
      const float af[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float sb = af[e] * S[r8 + e];
        rr = fmaf(sb, kf[e], rr);
        ss = fmaf(pre ? S[r8 + e] : sb, qf[e], ss);
        S[r8 + e] = sb;
      }
    }
#pragma unroll
    for (int off = 1; off < TPC; off <<= 1) {
      rr += __shfl_xor_sync(0xffffffffu, rr, off);
      ss += __shfl_xor_sync(0xffffffffu, ss, off);
    }
    const uint32_t voff = canon(t, j, C);
    float vt = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(svhi + voff));
    if (v_split) vt += __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(svlo + voff));
    const float u = vt - rr;  // u_t = beta^v v_t - S_bar^T k_t
#pragma unroll
    for (int r4 = 0; r4 < R; r4 += 4) {
      const float4 w4 = lds4(wr, r4);
      S[r4] = fmaf(w4.x, u, S[r4]);
      S[r4 + 1] = fmaf(w4.y, u, S[r4 + 1]);
      S[r4 + 2] = fmaf(w4.z, u, S[r4 + 2]);
      S[r4 + 3] = fmaf(w4.w, u, S[r4 + 3]);
    }
    // o_t = S_t^T q_t = S_bar^T q_t + (w . q) u_t; before the update: S_{t-1}^T q_t
    if (part == 0) orow[(int64_t)t * H * dv] = __float2bfloat16_rn(pre ? ss : fmaf(s_wq[t], u, ss));
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < R; ++r) sX[(k0 + r) * LDX + j] = S[r];
  __syncthreads();
  {
    const int k = 32 * q4 + lane;
    const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
#pragma unroll
    for (int cb = 0; cb < NV / 64; ++cb) {
      const int col = ch * (NV / 2) + 32 * cb;
      float x[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) x[e] = sX[k * LDX + col + e];
      tmem_st32(tmem_s + lane_base + col, x);
    }
  }
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
  __shared__ __align__(16) float s_lam[2][DK];   // gamma_C / gamma_m per key channel
  __shared__ __align__(16) float s_gm[DK];       // gamma_m per key channel
  __shared__ __align__(16) float s_grp[8][DK];   // per-8-token decay products
  __shared__ __align__(16) float s_Y[2048];
  __shared__ float s_wq[C];                      // w_t . q_t of a chunk on the exact path

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, ch = warp >> 2;
  const int pre = a.pre_read ? 1 : 0;  // o_t before the token's update: strictly causal P, Q+ with r_{t-1}
  const int T = a.T, H = a.H, dv = a.dv;
  // one CTA per (b, h) and slice of NV value columns (columns of the state evolve independently)
  const int nslices = dv / NV;
  const int bh = blockIdx.x / nslices, b = bh / H, h = bh % H;
  const int col0 = (blockIdx.x % nslices) * NV;
  const int nchunks = (T + C - 1) / C;

  if (tid == 0) {
    mbar_init(&bar_qk, 1);
    mbar_init(&bar_v, 1);
    mbar_init(&bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&s_tmem, kTmemCols);
  // rows 0..63 of the [T; P] tile: the 8x8 blocks above the block diagonal of T are zero and the
  // inverse never writes them; set at the start and again after the exact path has used the tile's
  // memory
  auto zero_t_upper = [&]() {
    for (int e = tid; e < 64 * 8; e += kThreads) {
      const int t = e >> 3, x8 = e & 7;
      if (x8 > (t >> 3)) *reinterpret_cast<uint4*>(sm + Ly::TP + canon_chunk(t, x8, 128)) = make_uint4(0, 0, 0, 0);
    }
  };
  zero_t_upper();
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t lane_base = (uint32_t)(32 * q4) << 16;

  // Raw k, q staging (STK, STQ) by TMA feeds the prep, which writes [K+; Q+] into KQ.
  uint8_t* const kq = sm + Ly::KQ;
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
    for (int x = 0; x < NV / 64; ++x)
      tma_load_4d(sm + Ly::STV + x * C * 128, &tm_v, &bar_v, col0 + 64 * x, h, c * C, b);
  };

  // gate values of a chunk for this thread (tokens 8 warp .. + 7, channels 4 lane .. + 3; beta^v for
  // value columns col0 + 4 lane .. + 3), loaded one chunk ahead so that their latency overlaps the
  // previous chunk's products
  // (beta^v too when the value columns are split: with 128 columns the registers are not there)
  constexpr bool kAheadBv = NV < 128;
  float4 g_al[8], g_ws[8], g_dd[8], g_bv[8];
  auto load_gates = [&](int c) {
    const int nvalid = max(0, min(8, min(C, T - c * C) - 8 * warp));
    const int64_t tok0 = ((int64_t)b * T + c * C + (nvalid > 0 ? 8 * warp : 0)) * H + h;
    gate4x8(g_al, a.alpha_p, a.alpha, tok0, H, DK, 4 * lane, nvalid, 1.f);
    gate4x8(g_ws, a.beta_k_p, a.beta_k, tok0, H, DK, 4 * lane, nvalid, 0.f);
    gate4x8(g_dd, a.key_scale_p, a.key_scale, tok0, H, DK, 4 * lane, nvalid, 0.f);
    if (kAheadBv && a.beta_v != DN_GATE_ONE && 4 * lane < NV)
      gate4x8(g_bv, a.beta_v_p, a.beta_v, tok0, H, dv, col0 + 4 * lane, nvalid, 0.f);
  };
  if (nchunks > 0) load_gates(0);

  uint32_t ph_qk = 0, ph_v = 0, ph_mma = 0;
  bool qk_pending = false, v_pending = false, mma_pending = false;
  bool o_pending = false;  // the previous chunk's outputs are still in D1 (stored during this chunk)
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

  // S_m = Diag(lambda_prev * gamma_m) S for rows 32 q4 .. +32, columns of half ch: the state in
  // chunk c's frame, in TMEM (fp32) and as the bf16 operand tile
  auto state_to_frame = [&](int c) {
    const int cur = c & 1, prev = cur ^ 1;
    const int k = 32 * q4 + lane;
    const float mu = (c == 0) ? s_gm[k] : s_lam[prev][k] * s_gm[k];
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
          uint4 pk = make_uint4(pack_bf16(x[8 * q8], x[8 * q8 + 1]), pack_bf16(x[8 * q8 + 2], x[8 * q8 + 3]),
                                pack_bf16(x[8 * q8 + 4], x[8 * q8 + 5]), pack_bf16(x[8 * q8 + 6], x[8 * q8 + 7]));
          *reinterpret_cast<uint4*>(orow + col + 8 * q8) = pk;
        }
      }
    }
  };

  // Gram [K+; Q+] W-^T of the current chunk -> TMEM scratch; thread 0 only
  auto issue_gram = [&]() {
#pragma unroll
    for (int kk = 0; kk < DK; kk += 16) {
      const uint64_t ad = sdesc(smem_u32(kq) + (kk >> 6) * (128 * 128) + (kk & 63) * 2, 16, 1024);
      const uint64_t bd = sdesc(smem_u32(sm + Ly::WHI) + (kk >> 6) * (C * 128) + (kk & 63) * 2, 16, 1024);
      mma_bf16(tmem + Ly::TM_SCR, ad, bd, id_gram, kk > 0);
    }
  };

  for (int c = 0; c < nchunks; ++c) {
    const int t0 = c * C;
    const int n = min(C, T - t0);
    const int cur = c & 1;

    // ---- P0: this chunk's q, k, v have landed
    {
      bool ok = mbar_wait_bounded(&bar_qk, ph_qk, a.wait_ns) && mbar_wait_bounded(&bar_v, ph_v, a.wait_ns);
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      ph_qk ^= 1;
      ph_v ^= 1;
      qk_pending = v_pending = false;
    }

    // ---- the next chunk's gate rows into L2, ahead of their loads at the end of this chunk:
    // lane l of warp tg takes the 128-byte line l % 4 of token 8 tg + l / 4 of every per-channel gate
    if (c + 1 < nchunks) {
      const int j = 8 * warp + (lane >> 2), line = lane & 3;
      if (t0 + C + j < T) {
        const int64_t tok = ((int64_t)b * T + t0 + C + j) * H + h;
        if (a.alpha == DN_GATE_CHANNEL) prefetch_l2(a.alpha_p + tok * DK + 32 * line);
        if (a.beta_k == DN_GATE_CHANNEL) prefetch_l2(a.beta_k_p + tok * DK + 32 * line);
        if (a.key_scale == DN_GATE_CHANNEL) prefetch_l2(a.key_scale_p + tok * DK + 32 * line);
        if (a.beta_v == DN_GATE_CHANNEL && 32 * line < dv) prefetch_l2(a.beta_v_p + tok * dv + 32 * line);
      }
    }

    // ---- P1: decay factors and the operand tiles (or, for a chunk of too strong a decay, the rows the
    // exact path reads)
    bool extreme;
    {
      // per-channel path: thread (g4, tg) owns channels 4g4..4g4+3 of tokens 8tg..8tg+7
      const int g4 = lane, tg = warp, cb0 = 4 * g4;
      if (bv_split && cb0 < NV) {
        // V~ = beta^v (.) v, split hi (in place) / lo
        if (!kAheadBv) {
          const int nvalid = max(0, min(8, n - 8 * tg));
          const int64_t tok0 = ((int64_t)b * T + t0 + (nvalid > 0 ? 8 * tg : 0)) * H + h;
          gate4x8(g_bv, a.beta_v_p, a.beta_v, tok0, H, dv, col0 + cb0, nvalid, 0.f);
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int j = 8 * tg + i;
          const float4 bv = g_bv[i];
          const uint32_t off2 = canon(j, cb0, C);
          const float4 vv = unpack4(*reinterpret_cast<const uint2*>(sm + Ly::STV + off2));
          uint2 hi, lo;
          split4(mul4(vv, bv), hi, lo);
          *reinterpret_cast<uint2*>(sm + Ly::STV + off2) = hi;
          *reinterpret_cast<uint2*>(sm + Ly::VLO + off2) = lo;
        }
      }
      // tokens 8 tg .. 8 tg + 7 of this chunk (gates loaded during the previous chunk)
      float4 al[8], ws[8], dd[8];
      uint2 kr[8], qr[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) al[i] = g_al[i], ws[i] = g_ws[i], dd[i] = g_dd[i];
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
      // every factor of the tensor-core path: r_t (second half) or 1 / r_t (first half), gamma_m and
      // gamma_C / gamma_m; one outside [2^-50, 2^50] sends the chunk to the exact path
      bool ok = true;
#pragma unroll
      for (int i = 0; i < 8; ++i) ok = ok && in_range4(mul4(off, loc[i]));
      if (tg == 0) {
        float4 gm = f4(1.f), lm = f4(1.f);
#pragma unroll
        for (int g = 0; g < 4; ++g) gm = mul4(gm, lds4(&s_grp[g][0], cb0));
#pragma unroll
        for (int g = 4; g < 8; ++g) lm = mul4(lm, lds4(&s_grp[g][0], cb0));
        sts4(s_gm, cb0, gm);
        sts4(&s_lam[cur][0], cb0, lm);
        ok = ok && in_range4(gm) && in_range4(lm);
      }
      extreme = __syncthreads_or(!ok);
      if (extreme) {
        // alpha and w = beta^k d k as fp32 rows [C][DK] over the [K+; Q+] and W- tiles, and w . q
        float* sAl = reinterpret_cast<float*>(sm + Ly::KQ);
        float* sWk = reinterpret_cast<float*>(sm + Ly::WHI);
        float wq[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int j = 8 * tg + i;
          const float4 kk = unpack4(kr[i]), qq = unpack4(qr[i]);
          const float4 wv = mul4(ws[i], kk);
          sts4(sAl, j * DK + cb0, al[i]);
          sts4(sWk, j * DK + cb0, wv);
          wq[i] = wv.x * qq.x + wv.y * qq.y + wv.z * qq.z + wv.w * qq.w;
        }
#pragma unroll
        for (int off2 = 16; off2 > 0; off2 >>= 1)
#pragma unroll
          for (int i = 0; i < 8; ++i) wq[i] += __shfl_xor_sync(0xffffffffu, wq[i], off2);
        if (lane == 0)
#pragma unroll
          for (int i = 0; i < 8; ++i) s_wq[8 * tg + i] = wq[i];
      } else
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
        // Q+ = q (.) r_t; for the pre-update read-out q (.) r_{t-1} = q (.) r_t / alpha_t
        *reinterpret_cast<uint2*>(kq + canon(64 + j, cb0, 128)) = pack4(pre ? mul4(qq, mul4(r, rcp4(al[i]))) : mul4(qq, r));
        uint2 hi, lo;
        split4(mul4(mul4(ws[i], kk), rinv), hi, lo);
        *reinterpret_cast<uint2*>(sm + Ly::WHI + canon(j, cb0, C)) = hi;
        *reinterpret_cast<uint2*>(sm + Ly::WLO + canon(j, cb0, C)) = lo;
      }
    }
    __syncthreads();

    if (extreme) {
      // ---- exact path for this chunk: the previous chunk's outputs first (they are still in D1)
      if (o_pending && q4 >= 2) store_o(c - 1);
      o_pending = false;
      tc_fence_before();
      exact_chunk<DK, NV>(a, sm + Ly::STK, sm + Ly::STQ, sm + Ly::STV, sm + Ly::VLO, bv_split,
                          reinterpret_cast<const float*>(sm + Ly::KQ), reinterpret_cast<const float*>(sm + Ly::WHI),
                          s_wq, reinterpret_cast<float*>(sm + Ly::TP), &s_lam[cur ^ 1][0], tmem + Ly::TM_S, c, n, b,
                          h, bh, col0, tid);
      // the state in tensor memory is now the true state: no pending chunk-end factor
      if (tid < DK) s_lam[cur][tid] = 1.f;
      __syncthreads();  // every thread is done with the transpose buffer over the [T; P] tile
      zero_t_upper();
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      // the staging tiles were read by the exact path: the next chunk's q, k, v may land now
      if (tid == 0 && c + 1 < nchunks) {
        issue_qk(c + 1);
        issue_v(c + 1);
      }
      if (c + 1 < nchunks) qk_pending = v_pending = true;
      load_gates(min(c + 1, nchunks - 1));
      continue;
    }

    // ---- P1.5: (the state is brought into this chunk's frame while the T MMAs run, below)
    fence_proxy_async();
    __syncthreads();

    // ---- P2: Gram [K+; Q+] W-^T -> scratch
    {
      if (tid == 0) {
        // the raw q, k staging was consumed by the prep; prefetch the next chunk's
        if (c + 1 < nchunks) {
          fence_proxy_async();
          issue_qk(c + 1);
        }
        issue_gram();
        mma_commit(&bar_mma);
      }
      if (c + 1 < nchunks) qk_pending = true;
      mma_pending = true;
      bool ok = mbar_wait_bounded(&bar_mma, ph_mma, a.wait_ns);
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
        for (int e4 = 0; e4 < 8; ++e4) {
          float y[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = i0 + 4 * e4 + e;
            y[e] = (i < t) ? x[4 * e4 + e] : 0.f;
          }
          sts4(sL, xi(t, i0 + 4 * e4), make_float4(y[0], y[1], y[2], y[3]));
        }
      } else {
        const int t = 32 * (q4 - 2) + lane;
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          float y[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) y[e] = (i0 + 8 * q8 + e <= t - pre) ? x[8 * q8 + e] : 0.f;
          uint4 pk = make_uint4(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]), pack_bf16(y[4], y[5]),
                                pack_bf16(y[6], y[7]));
          *reinterpret_cast<uint4*>(sm + Ly::TP + canon_chunk(64 + t, i0 / 8 + q8, 128)) = pk;
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    unit_lower_inverse<false, 8>(sL, sT, s_Y, sm + Ly::TP, nullptr, nullptr, nullptr, tid, 0);
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- P4: Wk = [T; P] K+ -> scratch;  U0 = [T; P] V~ -> U0
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < C; kk += 16) {
        const uint64_t ad = sdesc(smem_u32(sm + Ly::TP) + kk * 2, 16, 1024);
        const uint64_t bk = sdesc(smem_u32(kq) + kk * 128, 128 * 128, 1024);
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
    // while those MMAs run: the previous chunk's outputs (D1 rows 64..127) and the state in this
    // chunk's frame (S_acc columns; no overlap with the TMEM the MMAs write)
    if (o_pending && q4 >= 2) store_o(c - 1);
    state_to_frame(c);
    {
      bool ok = mbar_wait_bounded(&bar_mma, ph_mma, a.wait_ns);
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
      bool ok = mbar_wait_bounded(&bar_mma, ph_mma, a.wait_ns);
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
        const uint64_t buh = sdesc(smem_u32(sm + Ly::UHI) + kk * 128, C * 128, 1024);
        const uint64_t bul = sdesc(smem_u32(sm + Ly::ULO) + kk * 128, C * 128, 1024);
        const uint64_t awh = sdesc(smem_u32(sm + Ly::WHI) + kk * 128, C * 128, 1024);
        const uint64_t awl = sdesc(smem_u32(sm + Ly::WLO) + kk * 128, C * 128, 1024);
        mma_bf16(tmem + Ly::TM_S, awh, buh, id_state, 1);
        mma_bf16(tmem + Ly::TM_S, awh, bul, id_state, 1);
        mma_bf16(tmem + Ly::TM_S, awl, buh, id_state, 1);
      }
      mma_commit(&bar_mma);
    }
    mma_pending = true;
    // (unconditional, the last chunk re-reading itself: the arrays are then dead from P1 to here)
    load_gates(min(c + 1, nchunks - 1));
    {
      bool ok = mbar_wait_bounded(&bar_mma, ph_mma, a.wait_ns);
      if (__syncthreads_or(!ok)) {
        failed = true;
        break;
      }
      ph_mma ^= 1;
      mma_pending = false;
      tc_fence_after();
    }

    // ---- P9: (this chunk's outputs are stored during the next chunk's P4 products, or after the loop)
    o_pending = true;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  if (!failed && nchunks > 0) {
    if (o_pending && q4 >= 2) store_o(nchunks - 1);
    // S_T = Diag(gamma_C / gamma_m) S_acc of the last chunk
    const int k = 32 * q4 + lane;
    const float lam = s_lam[(nchunks - 1) & 1][k];
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
    if (v_pending) mbar_wait_bounded(&bar_v, ph_v, kWaitNs);
    if (mma_pending) mbar_wait_bounded(&bar_mma, ph_mma, kWaitNs);
    if (tid == 0) atomicExch(a.status, kDevTimeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ================================================================== split evaluation (workspace)
// With a workspace, the state-independent part of every chunk -- the decay factors, the operand tiles,
// the Gram product and the UT inverse -- runs first for all chunks at once (prep_tc_kernel, one CTA
// per (b, h, chunk)), which writes one record per chunk; chain_tc_kernel then walks each sequence's
// chunks with the state in tensor memory and bulk-loads each record's parts a step ahead of their
// use, so that a step of the chain is the Wk / U0 products, the state products and the U conversion.
// A chunk out of the factors' range is marked in its record, which then carries the exact path's
// operands instead (raw k and q tiles, alpha and w rows, w . q), and the chain evaluates it token by
// token as the fused kernel does.
template <int DK>
struct XRec {
  static constexpr uint32_t KQ = 0;                   // [K+; Q+] bf16 [128][DK]; exact: raw k, raw q [C][DK]
  static constexpr uint32_t TP = KQ + 128 * DK * 2;   // [T; P] bf16 [128][C]
  static constexpr uint32_t WHI = TP + 128 * C * 2;   // W- hi [C][DK]
  static constexpr uint32_t WLO = WHI + C * DK * 2;   // W- lo [C][DK]
  static constexpr uint32_t F = WLO + C * DK * 2;     // gamma_m [DK], gamma_C / gamma_m [DK], w . q [C], flag
  static constexpr uint32_t F_GM = 0, F_LAM = DK * 4, F_WQ = 2 * DK * 4, F_FLAG = 2 * DK * 4 + C * 4;
  static constexpr uint32_t FBYTES = 2048;
  static_assert(F_FLAG + 16 <= FBYTES, "factor block");
  static constexpr uint32_t V = F + FBYTES;           // V~ hi [C][d_v], then lo [C][d_v] (beta^v given)
  __host__ __device__ static constexpr size_t vbytes(int dv, bool bv) { return bv ? (size_t)2 * C * dv * 2 : 0; }
  // alpha rows then w = beta^k d k rows, fp32 [C][DK] each (written for exact chunks only)
  __host__ __device__ static constexpr size_t x_off(int dv, bool bv) { return V + vbytes(dv, bv); }
  __host__ __device__ static constexpr size_t stride(int dv, bool bv) { return x_off(dv, bv) + (size_t)2 * C * DK * 4; }
};

template <int DK>
struct PLayout {
  static constexpr int KQ = 0;                  // [K+; Q+] (the Gram's A), then the inverse's fp32 L and T
  static constexpr int WHI = KQ + 128 * DK * 2;  // W- hi (the Gram's B), then the inverse's scratch
  static constexpr int TP = WHI + C * DK * 2;    // [T; P]; before P3 the per-8-token decay products
  static constexpr int TOTAL = TP + 128 * C * 2;
  static_assert(2 * C * C * 4 <= 128 * DK * 2 && 2048 * 4 <= C * DK * 2 && 8 * DK * 4 <= 128 * C * 2, "overlays");
};

template <int DK>
__global__ void __launch_bounds__(kThreads, 2) prep_tc_kernel(const Args a, uint8_t* ws, int nchunks) {
  using Ly = PLayout<DK>;
  using R = XRec<DK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_mma;
  __shared__ uint32_t s_tmem;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, ch = warp >> 2;
  const int c = blockIdx.x % nchunks, bh = blockIdx.x / nchunks, b = bh / a.H, h = bh % a.H;
  const int T = a.T, H = a.H, dv = a.dv, t0 = c * C, n = min(C, T - t0);
  const int pre = a.pre_read ? 1 : 0;
  const bool bv = a.beta_v != DN_GATE_ONE;
  uint8_t* const rec = ws + ((size_t)bh * nchunks + c) * R::stride(dv, bv);
  float* const rf = reinterpret_cast<float*>(rec + R::F);
  float* const s_grp = reinterpret_cast<float*>(sm + Ly::TP);  // [8][DK]
  if (tid == 0) {
    mbar_init(&bar_mma, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&s_tmem, 64);
  // ---- P1: thread (lane, warp) owns channels 4 lane .. + 3 of tokens 8 warp .. + 7
  const int tg = warp, cb0 = 4 * lane;
  const int nvalid = max(0, min(8, n - 8 * tg));
  const int64_t tok0 = ((int64_t)b * T + t0 + (nvalid > 0 ? 8 * tg : 0)) * H + h;
  // V~ = beta^v (.) v, split hi / lo, for the value columns 4 lane .. + 3 (both paths read it)
  if (bv && cb0 < dv) {
    float4 bvs[8];
    uint2 vr[8];
    gate4x8(bvs, a.beta_v_p, a.beta_v, tok0, H, dv, cb0, nvalid, 0.f);
    const __nv_bfloat16* vp = static_cast<const __nv_bfloat16*>(a.v);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ic = i < nvalid ? i : max(nvalid - 1, 0);
      vr[i] = __ldg(reinterpret_cast<const uint2*>(vp + (tok0 + (int64_t)ic * H) * dv + cb0));
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = 8 * tg + i;
      uint2 hi, lo;
      split4(mul4(unpack4(vr[i]), bvs[i]), hi, lo);
      const uint32_t o2 = canon(j, cb0, C);
      *reinterpret_cast<uint2*>(rec + R::V + o2) = hi;
      *reinterpret_cast<uint2*>(rec + R::V + (uint32_t)(C * dv * 2) + o2) = lo;
    }
  }

  float4 al[8], ws4[8], dd[8];
  uint2 kr[8], qr[8];
  gate4x8(al, a.alpha_p, a.alpha, tok0, H, DK, cb0, nvalid, 1.f);
  gate4x8(ws4, a.beta_k_p, a.beta_k, tok0, H, DK, cb0, nvalid, 0.f);
  gate4x8(dd, a.key_scale_p, a.key_scale, tok0, H, DK, cb0, nvalid, 0.f);
  {
    const __nv_bfloat16* kp = static_cast<const __nv_bfloat16*>(a.k);
    const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(a.q);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ic = i < nvalid ? i : max(nvalid - 1, 0);
      const int64_t off = (tok0 + (int64_t)ic * H) * DK + cb0;
      kr[i] = __ldg(reinterpret_cast<const uint2*>(kp + off));
      qr[i] = __ldg(reinterpret_cast<const uint2*>(qp + off));
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i >= nvalid) kr[i] = qr[i] = make_uint2(0, 0);
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) ws4[i] = mul4(ws4[i], dd[i]);
  // products inside the group: prefix (second half) or exclusive suffix (first half)
  float4 loc[8];
  {
    float4 p = f4(1.f);
    if (tg >= 4) {
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        p = mul4(p, al[i]);
        loc[i] = p;
      }
    } else {
#pragma unroll
      for (int i = 7; i >= 0; --i) {
        loc[i] = p;
        p = mul4(p, al[i]);
      }
    }
    sts4(s_grp + tg * DK, cb0, p);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  float4 off = f4(1.f);
  if (tg >= 4) {
    for (int g = 4; g < tg; ++g) off = mul4(off, lds4(s_grp + g * DK, cb0));
  } else {
    for (int g = tg + 1; g < 4; ++g) off = mul4(off, lds4(s_grp + g * DK, cb0));
  }
  bool ok = true;
#pragma unroll
  for (int i = 0; i < 8; ++i) ok = ok && in_range4(mul4(off, loc[i]));
  if (tg == 0) {
    float4 gm = f4(1.f), lm = f4(1.f);
#pragma unroll
    for (int g = 0; g < 4; ++g) gm = mul4(gm, lds4(s_grp + g * DK, cb0));
#pragma unroll
    for (int g = 4; g < 8; ++g) lm = mul4(lm, lds4(s_grp + g * DK, cb0));
    *reinterpret_cast<float4*>(rf + R::F_GM / 4 + cb0) = gm;  // (the record, global memory)
    *reinterpret_cast<float4*>(rf + R::F_LAM / 4 + cb0) = lm;
    ok = ok && in_range4(gm) && in_range4(lm);
  }
  const bool extreme = __syncthreads_or(!ok);
  if (tid == 0) reinterpret_cast<int*>(rf)[R::F_FLAG / 4] = extreme ? 1 : 0;

  if (extreme) {
    // the exact path's operands: raw k and q tiles, alpha and w rows (fp32), w . q per token
    float* xa = reinterpret_cast<float*>(rec + R::x_off(dv, bv));
    float* xw = xa + C * DK;
    float wq[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int j = 8 * tg + i;
      *reinterpret_cast<uint2*>(rec + R::KQ + canon(j, cb0, C)) = kr[i];
      *reinterpret_cast<uint2*>(rec + R::KQ + C * DK * 2 + canon(j, cb0, C)) = qr[i];
      const float4 kk = unpack4(kr[i]), qq = unpack4(qr[i]);
      const float4 wv = mul4(ws4[i], kk);
      *reinterpret_cast<float4*>(xa + j * DK + cb0) = al[i];
      *reinterpret_cast<float4*>(xw + j * DK + cb0) = wv;
      wq[i] = wv.x * qq.x + wv.y * qq.y + wv.z * qq.z + wv.w * qq.w;
    }
#pragma unroll
    for (int o2 = 16; o2 > 0; o2 >>= 1)
#pragma unroll
      for (int i = 0; i < 8; ++i) wq[i] += __shfl_xor_sync(0xffffffffu, wq[i], o2);
    if (lane == 0)
#pragma unroll
      for (int i = 0; i < 8; ++i) rf[R::F_WQ / 4 + 8 * tg + i] = wq[i];
  } else {
    // K+ and Q+ (shared memory, the Gram's A, and the record), W- hi (shared memory, the Gram's B, and
    // the record), W- lo (the record)
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
      const uint2 kpk = pack4(mul4(kk, r));
      // Q+ = q (.) r_t; for the pre-update read-out q (.) r_{t-1} = q (.) r_t / alpha_t
      const uint2 qpk = pack4(pre ? mul4(qq, mul4(r, rcp4(al[i]))) : mul4(qq, r));
      const uint32_t ok_ = canon(j, cb0, 128), oq = canon(64 + j, cb0, 128);
      *reinterpret_cast<uint2*>(sm + Ly::KQ + ok_) = kpk;
      *reinterpret_cast<uint2*>(sm + Ly::KQ + oq) = qpk;
      *reinterpret_cast<uint2*>(rec + R::KQ + ok_) = kpk;
      *reinterpret_cast<uint2*>(rec + R::KQ + oq) = qpk;
      uint2 hi, lo;
      split4(mul4(mul4(ws4[i], kk), rinv), hi, lo);
      const uint32_t ow = canon(j, cb0, C);
      *reinterpret_cast<uint2*>(sm + Ly::WHI + ow) = hi;
      *reinterpret_cast<uint2*>(rec + R::WHI + ow) = hi;
      *reinterpret_cast<uint2*>(rec + R::WLO + ow) = lo;
    }
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  bool failed = false;
  if (!extreme) {
    // ---- Gram [K+; Q+] W-^T -> tensor memory (64 columns)
    const uint32_t id_gram = idesc_bf16(128, 64, 0, 0);
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < DK; kk += 16) {
        const uint64_t ad = sdesc(smem_u32(sm + Ly::KQ) + (kk >> 6) * (128 * 128) + (kk & 63) * 2, 16, 1024);
        const uint64_t bd = sdesc(smem_u32(sm + Ly::WHI) + (kk >> 6) * (C * 128) + (kk & 63) * 2, 16, 1024);
        mma_bf16(tmem, ad, bd, id_gram, kk > 0);
      }
      mma_commit(&bar_mma);
    }
    // rows 0..63 of [T; P]: the 8x8 blocks above the block diagonal of T are zero (the inverse never
    // writes them; the group products that overlaid the tile are dead)
    for (int e = tid; e < 64 * 8; e += kThreads) {
      const int t = e >> 3, x8 = e & 7;
      if (x8 > (t >> 3)) *reinterpret_cast<uint4*>(sm + Ly::TP + canon_chunk(t, x8, 128)) = make_uint4(0, 0, 0, 0);
    }
    const bool okw = mbar_wait_bounded(&bar_mma, 0, a.wait_ns);
    failed = __syncthreads_or(!okw);
    if (!failed) {
      tc_fence_after();
      // A (strict lower) -> fp32 sL over the [K+; Q+] tile; P (lower incl.) -> bf16 rows 64..127 of [T; P]
      float* sL = reinterpret_cast<float*>(sm + Ly::KQ);
      float* sT = sL + C * C;
      {
        float x[32];
        const uint32_t lane_base = (uint32_t)(32 * q4) << 16;
        tmem_ld32(tmem + lane_base + 32 * ch, x);
        const int i0 = 32 * ch;
        if (q4 < 2) {
          const int t = 32 * q4 + lane;
#pragma unroll
          for (int e4 = 0; e4 < 8; ++e4) {
            float y[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = i0 + 4 * e4 + e;
              y[e] = (i < t) ? x[4 * e4 + e] : 0.f;
            }
            sts4(sL, xi(t, i0 + 4 * e4), make_float4(y[0], y[1], y[2], y[3]));
          }
        } else {
          const int t = 32 * (q4 - 2) + lane;
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = (i0 + 8 * q8 + e <= t - pre) ? x[8 * q8 + e] : 0.f;
            uint4 pk = make_uint4(pack_bf16(y[0], y[1]), pack_bf16(y[2], y[3]), pack_bf16(y[4], y[5]),
                                  pack_bf16(y[6], y[7]));
            *reinterpret_cast<uint4*>(sm + Ly::TP + canon_chunk(64 + t, i0 / 8 + q8, 128)) = pk;
          }
        }
      }
      tc_fence_before();
      __syncthreads();
      unit_lower_inverse<false, 8>(sL, sT, reinterpret_cast<float*>(sm + Ly::WHI), sm + Ly::TP, nullptr, nullptr,
                                   nullptr, tid, 0);
      fence_proxy_async();
      __syncthreads();
      // [T; P] -> the record
      if (tid == 0) {
        bulk_store(rec + R::TP, sm + Ly::TP, 128 * C * 2);
        bulk_commit();
      }
    } else {
      mbar_wait_bounded(&bar_mma, 0, kWaitNs);  // drain (bounded)
      if (tid == 0) atomicExch(a.status, kDevTimeout);
    }
  }
  if (tid == 0) bulk_wait_all();  // the record's copies are complete before the block leaves
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 64);
}

template <int DK, int NV>
struct XLayout {
  static constexpr int KQ = 0;                   // [K+; Q+] of the record, then [Wk; Q+]; exact: raw k, raw q
  static constexpr int TP0 = KQ + 128 * DK * 2;  // [T; P] of even chunks
  static constexpr int TP1 = TP0 + 128 * C * 2;  // [T; P] of odd chunks
  static constexpr int WHI = TP1 + 128 * C * 2;  // W- hi
  static constexpr int WLO = WHI + C * DK * 2;   // W- lo
  static constexpr int STV = WLO + C * DK * 2;   // V~ hi (the record) or raw v (TMA)
  static constexpr int VLO = STV + C * NV * 2;   // V~ lo
  static constexpr int UHI = VLO + C * NV * 2;   // U hi
  static constexpr int ULO = UHI + C * NV * 2;   // U lo
  static constexpr int SM = ULO + C * NV * 2;    // S_m bf16 [DK][NV]
  static constexpr int F0 = SM + DK * NV * 2 + 1024;  // factor blocks of even / odd chunks
  static constexpr int F1 = F0 + 2048;
  static constexpr int TOTAL = F1 + 2048;
  static constexpr int TM_S = 0, TM_D1 = NV, TM_U0 = 2 * NV, TM_SCR = 3 * NV;
  static_assert(TM_SCR + DK <= (int)kTmemCols, "tensor memory budget");
  // the exact path's fp32 state transpose (DK x (NV + 1)) overlays the U and S_m tiles
  static_assert(UHI + DK * (NV + 1) * 4 <= F0, "transpose buffer of the exact path");
};

template <int DK, int NV>
__global__ void __launch_bounds__(kThreads, 1)
    chain_tc_kernel(const __grid_constant__ CUtensorMap tm_v, const Args a, const uint8_t* ws) {
  using Ly = XLayout<DK, NV>;
  using R = XRec<DK>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_kq, bar_tp[2], bar_w, bar_v, bar_mma;
  __shared__ uint32_t s_tmem;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3, ch = warp >> 2;
  const int T = a.T, H = a.H, dv = a.dv;
  const int nslices = dv / NV;
  const int bh = blockIdx.x / nslices, b = bh / H, h = bh % H;
  const int col0 = (blockIdx.x % nslices) * NV;
  const int nchunks = (T + C - 1) / C;
  const bool bv = a.beta_v != DN_GATE_ONE;
  const size_t stride = R::stride(dv, bv);
  auto rec = [&](int c) { return ws + ((size_t)bh * nchunks + c) * stride; };
  auto fblk = [&](int c) { return reinterpret_cast<float*>(sm + ((c & 1) ? Ly::F1 : Ly::F0)); };

  if (tid == 0) {
    mbar_init(&bar_kq, 1);
    mbar_init(&bar_tp[0], 1);
    mbar_init(&bar_tp[1], 1);
    mbar_init(&bar_w, 1);
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
  uint8_t* const kq = sm + Ly::KQ;
  auto tp_of = [&](int c) { return sm + ((c & 1) ? Ly::TP1 : Ly::TP0); };

  // record parts (thread 0): [K+; Q+] and the factors; [T; P]; W- hi and lo; V~ (or raw v)
  auto issue_kq = [&](int c) {
    mbar_expect_tx(&bar_kq, 128 * DK * 2 + R::FBYTES);
    bulk_load(kq, rec(c) + R::KQ, 128 * DK * 2, &bar_kq);
    bulk_load(fblk(c), rec(c) + R::F, R::FBYTES, &bar_kq);
  };
  auto issue_tp = [&](int c) {
    mbar_expect_tx(&bar_tp[c & 1], 128 * C * 2);
    bulk_load(tp_of(c), rec(c) + R::TP, 128 * C * 2, &bar_tp[c & 1]);
  };
  auto issue_w = [&](int c) {
    mbar_expect_tx(&bar_w, 2 * C * DK * 2);
    bulk_load(sm + Ly::WHI, rec(c) + R::WHI, C * DK * 2, &bar_w);
    bulk_load(sm + Ly::WLO, rec(c) + R::WLO, C * DK * 2, &bar_w);
  };
  auto issue_v = [&](int c) {
    if (bv) {
      mbar_expect_tx(&bar_v, 2 * C * NV * 2);
      bulk_load(sm + Ly::STV, rec(c) + R::V + (col0 / 64) * (C * 128), C * NV * 2, &bar_v);
      bulk_load(sm + Ly::VLO, rec(c) + R::V + C * dv * 2 + (col0 / 64) * (C * 128), C * NV * 2, &bar_v);
    } else {
      mbar_expect_tx(&bar_v, (uint32_t)C * NV * 2);
#pragma unroll
      for (int x = 0; x < NV / 64; ++x)
        tma_load_4d(sm + Ly::STV + x * C * 128, &tm_v, &bar_v, col0 + 64 * x, h, c * C, b);
    }
  };

  uint32_t ph_kq = 0, ph_tp[2] = {0, 0}, ph_w = 0, ph_v = 0, ph_mma = 0;
  bool kq_p = false, tp_p[2] = {false, false}, w_p = false, v_p = false, mma_p = false;
  bool o_pending = false, failed = false;
  if (nchunks > 0) {
    if (tid == 0) {
      issue_kq(0);
      issue_tp(0);
      issue_w(0);
      issue_v(0);
      if (nchunks > 1) issue_tp(1);
    }
    kq_p = w_p = v_p = tp_p[0] = true;
    tp_p[1] = nchunks > 1;
  }

  const uint32_t id_wk = idesc_bf16(128, DK, 0, 1);
  const uint32_t id_nv = idesc_bf16(128, NV, 0, 1);
  const uint32_t id_state = idesc_bf16(128, NV, 1, 1);

  // S_m = Diag(lambda_prev gamma_m) S (rows 32 q4 .. + 31, columns of half ch): the state in chunk c's
  // frame, in tensor memory (fp32) and as the bf16 operand tile
  auto state_to_frame = [&](int c) {
    const int k = 32 * q4 + lane;
    const float gm = fblk(c)[R::F_GM / 4 + k];
    const float mu = (c == 0) ? gm : fblk(c - 1)[R::F_LAM / 4 + k] * gm;
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
  // o rows of chunk c from rows 64..127 of D1 (quadrants 2 and 3, columns of half ch)
  auto store_o = [&](int c) {
    const int t = 32 * (q4 - 2) + lane, t0c = c * C, nc = min(C, T - t0c);
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
          uint4 pk = make_uint4(pack_bf16(x[8 * q8], x[8 * q8 + 1]), pack_bf16(x[8 * q8 + 2], x[8 * q8 + 3]),
                                pack_bf16(x[8 * q8 + 4], x[8 * q8 + 5]), pack_bf16(x[8 * q8 + 6], x[8 * q8 + 7]));
          *reinterpret_cast<uint4*>(orow + col + 8 * q8) = pk;
        }
      }
    }
  };
  // a bounded wait by every thread; false (for all) if any thread's wait ran out
  auto wait_all = [&](uint64_t* bar, uint32_t ph) -> bool {
    return !__syncthreads_or(!mbar_wait_bounded(bar, ph, a.wait_ns));
  };

  for (int c = 0; c < nchunks; ++c) {
    const int n = min(C, T - c * C);
    // ---- this chunk's [K+; Q+] (or raw k, q) and factors
    if (!wait_all(&bar_kq, ph_kq)) {
      failed = true;
      break;
    }
    ph_kq ^= 1;
    kq_p = false;
    const float* fc = fblk(c);
    const bool extreme = reinterpret_cast<const int*>(fc)[R::F_FLAG / 4] != 0;
    // the next chunk's [T; P] into the buffer chunk c - 1 used (its products are done); the next
    // record's [K+; Q+] into L2 (it is loaded once this chunk's D1 product has read the tile)
    if (c + 1 < nchunks) {
      if (tid == 0) {
        if (c >= 1) issue_tp(c + 1);
        bulk_prefetch(rec(c + 1) + R::KQ, 128 * DK * 2);
        bulk_prefetch(rec(c + 1) + R::F, R::FBYTES);
      }
      tp_p[(c + 1) & 1] = true;
    }

    if (extreme) {
      // V~ (read by the exact path); [T; P] and W- of the record are not used, their loads are awaited
      if (!wait_all(&bar_v, ph_v) || !wait_all(&bar_tp[c & 1], ph_tp[c & 1]) || !wait_all(&bar_w, ph_w)) {
        failed = true;
        break;
      }
      ph_v ^= 1;
      ph_w ^= 1;
      ph_tp[c & 1] ^= 1;
      v_p = w_p = tp_p[c & 1] = false;
      if (o_pending && q4 >= 2) store_o(c - 1);
      o_pending = false;
      tc_fence_before();
      const float* xa = reinterpret_cast<const float*>(rec(c) + R::x_off(dv, bv));
      exact_chunk<DK, NV>(a, kq, kq + C * DK * 2, sm + Ly::STV, sm + Ly::VLO, bv, xa, xa + C * DK, fc + R::F_WQ / 4,
                          reinterpret_cast<float*>(sm + Ly::UHI), fblk(c - 1) + R::F_LAM / 4, tmem + Ly::TM_S, c, n, b,
                          h, bh, col0, tid);
      // the state in tensor memory is now the true state: no pending chunk-end factor
      if (tid < DK) fblk(c)[R::F_LAM / 4 + tid] = 1.f;
      fence_proxy_async();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (c + 1 < nchunks) {
        if (tid == 0) {
          issue_kq(c + 1);
          issue_w(c + 1);
          issue_v(c + 1);
        }
        kq_p = w_p = v_p = true;
      }
      continue;
    }

    // ---- Wk = [T; P] K+ -> scratch;  U0 = [T; P] V~ -> U0
    if (!wait_all(&bar_tp[c & 1], ph_tp[c & 1]) || !wait_all(&bar_v, ph_v)) {
      failed = true;
      break;
    }
    ph_v ^= 1;
    ph_tp[c & 1] ^= 1;
    tp_p[c & 1] = v_p = false;
    if (tid == 0) {
      const uint32_t tpa = smem_u32(tp_of(c));
#pragma unroll
      for (int kk = 0; kk < C; kk += 16) {
        const uint64_t ad = sdesc(tpa + kk * 2, 16, 1024);
        const uint64_t bk = sdesc(smem_u32(kq) + kk * 128, 128 * 128, 1024);
        mma_bf16(tmem + Ly::TM_SCR, ad, bk, id_wk, kk > 0);
      }
#pragma unroll
      for (int kk = 0; kk < C; kk += 16) {
        const uint64_t ad = sdesc(tpa + kk * 2, 16, 1024);
        const uint64_t bd = sdesc(smem_u32(sm + Ly::STV) + kk * 128, C * 128, 1024);
        mma_bf16(tmem + Ly::TM_U0, ad, bd, id_nv, kk > 0);
      }
      if (bv) {
#pragma unroll
        for (int kk = 0; kk < C; kk += 16) {
          const uint64_t ad = sdesc(tpa + kk * 2, 16, 1024);
          const uint64_t bd = sdesc(smem_u32(sm + Ly::VLO) + kk * 128, C * 128, 1024);
          mma_bf16(tmem + Ly::TM_U0, ad, bd, id_nv, 1);
        }
      }
      mma_commit(&bar_mma);
    }
    mma_p = true;
    // while those run: the previous chunk's outputs and the state in this chunk's frame
    if (o_pending && q4 >= 2) store_o(c - 1);
    state_to_frame(c);
    if (!wait_all(&bar_mma, ph_mma)) {
      failed = true;
      break;
    }
    ph_mma ^= 1;
    mma_p = false;
    tc_fence_after();
    if (c + 1 < nchunks) {
      if (tid == 0) issue_v(c + 1);
      v_p = true;
    }

    // ---- Wk -> bf16 into rows 0..63 of the [K+; Q+] tile (K+ is dead now)
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

    // ---- D1 = [Wk; Q+] S_m
    if (tid == 0) {
#pragma unroll
      for (int kk = 0; kk < DK; kk += 16) {
        const uint64_t ad = sdesc(smem_u32(kq) + (kk >> 6) * (128 * 128) + (kk & 63) * 2, 16, 1024);
        const uint64_t bd = sdesc(smem_u32(sm + Ly::SM) + kk * 128, DK * 128, 1024);
        mma_bf16(tmem + Ly::TM_D1, ad, bd, id_nv, kk > 0);
      }
      mma_commit(&bar_mma);
    }
    mma_p = true;
    if (!wait_all(&bar_mma, ph_mma)) {
      failed = true;
      break;
    }
    ph_mma ^= 1;
    mma_p = false;
    tc_fence_after();
    // the [Wk; Q+] tile and the factor block of chunk c - 1 are free: the next record's tile and factors
    if (c + 1 < nchunks) {
      if (tid == 0) issue_kq(c + 1);
      kq_p = true;
    }

    // ---- U = U0 - Wk S_m -> hi / lo tiles
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
          const uint32_t o2 = canon_chunk(t, col / 8 + q8, C);
          *reinterpret_cast<uint4*>(sm + Ly::UHI + o2) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(sm + Ly::ULO + o2) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    // ---- O = Q+ S_m + P U (rows 64..127 of D1); S_acc += W-^T U (split)
    if (!wait_all(&bar_w, ph_w)) {
      failed = true;
      break;
    }
    ph_w ^= 1;
    w_p = false;
    if (tid == 0) {
      const uint32_t tpa = smem_u32(tp_of(c));
#pragma unroll
      for (int kk = 0; kk < C; kk += 16) {
        const uint64_t ad = sdesc(tpa + kk * 2, 16, 1024);
        const uint64_t bd = sdesc(smem_u32(sm + Ly::UHI) + kk * 128, C * 128, 1024);
        mma_bf16(tmem + Ly::TM_D1, ad, bd, id_nv, 1);
      }
#pragma unroll
      for (int kk = 0; kk < C; kk += 16) {
        const uint64_t buh = sdesc(smem_u32(sm + Ly::UHI) + kk * 128, C * 128, 1024);
        const uint64_t bul = sdesc(smem_u32(sm + Ly::ULO) + kk * 128, C * 128, 1024);
        const uint64_t awh = sdesc(smem_u32(sm + Ly::WHI) + kk * 128, C * 128, 1024);
        const uint64_t awl = sdesc(smem_u32(sm + Ly::WLO) + kk * 128, C * 128, 1024);
        mma_bf16(tmem + Ly::TM_S, awh, buh, id_state, 1);
        mma_bf16(tmem + Ly::TM_S, awh, bul, id_state, 1);
        mma_bf16(tmem + Ly::TM_S, awl, buh, id_state, 1);
      }
      mma_commit(&bar_mma);
    }
    mma_p = true;
    if (!wait_all(&bar_mma, ph_mma)) {
      failed = true;
      break;
    }
    ph_mma ^= 1;
    mma_p = false;
    tc_fence_after();
    // W- hi and lo are free: the next record's
    if (c + 1 < nchunks) {
      if (tid == 0) issue_w(c + 1);
      w_p = true;
    }
    // (this chunk's outputs are stored during the next chunk's first products, or after the loop)
    o_pending = true;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
  }

  if (!failed && nchunks > 0) {
    if (o_pending && q4 >= 2) store_o(nchunks - 1);
    // S_T = Diag(gamma_C / gamma_m) S_acc of the last chunk
    const int k = 32 * q4 + lane;
    const float lam = fblk(nchunks - 1)[R::F_LAM / 4 + k];
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
    if (kq_p) mbar_wait_bounded(&bar_kq, ph_kq, kWaitNs);
    for (int i = 0; i < 2; ++i)
      if (tp_p[i]) mbar_wait_bounded(&bar_tp[i], ph_tp[i], kWaitNs);
    if (w_p) mbar_wait_bounded(&bar_w, ph_w, kWaitNs);
    if (v_p) mbar_wait_bounded(&bar_v, ph_v, kWaitNs);
    if (mma_p) mbar_wait_bounded(&bar_mma, ph_mma, kWaitNs);
    if (tid == 0) atomicExch(a.status, kDevTimeout);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- host side
template <int DK, int NV>
cudaError_t launch_impl(const Args& a, cudaStream_t s) {
  using Ly = Layout<DK, NV>;
  const int smem = Ly::TOTAL + 1024;
  // per call: the attribute is per device, and the call is cheap next to the kernel
  cudaError_t e =
      cudaFuncSetAttribute(chunk_tc_kernel<DK, NV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  CUtensorMap mq, mk, mv;
  if (!make_bthd_map(&mq, a.q, DK, a.H, a.T, a.B, C) || !make_bthd_map(&mk, a.k, DK, a.H, a.T, a.B, C) ||
      !make_bthd_map(&mv, a.v, a.dv, a.H, a.T, a.B, C))
    return cudaErrorInvalidValue;
  chunk_tc_kernel<DK, NV><<<a.B * a.H * (a.dv / NV), kThreads, smem, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

// Few sequences: twice their count still fits the SMs (148 when no device can be queried)
bool few_sequences(const Args& a) {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return (int64_t)a.B * a.H * 2 <= sms;
}

template <int NV>
cudaError_t launch_split_impl(const Args& a, uint8_t* ws, cudaStream_t s) {
  const int nc = (a.T + C - 1) / C;
  const int psmem = PLayout<128>::TOTAL + 1024, csmem = XLayout<128, NV>::TOTAL + 1024;
  cudaError_t e = cudaFuncSetAttribute(prep_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, psmem);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(chain_tc_kernel<128, NV>, cudaFuncAttributeMaxDynamicSharedMemorySize, csmem);
  if (e != cudaSuccess) return e;
  CUtensorMap mv;
  if (!make_bthd_map(&mv, a.v, a.dv, a.H, a.T, a.B, C)) return cudaErrorInvalidValue;
  prep_tc_kernel<128><<<(unsigned)((int64_t)a.B * a.H * nc), kThreads, psmem, s>>>(a, ws, nc);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  chain_tc_kernel<128, NV><<<a.B * a.H * (a.dv / NV), kThreads, csmem, s>>>(mv, a, ws);
  return cudaGetLastError();
}

}  // namespace

// The split evaluation is taken when few sequences leave SMs idle (B H 2 <= SMs, the fused kernel's
// column split): then the chunk-parallel prep runs on every SM and the chains only walk. With more
// sequences the fused kernel keeps every SM busy already and the prep's extra work does not pay
// (measured: kda, 128 sequences, 1.36 ms split against 1.34 ms fused).
bool split_tc_supported(const Args& a) {
  return chunk_tc_supported(a) && !per_token_tc(a) && few_sequences(a) &&
         (int64_t)a.B * a.H * ((a.T + C - 1) / C) < ((int64_t)1 << 31);  // (one prep CTA per chunk)
}

size_t split_tc_workspace_bytes(const Args& a) {
  return (size_t)a.B * a.H * ((a.T + C - 1) / C) * XRec<128>::stride(a.dv, a.beta_v != DN_GATE_ONE);
}

cudaError_t launch_split_tc(const Args& a, void* workspace, cudaStream_t s) {
  return launch_split_impl<64>(a, static_cast<uint8_t*>(workspace), s);  // 64 value columns per chain
}

bool chunk_tc_supported(const Args& a) {
  return a.io_bf16 && a.dk == 128 && (a.dv == 128 || a.dv == 64) && a.chunk == C && a.T > 0;
}

bool per_token_tc(const Args& a) {
  return chunk_tc_supported(a) && a.alpha != DN_GATE_CHANNEL && a.beta_k != DN_GATE_CHANNEL &&
         a.beta_v != DN_GATE_CHANNEL && a.key_scale != DN_GATE_CHANNEL;
}

cudaError_t launch_chunk_tc(const Args& a, cudaStream_t s) {
  // per-token gates only -> the pipelined raw-tile kernel (dn_chunk_sc.cu)
  const bool sc = a.alpha != DN_GATE_CHANNEL && a.beta_k != DN_GATE_CHANNEL && a.beta_v != DN_GATE_CHANNEL &&
                  a.key_scale != DN_GATE_CHANNEL;
  if (sc) return launch_chunk_sc(a, s);
  // few sequences: split the 128 value columns into two 64-column CTAs when that still fits in one
  // wave (each CTA repeats the column-independent prep, Gram and inverse)
  if (a.dv == 128 && !few_sequences(a)) return launch_impl<128, 128>(a, s);
  return launch_impl<128, 64>(a, s);
}

}  // namespace dn
