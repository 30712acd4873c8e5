// Tensor-core chunked prefill for per-token gates (GDN: scalar alpha, beta^k, beta^v, d; bf16 io,
// d_k = 128, d_v in {64, 128}) for sm_100a, with the chunk-local UT transform pipelined one chunk
// ahead of the state recurrence.
//
// One CTA owns one (b, h) sequence (and a slice of NV value columns) and walks its chunks of
// C = 64 tokens. Every gate is a scalar per token, so every decay factor is a scalar per token (or
// per token pair) and moves onto the small C x C matrices or onto rows of the raw tiles. With
// gamma_t = prod_{s <= t} alpha_s (from the chunk start, token t included), S the state entering
// the chunk and w_t = beta^k_t d_t k_t:
//
//   A_ti = (gamma_t / gamma_i) beta_i d_i (k_t . k_i)  (i < t),   T = (I + A)^{-1}
//   Wk = (T Diag(gamma)) K,   U0 = (T Diag(beta^v)) V,   U = U0 - Wk S
//   o_t = gamma_t S^T q_t + sum_{i <= t} (gamma_t / gamma_i) (q_t . w_i) u_i
//   S'  = gamma_C S + sum_i (gamma_C / gamma_i) w_i u_i^T
//
// (the chunk-parallel WY / UT evaluation of the gated delta rule: FG2-GDN page, sections 2.A and
// 3 item 2). Every factor above is a ratio of decay products, at most 1 for gates in (0, 1], and
// the products themselves are carried as mantissa and exponent (split_pow2), so no gate strength
// can overflow or underflow an intermediate: small factors round to zero, as the recurrence does.
// The output and the state update read one residual tile between them, U'_i = c_i u_i, and the
// powers of two that separate their two scalings move, exactly, onto rows of the raw tiles:
//
//   gamma_t = rho_t 2^{e_t},  gamma_C / gamma_i = mu_i 2^{n_i}   (rho, mu in [0.5, 1))
//   c_i = beta_i d_i mu_i,   K'_i = 2^{n_i} k_i,   Q'_t = 2^{e_t} q_t
//   P'_ti = (q_t . k_i) 2^{e_t - e_i} / (rho_i mu_i)   (i <= t)
//   o_t = rho_t (Q' S + P' U')_t,    S' = gamma_C S + K'^T U'
//
// (the read-out before the update uses gamma_{t-1} in place of gamma_t and i < t).
//
// Only the last lines depend on the state. Two warp groups therefore work one chunk apart:
//  * the state group (warps 0..7) runs the state chain of chunk c: the Wk and U0 products, the
//    state framing, D1 = [Wk; Q'] S, U', the O and state-update products and the o store;
//  * the transform group (warps 8..15) meanwhile prepares chunk c + 1: its decay factors, A and P'
//    from the Gram product [K; Q] K^T (issued by the state group right after chunk c's Wk / U0
//    products), and the inverse T, emitted as the bf16 operand tiles T Diag(gamma) and
//    T Diag(beta^v).
// Hand-offs are mbarriers: the transform group arrives on `tready` once chunk c + 1's tiles are in
// shared memory; the Gram of chunk c + 1 is committed after chunk c's Wk / U0 products, so its
// completion also tells the transform group that the T tiles of chunk c are no longer read.
// P' is double-buffered by chunk parity; the per-token factors are kept for four chunks.
//
// Precision: bf16 operands, fp32 accumulation; U' is split hi + lo for the state update (K' is raw k
// times a power of two, exact in bf16); T is inverted in fp32 (TF32 block merges) and rounded to
// bf16 once.
//
// Tensor memory (512 columns): S_acc | D1 | U0 | (Wk, d_v = 64 only) | Gram; Wk shares D1's columns
// when d_v = 128 (D1 is written only after Wk has been read).
// Every mbarrier wait is bounded in time; on expiry both groups leave their loops, the state group
// drains what it issued (bounded), the CTA sets the status word and frees its tensor memory.
#include "dn_common.cuh"
#include "dn_sc_factors.cuh"
#include "dn_tc_ptx.cuh"
#include "dn_ut_inverse.cuh"

namespace dn {
namespace {

using namespace tc;
using namespace ut;

constexpr int C = 64;
constexpr int DK = 128;
constexpr int kStateThreads = 256;   // warps 0..7
constexpr int kXformThreads = 256;   // warps 8..15
constexpr int kThreads = kStateThreads + kXformThreads;
constexpr int kBarState = 1, kBarXform = 2;   // hardware barriers of the two groups (0 = whole CTA)
constexpr uint32_t kTmemCols = 512;
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s: the bound of the drain waits after a failure

template <int NV>
struct ScLayout {
  static constexpr int STK = 0;                   // raw k [C][DK] (TMA), rows scaled to K': state-update operand
  static constexpr int STQ = STK + C * DK * 2;    // T Diag(beta^v) [128][C]: rows 0..63 bf16 hi, 64..127 lo (or 0)
  static constexpr int STV = STQ + 128 * C * 2;   // raw v [C][NV] (TMA)
  static constexpr int KQ0 = STV + C * NV * 2;    // [K; Q] (TMA), then [Wk; Q]: even chunks
  static constexpr int KQ1 = KQ0 + 128 * DK * 2;  //                               odd chunks
  static constexpr int TP = KQ1 + 128 * DK * 2;   // T Diag(gamma) | P' (even chunks) | P' (odd chunks), 64 rows each
  static constexpr int SMU = TP + 3 * C * C * 2;  // S bf16 [DK][NV]; after D1: U' hi, U' lo [C][NV]
  static constexpr int SMU_BYTES = (DK * NV * 2 > 2 * C * NV * 2) ? DK * NV * 2 : 2 * C * NV * 2;
  static constexpr int INV = SMU + SMU_BYTES;     // fp32 L and T of the inverse (64 x 64 each)
  static constexpr int TOTAL = INV + 2 * C * C * 4;
  static constexpr int TM_S = 0, TM_D1 = NV, TM_U0 = 2 * NV;
  static constexpr int TM_WK = (NV == 128) ? TM_D1 : 3 * NV;
  static constexpr int TM_GR = (NV == 128) ? 3 * NV : 3 * NV + DK;
  static_assert(TM_GR + 64 <= (int)kTmemCols, "tensor memory budget");
  // dynamic (plus 1 KB for alignment) and about 20 KB of static shared memory per CTA
  static_assert(TOTAL + 1024 + 20 * 1024 <= 227 * 1024, "shared memory budget");
};

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int NV>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_sc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const Args a) {
  using Ly = ScLayout<NV>;
  constexpr int NCB = NV / 64;  // 32-column TMEM loads per thread per NV-wide tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t bar_qk[2], bar_k, bar_v, bar_mma, bar_gram, bar_tready, bar_drain;
  __shared__ uint32_t s_tmem;
  __shared__ __align__(16) float s_Y[2048];  // inverse scratch
  // per-token factors by chunk index mod 4 (dn_sc_factors.cuh)
  __shared__ scf::Factors s_f[4];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int q4 = warp & 3;  // TMEM lane quadrant this warp may access
  const int pre = a.pre_read ? 1 : 0;  // o_t before the token's update: strictly causal P', gamma_{t-1}
  // a per-token beta^v is folded into T Diag(beta^v), kept as bf16 hi + lo (U0 = T~_hi V + T~_lo V)
  const bool bv_split = a.beta_v != DN_GATE_ONE;
  const int T = a.T, H = a.H, dv = a.dv;
  const int nslices = dv / NV;
  const int bh = blockIdx.x / nslices, b = bh / H, h = bh % H;
  const int col0 = (blockIdx.x % nslices) * NV;
  const int nchunks = (T + C - 1) / C;

  if (tid == 0) {
    mbar_init(&bar_qk[0], 1);
    mbar_init(&bar_qk[1], 1);
    mbar_init(&bar_k, 1);
    mbar_init(&bar_v, 1);
    mbar_init(&bar_mma, 1);
    mbar_init(&bar_gram, 1);
    mbar_init(&bar_tready, 1);
    mbar_init(&bar_drain, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&s_tmem, kTmemCols);
  // rows 0..63 of the T Diag(r) and T Diag(beta^v) tiles: the 8x8 blocks above the block diagonal
  // stay zero (the inverse never writes them); rows 64..127 of the T Diag(beta^v) tile are zero
  for (int e = tid; e < 64 * 8; e += kThreads) {
    const int t = e >> 3, x8 = e & 7;
    if (x8 > (t >> 3)) {
      *reinterpret_cast<uint4*>(sm + Ly::TP + canon_chunk(t, x8, 64)) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(sm + Ly::STQ + canon_chunk(t, x8, 128)) = make_uint4(0, 0, 0, 0);
    }
  }
  for (int i = tid; i < 64 * 128 / 16; i += kThreads)
    reinterpret_cast<uint4*>(sm + Ly::STQ + 64 * 128)[i] = make_uint4(0, 0, 0, 0);
  // the inverse's fp32 scratch (L, T): the blocks of T above the diagonal stay zero
  for (int i = tid; i < 2 * C * C * 4 / 16; i += kThreads)
    reinterpret_cast<uint4*>(sm + Ly::INV)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t lane_base = (uint32_t)(32 * q4) << 16;

  auto kq_buf = [&](int c) -> uint8_t* { return sm + ((c & 1) ? Ly::KQ1 : Ly::KQ0); };
  // [K; Q] tile of chunk c (one thread)
  auto issue_qk = [&](int c) {
    uint64_t* bar = &bar_qk[c & 1];
    uint8_t* kq = kq_buf(c);
    mbar_expect_tx(bar, 2u * C * DK * 2);
#pragma unroll
    for (int x = 0; x < DK / 64; ++x) {
      tma_load_4d(kq + x * 128 * 128, &tm_k, bar, 64 * x, h, c * C, b);
      tma_load_4d(kq + x * 128 * 128 + 64 * 128, &tm_q, bar, 64 * x, h, c * C, b);
    }
  };
  auto issue_k = [&](int c) {
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
  // Gram [K; Q] K^T of chunk c -> TM_GR (one thread)
  auto issue_gram = [&](int c) {
    const uint8_t* kq = kq_buf(c);
    const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
    for (int kk = 0; kk < DK; kk += 16) {
      const uint64_t d = sdesc(smem_u32(kq) + (kk >> 6) * (128 * 128) + (kk & 63) * 2, 16, 1024);
      mma_bf16(tmem + Ly::TM_GR, d, d, id, kk > 0);
    }
  };

  bool failed = false;
  if (warp < 8) {
    // ======================================================= state group
    const int ch = warp >> 2;  // column half of the TMEM tiles this warp covers
    uint32_t ph_qk[2] = {0, 0}, ph_k = 0, ph_v = 0, ph_mma = 0, ph_tr = 0;
    bool pend_qk[2] = {false, false}, pend_k = false, pend_v = false;
    bool ok0 = true;  // thread 0: its own waits (the [K; Q] tiles before a Gram) succeeded
    if (tid == 0 && nchunks > 0) {
      issue_qk(0);
      pend_qk[0] = true;
      if (nchunks > 1) {
        issue_qk(1);
        pend_qk[1] = true;
      }
      issue_k(0);
      issue_v(0);
      pend_k = pend_v = true;
      if (mbar_wait_bounded(&bar_qk[0], ph_qk[0], a.wait_ns)) {
        ph_qk[0] ^= 1;
        pend_qk[0] = false;
        tc_fence_after();
        issue_gram(0);
        mma_commit(&bar_gram);
      } else {
        ok0 = false;
      }
    }
    const uint32_t id_wk = idesc_bf16(128, DK, 0, 1);
    const uint32_t id_nv = idesc_bf16(128, NV, 0, 1);
    const uint32_t id_state = idesc_bf16(128, NV, 1, 1);

    for (int c = 0; c < nchunks; ++c) {
      const int t0 = c * C, cur = c & 3;
      uint8_t* const kq = kq_buf(c);

      // ---- M0: chunk c's T tiles, P and factors are ready; its v tile has landed
      {
        const bool ok = ok0 && mbar_wait_bounded(&bar_tready, ph_tr, a.wait_ns) &&
                        mbar_wait_bounded(&bar_v, ph_v, a.wait_ns);
        if (group_or(kBarState, kStateThreads, !ok)) {
          failed = true;
          break;
        }
        ph_tr ^= 1;
        ph_v ^= 1;
        pend_v = false;
        tc_fence_after();
      }

      // ---- M1: Wk = (T Diag gamma) K -> TM_WK, U0 = (T Diag beta^v) V -> TM_U0; then chunk c + 1's Gram
      // (its completion also tells the transform group that chunk c's T tiles are no longer read)
      if (tid == 0) {
#pragma unroll
        for (int kk = 0; kk < C; kk += 16) {
          const uint64_t ad = sdesc(smem_u32(sm + Ly::TP) + kk * 2, 16, 1024);
          const uint64_t bk = sdesc(smem_u32(kq) + kk * 128, 128 * 128, 1024);
          mma_bf16(tmem + Ly::TM_WK, ad, bk, id_wk, kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < C; kk += 16) {
          const uint64_t ad = sdesc(smem_u32(sm + Ly::STQ) + kk * 2, 16, 1024);
          const uint64_t bv = sdesc(smem_u32(sm + Ly::STV) + kk * 128, C * 128, 1024);
          mma_bf16(tmem + Ly::TM_U0, ad, bv, id_nv, kk > 0);
        }
        if (bv_split) {
          // + (lo part of T Diag(beta^v)) V: the lo rows sit in rows 64..127 of the tile, so this
          // 128-row operand starts there; its other 64 rows only reach unused rows of U0
#pragma unroll
          for (int kk = 0; kk < C; kk += 16) {
            const uint64_t ad = sdesc(smem_u32(sm + Ly::STQ) + 64 * 128 + kk * 2, 16, 1024);
            const uint64_t bv = sdesc(smem_u32(sm + Ly::STV) + kk * 128, C * 128, 1024);
            mma_bf16(tmem + Ly::TM_U0, ad, bv, id_nv, 1);
          }
        }
        mma_commit(&bar_mma);
        if (c + 1 < nchunks) {
          const int j = (c + 1) & 1;
          if (mbar_wait_bounded(&bar_qk[j], ph_qk[j], a.wait_ns)) {
            ph_qk[j] ^= 1;
            pend_qk[j] = false;
            issue_gram(c + 1);
            mma_commit(&bar_gram);
          } else {
            ok0 = false;
          }
        }
      }
      // meanwhile: the state entering the chunk -> bf16 operand tile in SMU, and gamma_C S -> TM_S
      // (fp32, where the state update accumulates); rows 32 q4 .. +32, columns of half ch
      {
        const int k = 32 * q4 + lane;
        const float gl = s_f[cur].glast;
        uint32_t xr[NCB][32];  // all TMEM loads of this thread in flight at once
        if (c == 0) {
#pragma unroll
          for (int cb = 0; cb < NCB; ++cb) {
            const int col = ch * (NV / 2) + 32 * cb;
            const float* src = a.S0 ? a.S0 + ((int64_t)bh * DK + k) * dv + col0 + col : nullptr;
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 f = src ? *reinterpret_cast<const float4*>(src + e) : make_float4(0.f, 0.f, 0.f, 0.f);
              xr[cb][e] = __float_as_uint(f.x), xr[cb][e + 1] = __float_as_uint(f.y);
              xr[cb][e + 2] = __float_as_uint(f.z), xr[cb][e + 3] = __float_as_uint(f.w);
            }
          }
        } else {
#pragma unroll
          for (int cb = 0; cb < NCB; ++cb) tmem_ld32_issue(tmem + lane_base + Ly::TM_S + ch * (NV / 2) + 32 * cb, xr[cb]);
#pragma unroll
          for (int cb = 0; cb < NCB; ++cb) tmem_wait_ld(xr[cb]);
        }
#pragma unroll
        for (int cb = 0; cb < NCB; ++cb) {
          const int col = ch * (NV / 2) + 32 * cb;
          float x[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(xr[cb][e]);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            uint4 pk = make_uint4(pack_bf16(x[8 * q8], x[8 * q8 + 1]), pack_bf16(x[8 * q8 + 2], x[8 * q8 + 3]),
                                  pack_bf16(x[8 * q8 + 4], x[8 * q8 + 5]), pack_bf16(x[8 * q8 + 6], x[8 * q8 + 7]));
            *reinterpret_cast<uint4*>(sm + Ly::SMU + canon_chunk(k, col / 8 + q8, DK)) = pk;
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) x[e] *= gl;
          tmem_st32_issue(tmem + lane_base + Ly::TM_S + col, x);
        }
        tmem_wait_st();
      }
      {
        const bool ok = mbar_wait_bounded(&bar_mma, ph_mma, a.wait_ns);
        if (group_or(kBarState, kStateThreads, !ok)) {
          failed = true;
          break;
        }
        ph_mma ^= 1;
        tc_fence_after();
      }
      if (tid == 0 && c + 1 < nchunks) {
        issue_v(c + 1);
        pend_v = true;
      }

      // ---- M2: Wk -> bf16 into rows 0..63 of the [K; Q] tile (K is not read again); meanwhile the
      // other warps scale rows 64..127 to Q' = 2^{e_t} q_t (this chunk's Gram is complete: its
      // transform arrived on tready)
      if (q4 >= 2) {
        const int t = 32 * (q4 - 2) + lane;
        const float sc = pow2f(s_f[cur].oex[t]);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          uint4* p = reinterpret_cast<uint4*>(kq + canon_chunk(64 + t, 8 * ch + j, 128));
          *p = scale_bf16x8(*p, sc);
        }
      }
      if (q4 < 2) {
        const int t = 32 * q4 + lane;
        uint32_t xr[DK / 64][32];
#pragma unroll
        for (int cb = 0; cb < DK / 64; ++cb) tmem_ld32_issue(tmem + lane_base + Ly::TM_WK + ch * (DK / 2) + 32 * cb, xr[cb]);
#pragma unroll
        for (int cb = 0; cb < DK / 64; ++cb) tmem_wait_ld(xr[cb]);
#pragma unroll
        for (int cb = 0; cb < DK / 64; ++cb) {
          const int col = ch * (DK / 2) + 32 * cb;
          const uint32_t* x = xr[cb];
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            uint4 pk = make_uint4(pack_bf16(__uint_as_float(x[8 * q8]), __uint_as_float(x[8 * q8 + 1])),
                                  pack_bf16(__uint_as_float(x[8 * q8 + 2]), __uint_as_float(x[8 * q8 + 3])),
                                  pack_bf16(__uint_as_float(x[8 * q8 + 4]), __uint_as_float(x[8 * q8 + 5])),
                                  pack_bf16(__uint_as_float(x[8 * q8 + 6]), __uint_as_float(x[8 * q8 + 7])));
            *reinterpret_cast<uint4*>(kq + canon_chunk(t, col / 8 + q8, 128)) = pk;
          }
        }
      }
      fence_proxy_async();
      tc_fence_before();
      group_sync(kBarState, kStateThreads);
      tc_fence_after();

      // ---- M3: D1 = [Wk; Q'] S -> TM_D1
      if (tid == 0) {
#pragma unroll
        for (int kk = 0; kk < DK; kk += 16) {
          const uint64_t ad = sdesc(smem_u32(kq) + (kk >> 6) * (128 * 128) + (kk & 63) * 2, 16, 1024);
          const uint64_t bd = sdesc(smem_u32(sm + Ly::SMU) + kk * 128, DK * 128, 1024);
          mma_bf16(tmem + Ly::TM_D1, ad, bd, id_nv, kk > 0);
        }
        mma_commit(&bar_mma);
      }
      {
        const bool ok = mbar_wait_bounded(&bar_mma, ph_mma, a.wait_ns);
        if (group_or(kBarState, kStateThreads, !ok)) {
          failed = true;
          break;
        }
        ph_mma ^= 1;
        tc_fence_after();
      }
      // this chunk's [K; Q] buffer is free: load chunk c + 2's into it
      if (tid == 0 && c + 2 < nchunks) {
        issue_qk(c + 2);
        pend_qk[c & 1] = true;
      }

      // ---- M4: U' = c (U0 - Wk S), rows 0..63 -> hi / lo tiles (the S tile is dead); meanwhile the
      // other warps wait for this chunk's raw k tile and scale its rows to K' = 2^{n_i} k_i
      bool ok_k = true;
      if (q4 >= 2) {
        ok_k = mbar_wait_bounded(&bar_k, ph_k, a.wait_ns);
        if (ok_k) {
          const int u = 32 * ((q4 - 2) + 2 * ch) + lane;
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int e = u + 128 * it, i = e >> 4;
            uint4* p = reinterpret_cast<uint4*>(sm + Ly::STK + canon_chunk(i, e & 15, C));
            *p = scale_bf16x8(*p, pow2f(s_f[cur].n[i]));
          }
        }
      }
      if (q4 < 2) {
        const int t = 32 * q4 + lane;
        const float us = s_f[cur].c[t];
#pragma unroll
        for (int cb = 0; cb < NV / 64; ++cb) {
          const int col = ch * (NV / 2) + 32 * cb;
          uint32_t u0r[32], d1r[32];
          tmem_ld32_issue(tmem + lane_base + Ly::TM_U0 + col, u0r);
          tmem_ld32_issue(tmem + lane_base + Ly::TM_D1 + col, d1r);
          tmem_wait_ld(u0r);
          tmem_wait_ld(d1r);
          float u0[32], d1[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) u0[e] = __uint_as_float(u0r[e]), d1[e] = __uint_as_float(d1r[e]);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 8 * q8 + 2 * e;
              split_bf16(us * (u0[i] - d1[i]), us * (u0[i + 1] - d1[i + 1]), hi[e], lo[e]);
            }
            const uint32_t off = canon_chunk(t, col / 8 + q8, C);
            *reinterpret_cast<uint4*>(sm + Ly::SMU + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(sm + Ly::SMU + C * NV * 2 + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          }
        }
      }
      fence_proxy_async();
      {
        tc_fence_before();
        if (group_or(kBarState, kStateThreads, !ok_k)) {
          failed = true;
          break;
        }
        ph_k ^= 1;
        pend_k = false;
        tc_fence_after();
      }

      // ---- M5: D1 rows 64..127 += P' U' (O); S_acc += K'^T U' (hi and lo)
      if (tid == 0) {
        const uint32_t pa = smem_u32(sm + Ly::TP) + (uint32_t)(c & 1) * (C * C * 2);  // rows 64..127 = P
#pragma unroll
        for (int kk = 0; kk < C; kk += 16) {
          const uint64_t ad = sdesc(pa + kk * 2, 16, 1024);
          const uint64_t bd = sdesc(smem_u32(sm + Ly::SMU) + kk * 128, C * 128, 1024);
          mma_bf16(tmem + Ly::TM_D1, ad, bd, id_nv, 1);
        }
#pragma unroll
        for (int kk = 0; kk < C; kk += 16) {
          const uint64_t ak = sdesc(smem_u32(sm + Ly::STK) + kk * 128, C * 128, 1024);
          const uint64_t buh = sdesc(smem_u32(sm + Ly::SMU) + kk * 128, C * 128, 1024);
          const uint64_t bul = sdesc(smem_u32(sm + Ly::SMU + C * NV * 2) + kk * 128, C * 128, 1024);
          mma_bf16(tmem + Ly::TM_S, ak, buh, id_state, 1);
          mma_bf16(tmem + Ly::TM_S, ak, bul, id_state, 1);
        }
        mma_commit(&bar_mma);
      }
      {
        const bool ok = mbar_wait_bounded(&bar_mma, ph_mma, a.wait_ns);
        if (group_or(kBarState, kStateThreads, !ok)) {
          failed = true;
          break;
        }
        ph_mma ^= 1;
        tc_fence_after();
      }
      if (tid == 0 && c + 1 < nchunks) {
        issue_k(c + 1);
        pend_k = true;
      }

      // ---- M6: o rows of chunk c = rho_t x (rows 64..127 of D1), warps of quadrants 2 and 3; the
      // TMEM load is warp-collective: every lane loads, only rows of real tokens store
      if (q4 >= 2) {
        const int t = 32 * (q4 - 2) + lane, nc = min(C, T - t0);
        const float os = s_f[cur].orho[t];  // mantissa of gamma_t (of gamma_{t-1} before the update)
        __nv_bfloat16* orow =
            reinterpret_cast<__nv_bfloat16*>(a.o) + (((int64_t)b * T + t0 + t) * H + h) * dv + col0;
        uint32_t xr[NCB][32];
#pragma unroll
        for (int cb = 0; cb < NCB; ++cb) tmem_ld32_issue(tmem + lane_base + Ly::TM_D1 + ch * (NV / 2) + 32 * cb, xr[cb]);
#pragma unroll
        for (int cb = 0; cb < NCB; ++cb) tmem_wait_ld(xr[cb]);
        if (t < nc) {
#pragma unroll
          for (int cb = 0; cb < NCB; ++cb) {
            const int col = ch * (NV / 2) + 32 * cb;
            float x[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) x[e] = os * __uint_as_float(xr[cb][e]);
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
      group_sync(kBarState, kStateThreads);
      tc_fence_after();
    }

    if (!failed && nchunks > 0) {
      // S_T = S_acc of the last chunk
      const int k = 32 * q4 + lane;
#pragma unroll
      for (int cb = 0; cb < NV / 64; ++cb) {
        const int col = ch * (NV / 2) + 32 * cb;
        float x[32];
        tmem_ld32(tmem + lane_base + Ly::TM_S + col, x);
        float* dst = a.S + ((int64_t)bh * DK + k) * dv + col0 + col;
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
      }
    }
    if (failed && tid == 0) {
      // drain: every tensor-core op this thread issued (a commit tracks all earlier ones), then
      // every TMA load still in flight (bounded)
      mma_commit(&bar_drain);
      mbar_wait_bounded(&bar_drain, 0, kWaitNs);
      for (int j = 0; j < 2; ++j)
        if (pend_qk[j]) mbar_wait_bounded(&bar_qk[j], ph_qk[j], kWaitNs);
      if (pend_k) mbar_wait_bounded(&bar_k, ph_k, kWaitNs);
      if (pend_v) mbar_wait_bounded(&bar_v, ph_v, kWaitNs);
    }
  } else {
    // ======================================================= transform group
    const int gt = tid - kStateThreads, gw = gt >> 5, gch = gw >> 2;  // q4 == gw & 3
    uint32_t ph_gr = 0;
    // Thread j < 64 (warps 8, 9) holds token j's gates of the next chunk in registers, loaded one
    // chunk ahead of their use.
    scf::Gates gx;
    if (gt < 64 && nchunks > 0) gx = scf::load_gates(a, b, h, 0, gt);

    for (int n = 0; n < nchunks; ++n) {
      const int cur = n & 3;
      if (gt < 64) {
        const scf::Gates g = gx;
        if (n + 1 < nchunks) gx = scf::load_gates(a, b, h, n + 1, gt);
        scf::token_factors(g, gt, lane, pre, s_f[cur]);
      }
      // ---- X1: the Gram of chunk n has completed, and with it chunk n - 1's Wk / U0 products
      {
        const bool ok = mbar_wait_bounded(&bar_gram, ph_gr, a.wait_ns);
        if (group_or(kBarXform, kXformThreads, !ok)) {
          failed = true;
          break;
        }
        ph_gr ^= 1;
        tc_fence_after();
      }
      // ---- X2: A (strict lower) -> fp32 L; P' (lower incl., or strictly lower before the update) ->
      // bf16 P' tile of parity n & 1 (last read by chunk n - 2's O product, long complete)
      float* sL = reinterpret_cast<float*>(sm + Ly::INV);
      float* sT = sL + C * C;
      scf::extract_ap(s_f[cur], tmem + Ly::TM_GR, q4, gch, lane, pre, sL, sm + Ly::TP + (1 + (n & 1)) * (C * C * 2));
      tc_fence_before();
      // ---- X3: T = (I + A)^{-1} -> T Diag(gamma) (TP rows 0..63) and T Diag(beta^v) (STQ rows 0..63)
      if (bv_split)
        unit_lower_inverse<true, 8, false, true>(sL, sT, s_Y, sm + Ly::TP, sm + Ly::STQ, s_f[cur].gam, s_f[cur].bv,
                                                 gt, kBarXform);
      else
        unit_lower_inverse<true, 8, false>(sL, sT, s_Y, sm + Ly::TP, sm + Ly::STQ, s_f[cur].gam, s_f[cur].bv, gt,
                                           kBarXform);
      fence_proxy_async();
      group_sync(kBarXform, kXformThreads);
      if (gt == 0) mbar_arrive(&bar_tready);
    }
  }

  if (failed && tid == 0) atomicExch(a.status, kDevTimeout);
  if (failed && tid == kStateThreads) atomicExch(a.status, kDevTimeout);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, kTmemCols);
}

// ---------------------------------------------------------------- host side
template <int NV>
cudaError_t launch_impl(const Args& a, cudaStream_t s) {
  using Ly = ScLayout<NV>;
  const int smem = Ly::TOTAL + 1024;
  cudaError_t e = cudaFuncSetAttribute(chunk_sc_kernel<NV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  CUtensorMap mq, mk, mv;
  if (!make_bthd_map(&mq, a.q, DK, a.H, a.T, a.B, C) || !make_bthd_map(&mk, a.k, DK, a.H, a.T, a.B, C) ||
      !make_bthd_map(&mv, a.v, a.dv, a.H, a.T, a.B, C))
    return cudaErrorInvalidValue;
  chunk_sc_kernel<NV><<<a.B * a.H * (a.dv / NV), kThreads, smem, s>>>(mq, mk, mv, a);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_chunk_sc(const Args& a, cudaStream_t s) {
  // few sequences: split the 128 value columns into two 64-column CTAs when that still fits in one
  // wave (each CTA repeats the column-independent transform)
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const bool split = a.dv == 128 && (int64_t)a.B * a.H * 2 <= sms;
  if (a.dv == 128 && !split) return launch_impl<128>(a, s);
  return launch_impl<64>(a, s);
}

}  // namespace dn
