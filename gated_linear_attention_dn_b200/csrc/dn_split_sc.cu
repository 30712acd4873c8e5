// Chunked prefill for per-token gates (GDN: scalar alpha, beta^k, beta^v, d; bf16 io, d_k = 128,
// d_v in {64, 128}) in two kernels, for callers that pass a workspace:
//
//  1. xform_sc_kernel, one CTA per (b, h, chunk), all chunks at once: the chunk's decay factors, the
//     Gram product [K; Q] K^T (tcgen05), A and P', and the UT transform T = (I + A)^{-1}; it writes
//     the bf16 operand tiles T Diag(gamma), P' and T Diag(beta^v) and the per-token factors the state
//     chain needs into the chunk's workspace record.
//  2. chain_sc_kernel, one CTA per (b, h) and slice of NV value columns: the state recurrence over the
//     chunks in order, with the fp32 state in tensor memory. The state-independent products of chunk
//     c + 1 (Wk = (T Diag gamma) K, U0 = (T Diag beta^v) V, and the bf16 conversions of Wk, Q' and K')
//     are issued while chunk c's state chain runs, so each chunk's sequential path is only: the
//     state framing, D1 = [Wk; Q'] S, U' = c (U0 - Wk S), and O += P' U', S += K'^T U'.
//
// The algebra and the factors are those of dn_chunk_sc.cu (dn_sc_factors.cuh): the chunk-parallel WY /
// UT evaluation of the gated delta rule (FG2-GDN page, sections 2.A and 3 item 2), with decay
// products carried as mantissa and exponent. Splitting the chunk-local transform off the sequential
// chain trades one extra pass over q and k and ~25 KB of workspace per chunk for a chain that no
// longer shares its SM with the transform.
//
// Workspace record of one (b, h, chunk), chunk-major per (b, h): T Diag(gamma) (bf16 64 x 64,
// 128-byte-swizzled canonical layout, as the MMA reads it), P' (same), T Diag(beta^v) (hi rows; then
// lo rows when beta^v is given), then the factor record (c_t, o scale, Q' and K' exponents, gamma_C).
// Every mbarrier wait is bounded in time; on expiry a kernel leaves its loop, drains what it issued,
// sets the status word and frees its tensor memory.
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
constexpr int kThreads = 256;
constexpr uint64_t kDrainNs = 2000000000ull;  // bound of the drain waits after a failure

// ------------------------------------------------------------------ workspace record
struct Rec {
  float c[C];     // U' row scale c_t = beta^k_t d_t mu_t
  float orho[C];  // o scale
  int oex[C];     // exponent of the power of two on q_t (Q')
  int n[C];       // exponent of the power of two on k_t (K')
  float glast;    // gamma_C
  float pad[3];
};
static_assert(sizeof(Rec) == 1040, "factor record");
constexpr int kRecTG = 0;      // T Diag(gamma)
constexpr int kRecP = 8192;    // P'
constexpr int kRecTB = 16384;  // T Diag(beta^v): hi rows, then lo rows when beta^v is given
__host__ __device__ constexpr int tb_bytes(bool bv) { return bv ? 16384 : 8192; }
__host__ __device__ constexpr int rec_factor_off(bool bv) { return kRecTB + tb_bytes(bv); }
__host__ __device__ constexpr size_t rec_stride(bool bv) { return (size_t)rec_factor_off(bv) + sizeof(Rec); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// L2 prefetch of a tile of a tensor map
__device__ __forceinline__ void tma_prefetch_4d(const CUtensorMap* map, int x, int y, int z, int w) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global [%0, {%1, %2, %3, %4}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z), "r"(w)
               : "memory");
}

// shared -> global TMA tile store (rows past the tensor's end are not written), its group commit, and
// the wait until every committed store has finished reading shared memory
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, const void* src, int x, int y, int z, int w) {
  asm volatile("cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z), "r"(w)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

// ================================================================== 1. transform kernel
// Shared memory holds only the [K; Q] tile (TMA), which the fp32 L and T arrays overlay once the
// Gram is done, and the inverse's scratch; P' and the T tiles go straight to the record, so four
// CTAs fit on an SM.
constexpr int kXformSmem = 128 * DK * 2;  // [K; Q] bf16 [128][DK]; after the Gram: fp32 L and T (64 x 64 each)
static_assert(kXformSmem >= 2 * C * C * 4, "L and T fit over the [K; Q] tile");
constexpr int kXformPerSm = 4;

template <bool BV>
__global__ void __launch_bounds__(kThreads, kXformPerSm) xform_sc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                                        const __grid_constant__ CUtensorMap tm_k,
                                                                        const Args a, uint8_t* ws, int ahead) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ __align__(8) uint64_t bar_kq, bar_g;
  __shared__ uint32_t s_tmem;
  __shared__ __align__(16) float s_Y[2048];
  __shared__ scf::Factors s_f;
  __shared__ __align__(16) float s_wg[C], s_pw[C];  // column factors of the fast extraction
  __shared__ int s_wide;                            // a decay exponent of the chunk is beyond +-100
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q4 = warp & 3, gch = warp >> 2;
  const int pre = a.pre_read ? 1 : 0;
  const int nchunks = (a.T + C - 1) / C;
  // blocks run chunk-major from the last chunk back to the first, so that the records (and q, k
  // tiles) the state chains read first are the last ones written, still in L2 when the chains start
  const int nbhs = a.B * a.H;
  const int c = nchunks - 1 - (int)(blockIdx.x / nbhs), bh = (int)(blockIdx.x % nbhs), b = bh / a.H, h = bh % a.H;
  uint8_t* const rec = ws + ((size_t)bh * nchunks + c) * rec_stride(BV);
  if (tid == 0) s_wide = 0;
  const int64_t nb = (int64_t)blockIdx.x + ahead;  // the block that takes this one's place on its SM
  const bool pf = ahead > 0 && nb < (int64_t)gridDim.x;
  const int nc = nchunks - 1 - (int)(nb / nbhs), nbh = (int)(nb % nbhs);

  // thread 0 starts the [K; Q] load at once; warps 2 and 3 load the gates meanwhile (the factor scan
  // runs there, so that thread 0 is free to issue the Gram as soon as the tile lands)
  if (tid == 0) {
    mbar_init(&bar_kq, 1);
    mbar_init(&bar_g, 1);
    fence_mbar_init();
    mbar_expect_tx(&bar_kq, 2u * C * DK * 2);
#pragma unroll
    for (int x = 0; x < DK / 64; ++x) {
      tma_load_4d(sm + x * 128 * 128, &tm_k, &bar_kq, 64 * x, h, c * C, b);
      tma_load_4d(sm + x * 128 * 128 + 64 * 128, &tm_q, &bar_kq, 64 * x, h, c * C, b);
    }
    // the successor block's tiles into L2
    if (pf) {
#pragma unroll
      for (int x = 0; x < DK / 64; ++x) {
        tma_prefetch_4d(&tm_k, 64 * x, nbh % a.H, nc * C, nbh / a.H);
        tma_prefetch_4d(&tm_q, 64 * x, nbh % a.H, nc * C, nbh / a.H);
      }
    }
  }
  const bool fw = warp == 2 || warp == 3;  // the factor warps
  const int j = tid - 64;                  // their token
  scf::Gates g{};
  if (fw) {
    if (pf && nc * C + j < a.T) {  // the successor block's gates into L2 too
      const int64_t tok = ((int64_t)(nbh / a.H) * a.T + nc * C + j) * a.H + nbh % a.H;
      if (a.alpha == DN_GATE_SCALAR) prefetch_l2(a.alpha_p + tok);
      if (a.beta_k == DN_GATE_SCALAR) prefetch_l2(a.beta_k_p + tok);
      if (a.key_scale == DN_GATE_SCALAR) prefetch_l2(a.key_scale_p + tok);
      if (a.beta_v == DN_GATE_SCALAR) prefetch_l2(a.beta_v_p + tok);
    }
    g = scf::load_gates(a, b, h, c, j);
  }
  if (warp == 0) tmem_alloc(&s_tmem, 64);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  // Gram [K; Q] K^T -> tensor memory (M 128, N 64, K 128), while warps 2 and 3 scan the gates
  bool ok = true, issued = false;
  if (tid == 0) {
    ok = mbar_wait_bounded(&bar_kq, 0, a.wait_ns);
    if (ok) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
      for (int kk = 0; kk < DK; kk += 16) {
        const uint64_t d = sdesc(smem_u32(sm) + (kk >> 6) * (128 * 128) + (kk & 63) * 2, 16, 1024);
        mma_bf16(tmem, d, d, id, kk > 0);
      }
      mma_commit(&bar_g);
      issued = true;
    }
  }
  if (fw) {
    scf::token_factors(g, j, lane, pre, s_f);
    // the column factors of the fast extraction, and whether the chunk may use it
    const int ej = s_f.ex[j], oj = s_f.oex[j];
    s_wg[j] = s_f.ws[j] * s_f.rhoi[j] * pow2f(-ej);
    s_pw[j] = s_f.pinv[j] * pow2f(-ej);
    if (ej < -100 || ej > 100 || oj < -100 || oj > 100) s_wide = 1;
    // each thread copies the entries it wrote itself
    Rec* r = reinterpret_cast<Rec*>(rec + rec_factor_off(BV));
    r->c[j] = s_f.c[j];
    r->orho[j] = s_f.orho[j];
    r->oex[j] = s_f.oex[j];
    r->n[j] = s_f.n[j];
    if (j == 63) r->glast = s_f.glast;
  }
  if (__syncthreads_or(!ok)) {
    // the [K; Q] load did not land in time: wait for it (bounded), report, free tensor memory
    if (tid == 0) {
      mbar_wait_bounded(&bar_kq, 0, kDrainNs);
      atomicExch(a.status, kDevTimeout);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 64);
    return;
  }
  ok = mbar_wait_bounded(&bar_g, 0, a.wait_ns);
  if (__syncthreads_or(!ok)) {
    if (tid == 0 && issued) {
      mbar_wait_bounded(&bar_g, 0, kDrainNs);
      atomicExch(a.status, kDevTimeout);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 64);
    return;
  }
  tc_fence_after();
  // A into L (the [K; Q] tile is free now: L and T take its place), and P' into the inverse's
  // scratch, which warps 2..7 copy to the record with whole-line stores while warps 0 and 1 start
  // the inverse
  float* sL = reinterpret_cast<float*>(sm);
  float* sT = sL + C * C;
  if (s_wide)
    scf::extract_ap(s_f, tmem, q4, gch, lane, pre, sL, reinterpret_cast<uint8_t*>(s_Y));
  else
    scf::extract_ap_fast(s_f, s_wg, s_pw, tmem, q4, gch, lane, pre, sL, reinterpret_cast<uint8_t*>(s_Y));
  tc_fence_before();
  __syncthreads();
  // tensor memory is no longer needed
  if (warp == 0) tmem_dealloc(tmem, 64);
  if (tid >= 64) {
    const uint4* src = reinterpret_cast<const uint4*>(s_Y);
    uint4* dst = reinterpret_cast<uint4*>(rec + kRecP);
    for (int i = tid - 64; i < C * C * 2 / 16; i += kThreads - 64) dst[i] = src[i];
  }
  unit_lower_inverse<false, 8, true, false, false>(sL, sT, s_Y, nullptr, nullptr, nullptr, nullptr, tid, 0);
  // T Diag(gamma) and T Diag(beta^v) (hi, and lo when beta^v is given) as bf16 operand tiles, one
  // 16-byte chunk (row t, columns 8 x8 .. +7) per thread and step: eight threads write one
  // 128-byte row, so the stores are whole lines
  for (int e = tid; e < C * 8; e += kThreads) {
    const int t = e >> 3, x8 = e & 7;
    uint4 tg = make_uint4(0, 0, 0, 0), tb = tg, tl = tg;
    if (x8 <= (t >> 3)) {
      const float4 v0 = *reinterpret_cast<const float4*>(sT + xi(t, 8 * x8));
      const float4 v1 = *reinterpret_cast<const float4*>(sT + xi(t, 8 * x8 + 4));
      const float y[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
      const float* gm = s_f.gam + 8 * x8;
      const float* bv = s_f.bv + 8 * x8;
      tg = make_uint4(pack_bf16(y[0] * gm[0], y[1] * gm[1]), pack_bf16(y[2] * gm[2], y[3] * gm[3]),
                      pack_bf16(y[4] * gm[4], y[5] * gm[5]), pack_bf16(y[6] * gm[6], y[7] * gm[7]));
      float z[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) z[e] = y[e] * bv[e];
      if (BV) {
        tc::split_bf16(z[0], z[1], tb.x, tl.x);
        tc::split_bf16(z[2], z[3], tb.y, tl.y);
        tc::split_bf16(z[4], z[5], tb.z, tl.z);
        tc::split_bf16(z[6], z[7], tb.w, tl.w);
      } else {
        tb = make_uint4(pack_bf16(z[0], z[1]), pack_bf16(z[2], z[3]), pack_bf16(z[4], z[5]), pack_bf16(z[6], z[7]));
      }
    }
    const uint32_t off = canon_chunk(t, x8, 128);
    *reinterpret_cast<uint4*>(rec + kRecTG + off) = tg;
    *reinterpret_cast<uint4*>(rec + kRecTB + off) = tb;
    if (BV) *reinterpret_cast<uint4*>(rec + kRecTB + 64 * 128 + off) = tl;
  }
}

// ================================================================== 2. state-chain kernel
template <int NV>
struct CLayout {
  static constexpr int KB0 = 0;                    // raw k [C][DK] (TMA), rows scaled to K'; chunks of parity 0
  static constexpr int KB1 = KB0 + C * DK * 2;     //                                          parity 1
  static constexpr int QB0 = KB1 + C * DK * 2;     // [Wk; Q'] [128][DK]: q by TMA into rows 64..127
  static constexpr int QB1 = QB0 + 128 * DK * 2;
  static constexpr int VB = QB1 + 128 * DK * 2;    // raw v [C][NV] (TMA)
  static constexpr int TG = VB + C * NV * 2;       // T Diag(gamma) [64][64]; P' of parity 0 and 1 follow it:
  static constexpr int PB0 = TG + C * C * 2;       // the O product of parity p reads the 128 rows starting
  static constexpr int PB1 = PB0 + C * C * 2;      // 64 rows before PB_p, whose rows 64..127 are P'
  // T Diag(beta^v): hi rows, 64 zero rows, lo rows, 64 zero rows (the U0 product reads 128
  // rows from the hi or the lo rows, and its rows 64..127 must come out zero)
  static constexpr int TB = PB1 + C * C * 2;
  static constexpr int TBLO = TB + 128 * C * 2;
  static constexpr int OST = TBLO + 128 * C * 2;   // o rows of a chunk [C][NV] bf16, staged for the TMA store
  static constexpr int SMU = OST + C * NV * 2;     // S bf16 [DK][NV]; after D1: U' hi, U' lo [C][NV]
  static constexpr int SMU_BYTES = (DK * NV * 2 > 2 * C * NV * 2) ? DK * NV * 2 : 2 * C * NV * 2;
  static constexpr int FR0 = SMU + SMU_BYTES;      // factor records of parity 0 and 1
  static constexpr int FR1 = FR0 + 1088;
  static constexpr int TOTAL = FR1 + 1088;
  static_assert(TOTAL + 1024 + 4096 <= 227 * 1024, "shared memory budget");
  // tensor memory: the state; two accumulators (chunk parity) where U0 lands and D1 and the O product
  // accumulate; Wk
  static constexpr int TM_S = 0, TM_U = NV, TM_WK = 3 * NV;
  static_assert(TM_WK + DK <= 512, "tensor memory budget");
};

// Warp roles. Warp w runs on SM sub-partition w % 4 and reaches tensor-memory lanes 32 (w % 4) ..
// +31, so the work is placed by lane quadrant:
//  * warps 0..7 run the state chain of each chunk: all of them frame the state (S rows are all 128
//    lanes) and meet at a barrier, after which thread 0 issues D1 = [Wk; Q'] S (warp 0 has nothing to
//    do until D1 is done anyway); quadrants 0 and 1 form U' (rows 0..63 of D1 and U0) and the group
//    meets again, after which thread 0 issues O += P' U' (rows 64..127 of D1; the o rows leave as soon
//    as it is done), then the state update (the next chunk's framing waits for it); quadrants 2 and 3
//    store the o rows while the state update runs;
//  * warps 8 and 9 (quadrants 0 and 1) convert each chunk's Wk (lanes 0..63 of its accumulator) to the
//    bf16 rows 0..63 of its [Wk; Q'] tile, ahead of the chain;
//  * warp 11 scales the q rows of each chunk to Q' and its k rows to K' (shared memory only);
//  * lane 0 of warp 10 issues every load (and L2 prefetches further ahead) and the state-independent
//    products of the next chunk, Wk(c + 1) and U0(c + 1), as soon as their tensor memory is free (so
//    their issue stalls never hold the chain's warps).
// Hand-overs across warps go through mbarriers; within warps 0..7 through a named barrier. Each
// mbarrier that completes once per chunk is waited on for chunk c only by threads whose progress
// keeps its completion for chunk c + 1 from happening first (a wait by parity cannot tell two
// completions apart).
constexpr int kChainThreads = 384;
constexpr int kLoaderWarp = 10;
constexpr int kScalerWarp = 11;
constexpr int kBarChain = 1;  // named barrier of warps 0..7
constexpr int kBarOut = 2;    // named barrier of the o-storing warps (quadrants 2, 3 of warps 0..7)

template <int NV>
__global__ void __launch_bounds__(kChainThreads, 1)
    chain_sc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o, const Args a,
                    const uint8_t* ws, int bv_split) {
  using Ly = CLayout<NV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  // loads (transaction counts); products (commits); hand-overs (arrivals)
  __shared__ __align__(8) uint64_t bar_kq[2], bar_fr[2], bar_tg, bar_vb, bar_p[2];
  // (the state update, the O product and the o stores of chunk c complete barrier [c & 1]: the loader
  // looks at them a chunk later than the chain, which can never lap it by two chunks)
  // (Wk(c) completes both bar_wk and bar_wkp[c & 1]: the scaling warp waits on the latter, which it
  // cannot fall two completions behind)
  __shared__ __align__(8) uint64_t bar_wk, bar_wkp[2], bar_u0, bar_d1, bar_os[2], bar_o[2], bar_drain, bar_drain2;
  // (the scaling warp arrives on bar_kconv and on bar_kconvp[c & 1]: the loader, which reloads chunk
  // c's factor record after it, waits on the latter)
  __shared__ __align__(8) uint64_t bar_kconv, bar_kconvp[2], bar_wkfree, bar_ufree, bar_wkconv;
  __shared__ uint32_t s_tmem;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q4 = warp & 3, ch = (warp >> 2) & 1;
  const int T = a.T, H = a.H, dv = a.dv;
  const int nslices = dv / NV;
  const int bh = blockIdx.x / nslices, b = bh / H, h = bh % H;
  const int col0 = (blockIdx.x % nslices) * NV;
  const int nchunks = (T + C - 1) / C;
  const size_t stride = rec_stride(bv_split != 0);
  const uint8_t* const rec0 = ws + (size_t)bh * nchunks * stride;
  const uint32_t tbb = (uint32_t)tb_bytes(bv_split != 0);
  const uint32_t lane_base = (uint32_t)(32 * q4) << 16;

  if (tid == 0) {
    for (int j = 0; j < 2; ++j) {
      mbar_init(&bar_kq[j], 1);
      mbar_init(&bar_fr[j], 1);
      mbar_init(&bar_p[j], 1);
      mbar_init(&bar_os[j], 1);
      mbar_init(&bar_o[j], 1);
    }
    mbar_init(&bar_d1, 1);
    mbar_init(&bar_drain, 1);
    mbar_init(&bar_tg, 1);
    mbar_init(&bar_vb, 1);
    mbar_init(&bar_wk, 1);
    mbar_init(&bar_wkp[0], 1);
    mbar_init(&bar_wkp[1], 1);
    mbar_init(&bar_u0, 1);
    mbar_init(&bar_drain2, 1);
    mbar_init(&bar_wkfree, 2);   // warps 8, 9: chunk c's Wk has been read (TM_WK free)
    mbar_init(&bar_wkconv, 2);   // warps 8, 9: chunk c's Wk rows of the [Wk; Q'] tile are written
    mbar_init(&bar_ufree, 1);    // thread 0: chunk c's U' is formed (the other accumulator is free)
    mbar_init(&bar_kconv, 1);    // the scaling warp: chunk c's K' and Q' rows are scaled
    mbar_init(&bar_kconvp[0], 1);
    mbar_init(&bar_kconvp[1], 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&s_tmem, 512);
  // the zero rows after the hi and after the lo rows of T Diag(beta^v)
  for (int i = tid; i < 64 * C * 2 / 16; i += kChainThreads) {
    reinterpret_cast<uint4*>(sm + Ly::TB + 64 * 128)[i] = make_uint4(0, 0, 0, 0);
    reinterpret_cast<uint4*>(sm + Ly::TBLO + 64 * 128)[i] = make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  auto kb = [&](int c) -> uint8_t* { return sm + ((c & 1) ? Ly::KB1 : Ly::KB0); };
  auto qb = [&](int c) -> uint8_t* { return sm + ((c & 1) ? Ly::QB1 : Ly::QB0); };

  auto pbuf = [&](int c) -> uint8_t* { return sm + ((c & 1) ? Ly::PB1 : Ly::PB0); };
  auto frec = [&](int c) -> const Rec* { return reinterpret_cast<const Rec*>(sm + ((c & 1) ? Ly::FR1 : Ly::FR0)); };
  auto rec = [&](int c) -> const uint8_t* { return rec0 + (size_t)c * stride; };
  // parity of the m-th completion (m = 0, 1, ...) of a barrier that completes once per chunk, and of a
  // double-buffered load barrier's completion for chunk c
  auto par = [](int m) -> uint32_t { return (uint32_t)(m & 1); };
  auto par2 = [](int c) -> uint32_t { return (uint32_t)((c >> 1) & 1); };
  auto wait = [&](uint64_t* bar, uint32_t parity) -> bool { return mbar_wait_bounded(bar, parity, a.wait_ns); };
  auto wait_idle = [&](uint64_t* bar, uint32_t parity) -> bool {
    return mbar_wait_bounded_idle(bar, parity, a.wait_ns);
  };

  bool failed = false;
  if (warp == kLoaderWarp) {
    // ======================================================= loads (one thread)
    if (lane == 0 && nchunks > 0) {
      // loads in flight, by the completion they will produce: the chunk of a double-buffered load (-1:
      // none), the chunk of bar_tg's load
      int pend_kq[2] = {-1, -1}, pend_fr[2] = {-1, -1}, pend_p[2] = {-1, -1}, pend_tg = -1, pend_vb = -1;
      auto issue_kq = [&](int c) {  // k and q of chunk c
        uint64_t* bar = &bar_kq[c & 1];
        mbar_expect_tx(bar, 2u * C * DK * 2);
#pragma unroll
        for (int x = 0; x < DK / 64; ++x) {
          tma_load_4d(kb(c) + x * C * 128, &tm_k, bar, 64 * x, h, c * C, b);
          tma_load_4d(qb(c) + x * 128 * 128 + 64 * 128, &tm_q, bar, 64 * x, h, c * C, b);
        }
        pend_kq[c & 1] = c;
      };
      auto issue_fr = [&](int c) {  // the factor record of chunk c
        uint64_t* bar = &bar_fr[c & 1];
        mbar_expect_tx(bar, (uint32_t)sizeof(Rec));
        bulk_load(const_cast<Rec*>(frec(c)), rec(c) + rec_factor_off(bv_split != 0), sizeof(Rec), bar);
        pend_fr[c & 1] = c;
      };
      auto issue_tg = [&](int c) {  // T Diag(gamma) of chunk c (completion c of bar_tg)
        mbar_expect_tx(&bar_tg, 8192);
        bulk_load(sm + Ly::TG, rec(c) + kRecTG, 8192, &bar_tg);
        pend_tg = c;
      };
      auto issue_vb = [&](int c) {  // v slice and T Diag(beta^v) of chunk c (completion c of bar_vb)
        mbar_expect_tx(&bar_vb, (uint32_t)C * NV * 2 + tbb);
#pragma unroll
        for (int x = 0; x < NV / 64; ++x) tma_load_4d(sm + Ly::VB + x * C * 128, &tm_v, &bar_vb, col0 + 64 * x, h, c * C, b);
        bulk_load(sm + Ly::TB, rec(c) + kRecTB, 8192, &bar_vb);
        if (bv_split) bulk_load(sm + Ly::TBLO, rec(c) + kRecTB + 8192, 8192, &bar_vb);
        pend_vb = c;
      };
      auto issue_p = [&](int c) {
        uint64_t* bar = &bar_p[c & 1];
        mbar_expect_tx(bar, 8192);
        bulk_load(pbuf(c), rec(c) + kRecP, 8192, bar);
        pend_p[c & 1] = c;
      };
      auto prefetch = [&](int c) {  // every tile of chunk c, into L2
#pragma unroll
        for (int x = 0; x < DK / 64; ++x) {
          tma_prefetch_4d(&tm_k, 64 * x, h, c * C, b);
          tma_prefetch_4d(&tm_q, 64 * x, h, c * C, b);
        }
#pragma unroll
        for (int x = 0; x < NV / 64; ++x) tma_prefetch_4d(&tm_v, col0 + 64 * x, h, c * C, b);
        bulk_prefetch(rec(c), (uint32_t)stride);
      };
      issue_kq(0);
      issue_fr(0);
      issue_tg(0);
      issue_vb(0);
      issue_p(0);
      if (nchunks > 1) {
        issue_kq(1);
        issue_fr(1);
        issue_p(1);
      }
      for (int c = 2; c < 4 && c < nchunks; ++c) prefetch(c);
      const uint32_t id_wk = idesc_bf16(128, DK, 0, 1);
      const uint32_t id_nv = idesc_bf16(128, NV, 0, 1);
      // Wk(c) = (T Diag gamma) K(c) -> TM_WK (lanes 0..63); U0(c) = (T Diag beta^v) V(c) ->
      // accumulator c & 1 (rows 64..127 zero)
      auto mma_wk = [&](int c) {
#pragma unroll
        for (int kk = 0; kk < C; kk += 16) {
          const uint64_t ad = sdesc(smem_u32(sm + Ly::TG) + kk * 2, 16, 1024);
          const uint64_t bk = sdesc(smem_u32(kb(c)) + kk * 128, C * 128, 1024);
          mma_bf16(tmem + Ly::TM_WK, ad, bk, id_wk, kk > 0);
        }
        mma_commit(&bar_wk);
        mma_commit(&bar_wkp[c & 1]);
      };
      auto mma_u0 = [&](int c) {
        const uint32_t vb = smem_u32(sm + Ly::VB), acc = tmem + Ly::TM_U + (c & 1) * NV;
        const uint32_t hi = smem_u32(sm + Ly::TB), lo = smem_u32(sm + Ly::TBLO);
#pragma unroll
        for (int kk = 0; kk < C; kk += 16)
          mma_bf16(acc, sdesc(hi + kk * 2, 16, 1024), sdesc(vb + kk * 128, C * 128, 1024), id_nv, kk > 0);
        if (bv_split) {
#pragma unroll
          for (int kk = 0; kk < C; kk += 16)
            mma_bf16(acc, sdesc(lo + kk * 2, 16, 1024), sdesc(vb + kk * 128, C * 128, 1024), id_nv, 1);
        }
        mma_commit(&bar_u0);
      };
      bool ok = true, issued = false;
      // Wk(0) and U0(0)
      ok = wait_idle(&bar_tg, par(0)) && wait_idle(&bar_kq[0], par2(0));
      if (ok) {
        pend_tg = pend_kq[0] = -1;
        tc_fence_after();
        mma_wk(0);
        issued = true;
        ok = wait_idle(&bar_vb, par(0));
      }
      if (ok) {
        pend_vb = -1;
        mma_u0(0);
        // v and T Diag(beta^v) of chunk 1 once U0(0) has read chunk 0's
        if (nchunks > 1) {
          ok = wait_idle(&bar_u0, par(0));
          if (ok) issue_vb(1);
        }
      }
      // per chunk c: Wk(c + 1) once chunk c's Wk is converted, then T Diag(gamma) of chunk c + 2 once
      // Wk(c + 1) has read chunk c + 1's; U0(c + 1) once U'(c) is formed, and then the factor record
      // of chunk c + 2; the buffers of chunk c once its products have read them (k, q: the state
      // update; v, T Diag(beta^v): U0(c); P': the O product)
      for (int c = 0; c < nchunks && ok; ++c) {
        const bool more = c + 1 < nchunks;
        if (c == 0 && more) {
          ok = wait_idle(&bar_wk, par(0));  // T Diag(gamma) of chunk 0 has been read
          if (!ok) break;
          issue_tg(1);
        }
        if (more) {
          ok = wait_idle(&bar_wkfree, par(c)) && wait_idle(&bar_tg, par(c + 1)) &&
               wait_idle(&bar_kq[(c + 1) & 1], par2(c + 1));
          if (!ok) break;
          pend_tg = pend_kq[(c + 1) & 1] = -1;
          tc_fence_after();
          mma_wk(c + 1);
          if (c + 4 < nchunks) prefetch(c + 4);
          ok = wait_idle(&bar_ufree, par(c)) && wait_idle(&bar_vb, par(c + 1));
          if (!ok) break;
          pend_vb = -1;
          tc_fence_after();
          mma_u0(c + 1);
          // chunk c's factor record has been read: by the chain up to U'(c) (its o scales are kept in
          // registers) and by the scaling warp
          if (c + 2 < nchunks) {
            ok = wait_idle(&bar_kconvp[c & 1], par2(c));
            if (!ok) break;
            issue_fr(c + 2);
          }
          if (c + 2 < nchunks) {  // v and T Diag(beta^v) of chunk c + 2 once U0(c + 1) has read chunk c + 1's
            ok = wait_idle(&bar_u0, par(c + 1));
            if (!ok) break;
            issue_vb(c + 2);
          }
          if (c + 2 < nchunks) {
            ok = wait_idle(&bar_wk, par(c + 1));
            if (!ok) break;
            issue_tg(c + 2);
          }
        }
        if (c + 2 < nchunks) {  // (U0(c) is done: the chain saw it before signalling bar_ufree)
          ok = wait_idle(&bar_os[c & 1], par2(c));
          if (!ok) break;
          issue_kq(c + 2);
          ok = wait_idle(&bar_o[c & 1], par2(c));
          if (!ok) break;
          issue_p(c + 2);
        }
      }
      if (!ok) {
        failed = true;
        if (issued) {  // every product this thread issued
          mma_commit(&bar_drain2);
          mbar_wait_bounded(&bar_drain2, 0, kDrainNs);
        }
        // drain every load in flight
        for (int j = 0; j < 2; ++j) {
          if (pend_kq[j] >= 0) mbar_wait_bounded(&bar_kq[j], par2(pend_kq[j]), kDrainNs);
          if (pend_fr[j] >= 0) mbar_wait_bounded(&bar_fr[j], par2(pend_fr[j]), kDrainNs);
          if (pend_p[j] >= 0) mbar_wait_bounded(&bar_p[j], par2(pend_p[j]), kDrainNs);
        }
        if (pend_tg >= 0) mbar_wait_bounded(&bar_tg, par(pend_tg), kDrainNs);
        if (pend_vb >= 0) mbar_wait_bounded(&bar_vb, par(pend_vb), kDrainNs);
      }
    }
  } else if (warp == kScalerWarp) {
    // ======================================================= q rows -> Q' = 2^{oex} q, k rows -> K' = 2^{n} k
    // 16-byte chunk e of a 64-row, 128-column tile: row e / 16, chunk e % 16; in batches of 8 loads
    // before their stores
    auto scale_rows = [&](uint8_t* tile, int row0, const int* ex) {
#pragma unroll 1
      for (int j0 = 0; j0 < 32; j0 += 8) {
        uint4 kv[8];
        float sc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int e = lane + 32 * (j0 + j), i = e >> 4;
          kv[j] = *reinterpret_cast<const uint4*>(tile + canon_chunk(row0 + i, e & 15, row0 + C));
          sc[j] = pow2f(ex[i]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int e = lane + 32 * (j0 + j), i = e >> 4;
          *reinterpret_cast<uint4*>(tile + canon_chunk(row0 + i, e & 15, row0 + C)) = scale_bf16x8(kv[j], sc[j]);
        }
      }
    };
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      // the q and k tiles and the factors of chunk c have landed
      ok = wait_idle(&bar_kq[c & 1], par2(c)) && wait_idle(&bar_fr[c & 1], par2(c));
      if (!ok) break;
      const Rec* fr = frec(c);
      scale_rows(qb(c), 64, fr->oex);  // rows 64..127 of the [Wk; Q'] tile (the tile has 128 rows)
      ok = wait_idle(&bar_wkp[c & 1], par2(c));  // Wk(c) has read the raw k rows
      if (!ok) break;
      scale_rows(kb(c), 0, fr->n);
      fence_proxy_async();
      // D1(c - 1) is done, so the chain has seen kconv(c - 1) before kconv(c) can complete
      ok = c == 0 || wait_idle(&bar_d1, par(c - 1));
      if (!ok) break;
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bar_kconv);
        mbar_arrive(&bar_kconvp[c & 1]);
      }
    }
    if (!ok && nchunks > 0) failed = true;
  } else if (warp == 8 || warp == 9) {
    // ======================================================= Wk(c) (lanes 0..63) -> bf16 rows 0..63 of [Wk; Q'](c)
    bool ok = true;
    const int t = 32 * q4 + lane;
    for (int c = 0; c < nchunks && ok; ++c) {
      // Wk(c) is done; U'(c - 1) is formed (so D1(c - 1) is done: it read this tile's buffer two chunks
      // ago, and the chain has seen wkconv(c - 1) before wkconv(c) can complete). Starting only then
      // keeps these warps off their sub-partitions while quadrants 0 and 1 form U'.
      ok = wait_idle(&bar_wk, par(c)) && (c == 0 || wait(&bar_ufree, par(c - 1)));
      if (!ok) break;
      tc_fence_after();
      uint8_t* const qt = qb(c);
      const float nc = -1.f;  // the rows are -Wk: D1 accumulates onto U0
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {  // two halves of 64 columns
        uint32_t xr[2][32];
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) tmem_ld32_issue(tmem + lane_base + Ly::TM_WK + 64 * hb + 32 * cb, xr[cb]);
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) tmem_wait_ld(xr[cb]);
        if (hb == 1) {  // every load of Wk(c) is complete: TM_WK is free for Wk(c + 1)
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&bar_wkfree);
        }
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) {
          const int col = 64 * hb + 32 * cb;
          const float* x = reinterpret_cast<const float*>(xr[cb]);
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            const float* y = x + 8 * q8;
            uint4 pk = make_uint4(pack_bf16(nc * y[0], nc * y[1]), pack_bf16(nc * y[2], nc * y[3]),
                                  pack_bf16(nc * y[4], nc * y[5]), pack_bf16(nc * y[6], nc * y[7]));
            *reinterpret_cast<uint4*>(qt + canon_chunk(t, col / 8 + q8, 128)) = pk;
          }
        }
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_wkconv);
    }
    if (!ok && nchunks > 0) failed = true;
  } else if (warp < 8) {
    // ======================================================= the state chain, warps 0..7: warp (q4, ch)
    // covers lanes 32 q4 .. +31 and value columns ch NV / 2 .. + NV / 2
    constexpr int NCB = NV / 64;  // 32-column blocks per warp
    const uint32_t id_nv = idesc_bf16(128, NV, 0, 1);
    const uint32_t id_state = idesc_bf16(128, NV, 1, 1);
    const int cw = ch * (NV / 2);  // this warp's first column
    bool issued = false;           // thread 0 has issued products (the drain then waits for them)
    // accumulator of chunk c: U0, then U0 - Wk S (rows 0..63; U' = c (U0 - Wk S)) and Q' S + P' U'
    // (rows 64..127)
    auto tm_u = [&](int c) -> uint32_t { return tmem + Ly::TM_U + (c & 1) * NV; };
    // o rows of chunk c from rows 64..127 of its accumulator (quadrants 2, 3, meeting at barrier
    // kBarOut), once O(c) is done: scaled by os (this row's o scale, read while the chunk's factor
    // record was in), rounded and staged in shared memory, then written by one TMA store per 64
    // columns (the tensor map clips the rows past the sequence's end); thread 64 issues the stores.
    // Every thread of quadrants 2 and 3 calls it with its failure state (the barrier takes all 128).
    auto store_o = [&](int c, bool ok_in, float os) -> bool {
      bool okw = ok_in && wait(&bar_o[c & 1], par2(c));
      if (tid == 64) bulk_wait_read_all();  // the previous chunk's store has read the staging tile
      if (group_or(kBarOut, 128, !okw)) return false;
      tc_fence_after();
      const int t = 32 * (q4 - 2) + lane;
      uint32_t xr[NCB][32];
#pragma unroll
      for (int cb = 0; cb < NCB; ++cb) tmem_ld32_issue(tm_u(c) + lane_base + cw + 32 * cb, xr[cb]);
#pragma unroll
      for (int cb = 0; cb < NCB; ++cb) tmem_wait_ld(xr[cb]);
#pragma unroll
      for (int cb = 0; cb < NCB; ++cb) {
        const int col = cw + 32 * cb;
#pragma unroll
        for (int q8 = 0; q8 < 4; ++q8) {
          const float* x = reinterpret_cast<const float*>(xr[cb]) + 8 * q8;
          uint4 pk = make_uint4(pack_bf16(os * x[0], os * x[1]), pack_bf16(os * x[2], os * x[3]),
                                pack_bf16(os * x[4], os * x[5]), pack_bf16(os * x[6], os * x[7]));
          *reinterpret_cast<uint4*>(sm + Ly::OST + canon_chunk(t, col / 8 + q8, C)) = pk;
        }
      }
      fence_proxy_async();
      tc_fence_before();
      group_sync(kBarOut, 128);
      if (tid == 64) {
#pragma unroll
        for (int x = 0; x < NV / 64; ++x) tma_store_4d(&tm_o, sm + Ly::OST + x * C * 128, col0 + 64 * x, h, c * C, b);
        bulk_commit();
      }
      return true;
    };
    // the chain's own barrier (warps 0..7); every thread brings its failure flag, all leave with the OR
    auto chain_sync = [&](bool bad) -> bool { return group_or(kBarChain, 256, bad); };

    // ok: this thread's waits so far succeeded; run: the group's vote at its last barrier (loops are left
    // only on a vote, so that every thread of the group reaches every barrier)
    bool ok = nchunks > 0, run = nchunks > 0;
    float os_prev = 0.f, os_cur = 0.f;  // o scales of this thread's row (quadrants 2, 3) for chunks c - 1, c
    for (int c = 0; run && c < nchunks; ++c) {
      // ---- the state entering chunk c -> bf16 operand tile; gamma_C S -> TM_S (fp32, where the state
      // update accumulates): after the state update of chunk c - 1
      if (ok && c > 0) ok = wait(&bar_os[(c - 1) & 1], par2(c - 1));
      ok = ok && wait(&bar_fr[c & 1], par2(c));
      if (ok) {
        tc_fence_after();
        const int k = 32 * q4 + lane;
        const float gl = frec(c)->glast;
        os_prev = os_cur;
        if (q4 >= 2) os_cur = frec(c)->orho[32 * (q4 - 2) + lane];
        uint32_t xr[NCB][32];  // every TMEM load of this thread in flight at once
        if (c == 0) {
#pragma unroll
          for (int cb = 0; cb < NCB; ++cb) {
            const float* src = a.S0 ? a.S0 + ((int64_t)bh * DK + k) * dv + col0 + cw + 32 * cb : nullptr;
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 f = src ? *reinterpret_cast<const float4*>(src + e) : make_float4(0.f, 0.f, 0.f, 0.f);
              xr[cb][e] = __float_as_uint(f.x), xr[cb][e + 1] = __float_as_uint(f.y);
              xr[cb][e + 2] = __float_as_uint(f.z), xr[cb][e + 3] = __float_as_uint(f.w);
            }
          }
        } else {
#pragma unroll
          for (int cb = 0; cb < NCB; ++cb) tmem_ld32_issue(tmem + lane_base + Ly::TM_S + cw + 32 * cb, xr[cb]);
#pragma unroll
          for (int cb = 0; cb < NCB; ++cb) tmem_wait_ld(xr[cb]);
        }
#pragma unroll
        for (int cb = 0; cb < NCB; ++cb) {
          const int col = cw + 32 * cb;
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
      fence_proxy_async();
      tc_fence_before();
      if (chain_sync(!ok)) {
        run = ok = false;
        break;
      }
      tc_fence_after();
      // ---- D1(c) = [-Wk; Q'](c) S, accumulated onto U0(c), once U0(c) is done, the Wk rows are
      // converted and the Q' and K' rows scaled
      if (tid == 0) {
        ok = wait(&bar_kconv, par(c)) && wait(&bar_wkconv, par(c)) && wait(&bar_u0, par(c));
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < DK; kk += 16) {
            const uint64_t ad = sdesc(smem_u32(qb(c)) + (kk >> 6) * (128 * 128) + (kk & 63) * 2, 16, 1024);
            const uint64_t bd = sdesc(smem_u32(sm + Ly::SMU) + kk * 128, DK * 128, 1024);
            mma_bf16(tm_u(c), ad, bd, id_nv, 1);
          }
          mma_commit(&bar_d1);
          issued = true;
        }
      }
      // ---- the previous chunk's o rows (quadrants 2, 3, idle until the next barrier): they lie in the
      // other accumulator, which U0(c + 1) overwrites only after this chunk's U' is formed
      if (c > 0 && q4 >= 2) ok = store_o(c - 1, ok, os_prev);
      // ---- U' = c (U0 - Wk S) (rows 0..63 of the accumulator) -> hi / lo tiles (the S tile is dead
      // once D1 is done)
      ok = ok && wait(&bar_d1, par(c));
      if (ok && q4 < 2) {
        tc_fence_after();
        const int t = 32 * q4 + lane;
        const float us = frec(c)->c[t];
        uint32_t ur[NCB][32];  // every TMEM load of this thread in flight at once
#pragma unroll
        for (int cb = 0; cb < NCB; ++cb) tmem_ld32_issue(tm_u(c) + lane_base + cw + 32 * cb, ur[cb]);
#pragma unroll
        for (int cb = 0; cb < NCB; ++cb) tmem_wait_ld(ur[cb]);
#pragma unroll
        for (int cb = 0; cb < NCB; ++cb) {
          const int col = cw + 32 * cb;
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 8 * q8 + 2 * e;
              split_bf16(us * __uint_as_float(ur[cb][i]), us * __uint_as_float(ur[cb][i + 1]), hi[e], lo[e]);
            }
            const uint32_t off = canon_chunk(t, col / 8 + q8, C);
            *reinterpret_cast<uint4*>(sm + Ly::SMU + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(sm + Ly::SMU + C * NV * 2 + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
          }
        }
      }
      fence_proxy_async();
      tc_fence_before();
      if (chain_sync(!ok)) {
        run = ok = false;
        break;
      }
      tc_fence_after();
      // ---- O += P' U' (rows 64..127 of the accumulator) -> bar_o; then S_acc += K'^T U' (hi and lo)
      // -> bar_os, which so also covers O: the next framing overwrites the U' tiles
      if (tid == 0) {
        ok = wait(&bar_p[c & 1], par2(c));
        if (ok) {
          tc_fence_after();
          const uint32_t pa = smem_u32(pbuf(c)) - C * C * 2;  // rows 64..127 of this operand are P'
#pragma unroll
          for (int kk = 0; kk < C; kk += 16)
            mma_bf16(tm_u(c), sdesc(pa + kk * 2, 16, 1024), sdesc(smem_u32(sm + Ly::SMU) + kk * 128, C * 128, 1024),
                     id_nv, 1);
          mma_commit(&bar_o[c & 1]);
          const uint32_t kt = smem_u32(kb(c));
#pragma unroll
          for (int kk = 0; kk < C; kk += 16) {
            const uint64_t ak = sdesc(kt + kk * 128, C * 128, 1024);
            mma_bf16(tmem + Ly::TM_S, ak, sdesc(smem_u32(sm + Ly::SMU) + kk * 128, C * 128, 1024), id_state, 1);
            mma_bf16(tmem + Ly::TM_S, ak, sdesc(smem_u32(sm + Ly::SMU + C * NV * 2) + kk * 128, C * 128, 1024),
                     id_state, 1);
          }
          mma_commit(&bar_os[c & 1]);
          mbar_arrive(&bar_ufree);  // U'(c) is formed
        }
      }
    }
    if (run) {  // (a group decision: every o-storing thread enters the barrier in store_o)
      // the last chunk's o rows and S_T = S_acc
      if (q4 >= 2) ok = store_o(nchunks - 1, ok, os_cur);
      ok = ok && wait(&bar_os[(nchunks - 1) & 1], par2(nchunks - 1));
      if (ok) {
        tc_fence_after();
        const int k = 32 * q4 + lane;
#pragma unroll
        for (int cb = 0; cb < NCB; ++cb) {
          const int col = cw + 32 * cb;
          float x[32];
          tmem_ld32(tmem + lane_base + Ly::TM_S + col, x);
          float* dst = a.S + ((int64_t)bh * DK + k) * dv + col0 + col;
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(dst + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
        }
      }
    }
    if (tid == 64) bulk_wait_all();  // the o stores are complete before the CTA leaves
    if (!ok && nchunks > 0) failed = true;
    if (!ok && tid == 0 && issued) {
      // drain: every tensor-core product thread 0 issued (one commit tracks them all)
      mma_commit(&bar_drain);
      mbar_wait_bounded(&bar_drain, 0, kDrainNs);
    }
  }
  if (failed && (tid & 31) == 0) atomicExch(a.status, kDevTimeout);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side
template <bool BV>
cudaError_t launch_xform(const Args& a, const CUtensorMap& mq, const CUtensorMap& mk, uint8_t* ws, cudaStream_t s) {
  const int smem = kXformSmem + 1024;
  cudaError_t e = cudaFuncSetAttribute(xform_sc_kernel<BV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t nblk = (int64_t)a.B * a.H * ((a.T + C - 1) / C);
  // blocks resident at once: a block's successor on its SM slot is about this many blocks later
  int dev = 0, sms = 148, per_sm = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, xform_sc_kernel<BV>, kThreads, smem) != cudaSuccess)
    per_sm = 0;
  xform_sc_kernel<BV><<<(unsigned)nblk, kThreads, smem, s>>>(mq, mk, a, ws, sms * per_sm);
  return cudaGetLastError();
}

template <int NV>
cudaError_t launch_chain(const Args& a, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& mo, const uint8_t* ws, cudaStream_t s) {
  const int smem = CLayout<NV>::TOTAL + 1024;
  cudaError_t e = cudaFuncSetAttribute(chain_sc_kernel<NV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  chain_sc_kernel<NV><<<a.B * a.H * (a.dv / NV), kChainThreads, smem, s>>>(mq, mk, mv, mo, a, ws,
                                                                       a.beta_v != DN_GATE_ONE ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace

size_t split_sc_workspace_bytes(const Args& a) {
  return (size_t)a.B * a.H * ((a.T + C - 1) / C) * rec_stride(a.beta_v != DN_GATE_ONE);
}

cudaError_t launch_split_sc(const Args& a, void* workspace, cudaStream_t s) {
  CUtensorMap mq, mk, mv, mo;
  if (!make_bthd_map(&mq, a.q, DK, a.H, a.T, a.B, C) || !make_bthd_map(&mk, a.k, DK, a.H, a.T, a.B, C) ||
      !make_bthd_map(&mv, a.v, a.dv, a.H, a.T, a.B, C) || !make_bthd_map(&mo, a.o, a.dv, a.H, a.T, a.B, C))
    return cudaErrorInvalidValue;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t e = (a.beta_v != DN_GATE_ONE) ? launch_xform<true>(a, mq, mk, ws, s) : launch_xform<false>(a, mq, mk, ws, s);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const bool split = a.dv == 128 && (int64_t)a.B * a.H * 2 <= sms;
  if (a.dv == 128 && !split) return launch_chain<128>(a, mq, mk, mv, mo, ws, s);
  return launch_chain<64>(a, mq, mk, mv, mo, ws, s);
}

}  // namespace dn
