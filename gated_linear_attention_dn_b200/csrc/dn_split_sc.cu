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

// global -> shared bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned)
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// L2 prefetches: a tile of a tensor map, and a range of global memory (16-byte aligned, multiple of 16)
__device__ __forceinline__ void tma_prefetch_4d(const CUtensorMap* map, int x, int y, int z, int w) {
  asm volatile("cp.async.bulk.prefetch.tensor.4d.L2.global [%0, {%1, %2, %3, %4}];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(x), "r"(y), "r"(z), "r"(w)
               : "memory");
}

__device__ __forceinline__ void bulk_prefetch(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
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
template <bool BV>
struct XLayout {
  static constexpr int KQ = 0;               // [K; Q] bf16 [128][DK] (TMA); after the Gram: fp32 L and T (64 x 64 each)
  static constexpr int TG = KQ + 128 * DK * 2;  // T Diag(gamma) [64][64]
  static constexpr int PB = TG + C * C * 2;     // P' [64][64]
  static constexpr int TB = PB + C * C * 2;     // T Diag(beta^v) [64 or 128][64]
  static constexpr int TOTAL = TB + tb_bytes(BV);
  static_assert(TG - KQ >= 2 * C * C * 4, "L and T fit over the [K; Q] tile");
  static_assert(TOTAL - TG == rec_factor_off(BV), "record tiles are contiguous");
};

template <bool BV>
__global__ void __launch_bounds__(kThreads) xform_sc_kernel(const __grid_constant__ CUtensorMap tm_q,
                                                            const __grid_constant__ CUtensorMap tm_k, const Args a,
                                                            uint8_t* ws) {
  using Ly = XLayout<BV>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  __shared__ __align__(8) uint64_t bar_kq, bar_g;
  __shared__ uint32_t s_tmem;
  __shared__ __align__(16) float s_Y[2048];
  __shared__ scf::Factors s_f;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, q4 = warp & 3, gch = warp >> 2;
  const int pre = a.pre_read ? 1 : 0;
  const int nchunks = (a.T + C - 1) / C;
  const int bh = blockIdx.x / nchunks, c = blockIdx.x % nchunks, b = bh / a.H, h = bh % a.H;
  uint8_t* const rec = ws + (size_t)blockIdx.x * rec_stride(BV);

  if (tid == 0) {
    mbar_init(&bar_kq, 1);
    mbar_init(&bar_g, 1);
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&s_tmem, 64);
  // the 8x8 blocks above the block diagonal of the T tiles (the inverse does not write them)
  for (int e = tid; e < 64 * 8; e += kThreads) {
    const int t = e >> 3, x8 = e & 7;
    if (x8 > (t >> 3)) {
      *reinterpret_cast<uint4*>(sm + Ly::TG + canon_chunk(t, x8, 128)) = make_uint4(0, 0, 0, 0);
      *reinterpret_cast<uint4*>(sm + Ly::TB + canon_chunk(t, x8, 128)) = make_uint4(0, 0, 0, 0);
      if (BV) *reinterpret_cast<uint4*>(sm + Ly::TB + canon_chunk(64 + t, x8, 128)) = make_uint4(0, 0, 0, 0);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  if (tid == 0) {
    mbar_expect_tx(&bar_kq, 2u * C * DK * 2);
#pragma unroll
    for (int x = 0; x < DK / 64; ++x) {
      tma_load_4d(sm + Ly::KQ + x * 128 * 128, &tm_k, &bar_kq, 64 * x, h, c * C, b);
      tma_load_4d(sm + Ly::KQ + x * 128 * 128 + 64 * 128, &tm_q, &bar_kq, 64 * x, h, c * C, b);
    }
  }
  if (tid < 64) scf::token_factors(scf::load_gates(a, b, h, c, tid), tid, lane, pre, s_f);
  __syncthreads();
  if (tid < 64) {
    Rec* r = reinterpret_cast<Rec*>(rec + rec_factor_off(BV));
    r->c[tid] = s_f.c[tid];
    r->orho[tid] = s_f.orho[tid];
    r->oex[tid] = s_f.oex[tid];
    r->n[tid] = s_f.n[tid];
    if (tid == 0) r->glast = s_f.glast;
  }
  // Gram [K; Q] K^T -> tensor memory (M 128, N 64, K 128)
  bool ok = true, issued = false;
  if (tid == 0) {
    ok = mbar_wait_bounded(&bar_kq, 0, a.wait_ns);
    if (ok) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 64, 0, 0);
#pragma unroll
      for (int kk = 0; kk < DK; kk += 16) {
        const uint64_t d = sdesc(smem_u32(sm + Ly::KQ) + (kk >> 6) * (128 * 128) + (kk & 63) * 2, 16, 1024);
        mma_bf16(tmem, d, d, id, kk > 0);
      }
      mma_commit(&bar_g);
      issued = true;
    }
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
  // A and P' (the [K; Q] tile is free now: L and T take its place)
  float* sL = reinterpret_cast<float*>(sm + Ly::KQ);
  float* sT = sL + C * C;
  scf::extract_ap(s_f, tmem, q4, gch, lane, pre, sL, sm + Ly::PB);
  tc_fence_before();
  __syncthreads();
  unit_lower_inverse<true, 8, true, BV>(sL, sT, s_Y, sm + Ly::TG, sm + Ly::TB, s_f.gam, s_f.bv, tid, 0);
  __syncthreads();
  // the tiles to the record, 16 bytes per thread and step
  {
    const uint4* src = reinterpret_cast<const uint4*>(sm + Ly::TG);
    uint4* dst = reinterpret_cast<uint4*>(rec);
    for (int i = tid; i < rec_factor_off(BV) / 16; i += kThreads) dst[i] = src[i];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 64);
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
  static constexpr int TB = PB1 + C * C * 2;       // T Diag(beta^v) [128][64] (lo rows 64..127, or zero)
  static constexpr int OST = TB + 128 * C * 2;     // o rows of a chunk [C][NV] bf16, staged for the TMA store
  static constexpr int SMU = OST + C * NV * 2;     // S bf16 [DK][NV]; after D1: U' hi, U' lo [C][NV]
  static constexpr int SMU_BYTES = (DK * NV * 2 > 2 * C * NV * 2) ? DK * NV * 2 : 2 * C * NV * 2;
  static constexpr int FR0 = SMU + SMU_BYTES;      // factor records of parity 0 and 1
  static constexpr int FR1 = FR0 + 1088;
  static constexpr int TOTAL = FR1 + 1088;
  // the lo operand of T Diag(beta^v) reads 64 rows past TB: they lie in OST
  static_assert(C * NV * 2 >= 64 * C * 2, "operand overrun stays in shared memory");
  static_assert(TOTAL + 1024 + 4096 <= 227 * 1024, "shared memory budget");
  static constexpr int TM_S = 0, TM_D1 = NV, TM_U0 = 2 * NV, TM_WK = 3 * NV;
  static_assert(TM_WK + DK <= 512, "tensor memory budget");
};

// Warp roles. Warp w runs on SM sub-partition w % 4 and reaches tensor-memory lanes 32 (w % 4) ..
// +31, so the work is placed by lane quadrant:
//  * warps 0..7 run the state chain of each chunk: all of them frame the state (S rows are all 128
//    lanes) and meet at a barrier, after which thread 0 issues D1 = [Wk; Q'] S (warp 0 has nothing to
//    do until D1 is done anyway); quadrants 0 and 1 form U' (rows 0..63 of D1 and U0) and the group
//    meets again, after which thread 0 issues O += P' U' (rows 64..127 of D1; the o rows leave as soon
//    as it is done), then the state update (the next chunk's framing waits for it); quadrants 0 and 1
//    then convert the next chunk's Wk (lanes 0..63) and scale its q rows to Q', while quadrants 2 and 3
//    store the o rows;
//  * warp 11 (quadrant 3) scales the k rows of each chunk to K' (shared memory only);
//  * lane 0 of warp 10 issues every load (and L2 prefetches further ahead) and the state-independent
//    products of the next chunk, Wk(c + 1) and U0(c + 1), as soon as thread 0 signals that their
//    tensor memory is free (so their issue stalls never hold the chain's warps);
//  * warps 8 and 9 only place warps 10 and 11 on their sub-partitions.
// Hand-overs across warps go through mbarriers; within warps 0..7 through a named barrier.
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
  constexpr int NCB = NV / 64;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = align1024(smem_raw);
  // loads (transaction counts); products (commits); hand-overs (arrivals)
  __shared__ __align__(8) uint64_t bar_kq[2], bar_fr[2], bar_tg, bar_vb, bar_p[2];
  // (the state update, the O product and the o stores of chunk c complete barrier [c & 1]: the loader
  // looks at them a chunk later than the chain, which can never lap it by two chunks)
  __shared__ __align__(8) uint64_t bar_wk, bar_u0, bar_d1, bar_os[2], bar_o[2], bar_drain, bar_drain2;
  __shared__ __align__(8) uint64_t bar_kconv, bar_ostored[2], bar_wkfree, bar_ufree;
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
      mbar_init(&bar_ostored[j], 1);  // the thread that issues the o tile's store
    }
    mbar_init(&bar_tg, 1);
    mbar_init(&bar_vb, 1);
    mbar_init(&bar_wk, 1);
    mbar_init(&bar_u0, 1);
    mbar_init(&bar_d1, 1);
    mbar_init(&bar_drain, 1);
    mbar_init(&bar_drain2, 1);
    mbar_init(&bar_wkfree, 1);   // thread 0: chunk c's Wk is converted (TM_WK free)
    mbar_init(&bar_ufree, 1);    // thread 0: chunk c's U' is formed (TM_U0 free)
    mbar_init(&bar_kconv, 1);    // the k-scaling warp
    fence_mbar_init();
  }
  if (warp == 0) tmem_alloc(&s_tmem, 512);
  if (!bv_split) {  // no lo part: rows 64..127 of the T Diag(beta^v) tile stay zero
    for (int i = tid; i < 64 * C * 2 / 16; i += kChainThreads)
      reinterpret_cast<uint4*>(sm + Ly::TB + 64 * 128)[i] = make_uint4(0, 0, 0, 0);
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
        bulk_load(sm + Ly::TB, rec(c) + kRecTB, tbb, &bar_vb);
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
      // Wk(c) = (T Diag gamma) K(c) -> TM_WK (lanes 0..63); U0(c) = (T Diag beta^v) V(c) -> TM_U0
      auto mma_wk = [&](int c) {
#pragma unroll
        for (int kk = 0; kk < C; kk += 16) {
          const uint64_t ad = sdesc(smem_u32(sm + Ly::TG) + kk * 2, 16, 1024);
          const uint64_t bk = sdesc(smem_u32(kb(c)) + kk * 128, C * 128, 1024);
          mma_bf16(tmem + Ly::TM_WK, ad, bk, id_wk, kk > 0);
        }
        mma_commit(&bar_wk);
      };
      auto mma_u0 = [&](int c) {
        const uint32_t tb = smem_u32(sm + Ly::TB), vb = smem_u32(sm + Ly::VB);
        (void)c;
#pragma unroll
        for (int kk = 0; kk < C; kk += 16)
          mma_bf16(tmem + Ly::TM_U0, sdesc(tb + kk * 2, 16, 1024), sdesc(vb + kk * 128, C * 128, 1024), id_nv, kk > 0);
        if (bv_split) {
#pragma unroll
          for (int kk = 0; kk < C; kk += 16)
            mma_bf16(tmem + Ly::TM_U0, sdesc(tb + 64 * 128 + kk * 2, 16, 1024), sdesc(vb + kk * 128, C * 128, 1024),
                     id_nv, 1);
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
      // Wk(c + 1) has read chunk c + 1's; U0(c + 1) once U'(c) is formed; the buffers of chunk c once
      // its products have read them (k, q: the state update; v, T Diag(beta^v): U0(c); P': the O
      // product) and its factor record once its o rows are out
      for (int c = 0; c < nchunks && ok; ++c) {
        const bool more = c + 1 < nchunks;
        if (c == 0 && more) {
          ok = wait_idle(&bar_wk, par(0));  // T Diag(gamma) of chunk 0 has been read
          if (!ok) break;
          issue_tg(1);
        }
        if (more) {
          ok = wait_idle(&bar_wkfree, par(c)) && wait_idle(&bar_tg, par(c + 1)) && wait_idle(&bar_kq[(c + 1) & 1], par2(c + 1));
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
          ok = wait_idle(&bar_ostored[c & 1], par2(c));
          if (!ok) break;
          issue_fr(c + 2);
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
    // ======================================================= k rows of each chunk -> K' = 2^{n} k
    bool ok = true;
    for (int c = 0; c < nchunks && ok; ++c) {
      // its k tile and factors have landed, and Wk(c) has read the raw k rows
      ok = wait_idle(&bar_kq[c & 1], par2(c)) && wait_idle(&bar_fr[c & 1], par2(c)) && wait_idle(&bar_wk, par(c));
      if (!ok) break;
      const Rec* fr = frec(c);
      uint8_t* const kt = kb(c);
      // in batches of 8 loads before their stores
#pragma unroll 1
      for (int j0 = 0; j0 < 32; j0 += 8) {
        uint4 kv[8];
        float sc[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int e = lane + 32 * (j0 + j), i = e >> 4;
          kv[j] = *reinterpret_cast<const uint4*>(kt + canon_chunk(i, e & 15, C));
          sc[j] = pow2f(fr->n[i]);
        }
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int e = lane + 32 * (j0 + j), i = e >> 4;
          *reinterpret_cast<uint4*>(kt + canon_chunk(i, e & 15, C)) = scale_bf16x8(kv[j], sc[j]);
        }
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_kconv);
    }
    if (!ok && nchunks > 0) failed = true;
  } else if (warp < 8) {
    // ======================================================= the state chain, warps 0..7
    const uint32_t id_nv = idesc_bf16(128, NV, 0, 1);
    const uint32_t id_state = idesc_bf16(128, NV, 1, 1);
    bool issued = false;  // thread 0 has issued products (the drain then waits for them)
    // chunk c's Wk (lanes 0..63) -> bf16 rows 0..63 of its [Wk; Q'] tile and its q rows scaled to
    // Q' = 2^{oex} q (rows 64..127): quadrants 0 and 1, once Wk(c), k, q and the factors are in
    auto convert = [&](int c) -> bool {
      if (q4 >= 2) return true;
      if (!(wait(&bar_wk, par(c)) && wait(&bar_kq[c & 1], par2(c)) && wait(&bar_fr[c & 1], par2(c)))) return false;
      tc_fence_after();
      uint8_t* const qt = qb(c);
      const int t = 32 * q4 + lane;
      {
        uint4 qv[8];  // this thread's half row of q: every load in flight before any store
#pragma unroll
        for (int j = 0; j < 8; ++j) qv[j] = *reinterpret_cast<const uint4*>(qt + canon_chunk(64 + t, 8 * ch + j, 128));
        const float sc = pow2f(frec(c)->oex[t]);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4*>(qt + canon_chunk(64 + t, 8 * ch + j, 128)) = scale_bf16x8(qv[j], sc);
      }
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
          *reinterpret_cast<uint4*>(qt + canon_chunk(t, col / 8 + q8, 128)) = pk;
        }
      }
      return true;
    };
    // o rows of chunk c from rows 64..127 of D1 (quadrants 2, 3, meeting at barrier kBarOut), once O(c)
    // is done: scaled, rounded and staged in shared memory, then written by one TMA store per 64
    // columns (the tensor map clips the rows past the sequence's end); thread 64 issues the stores.
    // Every thread of quadrants 2 and 3 calls it with its failure state (the barrier takes all 128).
    auto store_o = [&](int c, bool ok_in) -> bool {
      bool okw = ok_in && wait(&bar_o[c & 1], par2(c));
      if (tid == 64) bulk_wait_read_all();  // the previous chunk's store has read the staging tile
      if (group_or(kBarOut, 128, !okw)) return false;
      tc_fence_after();
      const int t = 32 * (q4 - 2) + lane;
      const float os = frec(c)->orho[t];
      uint32_t xr[NCB][32];
#pragma unroll
      for (int cb = 0; cb < NCB; ++cb) tmem_ld32_issue(tmem + lane_base + Ly::TM_D1 + ch * (NV / 2) + 32 * cb, xr[cb]);
#pragma unroll
      for (int cb = 0; cb < NCB; ++cb) tmem_wait_ld(xr[cb]);
#pragma unroll
      for (int cb = 0; cb < NCB; ++cb) {
        const int col = ch * (NV / 2) + 32 * cb;
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
        mbar_arrive(&bar_ostored[c & 1]);  // the factor record's o scales have been read
      }
      return true;
    };
    // the chain's own barrier (warps 0..7); every thread brings its failure flag, all leave with the OR
    auto chain_sync = [&](bool bad) -> bool { return group_or(kBarChain, 256, bad); };

    // ok: this thread's waits so far succeeded; run: the group's vote at its last barrier (loops are left
    // only on a vote, so that every thread of the group reaches every barrier)
    bool ok = nchunks > 0, run = false;
    // ---- prologue: chunk 0's conversions
    if (ok) {
      ok = convert(0);
      fence_proxy_async();
      tc_fence_before();
      run = ok = !chain_sync(!ok);
      tc_fence_after();
    }
    for (int c = 0; run && c < nchunks; ++c) {
      const bool more = c + 1 < nchunks;
      // ---- the previous chunk's o rows (quadrants 2, 3): O(c - 1) is done before the state update of
      // chunk c - 1, which they overlap; D1(c) overwrites their rows after the next barrier
      if (c > 0 && q4 >= 2) ok = store_o(c - 1, ok);
      // ---- the state entering chunk c -> bf16 operand tile; gamma_C S -> TM_S (fp32, where the state
      // update accumulates): after the state update of chunk c - 1
      if (ok && c > 0) ok = wait(&bar_os[(c - 1) & 1], par2(c - 1));
      ok = ok && wait(&bar_fr[c & 1], par2(c));
      if (ok) {
        tc_fence_after();
        const int k = 32 * q4 + lane;
        const float gl = frec(c)->glast;
        uint32_t xr[NCB][32];  // every TMEM load of this thread in flight at once
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
      fence_proxy_async();
      tc_fence_before();
      if (chain_sync(!ok)) {
        run = ok = false;
        break;
      }
      tc_fence_after();
      // ---- D1(c) = [Wk; Q'](c) S (its K' rows are scaled too); TM_WK is free for Wk(c + 1)
      if (tid == 0) {
        ok = wait(&bar_kconv, par(c));
        if (ok) {
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < DK; kk += 16) {
            const uint64_t ad = sdesc(smem_u32(qb(c)) + (kk >> 6) * (128 * 128) + (kk & 63) * 2, 16, 1024);
            const uint64_t bd = sdesc(smem_u32(sm + Ly::SMU) + kk * 128, DK * 128, 1024);
            mma_bf16(tmem + Ly::TM_D1, ad, bd, id_nv, kk > 0);
          }
          mma_commit(&bar_d1);
          issued = true;
          mbar_arrive(&bar_wkfree);
        }
      }
      // ---- U' = c (U0 - Wk S) -> hi / lo tiles (the S tile is dead once D1 is done)
      ok = ok && wait(&bar_d1, par(c)) && wait(&bar_u0, par(c));
      if (ok && q4 < 2) {
        tc_fence_after();
        const int t = 32 * q4 + lane;
        const float us = frec(c)->c[t];
        uint32_t u0r[NCB][32], d1r[NCB][32];  // every TMEM load of this thread in flight at once
#pragma unroll
        for (int cb = 0; cb < NCB; ++cb) {
          tmem_ld32_issue(tmem + lane_base + Ly::TM_U0 + ch * (NV / 2) + 32 * cb, u0r[cb]);
          tmem_ld32_issue(tmem + lane_base + Ly::TM_D1 + ch * (NV / 2) + 32 * cb, d1r[cb]);
        }
#pragma unroll
        for (int cb = 0; cb < NCB; ++cb) {
          tmem_wait_ld(u0r[cb]);
          tmem_wait_ld(d1r[cb]);
        }
#pragma unroll
        for (int cb = 0; cb < NCB; ++cb) {
          const int col = ch * (NV / 2) + 32 * cb;
#pragma unroll
          for (int q8 = 0; q8 < 4; ++q8) {
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int i = 8 * q8 + 2 * e;
              split_bf16(us * (__uint_as_float(u0r[cb][i]) - __uint_as_float(d1r[cb][i])),
                         us * (__uint_as_float(u0r[cb][i + 1]) - __uint_as_float(d1r[cb][i + 1])), hi[e], lo[e]);
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
      // ---- O += P' U' (rows 64..127 of D1) -> bar_o; then S_acc += K'^T U' (hi and lo) -> bar_os, which
      // so also covers O: the next framing overwrites the U' tiles; then U0(c + 1)
      if (tid == 0) {
        ok = wait(&bar_p[c & 1], par2(c));
        if (ok) {
          tc_fence_after();
          const uint32_t pa = smem_u32(pbuf(c)) - C * C * 2;  // rows 64..127 of this operand are P'
#pragma unroll
          for (int kk = 0; kk < C; kk += 16)
            mma_bf16(tmem + Ly::TM_D1, sdesc(pa + kk * 2, 16, 1024),
                     sdesc(smem_u32(sm + Ly::SMU) + kk * 128, C * 128, 1024), id_nv, 1);
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
          mbar_arrive(&bar_ufree);  // TM_U0 is free: U'(c) has been formed
        }
      }
      // ---- chunk c + 1's conversions (quadrants 0, 1) while the products of chunk c run; a failure here
      // reaches the group at its next barrier
      if (ok && more) ok = convert(c + 1);
    }
    if (run) {  // (a group decision: every o-storing thread enters the barrier in store_o)
      // the last chunk's o rows and S_T = S_acc
      if (q4 >= 2) ok = store_o(nchunks - 1, ok);
      ok = ok && wait(&bar_os[(nchunks - 1) & 1], par2(nchunks - 1));
      if (ok) {
        tc_fence_after();
        const int k = 32 * q4 + lane;
#pragma unroll
        for (int cb = 0; cb < NCB; ++cb) {
          const int col = ch * (NV / 2) + 32 * cb;
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
  const int smem = XLayout<BV>::TOTAL + 1024;
  cudaError_t e = cudaFuncSetAttribute(xform_sc_kernel<BV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int64_t nblk = (int64_t)a.B * a.H * ((a.T + C - 1) / C);
  xform_sc_kernel<BV><<<(unsigned)nblk, kThreads, smem, s>>>(mq, mk, a, ws);
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
