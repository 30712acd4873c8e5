// OSDN phase 1: the diagonal preconditioner sequence d_t of every (b, h) (OSDN page, section 2.2
// "decoupled hypergradient feedback", two-phase implementation item 1, and section 2.3 "adaptive
// preconditioner forgetting"). Token t is written with d_t (the key scale d of the main
// recurrence); then, with a_t = k_t (.) k_t,
//   e_t = c_t (1 - beta_t <d_t, a_t>),  c_t = eta beta_t / ||k_t||^2   (0 when k_t = 0)
//   d_{t+1} = r_t d_t + e_t a_t
// which is d_{t+1} = r_t d_t - eta grad h_t(d_t) for the closed-form surrogate
// h_t(d) = ((1 - beta_t <d, a_t>)^2 - 1) / (2 ||k_t||^2) (r_t = 1 without forgetting).
//
// The only sequential dependence is the scalar <d_t, a_t>. Over a block of m = 32 tokens
// starting at t0, with rho_t = prod_{t0<=j<t} r_j, R(i+1, t) = prod_{i<j<t} r_j, G = Gram of the a_t,
// W_ti = R(i+1, t) G_ti (i < t) and P_t = <d_{t0}, a_t>:
//   <d_t, a_t> = rho_t P_t + sum_{i<t} W_ti e_i
//   => (I + Diag(c beta) W) e = c - Diag(c beta rho) P
//   => e = u0 - B P,  u0 = T c,  B = T Diag(c beta rho),  T = (I + Diag(c beta) W)^{-1}.
// u0 and B do not depend on d, so they are formed for all blocks of all heads at once
// (osdn_block_kernel, one warp per block, into the caller's workspace). The scan
// (osdn_scan_kernel, one CTA per (b, h), two threads per key channel) then needs per block only
// P (transposed warp reductions), e = u0 - B P (one warp), and the per-channel recurrences that
// write d_t for the 32 tokens, in two halves of 16 that run at once; the next blocks' k tiles,
// B and u0 arrive ahead through a cp.async ring.
#include <mutex>

#include "dn_common.cuh"
#include "dn_tc_ptx.cuh"

namespace dn {
namespace {

constexpr int kM = 32;              // tokens per block
constexpr int kBlockFloats = kM * kM + kM;  // B (column-major: element (t, s) at s * 32 + t), then u0

__device__ __forceinline__ float load_k(const void* k, int64_t i, int bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(k)[i]);
  return reinterpret_cast<const float*>(k)[i];
}

// ------------------------------------------------------------------ block kernel
// 4 warps per CTA, one block of 32 tokens per warp; lane t = token t0 + t.
template <int DK>
struct BlockSmem {
  static constexpr int AP = DK + 4;  // padded row of a (16-byte aligned, spreads rows over banks)
  static constexpr int A = kM * AP, L = kM * (kM + 1);
  static constexpr int BYTES = 4 * (A + L) * (int)sizeof(float);  // 4 warps
};

template <int DK>
__global__ void __launch_bounds__(128) osdn_block_kernel(const void* k, const float* beta, const float* ret,
                                                         float eta, int B, int T, int H, int io_bf16,
                                                         float* ws) {
  using Sm = BlockSmem<DK>;
  constexpr int AP = Sm::AP;
  extern __shared__ __align__(16) float smem_raw[];
  float* const smem = smem_raw;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nblk = (T + kM - 1) / kM;
  const int64_t blk = (int64_t)blockIdx.x * 4 + warp;
  if (blk >= (int64_t)B * H * nblk) return;  // whole warps only: no barrier below spans warps
  const int bh = (int)(blk / nblk), j = (int)(blk % nblk), b = bh / H, h = bh % H;
  const int t = j * kM + lane;
  const bool valid = t < T;
  float (*a)[AP] = reinterpret_cast<float (*)[AP]>(smem + warp * Sm::A);
  float (*L)[kM + 1] = reinterpret_cast<float (*)[kM + 1]>(smem + 4 * Sm::A + warp * Sm::L);

  // a_t = k_t (.) k_t, ||k_t||^2, c_t, beta_t, r_t (padding tokens: a = 0, c = 0, r = 1)
  float nrm = 0.f;
  const int64_t row = (((int64_t)b * T + t) * H + h) * DK;
  if (valid && io_bf16) {
    const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(k) + row);
    uint4 raw[DK / 8];  // the whole row in flight before any of it is used
#pragma unroll
    for (int c8 = 0; c8 < DK / 8; ++c8) raw[c8] = __ldg(src + c8);
#pragma unroll
    for (int c8 = 0; c8 < DK / 8; ++c8) {
      const uint4 u = raw[c8];
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      float v[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = __uint_as_float(w[e] << 16);
        v[2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float sq = v[e] * v[e];
        nrm += sq;
        a[lane][8 * c8 + e] = sq;
      }
    }
  } else {
    for (int c = 0; c < DK; ++c) {
      const float x = valid ? load_k(k, row + c, io_bf16) : 0.f;
      nrm += x * x;
      a[lane][c] = x * x;
    }
  }
  const int64_t tok = ((int64_t)b * T + t) * H + h;
  const float bt = valid ? beta[tok] : 0.f;
  const float rt = valid && ret ? ret[tok] : 1.f;
  const float ct = (valid && nrm > 0.f) ? eta * bt / nrm : 0.f;
  // rho_t = prod_{s<t} r_s within the block (exclusive product scan)
  float incl = rt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const float y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl *= y;
  }
  const float prev_incl = __shfl_up_sync(0xffffffffu, incl, 1);  // every lane takes part in the shuffle
  const float rho = lane == 0 ? 1.f : prev_incl;
  __syncwarp();

  // Gram row t: g[i] = <a_t, a_i>
  float g[kM];
#pragma unroll
  for (int i = 0; i < kM; ++i) g[i] = 0.f;
  for (int c4 = 0; c4 < DK; c4 += 4) {
    const float4 at = *reinterpret_cast<const float4*>(&a[lane][c4]);
#pragma unroll
    for (int i = 0; i < kM; ++i) {
      const float4 ai = *reinterpret_cast<const float4*>(&a[i][c4]);
      g[i] = fmaf(at.x, ai.x, fmaf(at.y, ai.y, fmaf(at.z, ai.z, fmaf(at.w, ai.w, g[i]))));
    }
  }
  // L_ti = c_t beta_t R(i+1, t) G_ti for i < t; R built from i = t - 1 downwards
  {
    const float cb = ct * bt;
    float R = 1.f;
#pragma unroll
    for (int i = kM - 1; i >= 0; --i) {
      const float ri = __shfl_sync(0xffffffffu, rt, i);
      if (i < lane) {
        L[lane][i] = cb * R * g[i];
        R *= ri;
      } else {
        L[lane][i] = 0.f;
      }
    }
  }
  __syncwarp();
  // T = (I + L)^{-1}: lane s forms column s by forward substitution
  float x[kM];
#pragma unroll
  for (int r = 0; r < kM; ++r) {
    float s0 = (r == lane) ? 1.f : 0.f, s1 = 0.f;
#pragma unroll
    for (int i = 0; i < r; ++i) {
      if (i & 1)
        s1 = fmaf(-L[r][i], x[i], s1);
      else
        s0 = fmaf(-L[r][i], x[i], s0);
    }
    x[r] = s0 + s1;
  }
  // B[:, s] = T[:, s] c_s beta_s rho_s (lane s writes column s, stored column-major so that the
  // scan's lanes read rows without bank conflicts); u0 = T c (row sums, through shared memory)
  float* out = ws + blk * kBlockFloats;
  const float colscale = ct * bt * rho;
  __syncwarp();
#pragma unroll
  for (int r = 0; r < kM; r += 4)
    *reinterpret_cast<float4*>(out + lane * kM + r) =
        make_float4(x[r] * colscale, x[r + 1] * colscale, x[r + 2] * colscale, x[r + 3] * colscale);
#pragma unroll
  for (int r = 0; r < kM; ++r) L[r][lane] = x[r] * ct;  // reuse L for T Diag(c)
  __syncwarp();
  float u0 = 0.f;
#pragma unroll
  for (int s = 0; s < kM; ++s) u0 += L[lane][s];
  out[kM * kM + lane] = u0;
}

// ------------------------------------------------------------------ scan kernel
// One CTA of 2 DK threads per (b, h): thread (half, ch) owns key channel ch of d over tokens
// 16 half .. +16 of every block (the second half starts from d at token 16, formed directly from the
// block's start state, the first half's e and its k rows). A ring of kStages shared-
// memory stages holds the k tile, B, u0 and retentions of the next blocks, copied with cp.async
// kStages - 1 blocks ahead (one commit group per block, empty past the end, so that a fixed
// wait_group count always means "this block's copies have landed").
constexpr int kStages = 4;

template <int DK, bool BF16>
struct ScanSmem {
  static constexpr int KT = kM * DK * (BF16 ? 2 : 4);  // k tile bytes
  static constexpr int BU = kBlockFloats * 4;          // B and u0
  static constexpr int RT = kM * 4;                    // retentions
  static constexpr int STAGE = KT + BU + RT;
  static constexpr int BYTES = kStages * STAGE;
  static_assert(KT % 16 == 0 && BU % 16 == 0 && STAGE % 16 == 0, "16-byte cp.async granularity");
};

template <int DK, bool BF16>
__global__ void __launch_bounds__(2 * DK) osdn_scan_kernel(const void* k, const float* ret, const float* d0, int B,
                                                           int T, int H, const float* ws, float* dout, float* dT) {
  using namespace tc;
  using Sm = ScanSmem<DK, BF16>;
  constexpr int NT = 2 * DK;   // two threads per key channel: tokens 0..15 and 16..31 of a block
  constexpr int NW = DK / 32;  // warps per half
  constexpr int HM = kM / 2;
  constexpr int ES = BF16 ? 2 : 4, ROW = DK * ES, ROW_CHUNKS = ROW / 16;
  extern __shared__ __align__(16) float smem_raw[];  // same declaration type as the block kernel's
  uint8_t* const smem = reinterpret_cast<uint8_t*>(smem_raw);
  __shared__ float s_part[2][NW][HM];
  __shared__ float s_e[kM];
  __shared__ float s_coef[HM];  // R(i + 1, 16) e_i: the first half's writes as seen at token 16
  __shared__ float s_rho16;     // prod_{j < 16} r_j
  __shared__ __align__(16) float s_d[DK];
  const int tid = threadIdx.x, ch = tid % DK, half = tid / DK, lane = tid & 31, wih = (tid % DK) >> 5;
  const int bh = blockIdx.x, b = bh / H, h = bh % H;
  const int nblk = (T + kM - 1) / kM;
  auto s_k = [&](int st) { return smem + st * Sm::STAGE; };
  auto s_bu = [&](int st) { return reinterpret_cast<float*>(smem + st * Sm::STAGE + Sm::KT); };
  auto s_r = [&](int st) { return reinterpret_cast<float*>(smem + st * Sm::STAGE + Sm::KT + Sm::BU); };
  auto k_at = [&](int st, int t) -> float {
    float x;
    if (BF16)
      x = __uint_as_float((uint32_t)reinterpret_cast<const unsigned short*>(s_k(st))[t * DK + ch] << 16);
    else
      x = reinterpret_cast<const float*>(s_k(st))[t * DK + ch];
    return x;
  };

  // copies of block j into stage j % kStages, committed as one group (an empty group past the end)
  auto issue = [&](int j) {
    if (j < nblk) {
      const int st = j % kStages, t0 = j * kM, nb = min(kM, T - t0);
      const uint8_t* kb = static_cast<const uint8_t*>(k);
      for (int c = tid; c < kM * ROW_CHUNKS; c += NT) {
        const int t = c / ROW_CHUNKS, part = c % ROW_CHUNKS;
        const bool v = t < nb;
        const uint8_t* src = v ? kb + (((int64_t)b * T + t0 + t) * H + h) * ROW + part * 16 : kb;
        cp_async_16_zfill(s_k(st) + t * ROW + part * 16, src, v ? 16u : 0u);
      }
      const float* wb = ws + ((int64_t)bh * nblk + j) * kBlockFloats;
      for (int c = tid; c < kBlockFloats / 4; c += NT) cp_async_16_zfill(s_bu(st) + 4 * c, wb + 4 * c, 16u);
      if (ret && tid < nb) cp_async_4(s_r(st) + tid, ret + ((int64_t)b * T + t0 + tid) * H + h);
    }
    cp_async_commit();
  };

  if (half == 0) s_d[ch] = d0 ? d0[(int64_t)bh * DK + ch] : 1.f;
#pragma unroll
  for (int j = 0; j < kStages - 1; ++j) issue(j);
  for (int j = 0; j < nblk; ++j) {
    const int st = j % kStages, t0 = j * kM, nb = min(kM, T - t0), tb = half * HM;
    cp_async_wait_group<kStages - 2>();
    __syncthreads();         // block j's tiles have landed; block j - 1 is done (its d_end is in s_d)
    issue(j + kStages - 1);  // into the stage block j - 1 used
    const float dstart = s_d[ch];
    float a[HM];
#pragma unroll
    for (int t = 0; t < HM; ++t) {
      const float x = k_at(st, tb + t);
      a[t] = x * x;
    }
    // the second half also takes the first half's a (its start d needs them after the last barrier)
    float a0[HM];
    if (half == 1) {
#pragma unroll
      for (int i = 0; i < HM; ++i) {
        const float x = k_at(st, i);
        a0[i] = x * x;
      }
    }
    // P_t = <d_{t0}, a_t> for this half's 16 tokens: a transposed butterfly over lanes 0..15's bit
    // pattern, then one exchange across lane bit 4; lane t (mod 16) ends with token t
    {
      float v[HM];
#pragma unroll
      for (int t = 0; t < HM; ++t) v[t] = dstart * a[t];
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) {
        const bool upper = (lane & off) != 0;
#pragma unroll
        for (int i = 0; i < off; ++i) {
          const float send = upper ? v[i] : v[i + off];
          const float keep = upper ? v[i + off] : v[i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
        }
      }
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], 16);
      if (lane < HM) s_part[half][wih][lane] = v[0];
    }
    __syncthreads();
    // e = u0 - B P (warp 0, lane t; B column-major), then the second half's start: R(i+1,16) e_i
    if (tid < 32) {
      // suffix products over lanes 0..15: suf_i = prod_{i<j<16} r_j (exclusive), rho16 = prod_{j<16} r_j
      // (they do not depend on P)
      const float rl = (ret && lane < HM) ? s_r(st)[lane] : 1.f;
      float incl = lane < HM ? rl : 1.f;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_down_sync(0xffffffffu, incl, off);
        if (lane + off < 32) incl *= y;
      }
      const float nxt = __shfl_down_sync(0xffffffffu, incl, 1);  // every lane takes part
      const float suf = lane == 31 ? 1.f : nxt;
      float P = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) P += s_part[lane / HM][w][lane % HM];
      // e_t = u0_t - sum_s B_ts P_s: P_s from lane s, four independent partial sums
      const float* bu = s_bu(st);
      float ep[4] = {bu[kM * kM + lane], 0.f, 0.f, 0.f};
#pragma unroll
      for (int s2 = 0; s2 < kM; ++s2)
        ep[s2 & 3] = fmaf(-bu[s2 * kM + lane], __shfl_sync(0xffffffffu, P, s2), ep[s2 & 3]);
      const float e = (ep[0] + ep[1]) + (ep[2] + ep[3]);
      s_e[lane] = e;
      if (lane < HM) s_coef[lane] = suf * e;
      if (lane == 0) s_rho16 = incl;
    }
    __syncthreads();
    // d_t for this half's tokens; the second half starts from d_{t0 + 16}
    // (every operand of the two dependent chains below is loaded first, so that each chain is a run
    // of fused multiply-adds and not a shared-memory round trip per token)
    float d;
    if (half == 0) {
      d = dstart;
    } else {
      float term[HM];
#pragma unroll
      for (int i = 0; i < HM; ++i) term[i] = s_coef[i] * a0[i];
      d = s_rho16 * dstart;
#pragma unroll
      for (int i = 0; i < HM; ++i) d += term[i];
    }
    float rt[HM], ea[HM];
    const float* rr = s_r(st);
#pragma unroll
    for (int t = 0; t < HM; ++t) {
      rt[t] = ret ? rr[tb + t] : 1.f;
      ea[t] = s_e[tb + t] * a[t];
    }
    float* o = dout + (((int64_t)b * T + t0 + tb) * H + h) * DK + ch;
    const int nt = min(HM, nb - tb);  // this half's real tokens (none past the end)
#pragma unroll
    for (int t = 0; t < HM; ++t) {
      if (t < nt) {
        o[(int64_t)t * H * DK] = d;
        d = fmaf(rt[t], d, ea[t]);
      }
    }
    // the block's final d: from the second half, or from the first when the block ends by token 16
    if ((half == 1 && nb > HM) || (half == 0 && nb <= HM)) s_d[ch] = d;
  }
  cp_async_wait_all();
  __syncthreads();
  if (dT && half == 0) dT[(int64_t)bh * DK + ch] = s_d[ch];
}

template <int DK, bool BF16>
cudaError_t launch_scan(const void* k, const float* ret, const float* d0, int B, int T, int H, const float* ws,
                        float* dout, float* dT, cudaStream_t s) {
  using Sm = ScanSmem<DK, BF16>;
  cudaError_t e = cudaFuncSetAttribute(osdn_scan_kernel<DK, BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Sm::BYTES);
  if (e != cudaSuccess) return e;
  osdn_scan_kernel<DK, BF16><<<B * H, 2 * DK, Sm::BYTES, s>>>(k, ret, d0, B, T, H, ws, dout, dT);
  return cudaGetLastError();
}

}  // namespace

size_t osdn_workspace_bytes(int B, int T, int H) {
  const int64_t nblk = (T + kM - 1) / kM;
  return (size_t)B * H * nblk * kBlockFloats * sizeof(float);
}

cudaError_t launch_osdn(const void* k, const float* beta, const float* ret, const float* d0, float eta, int B,
                        int T, int H, int dk, int io_bf16, float* ws, float* dout, float* dT, cudaStream_t s) {
  if ((int64_t)B * H == 0) return cudaSuccess;
  const int64_t nblk_all = (int64_t)B * H * ((T + kM - 1) / kM);
  if (nblk_all > 0) {
    const unsigned grid = (unsigned)((nblk_all + 3) / 4);
    cudaError_t e;
    if (dk == 128) {
      e = cudaFuncSetAttribute(osdn_block_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               BlockSmem<128>::BYTES);
      if (e != cudaSuccess) return e;
      osdn_block_kernel<128><<<grid, 128, BlockSmem<128>::BYTES, s>>>(k, beta, ret, eta, B, T, H, io_bf16, ws);
    } else {
      e = cudaFuncSetAttribute(osdn_block_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               BlockSmem<64>::BYTES);
      if (e != cudaSuccess) return e;
      osdn_block_kernel<64><<<grid, 128, BlockSmem<64>::BYTES, s>>>(k, beta, ret, eta, B, T, H, io_bf16, ws);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (dk == 128)
    return io_bf16 ? launch_scan<128, true>(k, ret, d0, B, T, H, ws, dout, dT, s)
                   : launch_scan<128, false>(k, ret, d0, B, T, H, ws, dout, dT, s);
  return io_bf16 ? launch_scan<64, true>(k, ret, d0, B, T, H, ws, dout, dT, s)
                 : launch_scan<64, false>(k, ret, d0, B, T, H, ws, dout, dT, s);
}

// ------------------------------------------------------------------ allocation-free entry point
// Some callers cannot allocate device memory at the moment they need this scan: a serving
// process whose allocator has handed out all of the GPU's memory up front, a host framework
// that forbids allocations inside its compute callbacks, or a latency-critical loop where an
// allocation's implicit device synchronisation is not allowed. dn_osdn_precond_noalloc serves
// them with a fixed scratch buffer that is part of the library's device image: every GPU that
// loads the library holds these 32 MiB until the process exits. Problems that need more
// (more than 7,943 blocks of 32 tokens over all heads) are rejected.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) unsigned char g_osdn_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {nullptr};
std::mutex g_scratch_mu;

// Device address of the scratch buffer on the current device (host code cannot use the
// array's name as a device pointer). Looked up once per device, on that device's first call.
dn_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_osdn_scratch) != cudaSuccess || !p) return DN_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return DN_OK;
}

}  // namespace
}  // namespace dn

extern "C" dn_status dn_osdn_precond_noalloc(const dn_osdn_desc* desc, const void* k, const float* beta,
                                             const float* retention, const float* d0, float* d, float* d_T,
                                             void* cuda_stream) {
  const size_t need = dn_osdn_precond_workspace_bytes(desc);
  if (!desc) return DN_ERR_INVALID_ARGUMENT;
  if (need > dn::kNoAllocScratchBytes) return DN_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = nullptr;
  if (need > 0) {
    const dn_status st = dn::scratch_address(&scratch);
    if (st != DN_OK) return st;
  }
  return dn_osdn_precond(desc, k, beta, retention, d0, d, d_T, scratch, dn::kNoAllocScratchBytes, cuda_stream);
}
