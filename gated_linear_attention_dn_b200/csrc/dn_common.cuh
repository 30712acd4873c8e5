// Shared device helpers and the host-side launch interface between the ABI
// shim (dn_abi.cu) and the kernels (one .cu file per kernel family).
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dn.h"

namespace dn {

// Device status codes written to the per-GPU status word (0 = fine): a bounded wait gave up, or a
// chunk's gates were outside the range a kernel's factorisation supports.
enum : int { kDevOk = 0, kDevTimeout = 1, kDevGateRange = 2 };

// Everything a kernel launch needs, already validated by the ABI shim.
struct Args {
  int B, T, H, dk, dv, chunk;
  int io_bf16;                    // 1: q/k/v/o are bf16, 0: fp32
  int alpha, beta_k, beta_v, key_scale;   // dn_gate modes
  int pre_read;                   // 1: o_t = S_{t-1}^T q_t (before the token's update)
  const void* q;
  const void* k;
  const void* v;
  const float* alpha_p;
  const float* beta_k_p;
  const float* beta_v_p;
  const float* key_scale_p;
  const float* S0;                // may be null (zero state)
  void* o;
  float* S;                       // S_T (chunk fwd) or the in/out state (decode)
  int* status;                    // device status word of the current GPU
  uint64_t wait_ns;               // bound of each mbarrier wait of the chunk kernels (0: one probe)
};

// The wait bound the launches take (dn_set_wait_limit_ns; 2 s unless changed).
uint64_t wait_limit_ns();

// Launchers (host). Each returns cudaSuccess or the launch error.
cudaError_t launch_decode(const Args& a, cudaStream_t s);
cudaError_t launch_seq_fwd(const Args& a, cudaStream_t s);
cudaError_t launch_chunk_tc(const Args& a, cudaStream_t s);
// per-token gates only (called by launch_chunk_tc)
cudaError_t launch_chunk_sc(const Args& a, cudaStream_t s);
// Whether a problem takes the per-token-gate tensor-core kernels (bf16, d_k = 128, every gate absent or
// one per token), and the split evaluation of it with a workspace (dn_split_sc.cu): its bytes and launch.
bool per_token_tc(const Args& a);
size_t split_sc_workspace_bytes(const Args& a);
cudaError_t launch_split_sc(const Args& a, void* workspace, cudaStream_t s);
// The split evaluation of the per-channel-gate problems (dn_chunk_tc.cu): whether it applies, its
// workspace bytes, and the launch of its two kernels.
bool split_tc_supported(const Args& a);
size_t split_tc_workspace_bytes(const Args& a);
cudaError_t launch_split_tc(const Args& a, void* workspace, cudaStream_t s);
// OSDN phase 1 (dn_osdn.cu): workspace bytes, and the launch of its two kernels.
size_t osdn_workspace_bytes(int B, int T, int H);
cudaError_t launch_osdn(const void* k, const float* beta, const float* ret, const float* d0, float eta, int B,
                        int T, int H, int dk, int io_bf16, float* ws, float* dout, float* dT, cudaStream_t s);
// Memory Caching read-out (dn_memcache.cu).
cudaError_t launch_mc_readout(const void* q, const float* M, const float* gates, void* o, int B, int T, int H,
                              int dk, int dv, int L, int bf16, int* status, uint64_t wait_ns, cudaStream_t s);
// Small states (d_k, d_v in {8, 16}; dn_small.cu): chunk fwd and decode alike.
bool small_state_supported(const Args& a);
cudaError_t launch_small_state(const Args& a, cudaStream_t s);
// Whether the tensor-core chunk kernels take this problem (else the sequential kernel does).
bool chunk_tc_supported(const Args& a);
// TMA tensor map over a [B, T, H, d] bf16 tensor, 128-byte swizzle, box of 64 channels x 1 head x
// box_tokens tokens x 1 sequence, zero fill past the end (dn_tma.cu). False if encoding fails.
bool make_bthd_map(CUtensorMap* m, const void* base, int d, int H, int T, int B, int box_tokens);

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ float io_load(const void* p, int64_t i, int bf16) {
  if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  return reinterpret_cast<const float*>(p)[i];
}

__device__ __forceinline__ void io_store(void* p, int64_t i, float x, int bf16) {
  if (bf16) {
    reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
  } else {
    reinterpret_cast<float*>(p)[i] = x;
  }
}

// Gate value for (row, token, channel): mode 0 -> 1, 1 -> one per token, 2 -> one per channel.
__device__ __forceinline__ float gate_load(const float* g, int mode, int64_t tok, int width, int ch) {
  if (mode == DN_GATE_ONE) return 1.0f;
  if (mode == DN_GATE_SCALAR) return g[tok];
  return g[tok * width + ch];
}

// ---------------------------------------------------------------- decay products without range limits
// A product of gates is carried as m * 2^e with m in [0.5, 1) and an integer exponent, so a chunk's
// cumulative decay never under- or overflows however strong the gates are; only the final factors,
// which are at most 1 in size, are formed as floats.

// x = m * 2^e for x > 0 (subnormals included). A gate that is 0 (or not positive) becomes
// 0.5 * 2^-1000: every product that contains it then rounds to zero, as it should.
__device__ __forceinline__ void split_pow2(float x, float& m, int& e) {
  if (!(x > 0.f)) {
    m = 0.5f;
    e = -1000;
    return;
  }
  int s = 0;
  if (x < 1.17549435e-38f) {  // subnormal: scale into the normal range first (exact)
    x *= 18446744073709551616.f;  // 2^64
    s = 64;
  }
  const int bits = __float_as_int(x);
  e = ((bits >> 23) & 0xff) - 126 - s;
  m = __int_as_float((bits & 0x007fffff) | 0x3f000000);
}

// (m, e) *= (m2, e2), renormalised so that m stays in [0.5, 1).
__device__ __forceinline__ void mul_pow2(float& m, int& e, float m2, int e2) {
  m *= m2;
  e += e2;
  if (m < 0.5f) {
    m *= 2.f;
    e -= 1;
  }
}

// 2^k as a float: exact for -126 <= k <= 127, 0 below (those factors are negligible next to 1),
// 2^127 above.
__device__ __forceinline__ float pow2f(int k) { return __int_as_float(min(max(k + 127, 0), 254) << 23); }

// Streaming 16-byte global load that does not allocate in L1 (the state is touched once).
// Not the non-coherent path: the decode kernel writes the same addresses later.
__device__ __forceinline__ float4 ld_stream_f4(const float* p) {
  float4 r;
  asm volatile("ld.global.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(r.x), "=f"(r.y), "=f"(r.z), "=f"(r.w)
               : "l"(p));
  return r;
}

// Streaming 16-byte global store (evict-first / cache-streaming).
__device__ __forceinline__ void st_stream_f4(float* p, float4 v) {
  asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
               "f"(v.w)
               : "memory");
}

}  // namespace dn
