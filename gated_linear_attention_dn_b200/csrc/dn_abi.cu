// C ABI shim: argument validation, the per-GPU status word, and dispatch to
// the kernels. Nothing here allocates device memory.
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "dn_bwd.cuh"
#include "dn_common.cuh"

// One status word per GPU that loads the library; kernels set it when a
// bounded wait gives up.
__device__ int g_dn_status;

namespace {

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices] = {nullptr};
std::mutex g_status_mu;  // guards the first lookup on each device
std::atomic<uint64_t> g_wait_ns{2000000000ull};

// Device address of the status word on the current device, looked up once per device.
dn_status status_ptr(int** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_status_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_dn_status) != cudaSuccess) return DN_ERR_CUDA;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_status_ptr[dev];
  return DN_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool gate_ok(int mode) { return mode == DN_GATE_ONE || mode == DN_GATE_SCALAR || mode == DN_GATE_CHANNEL; }

dn_status check_desc(const dn_desc* d, bool decode) {
  if (!d) return DN_ERR_INVALID_ARGUMENT;
  if (d->B < 1 || d->H < 1 || d->T < 0) return DN_ERR_INVALID_ARGUMENT;
  if (decode && d->T != 1) return DN_ERR_INVALID_ARGUMENT;
  if (d->d_k <= 0 || d->d_v <= 0) return DN_ERR_INVALID_ARGUMENT;
  if (d->io_dtype != DN_F32 && d->io_dtype != DN_BF16) return DN_ERR_INVALID_ARGUMENT;
  if (!gate_ok(d->alpha) || !gate_ok(d->beta_k) || !gate_ok(d->beta_v) || !gate_ok(d->key_scale))
    return DN_ERR_INVALID_ARGUMENT;
  if (d->chunk < 0) return DN_ERR_INVALID_ARGUMENT;
  if (d->readout != DN_READ_POST && d->readout != DN_READ_PRE) return DN_ERR_INVALID_ARGUMENT;
  const bool big = (d->d_k == 64 || d->d_k == 128) && (d->d_v == 64 || d->d_v == 128);
  const bool small = (d->d_k == 8 || d->d_k == 16) && (d->d_v == 8 || d->d_v == 16);
  if (!big && !small) return DN_ERR_UNSUPPORTED;
  if (!(d->chunk == 0 || d->chunk == 16 || d->chunk == 32 || d->chunk == 64)) return DN_ERR_UNSUPPORTED;
  // sizes must stay addressable with 32-bit grid math and 64-bit offsets
  const int64_t heads = (int64_t)d->B * d->H;
  if (heads * 2 >= (int64_t)1 << 31) return DN_ERR_UNSUPPORTED;
  if ((int64_t)d->B * d->T * d->H * (d->d_k > d->d_v ? d->d_k : d->d_v) >= ((int64_t)1 << 46))
    return DN_ERR_UNSUPPORTED;
  return DN_OK;
}

// A gate pointer is present exactly when its mode is not DN_GATE_ONE (for T == 0
// no token data is read and gate pointers may be anything, NULL included).
dn_status check_gate_ptr(int mode, const void* p, int T) {
  if (T > 0 && (mode == DN_GATE_ONE) != (p == nullptr)) return DN_ERR_INVALID_ARGUMENT;
  // per-channel gates are read in 16-byte vectors; per-token gates only need fp32 alignment
  if (p && mode == DN_GATE_CHANNEL && !aligned16(p)) return DN_ERR_MISALIGNED;
  if (p && (reinterpret_cast<uintptr_t>(p) & 3u) != 0) return DN_ERR_MISALIGNED;
  return DN_OK;
}

dn_status fill_args(const dn_desc* d, const void* q, const void* k, const void* v, const float* alpha,
                    const float* beta_k, const float* beta_v, const float* key_scale, dn::Args* a) {
  dn_status st;
  if ((st = check_gate_ptr(d->alpha, alpha, d->T)) != DN_OK) return st;
  if ((st = check_gate_ptr(d->beta_k, beta_k, d->T)) != DN_OK) return st;
  if ((st = check_gate_ptr(d->beta_v, beta_v, d->T)) != DN_OK) return st;
  if ((st = check_gate_ptr(d->key_scale, key_scale, d->T)) != DN_OK) return st;
  if (d->T > 0) {
    if (!q || !k || !v) return DN_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return DN_ERR_MISALIGNED;
  }
  memset(a, 0, sizeof(*a));
  a->B = d->B;
  a->T = d->T;
  a->H = d->H;
  a->dk = d->d_k;
  a->dv = d->d_v;
  a->chunk = d->chunk == 0 ? 64 : d->chunk;
  a->io_bf16 = d->io_dtype == DN_BF16;
  a->alpha = d->alpha;
  a->beta_k = d->beta_k;
  a->beta_v = d->beta_v;
  a->key_scale = d->key_scale;
  a->pre_read = d->readout == DN_READ_PRE;
  a->q = q;
  a->k = k;
  a->v = v;
  a->alpha_p = alpha;
  a->beta_k_p = beta_k;
  a->beta_v_p = beta_v;
  a->key_scale_p = key_scale;
  a->wait_ns = dn::wait_limit_ns();
  return DN_OK;
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t pa = reinterpret_cast<uintptr_t>(a), pb = reinterpret_cast<uintptr_t>(b);
  return pa < pb + nb && pb < pa + na;
}

}  // namespace

namespace dn {
uint64_t wait_limit_ns() { return g_wait_ns.load(std::memory_order_relaxed); }
}  // namespace dn

extern "C" {

int dn_version(void) { return 200; }

dn_status dn_set_wait_limit_ns(unsigned long long ns) {
  g_wait_ns.store(ns, std::memory_order_relaxed);
  return DN_OK;
}

const char* dn_status_string(dn_status s) {
  switch (s) {
    case DN_OK: return "DN_OK";
    case DN_ERR_INVALID_ARGUMENT: return "DN_ERR_INVALID_ARGUMENT";
    case DN_ERR_UNSUPPORTED: return "DN_ERR_UNSUPPORTED";
    case DN_ERR_MISALIGNED: return "DN_ERR_MISALIGNED";
    case DN_ERR_WORKSPACE_TOO_SMALL: return "DN_ERR_WORKSPACE_TOO_SMALL";
    case DN_ERR_CUDA: return "DN_ERR_CUDA";
    case DN_ERR_DEVICE_TIMEOUT: return "DN_ERR_DEVICE_TIMEOUT";
    case DN_ERR_GATE_RANGE: return "DN_ERR_GATE_RANGE";
  }
  return "DN_ERR_UNKNOWN";
}

size_t dn_chunk_fwd_workspace_bytes(const dn_desc* desc) {
  if (check_desc(desc, false) != DN_OK) return 0;
  dn::Args a;
  memset(&a, 0, sizeof(a));
  a.B = desc->B, a.T = desc->T, a.H = desc->H, a.dk = desc->d_k, a.dv = desc->d_v;
  a.chunk = desc->chunk == 0 ? 64 : desc->chunk;
  a.io_bf16 = desc->io_dtype == DN_BF16;
  a.alpha = desc->alpha, a.beta_k = desc->beta_k, a.beta_v = desc->beta_v, a.key_scale = desc->key_scale;
  if (dn::small_state_supported(a)) return 0;
  if (dn::per_token_tc(a)) return dn::split_sc_workspace_bytes(a);
  if (dn::split_tc_supported(a)) return dn::split_tc_workspace_bytes(a);
  if (dn::chunk_fwd32_supported(a)) return dn::chunk_fwd32_workspace_bytes(a);
  return 0;
}

dn_status dn_chunk_fwd(const dn_desc* desc, const void* q, const void* k, const void* v,
                       const float* alpha, const float* beta_k, const float* beta_v,
                       const float* key_scale, const float* S0, void* o, float* S_T,
                       void* workspace, size_t workspace_bytes, void* cuda_stream) {
  dn_status st = check_desc(desc, false);
  if (st != DN_OK) return st;
  dn::Args a;
  if ((st = fill_args(desc, q, k, v, alpha, beta_k, beta_v, key_scale, &a)) != DN_OK) return st;
  if (!S_T) return DN_ERR_INVALID_ARGUMENT;
  if (!aligned16(S_T) || (S0 && !aligned16(S0))) return DN_ERR_MISALIGNED;
  if (desc->T > 0) {
    if (!o) return DN_ERR_INVALID_ARGUMENT;
    if (!aligned16(o)) return DN_ERR_MISALIGNED;
    const size_t es = desc->io_dtype == DN_BF16 ? 2 : 4;
    const size_t n_o = (size_t)desc->B * desc->T * desc->H * desc->d_v * es;
    const size_t n_qk = (size_t)desc->B * desc->T * desc->H * desc->d_k * es;
    const size_t n_S = (size_t)desc->B * desc->H * desc->d_k * desc->d_v * 4;
    if (ranges_overlap(o, n_o, q, n_qk) || ranges_overlap(o, n_o, k, n_qk) ||
        ranges_overlap(o, n_o, v, n_o) || ranges_overlap(o, n_o, S_T, n_S))
      return DN_ERR_INVALID_ARGUMENT;
    // S_T is written while every input is still read
    const size_t n_tok = (size_t)desc->B * desc->T * desc->H;
    const void* ins[7] = {q, k, v, alpha, beta_k, beta_v, key_scale};
    const size_t in_n[7] = {n_qk, n_qk, n_o, n_tok * 4 * (desc->alpha == DN_GATE_CHANNEL ? desc->d_k : 1),
                            n_tok * 4 * (desc->beta_k == DN_GATE_CHANNEL ? desc->d_k : 1),
                            n_tok * 4 * (desc->beta_v == DN_GATE_CHANNEL ? desc->d_v : 1),
                            n_tok * 4 * (desc->key_scale == DN_GATE_CHANNEL ? desc->d_k : 1)};
    for (int i = 0; i < 7; ++i)
      if (ranges_overlap(S_T, n_S, ins[i], in_n[i])) return DN_ERR_INVALID_ARGUMENT;
    // a workspace is read and written while every input and output is live
    if (workspace) {
      const size_t need = dn_chunk_fwd_workspace_bytes(desc);
      if (need > 0) {
        if (workspace_bytes < need) return DN_ERR_WORKSPACE_TOO_SMALL;
        if (!aligned16(workspace)) return DN_ERR_MISALIGNED;
        for (int i = 0; i < 7; ++i)
          if (ranges_overlap(workspace, need, ins[i], in_n[i])) return DN_ERR_INVALID_ARGUMENT;
        if (ranges_overlap(workspace, need, o, n_o) || ranges_overlap(workspace, need, S_T, n_S) ||
            ranges_overlap(workspace, need, S0, S0 ? n_S : 0))
          return DN_ERR_INVALID_ARGUMENT;
      }
    }
  }
  {  // in place (S_T == S0) is supported; a partial overlap is not
    const size_t n_S = (size_t)desc->B * desc->H * desc->d_k * desc->d_v * 4;
    if (S0 && S0 != S_T && ranges_overlap(S0, n_S, S_T, n_S)) return DN_ERR_INVALID_ARGUMENT;
  }
  if ((st = status_ptr(&a.status)) != DN_OK) return st;
  a.S0 = S0;
  a.S = S_T;
  a.o = o;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const size_t n_S = (size_t)desc->B * desc->H * desc->d_k * desc->d_v * sizeof(float);
  if (desc->T == 0) {
    cudaError_t e = S0 ? (S0 == S_T ? cudaSuccess : cudaMemcpyAsync(S_T, S0, n_S, cudaMemcpyDeviceToDevice, s))
                       : cudaMemsetAsync(S_T, 0, n_S, s);
    return e == cudaSuccess ? DN_OK : DN_ERR_CUDA;
  }
  cudaError_t e;
  if (dn::small_state_supported(a)) {
    e = dn::launch_small_state(a, s);
  } else if (workspace && dn::per_token_tc(a)) {
    e = dn::launch_split_sc(a, workspace, s);
  } else if (workspace && dn::split_tc_supported(a)) {
    e = dn::launch_split_tc(a, workspace, s);
  } else if (a.io_bf16 && dn::chunk_tc_supported(a)) {
    e = dn::launch_chunk_tc(a, s);
  } else if (workspace && dn::chunk_fwd32_supported(a)) {
    e = dn::launch_chunk_fwd32(a, static_cast<float*>(workspace), s);
  } else {
    e = dn::launch_seq_fwd(a, s);
  }
  return e == cudaSuccess ? DN_OK : DN_ERR_CUDA;
}

dn_status dn_decode_step(const dn_desc* desc, const void* q, const void* k, const void* v,
                         const float* alpha, const float* beta_k, const float* beta_v,
                         const float* key_scale, float* S, void* o, void* cuda_stream) {
  dn_status st = check_desc(desc, true);
  if (st != DN_OK) return st;
  dn::Args a;
  if ((st = fill_args(desc, q, k, v, alpha, beta_k, beta_v, key_scale, &a)) != DN_OK) return st;
  if (!S || !o) return DN_ERR_INVALID_ARGUMENT;
  if (!aligned16(S) || !aligned16(o)) return DN_ERR_MISALIGNED;
  {  // o is written while S, q, k and v are still read (by the other column slice of the same head)
    const size_t es = desc->io_dtype == DN_BF16 ? 2 : 4;
    const size_t nh = (size_t)desc->B * desc->H;
    const size_t n_o = nh * desc->d_v * es, n_k = nh * desc->d_k * es;
    const size_t n_S = nh * desc->d_k * desc->d_v * 4;
    if (ranges_overlap(o, n_o, S, n_S) || ranges_overlap(o, n_o, q, n_k) || ranges_overlap(o, n_o, k, n_k) ||
        ranges_overlap(o, n_o, v, n_o))
      return DN_ERR_INVALID_ARGUMENT;
  }
  if ((st = status_ptr(&a.status)) != DN_OK) return st;
  a.S0 = S;
  a.S = S;
  a.o = o;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  cudaError_t e = dn::small_state_supported(a) ? dn::launch_small_state(a, s) : dn::launch_decode(a, s);
  return e == cudaSuccess ? DN_OK : DN_ERR_CUDA;
}

}  // extern "C"

namespace {

bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

dn_status check_osdn_desc(const dn_osdn_desc* d) {
  if (!d) return DN_ERR_INVALID_ARGUMENT;
  if (d->B < 1 || d->H < 1 || d->T < 0) return DN_ERR_INVALID_ARGUMENT;
  if (d->io_dtype != DN_F32 && d->io_dtype != DN_BF16) return DN_ERR_INVALID_ARGUMENT;
  if (!isfinite(d->eta) || d->eta < 0.f) return DN_ERR_INVALID_ARGUMENT;
  if (d->d_k != 64 && d->d_k != 128) return DN_ERR_UNSUPPORTED;
  const int64_t heads = (int64_t)d->B * d->H;
  const int64_t blocks = heads * ((d->T + 31) / 32);
  if (heads >= ((int64_t)1 << 31) || blocks >= ((int64_t)1 << 32)) return DN_ERR_UNSUPPORTED;
  if ((int64_t)d->B * d->T * d->H * d->d_k >= ((int64_t)1 << 46)) return DN_ERR_UNSUPPORTED;
  return DN_OK;
}

}  // namespace

extern "C" {

size_t dn_osdn_precond_workspace_bytes(const dn_osdn_desc* desc) {
  if (check_osdn_desc(desc) != DN_OK) return 0;
  return dn::osdn_workspace_bytes(desc->B, desc->T, desc->H);
}

dn_status dn_osdn_precond(const dn_osdn_desc* desc, const void* k, const float* beta,
                          const float* retention, const float* d0, float* d, float* d_T,
                          void* workspace, size_t workspace_bytes, void* cuda_stream) {
  dn_status st = check_osdn_desc(desc);
  if (st != DN_OK) return st;
  if (!aligned4(retention) || !aligned4(d0) || !aligned4(d_T)) return DN_ERR_MISALIGNED;
  if (desc->T > 0) {
    if (!k || !beta || !d) return DN_ERR_INVALID_ARGUMENT;
    if (!aligned16(k)) return DN_ERR_MISALIGNED;
    if (!aligned4(beta) || !aligned4(d)) return DN_ERR_MISALIGNED;
    const size_t need = dn::osdn_workspace_bytes(desc->B, desc->T, desc->H);
    if (!workspace || workspace_bytes < need) return DN_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(workspace)) return DN_ERR_MISALIGNED;
    const size_t n_d = (size_t)desc->B * desc->T * desc->H * desc->d_k * sizeof(float);
    const size_t n_k = (size_t)desc->B * desc->T * desc->H * desc->d_k * (desc->io_dtype == DN_BF16 ? 2 : 4);
    if (ranges_overlap(d, n_d, workspace, need) || ranges_overlap(d, n_d, k, n_k)) return DN_ERR_INVALID_ARGUMENT;
  } else if (!d_T) {
    return DN_OK;  // nothing to compute, nothing to write
  }
  cudaError_t e = dn::launch_osdn(k, beta, retention, d0, desc->eta, desc->B, desc->T, desc->H, desc->d_k,
                                  desc->io_dtype == DN_BF16, static_cast<float*>(workspace), d, d_T,
                                  static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? DN_OK : DN_ERR_CUDA;
}

dn_status dn_mc_readout(const dn_mc_desc* d, const void* q, const float* M, const float* gates, void* o,
                        void* cuda_stream) {
  if (!d) return DN_ERR_INVALID_ARGUMENT;
  if (d->B < 1 || d->H < 1 || d->T < 0 || d->seg_len < 1) return DN_ERR_INVALID_ARGUMENT;
  if (d->io_dtype != DN_F32 && d->io_dtype != DN_BF16) return DN_ERR_INVALID_ARGUMENT;
  if (!((d->d_k == 64 || d->d_k == 128) && (d->d_v == 64 || d->d_v == 128))) return DN_ERR_UNSUPPORTED;
  const int64_t tiles = (int64_t)d->B * d->H * ((d->T + 63) / 64);
  if (tiles >= ((int64_t)1 << 31) || (int64_t)d->B * d->T * d->H * d->d_v >= ((int64_t)1 << 46))
    return DN_ERR_UNSUPPORTED;
  if (d->T <= d->seg_len) return DN_OK;  // no token has an earlier segment
  if (!q || !M || !o) return DN_ERR_INVALID_ARGUMENT;
  if (!aligned16(M)) return DN_ERR_MISALIGNED;
  const size_t es = d->io_dtype == DN_BF16 ? 2 : 4;
  if ((reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(o)) & (es - 1)) return DN_ERR_MISALIGNED;
  if (gates && !aligned4(gates)) return DN_ERR_MISALIGNED;
  const size_t n_o = (size_t)d->B * d->T * d->H * d->d_v * es;
  const size_t n_q = (size_t)d->B * d->T * d->H * d->d_k * es;
  if (ranges_overlap(o, n_o, q, n_q)) return DN_ERR_INVALID_ARGUMENT;
  int* status = nullptr;
  dn_status st = status_ptr(&status);
  if (st != DN_OK) return st;
  cudaError_t e = dn::launch_mc_readout(q, M, gates, o, d->B, d->T, d->H, d->d_k, d->d_v, d->seg_len,
                                        d->io_dtype == DN_BF16, status, dn::wait_limit_ns(),
                                        static_cast<cudaStream_t>(cuda_stream));
  return e == cudaSuccess ? DN_OK : DN_ERR_CUDA;
}

}  // extern "C"

namespace {

bool small_dims(const dn_desc* d) { return (d->d_k == 8 || d->d_k == 16) && (d->d_v == 8 || d->d_v == 16); }

// The backward covers the tensor-core sizes (chunked kernels) and the small states (sequential
// kernel), either read-out.
dn_status check_bwd_desc(const dn_desc* d) {
  dn_status st = check_desc(d, false);
  if (st != DN_OK) return st;
  if (small_dims(d)) return DN_OK;
  if (!(d->chunk == 0 || d->chunk == 64)) return DN_ERR_UNSUPPORTED;  // (its chunks are 64 tokens)
  const int64_t blocks = (int64_t)d->B * d->H * ((d->T + 63) / 64);
  if (blocks >= ((int64_t)1 << 31)) return DN_ERR_UNSUPPORTED;
  return DN_OK;
}

// A gate gradient is given exactly when its gate is.
dn_status check_grad_ptr(int mode, const float* g) {
  if ((mode == DN_GATE_ONE) != (g == nullptr)) return DN_ERR_INVALID_ARGUMENT;
  if (g && !aligned4(g)) return DN_ERR_MISALIGNED;
  return DN_OK;
}

}  // namespace

extern "C" {

size_t dn_chunk_bwd_workspace_bytes(const dn_desc* desc) {
  if (check_bwd_desc(desc) != DN_OK) return 0;
  if (small_dims(desc)) return dn::small_bwd_workspace_bytes(desc->B, desc->T, desc->H, desc->d_k, desc->d_v);
  return dn::chunk_bwd_workspace_bytes(desc->B, desc->T, desc->H, desc->d_k, desc->d_v);
}

dn_status dn_chunk_bwd(const dn_desc* desc, const void* q, const void* k, const void* v, const float* alpha,
                       const float* beta_k, const float* beta_v, const float* key_scale, const float* S0,
                       const void* dO, const float* dS_T, void* dq, void* dk, void* dv, float* d_alpha,
                       float* d_beta_k, float* d_beta_v, float* d_key_scale, float* dS0, void* workspace,
                       size_t workspace_bytes, void* cuda_stream) {
  dn_status st = check_bwd_desc(desc);
  if (st != DN_OK) return st;
  dn::Args a;
  if ((st = fill_args(desc, q, k, v, alpha, beta_k, beta_v, key_scale, &a)) != DN_OK) return st;
  if ((S0 && !aligned16(S0)) || (dS_T && !aligned16(dS_T)) || (dS0 && !aligned16(dS0))) return DN_ERR_MISALIGNED;
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  const size_t n_S = (size_t)desc->B * desc->H * desc->d_k * desc->d_v * sizeof(float);
  if (desc->T == 0) {  // no tokens: dS0 = dS_T
    if (!dS0) return DN_OK;
    cudaError_t e = dS_T ? (dS_T == dS0 ? cudaSuccess : cudaMemcpyAsync(dS0, dS_T, n_S, cudaMemcpyDeviceToDevice, s))
                         : cudaMemsetAsync(dS0, 0, n_S, s);
    return e == cudaSuccess ? DN_OK : DN_ERR_CUDA;
  }
  if (!dO || !dq || !dk || !dv) return DN_ERR_INVALID_ARGUMENT;
  if (!aligned16(dO) || !aligned16(dq) || !aligned16(dk) || !aligned16(dv)) return DN_ERR_MISALIGNED;
  if ((st = check_grad_ptr(desc->alpha, d_alpha)) != DN_OK) return st;
  if ((st = check_grad_ptr(desc->beta_k, d_beta_k)) != DN_OK) return st;
  if ((st = check_grad_ptr(desc->beta_v, d_beta_v)) != DN_OK) return st;
  if ((st = check_grad_ptr(desc->key_scale, d_key_scale)) != DN_OK) return st;
  const size_t need = dn_chunk_bwd_workspace_bytes(desc);
  if (!workspace || workspace_bytes < need) return DN_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned16(workspace)) return DN_ERR_MISALIGNED;
  {  // the gradients of q, k, v are written while every input, dO and the workspace are still read
    const size_t es = desc->io_dtype == DN_BF16 ? 2 : 4;
    const size_t n_k = (size_t)desc->B * desc->T * desc->H * desc->d_k * es;
    const size_t n_v = (size_t)desc->B * desc->T * desc->H * desc->d_v * es;
    const void* outs[3] = {dq, dk, dv};
    const size_t out_n[3] = {n_k, n_k, n_v};
    const void* ins[6] = {q, k, v, dO, workspace, S0};
    const size_t in_n[6] = {n_k, n_k, n_v, n_v, need, S0 ? n_S : 0};
    for (int i = 0; i < 3; ++i) {
      for (int j = 0; j < 6; ++j)
        if (ranges_overlap(outs[i], out_n[i], ins[j], in_n[j])) return DN_ERR_INVALID_ARGUMENT;
      for (int j = i + 1; j < 3; ++j)
        if (ranges_overlap(outs[i], out_n[i], outs[j], out_n[j])) return DN_ERR_INVALID_ARGUMENT;
    }
  }
  a.S0 = S0;
  if ((st = status_ptr(&a.status)) != DN_OK) return st;
  cudaError_t e =
      small_dims(desc)
          ? dn::launch_small_bwd(a, dO, dS_T, dq, dk, dv, d_alpha, d_beta_k, d_beta_v, d_key_scale, dS0,
                                 static_cast<float*>(workspace), s)
          : dn::launch_chunk_bwd(a, dO, dS_T, dq, dk, dv, d_alpha, d_beta_k, d_beta_v, d_key_scale, dS0,
                                 static_cast<float*>(workspace), s);
  return e == cudaSuccess ? DN_OK : DN_ERR_CUDA;
}

dn_status dn_stream_status(void* cuda_stream) {
  cudaStream_t s = static_cast<cudaStream_t>(cuda_stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return DN_ERR_CUDA;
  if (cudaGetLastError() != cudaSuccess) return DN_ERR_CUDA;
  int* p = nullptr;
  dn_status st = status_ptr(&p);
  if (st != DN_OK) return st;
  int word = 0;
  if (cudaMemcpy(&word, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return DN_ERR_CUDA;
  if (word != dn::kDevOk) {
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return DN_ERR_CUDA;
    return word == dn::kDevGateRange ? DN_ERR_GATE_RANGE : DN_ERR_DEVICE_TIMEOUT;
  }
  return DN_OK;
}

}  // extern "C"
