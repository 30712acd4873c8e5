// Host-side launch interface of the chunked backward (dn_bwd.cu), used by the ABI shim.
#pragma once

#include "dn_common.cuh"

namespace dn {

// Workspace bytes of the backward: per (b, h) and chunk of 64 tokens, the chunk's UT transform and
// score matrix (64 x 64 each), S_m and its adjoint (d_k x d_v each), U and dV~ (64 x d_v each), fp32.
size_t chunk_bwd_workspace_bytes(int B, int T, int H, int dk, int dv);

// Launches the four kernels of the backward on stream s. Gradient pointers of absent gates are null;
// dS_T and gS0 may be null.
cudaError_t launch_chunk_bwd(const Args& f, const void* dO, const float* dS_T, void* gq, void* gk, void* gv,
                             float* galpha, float* gbeta_k, float* gbeta_v, float* gkey_scale, float* gS0, float* ws,
                             cudaStream_t s);

// The chunked forward in fp32 (fp32 io, or bf16 with d_k = 64) on the backward's chunk machinery:
// the prep kernel (every chunk's K+, Q+, W-, T and P), the state chain (S_m and U per chunk, S_T),
// and the outputs O = Q+ S_m + P U per chunk; a chunk whose decay is beyond the factorisation's
// range is evaluated token by token in the state chain. Workspace: the backward's plus one int per
// chunk.
bool chunk_fwd32_supported(const Args& a);
size_t chunk_fwd32_workspace_bytes(const Args& a);
cudaError_t launch_chunk_fwd32(const Args& f, float* ws, cudaStream_t s);

// Small states (d_k, d_v in {8, 16}; dn_small_bwd.cu), either read-out: the state entering every
// token is kept in the workspace (B * H * T * d_k * d_v fp32).
size_t small_bwd_workspace_bytes(int B, int T, int H, int dk, int dv);
cudaError_t launch_small_bwd(const Args& a, const void* dO, const float* dS_T, void* gq, void* gk, void* gv,
                             float* galpha, float* gbeta_k, float* gbeta_v, float* gkey_scale, float* gS0, float* ws,
                             cudaStream_t s);

}  // namespace dn
