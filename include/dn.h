/*
 * dn.h -- C ABI of the B200 (sm_100a) gated delta-rule library (libdn.so).
 *
 * The recurrence (key-major state S in R^{d_k x d_v}, fp32), per batch b,
 * head h and token t:
 *
 *   S_bar_t = Diag(alpha_t) S_{t-1}
 *   w_t     = beta^k_t (.) d_t (.) k_t
 *   u_t     = beta^v_t (.) v_t - S_bar_t^T k_t
 *   S_t     = S_bar_t + w_t u_t^T
 *           = (I - w_t k_t^T) Diag(alpha_t) S_{t-1} + w_t (beta^v_t (.) v_t)^T
 *   o_t     = S_t^T q_t                       (read-out after the update, no 1/sqrt(d_k))
 *
 * Sources of each term:
 *   - the delta rule as one online-gradient step on 0.5 ||S k - v||^2, with a
 *     scalar write gate beta (OSDN page, section 1; delta-mem page, section 2.A);
 *   - scalar forget gate alpha_t (Gated DeltaNet) and per-key-channel decay
 *     alpha_t in R^{d_k} (KDA) (FG2-GDN page, section 1); decay is applied to the
 *     state before the delta step (Sparse Delta Memory page, "Gated Delta Updates");
 *   - vector beta^k (erase strength) and beta^v (write strength) of FG2-GDN+
 *     (FG2-GDN page, section 2.B); FG2-GDN's symmetric form with k~ = sqrt(beta) (.) k,
 *     v~ = sqrt(beta) (.) v (section 2.A) is this recurrence fed k' = k~,
 *     beta^k = 1, beta^v = sqrt(beta);
 *   - OSDN preconditioned write key k~ = d (.) k, where the residual keeps the raw
 *     key (OSDN page, section 2.1, right-preconditioning identity).
 *
 * dn_chunk_fwd evaluates a whole sequence in chunkwise-parallel (WY / UT
 * transform) form, the chunk algorithm the FG2-GDN page (sections 2.A and 3
 * item 2) and the OSDN page (section 2.1) rely on; dn_decode_step advances a
 * resident state by one token.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates no device memory and keeps no per-call state. The only global
 *     state is one device status word per GPU (see dn_stream_status) and the
 *     static scratch buffer of dn_osdn_precond_noalloc.
 *   - Row-major layouts, innermost dimension last:
 *       q, k      [B, T, H, d_k]        io dtype
 *       v, o      [B, T, H, d_v]        io dtype
 *       alpha     [B, T, H] (DN_GATE_SCALAR) or [B, T, H, d_k] (DN_GATE_CHANNEL), fp32
 *       beta_k    [B, T, H] or [B, T, H, d_k], fp32
 *       beta_v    [B, T, H] or [B, T, H, d_v], fp32
 *       key_scale [B, T, H] or [B, T, H, d_k], fp32   (OSDN d_t)
 *       S0, S_T, S [B, H, d_k, d_v], fp32
 *     A gate whose mode is DN_GATE_ONE is absent (every value 1) and its pointer
 *     must be NULL. With T == 0 no token data is read: q, k, v, o and the gate
 *     pointers are ignored (they may be NULL).
 *   - q, k, v, o, S0, S_T, S and per-channel gates must be 16-byte aligned;
 *     per-token (DN_GATE_SCALAR) gates need only 4-byte alignment, so a gate
 *     tensor sliced at any token offset is accepted.
 *   - Calls are asynchronous on `cuda_stream` (a cudaStream_t; NULL = legacy
 *     default stream). Argument errors are returned synchronously before any
 *     launch; a failed launch returns DN_ERR_CUDA. A device-side bounded wait
 *     that gives up is reported later by dn_stream_status.
 *   - Numerics: fp32 state, fp32 accumulation. bf16 io runs the tensor-core
 *     chunk kernel (bf16 operands; the state-update product uses a hi/lo bf16
 *     split); fp32 io runs an fp32 CUDA-core kernel. Small states (d_k, d_v in
 *     {8, 16}, e.g. the delta-mem page's 8 x 8 memory) run an fp32 CUDA-core
 *     kernel with one warp per head, for the chunked call and the decode step.
 *   - Gates: alpha >= 0 (0 resets the state), finite. The forward and the decode
 *     step hold for any such decay, however strong: per-token gates carry the
 *     chunk's decay products as mantissa and exponent, and a chunk whose
 *     per-channel decay over half a chunk falls below 2^-50 is evaluated exactly,
 *     token by token, instead of through the tensor-core factorisation.
 */
#ifndef DN_H_
#define DN_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DN_OK = 0,
  DN_ERR_INVALID_ARGUMENT = 1,   /* null/inconsistent pointer or size, bad enum */
  DN_ERR_UNSUPPORTED = 2,        /* valid but not implemented (d_k, d_v, chunk, dtype) */
  DN_ERR_MISALIGNED = 3,         /* a pointer is not 16-byte aligned */
  DN_ERR_WORKSPACE_TOO_SMALL = 4,
  DN_ERR_CUDA = 5,               /* a CUDA runtime call or launch failed */
  DN_ERR_DEVICE_TIMEOUT = 6,     /* a kernel's bounded wait gave up (reported by dn_stream_status) */
  DN_ERR_GATE_RANGE = 7          /* dn_chunk_bwd only: a chunk's decay is beyond what its factorisation
                                    holds in fp32 (reported by dn_stream_status; see dn_chunk_bwd) */
} dn_status;

typedef enum { DN_F32 = 0, DN_BF16 = 1 } dn_dtype;

/* How a gate is given: absent (1), one value per (b, t, h), or one per channel. */
typedef enum { DN_GATE_ONE = 0, DN_GATE_SCALAR = 1, DN_GATE_CHANNEL = 2 } dn_gate;

/*
 * When o_t reads the state. DN_READ_POST: o_t = S_t^T q_t, after the token's update (the
 * default). DN_READ_PRE: o_t = S_{t-1}^T q_t, before the token's decay and write -- the read of
 * the delta-mem page (section 2.C, r_t = S_{t-1} q^m_t). delta-mem's update
 * S_t = lambda_t S_{t-1} + beta_t (v_t - S_{t-1} k_t) k_t^T (section 2.A; undecayed residual) is
 * this recurrence with alpha = lambda, beta^k = beta / lambda, beta^v = lambda (lambda > 0).
 * The forward takes either read-out for any alpha >= 0; dn_chunk_bwd needs alpha > 0.
 */
typedef enum { DN_READ_POST = 0, DN_READ_PRE = 1 } dn_readout;

typedef struct {
  int B, T, H;        /* batch, tokens per sequence, heads; B, H >= 1, T >= 0 */
  int d_k, d_v;       /* head dims; supported: d_k, d_v in {64, 128}, or both in {8, 16} (small states) */
  int chunk;          /* chunk length of the WY form: 16, 32 or 64; 0 selects the default, 64. 16 and 32 run the
                         chunk form in fp32 (below); small states and the sequential kernel have no chunks;
                         dn_chunk_bwd takes 0 or 64 */
  dn_dtype io_dtype;  /* dtype of q, k, v and o */
  dn_gate alpha;      /* forget gate: scalar (GDN) or per key channel (KDA) */
  dn_gate beta_k;     /* erase / write strength on the key side (GDN beta; FG2-GDN+ beta^k) */
  dn_gate beta_v;     /* write strength on the value side (FG2-GDN+ beta^v); CHANNEL means d_v wide */
  dn_gate key_scale;  /* OSDN preconditioner d_t on the write key; CHANNEL means d_k wide */
  dn_readout readout; /* read-out after (default, 0) or before the token's update */
} dn_desc;

/*
 * Bytes of workspace dn_chunk_fwd can use for this descriptor (0 for an invalid
 * descriptor, and for problems that have no use for one).
 *
 * Problems on the per-token-gate tensor-core path (bf16 io, d_k = 128, d_v in
 * {64, 128}, every gate absent or one per token: GDN) have two evaluations:
 *  - with a workspace of at least this size: a chunk-parallel transform kernel
 *    (decay factors, Gram product, UT inverse of every chunk at once) writes
 *    ~25 KB per (b, h, chunk of 64 tokens) -- 33 KB when beta^v is given -- and a
 *    state-chain kernel reads it back; the faster form;
 *  - with workspace == NULL: one fused kernel per (b, h) that keeps everything on
 *    chip, at some cost in speed.
 * Problems in fp32 io, and bf16 with d_k = 64 (d_k, d_v in {64, 128}), also have two, and
 * so does every problem with d_k, d_v in {64, 128} and chunk = 16 or 32:
 *  - with a workspace of at least this size: the chunk form in fp32 (split-TF32 warp
 *    tensor-core products, about fp32 accuracy) with chunks of C = chunk tokens: a kernel
 *    forms every chunk's decay-scaled keys, queries and write keys, UT transform and scores,
 *    the state chain walks the chunks, and a third kernel forms the outputs. The workspace
 *    holds, per (b, h, chunk), 4 * (2 C^2 + d_k d_v + C d_v + 3 C d_k + 2 d_k) bytes (115 KB
 *    at C = 64 and d = 64, 230 KB at d = 128) plus one int, rounded up to 16 bytes in all; a
 *    chunk whose decay over half a chunk exceeds e^80 per channel is evaluated token by token
 *    inside the chain;
 *  - with workspace == NULL: the sequential fp32 kernel, token by token.
 * Problems with a per-channel gate at bf16 d_k = 128 (KDA, FG2-GDN+, OSDN) whose sequences
 * are few (B * H * 2 <= the device's SM count) have two as well:
 *  - with a workspace of at least this size: a chunk-parallel kernel writes, per (b, h, chunk
 *    of 64 tokens), the decay-scaled [K+; Q+] tile, the [T; P] tile, W- (bf16 hi and lo), a
 *    2 KB factor block, V~ (hi and lo, when beta^v is given) and room for a chunk out of the
 *    factors' range (its raw k, q tiles and fp32 alpha and w rows): 146 KB per chunk, 178 KB
 *    with beta^v at d_v = 128; state-chain kernels of 64 value columns then read it back;
 *  - with workspace == NULL, and for more sequences (where this returns 0): one fused kernel
 *    per (b, h) and slice of value columns.
 * Both give the same results up to rounding. Other problems (small states) take no workspace.
 */
size_t dn_chunk_fwd_workspace_bytes(const dn_desc* desc);

/*
 * Chunked prefill (FG2-GDN page, sections 2.A and 3 item 2: the DPLR update that
 * keeps the WY chunk-parallel algorithm; OSDN page, section 2.1: only K -> d (.) K
 * changes in the block Gram matrix and intra-block scores).
 *
 * In:  q, k, v, gates as laid out above; S0 = initial state or NULL (zero).
 * Out: o [B,T,H,d_v] (io dtype), S_T [B,H,d_k,d_v] fp32 (final state).
 * S_T may alias S0 exactly (in-place resume); any other overlap of S_T with S0
 * or with an input, and any overlap of o with q, k, v or S_T, is rejected with
 * DN_ERR_INVALID_ARGUMENT. `workspace`: NULL, or (when
 * dn_chunk_fwd_workspace_bytes() is not 0) a 16-byte-aligned device buffer of at
 * least that many bytes, owned by the caller, whose contents on entry do not
 * matter and which overlaps no input or output (DN_ERR_WORKSPACE_TOO_SMALL,
 * DN_ERR_MISALIGNED, DN_ERR_INVALID_ARGUMENT otherwise); it is ignored when the
 * size is 0.
 * T == 0 copies S0 (or zeros) into S_T and writes no o.
 */
dn_status dn_chunk_fwd(const dn_desc* desc, const void* q, const void* k, const void* v,
                       const float* alpha, const float* beta_k, const float* beta_v,
                       const float* key_scale, const float* S0, void* o, float* S_T,
                       void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * One recurrent step (desc->T must be 1): S <- S_1, o <- S_1^T q, in place.
 * In:  q, k [B,1,H,d_k], v [B,1,H,d_v], gates for one token, S [B,H,d_k,d_v] fp32.
 * Out: S updated in place, o [B,1,H,d_v] (io dtype); o must not overlap S, q, k
 * or v (DN_ERR_INVALID_ARGUMENT).
 * Each (b, h) state is read once and written once (HBM-streaming kernel).
 */
dn_status dn_decode_step(const dn_desc* desc, const void* q, const void* k, const void* v,
                         const float* alpha, const float* beta_k, const float* beta_v,
                         const float* key_scale, float* S, void* o, void* cuda_stream);

/*
 * OSDN phase 1 (OSDN page, section 2.2 "decoupled hypergradient feedback", the
 * first of its two phases, and section 2.3 "adaptive preconditioner
 * forgetting"): the per-token diagonal preconditioner d_t of every (b, h), which
 * dn_chunk_fwd / dn_decode_step then take as the key scale (DN_GATE_CHANNEL).
 * Token t is written with d_t; then one online-gradient-descent step on the
 * closed-form surrogate h_t(d) = ((1 - beta_t <d, k_t (.) k_t>)^2 - 1) / (2 ||k_t||^2):
 *
 *   d_{t+1} = r_t d_t + eta beta_t (1 - beta_t <d_t, k_t (.) k_t>) (k_t (.) k_t) / ||k_t||^2
 *
 * (r_t = 1 without forgetting; a token with k_t = 0 only applies r_t). The page
 * prints the forgetting variant with "+ eta grad h"; this is the descent reading.
 *
 * In:  k [B,T,H,d_k] (io dtype); beta [B,T,H] fp32 (the scalar write strength);
 *      retention [B,T,H] fp32 or NULL (r = 1); d0 [B,H,d_k] fp32 or NULL (ones).
 * Out: d [B,T,H,d_k] fp32 (d_t of every token); d_T [B,H,d_k] fp32 or NULL
 *      (the preconditioner after the last token, for a later call's d0; may
 *      alias d0).
 * Scratch: `workspace` of at least dn_osdn_precond_workspace_bytes() bytes,
 * 16-byte aligned, owned by the caller; its contents on entry do not matter.
 * Supported: d_k in {64, 128}; k 16-byte aligned; beta, retention, d0, d, d_T
 * 4-byte aligned. T == 0 copies d0 (or ones) into d_T. Asynchronous on the stream.
 */
typedef struct {
  int B, T, H;        /* batch, tokens per sequence, heads; B, H >= 1, T >= 0 */
  int d_k;            /* key head dim: 64 or 128 */
  dn_dtype io_dtype;  /* dtype of k */
  float eta;          /* step size of the preconditioner's online-gradient descent (finite, >= 0) */
} dn_osdn_desc;

/* Bytes of workspace dn_osdn_precond needs: 4224 per head per 32 tokens. 0 for an invalid descriptor. */
size_t dn_osdn_precond_workspace_bytes(const dn_osdn_desc* desc);

dn_status dn_osdn_precond(const dn_osdn_desc* desc, const void* k, const float* beta,
                          const float* retention, const float* d0, float* d, float* d_T,
                          void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * dn_osdn_precond without a caller-provided workspace: the same computation and
 * results, with the scratch taken from a fixed 32 MiB buffer built into the
 * library. The pages have no counterpart to this entry point; it exists for
 * callers that cannot allocate device memory when they run the scan -- e.g. a
 * serving process whose allocator reserved the whole GPU at start-up, or a host
 * framework that forbids allocations inside its compute callbacks.
 *
 *  - Nothing is allocated: the buffer is a static device array that every GPU
 *    which loads libdn.so holds until the process exits.
 *  - Limit: problems whose dn_osdn_precond_workspace_bytes() exceeds 32 MiB (more
 *    than 7,943 blocks of 32 tokens summed over all (b, h)) are rejected with
 *    DN_ERR_WORKSPACE_TOO_SMALL before anything runs.
 *  - The first call on each device looks up the buffer's device address on the
 *    current device (one cudaGetSymbolAddress); make that first call before any
 *    stream capture.
 *  - All calls share the one buffer. Calls whose executions overlap on the GPU
 *    (different streams, or different host threads) race on it and give wrong
 *    results: serialise them. Its contents between calls do not matter; nothing
 *    needs clearing.
 * Arguments and errors are otherwise those of dn_osdn_precond.
 */
dn_status dn_osdn_precond_noalloc(const dn_osdn_desc* desc, const void* k, const float* beta,
                                  const float* retention, const float* d0, float* d, float* d_T,
                                  void* cuda_stream);

/*
 * Memory Caching read-out (Memory Caching page, section 2 "retrieval" and section 3: the
 * residual memory and the gated residual memory): the sequence is cut into segments of L
 * tokens, every segment's memory runs the recurrence from the initial state, and its final
 * state M_s is cached; a token t of segment j = t / L adds the gated read of the earlier
 * segments' memories to its own output:
 *
 *   o_t += sum_{s < j} g[b, t, h, s] M_s^T q_t          (g = 1 when gates is NULL)
 *
 * The online part and the cache come from dn_chunk_fwd on the sequence viewed as B * N
 * sequences of L tokens (q, k, v, gates as [B*N, L, H, d] views of the same memory when T is a
 * multiple of L): its o is the online read-out and its S_T is M [B, N, H, d_k, d_v].
 *
 * In:  q [B,T,H,d_k] (io dtype), M [B,N,H,d_k,d_v] fp32 (N = ceil(T / seg_len)), gates
 *      [B,T,H,N] fp32 or NULL.   In/out: o [B,T,H,d_v] (io dtype), accumulated in place.
 * Supported: d_k, d_v in {64, 128}; M 16-byte aligned. fp32 arithmetic.
 */
typedef struct {
  int B, T, H;        /* B, H >= 1, T >= 0 */
  int d_k, d_v;       /* 64 or 128 each */
  int seg_len;        /* L >= 1 */
  dn_dtype io_dtype;  /* dtype of q and o */
} dn_mc_desc;

dn_status dn_mc_readout(const dn_mc_desc* desc, const void* q, const float* M, const float* gates, void* o,
                        void* cuda_stream);

/*
 * Chunked backward (training pass) of dn_chunk_fwd: the gradients of the scalar
 *
 *   L = sum_{b,t,h} <dO_t, o_t> + sum_{b,h} <dS_T, S_T>
 *
 * with respect to q, k, v, every gate given, and S0. The FG2-GDN page (section 3
 * item 2) names chunk-parallel training for this DPLR update but prints no backward;
 * this is the chain rule through the same chunk form (C = 64) that the forward uses.
 *
 * In:  desc, q, k, v, gates, S0 exactly as given to dn_chunk_fwd (S0 may be NULL);
 *      dO [B,T,H,d_v] (io dtype); dS_T [B,H,d_k,d_v] fp32 or NULL (zero).
 * Out: dq, dk [B,T,H,d_k] and dv [B,T,H,d_v] (io dtype); d_alpha, d_beta_k,
 *      d_beta_v, d_key_scale fp32, each shaped like its gate ([B,T,H] for a
 *      per-token gate, [B,T,H,n] per channel), given exactly when the gate is
 *      (NULL when it is DN_GATE_ONE); dS0 [B,H,d_k,d_v] fp32 or NULL (not wanted).
 * Scratch: `workspace` of at least dn_chunk_bwd_workspace_bytes() bytes, 16-byte
 * aligned, owned by the caller; its contents on entry do not matter. Small states: the
 * state entering every token (B * H * T * d_k * d_v fp32). Otherwise, per (b, h) and
 * chunk of 64 tokens, fp32: the UT transform and score matrix (64 x 64 each), the
 * decay-scaled keys, queries and write keys and their decay factors (64 x d_k each), the
 * state and its adjoint (d_k x d_v each), and the residuals and their adjoints (64 x d_v each).
 * Supported: both read-outs (desc->readout as given to the forward); d_k, d_v in {64, 128}
 * (chunked kernels, chunk 0 or 64; 16 and 32 return DN_ERR_UNSUPPORTED) or both in {8, 16} (small states: one warp per head, sequential, the state
 * entering every token kept in the workspace); alpha > 0. The chunked kernels reference each chunk's
 * decay to a point inside it, in fp32: a chunk where the decay between that point and any of its
 * tokens exceeds e^80 per channel (mean log alpha below about -2.5 per token) sets
 * DN_ERR_GATE_RANGE for dn_stream_status and its gradients are not valid. dq, dk, dv must not overlap each other, q, k, v,
 * dO, S0 or the workspace. fp32 arithmetic throughout. T == 0 writes dS0 = dS_T (or
 * zeros). Asynchronous on the stream.
 */
size_t dn_chunk_bwd_workspace_bytes(const dn_desc* desc);

dn_status dn_chunk_bwd(const dn_desc* desc, const void* q, const void* k, const void* v,
                       const float* alpha, const float* beta_k, const float* beta_v,
                       const float* key_scale, const float* S0, const void* dO, const float* dS_T,
                       void* dq, void* dk, void* dv, float* d_alpha, float* d_beta_k, float* d_beta_v,
                       float* d_key_scale, float* dS0, void* workspace, size_t workspace_bytes,
                       void* cuda_stream);

/*
 * Synchronises `cuda_stream`, then reports (and clears) the device status word
 * that kernels set when a bounded wait gives up (DN_ERR_DEVICE_TIMEOUT) or when
 * dn_chunk_bwd meets a chunk beyond its range (DN_ERR_GATE_RANGE), or
 * DN_ERR_CUDA if the stream holds a CUDA error. DN_OK otherwise.
 * The status word's device address is looked up on the first call of any entry
 * point on each device: make that first call before any stream capture.
 */
dn_status dn_stream_status(void* cuda_stream);

/*
 * Diagnostics: the bound of every mbarrier wait in the tensor-core chunk kernels
 * (default 2 s, far above any legitimate wait). A wait that runs out makes the
 * kernel leave its loop, drain what it issued (those waits keep the 2 s bound),
 * free its tensor memory and set DN_ERR_DEVICE_TIMEOUT for dn_stream_status;
 * 0 makes each wait a single non-blocking probe, so a test can take that path
 * on purpose. Applies to launches made after the call, process-wide.
 */
dn_status dn_set_wait_limit_ns(unsigned long long ns);

/* Static, human-readable name of a status code. Never NULL. */
const char* dn_status_string(dn_status status);

/* Library version, major * 10000 + minor * 100 + patch. */
int dn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* DN_H_ */
