"""fp64 CPU oracle of the gated delta-rule recurrence.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers. Nothing here is shared with the CUDA
path, and nothing here imports it.

Three evaluations live here, each independent of the CUDA path:

* ``fwd`` -- the definition itself: a sequential fp64 loop over tokens per
  (batch, head), in plain C (``dn_oracle.c``), OpenMP across heads. This is the
  oracle that parity tests compare the GPU against.
* ``osdn_precond`` -- OSDN phase 1, the preconditioner sequence d_t that the
  OSDN key scale takes (sequential fp64 loop in the same C file).
* ``bwd`` -- the reverse mode of the definition: the gradients of
  sum <dO, o> + <dS_T, S_T> with respect to every input, by the chain rule
  walked token by token from the end (same C file).
* ``chunked.fwd`` -- the chunkwise-parallel (WY / UT-transform) evaluation of
  the same recurrence in NumPy fp64, following the chunk algebra the kernels
  use. It is never compared against the GPU; it exists so that tests can show
  the chunk algebra equals the sequential definition on small inputs.

Every input array uses the public layouts: q, k [B,T,H,dk]; v [B,T,H,dv];
gates [B,T,H] (one per token) or [B,T,H,n] (one per channel) or None (absent,
i.e. 1); S0 [B,H,dk,dv] or None (zero). Arrays may be float32/float64 or bf16
bit patterns (np.uint16), which are widened exactly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libdnoracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile dn_oracle.c into libdnoracle.so (gcc -O2, OpenMP)."""
    src = os.path.join(_HERE, "dn_oracle.c")
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(src):
        subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _LIB_PATH, src, "-lm"],
                       check=True)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.dn_oracle_heads.argtypes = [I, I, I, I, P, P, P, P, I, P, I, P, I, P, I, P, P, I, I]
            lib.dn_oracle_heads.restype = I
            lib.dn_oracle_max_threads.restype = I
            lib.dn_oracle_osdn_heads.argtypes = [I, I, I, P, P, P, ctypes.c_double, P, P, I]
            lib.dn_oracle_osdn_heads.restype = I
            lib.dn_oracle_bwd_heads.argtypes = [I, I, I, I, P, P, P, P, I, P, I, P, I, P, I, P, P, P, I,
                                                P, P, P, P, P, P, P, P, I]
            lib.dn_oracle_bwd_heads.restype = I
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().dn_oracle_max_threads())


def widen(x, bf16: bool | None = None) -> np.ndarray | None:
    """Exact conversion to float64 (bf16 bit patterns arrive as np.uint16)."""
    if x is None:
        return None
    x = np.asarray(x)
    if x.dtype == np.uint16 or bf16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def _per_head(x, heads, width_expected):
    """[B,T,H(,n)] -> [NH,T,n] contiguous fp64 for the selected (b, h) pairs; width."""
    if x is None:
        return None, 0
    x = np.asarray(x)
    if x.ndim == 3:
        g = np.stack([widen(x[b, :, h]) for (b, h) in heads])[..., None]
        return np.ascontiguousarray(g), 1
    assert x.shape[-1] == width_expected, (x.shape, width_expected)
    g = np.stack([widen(x[b, :, h, :]) for (b, h) in heads])
    return np.ascontiguousarray(g), width_expected


def fwd(q, k, v, alpha=None, beta_k=None, beta_v=None, key_scale=None, S0=None,
        heads=None, nthreads: int = 0, readout: str = "post"):
    """Sequential fp64 recurrence. Returns (o, S_T).

    readout="post": o_t = S_t^T q_t (after the token's update); "pre": o_t = S_{t-1}^T q_t.

    With ``heads=None`` every (b, h) runs and o is [B,T,H,dv], S_T [B,H,dk,dv].
    With ``heads=[(b, h), ...]`` only those run and o is [NH,T,dv], S_T [NH,dk,dv].
    """
    q = np.asarray(q)
    B, T, H, dk = q.shape
    dv = np.asarray(v).shape[-1]
    all_heads = heads is None
    if all_heads:
        heads = [(b, h) for b in range(B) for h in range(H)]
    NH = len(heads)
    qh, _ = _per_head(q, heads, dk)
    kh, _ = _per_head(k, heads, dk)
    vh, _ = _per_head(v, heads, dv)
    qh, kh, vh = qh.reshape(NH, T, dk), kh.reshape(NH, T, dk), vh.reshape(NH, T, dv)
    ah, aw = _per_head(alpha, heads, dk)
    bkh, bkw = _per_head(beta_k, heads, dk)
    bvh, bvw = _per_head(beta_v, heads, dv)
    dh, dw = _per_head(key_scale, heads, dk)
    if S0 is None:
        S = np.zeros((NH, dk, dv), dtype=np.float64)
    else:
        S0 = np.asarray(S0)
        S = np.ascontiguousarray(np.stack([widen(S0[b, h]) for (b, h) in heads]))
    o = np.zeros((NH, T, dv), dtype=np.float64)

    def ptr(a):
        return None if a is None else a.ctypes.data

    if readout not in ("post", "pre"):
        raise ValueError("readout must be 'post' or 'pre'")
    rc = _load().dn_oracle_heads(NH, T, dk, dv, ptr(qh), ptr(kh), ptr(vh), ptr(ah), aw, ptr(bkh), bkw,
                                 ptr(bvh), bvw, ptr(dh), dw, S.ctypes.data, o.ctypes.data,
                                 int(readout == "pre"), nthreads)
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    if not all_heads:
        return o, S
    o_full = np.empty((B, T, H, dv), dtype=np.float64)
    S_full = np.empty((B, H, dk, dv), dtype=np.float64)
    for n, (b, h) in enumerate(heads):
        o_full[b, :, h, :] = o[n]
        S_full[b, h] = S[n]
    return o_full, S_full


def bwd(q, k, v, alpha=None, beta_k=None, beta_v=None, key_scale=None, S0=None, dO=None, dS_T=None,
        heads=None, nthreads: int = 0, readout: str = "post"):
    """Reverse mode in fp64: the gradients of L = sum <dO, o> + <dS_T, S_T> (dS_T None: zero).

    Returns a dict with the gradient of every input under its own name ("q", "k", "v", "alpha",
    "beta_k", "beta_v", "key_scale", "S0"), each shaped like that input (None for an absent gate;
    "S0" is always [B,H,dk,dv]). With ``heads=[(b, h), ...]`` only those run and the leading
    [B,...,H] axes become one [NH] axis, as in ``fwd``.
    """
    q = np.asarray(q)
    B, T, H, dk = q.shape
    dv = np.asarray(v).shape[-1]
    all_heads = heads is None
    if all_heads:
        heads = [(b, h) for b in range(B) for h in range(H)]
    NH = len(heads)
    qh, _ = _per_head(q, heads, dk)
    kh, _ = _per_head(k, heads, dk)
    vh, _ = _per_head(v, heads, dv)
    dOh, _ = _per_head(dO, heads, dv)
    qh, kh, vh, dOh = (x.reshape(NH, T, -1) for x in (qh, kh, vh, dOh))
    gates = {}
    for name, x, n in (("alpha", alpha, dk), ("beta_k", beta_k, dk), ("beta_v", beta_v, dv),
                       ("key_scale", key_scale, dk)):
        gates[name] = _per_head(x, heads, n)

    def mats(x):
        if x is None:
            return None
        x = np.asarray(x)
        return np.ascontiguousarray(np.stack([widen(x[b, h]) for (b, h) in heads]))

    S0h, dSTh = mats(S0), mats(dS_T)
    out = {"q": np.zeros((NH, T, dk)), "k": np.zeros((NH, T, dk)), "v": np.zeros((NH, T, dv)),
           "S0": np.zeros((NH, dk, dv))}
    for name, (g, w) in gates.items():
        out[name] = None if g is None else np.zeros((NH, T, w))

    def ptr(a):
        return None if a is None else a.ctypes.data

    if readout not in ("post", "pre"):
        raise ValueError("readout must be 'post' or 'pre'")
    (ah, aw), (bkh, bkw), (bvh, bvw), (dh, dw) = (gates[n] for n in ("alpha", "beta_k", "beta_v", "key_scale"))
    rc = _load().dn_oracle_bwd_heads(NH, T, dk, dv, ptr(qh), ptr(kh), ptr(vh), ptr(ah), aw, ptr(bkh), bkw,
                                     ptr(bvh), bvw, ptr(dh), dw, ptr(S0h), ptr(dOh), ptr(dSTh),
                                     int(readout == "pre"), ptr(out["q"]), ptr(out["k"]), ptr(out["v"]),
                                     ptr(out["alpha"]), ptr(out["beta_k"]), ptr(out["beta_v"]),
                                     ptr(out["key_scale"]), ptr(out["S0"]), nthreads)
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    for name, x in (("alpha", alpha), ("beta_k", beta_k), ("beta_v", beta_v), ("key_scale", key_scale)):
        if x is not None and np.asarray(x).ndim == 3:
            out[name] = out[name][..., 0]
    if not all_heads:
        return out
    full = {}
    for name, g in out.items():
        if g is None:
            full[name] = None
            continue
        if name == "S0":
            f = np.empty((B, H) + g.shape[1:])
            for n, (b, h) in enumerate(heads):
                f[b, h] = g[n]
        else:
            f = np.empty((B, T, H) + g.shape[2:])
            for n, (b, h) in enumerate(heads):
                f[b, :, h] = g[n]
        full[name] = f
    return full


def osdn_precond(k, beta, retention=None, d0=None, eta: float = 0.5, heads=None, nthreads: int = 0):
    """OSDN phase 1 in fp64: the preconditioner d_t used by every token, and the final d_T.

    k [B,T,H,dk] (bf16 bits or float), beta [B,T,H] (the scalar write strength), retention
    [B,T,H] or None (no forgetting, r = 1), d0 [B,H,dk] or None (ones). Returns (d [B,T,H,dk],
    d_T [B,H,dk]); with ``heads=[(b, h), ...]`` only those run and the shapes are [NH,T,dk],
    [NH,dk].
    """
    k = np.asarray(k)
    B, T, H, dk = k.shape
    all_heads = heads is None
    if all_heads:
        heads = [(b, h) for b in range(B) for h in range(H)]
    NH = len(heads)
    kh = np.ascontiguousarray(np.stack([widen(k[b, :, h]) for (b, h) in heads])).reshape(NH, T, dk)
    bh = np.ascontiguousarray(np.stack([widen(np.asarray(beta)[b, :, h]) for (b, h) in heads]))
    rh = None
    if retention is not None:
        rh = np.ascontiguousarray(np.stack([widen(np.asarray(retention)[b, :, h]) for (b, h) in heads]))
    if d0 is None:
        d = np.ones((NH, dk), dtype=np.float64)
    else:
        d = np.ascontiguousarray(np.stack([widen(np.asarray(d0)[b, h]) for (b, h) in heads]))
    dseq = np.zeros((NH, T, dk), dtype=np.float64)
    rc = _load().dn_oracle_osdn_heads(NH, T, dk, kh.ctypes.data, bh.ctypes.data,
                                      None if rh is None else rh.ctypes.data, float(eta), d.ctypes.data,
                                      dseq.ctypes.data, nthreads)
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    if not all_heads:
        return dseq, d
    d_full = np.empty((B, T, H, dk), dtype=np.float64)
    dT_full = np.empty((B, H, dk), dtype=np.float64)
    for n, (b, h) in enumerate(heads):
        d_full[b, :, h, :] = dseq[n]
        dT_full[b, h] = d[n]
    return d_full, dT_full


def rel_l2(x, ref) -> float:
    """||x - ref||_2 / ||ref||_2 over the whole tensor, in fp64."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    num = np.linalg.norm((x - ref).ravel())
    return float(num / den) if den > 0 else float(num)


from . import chunked  # noqa: E402  (NumPy chunked evaluation, test-only)
from . import memcache  # noqa: E402  (Memory Caching over the recurrence, test-only)
