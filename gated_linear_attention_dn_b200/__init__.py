"""Python binding of libdn.so, the B200 (sm_100a) gated delta-rule library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in include/dn.h. PyTorch supplies device
memory and streams. There is no CPU path: if libdn.so is missing or cannot be
loaded, every call raises.

Entry points (same names as the C ABI):
    dn_chunk_fwd(q, k, v, alpha=None, beta_k=None, beta_v=None, key_scale=None,
                 S0=None, o=None, S_T=None, stream=None) -> (o, S_T)
    dn_decode_step(q, k, v, alpha=None, beta_k=None, beta_v=None, key_scale=None,
                   S=..., o=None, stream=None) -> o          (S updated in place)
    dn_chunk_bwd(q, k, v, alpha=None, beta_k=None, beta_v=None, key_scale=None, S0=None,
                 dO=..., dS_T=None, workspace=None, stream=None) -> dict of gradients
    dn_osdn_precond(k, beta, retention=None, d0=None, eta=0.5, d=None, d_T=None,
                    workspace=None, stream=None) -> (d, d_T)   (OSDN phase 1)
    dn_mc_readout(q, M, gates=None, o=..., seg_len=L, stream=None) -> o     (Memory Caching read-out)
    mc_fwd(q, k, v, ..., seg_len=L, gates=None) -> (o, M)   (segments + cached read-out)
    dn_stream_status(stream=None) -> int
    dn_status_string(code) -> str
    dn_set_wait_limit_ns(ns)        (diagnostics: bound of the chunk kernels' mbarrier waits)

Layouts: q, k [B,T,H,d_k]; v [B,T,H,d_v]; gates [B,T,H] (one per token),
[B,T,H,n] (one per channel) or None (absent = 1); states [B,H,d_k,d_v] fp32.
q/k/v/o are bf16 or fp32 CUDA tensors; gates fp32.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdn.so")

DN_OK, DN_ERR_INVALID_ARGUMENT, DN_ERR_UNSUPPORTED, DN_ERR_MISALIGNED = 0, 1, 2, 3
DN_ERR_WORKSPACE_TOO_SMALL, DN_ERR_CUDA, DN_ERR_DEVICE_TIMEOUT, DN_ERR_GATE_RANGE = 4, 5, 6, 7
DEFAULT_WAIT_NS = 2_000_000_000
DN_F32, DN_BF16 = 0, 1
DN_GATE_ONE, DN_GATE_SCALAR, DN_GATE_CHANNEL = 0, 1, 2
DN_READ_POST, DN_READ_PRE = 0, 1
_READOUT = {"post": DN_READ_POST, "pre": DN_READ_PRE}

EXPORTED = ("dn_chunk_fwd_workspace_bytes", "dn_chunk_fwd", "dn_decode_step", "dn_chunk_bwd_workspace_bytes",
            "dn_chunk_bwd", "dn_osdn_precond_workspace_bytes", "dn_osdn_precond", "dn_osdn_precond_noalloc",
            "dn_mc_readout", "dn_stream_status", "dn_status_string", "dn_version", "dn_set_wait_limit_ns")


class DnDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("d_k", ctypes.c_int),
                ("d_v", ctypes.c_int), ("chunk", ctypes.c_int), ("io_dtype", ctypes.c_int),
                ("alpha", ctypes.c_int), ("beta_k", ctypes.c_int), ("beta_v", ctypes.c_int),
                ("key_scale", ctypes.c_int), ("readout", ctypes.c_int)]


class DnOsdnDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("d_k", ctypes.c_int),
                ("io_dtype", ctypes.c_int), ("eta", ctypes.c_float)]


class DnMcDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int), ("d_k", ctypes.c_int),
                ("d_v", ctypes.c_int), ("seg_len", ctypes.c_int), ("io_dtype", ctypes.c_int)]


class DnError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {dn_status_string(code)} ({code})")
        self.code = code


_lib = None


def load(path: str = LIB_PATH):
    """Load libdn.so (raises if it is absent: there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libdn.so not built at {path}; run `python -m gated_linear_attention_dn_b200.build`")
    lib = ctypes.CDLL(path)
    P, I = ctypes.c_void_p, ctypes.c_int
    D = ctypes.POINTER(DnDesc)
    lib.dn_chunk_fwd_workspace_bytes.argtypes = [D]
    lib.dn_chunk_fwd_workspace_bytes.restype = ctypes.c_size_t
    lib.dn_chunk_fwd.argtypes = [D, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.dn_chunk_fwd.restype = I
    lib.dn_decode_step.argtypes = [D, P, P, P, P, P, P, P, P, P, P]
    lib.dn_decode_step.restype = I
    lib.dn_chunk_bwd_workspace_bytes.argtypes = [D]
    lib.dn_chunk_bwd_workspace_bytes.restype = ctypes.c_size_t
    lib.dn_chunk_bwd.argtypes = [D] + [P] * 19 + [ctypes.c_size_t, P]
    lib.dn_chunk_bwd.restype = I
    O = ctypes.POINTER(DnOsdnDesc)
    lib.dn_osdn_precond_workspace_bytes.argtypes = [O]
    lib.dn_osdn_precond_workspace_bytes.restype = ctypes.c_size_t
    lib.dn_osdn_precond.argtypes = [O, P, P, P, P, P, P, P, ctypes.c_size_t, P]
    lib.dn_osdn_precond.restype = I
    lib.dn_mc_readout.argtypes = [ctypes.POINTER(DnMcDesc), P, P, P, P, P]
    lib.dn_mc_readout.restype = I
    lib.dn_stream_status.argtypes = [P]
    lib.dn_stream_status.restype = I
    lib.dn_status_string.argtypes = [I]
    lib.dn_status_string.restype = ctypes.c_char_p
    lib.dn_version.restype = I
    lib.dn_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
    lib.dn_set_wait_limit_ns.restype = I
    _lib = lib
    return lib


def dn_status_string(code: int) -> str:
    return load().dn_status_string(int(code)).decode()


def dn_set_wait_limit_ns(ns: int) -> None:
    """Bound of every mbarrier wait of the tensor-core chunk kernels for later launches (default
    DEFAULT_WAIT_NS; 0 = one non-blocking probe per wait). A diagnostics hook for the timeout path."""
    code = load().dn_set_wait_limit_ns(int(ns))
    if code != DN_OK:
        raise DnError(code, "dn_set_wait_limit_ns")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _gate_mode(g, B, T, H, width, name):
    if g is None:
        return DN_GATE_ONE
    if g.dtype != torch.float32 or not g.is_contiguous():
        raise TypeError(f"{name} must be a contiguous float32 tensor")
    if tuple(g.shape) == (B, T, H):
        return DN_GATE_SCALAR
    if tuple(g.shape) == (B, T, H, width):
        return DN_GATE_CHANNEL
    raise ValueError(f"{name} has shape {tuple(g.shape)}; expected {(B, T, H)} or {(B, T, H, width)}")


def make_desc(q, v, alpha, beta_k, beta_v, key_scale, chunk: int = 0, readout: str = "post") -> DnDesc:
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if q.dtype == torch.bfloat16:
        io = DN_BF16
    elif q.dtype == torch.float32:
        io = DN_F32
    else:
        raise TypeError("q/k/v must be bfloat16 or float32")
    return DnDesc(B, T, H, dk, dv, chunk, io,
                  _gate_mode(alpha, B, T, H, dk, "alpha"), _gate_mode(beta_k, B, T, H, dk, "beta_k"),
                  _gate_mode(beta_v, B, T, H, dv, "beta_v"), _gate_mode(key_scale, B, T, H, dk, "key_scale"),
                  _READOUT[readout])


def _check_io(q, k, v):
    for n, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_contiguous():
            raise TypeError(f"{n} must be contiguous")
        if t.dtype != q.dtype:
            raise TypeError("q, k, v must share a dtype")
    if k.shape != q.shape or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k, v shapes disagree")


def dn_chunk_fwd_workspace_bytes(desc: DnDesc) -> int:
    return int(load().dn_chunk_fwd_workspace_bytes(ctypes.byref(desc)))


def dn_chunk_fwd(q, k, v, alpha=None, beta_k=None, beta_v=None, key_scale=None, S0=None, o=None,
                 S_T=None, stream=None, chunk: int = 0, workspace=None, readout: str = "post"):
    """Chunked prefill. Returns (o [B,T,H,d_v] io dtype, S_T [B,H,d_k,d_v] fp32).

    readout="post": o_t = S_t^T q_t; "pre": o_t = S_{t-1}^T q_t (before the token's update).
    workspace: None allocates the dn_chunk_fwd_workspace_bytes() the problem can use (the split
    transform + state-chain evaluation); False passes none (the fused one-kernel evaluation); a
    uint8 CUDA tensor is used as given."""
    lib = load()
    _check_io(q, k, v)
    desc = make_desc(q, v, alpha, beta_k, beta_v, key_scale, chunk, readout)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if o is None:
        o = torch.empty((B, T, H, dv), dtype=q.dtype, device=q.device)
    if S_T is None:
        S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    ws_bytes = dn_chunk_fwd_workspace_bytes(desc)
    if workspace is False:
        workspace = None
    elif ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    rc = lib.dn_chunk_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta_k),
                          _ptr(beta_v), _ptr(key_scale), _ptr(S0), _ptr(o), _ptr(S_T), _ptr(workspace),
                          workspace.numel() if workspace is not None else 0, _stream_handle(stream))
    if rc != DN_OK:
        raise DnError(rc, "dn_chunk_fwd")
    return o, S_T


def dn_decode_step(q, k, v, alpha=None, beta_k=None, beta_v=None, key_scale=None, S=None, o=None,
                   stream=None, readout: str = "post"):
    """One recurrent step; S [B,H,d_k,d_v] fp32 is updated in place. Returns o [B,1,H,d_v]
    (readout="pre": o = S^T q from the state before this step)."""
    lib = load()
    _check_io(q, k, v)
    if S is None:
        raise ValueError("decode needs the resident state S")
    desc = make_desc(q, v, alpha, beta_k, beta_v, key_scale, 0, readout)
    if o is None:
        o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    rc = lib.dn_decode_step(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta_k),
                            _ptr(beta_v), _ptr(key_scale), _ptr(S), _ptr(o), _stream_handle(stream))
    if rc != DN_OK:
        raise DnError(rc, "dn_decode_step")
    return o


def dn_chunk_bwd_workspace_bytes(desc: DnDesc) -> int:
    return int(load().dn_chunk_bwd_workspace_bytes(ctypes.byref(desc)))


def dn_chunk_bwd(q, k, v, alpha=None, beta_k=None, beta_v=None, key_scale=None, S0=None, dO=None, dS_T=None,
                 workspace=None, want_dS0: bool = True, out=None, stream=None, readout: str = "post"):
    """Backward of dn_chunk_fwd with the same read-out: the gradients of sum <dO, o> + <dS_T, S_T>.
    dO [B,T,H,d_v] in the io dtype; dS_T [B,H,d_k,d_v] fp32 or None (zero).

    Returns {"q", "k", "v"} (io dtype, shaped like the inputs), {"alpha", "beta_k", "beta_v",
    "key_scale"} (fp32, shaped like each gate; None for an absent gate) and "S0" (fp32
    [B,H,d_k,d_v], or None when want_dS0 is False). The workspace (dn_chunk_bwd_workspace_bytes)
    is allocated here when not given; so are the outputs, unless `out` (a dict returned by an
    earlier call of the same shapes) is passed to be written again.
    """
    lib = load()
    _check_io(q, k, v)
    desc = make_desc(q, v, alpha, beta_k, beta_v, key_scale, 0, readout)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if dO is None or not dO.is_contiguous() or dO.dtype != q.dtype or tuple(dO.shape) != (B, T, H, dv):
        raise ValueError("dO must be a contiguous [B,T,H,d_v] tensor of q's dtype")
    if dS_T is not None and (dS_T.dtype != torch.float32 or not dS_T.is_contiguous()
                             or tuple(dS_T.shape) != (B, H, dk, dv)):
        raise ValueError("dS_T must be a contiguous float32 [B,H,d_k,d_v] tensor")
    if out is None:
        out = {"q": torch.empty_like(q), "k": torch.empty_like(k), "v": torch.empty_like(v)}
        for name, g in (("alpha", alpha), ("beta_k", beta_k), ("beta_v", beta_v), ("key_scale", key_scale)):
            out[name] = None if g is None else torch.empty_like(g)
        out["S0"] = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device) if want_dS0 else None
    else:
        for name, ref in (("q", q), ("k", k), ("v", v), ("alpha", alpha), ("beta_k", beta_k), ("beta_v", beta_v),
                          ("key_scale", key_scale)):
            t = out.get(name)
            if (t is None) != (ref is None) or (t is not None and (t.shape != ref.shape or t.dtype != ref.dtype
                                                                   or not t.is_contiguous())):
                raise ValueError(f"out[{name!r}] does not match {name}")
        t = out.get("S0")
        if t is not None and (t.dtype != torch.float32 or not t.is_contiguous() or tuple(t.shape) != (B, H, dk, dv)):
            raise ValueError("out['S0'] must be a contiguous float32 [B,H,d_k,d_v] tensor or None")
    ws_bytes = dn_chunk_bwd_workspace_bytes(desc)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    rc = lib.dn_chunk_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta_k), _ptr(beta_v),
                          _ptr(key_scale), _ptr(S0), _ptr(dO), _ptr(dS_T), _ptr(out["q"]), _ptr(out["k"]),
                          _ptr(out["v"]), _ptr(out["alpha"]), _ptr(out["beta_k"]), _ptr(out["beta_v"]),
                          _ptr(out["key_scale"]), _ptr(out["S0"]), _ptr(workspace),
                          ws_bytes if workspace is not None else 0, _stream_handle(stream))
    if rc != DN_OK:
        raise DnError(rc, "dn_chunk_bwd")
    return out


def dn_osdn_precond_workspace_bytes(desc: DnOsdnDesc) -> int:
    return int(load().dn_osdn_precond_workspace_bytes(ctypes.byref(desc)))


def dn_osdn_precond(k, beta, retention=None, d0=None, eta: float = 0.5, d=None, d_T=None, workspace=None,
                    stream=None):
    """OSDN phase 1: the preconditioner d_t of every token. Returns (d [B,T,H,d_k], d_T [B,H,d_k]) fp32.

    k [B,T,H,d_k] bf16 or fp32; beta [B,T,H] fp32; retention [B,T,H] fp32 or None; d0 [B,H,d_k] fp32 or
    None (ones). The workspace (dn_osdn_precond_workspace_bytes) is allocated here when not given.
    """
    lib = load()
    if not k.is_contiguous():
        raise TypeError("k must be contiguous")
    B, T, H, dk = k.shape
    io = DN_BF16 if k.dtype == torch.bfloat16 else DN_F32 if k.dtype == torch.float32 else None
    if io is None:
        raise TypeError("k must be bfloat16 or float32")
    for n, g, shape in (("beta", beta, (B, T, H)), ("retention", retention, (B, T, H)), ("d0", d0, (B, H, dk))):
        if g is None:
            continue
        if g.dtype != torch.float32 or not g.is_contiguous() or tuple(g.shape) != shape:
            raise ValueError(f"{n} must be a contiguous float32 tensor of shape {shape}")
    desc = DnOsdnDesc(B, T, H, dk, io, float(eta))
    if d is None:
        d = torch.empty((B, T, H, dk), dtype=torch.float32, device=k.device)
    if d_T is None:
        d_T = torch.empty((B, H, dk), dtype=torch.float32, device=k.device)
    ws_bytes = dn_osdn_precond_workspace_bytes(desc)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=k.device)
    rc = lib.dn_osdn_precond(ctypes.byref(desc), _ptr(k), _ptr(beta), _ptr(retention), _ptr(d0), _ptr(d),
                             _ptr(d_T), _ptr(workspace), ws_bytes if workspace is not None else 0,
                             _stream_handle(stream))
    if rc != DN_OK:
        raise DnError(rc, "dn_osdn_precond")
    return d, d_T


def dn_mc_readout(q, M, gates=None, o=None, seg_len: int = 64, stream=None):
    """o [B,T,H,d_v] += sum_{s < t // seg_len} gates[b,t,h,s] M[b,s,h]^T q_t, in place (gates None: 1)."""
    lib = load()
    B, T, H, dk = q.shape
    dv = M.shape[-1]
    io = DN_BF16 if q.dtype == torch.bfloat16 else DN_F32
    if o is None or not o.is_contiguous() or o.dtype != q.dtype or tuple(o.shape) != (B, T, H, dv):
        raise ValueError("o must be a contiguous [B,T,H,d_v] tensor of q's dtype (it is accumulated into)")
    N = (T + seg_len - 1) // seg_len
    if M.dtype != torch.float32 or not M.is_contiguous() or tuple(M.shape) != (B, N, H, dk, dv):
        raise ValueError(f"M must be a contiguous float32 tensor of shape {(B, N, H, dk, dv)}")
    if gates is not None and (gates.dtype != torch.float32 or not gates.is_contiguous()
                              or tuple(gates.shape) != (B, T, H, N)):
        raise ValueError(f"gates must be a contiguous float32 tensor of shape {(B, T, H, N)}")
    desc = DnMcDesc(B, T, H, dk, dv, seg_len, io)
    rc = lib.dn_mc_readout(ctypes.byref(desc), _ptr(q), _ptr(M), _ptr(gates), _ptr(o), _stream_handle(stream))
    if rc != DN_OK:
        raise DnError(rc, "dn_mc_readout")
    return o


def mc_fwd(q, k, v, alpha=None, beta_k=None, beta_v=None, key_scale=None, S0=None, seg_len: int = 64,
           gates=None, readout: str = "post", stream=None):
    """Memory Caching over the recurrence: every segment of seg_len tokens runs from S0 (or zero)
    and its final state is cached; each token adds the gated read of the earlier segments'
    memories. Returns (o [B,T,H,d_v], M [B,N,H,d_k,d_v]). T must be a multiple of seg_len."""
    B, T, H, dk = q.shape
    if seg_len <= 0 or T % seg_len:
        raise ValueError("T must be a positive multiple of seg_len")
    N = T // seg_len

    def seg(x):  # [B, T, ...] -> [B*N, L, ...], the same memory
        return None if x is None else x.view(B * N, seg_len, *x.shape[2:])

    S0r = None if S0 is None else S0.repeat_interleave(N, dim=0).contiguous()
    o, M = dn_chunk_fwd(seg(q), seg(k), seg(v), seg(alpha), seg(beta_k), seg(beta_v), seg(key_scale), S0r,
                        stream=stream, readout=readout)
    o = o.view(B, T, H, -1)
    M = M.view(B, N, H, dk, -1)
    dn_mc_readout(q, M, gates, o, seg_len, stream)
    return o, M


def dn_stream_status(stream=None) -> int:
    return int(load().dn_stream_status(_stream_handle(stream)))


def dn_version() -> int:
    return int(load().dn_version())
