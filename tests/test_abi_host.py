"""C ABI checks that need no GPU: the library loads, exports every declared
entry point, and rejects bad arguments before touching the device."""
import ctypes
import os
import re

import numpy as np
import pytest

import gated_linear_attention_dn_b200 as dn
from gated_linear_attention_dn_b200 import build as dnbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    dnbuild.build()
    return dn.load()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(dn_[a-z_0-9]+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert {"dn_chunk_fwd", "dn_decode_step", "dn_stream_status", "dn_status_string"} <= names
    for n in names:
        assert hasattr(lib, n), f"libdn.so does not export {n}"
    for n in dn.EXPORTED:
        assert n in names


def test_status_strings(lib):
    assert dn.dn_status_string(0) == "DN_OK"
    assert dn.dn_status_string(6) == "DN_ERR_DEVICE_TIMEOUT"
    assert dn.dn_status_string(99) == "DN_ERR_UNKNOWN"
    assert dn.dn_version() >= 100


class _Buf:
    """16-byte aligned host scratch whose address stands in for a device pointer;
    validation failures return before any pointer is dereferenced or any CUDA call."""

    def __init__(self, n=4096):
        self.raw = np.zeros(n + 64, dtype=np.uint8)
        base = self.raw.ctypes.data
        self.addr = (base + 15) & ~15

    def p(self, off=0):
        return ctypes.c_void_p(self.addr + off)


def _desc(**kw):
    d = dict(B=1, T=8, H=2, d_k=64, d_v=64, chunk=0, io_dtype=dn.DN_BF16, alpha=dn.DN_GATE_SCALAR,
             beta_k=dn.DN_GATE_SCALAR, beta_v=dn.DN_GATE_ONE, key_scale=dn.DN_GATE_ONE)
    d.update(kw)
    return dn.DnDesc(**d)


def _call(lib, desc, off=None, **ptrs):
    bufs = {n: _Buf() for n in ("q", "k", "v", "a", "bk", "bv", "d", "s0", "o", "st")}
    p = {n: b.p() for n, b in bufs.items()}
    p["bv"] = None
    p["d"] = None
    p.update(ptrs)
    return lib.dn_chunk_fwd(ctypes.byref(desc) if desc is not None else None, p["q"], p["k"], p["v"],
                            p["a"], p["bk"], p["bv"], p["d"], p["s0"], p["o"], p["st"], None, 0, None)


def test_rejects_bad_descriptors(lib):
    assert _call(lib, None) == dn.DN_ERR_INVALID_ARGUMENT
    assert _call(lib, _desc(B=0)) == dn.DN_ERR_INVALID_ARGUMENT
    assert _call(lib, _desc(T=-1)) == dn.DN_ERR_INVALID_ARGUMENT
    assert _call(lib, _desc(io_dtype=7)) == dn.DN_ERR_INVALID_ARGUMENT
    assert _call(lib, _desc(alpha=5)) == dn.DN_ERR_INVALID_ARGUMENT
    assert _call(lib, _desc(d_k=96)) == dn.DN_ERR_UNSUPPORTED
    assert _call(lib, _desc(d_v=256)) == dn.DN_ERR_UNSUPPORTED
    assert _call(lib, _desc(chunk=48)) == dn.DN_ERR_UNSUPPORTED
    assert _call(lib, _desc(chunk=128)) == dn.DN_ERR_UNSUPPORTED
    assert _call(lib, _desc(chunk=-1)) == dn.DN_ERR_INVALID_ARGUMENT
    assert _call(lib, _desc(readout=2)) == dn.DN_ERR_INVALID_ARGUMENT
    assert _call(lib, _desc(d_k=8, d_v=64)) == dn.DN_ERR_UNSUPPORTED  # small and large dims do not mix
    assert _call(lib, _desc(d_k=32, d_v=32)) == dn.DN_ERR_UNSUPPORTED


def test_rejects_bad_pointers(lib):
    b = _Buf()
    # gate present iff its mode is not DN_GATE_ONE
    assert _call(lib, _desc(), a=None) == dn.DN_ERR_INVALID_ARGUMENT
    assert _call(lib, _desc(), bv=b.p()) == dn.DN_ERR_INVALID_ARGUMENT
    assert _call(lib, _desc(), q=None) == dn.DN_ERR_INVALID_ARGUMENT
    assert _call(lib, _desc(), o=None) == dn.DN_ERR_INVALID_ARGUMENT
    assert _call(lib, _desc(), st=None) == dn.DN_ERR_INVALID_ARGUMENT
    assert _call(lib, _desc(), k=b.p(4)) == dn.DN_ERR_MISALIGNED
    assert _call(lib, _desc(), a=b.p(2)) == dn.DN_ERR_MISALIGNED
    assert _call(lib, _desc(alpha=dn.DN_GATE_CHANNEL), a=b.p(8)) == dn.DN_ERR_MISALIGNED
    assert _call(lib, _desc(), o=b.p(2)) == dn.DN_ERR_MISALIGNED
    # o overlapping q
    q = _Buf()
    assert _call(lib, _desc(), q=q.p(), o=q.p(16)) == dn.DN_ERR_INVALID_ARGUMENT


def test_decode_rejects_bad_arguments(lib):
    b = _Buf()
    d = _desc(T=2)
    args = [b.p(), b.p(), b.p(), b.p(), b.p(), None, None, b.p(), b.p(), None]
    assert lib.dn_decode_step(ctypes.byref(d), *args) == dn.DN_ERR_INVALID_ARGUMENT  # T must be 1
    d = _desc(T=1)
    bad = list(args)
    bad[7] = b.p(4)  # misaligned S
    assert lib.dn_decode_step(ctypes.byref(d), *bad) == dn.DN_ERR_MISALIGNED
    bad = list(args)
    bad[7] = None
    assert lib.dn_decode_step(ctypes.byref(d), *bad) == dn.DN_ERR_INVALID_ARGUMENT


def _fwd32_bytes(B, T, H, dk, dv, C=64):
    """The fp32 chunked forward's workspace: per (b, h, chunk of C tokens) T, P (C x C), S_m (d_k x d_v),
    U (C x d_v), K+, Q+, W- (C x d_k), e^r, lam (d_k), fp32; then one int per chunk; the whole rounded
    up to 16 bytes."""
    nc = -(-T // C)
    per = 2 * C * C + dk * dv + C * dv + 3 * C * dk + 2 * dk
    return (B * H * nc * (per * 4 + 4) + 15) // 16 * 16


def test_workspace_query(lib):
    # bf16 with d_k = 64 and fp32 io take the fp32 chunked forward through a workspace
    assert dn.dn_chunk_fwd_workspace_bytes(_desc()) == _fwd32_bytes(1, 8, 2, 64, 64)
    assert dn.dn_chunk_fwd_workspace_bytes(_desc(io_dtype=dn.DN_F32, d_k=128, d_v=64, T=130)) == \
        _fwd32_bytes(1, 130, 2, 128, 64)
    # small states take none; per-channel bf16 d_k = 128 takes one record per (b, h, chunk): [K+; Q+],
    # [T; P], W- hi and lo, the factor block, V~ hi and lo when beta^v is given, alpha and w rows
    assert dn.dn_chunk_fwd_workspace_bytes(_desc(d_k=8, d_v=8)) == 0
    rec = 32768 + 16384 + 2 * 16384 + 2048 + 2 * 64 * 128 * 4
    assert dn.dn_chunk_fwd_workspace_bytes(_desc(d_k=128, d_v=128, alpha=dn.DN_GATE_CHANNEL)) == 1 * 2 * 1 * rec
    assert dn.dn_chunk_fwd_workspace_bytes(_desc(d_k=128, d_v=64, T=130, alpha=dn.DN_GATE_CHANNEL,
                                                 beta_v=dn.DN_GATE_CHANNEL)) == 1 * 2 * 3 * (rec + 2 * 64 * 64 * 2)
    # (taken for few sequences only, B H 2 <= SMs; more take the fused kernel without a workspace)
    assert dn.dn_chunk_fwd_workspace_bytes(_desc(B=80, H=1, d_k=128, d_v=128, alpha=dn.DN_GATE_CHANNEL)) == 0
    assert dn.dn_chunk_fwd_workspace_bytes(_desc(T=0)) == 0
    assert lib.dn_chunk_fwd_workspace_bytes(None) == 0


def test_chunk_lengths(lib):
    """chunk in {16, 32}: the chunk form in fp32 with that chunk length, for every d_k, d_v and io dtype
    (bf16 d_k = 128 included: the tensor-core kernels' tiles are 64 tokens); 0 means 64; small states
    have no chunks; the backward's chunks are 64 tokens."""
    for C in (16, 32):
        for io in (dn.DN_BF16, dn.DN_F32):
            for dk, dv in ((64, 64), (64, 128), (128, 64), (128, 128)):
                for al in (dn.DN_GATE_SCALAR, dn.DN_GATE_CHANNEL):
                    d = _desc(chunk=C, io_dtype=io, d_k=dk, d_v=dv, T=130, alpha=al)
                    assert dn.dn_chunk_fwd_workspace_bytes(d) == _fwd32_bytes(1, 130, 2, dk, dv, C), (C, io, dk, dv)
    assert dn.dn_chunk_fwd_workspace_bytes(_desc(chunk=64)) == dn.dn_chunk_fwd_workspace_bytes(_desc(chunk=0))
    assert dn.dn_chunk_fwd_workspace_bytes(_desc(chunk=16, d_k=8, d_v=8)) == 0
    assert lib.dn_chunk_bwd_workspace_bytes(ctypes.byref(_desc(chunk=32))) == 0  # rejected
    assert lib.dn_chunk_bwd_workspace_bytes(ctypes.byref(_desc(chunk=64))) > 0
    assert lib.dn_chunk_bwd_workspace_bytes(ctypes.byref(_desc(chunk=16, d_k=8, d_v=8))) > 0


def test_binding_has_no_cpu_path(tmp_path):
    with pytest.raises(RuntimeError):
        dn.load.__wrapped__ if hasattr(dn.load, "__wrapped__") else None
        saved = dn._lib
        try:
            dn._lib = None
            dn.load(str(tmp_path / "missing.so"))
        finally:
            dn._lib = saved


def _odesc(B=1, T=64, H=2, dk=128, io=dn.DN_BF16, eta=0.5):
    return dn.DnOsdnDesc(B, T, H, dk, io, eta)


def test_osdn_workspace_and_validation(lib):
    # 4224 bytes per head per 32 tokens (a 32x32 fp32 matrix and a 32-vector)
    assert dn.dn_osdn_precond_workspace_bytes(_odesc(B=2, T=65, H=3)) == 2 * 3 * 3 * 4224
    assert dn.dn_osdn_precond_workspace_bytes(_odesc(dk=96)) == 0
    assert lib.dn_osdn_precond_workspace_bytes(None) == 0
    P = ctypes.c_void_p
    good = P(1 << 20)  # a 16-byte-aligned address the library only inspects, never touches here
    ws = dn.dn_osdn_precond_workspace_bytes(_odesc())

    def call(desc, k=good, beta=good, ret=None, d0=None, d=P(1 << 30), dT=None, w=P(1 << 24), wb=ws):
        return lib.dn_osdn_precond(ctypes.byref(desc), k, beta, ret, d0, d, dT, w, wb, None)

    assert call(_odesc(B=0)) == dn.DN_ERR_INVALID_ARGUMENT
    assert call(_odesc(T=-1)) == dn.DN_ERR_INVALID_ARGUMENT
    assert call(_odesc(eta=float("nan"))) == dn.DN_ERR_INVALID_ARGUMENT
    assert call(_odesc(eta=-1.0)) == dn.DN_ERR_INVALID_ARGUMENT
    assert call(_odesc(io=7)) == dn.DN_ERR_INVALID_ARGUMENT
    assert call(_odesc(dk=96)) == dn.DN_ERR_UNSUPPORTED
    assert call(_odesc(), k=None) == dn.DN_ERR_INVALID_ARGUMENT
    assert call(_odesc(), beta=None) == dn.DN_ERR_INVALID_ARGUMENT
    assert call(_odesc(), d=None) == dn.DN_ERR_INVALID_ARGUMENT
    assert call(_odesc(), k=P((1 << 20) + 8)) == dn.DN_ERR_MISALIGNED
    assert call(_odesc(), beta=P((1 << 20) + 2)) == dn.DN_ERR_MISALIGNED
    assert call(_odesc(), ret=P((1 << 20) + 1)) == dn.DN_ERR_MISALIGNED
    assert call(_odesc(), w=None) == dn.DN_ERR_WORKSPACE_TOO_SMALL
    assert call(_odesc(), wb=ws - 1) == dn.DN_ERR_WORKSPACE_TOO_SMALL
    assert call(_odesc(), w=P((1 << 24) + 4)) == dn.DN_ERR_MISALIGNED
    assert call(_odesc(), d=P(1 << 24)) == dn.DN_ERR_INVALID_ARGUMENT  # output overlaps the workspace
    # T == 0 with no d_T: nothing to do
    assert call(_odesc(T=0), k=None, beta=None, d=None, w=None, wb=0) == dn.DN_OK


def _bwd_call(lib, desc, ws_bytes=None, **ptrs):
    names = ("q", "k", "v", "a", "bk", "bv", "d", "s0", "dO", "dST", "gq", "gk", "gv", "ga", "gbk", "gbv", "gd",
             "gs0", "ws")
    bufs = {n: _Buf() for n in names}
    p = {n: b.p() for n, b in bufs.items()}
    for n in ("bv", "d", "gbv", "gd"):  # the default descriptor has no beta^v and no key scale
        p[n] = None
    p.update(ptrs)
    if ws_bytes is None:
        ws_bytes = lib.dn_chunk_bwd_workspace_bytes(ctypes.byref(desc))
    return lib.dn_chunk_bwd(ctypes.byref(desc), *(p[n] for n in names), ws_bytes, None)


def test_bwd_workspace_bytes(lib):
    d = _desc(B=2, T=130, H=3, d_k=128, d_v=64)
    nc = 3  # ceil(130 / 64)
    # per chunk: T, P (64 x 64); S_m, dX (d_k x d_v); U, dV~ (64 x d_v); K+, Q+, W-, e^h (64 x d_k); e^r, lam (d_k)
    per = 2 * 64 * 64 + 2 * 128 * 64 + 2 * 64 * 64 + 4 * 64 * 128 + 2 * 128
    assert lib.dn_chunk_bwd_workspace_bytes(ctypes.byref(d)) == 2 * 3 * nc * per * 4
    # small states keep the state entering every token: B * H * T * d_k * d_v floats
    assert lib.dn_chunk_bwd_workspace_bytes(ctypes.byref(_desc(d_k=8, d_v=16))) == 1 * 2 * 8 * 8 * 16 * 4
    assert lib.dn_chunk_bwd_workspace_bytes(ctypes.byref(_desc(d_k=16, d_v=8, readout=dn.DN_READ_PRE))) == 2 * 8 * 128 * 4


def test_bwd_rejects_bad_arguments(lib):
    assert lib.dn_chunk_bwd_workspace_bytes(ctypes.byref(_desc(readout=dn.DN_READ_PRE))) > 0  # both read-outs
    assert _bwd_call(lib, _desc(d_k=16, d_v=64), ws_bytes=1 << 20) == dn.DN_ERR_UNSUPPORTED  # mixed small and big
    assert _bwd_call(lib, _desc(B=0)) == dn.DN_ERR_INVALID_ARGUMENT
    assert _bwd_call(lib, _desc(), dO=None) == dn.DN_ERR_INVALID_ARGUMENT
    assert _bwd_call(lib, _desc(), gq=None) == dn.DN_ERR_INVALID_ARGUMENT
    # a gate gradient is given exactly when its gate is
    assert _bwd_call(lib, _desc(), ga=None) == dn.DN_ERR_INVALID_ARGUMENT
    assert _bwd_call(lib, _desc(), gbv=_Buf().p()) == dn.DN_ERR_INVALID_ARGUMENT
    assert _bwd_call(lib, _desc(), gbk=_Buf().p(2)) == dn.DN_ERR_MISALIGNED
    assert _bwd_call(lib, _desc(), gq=_Buf().p(8)) == dn.DN_ERR_MISALIGNED
    assert _bwd_call(lib, _desc(), dST=_Buf().p(4)) == dn.DN_ERR_MISALIGNED
    need = lib.dn_chunk_bwd_workspace_bytes(ctypes.byref(_desc()))
    assert _bwd_call(lib, _desc(), ws_bytes=need - 1) == dn.DN_ERR_WORKSPACE_TOO_SMALL
    assert _bwd_call(lib, _desc(), ws=None) == dn.DN_ERR_WORKSPACE_TOO_SMALL
    # the q gradient may not overlap q (it is written while q is still read)
    shared = _Buf(1 << 16)
    assert _bwd_call(lib, _desc(), q=shared.p(), gq=shared.p(256)) == dn.DN_ERR_INVALID_ARGUMENT
    # no tokens and no dS0 wanted: nothing to do
    assert _bwd_call(lib, _desc(T=0), gs0=None) == dn.DN_OK


def test_binding_bwd_checks_arguments_before_the_library(lib):
    """dn_chunk_bwd's argument checks raise before any call into libdn.so (CPU tensors are enough)."""
    import torch
    q = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16)
    v = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16)
    a = torch.ones(1, 8, 2)
    with pytest.raises(ValueError, match="dO"):
        dn.dn_chunk_bwd(q, q, v, a, a, dO=None)
    with pytest.raises(ValueError, match="dO"):
        dn.dn_chunk_bwd(q, q, v, a, a, dO=torch.zeros(1, 8, 2, 64))  # fp32 dO for bf16 inputs
    with pytest.raises(ValueError, match="dS_T"):
        dn.dn_chunk_bwd(q, q, v, a, a, dO=v, dS_T=torch.zeros(1, 2, 64, 32))
    with pytest.raises(ValueError, match="out"):
        dn.dn_chunk_bwd(q, q, v, a, a, dO=v, out={"q": q, "k": q, "v": v, "alpha": None, "beta_k": a})
    with pytest.raises(TypeError):
        dn.dn_chunk_bwd(q, q.float(), v, a, a, dO=v)


def test_decode_rejects_o_overlapping_its_inputs(lib):
    # o is written by one column slice of a head while the other slice still reads S, q, k, v
    d = _desc(T=1, alpha=dn.DN_GATE_CHANNEL, beta_k=dn.DN_GATE_CHANNEL)
    bufs = {n: _Buf(1 << 16) for n in ("q", "k", "v", "a", "bk", "S", "o")}

    def call(**over):
        p = {n: b.p() for n, b in bufs.items()}
        p.update(over)
        return lib.dn_decode_step(ctypes.byref(d), p["q"], p["k"], p["v"], p["a"], p["bk"], None, None, p["S"],
                                  p["o"], None)

    for name in ("S", "q", "k", "v"):
        assert call(o=bufs[name].p(32)) == dn.DN_ERR_INVALID_ARGUMENT, name


def test_chunk_fwd_rejects_state_overlaps(lib):
    s = _Buf(1 << 17)
    nS = 1 * 2 * 64 * 64 * 4
    # S0 partly overlapping S_T (exact aliasing, S_T == S0, is the supported in-place form)
    assert _call(lib, _desc(), s0=s.p(0), st=s.p(nS // 2)) == dn.DN_ERR_INVALID_ARGUMENT
    assert _call(lib, _desc(), s0=s.p(0), st=s.p(0)) != dn.DN_ERR_INVALID_ARGUMENT
    # S_T overlapping an input it is written while reading
    q = _Buf(1 << 17)
    assert _call(lib, _desc(), q=q.p(), st=q.p(64)) == dn.DN_ERR_INVALID_ARGUMENT
    a = _Buf(1 << 17)
    assert _call(lib, _desc(), a=a.p(), st=a.p(16)) == dn.DN_ERR_INVALID_ARGUMENT


def test_gate_range_status_and_wait_hook(lib):
    assert dn.dn_status_string(dn.DN_ERR_GATE_RANGE) == "DN_ERR_GATE_RANGE"
    # the diagnostics hook only records the bound; put the default back
    dn.dn_set_wait_limit_ns(0)
    dn.dn_set_wait_limit_ns(dn.DEFAULT_WAIT_NS)


def test_chunk_fwd_workspace_checks(lib):
    d = _desc(d_k=128, d_v=128, T=100)
    need = lib.dn_chunk_fwd_workspace_bytes(ctypes.byref(d))
    assert need == 2 * 2 * 25616  # B H chunks x record
    assert lib.dn_chunk_fwd_workspace_bytes(ctypes.byref(_desc(d_k=128, d_v=128, io_dtype=dn.DN_F32))) == \
        _fwd32_bytes(1, 8, 2, 128, 128)
    big = np.zeros(1 << 20, dtype=np.uint8)
    ws = ctypes.c_void_p((big.ctypes.data + 15) & ~15)
    bufs = {n: _Buf(1 << 18) for n in ("q", "k", "v", "a", "bk", "o", "st")}
    p = {n: b.p() for n, b in bufs.items()}

    def call(w, nbytes):
        return lib.dn_chunk_fwd(ctypes.byref(d), p["q"], p["k"], p["v"], p["a"], p["bk"], None, None, None, p["o"],
                                p["st"], w, nbytes, None)

    assert call(ws, need - 16) == dn.DN_ERR_WORKSPACE_TOO_SMALL
    assert call(ctypes.c_void_p(ws.value + 8), need) == dn.DN_ERR_MISALIGNED
    assert call(bufs["q"].p(), need) == dn.DN_ERR_INVALID_ARGUMENT  # overlaps q
