"""The allocation-free OSDN scan (dn_osdn_precond_noalloc), called through the C ABI.

This entry point is for callers that cannot allocate device memory when they run the
scan (their allocator owns the whole GPU, or their framework forbids allocations inside
compute callbacks): it takes its scratch from a fixed buffer inside the library instead
of a caller workspace. It runs the same kernels on the same inputs as dn_osdn_precond
and keeps nothing between calls, so its results must equal those of dn_osdn_precond bit
for bit, including on a second call that finds the first call's data in the buffer (any
leftover read would show as a difference).

The file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import dn_inputs as di
import gated_linear_attention_dn_b200 as dn


def _lib():
    lib = dn.load()
    O = ctypes.POINTER(dn.DnOsdnDesc)
    P = ctypes.c_void_p
    lib.dn_osdn_precond_noalloc.argtypes = [O, P, P, P, P, P, P, P]
    lib.dn_osdn_precond_noalloc.restype = ctypes.c_int
    return lib


def _inputs(T, H, seed):
    w = di.WORKLOADS["osdn_phase1"].scaled(B=1, T=T, H=H)
    x = di.make_osdn_inputs(w)
    k = torch.from_numpy(x["k"].view(np.int16)).view(torch.bfloat16).cuda()
    beta = torch.from_numpy(x["beta"]).cuda()
    ret = torch.from_numpy(x["retention"]).cuda()
    d0 = torch.from_numpy(np.random.default_rng(seed).uniform(0.5, 1.5, (1, H, 128)).astype(np.float32)).cuda()
    return w, k, beta, ret, d0, x["eta"]


def _noalloc(lib, w, k, beta, ret, d0, eta):
    d = torch.full((w.B, w.T, w.H, w.dk), float("nan"), dtype=torch.float32, device="cuda")
    dT = torch.full((w.B, w.H, w.dk), float("nan"), dtype=torch.float32, device="cuda")
    desc = dn.DnOsdnDesc(w.B, w.T, w.H, w.dk, dn.DN_BF16, eta)
    P = ctypes.c_void_p
    rc = lib.dn_osdn_precond_noalloc(ctypes.byref(desc), P(k.data_ptr()), P(beta.data_ptr()), P(ret.data_ptr()),
                                     P(d0.data_ptr()), P(d.data_ptr()), P(dT.data_ptr()),
                                     P(torch.cuda.current_stream().cuda_stream))
    assert rc == dn.DN_OK, dn.dn_status_string(rc)
    assert dn.dn_stream_status() == dn.DN_OK
    return d, dT


def _rel(x, ref):
    return float(torch.linalg.vector_norm((x - ref).double()) / torch.linalg.vector_norm(ref.double()))


@pytest.mark.gpu
def test_noalloc_matches_the_workspace_entry_point_twice_in_a_row():
    lib = _lib()
    # two different problems back to back: the second finds the first one's data in the buffer
    for T, H, seed in ((1000, 4, 1), (333, 6, 2)):
        w, k, beta, ret, d0, eta = _inputs(T, H, seed)
        d, dT = _noalloc(lib, w, k, beta, ret, d0, eta)
        d_ref, dT_ref = dn.dn_osdn_precond(k, beta, ret, d0, eta=eta)
        torch.cuda.synchronize()
        assert torch.isfinite(d).all() and torch.isfinite(dT).all()
        e, eT = _rel(d, d_ref), _rel(dT, dT_ref)
        print(f"[no-alloc] T={T} H={H}: d rel-L2 {e:.3e}, d_T rel-L2 {eT:.3e} (must be identical)")
        assert torch.equal(d, d_ref) and torch.equal(dT, dT_ref)


def test_noalloc_rejects_problems_beyond_its_buffer():
    lib = _lib()
    # 32 MiB hold 7,943 blocks of 32 tokens: one head of 7,944 blocks is one too many
    desc = dn.DnOsdnDesc(1, 7944 * 32, 1, 128, dn.DN_BF16, 0.5)
    P = ctypes.c_void_p
    big = P(1 << 20)
    rc = lib.dn_osdn_precond_noalloc(ctypes.byref(desc), big, big, None, None, big, None, None)
    assert rc == dn.DN_ERR_WORKSPACE_TOO_SMALL
    assert lib.dn_osdn_precond_noalloc(None, big, big, None, None, big, None, None) == dn.DN_ERR_INVALID_ARGUMENT
