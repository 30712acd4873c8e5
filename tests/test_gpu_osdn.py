"""GPU parity of OSDN phase 1 (dn_osdn_precond) against the fp64 oracle, through the C ABI.

The scan runs in fp32 on the GPU; d is compared with the oracle's fp64 sequence element by
element (rel-L2 over the whole tensor, tolerance TOL_D), at sizes that cross the 32-token
blocks with ragged tails, at the full osdn_phase1 size on sampled heads, and end to end: the
GPU's d fed to the chunked prefill as the OSDN key scale against the oracle doing the same.
"""
import numpy as np
import pytest
import torch

import dn_inputs as di
import gated_linear_attention_dn_b200 as dn
import oracle
from tests.gpu_util import check, dev, host_f64, sampled_heads

pytestmark = pytest.mark.gpu

TOL_D = 1e-4  # fp32 scan against fp64: rounding of ~T fp32 steps, contracted by the update


def _case(T, H=2, dk=128, B=1, io="bf16", retention=True, d0=False, seed=0):
    w = di.WORKLOADS["osdn_phase1"].scaled(B=B, T=T, H=H, dk=dk, io=io)
    x = di.make_osdn_inputs(w)
    if not retention:
        x["retention"] = None
    x["d0"] = None
    if d0:
        x["d0"] = np.random.default_rng(seed).uniform(0.5, 1.5, (B, H, dk)).astype(np.float32)
    return w, x


def _run(x):
    d, dT = dn.dn_osdn_precond(dev(x["k"]), dev(x["beta"]), dev(x["retention"]), dev(x["d0"]), eta=x["eta"])
    assert dn.dn_stream_status() == dn.DN_OK
    return d, dT


def _check_d(d, dT, x, heads=None):
    ref, refT = oracle.osdn_precond(x["k"], x["beta"], x["retention"], x["d0"], eta=x["eta"], heads=heads)
    got, gotT = host_f64(d), host_f64(dT)
    if heads is not None:
        got = np.stack([got[b, :, h] for (b, h) in heads])
        gotT = np.stack([gotT[b, h] for (b, h) in heads])
    e, eT = oracle.rel_l2(got, ref), oracle.rel_l2(gotT, refT)
    # the part that learning changed, measured against its own size (d starts at 1 or d0)
    base = np.ones_like(ref) if x["d0"] is None else None
    print(f"[parity] d rel-L2 {e:.3e}, d_T rel-L2 {eT:.3e} (tol {TOL_D:.0e})")
    assert e <= TOL_D and eT <= TOL_D
    if base is not None and ref.shape[1] > 64:
        moved = oracle.rel_l2(ref, base)
        assert moved > 1e-3, "the scan must actually move d away from its start on this workload"
    return e


@pytest.mark.parametrize("T", [1, 31, 32, 33, 100, 1000])
def test_osdn_small_ragged(T):
    w, x = _case(T)
    _check_d(*_run(x), x)


@pytest.mark.parametrize("dk,io,retention,d0", [(64, "bf16", True, False), (128, "f32", False, True),
                                                (64, "f32", True, True), (128, "bf16", False, False)])
def test_osdn_variants(dk, io, retention, d0):
    w, x = _case(300, H=3, dk=dk, io=io, retention=retention, d0=d0, seed=dk)
    _check_d(*_run(x), x)


def test_osdn_empty_sequence():
    w, x = _case(0, H=2, d0=True)
    d, dT = _run(x)
    np.testing.assert_array_equal(host_f64(dT), x["d0"].astype(np.float64))
    w, x = _case(0, H=2, d0=False)
    d, dT = _run(x)
    np.testing.assert_array_equal(host_f64(dT), np.ones((1, 2, 128)))


def test_osdn_resume():
    w, x = _case(200, H=2)
    d_all, dT_all = _run(x)
    x1 = {n: (v[:, :77] if isinstance(v, np.ndarray) else v) for n, v in x.items()}
    d1, dT1 = _run(x1)
    x2 = {n: (v[:, 77:] if isinstance(v, np.ndarray) else v) for n, v in x.items()}
    d2, dT2 = dn.dn_osdn_precond(dev(x2["k"]), dev(x2["beta"]), dev(x2["retention"]), dT1, eta=x["eta"])
    torch.testing.assert_close(torch.cat([d1, d2], dim=1), d_all, rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(dT2, dT_all, rtol=1e-5, atol=1e-6)


def test_osdn_full_size_sampled_heads():
    w = di.WORKLOADS["osdn_phase1"]
    x = di.make_osdn_inputs(w)
    x["d0"] = None
    d, dT = _run(x)
    _check_d(d, dT, x, heads=sampled_heads(w, 3, seed=11))


def test_osdn_feeds_the_chunked_prefill():
    """Phase 1 then phase 2 on the GPU against the oracle doing both (OSDN page, section 2.2)."""
    wf = di.WORKLOADS["fg2_osdn_long"].scaled(T=1000, H=2)
    xf = di.make_inputs(wf)
    w1 = di.WORKLOADS["osdn_phase1"].scaled(T=1000, H=2)
    x1 = di.make_osdn_inputs(w1)
    assert np.array_equal(x1["k"], xf["k"])
    x1["d0"] = None
    d, _ = _run(x1)
    dref, _ = oracle.osdn_precond(x1["k"], x1["beta"], x1["retention"], None, eta=x1["eta"])
    xd = {n: dev(v) for n, v in xf.items()}
    o, ST = dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], d, xd["S0"])
    assert dn.dn_stream_status() == dn.DN_OK
    o_ref, S_ref = oracle.fwd(xf["q"], xf["k"], xf["v"], xf["alpha"], xf["beta_k"], xf["beta_v"], dref, xf["S0"])
    check(o, ST, o_ref, S_ref, "bf16")
