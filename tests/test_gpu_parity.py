"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small cases run every head through the oracle and span several chunks plus a
ragged tail; the full-size workloads (the sizes bench.py times) compare a
sample of heads, each over its whole sequence. Tolerances (relative L2 over the
compared tensor): fp32 io 1e-4 on o and S_T; bf16 io 2e-2 on o, 1e-3 on S_T.
"""
import numpy as np
import pytest
import torch

import dn_inputs as di
import gated_linear_attention_dn_b200 as dn
import oracle
from tests.gpu_util import TOL, check, host_f64, run_chunk, sampled_heads, to_device

pytestmark = pytest.mark.gpu


def _small(name, **sizes):
    w = di.WORKLOADS[name].scaled(**sizes)
    x = di.make_inputs(w)
    o_ref, S_ref = oracle.fwd(**x)
    o, ST = run_chunk(to_device(x))
    return check(o, ST, o_ref, S_ref, w.io)


def test_gdn_fp32_small_full_config():
    _small("gdn_fp32_small")


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 130, 1000])
def test_gdn_prefill_ragged(T):
    _small("gdn_prefill", B=1, H=2, T=T)


@pytest.mark.parametrize("T", [1, 65, 300])
def test_kda_small(T):
    _small("kda", B=1, H=2, T=T)


@pytest.mark.parametrize("T", [1, 65, 300])
def test_fg2_osdn_small(T):
    _small("fg2_osdn_long", B=1, H=2, T=T)


@pytest.mark.parametrize("dk,dv", [(64, 128), (128, 64), (64, 64)])
@pytest.mark.parametrize("name", ["gdn_prefill", "fg2_osdn_long"])
def test_head_dims(name, dk, dv):
    _small(name, B=2, H=3, T=130, dk=dk, dv=dv)


@pytest.mark.parametrize("name", ["gdn_fp32_small", "gdn_prefill"])
def test_zero_length_copies_state(name):
    w = di.WORKLOADS[name].scaled(B=1, H=2, T=0, s0_std=0.02)
    x = di.make_inputs(w)
    xd = to_device(x)
    o, ST = run_chunk(xd)
    torch.testing.assert_close(ST, xd["S0"], rtol=0, atol=0)


def test_resume_in_place():
    """fwd(T1) then fwd(T2, S0 = S_T1, S_T aliasing S0) equals fwd(T1 + T2)."""
    w = di.WORKLOADS["kda"].scaled(B=1, H=2, T=200)
    x = di.make_inputs(w)
    o_ref, S_ref = oracle.fwd(**x)
    xd = to_device(x)
    cut = 77
    part = lambda a, s: None if a is None else a[:, s].contiguous()
    S = xd["S0"].clone()
    os_ = []
    for s in (slice(0, cut), slice(cut, None)):
        o, _ = dn.dn_chunk_fwd(part(xd["q"], s), part(xd["k"], s), part(xd["v"], s), part(xd["alpha"], s),
                               part(xd["beta_k"], s), part(xd["beta_v"], s), part(xd["key_scale"], s),
                               S0=S, S_T=S)
        os_.append(o)
    assert dn.dn_stream_status() == dn.DN_OK
    check(torch.cat(os_, dim=1), S, o_ref, S_ref, "bf16")


def test_gated_newton_condition_full_size():
    """OSDN page, theorem 5.2 condition: with <beta^k (.) d, k^2> = 1 and q = k, o_t = beta^v (.) v_t
    for any state, at the full long-context size."""
    w = di.WORKLOADS["fg2_osdn_long"]
    x = di.make_inputs(w.scaled(T=4096))
    xd = to_device(x)
    k32 = xd["k"].float()
    # scalar beta^k chosen per token so that beta^k <d, k^2> = 1
    bk = 1.0 / (xd["key_scale"] * k32 * k32).sum(-1)
    o, _ = dn.dn_chunk_fwd(xd["k"], xd["k"], xd["v"], xd["alpha"], bk.contiguous(), xd["beta_v"],
                           xd["key_scale"], xd["S0"])
    assert dn.dn_stream_status() == dn.DN_OK
    expect = (xd["beta_v"] * xd["v"].float()).double()
    err = (o.double() - expect).norm() / expect.norm()
    assert err.item() < TOL["bf16"]["o"]


@pytest.mark.parametrize("name,nheads", [("gdn_prefill", 6), ("kda", 4), ("fg2_osdn_long", 2)])
def test_full_size_sampled_heads(name, nheads):
    w = di.WORKLOADS[name]
    x = di.make_inputs(w)
    xd = to_device(x)
    o, ST = run_chunk(xd)
    heads = sampled_heads(w, nheads, seed=1)
    o_ref, S_ref = oracle.fwd(**x, heads=heads)
    og = torch.stack([o[b, :, h] for (b, h) in heads])
    Sg = torch.stack([ST[b, h] for (b, h) in heads])
    check(og, Sg, o_ref, S_ref, w.io)
    assert torch.isfinite(o.float()).all() and torch.isfinite(ST).all()


# ------------------------------------------------------------------- decode

def _decode_inputs(w, step):
    x = di.make_inputs(w, step=step)
    return x


def test_decode_one_step_equals_chunk_T1():
    """A decode step equals the chunked forward at T = 1 (both on the GPU)."""
    w = di.WORKLOADS["decode"].scaled(B=8)
    x = di.make_inputs(w, step=0)
    xd = to_device(x)
    S = xd["S0"].clone()
    o_dec = dn.dn_decode_step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"],
                              xd["key_scale"], S=S)
    o_chk, S_chk = run_chunk(xd)
    # the decode step is fp32 on CUDA cores; the chunked kernel uses bf16 tensor-core operands,
    # so the two agree to the bf16 tolerances, and each matches the oracle on its own
    assert oracle.rel_l2(host_f64(o_dec), host_f64(o_chk)) < TOL["bf16"]["o"]
    assert oracle.rel_l2(host_f64(S), host_f64(S_chk)) < TOL["bf16"]["S"]
    o_ref, S_ref = oracle.fwd(**x)
    check(o_dec, S, o_ref, S_ref, "bf16")
    check(o_chk, S_chk, o_ref, S_ref, "bf16")


@pytest.mark.parametrize("B,steps", [(4, 100), (1024, 3)])
def test_decode_steps_vs_oracle(B, steps):
    """100 in-place decode steps against the oracle chained over the same per-step inputs."""
    w = di.WORKLOADS["decode"].scaled(B=B)
    heads = sampled_heads(w, 8, seed=2) if B > 8 else None
    S = None
    S_ref = None
    errs = []
    for step in range(steps):
        x = di.make_inputs(w, step=step)
        xd = to_device(x)
        if step == 0:
            S = xd["S0"].clone()
            if heads is None:
                S_ref = oracle.widen(x["S0"])
            else:
                S_ref = np.stack([oracle.widen(x["S0"][b, h]) for (b, h) in heads])[:, None]
        o = dn.dn_decode_step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"],
                              xd["key_scale"], S=S)
        if heads is None:
            o_ref, S_ref = oracle.fwd(**dict(x, S0=S_ref))
            errs.append(oracle.rel_l2(host_f64(o), o_ref))
        else:
            sub = {n: (None if a is None else np.stack([a[b:b + 1, :, h:h + 1] for (b, h) in heads])[:, 0])
                   for n, a in x.items() if n != "S0"}
            # sub arrays: [NH, 1, 1, d] -> treat each sampled head as its own batch entry
            o_ref, S_new = oracle.fwd(**sub, S0=S_ref)
            S_ref = S_new
            og = torch.stack([o[b, :, h] for (b, h) in heads])
            errs.append(oracle.rel_l2(host_f64(og), o_ref[:, :, 0]))
    assert dn.dn_stream_status() == dn.DN_OK
    assert max(errs) < TOL["bf16"]["o"]
    if heads is None:
        assert oracle.rel_l2(host_f64(S), S_ref) < TOL["bf16"]["S"]
    else:
        Sg = torch.stack([S[b, h] for (b, h) in heads])
        assert oracle.rel_l2(host_f64(Sg), S_ref[:, 0]) < TOL["bf16"]["S"]


def test_decode_fp32_io():
    w = di.WORKLOADS["decode"].scaled(B=3, io="f32")
    x = di.make_inputs(w)
    xd = to_device(x)
    S = xd["S0"].clone()
    o = dn.dn_decode_step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"],
                          xd["key_scale"], S=S)
    o_ref, S_ref = oracle.fwd(**x)
    check(o, S, o_ref, S_ref, "f32")
