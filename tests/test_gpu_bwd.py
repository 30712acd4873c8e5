"""GPU parity of the backward (dn_chunk_bwd, through the C ABI: the chunked kernels for d in {64, 128},
the sequential small-state kernel for d in {8, 16}, both read-outs) against the fp64 oracle's reverse
mode (oracle.bwd), element by element over every gradient.

Tolerances (rel-L2 over the whole tensor): the kernels compute in fp32 throughout (their dense
products are TF32 tensor-core products with a hi/lo split, about fp32 accuracy), and the same
chunk algebra run in fp32 NumPy lands near 5e-7 of the fp64 result. So every fp32 output (gate
gradients, dS0, and dq/dk/dv for fp32 inputs) must be within 1e-4. bf16 dq/dk/dv are rounded to
bf16 on output, whose relative rounding error is up to 2^-9 per element (about 1.5e-3 rel-L2);
they must be within 1e-2.
"""
import numpy as np
import pytest
import torch

import dn_inputs as di
import gated_linear_attention_dn_b200 as dn
import oracle
from tests.gpu_util import dev, host_f64, sampled_heads, to_device

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-4
TOL_IO = {"f32": 1e-4, "bf16": 1e-2}
NAMES = ("q", "k", "v", "alpha", "beta_k", "beta_v", "key_scale", "S0")


def _run(x, g, readout="post"):
    xd = to_device(x)
    gd = to_device(g)
    out = dn.dn_chunk_bwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                          xd["S0"], dO=gd["dO"], dS_T=gd["dS_T"], readout=readout)
    assert dn.dn_stream_status() == dn.DN_OK
    return out


def _compare(out, ref, io, heads=None):
    worst = {}
    for name in NAMES:
        if ref[name] is None:
            assert out[name] is None, name
            continue
        got = host_f64(out[name])
        if heads is not None:
            if name == "S0":
                got = np.stack([got[b, h] for (b, h) in heads])
            else:
                got = np.stack([got[b, :, h] for (b, h) in heads])
        tol = TOL_IO[io] if name in ("q", "k", "v") else TOL_F32
        e = oracle.rel_l2(got, ref[name])
        worst[name] = e
        assert np.isfinite(got).all(), name
        assert e <= tol, f"{name}: rel-L2 {e:.3e} > {tol}"
    print("[parity] bwd rel-L2 " + " ".join(f"{n} {e:.1e}" for n, e in worst.items()))


@pytest.mark.parametrize("name,kw", [
    ("gdn_fp32_small", {}),                              # fp32, d 64, 4 chunks
    ("gdn_prefill", dict(B=1, H=2, T=200)),              # bf16 scalar gates, ragged tail (200 = 3 x 64 + 8)
    ("kda", dict(B=1, H=2, T=130)),                      # channel decay, S0
    ("fg2_osdn_long", dict(B=1, H=2, T=150)),            # channel beta^k, beta^v, key scale, S0
    ("fg2_osdn_long", dict(B=1, H=1, T=37)),             # one partial chunk
    ("fg2_osdn_long", dict(B=2, H=1, T=1)),              # one token
    ("kda", dict(B=1, H=2, T=100, dv=64)),               # d_k 128, d_v 64
    ("gdn_prefill", dict(B=1, H=3, T=70, dk=64)),        # d_k 64, d_v 128
])
def test_bwd_matches_oracle(name, kw):
    w = di.WORKLOADS[name].scaled(**kw)
    x = di.make_inputs(w)
    g = di.make_bwd_inputs(w)
    out = _run(x, g)
    ref = oracle.bwd(**x, dO=g["dO"], dS_T=g["dS_T"])
    _compare(out, ref, w.io)


@pytest.mark.parametrize("name,kw", [
    ("gdn_prefill", dict(B=1, H=2, T=200)),              # bf16 scalar gates, ragged tail
    ("kda", dict(B=1, H=2, T=130)),                      # channel decay, S0
    ("fg2_osdn_long", dict(B=1, H=2, T=150)),            # every gate per channel
    ("gdn_fp32_small", dict(dv=128)),                    # fp32, d_k 64, d_v 128
])
def test_bwd_pre_readout_matches_oracle(name, kw):
    """o_t = S_{t-1}^T q_t (the delta-mem page's read): the same four kernels with Q+ / alpha and a strict P."""
    w = di.WORKLOADS[name].scaled(**kw)
    x = di.make_inputs(w)
    g = di.make_bwd_inputs(w)
    out = _run(x, g, readout="pre")
    ref = oracle.bwd(**x, dO=g["dO"], dS_T=g["dS_T"], readout="pre")
    _compare(out, ref, w.io)


@pytest.mark.parametrize("readout", ["post", "pre"])
@pytest.mark.parametrize("name,kw", [
    ("gdn_fp32_small", dict(B=2, H=3, T=300, dk=8, dv=8)),         # the delta-mem page's 8 x 8 memory
    ("fg2_osdn_long", dict(B=1, H=2, T=130, dk=16, dv=8)),        # every gate per channel, bf16
    ("kda", dict(B=1, H=5, T=77, dk=16, dv=16)),                  # channel decay, S0
])
def test_bwd_small_states_match_oracle(name, kw, readout):
    w = di.WORKLOADS[name].scaled(**kw)
    x = di.make_inputs(w)
    g = di.make_bwd_inputs(w)
    out = _run(x, g, readout=readout)
    ref = oracle.bwd(**x, dO=g["dO"], dS_T=g["dS_T"], readout=readout)
    _compare(out, ref, w.io)


def test_bwd_per_token_gates_everywhere():
    """Every gate one value per token (beta^v and the key scale included), fp32, S0 given."""
    w = di.WORKLOADS["gdn_fp32_small"].scaled(B=2, H=2, T=150)
    x = di.make_inputs(w)
    shp = (w.B, w.T, w.H)
    x["beta_v"] = di.fill(shp, w.seed("beta_v"), di.GEN_SIGMOID, dtype="f32")
    x["key_scale"] = di.fill(shp, w.seed("key_scale"), di.GEN_NORMAL, 1.0, 0.1, dtype="f32")
    x["S0"] = di.fill((w.B, w.H, w.dk, w.dv), w.seed("S0"), di.GEN_NORMAL, 0.0, 0.05, dtype="f32")
    g = di.make_bwd_inputs(w)
    out = _run(x, g)
    ref = oracle.bwd(**x, dO=g["dO"], dS_T=g["dS_T"])
    _compare(out, ref, w.io)


def test_bwd_without_final_state_adjoint_or_dS0():
    w = di.WORKLOADS["kda"].scaled(B=1, H=2, T=96)
    x = di.make_inputs(w)
    g = di.make_bwd_inputs(w)
    xd = to_device(x)
    out = dn.dn_chunk_bwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                          xd["S0"], dO=dev(g["dO"]), dS_T=None, want_dS0=False)
    assert dn.dn_stream_status() == dn.DN_OK
    assert out["S0"] is None
    ref = oracle.bwd(**x, dO=g["dO"], dS_T=None)
    ref["S0"] = None
    _compare(out, ref, w.io)


def test_bwd_no_tokens_passes_the_state_adjoint_through():
    w = di.WORKLOADS["gdn_prefill"].scaled(B=1, H=2, T=0)
    x = di.make_inputs(w)
    g = di.make_bwd_inputs(w)
    out = _run(x, g)
    np.testing.assert_array_equal(host_f64(out["S0"]), g["dS_T"].astype(np.float64))


def test_bwd_full_size_sampled_heads():
    """The configuration the benchmark times (B=8, H=16, T=4096, d=128, bf16, scalar gates): every
    gradient of a sample of heads (first and last included) against the oracle."""
    w = di.WORKLOADS["gdn_prefill"]
    x = di.make_inputs(w)
    g = di.make_bwd_inputs(w)
    out = _run(x, g)
    heads = sampled_heads(w, 3, seed=11)
    ref = oracle.bwd(**x, dO=g["dO"], dS_T=g["dS_T"], heads=heads)
    _compare(out, ref, w.io, heads=heads)
    torch.cuda.empty_cache()
