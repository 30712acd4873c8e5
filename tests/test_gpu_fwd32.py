"""The chunked forward in fp32 (fp32 io, and bf16 with d_k = 64), through the C ABI: with a workspace
(the binding's default) dn_chunk_fwd evaluates the chunk form on the backward's chunk kernels (every
chunk's K+, Q+, W-, T and P; the state chain; O = Q+ S_m + P U), without one the sequential kernel.
Both are compared with the fp64 oracle on ragged lengths, both read-outs, every d_k, d_v in
{64, 128}, every gate, and decay strong enough that chunks leave the factorisation's range and are
evaluated token by token inside the chain (exact zeros included)."""
import numpy as np
import pytest

import dn_inputs as di
import gated_linear_attention_dn_b200 as dn
import oracle
from tests.gpu_util import TOL, check, host_f64, sampled_heads, to_device

pytestmark = pytest.mark.gpu


def _both(w, x, readout="post"):
    xd = to_device(x)
    args = (xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"], xd["S0"])
    desc = dn.make_desc(xd["q"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"])
    assert dn.dn_chunk_fwd_workspace_bytes(desc) > 0  # this problem has the chunked fp32 path
    o_c, S_c = dn.dn_chunk_fwd(*args, readout=readout)                   # chunked (workspace allocated)
    o_s, S_s = dn.dn_chunk_fwd(*args, readout=readout, workspace=False)  # sequential
    assert dn.dn_stream_status() == dn.DN_OK
    o_ref, S_ref = oracle.fwd(**x, readout=readout)
    check(o_c, S_c, o_ref, S_ref, w.io)
    check(o_s, S_s, o_ref, S_ref, w.io)
    assert oracle.rel_l2(host_f64(o_c), host_f64(o_s)) < TOL[w.io]["o"]
    assert oracle.rel_l2(host_f64(S_c), host_f64(S_s)) < TOL[w.io]["S"]


@pytest.mark.parametrize("T", [1, 63, 64, 65, 256, 1000])
def test_fp32_config_ragged(T):
    w = di.WORKLOADS["gdn_fp32_small"].scaled(T=T)
    _both(w, di.make_inputs(w))


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("readout", ["post", "pre"])
def test_fp32_every_gate_and_size(dk, dv, readout):
    w = di.WORKLOADS["fg2_osdn_long"].scaled(B=1, H=2, T=200, dk=dk, dv=dv, io="f32")
    _both(w, di.make_inputs(w), readout)


@pytest.mark.parametrize("name", ["gdn_prefill", "kda"])
def test_bf16_dk64(name):
    w = di.WORKLOADS[name].scaled(B=2, H=2, T=300, dk=64, dv=128)
    _both(w, di.make_inputs(w))


@pytest.mark.parametrize("kind", [(di.GEN_UNIFORM, 0.01, 0.3), (di.GEN_UNIFORM, 1e-8, 1e-3)], ids=["strong", "extreme"])
@pytest.mark.parametrize("name", ["gdn_fp32_small", "kda"])
@pytest.mark.parametrize("readout", ["post", "pre"])
def test_strong_decay_exact_chunks(kind, name, readout):
    io = "f32" if name == "gdn_fp32_small" else "bf16"
    w = di.WORKLOADS[name].scaled(B=1, H=2, T=200, dk=64, dv=64, io=io, alpha_kind=kind, s0_std=0.5)
    _both(w, di.make_inputs(w), readout)


def test_zero_gates_reset():
    w = di.WORKLOADS["gdn_fp32_small"].scaled(T=200, s0_std=0.5)
    x = di.make_inputs(w)
    al = x["alpha"].copy()
    al[:, 70] = 0.0   # a full reset inside the second chunk
    al[:, 140:150] = 0.0
    x["alpha"] = al
    _both(w, x)


def test_resume_in_place():
    """S_T written over S0 (the caller resumes a sequence): two halves equal the whole."""
    w = di.WORKLOADS["gdn_fp32_small"].scaled(T=300, s0_std=0.5)
    x = di.make_inputs(w)
    xd = to_device(x)
    o_ref, S_ref = oracle.fwd(**x)
    S = xd["S0"].clone()
    o_parts = []
    for lo, hi in ((0, 130), (130, 300)):
        sl = lambda t: None if t is None else t[:, lo:hi].contiguous()
        o, _ = dn.dn_chunk_fwd(sl(xd["q"]), sl(xd["k"]), sl(xd["v"]), sl(xd["alpha"]), sl(xd["beta_k"]),
                               sl(xd["beta_v"]), sl(xd["key_scale"]), S, S_T=S)
        o_parts.append(o)
    assert dn.dn_stream_status() == dn.DN_OK
    import torch
    check(torch.cat(o_parts, dim=1), S, o_ref, S_ref, w.io)


def _chunked(w, x, C, readout="post"):
    """dn_chunk_fwd with chunk = C against the oracle, and against the default chunk length (64): the
    chunk length changes only the rounding."""
    xd = to_device(x)
    args = (xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"], xd["S0"])
    desc = dn.make_desc(xd["q"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"], chunk=C)
    assert dn.dn_chunk_fwd_workspace_bytes(desc) > 0  # the chunk form in fp32 with chunks of C tokens
    o_c, S_c = dn.dn_chunk_fwd(*args, readout=readout, chunk=C)
    o_d, S_d = dn.dn_chunk_fwd(*args, readout=readout)
    assert dn.dn_stream_status() == dn.DN_OK
    o_ref, S_ref = oracle.fwd(**x, readout=readout)
    check(o_c, S_c, o_ref, S_ref, w.io)
    assert oracle.rel_l2(host_f64(o_c), host_f64(o_d)) < 2 * TOL[w.io]["o"]
    assert oracle.rel_l2(host_f64(S_c), host_f64(S_d)) < 2 * TOL[w.io]["S"]


@pytest.mark.parametrize("C", [16, 32])
@pytest.mark.parametrize("T", [1, 15, 16, 17, 33, 100, 1000])
def test_chunk_length_ragged(C, T):
    w = di.WORKLOADS["gdn_fp32_small"].scaled(T=T, s0_std=0.5)
    _chunked(w, di.make_inputs(w), C)


@pytest.mark.parametrize("C", [16, 32])
@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
@pytest.mark.parametrize("name", ["gdn_prefill", "kda", "fg2_osdn_long"])
def test_chunk_length_every_size_and_gate(C, dk, dv, name):
    """bf16 io (d_k = 128 too, which takes the tensor-core kernels at 64) and every gate mode."""
    w = di.WORKLOADS[name].scaled(B=1, H=2, T=200, dk=dk, dv=dv)
    _chunked(w, di.make_inputs(w), C)


@pytest.mark.parametrize("C", [16, 32])
@pytest.mark.parametrize("readout", ["post", "pre"])
def test_chunk_length_readouts_fp32(C, readout):
    w = di.WORKLOADS["fg2_osdn_long"].scaled(B=1, H=2, T=150, dk=128, dv=64, io="f32")
    _chunked(w, di.make_inputs(w), C, readout)


@pytest.mark.parametrize("C", [16, 32])
@pytest.mark.parametrize("kind", [(di.GEN_UNIFORM, 0.01, 0.3), (di.GEN_UNIFORM, 1e-8, 1e-3)], ids=["strong", "extreme"])
def test_chunk_length_strong_decay(C, kind):
    """Decay strong enough that some chunks leave the factorisation's range (evaluated token by token)."""
    w = di.WORKLOADS["kda"].scaled(B=1, H=2, T=200, dk=64, dv=64, alpha_kind=kind, s0_std=0.5)
    _chunked(w, di.make_inputs(w), C, "pre")


def test_chunk_length_full_size_sampled():
    """The gdn_prefill workload at its full size (B=8, H=16, T=4096, d=128) with 32-token chunks, on
    sampled heads, each over its whole sequence."""
    import torch
    w = di.WORKLOADS["gdn_prefill"]
    x = di.make_inputs(w)
    xd = to_device(x)
    o, ST = dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                            xd["S0"], chunk=32)
    assert dn.dn_stream_status() == dn.DN_OK
    heads = sampled_heads(w, 4, seed=3)
    o_ref, S_ref = oracle.fwd(**x, heads=heads)
    og = torch.stack([o[b, :, h] for (b, h) in heads])
    Sg = torch.stack([ST[b, h] for (b, h) in heads])
    check(og, Sg, o_ref, S_ref, w.io)
