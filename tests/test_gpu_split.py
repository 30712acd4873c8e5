"""The two evaluations of the per-token-gate chunked prefill, through the C ABI: the split one (a
chunk-parallel transform kernel writing each chunk's UT-transform tiles and factors to the caller's
workspace, then the state-chain kernel) and the fused one (no workspace: one kernel per head). Each is
compared with the fp64 oracle, and the two with each other, on ragged lengths, both read-outs,
strong decay and every per-token gate; the workspace's neighbours stay untouched; a bounded wait
made to run out in either kernel of the split path reports DN_ERR_DEVICE_TIMEOUT."""
import numpy as np
import pytest
import torch

import dn_inputs as di
import gated_linear_attention_dn_b200 as dn
import oracle
from tests.gpu_util import TOL, check, host_f64, to_device

pytestmark = pytest.mark.gpu


def _both(w, x, readout="post"):
    xd = to_device(x)
    args = (xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"], xd["S0"])
    o_s, S_s = dn.dn_chunk_fwd(*args, readout=readout)                   # split (workspace allocated)
    o_f, S_f = dn.dn_chunk_fwd(*args, readout=readout, workspace=False)  # fused
    assert dn.dn_stream_status() == dn.DN_OK
    o_ref, S_ref = oracle.fwd(**x, readout=readout)
    check(o_s, S_s, o_ref, S_ref, w.io)
    check(o_f, S_f, o_ref, S_ref, w.io)
    # the two evaluations round differently but must agree to the same bounds
    assert oracle.rel_l2(host_f64(o_s), host_f64(o_f)) < TOL[w.io]["o"]
    assert oracle.rel_l2(host_f64(S_s), host_f64(S_f)) < TOL[w.io]["S"]


def test_workspace_size_is_positive_for_per_token_gates():
    w = di.WORKLOADS["gdn_prefill"]
    xd = to_device(di.make_inputs(w.scaled(B=1, T=70)))
    desc = dn.make_desc(xd["q"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"])
    assert dn.dn_chunk_fwd_workspace_bytes(desc) == 1 * 16 * 2 * 25616


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 130, 1000])
def test_split_and_fused_ragged(T):
    w = di.WORKLOADS["gdn_prefill"].scaled(B=1, H=2, T=T)
    _both(w, di.make_inputs(w))


@pytest.mark.parametrize("B,H", [(1, 3), (40, 2)])  # value columns split over two CTAs, and not
@pytest.mark.parametrize("readout", ["post", "pre"])
def test_split_and_fused_every_gate(B, H, readout):
    w = di.WORKLOADS["gdn_prefill"].scaled(B=B, H=H, T=257, s0_std=0.5, beta_v=di.GATE_SCALAR,
                                           key_scale=di.GATE_SCALAR)
    _both(w, di.make_inputs(w), readout)


@pytest.mark.parametrize("kind", [(di.GEN_UNIFORM, 0.01, 0.3), (di.GEN_UNIFORM, 1e-8, 1e-3)], ids=["strong", "extreme"])
@pytest.mark.parametrize("readout", ["post", "pre"])
def test_split_and_fused_strong_decay(kind, readout):
    w = di.WORKLOADS["gdn_prefill"].scaled(B=40, H=2, T=300, alpha_kind=kind, s0_std=0.5)
    _both(w, di.make_inputs(w), readout)


def test_split_full_size_sampled_heads_against_fused():
    """The bench's configuration: every head of the split path against the fused path, and sampled
    heads against the oracle."""
    w = di.WORKLOADS["gdn_prefill"]
    x = di.make_inputs(w)
    xd = to_device(x)
    args = (xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"], xd["S0"])
    o_s, S_s = dn.dn_chunk_fwd(*args)
    o_f, S_f = dn.dn_chunk_fwd(*args, workspace=False)
    assert dn.dn_stream_status() == dn.DN_OK
    assert oracle.rel_l2(host_f64(o_s), host_f64(o_f)) < TOL["bf16"]["o"]
    assert oracle.rel_l2(host_f64(S_s), host_f64(S_f)) < TOL["bf16"]["S"]
    heads = [(0, 0), (3, 7), (7, 15)]
    o_ref, S_ref = oracle.fwd(**x, heads=heads)
    check(torch.stack([o_s[b, :, h] for b, h in heads]), torch.stack([S_s[b, h] for b, h in heads]), o_ref, S_ref,
          "bf16")


def test_workspace_neighbours_untouched():
    w = di.WORKLOADS["gdn_prefill"].scaled(B=2, H=3, T=200, beta_v=di.GATE_SCALAR)
    x = di.make_inputs(w)
    xd = to_device(x)
    desc = dn.make_desc(xd["q"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"])
    n = dn.dn_chunk_fwd_workspace_bytes(desc)
    pad = 4096
    buf = torch.full((n + 2 * pad,), 0xA5, dtype=torch.uint8, device="cuda")
    o, ST = dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                            xd["S0"], workspace=buf[pad:pad + n])
    assert dn.dn_stream_status() == dn.DN_OK
    assert bool((buf[:pad] == 0xA5).all()) and bool((buf[pad + n:] == 0xA5).all())
    o_ref, S_ref = oracle.fwd(**x)
    check(o, ST, o_ref, S_ref, "bf16")


def test_split_wait_timeout_reports_status_and_recovers():
    w = di.WORKLOADS["gdn_prefill"].scaled(B=1, H=2, T=300)
    x = di.make_inputs(w)
    xd = to_device(x)
    args = (xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"], xd["S0"])
    dn.dn_set_wait_limit_ns(0)
    try:
        dn.dn_chunk_fwd(*args)
        st = dn.dn_stream_status()
    finally:
        dn.dn_set_wait_limit_ns(dn.DEFAULT_WAIT_NS)
    assert st == dn.DN_ERR_DEVICE_TIMEOUT
    o, ST = dn.dn_chunk_fwd(*args)
    assert dn.dn_stream_status() == dn.DN_OK
    o_ref, S_ref = oracle.fwd(**x)
    check(o, ST, o_ref, S_ref, "bf16")
