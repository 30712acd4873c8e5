"""GPU parity on the method's edge cases, through the C ABI, against the fp64 oracle or a closed form.

* Strong decay: gates far below the configured ones (alpha ~ U(0.01, 0.3), and U(1e-8, 1e-3)),
  per token (the per-token-gate kernel, whose decay products carry their own exponent) and per
  channel (the per-channel-gate kernel, which evaluates such chunks exactly, token by token), both
  read-outs, with the value columns split over two CTAs and not; gates with exact zeros (a full
  reset); chunks that switch between the tensor-core and the exact path inside one sequence.
  Any gate in [0, 1] is a valid forget gate of the recurrence (Sparse Delta Memory page, "Gated
  Delta Updates": decay, then the delta step); none may give a non-finite output.
* beta^k = 0: no write, S_t = Diag(prod alpha) S0 and o_t = S_t^T q_t (closed form).
* 100 decode steps equal one chunked call over the same 100 tokens.
* The decode workload's 100 in-place steps at its full batch (1024 sequences), sampled heads.
* A bounded wait made to run out reports DN_ERR_DEVICE_TIMEOUT and leaves the GPU usable.
* Guard bands: outputs written into the middle of larger buffers leave the neighbours untouched.
* The backward reports DN_ERR_GATE_RANGE for a chunk beyond its fp32 factorisation.
"""
import numpy as np
import pytest
import torch

import dn_inputs as di
import gated_linear_attention_dn_b200 as dn
import oracle
from tests.gpu_util import TOL, check, dev, host_f64, run_chunk, sampled_heads, to_device

pytestmark = pytest.mark.gpu

STRONG = (di.GEN_UNIFORM, 0.01, 0.3)
EXTREME = (di.GEN_UNIFORM, 1e-8, 1e-3)


def _parity(w, x, readout="post"):
    xd = to_device(x)
    o, ST = dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                            xd["S0"], readout=readout)
    assert dn.dn_stream_status() == dn.DN_OK
    o_ref, S_ref = oracle.fwd(**x, readout=readout)
    return check(o, ST, o_ref, S_ref, w.io)


# (B, H): 2 heads split the value columns over two CTAs, 80 heads do not
@pytest.mark.parametrize("B,H", [(1, 2), (40, 2)])
@pytest.mark.parametrize("kind", [STRONG, EXTREME], ids=["strong", "extreme"])
@pytest.mark.parametrize("readout", ["post", "pre"])
def test_strong_decay_per_token_gates(B, H, kind, readout):
    w = di.WORKLOADS["gdn_prefill"].scaled(B=B, H=H, T=300, alpha_kind=kind, s0_std=0.5)
    _parity(w, di.make_inputs(w), readout)


@pytest.mark.parametrize("readout", ["post", "pre"])
def test_strong_decay_per_token_gates_every_gate(readout):
    """beta^v and d given per token too (the T Diag(beta^v) hi/lo split and the scaled write key)."""
    w = di.WORKLOADS["gdn_prefill"].scaled(B=1, H=3, T=257, alpha_kind=STRONG, s0_std=0.5,
                                           beta_v=di.GATE_SCALAR, key_scale=di.GATE_SCALAR)
    _parity(w, di.make_inputs(w), readout)


@pytest.mark.parametrize("name", ["kda", "fg2_osdn_long"])
@pytest.mark.parametrize("B,H", [(1, 2), (40, 2)])
@pytest.mark.parametrize("kind", [STRONG, EXTREME], ids=["strong", "extreme"])
@pytest.mark.parametrize("readout", ["post", "pre"])
def test_strong_decay_per_channel_gates(name, B, H, kind, readout):
    w = di.WORKLOADS[name].scaled(B=B, H=H, T=300, alpha_kind=kind, s0_std=0.5)
    _parity(w, di.make_inputs(w), readout)


@pytest.mark.parametrize("name", ["gdn_prefill", "kda"])
@pytest.mark.parametrize("readout", ["post", "pre"])
def test_zero_gates_reset_the_state(name, readout):
    """alpha = 0 on some tokens (and channels): the state before them is forgotten exactly."""
    w = di.WORKLOADS[name].scaled(B=1, H=2, T=200, s0_std=0.5)
    x = di.make_inputs(w)
    a = x["alpha"].reshape(-1).copy()
    a[::37] = 0.0
    x["alpha"] = a.reshape(x["alpha"].shape)
    _parity(w, x, readout)


@pytest.mark.parametrize("B,H", [(1, 2), (40, 2)])
@pytest.mark.parametrize("readout", ["post", "pre"])
def test_per_channel_chunks_switch_paths(B, H, readout):
    """Mild decay except in chunk 1 (tokens 64..127) and the ragged last chunk, where 8 key channels
    decay strongly: chunks alternate between the tensor-core path and the exact path."""
    w = di.WORKLOADS["kda"].scaled(B=B, H=H, T=290, s0_std=0.5)
    x = di.make_inputs(w)
    a = x["alpha"].copy()
    strong = di.fill(a.shape, 12345, di.GEN_UNIFORM, 0.01, 0.3)
    for t0, t1 in ((64, 128), (256, 290)):
        a[:, t0:t1, :, :8] = strong[:, t0:t1, :, :8]
    x["alpha"] = a
    _parity(w, x, readout)


# ------------------------------------------------------------------- beta^k = 0: pure decay

@pytest.mark.parametrize("name", ["gdn_prefill", "kda"])
def test_no_write_is_pure_decay(name):
    """beta^k = 0 leaves only the decay: S_t = Diag(prod_{s<=t} alpha_s) S0, o_t = S_t^T q_t."""
    w = di.WORKLOADS[name].scaled(B=1, H=2, T=200, s0_std=0.5)
    x = di.make_inputs(w)
    x["beta_k"] = np.zeros_like(x["beta_k"])
    xd = to_device(x)
    o, ST = run_chunk(xd)
    q = oracle.widen(x["q"])
    S0 = x["S0"].astype(np.float64)
    a = x["alpha"].astype(np.float64)
    if a.ndim == 3:
        a = np.repeat(a[..., None], w.dk, axis=-1)
    gam = np.cumprod(a, axis=1)                                   # [B,T,H,dk]
    o_ref = np.einsum("bthk,bthk,bhkv->bthv", q, gam, S0)
    S_ref = gam[:, -1][..., None] * S0
    check(o, ST, o_ref, S_ref, "bf16")


# ------------------------------------------------------------------- decode

def test_hundred_decode_steps_equal_one_chunked_call():
    """100 in-place decode steps and one dn_chunk_fwd over the same 100 tokens give the same outputs and
    final state (each within the bf16 tolerances of the oracle and of each other)."""
    w = di.WORKLOADS["decode"].scaled(B=4)
    steps = [di.make_inputs(w, step=s) for s in range(100)]
    cat = {n: (None if steps[0][n] is None else np.concatenate([s[n] for s in steps], axis=1))
           for n in ("q", "k", "v", "alpha", "beta_k", "beta_v", "key_scale")}
    cat["S0"] = steps[0]["S0"]
    o_ref, S_ref = oracle.fwd(**cat)
    xd = to_device(cat)
    S = xd["S0"].clone()
    outs = []
    for s in steps:
        sd = to_device({n: a for n, a in s.items() if n != "S0"})
        outs.append(dn.dn_decode_step(sd["q"], sd["k"], sd["v"], sd["alpha"], sd["beta_k"], sd["beta_v"],
                                      sd["key_scale"], S=S))
    o_dec = torch.cat(outs, dim=1)
    o_chk, S_chk = run_chunk(xd)
    assert dn.dn_stream_status() == dn.DN_OK
    check(o_dec, S, o_ref, S_ref, "bf16")
    check(o_chk, S_chk, o_ref, S_ref, "bf16")
    assert oracle.rel_l2(host_f64(o_dec), host_f64(o_chk)) < TOL["bf16"]["o"]
    assert oracle.rel_l2(host_f64(S), host_f64(S_chk)) < TOL["bf16"]["S"]


def test_decode_full_batch_hundred_steps():
    """The decode workload as bench.py times it (1024 sequences x 32 heads, 100 in-place steps), against
    the oracle chained over the same per-step inputs on sampled heads; every step's o and the final S."""
    w = di.WORKLOADS["decode"]
    heads = sampled_heads(w, 8, seed=5)
    bi = np.array([b for b, _ in heads])
    hi = np.array([h for _, h in heads])
    S = None
    S_ref = None
    worst = 0.0
    for step in range(w.steps):
        x = di.make_inputs(w, step=step)
        xd = to_device(x)
        if step == 0:
            S = xd["S0"].clone()
            S_ref = x["S0"][bi, hi].astype(np.float64)[:, None]          # [NH,1,dk,dv]
        o = dn.dn_decode_step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                              S=S)
        sub = {n: (None if a is None else a[bi, :, hi][:, :, None]) for n, a in x.items() if n != "S0"}
        o_ref, S_ref = oracle.fwd(**sub, S0=S_ref)                         # each sampled head as a batch entry
        og = host_f64(o)[bi, :, hi]                                        # [NH,1,dv]
        e = max(oracle.rel_l2(og[i], o_ref[i, :, 0]) for i in range(len(heads)))
        worst = max(worst, e)
    assert dn.dn_stream_status() == dn.DN_OK
    print(f"[parity] decode full batch: worst per-head o rel-L2 over 100 steps {worst:.3e}")
    assert worst < TOL["bf16"]["o"]
    Sg = host_f64(S)[bi, hi]
    eS = max(oracle.rel_l2(Sg[i], S_ref[i, 0]) for i in range(len(heads)))
    print(f"[parity] decode full batch: worst per-head S rel-L2 after 100 steps {eS:.3e}")
    assert eS < TOL["bf16"]["S"]


# ------------------------------------------------------------------- failure path

@pytest.mark.parametrize("name", ["gdn_prefill", "kda"])
def test_wait_timeout_reports_status_and_recovers(name):
    """With every mbarrier wait reduced to one non-blocking probe, the first wait (on a TMA load just
    issued) gives up: the kernel drains what it issued, frees its tensor memory and sets the status
    word; the next call with the default bound runs normally and matches the oracle."""
    w = di.WORKLOADS[name].scaled(B=1, H=2, T=200)
    x = di.make_inputs(w)
    xd = to_device(x)
    dn.dn_set_wait_limit_ns(0)
    try:
        dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                        xd["S0"])
        st = dn.dn_stream_status()
    finally:
        dn.dn_set_wait_limit_ns(dn.DEFAULT_WAIT_NS)
    assert st == dn.DN_ERR_DEVICE_TIMEOUT
    assert dn.dn_stream_status() == dn.DN_OK  # reading the status cleared it
    o, ST = run_chunk(xd)
    o_ref, S_ref = oracle.fwd(**x)
    check(o, ST, o_ref, S_ref, w.io)


def test_backward_reports_gate_range():
    """A chunk whose decay is beyond the backward's fp32 factorisation is reported, not returned as if
    valid."""
    w = di.WORKLOADS["kda"].scaled(B=1, H=2, T=130, alpha_kind=EXTREME)
    x = di.make_inputs(w)
    g = di.make_bwd_inputs(w)
    xd, gd = to_device(x), to_device(g)
    dn.dn_chunk_bwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"], xd["S0"],
                    dO=gd["dO"], dS_T=gd["dS_T"])
    assert dn.dn_stream_status() == dn.DN_ERR_GATE_RANGE
    assert dn.dn_stream_status() == dn.DN_OK


# ------------------------------------------------------------------- guard bands

PAD = 4096  # elements of canary before and after every output


def _guarded(shape, dtype, canary):
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * PAD,), canary, dtype=dtype, device="cuda")
    return buf, buf[PAD:PAD + n].view(shape)


def _bands_intact(buf, n, canary):
    return bool((buf[:PAD] == canary).all()) and bool((buf[PAD + n:] == canary).all())


@pytest.mark.parametrize("name,B,H,T", [("gdn_prefill", 1, 2, 130), ("gdn_prefill", 40, 2, 65),
                                        ("gdn_prefill", 40, 2, 63), ("kda", 1, 3, 200), ("fg2_osdn_long", 2, 2, 63),
                                        ("fg2_osdn_long", 40, 2, 70), ("gdn_fp32_small", 1, 2, 77)])
def test_forward_writes_stay_in_bounds(name, B, H, T):
    w = di.WORKLOADS[name].scaled(B=B, H=H, T=T)
    x = di.make_inputs(w)
    xd = to_device(x)
    dt = xd["q"].dtype
    ob, o = _guarded((B, T, H, w.dv), dt, -7.0)
    sb, ST = _guarded((B, H, w.dk, w.dv), torch.float32, -7.0)
    dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"], xd["S0"],
                    o=o, S_T=ST)
    assert dn.dn_stream_status() == dn.DN_OK
    assert _bands_intact(ob, o.numel(), -7.0) and _bands_intact(sb, ST.numel(), -7.0)
    o_ref, S_ref = oracle.fwd(**x)
    check(o, ST, o_ref, S_ref, w.io)


def test_decode_writes_stay_in_bounds():
    w = di.WORKLOADS["decode"].scaled(B=5)
    x = di.make_inputs(w)
    xd = to_device(x)
    sb, S = _guarded(tuple(xd["S0"].shape), torch.float32, -7.0)
    S.copy_(xd["S0"])
    ob, o = _guarded((w.B, 1, w.H, w.dv), torch.bfloat16, -7.0)
    dn.dn_decode_step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"], S=S, o=o)
    assert dn.dn_stream_status() == dn.DN_OK
    assert _bands_intact(sb, S.numel(), -7.0) and _bands_intact(ob, o.numel(), -7.0)
    o_ref, S_ref = oracle.fwd(**x)
    check(o, S, o_ref, S_ref, "bf16")


@pytest.mark.parametrize("name,T", [("gdn_prefill", 130), ("fg2_osdn_long", 70)])
def test_backward_writes_stay_in_bounds(name, T):
    w = di.WORKLOADS[name].scaled(B=1, H=2, T=T)
    x = di.make_inputs(w)
    g = di.make_bwd_inputs(w)
    xd, gd = to_device(x), to_device(g)
    out, bufs = {}, {}
    for n in ("q", "k", "v", "alpha", "beta_k", "beta_v", "key_scale"):
        if xd[n] is None:
            out[n] = None
            continue
        bufs[n], out[n] = _guarded(tuple(xd[n].shape), xd[n].dtype, -7.0)
    bufs["S0"], out["S0"] = _guarded((1, 2, w.dk, w.dv), torch.float32, -7.0)
    dn.dn_chunk_bwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"], xd["S0"],
                    dO=gd["dO"], dS_T=gd["dS_T"], out=out)
    assert dn.dn_stream_status() == dn.DN_OK
    for n, b in bufs.items():
        assert _bands_intact(b, out[n].numel(), -7.0), n
        assert torch.isfinite(out[n].float()).all(), n
