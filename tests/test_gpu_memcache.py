"""GPU parity of Memory Caching (segment memories by dn_chunk_fwd on the segment view, cached
read-out by dn_mc_readout) against the fp64 oracle (oracle/memcache.py), through the C ABI."""
import numpy as np
import pytest

import dn_inputs as di
import gated_linear_attention_dn_b200 as dn
import oracle
from tests.gpu_util import TOL, dev, host_f64, to_device

pytestmark = pytest.mark.gpu


def _case(name, L, gated, **kw):
    w = di.WORKLOADS[name].scaled(**kw)
    x = di.make_inputs(w)
    N = w.T // L
    g = None
    if gated:
        g = np.random.default_rng(7).uniform(0.0, 1.0, (w.B, w.T, w.H, N)).astype(np.float32)
    return w, x, g


@pytest.mark.parametrize("name,L,gated,kw", [
    ("gdn_prefill", 256, True, dict(B=1, H=2, T=1024)),
    ("gdn_prefill", 128, False, dict(B=2, H=2, T=512)),
    ("kda", 192, True, dict(B=1, H=2, T=576)),
    ("gdn_fp32_small", 64, True, dict(T=256)),
])
def test_mc_fwd_matches_oracle(name, L, gated, kw):
    w, x, g = _case(name, L, gated, **kw)
    xd = to_device(x)
    o, M = dn.mc_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"], xd["S0"],
                     seg_len=L, gates=dev(g))
    assert dn.dn_stream_status() == dn.DN_OK
    o_ref, M_ref = oracle.memcache.mc_fwd(**x, seg_len=L, gates=g)
    tol = TOL[w.io]
    eo, eM = oracle.rel_l2(host_f64(o), o_ref), oracle.rel_l2(host_f64(M), M_ref)
    print(f"[parity] mc o rel-L2 {eo:.3e} (tol {tol['o']:.0e}), M rel-L2 {eM:.3e} (tol {tol['S']:.0e})")
    assert eo <= tol["o"] and eM <= tol["S"]


def test_readout_alone_fp32():
    """The cached read-out by itself, on exact fp32 memories, against the sum written out."""
    r = np.random.default_rng(3)
    B, T, H, dk, dv, L = 2, 320, 3, 128, 64, 64
    N = T // L
    q = r.standard_normal((B, T, H, dk)).astype(np.float32)
    M = r.standard_normal((B, N, H, dk, dv)).astype(np.float32) * 0.1
    g = r.uniform(0, 1, (B, T, H, N)).astype(np.float32)
    o0 = r.standard_normal((B, T, H, dv)).astype(np.float32)
    o = dev(o0.copy())
    dn.dn_mc_readout(dev(q), dev(M), dev(g), o, seg_len=L)
    assert dn.dn_stream_status() == dn.DN_OK
    ref = o0.astype(np.float64)
    for t in range(T):
        for s in range(t // L):
            ref[:, t] += g[:, t, :, s][..., None] * np.einsum("bhk,bhkv->bhv", q[:, t].astype(np.float64), M[:, s])
    err = oracle.rel_l2(host_f64(o), ref)
    print(f"[parity] mc read-out rel-L2 {err:.3e}")
    assert err <= 1e-5


@pytest.mark.parametrize("dk,dv", [(128, 128), (128, 64), (64, 128), (64, 64)])
@pytest.mark.parametrize("L,gated", [(128, False), (64, False), (100, False), (256, True), (100, True)])
def test_readout_alone_bf16(dk, dv, L, gated):
    """The tensor-core read-out (bf16 io) by itself against the sum written out in fp64 from the same
    bf16 inputs: tiles inside one segment (one product of the summed memories), tiles over several
    segments and ragged segment lengths (a product per memory, rows masked), and gates; the
    tolerance is the bf16 rounding of the output."""
    import torch
    r = np.random.default_rng(11 + dk + dv + L)
    B, H, T = 2, 3, 640 + 37
    N = -(-T // L)
    qb = torch.from_numpy(r.standard_normal((B, T, H, dk)).astype(np.float32)).bfloat16()
    o0 = torch.from_numpy(r.standard_normal((B, T, H, dv)).astype(np.float32)).bfloat16()
    M = r.standard_normal((B, N, H, dk, dv)).astype(np.float32) * 0.1
    g = r.uniform(0, 1, (B, T, H, N)).astype(np.float32) if gated else None
    o = o0.cuda()
    dn.dn_mc_readout(qb.cuda(), dev(M), dev(g), o, seg_len=L)
    assert dn.dn_stream_status() == dn.DN_OK
    q64 = qb.double().numpy()
    ref = o0.double().numpy().copy()
    for t in range(T):
        for s in range(t // L):
            w = g[:, t, :, s][..., None] if gated else 1.0
            ref[:, t] += w * np.einsum("bhk,bhkv->bhv", q64[:, t], M[:, s])
    err = oracle.rel_l2(host_f64(o), ref)
    print(f"[parity] mc read-out bf16 d_k={dk} d_v={dv} L={L} gated={gated}: rel-L2 {err:.3e}")
    assert err <= 5e-3
    # rows of the first segment are untouched
    assert torch.equal(o[:, :L].cpu(), o0[:, :L])


def test_mc_full_size_sampled_batches():
    """The configuration the benchmark times (GDN prefill B=8, H=16, T=4096, four segments of 1024,
    residual memory): the whole batch on the GPU; the first and last batch rows (all heads, the
    whole sequence) against the oracle. Batch rows are independent, so the oracle runs only those."""
    w = di.WORKLOADS["gdn_prefill"]
    x = di.make_inputs(w)
    xd = to_device(x)
    o, M = dn.mc_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"], xd["S0"],
                     seg_len=1024)
    assert dn.dn_stream_status() == dn.DN_OK
    sel = [0, w.B - 1]
    xs = {n: (None if a is None else np.ascontiguousarray(a[sel])) for n, a in x.items()}
    o_ref, M_ref = oracle.memcache.mc_fwd(**xs, seg_len=1024)
    tol = TOL[w.io]
    eo = oracle.rel_l2(host_f64(o)[sel], o_ref)
    eM = oracle.rel_l2(host_f64(M)[sel], M_ref)
    print(f"[parity] mc full size o rel-L2 {eo:.3e} (tol {tol['o']:.0e}), M rel-L2 {eM:.3e} (tol {tol['S']:.0e})")
    assert eo <= tol["o"] and eM <= tol["S"]
