"""Pins of the Memory Caching oracle (oracle/memcache.py), CPU only.

They check the read-out with the cache against what the Memory Caching page fixes: one segment
is the plain recurrence (N = 1, "a standard RNN"); one-token segments give (gated) linear
attention (N = L, "a Transformer with global attention"), written out here as attention; a
memory that never changes is read once per segment it sits in; the read-out is linear in the
gates, and the residual memory is the all-ones gate. Planted mistakes must fail a pin.
"""
import os
import types

import numpy as np
import pytest

import oracle
from oracle import memcache


def _x(T=12, H=2, dk=6, dv=5, seed=0, gated=True):
    r = np.random.default_rng(seed)
    x = {"q": r.standard_normal((1, T, H, dk)), "k": r.standard_normal((1, T, H, dk)) / np.sqrt(dk),
         "v": r.standard_normal((1, T, H, dv))}
    if gated:
        x.update(alpha=r.uniform(0.8, 1.0, (1, T, H)), beta_k=r.uniform(0.1, 0.9, (1, T, H)))
    return x


def pin_one_segment_is_the_recurrence(mc=memcache.mc_fwd):
    x = _x(seed=1)
    o, M = mc(**x, seg_len=12)
    o_ref, S_ref = oracle.fwd(**x)
    np.testing.assert_allclose(o, o_ref, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(M[:, 0], S_ref, rtol=1e-13, atol=1e-14)


def pin_one_token_segments_are_attention(mc=memcache.mc_fwd):
    T, H, dk, dv = 7, 2, 5, 4
    r = np.random.default_rng(2)
    q, k, v = r.standard_normal((1, T, H, dk)), r.standard_normal((1, T, H, dk)), r.standard_normal((1, T, H, dv))
    g = r.uniform(0.0, 1.0, (1, T, H, T))
    o, _ = mc(q, k, v, seg_len=1, gates=g)
    att = np.zeros((1, T, H, dv))
    for t in range(T):
        for s in range(t + 1):
            w = 1.0 if s == t else g[0, t, :, s]  # the token's own segment is its online memory
            att[0, t] += (w * np.einsum("hk,hk->h", q[0, t], k[0, s]))[:, None] * v[0, s]
    np.testing.assert_allclose(o, att, rtol=1e-12, atol=1e-13)


def pin_frozen_memory_is_read_per_segment(mc=memcache.mc_fwd):
    T, H, dk, dv, L = 10, 2, 4, 3, 3
    r = np.random.default_rng(3)
    q, k, v = r.standard_normal((1, T, H, dk)), r.standard_normal((1, T, H, dk)), r.standard_normal((1, T, H, dv))
    S0 = r.standard_normal((1, H, dk, dv))
    o, M = mc(q, k, v, beta_k=np.zeros((1, T, H)), S0=S0, seg_len=L)  # no writes: every memory is S0
    for t in range(T):
        j = t // L
        np.testing.assert_allclose(o[0, t], (j + 1) * np.einsum("hkv,hk->hv", S0[0], q[0, t]), rtol=1e-13)
    np.testing.assert_allclose(M, np.broadcast_to(S0[:, None], M.shape), rtol=1e-14)


def pin_linear_in_the_gates(mc=memcache.mc_fwd):
    x = _x(seed=4)
    N = 4
    r = np.random.default_rng(4)
    g1, g2 = r.uniform(0, 1, (1, 12, 2, N)), r.uniform(0, 1, (1, 12, 2, N))
    o0, _ = mc(**x, seg_len=3, gates=np.zeros_like(g1))
    o1, _ = mc(**x, seg_len=3, gates=g1)
    o2, _ = mc(**x, seg_len=3, gates=g2)
    o12, _ = mc(**x, seg_len=3, gates=g1 + g2)
    np.testing.assert_allclose(o12 - o0, (o1 - o0) + (o2 - o0), rtol=1e-11, atol=1e-12)
    oR, _ = mc(**x, seg_len=3, gates=None)
    o1s, _ = mc(**x, seg_len=3, gates=np.ones_like(g1))
    np.testing.assert_allclose(oR, o1s, rtol=1e-14)
    # with zero gates only the online memory remains: segment by segment, the recurrence from zero
    for j in range(N):
        sl = slice(3 * j, 3 * j + 3)
        o_seg, _ = oracle.fwd(**{n: a[:, sl] for n, a in x.items()})
        np.testing.assert_allclose(o0[:, sl], o_seg, rtol=1e-13, atol=1e-14)


PINS = [pin_one_segment_is_the_recurrence, pin_one_token_segments_are_attention,
        pin_frozen_memory_is_read_per_segment, pin_linear_in_the_gates]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_memcache_pin(pin):
    pin()


MUTATIONS = {
    "reads_own_segment": ("for s in range(j):", "for s in range(j + 1):"),
    "ignores_gates": ("                y = y * widen(gates)[:, t0:t1, :, s][..., None]", "                pass"),
    "memory_continues": ("        o_s, M_s = fwd(**args, S0=S0, readout=readout)",
                         "        o_s, M_s = fwd(**args, S0=(mems[-1] if mems else S0), readout=readout)"),
    "cache_skips_first_segment": ("    for j in range(1, N):", "    for j in range(2, N):"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_memcache_pins_catch_planted_mistake(name):
    old, new = MUTATIONS[name]
    src = open(os.path.join(os.path.dirname(oracle.__file__), "memcache.py")).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old}"
    mod = types.ModuleType("memcache_mutant")
    mod.__dict__.update(fwd=oracle.fwd, widen=oracle.widen, np=np)
    exec(compile(src.replace(old, new).replace("from . import fwd, widen", ""), "memcache_mutant", "exec"),
         mod.__dict__)
    failed = []
    for pin in PINS:
        try:
            pin(mod.mc_fwd)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake '{name}'"
