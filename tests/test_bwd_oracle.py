"""Pins of the oracle's reverse mode (oracle.bwd, dn_oracle_bwd_head in oracle/dn_oracle.c), CPU only.

The pages print no backward pass; what fixes it is the forward definition (itself pinned in
test_oracle_pins.py) and calculus:

* B1 -- central finite differences of L = sum <dO, o> + <dS_T, S_T> through the forward oracle,
  for every element of every input, every gate width and both read-outs; and on sampled elements
  of a sequence long enough to cross the reverse pass's recompute blocks.
* B2 -- the adjoint identity: for fixed keys and gates, (q) -> o and (v, S0) -> (o, S_T) are
  linear, so <dO, o(x)> + <dS_T, S_T(x)> equals <grad, x> exactly (up to rounding) for any x.
* B3 -- beta^k = 0 (no writes): the state only decays and every gradient has a closed form.
* B4 -- the chunked (UT/WY) reverse mode in NumPy (oracle/chunked.py), derived separately from
  the chunk equations, agrees with the sequential reverse mode.
Planted mistakes in the C reverse pass must fail one of B1-B3.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import chunked

NAMES = ("q", "k", "v", "alpha", "beta_k", "beta_v", "key_scale", "S0")


def _case(B=1, T=6, H=2, dk=3, dv=2, seed=0, gates="channel", s0=True):
    r = np.random.default_rng(seed)
    x = {"q": r.standard_normal((B, T, H, dk)), "k": r.standard_normal((B, T, H, dk)) / np.sqrt(dk),
         "v": r.standard_normal((B, T, H, dv)),
         "S0": r.standard_normal((B, H, dk, dv)) * 0.5 if s0 else None}
    if gates == "channel":
        x.update(alpha=r.uniform(0.6, 1.0, (B, T, H, dk)), beta_k=r.uniform(0.1, 0.9, (B, T, H, dk)),
                 beta_v=r.uniform(0.3, 1.2, (B, T, H, dv)), key_scale=r.uniform(0.7, 1.3, (B, T, H, dk)))
    elif gates == "scalar":
        x.update(alpha=r.uniform(0.6, 1.0, (B, T, H)), beta_k=r.uniform(0.1, 0.9, (B, T, H)),
                 beta_v=r.uniform(0.3, 1.2, (B, T, H)), key_scale=r.uniform(0.7, 1.3, (B, T, H)))
    else:
        x.update(alpha=None, beta_k=None, beta_v=None, key_scale=None)
    dO = r.standard_normal((B, T, H, dv))
    dS_T = r.standard_normal((B, H, dk, dv))
    return x, dO, dS_T


def _loss(x, dO, dS_T, readout):
    o, S = oracle.fwd(**x, readout=readout)
    return float(np.sum(o * dO) + np.sum(S * dS_T))


def _fd_check(x, dO, dS_T, readout, sample=None, seed=0, h=1e-6, rtol=1e-7):
    g = oracle.bwd(**x, dO=dO, dS_T=dS_T, readout=readout)
    r = np.random.default_rng(seed)
    for name in NAMES:
        a = x[name]
        if a is None:
            assert g[name] is None or name == "S0"
            continue
        idx_all = list(np.ndindex(a.shape))
        if sample is not None:
            pick = r.choice(len(idx_all), min(sample, len(idx_all)), replace=False)
            idx_all = [idx_all[i] for i in pick]
        idx = idx_all
        fd = np.empty(len(idx))
        an = np.empty(len(idx))
        for n, ix in enumerate(idx):
            y = dict(x)
            y[name] = a.copy()
            y[name][ix] += h
            lp = _loss(y, dO, dS_T, readout)
            y[name][ix] -= 2 * h
            lm = _loss(y, dO, dS_T, readout)
            fd[n] = (lp - lm) / (2 * h)
            an[n] = g[name][ix]
        scale = max(np.abs(fd).max(), 1e-30)
        assert np.abs(fd - an).max() <= rtol * scale, (name, np.abs(fd - an).max() / scale)


# B1 -- every element, every gate width, both read-outs
@pytest.mark.parametrize("gates", ["channel", "scalar", "none"])
@pytest.mark.parametrize("readout", ["post", "pre"])
def test_b1_finite_differences(gates, readout):
    x, dO, dS_T = _case(seed=1, gates=gates)
    _fd_check(x, dO, dS_T, readout)


# B1 -- a sequence that crosses the reverse pass's 64-token recompute blocks (sampled elements)
@pytest.mark.parametrize("readout", ["post", "pre"])
def test_b1_finite_differences_long(readout):
    x, dO, dS_T = _case(T=150, H=1, dk=2, dv=2, seed=2)
    x["alpha"] = np.random.default_rng(3).uniform(0.97, 1.0, x["alpha"].shape)
    _fd_check(x, dO, dS_T, readout, sample=12, seed=4)


# B2 -- adjoint identity for the linear maps q -> o and (v, S0) -> (o, S_T)
@pytest.mark.parametrize("readout", ["post", "pre"])
def test_b2_adjoint_identity(readout):
    x, dO, dS_T = _case(T=200, H=2, dk=12, dv=10, seed=5)
    g = oracle.bwd(**x, dO=dO, dS_T=dS_T, readout=readout)
    r = np.random.default_rng(6)
    dq = r.standard_normal(x["q"].shape)
    dv = r.standard_normal(x["v"].shape)
    dS0 = r.standard_normal(x["S0"].shape)
    o, _ = oracle.fwd(**dict(x, q=dq), readout=readout)
    lhs_q = float(np.sum(o * dO))  # o is linear in q for fixed (v, S0); S_T does not depend on q
    assert np.abs(oracle.fwd(**dict(x, q=np.zeros_like(dq)), readout=readout)[0]).max() == 0.0
    np.testing.assert_allclose(lhs_q, np.sum(g["q"] * dq), rtol=1e-11)
    lhs_vs = _loss(dict(x, v=dv, S0=dS0), dO, dS_T, readout)  # (v, S0) -> (o, S_T) is linear
    np.testing.assert_allclose(lhs_vs, np.sum(g["v"] * dv) + np.sum(g["S0"] * dS0), rtol=1e-11)


# B3 -- beta^k = 0: S_t = Diag(gamma_t) S0 with gamma_t = prod_{s<=t} alpha_s, and
#   dq_t = S_t dO_t (post) / S_{t-1} dO_t (pre),  dk = dv = dbeta^v = dd = 0,
#   dS0 = sum_t Diag(gamma_t') q_t dO_t^T + Diag(gamma_T) dS_T,
#   dbeta^k_t = d_t (.) k_t (.) (dS_t u_t) with dS_t the adjoint of S_t and u_t = beta^v v_t - S_bar_t^T k_t,
#   d log alpha_s = sum_{t >= s} gamma_t (.) rowsum(S0 (.) (q_t dO_t^T)) + gamma_T (.) rowsum(S0 (.) dS_T).
@pytest.mark.parametrize("mode", ["channel", "scalar"])
@pytest.mark.parametrize("readout", ["post", "pre"])
def test_b3_no_writes_closed_form(mode, readout):
    x, dO, dS_T = _case(T=9, H=1, dk=4, dv=3, seed=7, gates=mode)
    x["beta_k"] = np.zeros_like(x["beta_k"])
    g = oracle.bwd(**x, dO=dO, dS_T=dS_T, readout=readout)
    T, dk, dv = 9, 4, 3
    a = x["alpha"][0, :, 0]
    a = np.repeat(a[:, None], dk, axis=1) if a.ndim == 1 else a
    gam = np.cumprod(a, axis=0)                                  # gamma_t after token t
    gread = gam if readout == "post" else np.vstack([np.ones((1, dk)), gam[:-1]])
    S0, q, k, v = x["S0"][0, 0], x["q"][0, :, 0], x["k"][0, :, 0], x["v"][0, :, 0]
    dOh, dST = dO[0, :, 0], dS_T[0, 0]
    for t in range(T):
        np.testing.assert_allclose(g["q"][0, t, 0], (gread[t][:, None] * S0) @ dOh[t], rtol=1e-12, atol=1e-14)
    for name in ("k", "v"):
        assert np.abs(g[name]).max() < 1e-14
    assert np.abs(g["beta_v"]).max() < 1e-14 and np.abs(g["key_scale"]).max() < 1e-14
    dS0 = sum(gread[t][:, None] * np.outer(q[t], dOh[t]) for t in range(T)) + gam[-1][:, None] * dST
    np.testing.assert_allclose(g["S0"][0, 0], dS0, rtol=1e-12, atol=1e-14)
    # write-strength gradient at beta^k = 0
    bv = x["beta_v"][0, :, 0]
    bv = np.repeat(bv[:, None], dv, axis=1) if bv.ndim == 1 else bv
    dd = x["key_scale"][0, :, 0]
    dd = np.repeat(dd[:, None], dk, axis=1) if dd.ndim == 1 else dd
    dbk = np.zeros((T, dk))
    for t in range(T):
        dS_t = gam[-1][:, None] / gam[t][:, None] * dST
        for s in range(t + (0 if readout == "post" else 1), T):
            gs = gam[s] if readout == "post" else gam[s - 1]
            dS_t = dS_t + (gs / gam[t])[:, None] * np.outer(q[s], dOh[s])
        u = bv[t] * v[t] - (gam[t][:, None] * S0).T @ k[t]
        dbk[t] = dd[t] * k[t] * (dS_t @ u)
    got = g["beta_k"][0, :, 0]
    np.testing.assert_allclose(got, dbk.sum(axis=1) if got.ndim == 1 else dbk, rtol=1e-11, atol=1e-14)
    # decay gradient
    contrib = np.array([gread[t] * ((S0 @ dOh[t]) * q[t]) for t in range(T)])  # through o_t
    dlog = np.zeros((T, dk))
    for s in range(T):
        first = s if readout == "post" else s + 1
        dlog[s] = contrib[first:].sum(axis=0) + gam[-1] * np.sum(S0 * dST, axis=1)
    da = dlog / a
    got = g["alpha"][0, :, 0]
    np.testing.assert_allclose(got, da.sum(axis=1) if got.ndim == 1 else da, rtol=1e-11, atol=1e-14)


# B4 -- the chunked reverse mode against the sequential one, both read-outs
@pytest.mark.parametrize("readout", ["post", "pre"])
@pytest.mark.parametrize("T,C", [(1, 4), (5, 4), (64, 16), (65, 16), (130, 64), (37, 8)])
@pytest.mark.parametrize("gates", ["channel", "scalar", "none"])
def test_b4_chunked_reverse_matches(T, C, gates, readout):
    x, dO, dS_T = _case(T=T, H=2, dk=6, dv=5, seed=T + C, gates=gates)
    g = oracle.bwd(**x, dO=dO, dS_T=dS_T, readout=readout)
    gc = chunked.bwd(**x, dO=dO, dS_T=dS_T, C=C, readout=readout)
    for name in NAMES:
        if g[name] is None:
            assert gc[name] is None
            continue
        np.testing.assert_allclose(gc[name], g[name], rtol=1e-9, atol=1e-11, err_msg=name)


def test_golden_fixture_regression():
    """The committed fixture was written by tests/golden/make_golden.py (oracle and seeded inputs only)."""
    import json
    import dn_inputs as di
    with open(os.path.join(os.path.dirname(__file__), "golden", "oracle_bwd_tiny.json")) as f:
        gold = json.load(f)
    w = di.WORKLOADS[gold["workload"]].scaled(**gold["sizes"])
    x = di.make_inputs(w)
    gb = di.make_bwd_inputs(w)
    g = oracle.bwd(**x, dO=gb["dO"], dS_T=gb["dS_T"])
    assert sorted(gold["grad_norm"]) == sorted(n for n, a in g.items() if a is not None)
    for n, head in gold["grad_head"].items():
        np.testing.assert_allclose(g[n].ravel()[: len(head)], head, rtol=1e-12, atol=1e-15, err_msg=n)
        np.testing.assert_allclose(np.linalg.norm(g[n]), gold["grad_norm"][n], rtol=1e-12, err_msg=n)


SRC = os.path.join(os.path.dirname(oracle.__file__), "dn_oracle.c")
MUTATIONS = {
    "erase_adjoint_dropped": ("const double dsb = dS[(int64_t)i * dv + j] - kt[i] * du[j];",
                              "const double dsb = dS[(int64_t)i * dv + j];"),
    "key_gradient_sign": ("dkt[i] = bk * dd * dw[i] - acc;", "dkt[i] = bk * dd * dw[i] + acc;"),
    "decay_gradient_on_new_state": ("da += dsb * S_prev[(int64_t)i * dv + j];",
                                    "da += dsb * S_t[(int64_t)i * dv + j];"),
    "final_state_adjoint_dropped": ("dS[e] = dS_T ? dS_T[e] : 0.0;", "dS[e] = 0.0;"),
    "value_gradient_without_beta_v": ("dvt[j] = gate(beta_v, bv_w, t, j) * du[j];", "dvt[j] = du[j];"),
    "post_read_uses_old_state": ("const double* S_read = pre_read ? S_prev : S_t;",
                                 "const double* S_read = S_prev;"),
    "adjoint_not_decayed": ("dS[(int64_t)i * dv + j] = decay * dsb;", "dS[(int64_t)i * dv + j] = dsb;"),
    "beta_k_gradient_without_d": ("gate_grad(dbeta_k, bk_w, t, i, dd * kt[i] * dw[i]);",
                                  "gate_grad(dbeta_k, bk_w, t, i, kt[i] * dw[i]);"),
}

PINS = [lambda: test_b1_finite_differences("channel", "post"),
        lambda: test_b1_finite_differences("scalar", "pre"),
        lambda: test_b1_finite_differences_long("post"),
        lambda: test_b2_adjoint_identity("post"),
        lambda: test_b3_no_writes_closed_form("channel", "post")]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_bwd_pins_catch_planted_mistake(name, tmp_path, monkeypatch):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old}"
    (tmp_path / "mut.c").write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(tmp_path / "mut.c"), "-lm"],
                   check=True)
    lib = ctypes.CDLL(str(so))
    real = oracle._load()
    for fn in ("dn_oracle_heads", "dn_oracle_bwd_heads"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", lib)
    failed = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            failed.append(pin)
    assert failed, f"no pin caught the planted mistake '{name}'"
