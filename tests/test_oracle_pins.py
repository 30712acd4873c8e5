"""Pins of the fp64 oracle against what the pages and the mathematics fix.

None of these re-types the oracle's loop: each checks it against a closed form,
an identity printed on the pages, a special case with a textbook answer, or the
independent chunked (UT/WY) evaluation. A dropped decay, a wrong sign in the
residual, a transposed outer product, a gate applied to the wrong side or a
mixed-up (b, h) index each fails at least one of them.
"""
import numpy as np
import pytest

import dn_inputs as di
import oracle

RNG = np.random.default_rng(12345)


def _rand_case(B=1, T=7, H=2, dk=5, dv=6, seed=0, alpha="channel", bk="channel", bv="channel",
               d=True, s0=True):
    r = np.random.default_rng(seed)
    q = r.standard_normal((B, T, H, dk))
    k = r.standard_normal((B, T, H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    v = r.standard_normal((B, T, H, dv))

    def g(mode, width, lo, hi):
        if mode is None:
            return None
        if mode == "scalar":
            return r.uniform(lo, hi, (B, T, H))
        return r.uniform(lo, hi, (B, T, H, width))

    return dict(q=q, k=k, v=v, alpha=g(alpha, dk, 0.7, 1.0), beta_k=g(bk, dk, 0.1, 0.9),
                beta_v=g(bv, dv, 0.3, 1.2), key_scale=g("channel" if d else None, dk, 0.8, 1.2),
                S0=r.standard_normal((B, H, dk, dv)) * 0.3 if s0 else None)


# P1 -- beta^k = 0: no writes, the state only decays: S_t = Diag(prod_{s<=t} alpha_s) S0,
# o_t = S_t^T q_t (forget gate applied to the state, Sparse Delta Memory page,
# "Gated Delta Updates"; KDA channel decay, FG2-GDN page section 1).
@pytest.mark.parametrize("mode", ["scalar", "channel"])
def test_p1_zero_beta_pure_decay(mode):
    x = _rand_case(T=9, alpha=mode, seed=1)
    x["beta_k"] = np.zeros_like(x["beta_k"])
    o, ST = oracle.fwd(**x)
    B, T, H, dk = x["q"].shape
    for b in range(B):
        for h in range(H):
            a = x["alpha"][b, :, h]
            if a.ndim == 1:
                a = np.repeat(a[:, None], dk, axis=1)
            cum = np.cumprod(a, axis=0)  # [T, dk]
            for t in range(T):
                St = cum[t][:, None] * x["S0"][b, h]
                np.testing.assert_allclose(o[b, t, h], St.T @ x["q"][b, t, h], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(ST[b, h], cum[-1][:, None] * x["S0"][b, h], rtol=1e-12, atol=1e-14)


# P2 -- alpha = 1, beta = 1, S0 = 0, orthonormal keys: the delta rule stores each pair exactly,
# S_t^T k_i = v_i for i <= t and S_T = sum_i k_i v_i^T (delta rule as online regression,
# OSDN page section 1; a unit step on an orthonormal key set is exact recall).
def test_p2_orthonormal_recall():
    dk, dv, T = 8, 5, 6
    r = np.random.default_rng(2)
    Qm, _ = np.linalg.qr(r.standard_normal((dk, dk)))
    keys = Qm[:T]                       # orthonormal rows
    vals = r.standard_normal((T, dv))
    k = keys[None, :, None, :]
    v = vals[None, :, None, :]
    # read back every stored key through q: after step t, o_t = S_t^T q_t
    for i in range(T):
        q = np.repeat(keys[i][None, None, None, :], T, axis=1)
        o, ST = oracle.fwd(q, k, v)
        for t in range(T):
            expect = vals[i] if i <= t else np.zeros(dv)
            np.testing.assert_allclose(o[0, t, 0], expect, atol=1e-12)
    np.testing.assert_allclose(ST[0, 0], keys.T @ vals, atol=1e-12)


# P3 -- gated Newton condition beta <d, k^2> = 1 (OSDN page, section 3, theorem 5.2 condition):
# one step then maps k_t exactly onto beta^v (.) v_t, for any prior state and decay.
@pytest.mark.parametrize("with_d", [False, True])
def test_p3_gated_newton_condition(with_d):
    x = _rand_case(T=11, H=3, seed=3, d=with_d)
    kk = x["k"] ** 2
    dd = x["key_scale"] if with_d else np.ones_like(kk)
    # rescale beta^k per token so that <beta^k (.) d, k^2> = 1
    x["beta_k"] = x["beta_k"] / np.sum(x["beta_k"] * dd * kk, axis=-1, keepdims=True)
    x["q"] = x["k"].copy()
    o, _ = oracle.fwd(**x)
    np.testing.assert_allclose(o, x["beta_v"] * x["v"], rtol=1e-10, atol=1e-11)


def _one_step_value_major(S_vm, k, v, beta, d):
    """The OSDN page's printed step S - beta grad f(S) D, value-major S in R^{dv x dk},
    f(S) = 0.5 ||S k - v||^2, grad f(S) = (S k - v) k^T, D = diag(d)."""
    grad = np.outer(S_vm @ k - v, k)
    return S_vm - beta * grad @ np.diag(d)


# P4 -- residual contraction and the closed-form hypergradient surrogate (OSDN page,
# section 2.2): f(S_t) = (1 - beta <d, k^2>)^2 f(S_{t-1}), and
# h = (f(S_t) - f(S_{t-1})) / ||grad f(S_{t-1})||^2 = ((1 - beta <d,k^2>)^2 - 1) / (2 ||k||^2).
# Also the general form with decay and beta^v: S_t^T k - beta^v v
#   = (1 - <beta^k (.) d, k^2>) (S_bar^T k - beta^v v), checked token by token.
def test_p4_residual_contraction_and_hypergradient():
    r = np.random.default_rng(4)
    dk, dv = 6, 4
    for trial in range(20):
        S0 = r.standard_normal((1, 1, dk, dv))
        k = r.standard_normal(dk)
        v = r.standard_normal(dv)
        q = r.standard_normal(dk)
        beta = r.uniform(0.1, 1.5)
        d = r.uniform(0.5, 1.5, dk)
        _, S1 = oracle.fwd(q[None, None, None], k[None, None, None], v[None, None, None],
                           beta_k=np.full((1, 1, 1), beta), key_scale=d[None, None, None], S0=S0)
        f0 = 0.5 * np.sum((S0[0, 0].T @ k - v) ** 2)
        f1 = 0.5 * np.sum((S1[0, 0].T @ k - v) ** 2)
        c = 1.0 - beta * np.sum(d * k * k)
        np.testing.assert_allclose(f1, c * c * f0, rtol=1e-10)
        grad_sq = np.sum(np.outer(S0[0, 0].T @ k - v, k) ** 2)
        h = (f1 - f0) / grad_sq
        np.testing.assert_allclose(h, (c * c - 1.0) / (2.0 * np.sum(k * k)), rtol=1e-9, atol=1e-12)
    # general gated form, per token, chaining T = 1 calls
    x = _rand_case(T=10, H=1, seed=44)
    S = x["S0"].copy()
    for t in range(10):
        sl = {n: (None if a is None else a[:, t:t + 1]) for n, a in x.items() if n != "S0"}
        _, S_new = oracle.fwd(**sl, S0=S)
        kt = x["k"][0, t, 0]
        a = x["alpha"][0, t, 0]
        Sbar = a[:, None] * S[0, 0]
        bvv = x["beta_v"][0, t, 0] * x["v"][0, t, 0]
        lhs = S_new[0, 0].T @ kt - bvv
        rho = 1.0 - np.sum(x["beta_k"][0, t, 0] * x["key_scale"][0, t, 0] * kt * kt)
        np.testing.assert_allclose(lhs, rho * (Sbar.T @ kt - bvv), rtol=1e-9, atol=1e-12)
        S = S_new


# P5 -- vector beta equal to a constant reproduces scalar GDN; and the FG2-GDN printed update
# S_t = (I - k~ k~^T) Diag(alpha) S_{t-1} + k~ v~^T with k~ = sqrt(beta) (.) k, v~ = sqrt(beta) (.) v
# (FG2-GDN page, section 2.A), computed literally here for a NON-constant vector beta,
# equals the oracle fed k' = sqrt(beta) (.) k, beta^k = 1, beta^v = sqrt(beta).
def test_p5_vector_beta_constant_and_fg2_form():
    x = _rand_case(T=12, H=2, dk=6, dv=6, seed=5, d=False, bv=None)  # sqrt(beta) (.) v needs dk = dv
    c = 0.37
    xs = dict(x, beta_k=np.full(x["q"].shape[:3], c))
    xc = dict(x, beta_k=np.full(x["q"].shape, c))
    o1, S1 = oracle.fwd(**xs)
    o2, S2 = oracle.fwd(**xc)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)

    B, T, H, dk = x["q"].shape
    beta = np.random.default_rng(55).uniform(0.05, 0.95, (B, T, H, dk))
    kt = np.sqrt(beta) * x["k"]
    o3, S3 = oracle.fwd(x["q"], kt, x["v"], alpha=x["alpha"], beta_v=np.sqrt(beta), S0=x["S0"])
    for b in range(B):
        for h in range(H):
            S = x["S0"][b, h].copy()
            for t in range(T):
                kk = kt[b, t, h]
                vv = np.sqrt(beta[b, t, h]) * x["v"][b, t, h]
                S = (np.eye(dk) - np.outer(kk, kk)) @ np.diag(x["alpha"][b, t, h]) @ S + np.outer(kk, vv)
                np.testing.assert_allclose(o3[b, t, h], S.T @ x["q"][b, t, h], rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(S3[b, h], S, rtol=1e-11, atol=1e-12)


# P6 -- OSDN right-preconditioning identity (OSDN page, section 2.1): the value-major gradient
# step S - beta grad f(S) D, transposed, equals the key-major oracle with beta^k = beta, key
# scale d (no decay, beta^v = 1).
def test_p6_osdn_identity():
    r = np.random.default_rng(6)
    dk, dv, T = 7, 5, 9
    k = r.standard_normal((1, T, 1, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q = r.standard_normal((1, T, 1, dk))
    v = r.standard_normal((1, T, 1, dv))
    beta = r.uniform(0.2, 0.9, (1, T, 1))
    d = r.uniform(0.5, 1.5, (1, T, 1, dk))
    S0 = r.standard_normal((1, 1, dk, dv))
    o, ST = oracle.fwd(q, k, v, beta_k=beta, key_scale=d, S0=S0)
    S_vm = S0[0, 0].T.copy()
    for t in range(T):
        S_vm = _one_step_value_major(S_vm, k[0, t, 0], v[0, t, 0], beta[0, t, 0], d[0, t, 0])
        np.testing.assert_allclose(o[0, t, 0], S_vm @ q[0, t, 0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(ST[0, 0], S_vm.T, rtol=1e-12, atol=1e-12)


# P7 -- chunked (UT/WY) evaluation equals the sequential definition on tiny inputs.
# C = 1 is literally sequential; both reference points (chunk start, midpoint) are checked.
@pytest.mark.parametrize("T", [1, 5, 64, 65, 130])
@pytest.mark.parametrize("C", [1, 4, 16, 64])
@pytest.mark.parametrize("d", [4, 8])
def test_p7_chunked_equals_sequential(T, C, d):
    x = _rand_case(B=1, T=T, H=2, dk=d, dv=d, seed=7 + T + C + d)
    o, ST = oracle.fwd(**x)
    for ref in ("mid", "start"):
        o2, S2 = oracle.chunked.fwd(**x, C=C, ref=ref)
        assert oracle.rel_l2(o2, o) < 1e-10
        assert oracle.rel_l2(S2, ST) < 1e-10


def test_p7_chunked_scalar_gates_strong_decay():
    # strong decay (alpha down to 0.2): the midpoint reference keeps exponents bounded
    x = _rand_case(B=1, T=130, H=1, dk=8, dv=8, seed=77, alpha="scalar", bk="scalar", bv=None, d=False)
    x["alpha"] = np.random.default_rng(78).uniform(0.2, 0.5, x["alpha"].shape)
    o, ST = oracle.fwd(**x)
    o2, S2 = oracle.chunked.fwd(**x, C=64, ref="mid")
    assert oracle.rel_l2(o2, o) < 1e-9 and oracle.rel_l2(S2, ST) < 1e-9


# P8 -- resume: fwd(T1) then fwd(T2, S0 = S_T1) equals fwd(T1 + T2); the state is the checkpoint
# (learned / carried initial state M0, Sparse Delta Memory page; per-segment cached states,
# Memory Caching page section 2).
def test_p8_resume():
    x = _rand_case(B=2, T=13, H=2, seed=8)
    o, ST = oracle.fwd(**x)
    cut = 6
    a = {n: (None if v is None else v[:, :cut]) for n, v in x.items() if n != "S0"}
    b = {n: (None if v is None else v[:, cut:]) for n, v in x.items() if n != "S0"}
    oa, Sa = oracle.fwd(**a, S0=x["S0"])
    ob, Sb = oracle.fwd(**b, S0=Sa)
    np.testing.assert_allclose(np.concatenate([oa, ob], axis=1), o, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(Sb, ST, rtol=1e-13, atol=1e-14)


# P10 -- permutation equivariance over b and h (heads are independent): catches mixed-up
# (b, h) indexing in the per-head gather/scatter.
def test_p10_permutation_equivariance():
    x = _rand_case(B=3, T=5, H=4, seed=10)
    o, ST = oracle.fwd(**x)
    pb = np.array([2, 0, 1])
    ph = np.array([3, 1, 0, 2])

    def perm(a, bt_axes=True):
        if a is None:
            return None
        a = a[pb]
        return a[:, :, ph] if bt_axes else a[:, ph]

    xp = {n: perm(v, n != "S0") for n, v in x.items()}
    o2, S2 = oracle.fwd(**xp)
    np.testing.assert_allclose(o2, o[pb][:, :, ph], rtol=1e-14, atol=0)
    np.testing.assert_allclose(S2, ST[pb][:, ph], rtol=1e-14, atol=0)
    # subset evaluation returns the same heads
    heads = [(2, 3), (0, 1)]
    oh, Sh = oracle.fwd(**x, heads=heads)
    for n, (b, h) in enumerate(heads):
        np.testing.assert_allclose(oh[n], o[b, :, h], rtol=1e-14)
        np.testing.assert_allclose(Sh[n], ST[b, h], rtol=1e-14)


# P11 -- linearity: scaling (S0, beta^v (.) v) by a scales o and S_T by a.
def test_p11_linearity():
    x = _rand_case(B=1, T=9, H=2, seed=11)
    o, ST = oracle.fwd(**x)
    a = -2.5
    o2, S2 = oracle.fwd(**dict(x, v=a * x["v"], S0=a * x["S0"]))
    np.testing.assert_allclose(o2, a * o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S2, a * ST, rtol=1e-12, atol=1e-13)


# P12 -- dk = dv = 1 with constant inputs: s_t = a s_{t-1} + b with a = alpha (1 - beta d k^2),
# b = beta d k beta^v v, whose closed form is the geometric series a^t s0 + b (1 - a^t) / (1 - a).
def test_p12_scalar_closed_form():
    T = 40
    al, be, dd, kk, bvv, vv, qq, s0 = 0.93, 0.6, 1.1, 0.8, 0.9, -1.7, 0.45, 0.3
    ones = np.ones((1, T, 1, 1))
    o, ST = oracle.fwd(qq * ones, kk * ones, vv * ones, alpha=al * ones, beta_k=be * ones,
                       beta_v=bvv * ones, key_scale=dd * ones, S0=np.full((1, 1, 1, 1), s0))
    a = al * (1.0 - be * dd * kk * kk)
    b = be * dd * kk * bvv * vv
    t = np.arange(1, T + 1)
    s = a ** t * s0 + b * (1.0 - a ** t) / (1.0 - a)
    np.testing.assert_allclose(o[0, :, 0, 0], qq * s, rtol=1e-12)
    np.testing.assert_allclose(ST[0, 0, 0, 0], s[-1], rtol=1e-12)


# Delta-rule fixed point: with alpha = 1, beta = 1 and ||k|| = 1, rewriting the same pair
# leaves the state unchanged after the first write (the residual is already zero).
def test_delta_rule_idempotent_rewrite():
    r = np.random.default_rng(13)
    dk, dv, T = 6, 3, 4
    k = r.standard_normal(dk)
    k /= np.linalg.norm(k)
    v = r.standard_normal(dv)
    S0 = r.standard_normal((1, 1, dk, dv))
    K = np.tile(k, (1, T, 1, 1))
    V = np.tile(v, (1, T, 1, 1))
    o, ST = oracle.fwd(K, K, V, S0=S0)
    _, S1 = oracle.fwd(K[:, :1], K[:, :1], V[:, :1], S0=S0)
    np.testing.assert_allclose(ST, S1, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(o[0, :, 0], np.tile(v, (T, 1)), rtol=1e-12, atol=1e-13)


def test_oracle_consumes_bf16_bits_exactly():
    w = di.WORKLOADS["gdn_prefill"].scaled(B=1, T=3, H=1, dk=8, dv=8)
    x = di.make_inputs(w)
    assert x["q"].dtype == np.uint16
    o_bits, S_bits = oracle.fwd(**x)
    xf = {n: (None if v is None else oracle.widen(v)) for n, v in x.items()}
    o_f, S_f = oracle.fwd(**xf)
    np.testing.assert_array_equal(o_bits, o_f)
    np.testing.assert_array_equal(S_bits, S_f)


def test_golden_fixture_regression():
    """The committed fixture was written by tests/golden/make_golden.py (oracle only)."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_tiny.json")
    with open(path) as f:
        g = json.load(f)
    w = di.WORKLOADS[g["workload"]].scaled(**g["sizes"])
    x = di.make_inputs(w)
    o, ST = oracle.fwd(**x)
    np.testing.assert_allclose(o.ravel()[: len(g["o_head"])], g["o_head"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(ST.ravel()[: len(g["S_head"])], g["S_head"], rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(np.linalg.norm(o), g["o_norm"], rtol=1e-12)
    np.testing.assert_allclose(np.linalg.norm(ST), g["S_norm"], rtol=1e-12)
