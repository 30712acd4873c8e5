"""Pins of the OSDN phase-1 oracle (the preconditioner scan), CPU only.

The oracle (oracle.osdn_precond) follows the OSDN page, sections 2.2-2.3: token t
is written with d_t; then d_{t+1} = r_t d_t - eta grad h_t(d_t), with the closed-form
surrogate h_t(d) = ((1 - beta_t <d, k_t (.) k_t>)^2 - 1) / (2 ||k_t||^2). Its closed
form against the definition (f_t(S_t) - f_t(S_{t-1})) / ||grad f_t(S_{t-1})||^2 is
pinned in test_oracle_pins.py (P4). Here the scan itself is pinned against closed
forms, a fixed point, a finite-difference gradient and a descent property; the
mutation cases plant mistakes in a copy of the C oracle and check a pin fails.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle


def _keys(T, H=1, dk=8, seed=0, B=1):
    r = np.random.default_rng(seed)
    k = r.standard_normal((B, T, H, dk))
    return k / np.linalg.norm(k, axis=-1, keepdims=True)


def _h(d, k, beta):
    """The page's closed-form surrogate (used only to differentiate numerically)."""
    c = 1.0 - beta * np.sum(d * k * k)
    return (c * c - 1.0) / (2.0 * np.sum(k * k))


# O1 -- eta = 0: no learning, d_t = (prod_{j<t} r_j) d_0
def test_o1_no_learning_pure_retention():
    T, H, dk = 9, 2, 8
    r = np.random.default_rng(1)
    k = _keys(T, H, dk, seed=1)
    beta = r.uniform(0.1, 1.0, (1, T, H))
    ret = r.uniform(0.5, 1.0, (1, T, H))
    d0 = r.uniform(0.5, 2.0, (1, H, dk))
    d, dT = oracle.osdn_precond(k, beta, ret, d0, eta=0.0)
    for h in range(H):
        prod = 1.0
        for t in range(T):
            np.testing.assert_allclose(d[0, t, h], prod * d0[0, h], rtol=1e-14)
            prod *= ret[0, t, h]
        np.testing.assert_allclose(dT[0, h], prod * d0[0, h], rtol=1e-14)


# O2 -- the gated Newton condition beta <d, k (.) k> = 1 is a fixed point (zero gradient)
def test_o2_newton_fixed_point():
    T, dk = 12, 8
    k1 = _keys(1, 1, dk, seed=2)[0, 0, 0]
    k = np.broadcast_to(k1, (1, T, 1, dk)).copy()
    beta = np.full((1, T, 1), 0.7)
    d0 = np.full((1, 1, dk), 1.0 / (0.7 * np.sum(k1 * k1 * 1.0)))  # <d0, k^2> beta = 1 (||k|| = 1)
    d, dT = oracle.osdn_precond(k, beta, None, d0, eta=0.9)
    np.testing.assert_allclose(d[0, :, 0], np.broadcast_to(d0[0, 0], (T, dk)), rtol=1e-13)
    np.testing.assert_allclose(dT[0, 0], d0[0, 0], rtol=1e-13)


# O3 -- one repeated key, no retention: g_t = 1 - beta <d_t, k^2> contracts geometrically,
# g_t = g_0 rho^t with rho = 1 - eta beta^2 ||k^2||^2 / ||k||^2 (descent; ascent would grow)
@pytest.mark.parametrize("eta,beta", [(0.5, 0.8), (1.3, 0.6), (0.05, 1.0)])
def test_o3_geometric_contraction(eta, beta):
    T, dk = 40, 8
    r = np.random.default_rng(3)
    k1 = r.standard_normal(dk) * 0.7
    k = np.broadcast_to(k1, (1, T, 1, dk)).copy()
    d0 = r.uniform(0.2, 2.0, (1, 1, dk))
    d, _ = oracle.osdn_precond(k, np.full((1, T, 1), beta), None, d0, eta=eta)
    a = k1 * k1
    g = 1.0 - beta * (d[0, :, 0] @ a)
    rho = 1.0 - eta * beta * beta * np.sum(a * a) / np.sum(a)
    np.testing.assert_allclose(g, g[0] * rho ** np.arange(T), rtol=1e-11, atol=1e-14)


# O4 -- each step is minus eta times the gradient of the page's surrogate at d_t (central
# finite differences of h_t), on top of the retention
def test_o4_step_is_surrogate_gradient():
    T, H, dk = 6, 2, 5
    r = np.random.default_rng(4)
    k = r.standard_normal((1, T, H, dk))
    beta = r.uniform(0.1, 1.2, (1, T, H))
    ret = r.uniform(0.6, 1.0, (1, T, H))
    d0 = r.uniform(0.5, 1.5, (1, H, dk))
    eta = 0.37
    d, dT = oracle.osdn_precond(k, beta, ret, d0, eta=eta)
    nxt = np.concatenate([d[:, 1:], dT[:, None]], axis=1)
    eps = 1e-6
    for h in range(H):
        for t in range(T):
            dt, kt, bt = d[0, t, h], k[0, t, h], beta[0, t, h]
            grad = np.array([(_h(dt + eps * e, kt, bt) - _h(dt - eps * e, kt, bt)) / (2 * eps)
                             for e in np.eye(dk)])
            np.testing.assert_allclose(nxt[0, t, h], ret[0, t, h] * dt - eta * grad, rtol=1e-7, atol=1e-9)


# O5 -- with a small step and no retention the surrogate of the current token does not increase
def test_o5_descent_on_the_current_surrogate():
    T, dk = 50, 16
    k = _keys(T, 1, dk, seed=5)
    r = np.random.default_rng(5)
    beta = r.uniform(0.2, 1.0, (1, T, 1))
    d, dT = oracle.osdn_precond(k, beta, None, None, eta=0.2)
    nxt = np.concatenate([d[:, 1:], dT[:, None]], axis=1)
    for t in range(T):
        kt, bt = k[0, t, 0], beta[0, t, 0]
        assert _h(nxt[0, t, 0], kt, bt) <= _h(d[0, t, 0], kt, bt) + 1e-15


# O6 -- full forgetting (r = 0): d_{t+1} depends only on token t
def test_o6_full_forgetting():
    T, dk = 7, 6
    k = _keys(T, 1, dk, seed=6)
    beta = np.random.default_rng(6).uniform(0.2, 1.0, (1, T, 1))
    eta = 0.8
    d, dT = oracle.osdn_precond(k, beta, np.zeros((1, T, 1)), None, eta=eta)
    nxt = np.concatenate([d[:, 1:], dT[:, None]], axis=1)
    for t in range(T):
        kt, bt = k[0, t, 0], beta[0, t, 0]
        g = 1.0 - bt * np.sum(d[0, t, 0] * kt * kt)
        np.testing.assert_allclose(nxt[0, t, 0], eta * bt * g * kt * kt / np.sum(kt * kt), rtol=1e-13)


# O7 -- resume: the scan over T1 then T2 (d0 = d_T1) equals the scan over T1 + T2; a zero key
# changes nothing but the retention
def test_o7_resume_and_zero_key():
    T1, T2, H, dk = 5, 7, 2, 8
    k = _keys(T1 + T2, H, dk, seed=7)
    k[0, 3, 1] = 0.0
    r = np.random.default_rng(7)
    beta = r.uniform(0.2, 1.0, (1, T1 + T2, H))
    ret = r.uniform(0.8, 1.0, (1, T1 + T2, H))
    d, dT = oracle.osdn_precond(k, beta, ret, None, eta=0.6)
    d1, dT1 = oracle.osdn_precond(k[:, :T1], beta[:, :T1], ret[:, :T1], None, eta=0.6)
    d2, dT2 = oracle.osdn_precond(k[:, T1:], beta[:, T1:], ret[:, T1:], dT1, eta=0.6)
    np.testing.assert_allclose(np.concatenate([d1, d2], axis=1), d, rtol=1e-14)
    np.testing.assert_allclose(dT2, dT, rtol=1e-14)
    np.testing.assert_allclose(d[0, 4, 1], ret[0, 3, 1] * d[0, 3, 1], rtol=1e-14)


# O8 -- the surrogate is quadratic in d, so one step is affine in d:
#   d_{t+1} = (r_t I - (eta beta_t^2 / ||k_t||^2) a_t a_t^T) d_t + (eta beta_t / ||k_t||^2) a_t,  a_t = k_t (.) k_t.
# Hence the scan over any segment is an affine map d -> M d + m: affine combinations of start
# states map to the same combinations of end states, and chaining the segments' maps (each read off
# the scan itself from basis start states) reproduces the whole sequence -- the composition a
# segment-parallel scan would use.
def test_o8_affine_in_d_and_segment_composition():
    T, dk, L = 48, 8, 12
    k = _keys(T, 1, dk, seed=8)
    r = np.random.default_rng(8)
    beta = r.uniform(0.2, 1.0, (1, T, 1))
    ret = r.uniform(0.85, 1.0, (1, T, 1))
    eta = 0.7
    x, y = r.uniform(0.5, 2.0, (1, 1, dk)), r.uniform(0.5, 2.0, (1, 1, dk))
    for w in (0.3, -1.7, 2.5):  # affine (not only convex) combinations
        _, ex = oracle.osdn_precond(k, beta, ret, x, eta=eta)
        _, ey = oracle.osdn_precond(k, beta, ret, y, eta=eta)
        _, ez = oracle.osdn_precond(k, beta, ret, w * x + (1 - w) * y, eta=eta)
        np.testing.assert_allclose(ez, w * ex + (1 - w) * ey, rtol=1e-12, atol=1e-13)
    d_full, dT_full = oracle.osdn_precond(k, beta, ret, x, eta=eta)
    d = x[0, 0].copy()
    for s0 in range(0, T, L):
        seg = slice(s0, s0 + L)
        _, m = oracle.osdn_precond(k[:, seg], beta[:, seg], ret[:, seg], np.zeros((1, 1, dk)), eta=eta)
        M = np.stack([oracle.osdn_precond(k[:, seg], beta[:, seg], ret[:, seg], np.eye(dk)[i][None, None], eta=eta)[1][0, 0]
                      - m[0, 0] for i in range(dk)], axis=1)
        # the same map from the per-token matrices written out
        A, c = np.eye(dk), np.zeros(dk)
        for t in range(s0, s0 + L):
            kt = k[0, t, 0]
            at, nrm = kt * kt, np.sum(kt * kt)
            At = ret[0, t, 0] * np.eye(dk) - eta * beta[0, t, 0] ** 2 / nrm * np.outer(at, at)
            A, c = At @ A, At @ c + eta * beta[0, t, 0] / nrm * at
        np.testing.assert_allclose(M, A, rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(m[0, 0], c, rtol=1e-11, atol=1e-13)
        d = M @ d + m[0, 0]
    np.testing.assert_allclose(d, dT_full[0, 0], rtol=1e-11)


SRC = os.path.join(os.path.dirname(oracle.__file__), "dn_oracle.c")
MUTATIONS = {
    "ascent": ("d[i] = rt * d[i] - eta * grad;", "d[i] = rt * d[i] + eta * grad;"),
    "no_norm": ("-beta[t] * g * kt[i] * kt[i] / nrm", "-beta[t] * g * kt[i] * kt[i]"),
    "linear_key": ("-beta[t] * g * kt[i] * kt[i] / nrm", "-beta[t] * g * kt[i] / nrm"),
    "output_after_step": ("      out[i] = d[i];\n", ""),
    "retention_on_step": ("d[i] = rt * d[i] - eta * grad;", "d[i] = rt * (d[i] - eta * grad);"),
    "beta_once": ("const double g = 1.0 - beta[t] * dot;", "const double g = 1.0 - dot;"),
}
PINS = [test_o1_no_learning_pure_retention, test_o2_newton_fixed_point,
        lambda: test_o3_geometric_contraction(0.5, 0.8), test_o4_step_is_surrogate_gradient,
        test_o5_descent_on_the_current_surrogate, test_o6_full_forgetting, test_o7_resume_and_zero_key,
        test_o8_affine_in_d_and_segment_composition]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_osdn_pins_catch_planted_mistake(name, tmp_path, monkeypatch):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old}"
    mut = src.replace(old, new)
    if name == "output_after_step":  # write d_t after the step instead of before it
        mut = mut.replace("      d[i] = rt * d[i] - eta * grad;\n",
                          "      d[i] = rt * d[i] - eta * grad;\n      out[i] = d[i];\n")
    (tmp_path / "mut.c").write_text(mut)
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(tmp_path / "mut.c"), "-lm"],
                   check=True)
    lib = ctypes.CDLL(str(so))
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.dn_oracle_osdn_heads.argtypes = [I, I, I, P, P, P, ctypes.c_double, P, P, I]
    lib.dn_oracle_osdn_heads.restype = I
    oracle._load()
    monkeypatch.setattr(oracle, "_lib", lib)
    failed = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            failed.append(pin)
    assert failed, f"no pin caught the planted mistake '{name}'"
