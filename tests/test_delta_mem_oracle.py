"""Pins of the oracle's pre-update read-out and of the delta-mem mapping (CPU only).

The delta-mem page (section 2.A) updates a small value-major state with an undecayed residual,
S_t = lambda_t S_{t-1} + beta_t (v_t - S_{t-1} k_t) k_t^T, and reads it before the update,
r_t = S_{t-1} q_t (section 2.C). The recurrence here decays before the residual; the two agree
exactly under alpha = lambda, beta^k = beta / lambda, beta^v = lambda (lambda > 0), read out
before the update (readout="pre"). These tests pin the pre-update read-out against the
post-update one, and the mapping against the page's update written out literally.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle


def _case(T=9, H=2, dk=8, dv=8, seed=0, channel=False):
    r = np.random.default_rng(seed)
    x = {"q": r.standard_normal((1, T, H, dk)), "k": r.standard_normal((1, T, H, dk)) / np.sqrt(dk),
         "v": r.standard_normal((1, T, H, dv)),
         "alpha": r.uniform(0.8, 1.0, (1, T, H, dk) if channel else (1, T, H)),
         "beta_k": r.uniform(0.1, 1.0, (1, T, H)), "beta_v": None, "key_scale": None,
         "S0": r.standard_normal((1, H, dk, dv)) * 0.3}
    return x


# D1 -- the pre-update read-out of token t is the post-update read-out of token t - 1 asked with
# q_t; the first token reads S0; the final state does not depend on the read-out
@pytest.mark.parametrize("channel", [False, True])
def test_d1_pre_read_is_the_previous_state(channel):
    x = _case(seed=1, channel=channel)
    T = x["q"].shape[1]
    o_pre, S_pre = oracle.fwd(**x, readout="pre")
    o_post, S_post = oracle.fwd(**x)
    np.testing.assert_array_equal(S_pre, S_post)
    np.testing.assert_allclose(o_pre[0, 0], np.einsum("hij,hi->hj", x["S0"][0], x["q"][0, 0]), rtol=1e-13)
    for t in range(1, T):
        y = {n: (None if a is None else (a[:, :t].copy() if n != "S0" else a)) for n, a in x.items()}
        y["q"][:, t - 1] = x["q"][:, t]
        o_t, _ = oracle.fwd(**y)
        np.testing.assert_allclose(o_pre[:, t], o_t[:, t - 1], rtol=1e-12, atol=1e-14)


# D2 -- the delta-mem update and read written from its page, value-major, r x r states
# (r = 8, the page's size), against the oracle under the mapping
def test_d2_delta_mem_mapping():
    T, H, r_ = 40, 3, 8
    g = np.random.default_rng(2)
    q = g.standard_normal((1, T, H, r_))
    k = g.standard_normal((1, T, H, r_))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)  # the page normalises q and k
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = g.standard_normal((1, T, H, r_))
    lam = g.uniform(0.85, 1.0, (1, T, H))
    beta = g.uniform(0.05, 0.9, (1, T, H))
    S0 = g.standard_normal((1, H, r_, r_)) * 0.2  # value-major
    reads = np.zeros((1, T, H, r_))
    S_end = np.zeros_like(S0)
    for h in range(H):
        S = S0[0, h].copy()
        for t in range(T):
            kt, vt = k[0, t, h], v[0, t, h]
            reads[0, t, h] = S @ q[0, t, h]
            S = lam[0, t, h] * S + beta[0, t, h] * np.outer(vt - S @ kt, kt)
        S_end[0, h] = S
    o, S_T = oracle.fwd(q, k, v, alpha=lam, beta_k=beta / lam, beta_v=lam,
                        S0=np.ascontiguousarray(np.swapaxes(S0, -1, -2)), readout="pre")
    np.testing.assert_allclose(o, reads, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(np.swapaxes(S_T, -1, -2), S_end, rtol=1e-11, atol=1e-13)


SRC = os.path.join(os.path.dirname(oracle.__file__), "dn_oracle.c")
MUTATIONS = {
    "pre_read_after_decay": ("    if (pre_read) {\n      /* o_t = S_{t-1}^T q_t, before this token's decay and write */",
                             "    if (0) {\n      /* o_t = S_{t-1}^T q_t, before this token's decay and write */"),
    "pre_read_with_key": ("const double qpre = qt[i];", "const double qpre = kt[i];"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_delta_mem_pins_catch_planted_mistake(name, tmp_path, monkeypatch):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old}"
    mut = src.replace(old, new)
    if name == "pre_read_after_decay":  # read after the decay instead of before it
        mut = mut.replace("    /* w_t = beta^k (.) d (.) k */",
                          "    if (pre_read) {\n      for (int j = 0; j < dv; ++j) ot[j] = 0.0;\n"
                          "      for (int i = 0; i < dk; ++i)\n        for (int j = 0; j < dv; ++j)"
                          " ot[j] += S[(int64_t)i * dv + j] * qt[i];\n    }\n    /* w_t = beta^k (.) d (.) k */")
    (tmp_path / "mut.c").write_text(mut)
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(tmp_path / "mut.c"), "-lm"],
                   check=True)
    lib = ctypes.CDLL(str(so))
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.dn_oracle_heads.argtypes = [I, I, I, I, P, P, P, P, I, P, I, P, I, P, I, P, P, I, I]
    lib.dn_oracle_heads.restype = I
    oracle._load()
    monkeypatch.setattr(oracle, "_lib", lib)
    failed = []
    for pin in (lambda: test_d1_pre_read_is_the_previous_state(False), test_d2_delta_mem_mapping):
        try:
            pin()
        except AssertionError:
            failed.append(pin)
    assert failed, f"no pin caught the planted mistake '{name}'"
