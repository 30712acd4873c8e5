"""The pins must catch plausible mistakes in the oracle.

Each case plants one mistake in a temporary copy of oracle/dn_oracle.c (on the
CPU, in a temp directory), loads the mutated library in place of the real one,
and checks that at least one pin in test_oracle_pins.py fails on it.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "dn_oracle.c")

MUTATIONS = {
    "residual_sign": ("u[j] -= Si[j] * ki;", "u[j] += Si[j] * ki;"),
    "drop_key_scale": ("* gate(key_scale, d_w, t, i) * kt[i];", "* kt[i];"),
    "drop_beta_k": ("w[i] = gate(beta_k, bk_w, t, i) *", "w[i] = 1.0 *"),
    "drop_beta_v": ("u[j] = gate(beta_v, bv_w, t, j) * vt[j];", "u[j] = vt[j];"),
    "update_with_raw_key": ("Si[j] += wi * u[j];", "Si[j] += kt[i] * u[j];"),
    "channel_decay_collapsed": ("double a = gate(alpha, alpha_w, t, i);",
                                "double a = gate(alpha, alpha_w, t, 0);"),
    "readout_uses_key": ("double qi = qt[i];", "double qi = kt[i];"),
    "no_decay": ("for (int j = 0; j < dv; ++j) Si[j] *= a;", "(void)a;"),
}

PINS = [
    lambda: pins.test_p1_zero_beta_pure_decay("channel"),
    lambda: pins.test_p1_zero_beta_pure_decay("scalar"),
    pins.test_p2_orthonormal_recall,
    lambda: pins.test_p3_gated_newton_condition(True),
    pins.test_p4_residual_contraction_and_hypergradient,
    pins.test_p5_vector_beta_constant_and_fg2_form,
    pins.test_p6_osdn_identity,
    pins.test_p8_resume,
    pins.test_p11_linearity,
    pins.test_p12_scalar_closed_form,
    pins.test_delta_rule_idempotent_rewrite,
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path, monkeypatch):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old}"
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(mut), "-lm"],
                   check=True)
    lib = ctypes.CDLL(str(so))
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.dn_oracle_heads.argtypes = [I, I, I, I, P, P, P, P, I, P, I, P, I, P, I, P, P, I, I]
    lib.dn_oracle_heads.restype = I
    oracle._load()
    monkeypatch.setattr(oracle, "_lib", lib)
    failed = []
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            failed.append(pin)
    assert failed, f"no pin caught the planted mistake '{name}'"
