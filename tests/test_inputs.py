"""The seeded generator against its published definitions."""
import numpy as np
import torch

import dn_inputs as di


def test_splitmix64_reference_stream():
    # first outputs of Vigna's splitmix64 from state 0 (published reference values)
    assert di.splitmix_at(0, 0) == 0xE220A8397B1DCDAF
    assert di.splitmix_at(0, 1) == 0x6E789E6AA1B965F4
    assert di.splitmix_at(0, 2) == 0x06C45D188009454F


def test_box_muller_moments():
    z = di.fill((1 << 20,), 99, di.GEN_NORMAL, 0.0, 1.0, dtype="f64")
    assert abs(z.mean()) < 5e-3
    assert abs(z.std() - 1.0) < 5e-3
    assert abs(np.mean(z ** 4) - 3.0) < 0.05  # Gaussian kurtosis
    # the same element by its counter
    assert z[12345] == di.normal_at(99, 12345)


def test_counter_offset_regenerates_slices():
    full = di.fill((1000,), 7, di.GEN_NORMAL, 0.0, 1.0, dtype="f64")
    part = di.fill((300,), 7, di.GEN_NORMAL, 0.0, 1.0, dtype="f64", offset=500)
    np.testing.assert_array_equal(full[500:800], part)


def test_l2_rows_unit_norm_and_bf16_rne():
    x64 = di.fill((64, 128), 5, di.GEN_L2ROWS, dtype="f64", row=128)
    np.testing.assert_allclose(np.linalg.norm(x64, axis=1), 1.0, rtol=1e-14)
    xb = di.fill((64, 128), 5, di.GEN_L2ROWS, dtype="bf16", row=128)
    ref = torch.from_numpy(x64.astype(np.float32)).to(torch.bfloat16)
    np.testing.assert_array_equal(xb, ref.view(torch.int16).numpy().view(np.uint16))


def test_gate_recipes_ranges():
    a = di.fill((100000,), 3, di.GEN_EXP_NEG_SOFTPLUS, 0.1, dtype="f64")
    assert a.min() > 0.0 and a.max() < 1.0
    z = np.array([di.normal_at(3, i) for i in range(50)])
    np.testing.assert_allclose(a[:50], np.exp(-np.log1p(np.exp(z)) * 0.1), rtol=1e-14)
    s = di.fill((50,), 4, di.GEN_SIGMOID, dtype="f64")
    z = np.array([di.normal_at(4, i) for i in range(50)])
    np.testing.assert_allclose(s, 1 / (1 + np.exp(-z)), rtol=1e-14)
    u = di.fill((100000,), 8, di.GEN_UNIFORM, 0.9, 1.0, dtype="f64")
    assert u.min() >= 0.9 and u.max() < 1.0


def test_workload_shapes():
    w = di.WORKLOADS["fg2_osdn_long"].scaled(T=8)
    x = di.make_inputs(w)
    assert x["q"].shape == (2, 8, 16, 128) and x["q"].dtype == np.uint16
    assert x["alpha"].shape == (2, 8, 16, 128) and x["alpha"].dtype == np.float32
    assert x["beta_v"].shape == (2, 8, 16, 128)
    assert x["S0"].shape == (2, 16, 128, 128)
    w = di.WORKLOADS["gdn_prefill"].scaled(T=8, B=1)
    x = di.make_inputs(w)
    assert x["alpha"].shape == (1, 8, 16) and x["beta_v"] is None and x["S0"] is None
    w = di.WORKLOADS["decode"].scaled(B=4)
    x0, x1 = di.make_inputs(w, step=0), di.make_inputs(w, step=1)
    assert x0["q"].shape == (4, 1, 32, 128)
    assert not np.array_equal(x0["q"], x1["q"])
    assert x0["S0"] is not None and x1["S0"] is None


def test_backward_cotangents():
    """dO ~ N(0,1) in the storage dtype and dS_T ~ N(0, 0.1^2) fp32, deterministic, and drawn from
    seeds no forward tensor of any workload uses."""
    w = di.WORKLOADS["gdn_prefill"].scaled(B=2, T=512, H=4)
    g1, g2 = di.make_bwd_inputs(w), di.make_bwd_inputs(w)
    assert g1["dO"].dtype == np.uint16 and g1["dO"].shape == (2, 512, 4, 128)
    assert g1["dS_T"].dtype == np.float32 and g1["dS_T"].shape == (2, 4, 128, 128)
    np.testing.assert_array_equal(g1["dO"], g2["dO"])
    np.testing.assert_array_equal(g1["dS_T"], g2["dS_T"])
    dO = di.to_f64(g1["dO"], "bf16")
    assert abs(dO.mean()) < 0.01 and abs(dO.std() - 1.0) < 0.01
    assert abs(g1["dS_T"].std() - 0.1) < 0.002
    fwd_seeds = {w2.seed(n) for w2 in di.WORKLOADS.values()
                 for n in ("q", "k", "v", "alpha", "beta_k", "beta_v", "key_scale", "S0", "beta", "retention")}
    bwd_seeds = {w2.seed(n) for w2 in di.WORKLOADS.values() for n in ("dO", "dS_T")}
    assert not (fwd_seeds & bwd_seeds)
