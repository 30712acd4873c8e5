"""GPU parity of the pre-update read-out (o_t = S_{t-1}^T q_t, delta-mem page section 2.C) on every
kernel path, against the fp64 oracle with readout="pre", through the C ABI: the fp32 sequential
kernel, the per-token-gate and per-channel-gate tensor-core chunk kernels, and the decode step;
plus the delta-mem update (undecayed residual) through its mapping onto the recurrence."""
import numpy as np
import pytest

import dn_inputs as di
import gated_linear_attention_dn_b200 as dn
import oracle
from tests.gpu_util import check, dev, to_device

pytestmark = pytest.mark.gpu


def _pre(name, **kw):
    w = di.WORKLOADS[name].scaled(**kw)
    x = di.make_inputs(w)
    xd = to_device(x)
    o, ST = dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                            xd["S0"], readout="pre")
    assert dn.dn_stream_status() == dn.DN_OK
    o_ref, S_ref = oracle.fwd(**x, readout="pre")
    check(o, ST, o_ref, S_ref, w.io)


def test_pre_read_fp32_sequential():
    _pre("gdn_fp32_small", T=200)


@pytest.mark.parametrize("T", [1, 65, 500])
def test_pre_read_per_token_chunk(T):
    _pre("gdn_prefill", B=1, H=2, T=T)


@pytest.mark.parametrize("name", ["kda", "fg2_osdn_long"])
def test_pre_read_per_channel_chunk(name):
    _pre(name, B=1, H=2, T=300)


def test_pre_read_decode():
    w = di.WORKLOADS["decode"].scaled(B=4)
    S = None
    S_ref = None
    for step in range(3):
        x = di.make_inputs(w, step)
        if step == 0:
            S_ref = x["S0"].astype(np.float64)
            S = dev(x["S0"])
        xd = to_device({n: a for n, a in x.items() if n != "S0"})
        o = dn.dn_decode_step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                              S=S, readout="pre")
        assert dn.dn_stream_status() == dn.DN_OK
        o_ref, S_ref = oracle.fwd(**{n: a for n, a in x.items() if n != "S0"}, S0=S_ref, readout="pre")
        check(o, S, o_ref, S_ref, "bf16")


def test_delta_mem_mapping_on_the_gpu():
    """delta-mem's S_t = lambda S_{t-1} + beta (v - S_{t-1} k) k^T with r_t = S_{t-1} q_t, run as
    alpha = lambda, beta^k = beta / lambda, beta^v = lambda, readout="pre" (bf16 chunk kernel)."""
    w = di.WORKLOADS["gdn_prefill"].scaled(B=1, H=2, T=400)
    x = di.make_inputs(w)
    lam = np.clip(x["alpha"], 0.5, 1.0).astype(np.float32)
    beta = x["beta_k"]
    x.update(alpha=lam, beta_k=(beta / lam).astype(np.float32), beta_v=lam)
    xd = to_device(x)
    o, ST = dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], None, None,
                            readout="pre")
    assert dn.dn_stream_status() == dn.DN_OK
    # the page's update, value-major, in fp64
    q, k, v = (oracle.widen(x[n]) for n in ("q", "k", "v"))
    reads = np.zeros_like(oracle.widen(x["v"]))
    S_end = np.zeros((1, 2, 128, 128))
    for h in range(2):
        S = np.zeros((128, 128))
        for t in range(400):
            reads[0, t, h] = S @ q[0, t, h]
            S = lam[0, t, h] * S + beta[0, t, h] * np.outer(v[0, t, h] - S @ k[0, t, h], k[0, t, h])
        S_end[0, h] = S.T
    check(o, ST, reads, S_end, "bf16")
