"""GPU parity of the small-state kernel (d_k, d_v in {8, 16}; the delta-mem page's 8 x 8 memory)
against the fp64 oracle, through the C ABI: chunked calls with either read-out, per-channel
gates, the delta-mem configuration (pre-update read-out, undecayed residual by mapping), and
decode steps."""
import numpy as np
import pytest

import dn_inputs as di
import gated_linear_attention_dn_b200 as dn
import oracle
from tests.gpu_util import check, dev, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv,readout", [(8, 8, "pre"), (16, 8, "post"), (8, 16, "post"), (16, 16, "pre")])
def test_small_state_chunk(io, dk, dv, readout):
    w = di.WORKLOADS["kda"].scaled(B=2, H=3, T=700, dk=dk, dv=dv, io=io)
    x = di.make_inputs(w)
    xd = to_device(x)
    o, ST = dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                            xd["S0"], readout=readout)
    assert dn.dn_stream_status() == dn.DN_OK
    o_ref, S_ref = oracle.fwd(**x, readout=readout)
    check(o, ST, o_ref, S_ref, io)


def test_delta_mem_eight_by_eight():
    """delta-mem: S_t = lambda S_{t-1} + beta (v - S_{t-1} k) k^T, r_t = S_{t-1} q_t, 8 x 8 states."""
    w = di.WORKLOADS["gdn_fp32_small"].scaled(B=2, H=4, T=1000, dk=8, dv=8)
    x = di.make_inputs(w)
    lam = x["alpha"].astype(np.float32)
    beta = x["beta_k"]
    x.update(beta_k=(beta / lam).astype(np.float32), beta_v=lam)
    xd = to_device(x)
    o, ST = dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], None, None,
                            readout="pre")
    assert dn.dn_stream_status() == dn.DN_OK
    q, k, v = (x[n].astype(np.float64) for n in ("q", "k", "v"))
    reads = np.zeros_like(v)
    S_end = np.zeros((2, 4, 8, 8))
    for b in range(2):
        for h in range(4):
            S = np.zeros((8, 8))  # value-major, as on the page
            for t in range(1000):
                reads[b, t, h] = S @ q[b, t, h]
                S = lam[b, t, h] * S + beta[b, t, h] * np.outer(v[b, t, h] - S @ k[b, t, h], k[b, t, h])
            S_end[b, h] = S.T
    check(o, ST, reads, S_end, "f32")


def test_small_state_decode():
    w = di.WORKLOADS["decode"].scaled(B=6, dk=8, dv=8)
    S = None
    S_ref = None
    for step in range(4):
        x = di.make_inputs(w, step)
        if step == 0:
            S_ref = x["S0"].astype(np.float64)
            S = dev(x["S0"])
        xd = to_device({n: a for n, a in x.items() if n != "S0"})
        o = dn.dn_decode_step(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"], xd["key_scale"],
                              S=S)
        assert dn.dn_stream_status() == dn.DN_OK
        o_ref, S_ref = oracle.fwd(**{n: a for n, a in x.items() if n != "S0"}, S0=S_ref)
        check(o, S, o_ref, S_ref, "bf16")
