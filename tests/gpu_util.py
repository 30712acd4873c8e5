"""Helpers shared by the GPU tests: move seeded inputs to the device and run the
C ABI through the Python binding."""
import numpy as np
import torch

import gated_linear_attention_dn_b200 as dn
import oracle

TOL = {"f32": {"o": 1e-4, "S": 1e-4}, "bf16": {"o": 2e-2, "S": 1e-3}}


def dev(x, dtype=None):
    if x is None:
        return None
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def to_device(x: dict) -> dict:
    return {n: dev(v) for n, v in x.items()}


def host_f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def run_chunk(xd: dict):
    o, ST = dn.dn_chunk_fwd(xd["q"], xd["k"], xd["v"], xd["alpha"], xd["beta_k"], xd["beta_v"],
                            xd["key_scale"], xd["S0"])
    assert dn.dn_stream_status() == dn.DN_OK
    return o, ST


def check(o_gpu, S_gpu, o_ref, S_ref, io):
    eo = oracle.rel_l2(host_f64(o_gpu), o_ref)
    eS = oracle.rel_l2(host_f64(S_gpu), S_ref)
    tol = TOL[io]
    print(f"[parity] o rel-L2 {eo:.3e} (tol {tol['o']:.0e}), S rel-L2 {eS:.3e} (tol {tol['S']:.0e})")
    assert eo <= tol["o"], f"o rel-L2 {eo:.3e} > {tol['o']}"
    assert eS <= tol["S"], f"S_T rel-L2 {eS:.3e} > {tol['S']}"
    return eo, eS


def sampled_heads(w, n, seed=0):
    r = np.random.default_rng(seed)
    allh = [(b, h) for b in range(w.B) for h in range(w.H)]
    idx = r.choice(len(allh), size=min(n, len(allh)), replace=False)
    heads = [allh[i] for i in sorted(idx)]
    # always include the first and the last head (edges of the grid)
    for e in (allh[0], allh[-1]):
        if e not in heads:
            heads.append(e)
    return heads
