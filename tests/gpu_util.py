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


def per_head_rel_l2(got: np.ndarray, ref: np.ndarray, kind: str) -> np.ndarray:
    """rel-L2 of every head separately. o is [B,T,H,dv] (heads on axes 0 and 2) or, for a stack of
    sampled heads, [NH,T,dv]; a state is [B,H,dk,dv] or [NH,dk,dv]. A head whose reference is zero
    is compared by its absolute L2 norm."""
    if kind == "o" and got.ndim == 4:
        got, ref = np.moveaxis(got, 2, 1), np.moveaxis(ref, 2, 1)  # [B,H,T,dv]
    lead = 2 if got.ndim == 4 else 1
    g = got.reshape(int(np.prod(got.shape[:lead])), -1)
    r = ref.reshape(g.shape)
    num = np.linalg.norm(g - r, axis=1)
    den = np.linalg.norm(r, axis=1)
    return np.where(den > 0, num / np.where(den > 0, den, 1.0), num)


def check(o_gpu, S_gpu, o_ref, S_ref, io):
    """Pooled rel-L2 over the compared tensors, and the same bound on every head on its own (so a bad
    tail chunk of one head cannot hide in the pooled norm)."""
    og, Sg = host_f64(o_gpu), host_f64(S_gpu)
    assert np.isfinite(og).all() and np.isfinite(Sg).all(), "non-finite output"
    eo = oracle.rel_l2(og, o_ref)
    eS = oracle.rel_l2(Sg, S_ref)
    ho = per_head_rel_l2(og, np.asarray(o_ref), "o").max() if og.size else 0.0
    hS = per_head_rel_l2(Sg, np.asarray(S_ref), "S").max()
    tol = TOL[io]
    print(f"[parity] o rel-L2 {eo:.3e} (worst head {ho:.3e}, tol {tol['o']:.0e}), "
          f"S rel-L2 {eS:.3e} (worst head {hS:.3e}, tol {tol['S']:.0e})")
    assert eo <= tol["o"], f"o rel-L2 {eo:.3e} > {tol['o']}"
    assert eS <= tol["S"], f"S_T rel-L2 {eS:.3e} > {tol['S']}"
    assert ho <= tol["o"], f"o rel-L2 of the worst head {ho:.3e} > {tol['o']}"
    assert hS <= tol["S"], f"S_T rel-L2 of the worst head {hS:.3e} > {tol['S']}"
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
