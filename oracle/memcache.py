"""Memory Caching over the gated delta-rule memory, in fp64 (TEST INFRASTRUCTURE ONLY).

Memory Caching page, section 2: the sequence is cut into segments of L tokens; each segment's
memory is updated online by the recurrence and its final state M^(s) is cached; a token of
segment j reads its online memory and the cached memories of the earlier segments, weighted
by gates (section 3: residual memory sums them, g = 1; the gated residual memory weights each
past segment per token). The page's limits fix what "online" means: N = L segments must behave
like global attention, which holds when every segment's memory starts from the initial state
(a one-token segment's memory is then k v^T). So:

  online   o_t^on = the recurrence's read-out within segment j, from S0 (or zero) at its start
  cache    M^(s) = the state after segment s, from S0 (or zero) at its start
  read-out o_t = o_t^on + sum_{s < j} g_{t,s} M^(s)T q_t

Gates g [B,T,H,N] (None: all ones, the residual memory). The online part is oracle.fwd on each
segment; the cache read-out is the sum written out.
"""
from __future__ import annotations

import numpy as np

from . import fwd, widen


def segments(x, L):
    """[B,T,...] -> list of [B,L,...] views (the last segment may be shorter)."""
    if x is None:
        return None
    T = x.shape[1]
    return [x[:, s:s + L] for s in range(0, T, L)]


def mc_fwd(q, k, v, alpha=None, beta_k=None, beta_v=None, key_scale=None, S0=None, seg_len=64, gates=None,
           readout: str = "post"):
    """Returns (o [B,T,H,dv], M [B,N,H,dk,dv]): the read-out with the cache, and the cached memories."""
    T = np.asarray(q).shape[1]
    N = (T + seg_len - 1) // seg_len
    parts = {n: segments(None if a is None else np.asarray(a), seg_len)
             for n, a in dict(q=q, k=k, v=v, alpha=alpha, beta_k=beta_k, beta_v=beta_v,
                              key_scale=key_scale).items()}
    outs, mems = [], []
    for s in range(N):
        args = {n: (None if p is None else p[s]) for n, p in parts.items()}
        o_s, M_s = fwd(**args, S0=S0, readout=readout)
        outs.append(o_s)
        mems.append(M_s)
    o = np.concatenate(outs, axis=1)
    M = np.stack(mems, axis=1)  # [B, N, H, dk, dv]
    qf = widen(q)
    for j in range(1, N):
        t0, t1 = j * seg_len, min(T, (j + 1) * seg_len)
        for s in range(j):
            y = np.einsum("bthk,bhkv->bthv", qf[:, t0:t1], M[:, s])
            if gates is not None:
                y = y * widen(gates)[:, t0:t1, :, s][..., None]
            o[:, t0:t1] += y
    return o, M
