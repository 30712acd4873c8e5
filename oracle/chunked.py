"""Chunkwise-parallel (WY / UT-transform) evaluation of the gated delta rule, NumPy fp64.

TEST INFRASTRUCTURE ONLY. This is not the oracle the GPU is compared against;
it shows, on small inputs, that the chunk algebra reproduces the sequential
definition (``oracle.fwd``). The pages name the chunk-parallel scheme (FG2-GDN
page, section 2.A: the rank-1 structure that the WY representation needs, and
section 3 item 2: the diagonal-plus-low-rank structure reused by KDA's chunk
algorithm; OSDN page, section 2.1: only K -> K~ changes in the block Gram matrix
and the intra-block scores) but print no formulas for it; the algebra below is
derived from the recurrence.

Within one chunk of n tokens (t = 1..n), with start state S and per-key-channel
log-decay prefix g_t = sum_{s<=t} log alpha_s (g_0 = 0), pick a reference point
m in {0..n} and write e(x) = exp(x) elementwise:

  K+_t = k_t (.) e(g_t - g_m)          Q+_t = q_t (.) e(g_t - g_m)
  W-_t = w_t (.) e(g_m - g_t)          V~_t = beta^v_t (.) v_t,  w_t = beta^k_t (.) d_t (.) k_t
  S_m  = Diag(e(g_m)) S                (state decayed to the reference point)
  L    = strictly-lower(K+ W-^T)       T = (I + L)^{-1}       (the UT transform)
  U    = T (V~ - K+ S_m)               (all residuals u_t of the chunk)
  O    = Q+ S_m + lower-incl(Q+ W-^T) U
  S'   = Diag(e(g_n - g_m)) (S_m + W-^T U)

m = 0 is the chunk-start reference; m = n // 2 (the midpoint) keeps every
exponent within half a chunk of decay, which is the form the kernels use.
"""
from __future__ import annotations

import numpy as np


def _gate(x, t0, t1, width):
    """Gate values for tokens [t0, t1) of one head, broadcast to [n, width]."""
    if x is None:
        return np.ones((t1 - t0, width))
    x = np.asarray(x, dtype=np.float64)
    if x.ndim == 1:
        return np.repeat(x[t0:t1, None], width, axis=1)
    return x[t0:t1]


def head_fwd(q, k, v, alpha, beta_k, beta_v, key_scale, S, C: int, ref: str = "mid"):
    """One head. q, k [T,dk]; v [T,dv]; gates [T] or [T,n] or None; S [dk,dv] (copied).

    Returns (o [T,dv], S_T [dk,dv]).
    """
    T, dk = q.shape
    dv = v.shape[1]
    S = np.array(S, dtype=np.float64, copy=True)
    o = np.zeros((T, dv))
    for c0 in range(0, T, C):
        c1 = min(T, c0 + C)
        n = c1 - c0
        a = _gate(alpha, c0, c1, dk)
        g = np.concatenate([np.zeros((1, dk)), np.cumsum(np.log(a), axis=0)])  # g[0..n]
        m = n // 2 if ref == "mid" else 0
        gt = g[1:]                                                              # g_t, t = 1..n
        w = _gate(beta_k, c0, c1, dk) * _gate(key_scale, c0, c1, dk) * k[c0:c1]
        Kp = k[c0:c1] * np.exp(gt - g[m])
        Qp = q[c0:c1] * np.exp(gt - g[m])
        Wm = w * np.exp(g[m] - gt)
        Vt = _gate(beta_v, c0, c1, dv) * v[c0:c1]
        Sm = np.exp(g[m])[:, None] * S
        L = np.tril(Kp @ Wm.T, k=-1)
        Tm = np.linalg.inv(np.eye(n) + L)
        U = Tm @ (Vt - Kp @ Sm)
        P = np.tril(Qp @ Wm.T)
        o[c0:c1] = Qp @ Sm + P @ U
        S = np.exp(g[n] - g[m])[:, None] * (Sm + Wm.T @ U)
    return o, S


def fwd(q, k, v, alpha=None, beta_k=None, beta_v=None, key_scale=None, S0=None, C: int = 64,
        ref: str = "mid"):
    """All heads, public layouts (q [B,T,H,dk] ...), fp64 inputs. Returns (o, S_T)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    ST = np.zeros((B, H, dk, dv))

    def sl(x, b, h):
        if x is None:
            return None
        x = np.asarray(x, dtype=np.float64)
        return x[b, :, h] if x.ndim == 3 else x[b, :, h, :]

    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.asarray(S0, dtype=np.float64)[b, h]
            ob, Sb = head_fwd(q[b, :, h], k[b, :, h], v[b, :, h], sl(alpha, b, h), sl(beta_k, b, h),
                              sl(beta_v, b, h), sl(key_scale, b, h), S, C, ref)
            o[b, :, h] = ob
            ST[b, h] = Sb
    return o, ST


def head_bwd(q, k, v, alpha, beta_k, beta_v, key_scale, S, dO, dS_T, C: int, readout: str = "post"):
    """Reverse mode of the chunk algebra, either read-out.

    The chain rule through the chunk equations gives, with dS' the adjoint of the chunk-end state
    and lam = e(g_n - g_m):
      dX  = Diag(lam) dS'                          (adjoint of X = S_m + W-^T U)
      dU  = lower-incl(Q+ W-^T)^T dO + W- dX
      dV~ = T^T dU                                  (adjoint of V~ - K+ S_m, as U = T (V~ - K+ S_m))
      dS_m = Q+^T dO + dX - K+^T dV~,    dS = Diag(e(g_m)) dS_m
      dP  = lower-incl(dO U^T),          dL = -strictly-lower(dV~ U^T)
      dQ+ = dO S_m^T + dP W-,    dK+ = -dV~ S_m^T + dL W-,    dW- = U dX^T + dP^T Q+ + dL^T K+
    (dL uses T^T dT T^T with dT = dU ((I + L) U)^T, so T^T dT T^T = dV~ U^T.) The outputs do not
    depend on the reference point g_m, so its adjoint terms cancel and g_m is held fixed: the
    log-decay adjoint of token t is dh_t = Q+ (.) dQ+ + K+ (.) dK+ - W- (.) dW- (every channel), plus
    rowsum(dX (.) X) at the chunk's last token, and d log alpha_s is the sum over t >= s in the chunk.
    The pre read-out o_t = S_{t-1}^T q_t reads the state before token t's decay: Q+_t = q_t (.) e(h_t)
    / alpha_t and P = strictly-lower(Q+ W-^T), so dP is strictly lower, dq = e(h) / alpha (.) dQ+, and
    d log alpha_t also gets -Q+_t (.) dQ+_t, token t's own term (not summed over later tokens).

    Returns a dict of per-token gradients shaped [T, n] for every gate (channel form) and
    dS0 [dk, dv].
    """
    T, dk = q.shape
    dv = v.shape[1]
    S = np.array(S, dtype=np.float64, copy=True)
    nc = (T + C - 1) // C
    keep = []
    for c in range(nc):  # forward, keeping what the reverse needs
        c0, c1 = c * C, min(T, c * C + C)
        n = c1 - c0
        a = _gate(alpha, c0, c1, dk)
        g = np.cumsum(np.log(a), axis=0)                  # g_t, t = 0..n-1 (after token t)
        r = g[(n - 1) // 2]                               # the reference point, held fixed
        eh = np.exp(g - r)
        bkd = _gate(beta_k, c0, c1, dk) * _gate(key_scale, c0, c1, dk)
        w = bkd * k[c0:c1]
        eq = eh / a if readout == "pre" else eh   # the pre read-out stops the decay one token earlier
        Kp, Qp, Wm = k[c0:c1] * eh, q[c0:c1] * eq, w / eh
        Vt = _gate(beta_v, c0, c1, dv) * v[c0:c1]
        Sm = np.exp(r)[:, None] * S
        Tm = np.linalg.inv(np.eye(n) + np.tril(Kp @ Wm.T, k=-1))
        U = Tm @ (Vt - Kp @ Sm)
        X = Sm + Wm.T @ U
        lam = np.exp(g[-1] - r)
        keep.append((c0, c1, a, eh, eq, bkd, Kp, Qp, Wm, Tm, U, Sm, X, lam, r))
        S = lam[:, None] * X
    out = {n: np.zeros((T, w)) for n, w in (("q", dk), ("k", dk), ("v", dv), ("alpha", dk),
                                               ("beta_k", dk), ("beta_v", dv), ("key_scale", dk))}
    dS = np.zeros((dk, dv)) if dS_T is None else np.array(dS_T, dtype=np.float64)
    for c in reversed(range(nc)):
        c0, c1, a, eh, eq, bkd, Kp, Qp, Wm, Tm, U, Sm, X, lam, r = keep[c]
        dOc = dO[c0:c1]
        dX = lam[:, None] * dS
        diag = -1 if readout == "pre" else 0
        P = np.tril(Qp @ Wm.T, k=diag)
        dU = P.T @ dOc + Wm @ dX
        dVt = Tm.T @ dU
        dS = np.exp(r)[:, None] * (Qp.T @ dOc + dX - Kp.T @ dVt)
        dP = np.tril(dOc @ U.T, k=diag)
        dL = -np.tril(dVt @ U.T, k=-1)
        dQp = dOc @ Sm.T + dP @ Wm
        dKp = -dVt @ Sm.T + dL @ Wm
        dWm = U @ dX.T + dP.T @ Qp + dL.T @ Kp
        dh = Qp * dQp + Kp * dKp - Wm * dWm
        dh[-1] += np.sum(dX * X, axis=1)
        dlog = np.cumsum(dh[::-1], axis=0)[::-1]
        if readout == "pre":
            dlog = dlog - Qp * dQp
        dw = dWm / eh
        kc, vc = k[c0:c1], v[c0:c1]
        out["q"][c0:c1] = dQp * eq
        out["k"][c0:c1] = dKp * eh + bkd * dw
        out["alpha"][c0:c1] = dlog / a
        out["beta_k"][c0:c1] = _gate(key_scale, c0, c1, dk) * kc * dw
        out["key_scale"][c0:c1] = _gate(beta_k, c0, c1, dk) * kc * dw
        out["v"][c0:c1] = _gate(beta_v, c0, c1, dv) * dVt
        out["beta_v"][c0:c1] = vc * dVt
    out["S0"] = dS
    return out


def bwd(q, k, v, alpha=None, beta_k=None, beta_v=None, key_scale=None, S0=None, dO=None, dS_T=None,
        C: int = 64, readout: str = "post"):
    """All heads, public layouts: the gradients as ``oracle.bwd`` returns them."""
    q = np.asarray(q, dtype=np.float64)
    B, T, H, dk = q.shape
    dv = np.asarray(v).shape[-1]

    def sl(x, b, h):
        if x is None:
            return None
        x = np.asarray(x, dtype=np.float64)
        return x[b, :, h] if x.ndim == 3 else x[b, :, h, :]

    gates = dict(alpha=alpha, beta_k=beta_k, beta_v=beta_v, key_scale=key_scale)
    res = {"q": np.zeros((B, T, H, dk)), "k": np.zeros((B, T, H, dk)), "v": np.zeros((B, T, H, dv)),
           "S0": np.zeros((B, H, dk, dv))}
    for n, x in gates.items():
        res[n] = None if x is None else np.zeros(np.shape(x))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.asarray(S0, dtype=np.float64)[b, h]
            g = head_bwd(q[b, :, h], np.asarray(k, dtype=np.float64)[b, :, h],
                         np.asarray(v, dtype=np.float64)[b, :, h], *(sl(gates[n], b, h) for n in gates), S,
                         np.asarray(dO, dtype=np.float64)[b, :, h],
                         None if dS_T is None else np.asarray(dS_T, dtype=np.float64)[b, h], C, readout)
            for n in ("q", "k", "v"):
                res[n][b, :, h] = g[n]
            res["S0"][b, h] = g["S0"]
            for n, x in gates.items():
                if x is None:
                    continue
                gn = g[n]
                res[n][b, :, h] = gn.sum(axis=1) if np.ndim(x) == 3 else gn
    return res
