"""Gradients of the Gated DeltaNet-2 forward operator, fp64 numpy.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages train models with this operator (page "Gated DeltaNet-2：将擦除与写入分开",
section "词元路径与并行训练") but print no gradient formulas.  The plain
definition of the backward pass is reverse-mode differentiation of the token
recurrence (same page, section "在两个维度上独立控制"), written out here step by
step, per (sequence, head), in the order opposite to the forward.

Forward at token t (S_{t-1} -> S_t):

    alpha = exp(log_alpha_t)
    Sbar  = diag(alpha) S_{t-1}
    e     = b_t * k_t,   z = w_t * v_t
    r     = Sbar^T e
    u     = z - r
    S_t   = Sbar + k_t u^T
    o_t   = scale * S_t^T q_t          (the query reads the updated state)

Backward at token t, with dS the gradient reaching S_t from the later tokens
(and from hT) and dO_t the gradient of o_t:

    dS    += scale * q_t dO_t^T         (o_t reads S_t)
    dq_t   = scale * S_t dO_t
    dk_t   = dS u                        (S_t = Sbar + k_t u^T)
    du     = dS^T k_t
    dz     = du,   dr = -du
    dSbar  = dS + e dr^T                 (the direct term, and r = Sbar^T e)
    de     = Sbar dr
    db_t   = de * k_t,   dk_t += de * b_t
    dw_t   = dz * v_t,   dv_t  = dz * w_t
    dalpha = rowsum(dSbar * S_{t-1})     (Sbar = diag(alpha) S_{t-1})
    dlog_alpha_t = dalpha * alpha
    dS     = diag(alpha) dSbar           (what reaches S_{t-1})

and dh0 is dS after token 1.  Plain loops over tokens with numpy products:
for small cases only.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    return None if x is None else np.asarray(x, dtype=np.float64)


def _seq_one(q, k, v, la, b, w, scale, dO, dhT, h0):
    """One (sequence, head): inputs [T, d]; returns the gradients."""
    T, dk = q.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if h0 is None else h0.copy()
    states = [S]
    for t in range(T):
        alpha = np.exp(la[t])
        Sbar = alpha[:, None] * S
        e = b[t] * k[t]
        r = Sbar.T @ e
        S = Sbar + np.outer(k[t], w[t] * v[t] - r)
        states.append(S)
    g = {n: np.zeros_like(x) for n, x in (("q", q), ("k", k), ("v", v), ("log_alpha", la), ("b", b), ("w", w))}
    dS = np.zeros((dk, dv)) if dhT is None else dhT.copy()
    for t in range(T - 1, -1, -1):
        S_prev, S_t = states[t], states[t + 1]
        alpha = np.exp(la[t])
        Sbar = alpha[:, None] * S_prev
        e = b[t] * k[t]
        z = w[t] * v[t]
        u = z - Sbar.T @ e
        dS = dS + scale * np.outer(q[t], dO[t])
        g["q"][t] = scale * (S_t @ dO[t])
        dk_t = dS @ u
        du = dS.T @ k[t]
        dr = -du
        dSbar = dS + np.outer(e, dr)
        de = Sbar @ dr
        g["b"][t] = de * k[t]
        g["k"][t] = dk_t + de * b[t]
        g["w"][t] = du * v[t]
        g["v"][t] = du * w[t]
        g["log_alpha"][t] = np.sum(dSbar * S_prev, axis=1) * alpha
        dS = alpha[:, None] * dSbar
    g["h0"] = dS
    return g


def backward(q, k, v, log_alpha, b, w, scale, dO, dhT=None, h0=None, cu_seqlens=None):
    """Gradients of the forward operator's outputs (O [B, T, H, dv] and hT
    [N, H, dk, dv]) contracted with dO and dhT, with respect to every input.

    Layout as the forward: ``[B, T, H, d]``, or ``[1, T_total, H, d]`` with
    ``cu_seqlens``; dhT and h0 ``[N, H, dk, dv]`` (None: zero).  Returns a dict
    of fp64 arrays: q, k, v, log_alpha, b, w (input shapes) and h0
    ``[N, H, dk, dv]``.
    """
    q, k, v, la, b, w, dO = (_f64(x) for x in (q, k, v, log_alpha, b, w, dO))
    dhT, h0 = _f64(dhT), _f64(h0)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        spans = [(n, slice(None)) for n in range(B)]
        N = B
    else:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        assert B == 1
        N = len(cu) - 1
        spans = [(0, slice(int(cu[n]), int(cu[n + 1]))) for n in range(N)]
    out = {n: np.zeros_like(x) for n, x in (("q", q), ("k", k), ("v", v), ("log_alpha", la), ("b", b), ("w", w))}
    out["h0"] = np.zeros((N, H, dk, dv))
    for n, (bi, sl) in enumerate(spans):
        for h in range(H):
            pick = lambda x: x[bi, sl, h]  # noqa: E731
            g = _seq_one(pick(q), pick(k), pick(v), pick(la), pick(b), pick(w), scale, pick(dO),
                         None if dhT is None else dhT[n, h], None if h0 is None else h0[n, h])
            for name in ("q", "k", "v", "log_alpha", "b", "w"):
                out[name][bi, sl, h] = g[name]
            out["h0"][n, h] = g["h0"]
    return out
