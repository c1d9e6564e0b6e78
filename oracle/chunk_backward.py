"""Chunkwise backward of the Gated DeltaNet-2 forward operator, fp64 numpy.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The backward of the 64-token chunk form (``oracle/chunk_wy.py``), the algebra
a GPU backward over chunks evaluates: per (sequence, head) the forward states
at the chunk boundaries are recomputed, then the chunks are taken in reverse
order, each turning the gradient of its end state (dS1) and of its outputs
(dO) into the gradients of its inputs and of its start state (dS0).  It is
checked against ``oracle/backward.py``, the token-by-token reverse mode, which
finite differences of the forward recurrence pin.

Per chunk of n tokens (notation of ``chunk_wy``; D_ij^c = exp(g_ic - g_jc)
for j <= i, masks as in the forward):

    dQ~  = scale dO S0^T                 dP  = scale dO U^T   (j <= i)
    dU   = scale P^T dO + Kbar dS1       dKbar = U dS1^T
    dS0  = scale Q~^T dO + diag(gamma_n) dS1 - W^T dU
    dW   = -dU S0^T                      dU~ = dU
    dT   = dU~ Z^T + dW E~^T             dZ  = T^T dU~,   dE~ = T^T dW
    dA   = -T^T dT T^T  (j < i)          (T = (I + A)^-1)
    dE_ic += sum_j dA_ij K_jc D_ij^c
    dK_jc += sum_i (dA_ij E_ic + dP_ij Q_ic) D_ij^c
    dQ_ic += sum_j dP_ij K_jc D_ij^c
    dg_ic += sum_j M_ij^c,  dg_jc -= sum_i M_ij^c,
             M_ij^c = (dA_ij E_ic + dP_ij Q_ic) K_jc D_ij^c
    E~ = E gamma, Q~ = Q gamma, Kbar = K exp(g_n - g), gamma = exp(g),
    S1 = diag(gamma_n) S0 + ...: the chain rule through each scale, with
    g_n the last row of g
    E = b K, Z = w V;  g = cumsum(log_alpha): dlog_alpha = reverse cumsum of dg.
"""
from __future__ import annotations

import numpy as np

from oracle.chunk_wy import chunk_step


def chunk_step_backward(q, k, v, la, b, w, S0, scale, dO, dS1):
    """Gradients of one chunk (arrays [n, d] fp64, S0 and dS1 [dk, dv]).

    Returns a dict: q, k, v, log_alpha, b, w ([n, d]) and S0 ([dk, dv]).
    """
    n = q.shape[0]
    f = chunk_step(q, k, v, la, b, w, S0, scale)
    g, A, P, T, W, U = f["g"], f["A"], f["P"], f["T"], f["W"], f["U"]
    e = b * k
    z = w * v
    gam = np.exp(g)
    gn = g[-1]
    Et = e * gam
    Qt = q * gam
    kscale = np.exp(gn[None, :] - g)
    Kbar = k * kscale
    lower_incl = np.tril(np.ones((n, n), dtype=bool))
    lower_strict = np.tril(np.ones((n, n), dtype=bool), -1)
    diff = g[:, None, :] - g[None, :, :]
    D = np.where(lower_incl[:, :, None], np.exp(np.where(lower_incl[:, :, None], diff, 0.0)), 0.0)

    dQt = scale * dO @ S0.T
    dP = np.where(lower_incl, scale * dO @ U.T, 0.0)
    dU = scale * P.T @ dO + Kbar @ dS1
    dKbar = U @ dS1.T
    dS0 = scale * Qt.T @ dO + np.exp(gn)[:, None] * dS1 - W.T @ dU
    dgn = np.sum(dS1 * S0, axis=1) * np.exp(gn)       # S1 = diag(exp(g_n)) S0 + ...
    dW = -dU @ S0.T
    dT = dU @ z.T + dW @ Et.T
    dz = T.T @ dU
    dEt = T.T @ dW
    dA = np.where(lower_strict, -T.T @ dT @ T.T, 0.0)

    # through the pairwise-decayed products A and P
    dE = np.einsum("ij,jc,ijc->ic", dA, k, D)
    dK = np.einsum("ij,ic,ijc->jc", dA, e, D) + np.einsum("ij,ic,ijc->jc", dP, q, D)
    dQ = np.einsum("ij,jc,ijc->ic", dP, k, D)
    M = (dA[:, :, None] * e[:, None, :] + dP[:, :, None] * q[:, None, :]) * k[None, :, :] * D
    dg = M.sum(axis=1) - M.sum(axis=0)
    # through the per-channel scales
    dE += dEt * gam
    dQ += dQt * gam
    dg += (dEt * e + dQt * q) * gam
    dK += dKbar * kscale
    t = dKbar * k * kscale                               # Kbar = K exp(g_n - g)
    dg -= t
    dgn = dgn + t.sum(axis=0)
    dg[-1] += dgn
    # gates, and the cumulative sum
    db = dE * k
    dK += dE * b
    dw = dz * v
    dv = dz * w
    dla = np.cumsum(dg[::-1], axis=0)[::-1]
    return dict(q=dQ, k=dK, v=dv, log_alpha=dla, b=db, w=dw, S0=dS0)


def backward(q, k, v, log_alpha, b, w, scale, dO, dhT=None, h0=None, cu_seqlens=None, chunk=64):
    """Same interface and result as ``oracle.backward.backward``, evaluated
    chunk by chunk."""
    f64 = lambda x: None if x is None else np.asarray(x, dtype=np.float64)  # noqa: E731
    q, k, v, la, b, w, dO = (f64(x) for x in (q, k, v, log_alpha, b, w, dO))
    dhT, h0 = f64(dhT), f64(h0)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        spans = [(n, 0, T) for n in range(B)]
    else:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
        assert B == 1
        spans = [(0, int(cu[n]), int(cu[n + 1])) for n in range(len(cu) - 1)]
    N = len(spans)
    out = {n: np.zeros_like(x) for n, x in (("q", q), ("k", k), ("v", v), ("log_alpha", la), ("b", b), ("w", w))}
    out["h0"] = np.zeros((N, H, dk, dv))
    for n, (bi, t0, t1) in enumerate(spans):
        for h in range(H):
            sl = lambda x, a, c: x[bi, a:c, h]  # noqa: E731
            bounds = [(c0, min(c0 + chunk, t1)) for c0 in range(t0, t1, chunk)]
            # forward: the start state of every chunk
            S = np.zeros((dk, dv)) if h0 is None else h0[n, h].copy()
            starts = []
            for c0, c1 in bounds:
                starts.append(S)
                S = chunk_step(sl(q, c0, c1), sl(k, c0, c1), sl(v, c0, c1), sl(la, c0, c1), sl(b, c0, c1),
                               sl(w, c0, c1), S, scale)["S1"]
            # backward over the chunks in reverse order
            dS = np.zeros((dk, dv)) if dhT is None else dhT[n, h].copy()
            for (c0, c1), S0 in zip(reversed(bounds), reversed(starts)):
                r = chunk_step_backward(sl(q, c0, c1), sl(k, c0, c1), sl(v, c0, c1), sl(la, c0, c1),
                                        sl(b, c0, c1), sl(w, c0, c1), S0, scale, sl(dO, c0, c1), dS)
                for name in ("q", "k", "v", "log_alpha", "b", "w"):
                    out[name][bi, c0:c1, h] = r[name]
                dS = r["S0"]
            out["h0"][n, h] = dS
    return out
