"""Chunkwise WY restatement of the Gated Delta Rule-2 recurrence, fp64 numpy.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The pages state that training evaluates the recurrence in 64-token chunks in a
WY form, with the cumulative channel-wise decay absorbed into asymmetric erase
factors and an in-chunk triangular solve plus dense matrix products (page
"Gated DeltaNet-2：将擦除与写入分开", section "词元路径与并行训练"; page
"Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention",
arxivlens summary).  They do not print the algebra; it is derived here from
the token recurrence (section "在两个维度上独立控制" of the same page), per
(sequence, head) and chunk with start state S0, positions i = 1..n:

    g_i   = sum_{j<=i} lambda_j                      (in-chunk cumulative log-decay)
    e_i   = b_i * k_i,  z_i = w_i * v_i
    A_ij  = sum_c e_ic k_jc exp(g_ic - g_jc)           (j < i, strictly lower)
    P_ij  = sum_c q_ic k_jc exp(g_ic - g_jc)           (j <= i: the query sees token i)
    T     = (I + A)^-1                                 (unit lower triangular)
    E~_i  = e_i * exp(g_i)        ("erase factor" with the decay absorbed)
    W     = T E~,   U~ = T Z,   U = U~ - W S0          (u_i = z_i - r_i exactly)
    Q~_i  = q_i * exp(g_i)
    O     = scale * (Q~ S0 + P U)
    Kbar_j= k_j * exp(g_n - g_j)
    S1    = diag(exp(g_n)) S0 + Kbar^T U

Unrolling the recurrence inside a chunk gives (I + A) U = Z - E~ S0, which is
what the triangular solve inverts.  Every decay factor is formed pairwise as
exp(g_i - g_j) with j <= i, so no factor exceeds 1 (lambda <= 0).

The GPU path stores per chunk the quantities that do not depend on S0:
W, U~, Kbar, Q_eff = Q~ - P W and O_part = P U~ (so that
O = scale * (Q_eff S0 + O_part)), plus exp(g_n).  :func:`chunk_wy` returns
them (``return_intermediates=True``) for step-by-step parity tests.
"""
from __future__ import annotations

import numpy as np


def _tri_inverse_unit_lower(A: np.ndarray) -> np.ndarray:
    """(I + A)^-1 for strictly lower A, by a library solve against the identity."""
    n = A.shape[0]
    M = np.eye(n) + A
    return np.linalg.solve(M, np.eye(n))


def chunk_step(q, k, v, la, b, w, S0, scale):
    """One chunk of one (sequence, head).  Arrays are [n, d] fp64, S0 [dk, dv].

    Returns a dict with O, S1 and the S0-independent intermediates.
    """
    n = q.shape[0]
    g = np.cumsum(la, axis=0)                           # [n, dk]
    e = b * k
    z = w * v
    diff = g[:, None, :] - g[None, :, :]                # g_i - g_j, [n, n, dk]
    lower_incl = np.tril(np.ones((n, n), dtype=bool))
    # exp only where j <= i (there the exponent is <= 0); elsewhere the factor is 0
    decay = np.where(lower_incl[:, :, None], np.exp(np.where(lower_incl[:, :, None], diff, 0.0)), 0.0)
    A = np.einsum("ic,jc,ijc->ij", e, k, decay)
    A = np.tril(A, -1)
    P = np.einsum("ic,jc,ijc->ij", q, k, decay)
    P = np.tril(P, 0)
    T = _tri_inverse_unit_lower(A)
    gam = np.exp(g)                                     # [n, dk]
    Et = e * gam
    W = T @ Et
    Ut = T @ z
    U = Ut - W @ S0
    Qt = q * gam
    O = scale * (Qt @ S0 + P @ U)
    Kbar = k * np.exp(g[-1][None, :] - g)
    S1 = np.exp(g[-1])[:, None] * S0 + Kbar.T @ U
    return dict(O=O, S1=S1, g=g, A=A, P=P, T=T, W=W, Ut=Ut, U=U, Kbar=Kbar,
                Q_eff=Qt - P @ W, O_part=P @ Ut, gamma_last=np.exp(g[-1]))


def chunk_wy(q, k, v, log_alpha, b, w, scale, h0=None, cu_seqlens=None, chunk=64,
             return_intermediates=False):
    """Chunkwise WY evaluation in fp64.  Same interface as ``oracle.recurrent``.

    Chunks are aligned to each sequence's first token; the last chunk of a
    sequence may be shorter than ``chunk``.  With ``return_intermediates`` the
    third return value is a list, in (sequence, chunk) order, of dicts holding
    the per-chunk quantities for every head (arrays with a leading head axis)
    and the chunk's start state ``S0``.
    """
    f = lambda x: np.asarray(x, dtype=np.float64)  # noqa: E731
    q, k, v, la, b, w = (f(x) for x in (q, k, v, log_alpha, b, w))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if cu_seqlens is None:
        cu = np.arange(B + 1, dtype=np.int64) * T
    else:
        cu = np.asarray(cu_seqlens, dtype=np.int64)
    flat = lambda x: x.reshape(B * T, H, x.shape[-1])  # noqa: E731
    q, k, v, la, b, w = (flat(x) for x in (q, k, v, la, b, w))
    N = len(cu) - 1
    o = np.zeros((B * T, H, dv))
    hT = np.zeros((N, H, dk, dv))
    inter = []
    for s in range(N):
        S = np.zeros((H, dk, dv)) if h0 is None else f(h0).reshape(N, H, dk, dv)[s].copy()
        for c0 in range(int(cu[s]), int(cu[s + 1]), chunk):
            c1 = min(c0 + chunk, int(cu[s + 1]))
            rec = {"seq": s, "start": c0, "len": c1 - c0, "S0": S.copy()} if return_intermediates else None
            per_head = []
            for h in range(H):
                r = chunk_step(q[c0:c1, h], k[c0:c1, h], v[c0:c1, h], la[c0:c1, h],
                               b[c0:c1, h], w[c0:c1, h], S[h], scale)
                o[c0:c1, h] = r["O"]
                S[h] = r["S1"]
                per_head.append(r)
            if return_intermediates:
                for key in ("W", "Ut", "Kbar", "Q_eff", "O_part", "gamma_last", "A", "P", "T", "g"):
                    rec[key] = np.stack([r[key] for r in per_head])
                inter.append(rec)
        hT[s] = S
    o = o.reshape(B, T, H, dv)
    if return_intermediates:
        return o, hT, inter
    return o, hT
