"""Affine state map of a token range, fp64 numpy (two-level chunk scan).

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Per (sequence, head) the recurrence (page "Gated DeltaNet-2：将擦除与写入分开",
section "在两个维度上独立控制") updates the state by

    Sbar = diag(alpha_t) S,   S_t = Sbar - k_t (e_t^T Sbar) + k_t z_t^T,

with e_t = b_t * k_t and z_t = w_t * v_t: an affine function of S_{t-1},
S_t = L_t S_{t-1} + k_t z_t^T with the linear part L_t = (I - k_t e_t^T) diag(alpha_t).
Over a range of tokens the composition is again affine,

    S_end = Phi S_start + Psi,   Phi = L_last ... L_first   (dk x dk),
                                 Psi = the state reached from S_start = 0  (dk x dv),

and maps of consecutive ranges compose as (Phi2, Psi2) o (Phi1, Psi1) =
(Phi2 Phi1, Phi2 Psi1 + Psi2).  This is what a two-level scan over chunk
segments (or over ranks that each hold a range of a long sequence) passes
along: each range's map is computed independently, a short scan of the maps
gives every range its true start state, and each range then runs from there.
The pages train with 64-token chunks (section "词元路径与并行训练"); the
segment maps are derived here from the recurrence.

:func:`state_map` applies the token updates one by one to Phi (starting from
the identity) and to Psi (starting from zero); nothing is blocked or fused.
"""
from __future__ import annotations

import numpy as np


def _seq_slices(T, B, cu_seqlens):
    if cu_seqlens is None:
        return [(n, slice(0, T)) for n in range(B)]
    cu = np.asarray(cu_seqlens)
    return [(n, slice(int(cu[n]), int(cu[n + 1]))) for n in range(len(cu) - 1)]


def state_map(k, v, log_alpha, b, w, cu_seqlens=None):
    """Affine maps of whole sequences.

    k, log_alpha, b: [B, T, H, dk]; v, w: [B, T, H, dv] (any float dtype,
    upcast to fp64); cu_seqlens: None (B dense sequences) or [N + 1] with B = 1.
    Returns (Phi [N, H, dk, dk], Psi [N, H, dk, dv]) in fp64.
    """
    k, v, la, b, w = (np.asarray(a, dtype=np.float64) for a in (k, v, log_alpha, b, w))
    B, T, H, dk = k.shape
    dv = v.shape[-1]
    seqs = _seq_slices(T, B, cu_seqlens)
    N = len(seqs)
    Phi = np.zeros((N, H, dk, dk))
    Psi = np.zeros((N, H, dk, dv))
    for n, s in seqs:
        bi = 0 if cu_seqlens is not None else n
        for h in range(H):
            P = np.eye(dk)
            Q = np.zeros((dk, dv))
            for t in range(s.start, s.stop):
                kt = k[bi, t, h]
                et = b[bi, t, h] * kt
                zt = w[bi, t, h] * v[bi, t, h]
                alpha = np.exp(la[bi, t, h])
                Pb = alpha[:, None] * P                 # diag(alpha) Phi
                Qb = alpha[:, None] * Q                 # diag(alpha) Psi
                P = Pb - np.outer(kt, et @ Pb)          # (I - k e^T) diag(alpha) Phi
                Q = Qb - np.outer(kt, et @ Qb) + np.outer(kt, zt)
            Phi[n, h] = P
            Psi[n, h] = Q
    return Phi, Psi


def compose(first, second):
    """The map of a range followed by the next one: (Phi2 Phi1, Phi2 Psi1 + Psi2)."""
    P1, Q1 = first
    P2, Q2 = second
    return P2 @ P1, P2 @ Q1 + Q2


def apply(m, S):
    """Phi S + Psi (the end state of the range from start state S)."""
    P, Q = m
    return P @ S + Q
