"""The token path around the operator, fp64 numpy.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Page "Gated DeltaNet-2：将擦除与写入分开", section "词元路径与并行训练": the
query and the key each go through a linear projection, a short causal
convolution, SiLU and L2 normalisation; the value through a projection, the
convolution and SiLU; the operator's output then goes through RMS
normalisation, an output gate of its own (not the write gate) and a
projection.  The projections need trained weights and stay outside; this
module is the rest, per token:

    short_conv : y_t[c] = sum_{i=0}^{W-1} wt[c, i] * x_{t-i}[c]   (depthwise,
                 causal inside each sequence: x before the sequence's first
                 token is zero), over the H*d channels of the projection
    silu       : x * sigmoid(x)
    l2norm     : x / sqrt(sum_c x_c^2 + eps) over the d channels of a head
    rmsnorm    : x / sqrt(mean_c x_c^2 + eps) * weight[c] over dv channels
    gate       : rmsnorm(o) * sigmoid(g), g the output-gate projection

The pages do not print the convolution width, the epsilons or the gate's
activation; the readings taken are W = 4 (any W works here), eps = 1e-6 for
both norms, and a sigmoid gate like the erase and write gates.
"""
from __future__ import annotations

import numpy as np

EPS = 1e-6


def _seqs(B, T, cu_seqlens):
    if cu_seqlens is None:
        return [(n, 0, T) for n in range(B)]
    cu = np.asarray(cu_seqlens)
    return [(0, int(cu[n]), int(cu[n + 1])) for n in range(len(cu) - 1)]


def short_conv(x, weight, cu_seqlens=None):
    """Depthwise causal convolution.  x: [B, T, H, d]; weight: [H * d, W]."""
    x = np.asarray(x, dtype=np.float64)
    B, T, H, d = x.shape
    wt = np.asarray(weight, dtype=np.float64).reshape(H, d, -1)
    W = wt.shape[-1]
    y = np.zeros_like(x)
    for bi, t0, t1 in _seqs(B, T, cu_seqlens):
        for t in range(t0, t1):
            acc = np.zeros((H, d))
            for i in range(W):
                if t - i >= t0:
                    acc += wt[:, :, i] * x[bi, t - i]
            y[bi, t] = acc
    return y


def silu(x):
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def l2norm(x, eps=EPS):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def rmsnorm(x, weight, eps=EPS):
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * np.asarray(weight, dtype=np.float64)


def prologue(q_raw, k_raw, v_raw, wq, wk, wv, cu_seqlens=None):
    """(q, k, v) handed to the operator from the projections' outputs."""
    q = l2norm(silu(short_conv(q_raw, wq, cu_seqlens)))
    k = l2norm(silu(short_conv(k_raw, wk, cu_seqlens)))
    v = silu(short_conv(v_raw, wv, cu_seqlens))
    return q, k, v


def epilogue(o, g, weight):
    """Normalised, gated output (before the output projection).  o, g: [B, T, H, dv]; weight: [dv]."""
    return rmsnorm(o, weight) / (1.0 + np.exp(-np.asarray(g, dtype=np.float64)))
