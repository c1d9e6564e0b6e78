"""Seeded synthetic inputs for the Gated DeltaNet-2 forward operator.

This module is shared by the tests, ``bench.py`` and the oracle checks.  It
holds only input generation (random draws and the distribution shaping of the
workloads); none of the operator's arithmetic lives here.

Workloads (token budgets of the pages' throughput figure, page
"Gated DeltaNet-2：将擦除与写入分开", section "消融实验与训练吞吐量", Fig. 2:
2K x 8 and 16K x 1; heads and head sizes from section "实验比较的边界" /
the state-size paragraph: 16 heads, key and value dimension 128):

  0 tiny      B=1, H=2,  T=128,   dk=dv=64,  fp32 I/O
  1 2Kx8      B=8, H=16, T=2048,  dk=dv=128, bf16 I/O, h0 ~ N(0, 0.01^2)
  2 16Kx1     B=1, H=16, T=16384, dk=dv=128, bf16 I/O, strong decay variety, h0 = 0
  3 reduce    B=4, H=16, T=4096,  dk=dv=128, bf16 I/O, (a) b = w = beta per
              (token, head); (b) additionally a scalar decay per (token, head)
  4 varlen    32 sequences, lengths uniform on [256, 8192] excluding multiples
              of 64, packed with cu_seqlens; H=16, dk=dv=128, bf16 I/O, per-
              sequence h0 ~ N(0, 0.01^2); plus a 256-state decode batch.

Distributions (all draws from ``numpy.random.default_rng(seed)``, float32
standard normals, drawn in the order q, k, v, log_alpha, b, w, h0):
  q, k  : N(0,1), then divided by their L2 norm over the head dimension
  v     : N(0,1) (workload 0) or SiLU(N(0,1)) (bf16 workloads)
  log_alpha : -0.1 * softplus(N(0,1))   (mild), or
              -softplus(N(-2, 1.5))     (strong: per-channel decay from ~1 to ~0)
  b, w  : sigmoid(N(0,1)) per (token, head, channel); the ablation variants
          scale b by 2 (erase range [0, 2]) or replace b or w by its channel
          mean (make_inputs: erase_range, mean_gate)
  h0    : N(0, sigma) with sigma the standard deviation (0.01), fp32
"N(mu, s)" is read as mean and standard deviation.  bf16 tensors are rounded
to nearest-even from float32 and returned as float32 arrays holding exactly
representable bf16 values, so the oracle sees the same numbers as the GPU.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    r = (u + bias) & np.uint32(0xFFFF0000)
    return r.view(np.float32)


def _softplus(x):
    return np.logaddexp(np.float32(0.0), x).astype(np.float32)


def _sigmoid(x):
    return (1.0 / (1.0 + np.exp(-x))).astype(np.float32)


def _l2norm(x):
    n = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
    return (x / n).astype(np.float32)


@dataclass
class Inputs:
    """One operator invocation's inputs (numpy, host)."""
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    log_alpha: np.ndarray
    b: np.ndarray
    w: np.ndarray
    scale: float
    io: str                      # "f32" or "bf16": dtype of q, k, v and the output
    h0: Optional[np.ndarray] = None
    cu_seqlens: Optional[np.ndarray] = None
    beta: Optional[np.ndarray] = None             # scalar gate per (token, head)
    log_alpha_scalar: Optional[np.ndarray] = None  # scalar decay per (token, head)
    name: str = ""
    meta: dict = field(default_factory=dict)

    @property
    def shape(self):
        B, T, H, dk = self.q.shape
        return B, T, H, dk, self.v.shape[-1]

    @property
    def num_seqs(self):
        return self.q.shape[0] if self.cu_seqlens is None else len(self.cu_seqlens) - 1

    @property
    def tokens(self):
        B, T = self.q.shape[:2]
        return B * T


def make_inputs(B, T, H, dk, dv, io="bf16", seed=0, decay="mild", gates="channel",
                h0_std=None, lengths=None, v_act=None, erase_range=1.0, mean_gate=None) -> Inputs:
    """General generator.

    ``decay``: "mild" (-0.1*softplus(N(0,1))) or "strong" (-softplus(N(-2,1.5))).
    ``gates``: "channel" (b, w per channel), "kda" (b = w = beta per token-head,
    broadcast over channels), "gdn" (as "kda" and a scalar decay per token-head,
    broadcast over key channels).
    ``lengths``: if given, B must be 1 and T == sum(lengths); sequences are
    packed and ``cu_seqlens`` is set.
    ``v_act``: "silu" or None; defaults to "silu" for bf16 and None for f32.
    ``erase_range``: b = erase_range * sigmoid(N(0,1)) (the ablation widening
    the erase gate's range from [0, 1] to [0, 2] uses 2).
    ``mean_gate``: None, "erase" or "write": the ablation that averages one
    gate (b, the erase gate, or w, the write gate) over its channels at run
    time, broadcast back over them.  Page "Gated DeltaNet-2：将擦除与写入分开",
    section "消融实验与训练吞吐量".  Neither option changes the draws, so the
    other tensors are those of the plain call with the same seed.
    """
    rng = np.random.default_rng(seed)
    shp_k = (B, T, H, dk)
    shp_v = (B, T, H, dv)
    n = lambda s: rng.standard_normal(s, dtype=np.float32)  # noqa: E731
    q = _l2norm(n(shp_k))
    k = _l2norm(n(shp_k))
    v = n(shp_v)
    if v_act is None:
        v_act = "silu" if io == "bf16" else None
    if v_act == "silu":
        v = (v * _sigmoid(v)).astype(np.float32)
    beta = las = None
    if gates == "gdn":
        las_draw = n((B, T, H))
    else:
        la_draw = n(shp_k)
    if decay == "mild":
        f = lambda x: (-0.1 * _softplus(x)).astype(np.float32)  # noqa: E731
    elif decay == "strong":
        f = lambda x: (-_softplus(-2.0 + 1.5 * x)).astype(np.float32)  # noqa: E731
    else:
        raise ValueError(decay)
    if gates == "gdn":
        las = f(las_draw)
        la = np.broadcast_to(las[..., None], shp_k).astype(np.float32)
    else:
        la = f(la_draw)
    if gates == "channel":
        b = _sigmoid(n(shp_k))
        w = _sigmoid(n(shp_v))
    elif gates in ("kda", "gdn"):
        beta = _sigmoid(n((B, T, H)))
        b = np.broadcast_to(beta[..., None], shp_k).astype(np.float32)
        w = np.broadcast_to(beta[..., None], shp_v).astype(np.float32)
    else:
        raise ValueError(gates)
    if erase_range != 1.0:
        b = (np.float32(erase_range) * b).astype(np.float32)
    if mean_gate == "erase":
        b = np.broadcast_to(b.mean(axis=-1, dtype=np.float32)[..., None], shp_k).astype(np.float32)
    elif mean_gate == "write":
        w = np.broadcast_to(w.mean(axis=-1, dtype=np.float32)[..., None], shp_v).astype(np.float32)
    elif mean_gate is not None:
        raise ValueError(mean_gate)
    cu = None
    if lengths is not None:
        assert B == 1 and T == int(np.sum(lengths))
        cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    nseq = B if cu is None else len(cu) - 1
    h0 = None
    if h0_std is not None:
        h0 = (h0_std * n((nseq, H, dk, dv))).astype(np.float32)
    if io == "bf16":
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
    elif io != "f32":
        raise ValueError(io)
    return Inputs(q=q, k=k, v=v, log_alpha=la, b=b, w=w, scale=float(dk) ** -0.5, io=io,
                  h0=h0, cu_seqlens=cu, beta=beta, log_alpha_scalar=las)


def varlen_lengths(rng, count=32, lo=256, hi=8192, multiple=64):
    """Integers uniform on [lo, hi], redrawing multiples of ``multiple``."""
    out = []
    while len(out) < count:
        x = int(rng.integers(lo, hi + 1))
        if x % multiple != 0:
            out.append(x)
    return np.array(out, dtype=np.int64)


def config(i: int, variant: str = "a") -> Inputs:
    """The five named workloads (index as in the module docstring)."""
    if i == 0:
        x = make_inputs(1, 128, 2, 64, 64, io="f32", seed=0, decay="mild")
        x.name = "tiny fp32 B=1 T=128 H=2 d=64"
    elif i == 1:
        x = make_inputs(8, 2048, 16, 128, 128, io="bf16", seed=1, decay="mild", h0_std=0.01)
        x.name = "2Kx8 B=8 T=2048 H=16 d=128 bf16"
    elif i == 2:
        x = make_inputs(1, 16384, 16, 128, 128, io="bf16", seed=2, decay="strong")
        x.name = "16Kx1 B=1 T=16384 H=16 d=128 bf16"
    elif i == 3:
        gates = "kda" if variant == "a" else "gdn"
        x = make_inputs(4, 4096, 16, 128, 128, io="bf16", seed=3, decay="mild", gates=gates)
        x.name = f"reduction-{variant} B=4 T=4096 H=16 d=128 bf16"
    elif i == 4:
        rng = np.random.default_rng(4)
        lens = varlen_lengths(rng)
        x = make_inputs(1, int(lens.sum()), 16, 128, 128, io="bf16", seed=40, decay="mild",
                        h0_std=0.01, lengths=lens)
        x.name = f"varlen 32 seqs T_total={int(lens.sum())} H=16 d=128 bf16"
    else:
        raise ValueError(i)
    return x


@dataclass
class DecodeInputs:
    q: np.ndarray      # [B, H, dk]
    k: np.ndarray
    v: np.ndarray      # [B, H, dv]
    log_alpha: np.ndarray
    b: np.ndarray
    w: np.ndarray
    state: np.ndarray  # [B, H, dk, dv] fp32
    scale: float
    io: str


def decode_inputs(B=256, H=16, dk=128, dv=128, io="bf16", seed=41, state_std=0.01, **gate_kw) -> DecodeInputs:
    """Single-token decode batch: one token per state, same distributions as
    above (``gate_kw``: make_inputs' erase_range / mean_gate)."""
    x = make_inputs(B, 1, H, dk, dv, io=io, seed=seed, decay="mild", **gate_kw)
    rng = np.random.default_rng(seed + 1000)
    state = (state_std * rng.standard_normal((B, H, dk, dv), dtype=np.float32)).astype(np.float32)
    sq = lambda a: np.ascontiguousarray(a[:, 0])  # noqa: E731
    return DecodeInputs(q=sq(x.q), k=sq(x.k), v=sq(x.v), log_alpha=sq(x.log_alpha), b=sq(x.b),
                        w=sq(x.w), state=state, scale=x.scale, io=io)
