"""Pins for the backward oracle (``oracle/backward.py``), the first step of the
gate-aware backward pass.

The pages give no gradient formulas; the backward oracle differentiates the
token recurrence by hand.  It is pinned here against something other than
itself: central finite differences, in fp64, of the forward oracle (the C
recurrence, itself pinned in ``test_oracle_pins.py``), of the scalar loss
L = sum(O * dO) + sum(hT * dhT) with random dO and dhT.  Every element of
every input (and h0) on a tiny case, a sample of elements on a larger one with
strong decay and several heads, and the packed layout against separate
sequences.  Planted mistakes (a dropped term of the erase path, the chain rule
of the decay, the state the query reads, ...) must fail the check.
"""
import types

import numpy as np
import pytest

import oracle
from oracle import backward as bw_mod
from workloads import make_inputs

NAMES = ("q", "k", "v", "log_alpha", "b", "w")


def _case(B, T, H, dk, dv, seed, decay="mild", lengths=None, erase_range=1.0):
    x = make_inputs(B, T, H, dk, dv, io="f32", seed=seed, decay=decay, h0_std=0.3, lengths=lengths,
                    erase_range=erase_range)
    arrs = {n: getattr(x, n).astype(np.float64) for n in NAMES}
    arrs["h0"] = x.h0.astype(np.float64)
    rng = np.random.default_rng(seed + 500)
    N = x.num_seqs
    dO = rng.standard_normal(x.v.shape)
    dhT = rng.standard_normal((N, H, dk, dv))
    return x, arrs, dO, dhT


def _loss(x, arrs, dO, dhT):
    o, hT = oracle.recurrent(*(arrs[n] for n in NAMES), x.scale, h0=arrs["h0"], cu_seqlens=x.cu_seqlens)
    return float(np.sum(o * dO) + np.sum(hT * dhT))


def _fd_check(x, arrs, dO, dhT, grads, picks, eps=1e-6, rtol=1e-6):
    for name, idxs in picks.items():
        for idx in idxs:
            plus = {n: a.copy() for n, a in arrs.items()}
            minus = {n: a.copy() for n, a in arrs.items()}
            plus[name][idx] += eps
            minus[name][idx] -= eps
            fd = (_loss(x, plus, dO, dhT) - _loss(x, minus, dO, dhT)) / (2 * eps)
            got = grads[name][idx]
            assert abs(got - fd) <= rtol * max(1.0, abs(fd)), (name, idx, got, fd)


def _grads(x, arrs, dO, dhT, module=bw_mod):
    return module.backward(*(arrs[n] for n in NAMES), x.scale, dO, dhT=dhT, h0=arrs["h0"], cu_seqlens=x.cu_seqlens)


def _all_elements(arrs):
    return {n: list(np.ndindex(a.shape)) for n, a in arrs.items()}


def test_backward_matches_finite_differences_every_element():
    x, arrs, dO, dhT = _case(1, 5, 1, 3, 2, seed=81)
    grads = _grads(x, arrs, dO, dhT)
    _fd_check(x, arrs, dO, dhT, grads, _all_elements(arrs))


def test_backward_matches_finite_differences_sampled_strong_decay():
    x, arrs, dO, dhT = _case(2, 24, 2, 6, 5, seed=82, decay="strong")
    grads = _grads(x, arrs, dO, dhT)
    rng = np.random.default_rng(7)
    picks = {n: [tuple(int(rng.integers(s)) for s in a.shape) for _ in range(12)] for n, a in arrs.items()}
    _fd_check(x, arrs, dO, dhT, grads, picks)


def test_backward_matches_finite_differences_widened_erase_range():
    """The erase gate widened to (0, 2) (the gate ablation): the same
    derivative, now through erase factors up to a reflection."""
    x, arrs, dO, dhT = _case(1, 9, 2, 4, 3, seed=85, decay="strong", erase_range=2.0)
    assert arrs["b"].max() > 1.0
    grads = _grads(x, arrs, dO, dhT)
    _fd_check(x, arrs, dO, dhT, grads, _all_elements(arrs))


def test_backward_packed_equals_separate_sequences():
    lengths = [7, 0, 1, 9]
    x, arrs, dO, dhT = _case(1, sum(lengths), 2, 4, 3, seed=83, lengths=lengths)
    packed = _grads(x, arrs, dO, dhT)
    cu = x.cu_seqlens
    for n in range(len(lengths)):
        s = slice(int(cu[n]), int(cu[n + 1]))
        one = bw_mod.backward(*(arrs[m][:, s] for m in NAMES), x.scale, dO[:, s], dhT=dhT[n:n + 1],
                              h0=arrs["h0"][n:n + 1])
        for m in NAMES:
            assert np.array_equal(packed[m][:, s], one[m])
        assert np.array_equal(packed["h0"][n], one["h0"][0])


MUTANTS = {
    "erase path dropped": ("dSbar = dS + np.outer(e, dr)", "dSbar = dS"),
    "direct term dropped": ("dSbar = dS + np.outer(e, dr)", "dSbar = np.outer(e, dr)"),
    "decay chain rule without alpha": ('g["log_alpha"][t] = np.sum(dSbar * S_prev, axis=1) * alpha',
                                       'g["log_alpha"][t] = np.sum(dSbar * S_prev, axis=1)'),
    "decay gradient from the new state": ('g["log_alpha"][t] = np.sum(dSbar * S_prev, axis=1) * alpha',
                                          'g["log_alpha"][t] = np.sum(dSbar * S_t, axis=1) * alpha'),
    "query reads the old state": ('g["q"][t] = scale * (S_t @ dO[t])', 'g["q"][t] = scale * (S_prev @ dO[t])'),
    "write gate and value swapped": ('g["v"][t] = du * w[t]', 'g["v"][t] = du * v[t]'),
    "decay not carried back": ("dS = alpha[:, None] * dSbar", "dS = dSbar"),
    "erase gradient sign": ("\n        dr = -du\n", "\n        dr = du\n"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_finite_differences_catch_mutant(name):
    old, new = MUTANTS[name]
    src = open(bw_mod.__file__).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("backward_mutant")
    exec(compile(src.replace(old, new), "backward_mutant", "exec"), mod.__dict__)
    x, arrs, dO, dhT = _case(1, 5, 1, 3, 2, seed=81)
    grads = _grads(x, arrs, dO, dhT, module=mod)
    with pytest.raises(AssertionError):
        _fd_check(x, arrs, dO, dhT, grads, _all_elements(arrs))


# --- the chunkwise backward against the token backward ------------------------------

def _rel(a, b):
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


@pytest.mark.parametrize("T,chunk,decay,lengths,erase_range", [(23, 8, "mild", None, 1.0),
                                                                (150, 64, "strong", None, 1.0),
                                                                (None, 16, "strong", [40, 0, 1, 33], 1.0),
                                                                (100, 16, "strong", None, 2.0)])
def test_chunk_backward_equals_token_backward(T, chunk, decay, lengths, erase_range):
    from oracle.chunk_backward import backward as chunk_backward
    if lengths is not None:
        T = sum(lengths)
    x, arrs, dO, dhT = _case(1 if lengths else 2, T, 2, 6, 5, seed=84, decay=decay, lengths=lengths,
                             erase_range=erase_range)
    ref = _grads(x, arrs, dO, dhT)
    got = chunk_backward(*(arrs[n] for n in NAMES), x.scale, dO, dhT=dhT, h0=arrs["h0"],
                         cu_seqlens=x.cu_seqlens, chunk=chunk)
    for name in NAMES + ("h0",):
        assert _rel(got[name], ref[name]) <= 1e-9, (name, _rel(got[name], ref[name]))


CHUNK_MUTANTS = {
    "start-state gradient misses the W S0 path": (
        "dS0 = scale * Qt.T @ dO + np.exp(gn)[:, None] * dS1 - W.T @ dU",
        "dS0 = scale * Qt.T @ dO + np.exp(gn)[:, None] * dS1"),
    "pairwise decay not differentiated": ("dg = M.sum(axis=1) - M.sum(axis=0)", "dg = np.zeros_like(g)"),
    "query mask without the diagonal": ("dP = np.where(lower_incl, scale * dO @ U.T, 0.0)",
                                        "dP = np.where(lower_strict, scale * dO @ U.T, 0.0)"),
    "inverse's gradient not transposed": ("dA = np.where(lower_strict, -T.T @ dT @ T.T, 0.0)",
                                          "dA = np.where(lower_strict, -T @ dT @ T, 0.0)"),
}


@pytest.mark.parametrize("name", sorted(CHUNK_MUTANTS))
def test_token_backward_catches_chunk_mutant(name):
    from oracle import chunk_backward as cb_mod
    old, new = CHUNK_MUTANTS[name]
    src = open(cb_mod.__file__).read()
    assert src.count(old) == 1, old
    mod = types.ModuleType("chunk_backward_mutant")
    exec(compile(src.replace(old, new), "chunk_backward_mutant", "exec"), mod.__dict__)
    x, arrs, dO, dhT = _case(2, 23, 2, 6, 5, seed=84)
    ref = _grads(x, arrs, dO, dhT)
    got = mod.backward(*(arrs[n] for n in NAMES), x.scale, dO, dhT=dhT, h0=arrs["h0"], chunk=8)
    assert max(_rel(got[n], ref[n]) for n in NAMES + ("h0",)) > 1e-6
