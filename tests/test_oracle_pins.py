"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix.

None of these compares the oracle with a retyped copy of itself.  They use
  * the reductions the pages name (KDA, Gated DeltaNet, DeltaNet), each checked
    against a separately written scalar-gate oracle;
  * the delta-rule overwrite invariant (with unit keys, alpha = 1 and
    b = w = 1 the state maps k_t exactly to v_t, and a query equal to k_t
    reads scale * v_t from the updated state), and its reflection form at
    the top of the widened erase range (b = 2: a repeated token is the
    identity on the state);
  * closed forms of the degenerate cases b = 0 (decayed linear attention) and
    b = w = 0 (pure decay), written as cumulative sums, not as a loop;
  * an exact rational example with one-hot keys (tests/golden/basis_keys.json);
  * the state size the pages quote (16 heads x 128 x 128 = 262,144 values);
  * sequence splitting through h0/hT, and the chunkwise WY restatement.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle.chunk_wy import chunk_wy
from workloads import make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm((a - b).ravel()) / max(np.linalg.norm(b.ravel()), 1e-300))


def _run(x, **kw):
    return oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.scale, h0=x.h0,
                            cu_seqlens=x.cu_seqlens, **kw)


# --- reductions named on the pages ------------------------------------------------

def test_reduction_to_kda():
    """b = w = beta (one scalar per token-head) gives KDA."""
    x = make_inputs(2, 77, 3, 16, 12, io="f32", seed=11, gates="kda", h0_std=0.3)
    o, hT = _run(x)
    o2, hT2 = oracle.kda(x.q, x.k, x.v, x.log_alpha, x.beta, x.scale, h0=x.h0)
    assert rel(o, o2) < 1e-12 and rel(hT, hT2) < 1e-12


def test_reduction_to_gated_deltanet():
    """b = w = beta and a scalar decay gives Gated DeltaNet."""
    x = make_inputs(2, 77, 3, 16, 12, io="f32", seed=12, gates="gdn", decay="strong", h0_std=0.3)
    o, hT = _run(x)
    o2, hT2 = oracle.gdn(x.q, x.k, x.v, x.log_alpha_scalar, x.beta, x.scale, h0=x.h0)
    assert rel(o, o2) < 1e-12 and rel(hT, hT2) < 1e-12


def test_reduction_to_deltanet():
    """alpha = 1 and b = w = 1 gives plain DeltaNet."""
    x = make_inputs(1, 90, 2, 16, 16, io="f32", seed=13, h0_std=0.3)
    ones_k = np.ones_like(x.b)
    ones_v = np.ones_like(x.w)
    o, hT = oracle.recurrent(x.q, x.k, x.v, np.zeros_like(x.log_alpha), ones_k, ones_v,
                             x.scale, h0=x.h0)
    o2, hT2 = oracle.deltanet(x.q, x.k, x.v, x.scale, h0=x.h0)
    assert rel(o, o2) < 1e-12 and rel(hT, hT2) < 1e-12


def test_scalar_oracles_agree_with_each_other():
    """KDA with a decay equal across channels is Gated DeltaNet; GDN with
    alpha = beta = 1 is DeltaNet.  Ties the three scalar oracles together."""
    x = make_inputs(1, 60, 2, 8, 8, io="f32", seed=14, gates="gdn", h0_std=0.2)
    o1, h1 = oracle.kda(x.q, x.k, x.v, x.log_alpha, x.beta, x.scale, h0=x.h0)
    o2, h2 = oracle.gdn(x.q, x.k, x.v, x.log_alpha_scalar, x.beta, x.scale, h0=x.h0)
    assert rel(o1, o2) < 1e-12 and rel(h1, h2) < 1e-12
    z = np.zeros_like(x.beta)
    o3, h3 = oracle.gdn(x.q, x.k, x.v, z, np.ones_like(x.beta), x.scale, h0=x.h0)
    o4, h4 = oracle.deltanet(x.q, x.k, x.v, x.scale, h0=x.h0)
    assert rel(o3, o4) < 1e-12 and rel(h3, h4) < 1e-12


# --- textbook delta-rule invariant -----------------------------------------------

def test_delta_rule_overwrite_invariant():
    """With unit-norm keys, alpha = 1 and b = w = 1, the update overwrites the
    value stored under k_t: S_t^T k_t = v_t.  With q_t = k_t the output is
    therefore scale * v_t -- which holds only if the query reads the state
    after the update and the correction has the right sign."""
    x = make_inputs(1, 40, 2, 16, 8, io="f32", seed=15, h0_std=0.5)
    k = x.k.astype(np.float64)
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)      # unit norm in fp64
    zeros = np.zeros_like(x.log_alpha)
    ones_k, ones_v = np.ones_like(x.b), np.ones_like(x.w)
    o, hT = oracle.recurrent(k, k, x.v, zeros, ones_k, ones_v, 0.75, h0=x.h0)
    np.testing.assert_allclose(o, 0.75 * x.v.astype(np.float64), rtol=0, atol=1e-12)
    # and the final state maps the last key to the last value
    for h in range(2):
        np.testing.assert_allclose(hT[0, h].T @ k[0, -1, h], x.v[0, -1, h], rtol=0, atol=1e-12)


def test_full_range_erase_repeated_token_is_identity():
    """At the top of the widened erase range (b = 2 in every channel), with
    alpha = 1, w = 1 and a unit key, one token applies the reflection
    I - 2 k k^T to the state and writes k v^T.  The same token twice in a row
    therefore leaves the state as it was, and with q = k the two outputs are
    scale * (v - S^T k) and scale * S^T k, S the state before the pair.  A
    dropped erase, a wrong sign of the correction or a query that reads the
    old state breaks one of the three."""
    x = make_inputs(1, 24, 2, 16, 8, io="f32", seed=16, h0_std=0.5)
    k = x.k.astype(np.float64)
    k = k / np.linalg.norm(k, axis=-1, keepdims=True)
    k[:, 1::2] = k[:, 0::2]                                   # tokens come in identical pairs
    v = x.v.astype(np.float64)
    v[:, 1::2] = v[:, 0::2]
    zeros = np.zeros_like(x.log_alpha, dtype=np.float64)
    twos, ones_v = np.full(x.b.shape, 2.0), np.ones(x.w.shape)
    o, hT = oracle.recurrent(k, k, v, zeros, twos, ones_v, 0.5, h0=x.h0)
    np.testing.assert_allclose(hT, x.h0, rtol=0, atol=1e-12)
    h0 = x.h0[0].astype(np.float64)                           # [H, dk, dv]
    read = np.einsum("hkv,thk->thv", h0, k[0])                # S^T k with S = h0
    np.testing.assert_allclose(o[0, 0::2], 0.5 * (v[0, 0::2] - read[0::2]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(o[0, 1::2], 0.5 * read[1::2], rtol=0, atol=1e-12)


def test_gate_ablation_inputs():
    """The ablation inputs keep the plain call's draws: b scaled into (0, 2),
    or b / w replaced by their channel mean."""
    base = make_inputs(2, 30, 3, 16, 8, io="f32", seed=17)
    wide = make_inputs(2, 30, 3, 16, 8, io="f32", seed=17, erase_range=2.0)
    assert np.array_equal(wide.b, 2.0 * base.b) and np.array_equal(wide.w, base.w)
    assert wide.b.max() < 2.0 and wide.b.min() > 0.0
    me = make_inputs(2, 30, 3, 16, 8, io="f32", seed=17, mean_gate="erase")
    np.testing.assert_allclose(me.b, np.broadcast_to(base.b.mean(-1, keepdims=True), base.b.shape), rtol=1e-6)
    assert np.array_equal(me.w, base.w) and np.array_equal(me.k, base.k)
    mw = make_inputs(2, 30, 3, 16, 8, io="f32", seed=17, mean_gate="write")
    np.testing.assert_allclose(mw.w, np.broadcast_to(base.w.mean(-1, keepdims=True), base.w.shape), rtol=1e-6)
    assert np.array_equal(mw.b, base.b)


# --- closed forms of the degenerate gates --------------------------------------------

def _closed_form_no_erase(x):
    """b = 0: S_t = D_t S_{t-1} + k_t z_t^T, i.e.
    S_t = diag(exp(G_t)) h0 + sum_{s<=t} diag(exp(G_t - G_s)) k_s z_s^T
    with G the cumulative log-decay.  Evaluated directly, O(T^2)."""
    q, k, v, la, w = (np.asarray(a, dtype=np.float64) for a in (x.q, x.k, x.v, x.log_alpha, x.w))
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    h0 = np.zeros((B, H, dk, dv)) if x.h0 is None else x.h0.astype(np.float64)
    G = np.cumsum(la, axis=1)               # [B, T, H, dk]
    z = w * v
    o = np.zeros((B, T, H, dv))
    hT = np.zeros((B, H, dk, dv))
    for bi in range(B):
        for h in range(H):
            for t in range(T):
                S = np.exp(G[bi, t, h])[:, None] * h0[bi, h]
                dec = np.exp(G[bi, t, h][None, :] - G[bi, : t + 1, h])     # [t+1, dk]
                S = S + np.einsum("sc,sj->cj", dec * k[bi, : t + 1, h], z[bi, : t + 1, h])
                o[bi, t, h] = x.scale * S.T @ q[bi, t, h]
            hT[bi, h] = S
    return o, hT


def test_no_erase_is_decayed_linear_attention():
    x = make_inputs(2, 50, 2, 8, 6, io="f32", seed=16, decay="strong", h0_std=0.4)
    b0 = np.zeros_like(x.b)
    o, hT = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, b0, x.w, x.scale, h0=x.h0)
    o2, hT2 = _closed_form_no_erase(x)
    assert rel(o, o2) < 1e-12 and rel(hT, hT2) < 1e-12


def test_no_erase_no_write_is_pure_decay():
    """b = w = 0: S_t = D_t S_{t-1}, so hT = diag(exp(sum lambda)) h0."""
    x = make_inputs(1, 33, 3, 8, 5, io="f32", seed=17, h0_std=1.0)
    z_k, z_v = np.zeros_like(x.b), np.zeros_like(x.w)
    o, hT = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, z_k, z_v, x.scale, h0=x.h0)
    G = np.cumsum(x.log_alpha.astype(np.float64), axis=1)
    exp_hT = np.exp(G[:, -1])[..., None] * x.h0
    np.testing.assert_allclose(hT, exp_hT, rtol=1e-13, atol=1e-15)
    exp_o = x.scale * np.einsum("bthc,bhcj->bthj", x.q * np.exp(G), x.h0.astype(np.float64))
    np.testing.assert_allclose(o, exp_o, rtol=1e-12, atol=1e-15)


# --- exact rational example (one-hot keys) -------------------------------------------

def _basis_expected(spec):
    F = Fraction
    dk, dv = spec["dk"], spec["dv"]
    S = [[F(s) for s in row] for row in spec["h0"]]
    scale = F(spec["scale"])
    outs = []
    for tok in spec["tokens"]:
        i = tok["key_channel"]
        alpha = [F(a) for a in tok["alpha"]]
        b = [F(a) for a in tok["b"]]
        w = [F(a) for a in tok["w"]]
        v = [F(a) for a in tok["v"]]
        q = [F(a) for a in tok["q"]]
        Sbar = [[alpha[m] * S[m][j] for j in range(dv)] for m in range(dk)]
        S = [row[:] for row in Sbar]
        S[i] = [(1 - b[i]) * Sbar[i][j] + w[j] * v[j] for j in range(dv)]
        outs.append([scale * sum(S[m][j] * q[m] for m in range(dk)) for j in range(dv)])
    return outs, S


def test_basis_keys_exact_example():
    with open(os.path.join(GOLDEN, "basis_keys.json")) as f:
        spec = json.load(f)
    dk, dv = spec["dk"], spec["dv"]
    toks = spec["tokens"]
    T = len(toks)
    fl = lambda xs: [float(Fraction(a)) for a in xs]  # noqa: E731
    q = np.array([fl(t["q"]) for t in toks]).reshape(1, T, 1, dk)
    k = np.zeros((1, T, 1, dk))
    for t, tok in enumerate(toks):
        k[0, t, 0, tok["key_channel"]] = 1.0
    la = np.log(np.array([fl(t["alpha"]) for t in toks])).reshape(1, T, 1, dk)
    b = np.array([fl(t["b"]) for t in toks]).reshape(1, T, 1, dk)
    w = np.array([fl(t["w"]) for t in toks]).reshape(1, T, 1, dv)
    v = np.array([fl(t["v"]) for t in toks]).reshape(1, T, 1, dv)
    h0 = np.array([fl(r) for r in spec["h0"]]).reshape(1, 1, dk, dv)
    o, hT = oracle.recurrent(q, k, v, la, b, w, float(Fraction(spec["scale"])), h0=h0)
    outs, S = _basis_expected(spec)
    np.testing.assert_allclose(o[0, :, 0], np.array(outs, dtype=np.float64), rtol=0, atol=1e-13)
    np.testing.assert_allclose(hT[0, 0], np.array(S, dtype=np.float64), rtol=0, atol=1e-13)
    # the chunk restatement must agree as well (chunk smaller than T to cross a boundary)
    o2, hT2 = chunk_wy(q, k, v, la, b, w, float(Fraction(spec["scale"])), h0=h0, chunk=2)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(hT2, hT, rtol=0, atol=1e-13)


# --- sizes, splitting, varlen --------------------------------------------------------

def test_state_size_matches_pages():
    """16 heads with dk = dv = 128 hold 262,144 state values per sequence."""
    x = make_inputs(1, 2, 16, 128, 128, io="f32", seed=18)
    _, hT = _run(x)
    assert hT.shape == (1, 16, 128, 128)
    assert hT[0].size == 262_144


def test_split_through_state_equals_one_run():
    x = make_inputs(1, 100, 2, 8, 8, io="f32", seed=19, h0_std=0.3)
    o, hT = _run(x)
    sl = lambda a, s: None if a is None else a[:, s]  # noqa: E731
    s1, s2 = slice(0, 37), slice(37, 100)
    oa, ha = oracle.recurrent(*(sl(a, s1) for a in (x.q, x.k, x.v, x.log_alpha, x.b, x.w)), x.scale, h0=x.h0)
    ob, hb = oracle.recurrent(*(sl(a, s2) for a in (x.q, x.k, x.v, x.log_alpha, x.b, x.w)), x.scale, h0=ha)
    assert rel(np.concatenate([oa, ob], axis=1), o) < 1e-13
    assert rel(hb, hT) < 1e-13


def test_varlen_equals_separate_sequences():
    lens = [5, 64, 1, 70, 0, 33]
    x = make_inputs(1, sum(lens), 2, 8, 4, io="f32", seed=20, h0_std=0.3, lengths=lens)
    o, hT = _run(x)
    cu = x.cu_seqlens
    for n in range(len(lens)):
        s = slice(cu[n], cu[n + 1])
        on, hn = oracle.recurrent(*(a[:, s] for a in (x.q, x.k, x.v, x.log_alpha, x.b, x.w)),
                                  x.scale, h0=x.h0[n: n + 1])
        assert np.array_equal(on, o[:, s])
        assert np.array_equal(hn[0], hT[n])


def test_thread_count_does_not_change_results():
    x = make_inputs(3, 40, 4, 8, 8, io="f32", seed=21, h0_std=0.3)
    o1, h1 = _run(x, nthreads=1)
    o2, h2 = _run(x, nthreads=5)
    assert np.array_equal(o1, o2) and np.array_equal(h1, h2)


# --- chunkwise WY algebra equals the recurrence ---------------------------------------

@pytest.mark.parametrize("T,chunk,decay", [(150, 64, "mild"), (200, 64, "strong"), (67, 16, "mild"),
                                           (64, 64, "strong"), (1, 64, "mild")])
def test_chunk_wy_equals_recurrence(T, chunk, decay):
    x = make_inputs(1, T, 2, 16, 12, io="f32", seed=22 + T, decay=decay, h0_std=0.5)
    o, hT = _run(x)
    o2, hT2 = chunk_wy(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.scale, h0=x.h0, chunk=chunk)
    assert rel(o2, o) < 1e-10
    assert rel(hT2, hT) < 1e-10


def test_chunk_wy_varlen_and_intermediates():
    lens = [70, 3, 128, 65]
    x = make_inputs(1, sum(lens), 2, 8, 8, io="f32", seed=23, h0_std=0.5, lengths=lens)
    o, hT = _run(x)
    o2, hT2, inter = chunk_wy(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.scale, h0=x.h0,
                              cu_seqlens=x.cu_seqlens, return_intermediates=True)
    assert rel(o2, o) < 1e-10 and rel(hT2, hT) < 1e-10
    assert [r["len"] for r in inter] == [64, 6, 3, 64, 64, 64, 1]
    # the S0-independent factorisation reproduces each chunk's output
    for r in inter:
        s = slice(r["start"], r["start"] + r["len"])
        for h in range(2):
            O = x.scale * (r["Q_eff"][h] @ r["S0"][h] + r["O_part"][h])
            np.testing.assert_allclose(O, o[0, s, h], rtol=1e-10, atol=1e-12)
            S1 = r["gamma_last"][h][:, None] * r["S0"][h] + r["Kbar"][h].T @ (r["Ut"][h] - r["W"][h] @ r["S0"][h])
            assert np.all(np.isfinite(S1))
    # T really is the inverse of I + A (unit lower triangular)
    for r in inter:
        for h in range(2):
            n = r["len"]
            np.testing.assert_allclose((np.eye(n) + r["A"][h]) @ r["T"][h], np.eye(n), atol=1e-12)
            assert np.allclose(np.triu(r["T"][h], 1), 0) and np.allclose(np.diag(r["T"][h]), 1)


def test_recurrent_step_is_one_token():
    from workloads import decode_inputs
    d = decode_inputs(B=3, H=2, dk=8, dv=6, io="f32", seed=5, state_std=0.5)
    o, S = oracle.recurrent_step(d.q, d.k, d.v, d.log_alpha, d.b, d.w, d.scale, d.state)
    for bi in range(3):
        ob, hb = oracle.recurrent(d.q[bi][None, None], d.k[bi][None, None], d.v[bi][None, None],
                                  d.log_alpha[bi][None, None], d.b[bi][None, None], d.w[bi][None, None],
                                  d.scale, h0=d.state[bi][None])
        assert np.array_equal(ob[0, 0], o[bi]) and np.array_equal(hb[0], S[bi])
