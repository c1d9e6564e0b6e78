"""Pins of the state-map oracle (oracle/state_map.py), no GPU.

The map (Phi, Psi) of a token range must satisfy, whatever the inputs:
  * Phi h0 + Psi equals the final state of the token recurrence (the C
    oracle, separately written) started from h0, for any h0;
  * consecutive ranges compose: map([0, T)) = map([T1, T)) o map([0, T1));
  * b = 0 (nothing erased): Phi = diag(exp(sum of log_alpha)) and
    Psi = sum_t diag(exp(sum_{t' > t} log_alpha_t')) k_t z_t^T, closed forms;
  * alpha = 1, b = w = 1 and unit keys (plain DeltaNet): the last token's key
    is overwritten, k_T^T Phi = 0 and k_T^T Psi = v_T (the delta-rule
    invariant);
  * an empty range is the identity map.
A planted mistake in the oracle (sign of the erase, decay on the wrong side,
write gate dropped) fails one of these.
"""
import numpy as np
import pytest

import oracle
from oracle import state_map as sm
from workloads import make_inputs


def _inputs(T, seed, **kw):
    return make_inputs(1, T, 2, 8, 6, io="f32", seed=seed, decay="strong", h0_std=0.3, **kw)


def test_map_applied_to_h0_equals_recurrence():
    x = _inputs(37, 1)
    Phi, Psi = sm.state_map(x.k, x.v, x.log_alpha, x.b, x.w)
    _, hT = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.scale, h0=x.h0)
    got = np.einsum("nhij,nhjv->nhiv", Phi, x.h0.astype(np.float64)) + Psi
    np.testing.assert_allclose(got, hT, rtol=1e-11, atol=1e-12)


def test_packed_sequences_each_get_their_own_map():
    lengths = [5, 0, 19, 1]
    x = make_inputs(1, sum(lengths), 2, 8, 6, io="f32", seed=2, h0_std=0.3, lengths=lengths)
    Phi, Psi = sm.state_map(x.k, x.v, x.log_alpha, x.b, x.w, cu_seqlens=x.cu_seqlens)
    _, hT = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.scale, h0=x.h0, cu_seqlens=x.cu_seqlens)
    got = np.einsum("nhij,nhjv->nhiv", Phi, x.h0.astype(np.float64)) + Psi
    np.testing.assert_allclose(got, hT, rtol=1e-11, atol=1e-12)
    # the empty sequence: identity map
    np.testing.assert_array_equal(Phi[1], np.broadcast_to(np.eye(8), (2, 8, 8)))
    np.testing.assert_array_equal(Psi[1], 0.0)


@pytest.mark.parametrize("t1", [1, 16, 36])
def test_consecutive_ranges_compose(t1):
    x = _inputs(37, 3)
    whole = sm.state_map(x.k, x.v, x.log_alpha, x.b, x.w)
    cut = lambda a, s: a[:, s]  # noqa: E731
    first = sm.state_map(*(cut(a, slice(0, t1)) for a in (x.k, x.v, x.log_alpha, x.b, x.w)))
    second = sm.state_map(*(cut(a, slice(t1, 37)) for a in (x.k, x.v, x.log_alpha, x.b, x.w)))
    P, Q = sm.compose(first, second)
    np.testing.assert_allclose(P, whole[0], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(Q, whole[1], rtol=1e-11, atol=1e-13)


def test_no_erase_closed_form():
    x = _inputs(23, 4)
    b0 = np.zeros_like(x.b)
    Phi, Psi = sm.state_map(x.k, x.v, x.log_alpha, b0, x.w)
    la = x.log_alpha.astype(np.float64)
    k, v, w = (a.astype(np.float64) for a in (x.k, x.v, x.w))
    for h in range(2):
        np.testing.assert_allclose(Phi[0, h], np.diag(np.exp(la[0, :, h].sum(0))), rtol=1e-13)
        ref = np.zeros((8, 6))
        for t in range(23):
            tail = np.exp(la[0, t + 1:, h].sum(0))
            ref += np.outer(tail * k[0, t, h], w[0, t, h] * v[0, t, h])
        np.testing.assert_allclose(Psi[0, h], ref, rtol=1e-12, atol=1e-14)


def test_deltanet_overwrites_the_last_key():
    x = _inputs(11, 5)
    ones = np.ones_like(x.b)
    k = x.k.astype(np.float64)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)           # unit keys to fp64 precision
    Phi, Psi = sm.state_map(k, x.v, np.zeros_like(x.log_alpha), ones, np.ones_like(x.w))
    kT = k[0, -1]
    for h in range(2):
        np.testing.assert_allclose(kT[h] @ Phi[0, h], 0.0, atol=1e-13)
        np.testing.assert_allclose(kT[h] @ Psi[0, h], x.v[0, -1, h], rtol=1e-12, atol=1e-13)


def test_planted_mistakes_fail_the_pins():
    x = _inputs(21, 6)
    _, hT = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.scale, h0=x.h0)

    def err(k, v, la, b, w):
        Phi, Psi = sm.state_map(k, v, la, b, w)
        got = np.einsum("nhij,nhjv->nhiv", Phi, x.h0.astype(np.float64)) + Psi
        return np.abs(got - hT).max()

    assert err(x.k, x.v, x.log_alpha, x.b, x.w) < 1e-10
    assert err(x.k, x.v, x.log_alpha, -x.b, x.w) > 1e-4            # erase sign flipped
    assert err(x.k, x.v, x.log_alpha, x.b, np.ones_like(x.w)) > 1e-4   # write gate dropped
    assert err(x.k, x.v, 0.5 * x.log_alpha, x.b, x.w) > 1e-4       # half the decay
