"""Pins of the token-path oracle (oracle/token_path.py), no GPU.

  * the convolution against numpy's own 1-D convolution, channel by channel;
  * a one-tap kernel is the identity, a delayed tap shifts by one token with
    zero at every sequence start (causal, and packed sequences do not see each
    other);
  * SiLU: silu(0) = 0, silu(x) -> x for large x, silu(x) = x sigmoid(x);
  * L2 normalisation gives unit vectors (to eps) in the same direction;
  * RMS normalisation is scale invariant and gives mean square weight^2;
  * the gate at g = 0 halves the normalised output;
and a planted anti-causal convolution fails the shift pin.
"""
import numpy as np

from oracle import token_path as tp


def _x(B, T, H, d, seed):
    return np.random.default_rng(seed).standard_normal((B, T, H, d))


def test_conv_matches_numpy_convolve():
    x = _x(2, 30, 2, 3, 0)
    w = np.random.default_rng(1).standard_normal((6, 4))
    y = tp.short_conv(x, w)
    for bi in range(2):
        for h in range(2):
            for c in range(3):
                ref = np.convolve(x[bi, :, h, c], w[h * 3 + c])[:30]
                np.testing.assert_allclose(y[bi, :, h, c], ref, rtol=1e-13, atol=1e-13)


def test_conv_identity_and_shift_stay_inside_sequences():
    x = _x(1, 12, 1, 4, 2)
    cu = np.array([0, 5, 5, 12])
    ident = np.zeros((4, 4)); ident[:, 0] = 1
    np.testing.assert_array_equal(tp.short_conv(x, ident, cu), x)
    shift = np.zeros((4, 4)); shift[:, 1] = 1
    y = tp.short_conv(x, shift, cu)
    for a, b in ((0, 5), (5, 12)):
        np.testing.assert_array_equal(y[0, a], 0.0)
        np.testing.assert_array_equal(y[0, a + 1:b], x[0, a:b - 1])

    def anti_causal(x, weight):
        return tp.short_conv(x[:, ::-1], weight)[:, ::-1]
    assert np.abs(anti_causal(x, shift)[0, 1:5] - x[0, 0:4]).max() > 0.1


def test_silu():
    assert tp.silu(0.0) == 0.0
    np.testing.assert_allclose(tp.silu(40.0), 40.0, rtol=1e-15)
    x = np.linspace(-6, 6, 25)
    np.testing.assert_allclose(tp.silu(x), x / (1 + np.exp(-x)), rtol=1e-15)


def test_l2norm_unit_and_direction():
    x = _x(1, 7, 3, 16, 3)
    y = tp.l2norm(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=1e-6)
    cos = np.sum(x * y, -1) / np.linalg.norm(x, axis=-1)
    np.testing.assert_allclose(cos, 1.0, rtol=1e-6)


def test_rmsnorm_scale_invariance_and_mean_square():
    x = _x(1, 5, 2, 32, 4)
    w = np.linspace(0.5, 1.5, 32)
    np.testing.assert_allclose(tp.rmsnorm(7.5 * x, w), tp.rmsnorm(x, w), rtol=1e-6)
    y = tp.rmsnorm(x, np.ones(32))
    np.testing.assert_allclose(np.mean(y * y, -1), 1.0, rtol=1e-5)


def test_gate_at_zero_halves():
    o = _x(1, 3, 2, 8, 5)
    w = np.ones(8)
    np.testing.assert_allclose(tp.epilogue(o, np.zeros_like(o), w), 0.5 * tp.rmsnorm(o, w), rtol=1e-15)
