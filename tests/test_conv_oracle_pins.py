"""Pins of the short-convolution oracle (oracle/shortconv.py) against facts
that do not come from the oracle itself: central finite differences, numpy's
own convolution, identity and shift kernels, hand-worked SiLU values and the
segment-split identity of the boundary state."""
import numpy as np
import pytest

from oracle import shortconv as sc


def _rand(rng, B, H, T, d, K, with_state=True):
    x = rng.standard_normal((B, H, T, d))
    w = rng.standard_normal((H, d, K)) * 0.7
    ci = rng.standard_normal((B, H, K - 1, d)) if with_state else None
    dy = rng.standard_normal((B, H, T, d))
    dco = rng.standard_normal((B, H, K - 1, d))
    return x, w, ci, dy, dco


def _loss(x, w, ci, dy, dco, act):
    y, co = sc.conv_fwd(x, w, ci, act)
    return float(np.sum(y * dy) + np.sum(co * dco))


@pytest.mark.parametrize("act", ["silu", "none"])
@pytest.mark.parametrize("T,K", [(1, 2), (2, 4), (5, 4), (7, 3), (3, 5)])
def test_gradients_match_finite_differences(act, T, K):
    """Central differences of L = <y, dy> + <conv_out, dconv_out> in every input."""
    rng = np.random.default_rng(100 + T * 10 + K)
    x, w, ci, dy, dco = _rand(rng, 1, 2, T, 3, K)
    gr = sc.conv_bwd(x, w, ci, dy, dco, act)
    h = 1e-6
    for name, arr, g in (("x", x, gr["dx"]), ("w", w, gr["dw"]), ("conv_in", ci, gr["dconv_in"])):
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + h
            lp = _loss(x, w, ci, dy, dco, act)
            arr[idx] = old - h
            lm = _loss(x, w, ci, dy, dco, act)
            arr[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(num - g)) / max(np.max(np.abs(num)), 1e-12)
        assert err < 1e-6, (name, err)


def test_matches_numpy_convolve():
    """Without the activation, every channel is numpy's full convolution of the
    extended input with the taps, read at offsets K-1 .. K-1+T-1."""
    rng = np.random.default_rng(7)
    x, w, ci, _, _ = _rand(rng, 2, 2, 11, 3, 4)
    y, co = sc.conv_fwd(x, w, ci, "none")
    for b in range(2):
        for h in range(2):
            for c in range(3):
                xe = np.concatenate([ci[b, h, :, c], x[b, h, :, c]])
                ref = np.convolve(xe, w[h, c])[3:3 + 11]
                np.testing.assert_allclose(y[b, h, :, c], ref, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(co, x[:, :, -3:, :])


def test_identity_and_shift_kernels():
    rng = np.random.default_rng(8)
    x, _, ci, _, _ = _rand(rng, 1, 1, 6, 2, 3)
    for j in range(3):
        w = np.zeros((1, 2, 3))
        w[..., j] = 1.0
        y, _ = sc.conv_fwd(x, w, ci, "none")
        xe = np.concatenate([ci, x], axis=2)
        np.testing.assert_array_equal(y, xe[:, :, 2 - j:2 - j + 6, :])


def test_silu_values():
    """SiLU(z) = z sigma(z): 0 at 0; at z = ln 3, sigma = 3/4.  Its derivative
    sigma (1 + z (1 - sigma)) is 1/2 at 0."""
    x = np.array([0.0, np.log(3.0)]).reshape(1, 1, 2, 1)
    w = np.ones((1, 1, 1))
    y, _ = sc.conv_fwd(x, w, None, "silu")
    np.testing.assert_allclose(y.ravel(), [0.0, 0.75 * np.log(3.0)], rtol=0, atol=1e-15)
    gr = sc.conv_bwd(x, w, None, np.ones_like(x), None, "silu")
    s = 0.75
    np.testing.assert_allclose(gr["dx"].ravel(), [0.5, s * (1 + np.log(3.0) * (1 - s))], rtol=1e-15)


def test_empty_segment_passes_the_state_through():
    rng = np.random.default_rng(9)
    x, w, ci, dy, dco = _rand(rng, 1, 2, 0, 3, 4)
    y, co = sc.conv_fwd(x, w, ci, "silu")
    assert y.shape == (1, 2, 0, 3)
    np.testing.assert_array_equal(co, ci)
    gr = sc.conv_bwd(x, w, ci, dy, dco, "silu")
    np.testing.assert_array_equal(gr["dconv_in"], dco)
    assert np.all(gr["dw"] == 0)


@pytest.mark.parametrize("seg_len", [[5, 6], [1, 1, 9], [0, 4, 0, 7], [2, 1, 2, 6], [11]])
def test_segment_split_identity(seg_len):
    """Splitting the sequence and handing the convolution state on (and its
    gradient back) changes no result, including segments shorter than the
    state and empty ones."""
    rng = np.random.default_rng(10)
    x, w, ci, dy, dco = _rand(rng, 2, 2, 11, 3, 4)
    y1, co1, g1 = sc.segment_run(x, w, ci, dy, dco, N=1)
    yN, coN, gN = sc.segment_run(x, w, ci, dy, dco, N=len(seg_len), seg_len=seg_len)
    np.testing.assert_allclose(yN, y1, rtol=0, atol=1e-12)
    np.testing.assert_array_equal(coN, co1)
    for k in ("dx", "dw", "dconv_in"):
        np.testing.assert_allclose(gN[k], g1[k], rtol=0, atol=1e-12)
