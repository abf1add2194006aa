"""Pins of the per-channel-decay delta-rule oracle (oracle/kda.py): central
finite differences of every input, exact reduction to the scalar-decay oracle
(the independent C implementation) when all channels decay alike, closed forms
for beta = 0 and for the beta-off recurrence without decay, and the
segment-split identity."""
import numpy as np
import pytest

import oracle
from oracle import kda


def _rand(rng, B, H, T, dk, dv, beta=True, state=True):
    q = rng.standard_normal((B, H, T, dk)) * 0.5
    k = rng.standard_normal((B, H, T, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H, T, dv))
    g = -np.log1p(np.exp(rng.standard_normal((B, H, T, dk)) - 1.0))
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, H, T)))) if beta else None
    S = rng.standard_normal((B, H, dk, dv)) * 0.3 if state else None
    dO = rng.standard_normal((B, H, T, dv))
    dS = rng.standard_normal((B, H, dk, dv)) * 0.3
    return q, k, v, g, b, S, dO, dS


def _loss(q, k, v, g, b, S, dO, dS, scale):
    o, So = kda.kda_fwd(q, k, v, g, b, S, scale)
    return float(np.sum(o * dO) + np.sum(So * dS))


@pytest.mark.parametrize("beta", [True, False])
@pytest.mark.parametrize("T", [1, 3, 8])
def test_gradients_match_finite_differences(beta, T):
    rng = np.random.default_rng(40 + T + (10 if beta else 0))
    q, k, v, g, b, S, dO, dS = _rand(rng, 1, 1, T, 4, 3, beta)
    scale = 0.7
    gr = kda.kda_bwd(q, k, v, g, b, S, dO, dS, scale)
    h = 1e-6
    pairs = [("dq", q), ("dk", k), ("dv", v), ("dg", g), ("dS_in", S)] + ([("dbeta", b)] if beta else [])
    for name, arr in pairs:
        num = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            old = arr[idx]
            arr[idx] = old + h
            lp = _loss(q, k, v, g, b, S, dO, dS, scale)
            arr[idx] = old - h
            lm = _loss(q, k, v, g, b, S, dO, dS, scale)
            arr[idx] = old
            num[idx] = (lp - lm) / (2 * h)
        err = np.max(np.abs(num - gr[name])) / max(np.max(np.abs(num)), 1e-12)
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("beta", [True, False])
def test_equal_channel_decay_is_the_scalar_decay_layer(beta):
    """With the same log-decay on every key channel, the diagonal transition is
    the scalar one: outputs and gradients equal the C oracle's, and dg of the
    scalar layer is the sum over channels."""
    rng = np.random.default_rng(3)
    q, k, v, g, b, S, dO, dS = _rand(rng, 2, 2, 150, 8, 6, beta)
    gs = g[..., 0]
    g = np.repeat(gs[..., None], 8, axis=-1)
    o1, S1 = kda.kda_fwd(q, k, v, g, b, S, 0.5)
    o2, S2 = oracle.gdn_fwd(q, k, v, gs, b, S, 0.5)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-11)
    np.testing.assert_allclose(S1, S2, rtol=0, atol=1e-11)
    g1 = kda.kda_bwd(q, k, v, g, b, S, dO, dS, 0.5)
    g2 = oracle.gdn_bwd(q, k, v, gs, b, S, dO, dS, 0.5)
    for n in ("dq", "dk", "dv", "dS_in") + (("dbeta",) if beta else ()):
        np.testing.assert_allclose(g1[n], g2[n], rtol=0, atol=1e-10)
    np.testing.assert_allclose(g1["dg"].sum(-1), g2["dg"], rtol=0, atol=1e-10)


def test_beta_zero_closed_form():
    """beta = 0: nothing is erased or written, the state only decays per channel."""
    rng = np.random.default_rng(4)
    q, k, v, g, _, S, _, _ = _rand(rng, 1, 2, 20, 5, 3)
    b = np.zeros(q.shape[:3])
    o, So = kda.kda_fwd(q, k, v, g, b, S, 1.3)
    G = np.cumsum(g, axis=2)
    ref = 1.3 * np.einsum("bhtc,bhcj->bhtj", q * np.exp(G), S)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(So, np.exp(G[:, :, -1])[..., None] * S, rtol=0, atol=1e-12)


def test_beta_off_without_decay_is_linear_attention():
    rng = np.random.default_rng(5)
    q, k, v, _, _, S, _, _ = _rand(rng, 1, 1, 12, 4, 3, beta=False)
    g = np.zeros(q.shape)
    o, _ = kda.kda_fwd(q, k, v, g, None, S, 1.0)
    qk = np.einsum("bhtc,bhsc->bhts", q, k)
    ref = np.einsum("bhtc,bhcj->bhtj", q, S) + np.einsum("bhts,bhsj->bhtj", np.tril(qk), v)
    np.testing.assert_allclose(o, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("seg_len", [[70, 80], [1, 0, 100, 49], [64, 64, 22]])
def test_segment_split_identity(seg_len):
    rng = np.random.default_rng(6)
    args = _rand(rng, 1, 2, 150, 6, 5)
    q, k, v, g, b, S, dO, dS = args
    o1, S1, g1 = kda.segment_run(q, k, v, g, b, S, dO, dS, N=1)
    oN, SN, gN = kda.segment_run(q, k, v, g, b, S, dO, dS, N=len(seg_len), seg_len=seg_len)
    np.testing.assert_allclose(oN, o1, rtol=0, atol=1e-12)
    np.testing.assert_allclose(SN, S1, rtol=0, atol=1e-12)
    for n in g1:
        np.testing.assert_allclose(gN[n], g1[n], rtol=0, atol=1e-11)
