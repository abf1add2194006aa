"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

The pages print no worked example, so the oracle is fixed by:
  * hand-worked two-token examples (tests/golden/), exact dyadic values;
  * central finite differences of the scalar L = sum <o,dO> + <S_out,dS_out>,
    the concrete check the StateFlow review asks for (state gradient against an
    independent differentiation, < 1e-6 relative);
  * closed forms: the scalar-gated recurrence without the delta term is plain
    decay-masked linear attention (direct O(T^2) sums); the delta rule with
    beta = 0 only decays the incoming state;
  * the delta-rule retrieval invariant: beta = 1 and unit keys give S_t^T k_t = v_t;
  * single-token formulas written out, and linearity in (V, S_in);
  * the segment-split identity of StateFlow section 3.1 (exactness claim of
    section 4.1), N segments with state handoff == one pass;
  * the chunkwise Pre/ST/Out form (section 2.2), an independent derivation,
    agreeing for several chunk sizes and ragged lengths.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import chunkwise

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_case(rng, B=1, H=1, T=5, dk=4, dv=3, beta=True, g_scale=0.3, unit_k=False, s_in=0.5):
    q = rng.standard_normal((B, H, T, dk))
    k = rng.standard_normal((B, H, T, dk))
    if unit_k:
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, H, T, dv))
    g = -g_scale * np.abs(rng.standard_normal((B, H, T)))
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, H, T)))) if beta else None
    S_in = s_in * rng.standard_normal((B, H, dk, dv)) if s_in else None
    dO = rng.standard_normal((B, H, T, dv))
    dS = 0.3 * rng.standard_normal((B, H, dk, dv))
    return dict(q=q, k=k, v=v, g=g, beta=b, S_in=S_in, dO=dO, dS_out=dS)


def relerr(x, y):
    x = np.asarray(x, np.float64)
    y = np.asarray(y, np.float64)
    den = np.max(np.abs(y))
    if den == 0:
        return float(np.max(np.abs(x)))
    return float(np.max(np.abs(x - y)) / den)


# ---------------------------------------------------------------- golden ----

def test_golden_two_token_delta_rule():
    ex = json.load(open(os.path.join(GOLDEN, "two_token_example.json")))
    q = np.array(ex["q"], float)[None, None]
    k = np.array(ex["k"], float)[None, None]
    v = np.array(ex["v"], float)[None, None]
    g = np.log(np.array(ex["alpha"], float))[None, None]
    b = np.array(ex["beta"], float)[None, None]
    S_in = np.array(ex["S_in"], float)[None, None]
    o, S_out = oracle.gdn_fwd(q, k, v, g, b, S_in)
    np.testing.assert_allclose(o[0, 0], np.array(ex["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(S_out[0, 0], np.array(ex["S_out"]), rtol=0, atol=1e-14)


def test_golden_two_token_beta_off():
    ex = json.load(open(os.path.join(GOLDEN, "betaoff_two_token_example.json")))
    q = np.array(ex["q"], float)[None, None]
    k = np.array(ex["k"], float)[None, None]
    v = np.array(ex["v"], float)[None, None]
    g = np.log(np.array(ex["alpha"], float))[None, None]
    S_in = np.array(ex["S_in"], float)[None, None]
    o, S_out = oracle.gdn_fwd(q, k, v, g, None, S_in)
    np.testing.assert_allclose(o[0, 0], np.array(ex["o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(S_out[0, 0], np.array(ex["S_out"]), rtol=0, atol=1e-14)


# ------------------------------------------------------ finite differences --

def _loss_of(case, scale):
    o, S_out = oracle.gdn_fwd(case["q"], case["k"], case["v"], case["g"], case["beta"],
                              case["S_in"], scale)
    return oracle.loss(o, S_out, case["dO"], case["dS_out"])


@pytest.mark.parametrize("T", [1, 3, 8, 17])
@pytest.mark.parametrize("beta", [True, False])
def test_finite_differences(T, beta):
    rng = np.random.default_rng(100 + T + (7 if beta else 0))
    case = rand_case(rng, B=1, H=2, T=T, dk=4, dv=3, beta=beta)
    scale = 0.7
    gr = oracle.gdn_bwd(case["q"], case["k"], case["v"], case["g"], case["beta"], case["S_in"],
                        case["dO"], case["dS_out"], scale, ckpt=4)
    h = 1e-6
    names = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("S_in", "dS_in")]
    if beta:
        names.append(("beta", "dbeta"))
    for name, gname in names:
        x = case[name]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + h
            lp = _loss_of(case, scale)
            x[idx] = old - h
            lm = _loss_of(case, scale)
            x[idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        assert relerr(gr[gname], fd) < 1e-6, (name, relerr(gr[gname], fd))
    if not beta:
        assert gr["dbeta"] is None


def test_finite_differences_no_state():
    """S_in and dS_out absent (zeros) still give consistent gradients."""
    rng = np.random.default_rng(5)
    case = rand_case(rng, T=6, s_in=0)
    case["dS_out"] = None
    gr = oracle.gdn_bwd(case["q"], case["k"], case["v"], case["g"], case["beta"], None,
                        case["dO"], None)
    h = 1e-6
    x = case["v"]
    fd = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        idx = it.multi_index
        old = x[idx]
        x[idx] = old + h
        lp = _loss_of(case, 1.0)
        x[idx] = old - h
        lm = _loss_of(case, 1.0)
        x[idx] = old
        fd[idx] = (lp - lm) / (2 * h)
    assert relerr(gr["dv"], fd) < 1e-6


# ------------------------------------------------------------ closed forms --

@pytest.mark.parametrize("zero_g", [True, False])
def test_beta_off_is_decay_masked_linear_attention(zero_g):
    rng = np.random.default_rng(11)
    B, H, T, dk, dv = 1, 2, 13, 5, 4
    case = rand_case(rng, B, H, T, dk, dv, beta=False, g_scale=0.0 if zero_g else 0.4)
    q, k, v, g, S_in = case["q"], case["k"], case["v"], case["g"], case["S_in"]
    o, S_out = oracle.gdn_fwd(q, k, v, g, None, S_in)
    for b in range(B):
        for hh in range(H):
            G = np.cumsum(g[b, hh])
            for t in range(T):
                ref = np.exp(G[t]) * (S_in[b, hh].T @ q[b, hh, t])
                for s in range(t + 1):
                    ref = ref + np.exp(G[t] - G[s]) * np.dot(q[b, hh, t], k[b, hh, s]) * v[b, hh, s]
                np.testing.assert_allclose(o[b, hh, t], ref, rtol=1e-12, atol=1e-12)
            Sref = np.exp(G[-1]) * S_in[b, hh]
            for s in range(T):
                Sref = Sref + np.exp(G[-1] - G[s]) * np.outer(k[b, hh, s], v[b, hh, s])
            np.testing.assert_allclose(S_out[b, hh], Sref, rtol=1e-12, atol=1e-12)


def test_delta_rule_beta_zero_only_decays_state():
    rng = np.random.default_rng(12)
    case = rand_case(rng, 1, 2, 9, 4, 3, beta=True)
    beta0 = np.zeros_like(case["beta"])
    q, k, v, g, S_in = case["q"], case["k"], case["v"], case["g"], case["S_in"]
    o, S_out = oracle.gdn_fwd(q, k, v, g, beta0, S_in)
    G = np.cumsum(g, axis=-1)
    ref_o = np.exp(G)[..., None] * np.einsum("bhkv,bhtk->bhtv", S_in, q)
    np.testing.assert_allclose(o, ref_o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S_out, np.exp(G[..., -1])[..., None, None] * S_in, rtol=1e-12)
    gr = oracle.gdn_bwd(q, k, v, g, beta0, S_in, case["dO"], case["dS_out"])
    assert np.max(np.abs(gr["dv"])) == 0.0


@pytest.mark.parametrize("g_scale", [0.0, 0.5, 3.0])
def test_retrieval_invariant(g_scale):
    """beta = 1 and unit-norm keys: S_t^T k_t = v_t for any decay, so q = k gives o = v."""
    rng = np.random.default_rng(13)
    case = rand_case(rng, 1, 2, 20, 6, 5, beta=True, g_scale=g_scale, unit_k=True)
    ones = np.ones_like(case["beta"])
    o, _ = oracle.gdn_fwd(case["k"], case["k"], case["v"], case["g"], ones, case["S_in"])
    np.testing.assert_allclose(o, case["v"], rtol=0, atol=1e-12)


def test_single_token_forms():
    rng = np.random.default_rng(14)
    case = rand_case(rng, 1, 1, 1, 4, 3, beta=True)
    q, k, v = case["q"][0, 0, 0], case["k"][0, 0, 0], case["v"][0, 0, 0]
    a = np.exp(case["g"][0, 0, 0])
    b = case["beta"][0, 0, 0]
    S = case["S_in"][0, 0]
    P = np.eye(4) - b * np.outer(k, k)
    o_ref = b * np.dot(q, k) * v + a * (S.T @ (P @ q))
    S_ref = a * (P @ S) + b * np.outer(k, v)
    o, S_out = oracle.gdn_fwd(case["q"], case["k"], case["v"], case["g"], case["beta"],
                              case["S_in"], 1.0)
    np.testing.assert_allclose(o[0, 0, 0], o_ref, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S_out[0, 0], S_ref, rtol=1e-13, atol=1e-14)


def test_linearity_in_values_and_state():
    rng = np.random.default_rng(15)
    c1 = rand_case(rng, 1, 2, 11, 4, 3)
    c2 = rand_case(rng, 1, 2, 11, 4, 3)
    args = lambda c, v, s: (c1["q"], c1["k"], v, c1["g"], c1["beta"], s)
    o1, s1 = oracle.gdn_fwd(*args(c1, c1["v"], c1["S_in"]))
    o2, s2 = oracle.gdn_fwd(*args(c1, c2["v"], c2["S_in"]))
    o12, s12 = oracle.gdn_fwd(*args(c1, 2 * c1["v"] - c2["v"], 2 * c1["S_in"] - c2["S_in"]))
    np.testing.assert_allclose(o12, 2 * o1 - o2, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(s12, 2 * s1 - s2, rtol=1e-11, atol=1e-12)


def test_empty_sequence():
    rng = np.random.default_rng(16)
    case = rand_case(rng, 1, 2, 0, 4, 3)
    o, S_out = oracle.gdn_fwd(case["q"], case["k"], case["v"], case["g"], case["beta"], case["S_in"])
    assert o.shape == (1, 2, 0, 3)
    np.testing.assert_array_equal(S_out, case["S_in"])
    gr = oracle.gdn_bwd(case["q"], case["k"], case["v"], case["g"], case["beta"], case["S_in"],
                        case["dO"], case["dS_out"])
    np.testing.assert_array_equal(gr["dS_in"], case["dS_out"])


# ------------------------------------------------------ segment identity ----

@pytest.mark.parametrize("seg", [[40], [20, 20], [8, 8, 8, 16], [1, 13, 26], [0, 25, 0, 15]])
@pytest.mark.parametrize("beta", [True, False])
def test_segment_split_identity(seg, beta):
    rng = np.random.default_rng(17)
    case = rand_case(rng, 2, 2, 40, 5, 4, beta=beta, g_scale=0.05)
    o1, S1, g1 = oracle.segment_run(case["q"], case["k"], case["v"], case["g"], case["beta"],
                                    case["S_in"], case["dO"], case["dS_out"], seg_len=[40])
    oN, SN, gN = oracle.segment_run(case["q"], case["k"], case["v"], case["g"], case["beta"],
                                    case["S_in"], case["dO"], case["dS_out"], seg_len=seg)
    assert relerr(oN, o1) < 1e-12
    assert relerr(SN, S1) < 1e-12
    for name in ("dq", "dk", "dv", "dg", "dS_in") + (("dbeta",) if beta else ()):
        assert relerr(gN[name], g1[name]) < 1e-12, name


def test_segment_bounds():
    assert oracle.segment_bounds(10, N=3) == [(0, 4), (4, 7), (7, 10)]
    assert oracle.segment_bounds(8, seg_len=[0, 8]) == [(0, 0), (0, 8)]
    with pytest.raises(ValueError):
        oracle.segment_bounds(8, seg_len=[3, 3])


# -------------------------------------------------------- chunkwise form ----

@pytest.mark.parametrize("C", [16, 32, 64, 128])
@pytest.mark.parametrize("beta", [True, False])
def test_chunkwise_form_matches_token_recurrence(C, beta):
    rng = np.random.default_rng(18 + C)
    T = 2 * C + C // 2 + 3          # several chunks and a ragged tail
    case = rand_case(rng, 1, 2, T, 8, 6, beta=beta, g_scale=0.05, unit_k=True)
    args = (case["q"], case["k"], case["v"], case["g"], case["beta"], case["S_in"])
    o, S_out = oracle.gdn_fwd(*args, scale=0.5)
    oc, Sc = chunkwise.gdn_fwd(*args, scale=0.5, C=C)
    assert relerr(oc, o) < 1e-10
    assert relerr(Sc, S_out) < 1e-10
    gr = oracle.gdn_bwd(*args, case["dO"], case["dS_out"], scale=0.5)
    gc = chunkwise.gdn_bwd(*args, case["dO"], case["dS_out"], scale=0.5, C=C)
    for name in ("dq", "dk", "dv", "dg", "dS_in") + (("dbeta",) if beta else ()):
        assert relerr(gc[name], gr[name]) < 1e-9, (name, relerr(gc[name], gr[name]))


def test_chunkwise_strong_decay_no_overflow():
    """Decay of the workloads (about e^-140 per 64-token chunk) stays finite in the chunk form."""
    rng = np.random.default_rng(19)
    case = rand_case(rng, 1, 1, 100, 8, 8, beta=True, unit_k=True)
    case["g"] = -np.log1p(np.exp(rng.standard_normal((1, 1, 100)) + 2.0))
    args = (case["q"], case["k"], case["v"], case["g"], case["beta"], case["S_in"])
    o, S_out = oracle.gdn_fwd(*args)
    with np.errstate(over="raise", invalid="raise"):
        oc, Sc = chunkwise.gdn_fwd(*args, C=64)
        gc = chunkwise.gdn_bwd(*args, case["dO"], case["dS_out"], C=64)
    assert relerr(oc, o) < 1e-10 and relerr(Sc, S_out) < 1e-10
    gr = oracle.gdn_bwd(*args, case["dO"], case["dS_out"])
    for name in ("dq", "dk", "dv", "dg", "dbeta", "dS_in"):
        assert relerr(gc[name], gr[name]) < 1e-9, name
