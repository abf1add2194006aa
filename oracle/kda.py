"""fp64 oracle of the delta rule with a per-channel (diagonal) decay.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may use it; it shares no code with the CUDA
library and never imports it.

StateFlow (arXiv 2608.06838, section 2.1) lists the structured transitions F_t
of modern linear recurrences, S_t = S_{t-1} F_t + v_t k_t^T: scalar-identity
(Mamba-2), rank-1 (Gated Linear Attention), scalar-plus-low-rank (Gated
DeltaNet) and diagonal-plus-low-rank (Kimi Delta Attention, KDA).  The reading
taken here for the diagonal-plus-low-rank member, in the same orientation as
the rest of this oracle (state S in R^{dk x dv}, rows = key channels):

    alpha_t = exp(g_t)  in R^{dk}   (a log-decay per key channel)
    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
    o_t = scale * S_t^T q_t
and with the beta path off (per-channel decay without the delta term):
    S_t = Diag(alpha_t) S_{t-1} + k_t v_t^T

With every channel's log-decay equal this is exactly the scalar-decay layer
of ``oracle.gdn_fwd`` (a pin).  The backward gives the gradients of
L = sum_t <o_t, dO_t> + <S_out, dS_out> by the reverse-time adjoint, with D the
total gradient of S_t (the carry from later tokens plus scale q_t dO_t^T),
S' = Diag(alpha_t) S_{t-1}, u = S'^T k_t, w = D^T k_t:
    dq_t = scale S_t dO_t              dv_t = beta_t w
    dbeta_t = w . (v_t - u)            dk_t = beta_t (D (v_t - u) - S' w)
    dS' = D - beta_t k_t w^T           dg_t = alpha_t * rowsum(dS' * S_{t-1})
    carry <- Diag(alpha_t) dS'
(beta off: dk = D v, dv = D^T k, dS' = D.)  S_{t-1} is replayed forward from a
checkpoint every 64 tokens.
"""
from __future__ import annotations

import numpy as np

_W = 64  # checkpoint interval


def _split(x):
    B, H = x.shape[:2]
    return B, H, x.reshape((B * H,) + x.shape[2:])


def kda_fwd(q, k, v, g, beta=None, S_in=None, scale=1.0, checkpoints=False):
    """q, k: [B,H,T,dk]; v: [B,H,T,dv]; g: [B,H,T,dk] log-decays; beta: [B,H,T]
    or None; S_in: [B,H,dk,dv] or None.  Returns (o, S_out) (and the list of
    states at every 64th token when ``checkpoints``)."""
    B, H, qq = _split(np.asarray(q, np.float64))
    kk = np.asarray(k, np.float64).reshape(qq.shape)
    vv = np.asarray(v, np.float64).reshape((B * H,) + v.shape[2:])
    gg = np.asarray(g, np.float64).reshape(qq.shape)
    bb = None if beta is None else np.asarray(beta, np.float64).reshape(B * H, -1)
    T, dk = qq.shape[1], qq.shape[2]
    dv = vv.shape[2]
    S = np.zeros((B * H, dk, dv)) if S_in is None else np.asarray(S_in, np.float64).reshape(B * H, dk, dv).copy()
    o = np.zeros((B * H, T, dv))
    cps = []
    for t in range(T):
        if checkpoints and t % _W == 0:
            cps.append(S.copy())
        S = _step(S, kk[:, t], vv[:, t], gg[:, t], None if bb is None else bb[:, t])
        o[:, t] = scale * np.einsum("bcj,bc->bj", S, qq[:, t])
    o = o.reshape(B, H, T, dv)
    S_out = S.reshape(B, H, dk, dv)
    return (o, S_out, cps) if checkpoints else (o, S_out)


def _step(S, k, v, g, b):
    Sp = np.exp(g)[:, :, None] * S
    if b is None:
        return Sp + k[:, :, None] * v[:, None, :]
    u = np.einsum("bcj,bc->bj", Sp, k)
    return Sp + (b[:, None, None] * k[:, :, None]) * (v - u)[:, None, :]


def kda_bwd(q, k, v, g, beta, S_in, dO, dS_out=None, scale=1.0):
    """Gradients of sum <o, dO> + <S_out, dS_out>: dict dq, dk, dv, dg, dbeta
    (None when beta is None), dS_in."""
    q = np.asarray(q, np.float64)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    BH = B * H
    _, _, cps = kda_fwd(q, k, v, g, beta, S_in, scale, checkpoints=True)
    qq = q.reshape(BH, T, dk)
    kk = np.asarray(k, np.float64).reshape(BH, T, dk)
    vv = np.asarray(v, np.float64).reshape(BH, T, dv)
    gg = np.asarray(g, np.float64).reshape(BH, T, dk)
    bb = None if beta is None else np.asarray(beta, np.float64).reshape(BH, T)
    dOO = np.asarray(dO, np.float64).reshape(BH, T, dv)
    carry = np.zeros((BH, dk, dv)) if dS_out is None else np.asarray(dS_out, np.float64).reshape(BH, dk, dv).copy()
    out = {n: np.zeros((BH, T, dk)) for n in ("dq", "dk", "dg")}
    out["dv"] = np.zeros((BH, T, dv))
    out["dbeta"] = None if bb is None else np.zeros((BH, T))
    for w0 in reversed(range(0, T, _W)):
        w1 = min(T, w0 + _W)
        states = [cps[w0 // _W]]  # states[i] = S_{w0+i-1} (the state before token w0+i)
        for t in range(w0, w1):
            states.append(_step(states[-1], kk[:, t], vv[:, t], gg[:, t], None if bb is None else bb[:, t]))
        for t in reversed(range(w0, w1)):
            Sprev, St = states[t - w0], states[t - w0 + 1]
            D = carry + scale * qq[:, t, :, None] * dOO[:, t, None, :]
            out["dq"][:, t] = scale * np.einsum("bcj,bj->bc", St, dOO[:, t])
            a = np.exp(gg[:, t])
            Sp = a[:, :, None] * Sprev
            kt, vt = kk[:, t], vv[:, t]
            wv = np.einsum("bcj,bc->bj", D, kt)
            if bb is None:
                out["dk"][:, t] = np.einsum("bcj,bj->bc", D, vt)
                out["dv"][:, t] = wv
                dSp = D
            else:
                b = bb[:, t]
                u = np.einsum("bcj,bc->bj", Sp, kt)
                out["dv"][:, t] = b[:, None] * wv
                out["dbeta"][:, t] = np.sum(wv * (vt - u), axis=1)
                out["dk"][:, t] = b[:, None] * (np.einsum("bcj,bj->bc", D, vt - u) - np.einsum("bcj,bj->bc", Sp, wv))
                dSp = D - b[:, None, None] * kt[:, :, None] * wv[:, None, :]
            out["dg"][:, t] = a * np.sum(dSp * Sprev, axis=2)
            carry = a[:, :, None] * dSp
    res = {n: None if x is None else x.reshape((B, H) + x.shape[1:]) for n, x in out.items()}
    res["dS_in"] = carry.reshape(B, H, dk, dv)
    return res


def segment_run(q, k, v, g, beta, S_in, dO, dS_out=None, N=1, seg_len=None, scale=1.0):
    """N segments with the state handed forward and its gradient backward.
    Returns (o, S_out, grads)."""
    T = q.shape[2]
    if seg_len is None:
        base, rem = divmod(T, N)
        seg_len = [base + (1 if i < rem else 0) for i in range(N)]
    starts = np.cumsum([0] + list(seg_len))
    sl = lambda x, i: None if x is None else x[:, :, starts[i]:starts[i + 1]]
    states = [S_in]
    os_ = []
    for i in range(N):
        o, S = kda_fwd(sl(q, i), sl(k, i), sl(v, i), sl(g, i), sl(beta, i), states[i], scale)
        os_.append(o)
        states.append(S)
    grads = {n: [] for n in ("dq", "dk", "dv", "dg", "dbeta")}
    dS = dS_out
    for i in reversed(range(N)):
        gr = kda_bwd(sl(q, i), sl(k, i), sl(v, i), sl(g, i), sl(beta, i), states[i], sl(dO, i), dS, scale)
        for n in grads:
            grads[n].insert(0, gr[n])
        dS = gr["dS_in"]
    cat = {n: None if beta is None and n == "dbeta" else np.concatenate(x, axis=2) for n, x in grads.items()}
    cat["dS_in"] = dS
    return np.concatenate(os_, axis=2), states[N], cat
