"""fp64 oracle of the short causal convolution with a boundary state.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may use it; it shares no code with the CUDA
library and never imports it.

StateFlow (arXiv 2608.06838) names two kinds of state a sequence chunk hands to
the next one: the recurrent state and the boundary state of the local
convolution modules (section 1, the first challenge of applying sequence
pipelining to linear recurrence; section 3.3, where the boundary tensor B_r is
"compact recurrent and local-convolution boundary states").  The pages do not
spell the convolution out.  The reading taken here is the causal depthwise
short convolution of Gated DeltaNet-style layers, applied per channel before
the recurrence:

  per (batch b, head h, channel c), taps w[h, c, 0..K-1] (tap j multiplies the
  input j steps back), extended input xe_p for p = -(K-1) .. T-1 with
  xe_p = conv_in[K-1+p] for p < 0 (the last K-1 inputs of the previous chunk,
  oldest first) and xe_p = x_p otherwise:
      pre_t = sum_j w_j xe_{t-j},     y_t = act(pre_t)   (act: identity or SiLU)
      conv_out = xe_{T-(K-1)} .. xe_{T-1}   (the state handed to the next chunk)

The backward gives the gradients of L = sum_t <y_t, dy_t> + <conv_out, dconv_out>
with respect to x, w and conv_in (dconv_in is handed to the previous chunk).
Everything is plain loops over the definition, in fp64.
"""
from __future__ import annotations

import numpy as np


def _act(z, act):
    if act == "silu":
        return z / (1.0 + np.exp(-z))
    return z


def _dact(z, act):
    if act == "silu":
        s = 1.0 / (1.0 + np.exp(-z))
        return s * (1.0 + z * (1.0 - s))
    return np.ones_like(z)


def _extended(x, conv_in, K):
    """[B, H, K-1+T, d]: conv_in (zeros when None) followed by x."""
    B, H, T, d = x.shape
    ci = np.zeros((B, H, K - 1, d)) if conv_in is None else np.asarray(conv_in, np.float64)
    return np.concatenate([ci, np.asarray(x, np.float64)], axis=2)


def conv_fwd(x, w, conv_in=None, act="silu"):
    """x: [B,H,T,d]; w: [H,d,K]; conv_in: [B,H,K-1,d] or None.  Returns (y, conv_out)."""
    B, H, T, d = x.shape
    K = w.shape[-1]
    xe = _extended(x, conv_in, K)
    pre = np.zeros((B, H, T, d))
    for t in range(T):
        for j in range(K):
            # xe index of x_{t-j} is (t - j) + (K - 1)
            pre[:, :, t, :] += w[None, :, :, j] * xe[:, :, t - j + K - 1, :]
    y = _act(pre, act)
    conv_out = xe[:, :, T:T + K - 1, :].copy()
    return y, conv_out


def conv_bwd(x, w, conv_in, dy, dconv_out=None, act="silu"):
    """Gradients of sum <y, dy> + <conv_out, dconv_out>.  Returns dict dx, dw, dconv_in."""
    B, H, T, d = x.shape
    K = w.shape[-1]
    xe = _extended(x, conv_in, K)
    pre = np.zeros((B, H, T, d))
    for t in range(T):
        for j in range(K):
            pre[:, :, t, :] += w[None, :, :, j] * xe[:, :, t - j + K - 1, :]
    delta = np.asarray(dy, np.float64) * _dact(pre, act)
    dxe = np.zeros_like(xe)
    dw = np.zeros((H, d, K))
    for t in range(T):
        for j in range(K):
            dxe[:, :, t - j + K - 1, :] += w[None, :, :, j] * delta[:, :, t, :]
            dw[:, :, j] += np.sum(delta[:, :, t, :] * xe[:, :, t - j + K - 1, :], axis=0)
    if dconv_out is not None:
        # conv_out is the last K-1 entries of the extended input
        dxe[:, :, T:T + K - 1, :] += np.asarray(dconv_out, np.float64)
    return {"dx": dxe[:, :, K - 1:, :], "dw": dw, "dconv_in": dxe[:, :, :K - 1, :]}


def segment_run(x, w, conv_in, dy, dconv_out=None, N=1, seg_len=None, act="silu"):
    """The sequence as N segments with the convolution state handed forward and
    its gradient handed backward (the weight gradient summed over segments).
    Returns (y, conv_out, grads)."""
    B, H, T, d = x.shape
    K = w.shape[-1]
    if seg_len is None:
        base, rem = divmod(T, N)
        seg_len = [base + (1 if i < rem else 0) for i in range(N)]
    assert sum(seg_len) == T
    starts = np.cumsum([0] + list(seg_len))
    ys, states = [], [np.zeros((B, H, K - 1, d)) if conv_in is None else np.asarray(conv_in, np.float64)]
    for i in range(N):
        a, b = starts[i], starts[i + 1]
        y, co = conv_fwd(x[:, :, a:b], w, states[i], act)
        ys.append(y)
        states.append(co)
    out = {"dx": np.zeros((B, H, T, d)), "dw": np.zeros((H, d, K))}
    g = np.zeros((B, H, K - 1, d)) if dconv_out is None else np.asarray(dconv_out, np.float64)
    for i in reversed(range(N)):
        a, b = starts[i], starts[i + 1]
        gr = conv_bwd(x[:, :, a:b], w, states[i], dy[:, :, a:b], g, act)
        out["dx"][:, :, a:b] = gr["dx"]
        out["dw"] += gr["dw"]
        g = gr["dconv_in"]
    out["dconv_in"] = g
    return np.concatenate(ys, axis=2), states[N], out
