"""Chunkwise fp64 form of the gated delta-rule layer (numpy), a test aid.

TEST INFRASTRUCTURE.  It shares no code with the CUDA library and is pinned
against the token-by-token oracle (``oracle.gdn_fwd`` / ``oracle.gdn_bwd``) by
the tests: both must agree to ~1e-12 for every chunk size.  It exists so the
per-stage intermediates of the chunk form (W, U, V_new, the state entering each
chunk, dV_new, the state gradient leaving each chunk) can be inspected.

It follows the three-stage chunk decomposition of StateFlow (arXiv 2608.06838,
section 2.2): Omega_i = Pre(X_i); (S_{(i+1)T_C}, V_i^new) = ST(S_{iT_C}, Omega_i);
Y_i = Out(V_i^new, S_{iT_C}, Omega_i).  For Gated DeltaNet, Pre is the UT/WY
transform of the chunk (the WY form of delta-rule kernels noted on the Gated
Linear Attention citation page), written here from its derivation:

  per chunk of C tokens with local index i, j and chunk-local cumulative
  log-decay G_i = sum_{s<=i} g_s, gamma_i = exp(G_i), Gamma_ij = exp(G_i - G_j)
  for j <= i (0 above the diagonal):
    A     = strictly-lower( diag(beta) (K K^T * Gamma) )
    T     = (I + A)^{-1} diag(beta)
    W     = T (gamma * K)            U = T V
    V_new = U - W S0                                        (ST, first half)
    S_C   = gamma_C S0 + (K * exp(G_C - G))^T V_new         (ST, second half)
    O     = scale [ (gamma * Q) S0 + ((Q K^T) * Gamma) V_new ]   (Out)

The backward is the adjoint of exactly these operations (derivation in
``chunk_bwd``).  The beta-off variant (S_t = alpha_t S_{t-1} + k_t v_t^T) has
no erase term: T = I, W = 0, U = V, so V_new = V.
"""
from __future__ import annotations

import numpy as np


def _pad(x, C, axis):
    n = x.shape[axis]
    r = (-n) % C
    if r == 0:
        return x
    pad = [(0, 0)] * x.ndim
    pad[axis] = (0, r)
    return np.pad(x, pad)


def chunk_pre(k, v, g, beta):
    """Pre for one chunk of one head.  k:[C,dk] v:[C,dv] g:[C] beta:[C] or None."""
    C = k.shape[0]
    G = np.cumsum(g)
    gam = np.exp(G)
    # Gamma_ij = exp(G_i - G_j) for j <= i; above the diagonal the exponent is
    # replaced by 0 before exponentiating, so exp is never taken of a growth term
    mask = np.tril(np.ones((C, C), bool))
    diff = np.where(mask, G[:, None] - G[None, :], 0.0)
    Gam = np.where(mask, np.exp(diff), 0.0)
    if beta is None:
        # no erase term: nothing is subtracted from the values, V_new = V
        Tm = np.eye(C)
        A = np.zeros((C, C))
        Linv = np.eye(C)
        W = np.zeros_like(k)
    else:
        A = np.tril(beta[:, None] * (k @ k.T) * Gam, -1)
        Linv = np.linalg.solve(np.eye(C) + A, np.eye(C))
        Tm = Linv * beta[None, :]
        W = Tm @ (gam[:, None] * k)
    U = Tm @ v
    return {"G": G, "gam": gam, "Gam": Gam, "A": A, "Linv": Linv, "T": Tm, "W": W, "U": U}


def chunk_fwd(q, k, v, g, beta, S0, scale=1.0):
    """Pre + ST + Out for one chunk of one head.  Returns (o, S_C, intermediates)."""
    pre = chunk_pre(k, v, g, beta)
    G, gam, Gam = pre["G"], pre["gam"], pre["Gam"]
    Vn = pre["U"] - pre["W"] @ S0
    dec = np.exp(G[-1] - G)
    S_C = np.exp(G[-1]) * S0 + (k * dec[:, None]).T @ Vn
    qs = scale * q
    P = (qs @ k.T) * Gam
    o = (gam[:, None] * qs) @ S0 + P @ Vn
    pre.update({"V_new": Vn, "S0": S0, "P": P})
    return o, S_C, pre


def chunk_bwd(q, k, v, g, beta, S0, dO, dS_C, scale=1.0):
    """Adjoint of chunk_fwd for one chunk of one head.

    Returns (dq, dk, dv, dg, dbeta, dS0, intermediates).  With Qs = scale*Q,
    P = (Qs K^T) * Gamma, Khat = K * exp(G_C - G), Kt = gamma * K:
      dV_new = P^T dO + Khat dS_C
      dS0    = (gamma*Qs)^T dO + gamma_C dS_C - W^T dV_new
      M      = (dO V_new^T) * Gamma
      dQs    = gamma * (dO S0^T) + M K
      dW     = -dV_new S0^T ;  dU = dV_new
      dKt    = T^T dW ;  dV = T^T dU ;  dT = dW Kt^T + dU V^T
      T = Linv diag(beta):  dbeta_j += sum_r dT_rj Linv_rj ; dLinv = dT diag(beta)
      dA     = strictly-lower(-Linv^T dLinv Linv^T)
      A_ij = beta_i Gamma_ij (k_i.k_j):  dbeta_i += sum_j dA_ij Gamma_ij (k_i.k_j)
                                          Z_ij = dA_ij beta_i Gamma_ij
      dK     = M^T Qs + Khat-side (exp(G_C-G) * (V_new dS_C^T)) + gamma * dKt + (Z + Z^T) K
      dG     = row sums minus column sums of every Gamma-weighted product
               + gamma/gamma_C terms;  dg = reverse cumsum of dG within the chunk.
    """
    C = q.shape[0]
    pre = chunk_pre(k, v, g, beta)
    G, gam, Gam, Tm, W = pre["G"], pre["gam"], pre["Gam"], pre["T"], pre["W"]
    Linv = pre["Linv"]
    Vn = pre["U"] - W @ S0
    qs = scale * q
    QK = qs @ k.T
    P = QK * Gam
    dec = np.exp(G[-1] - G)
    gC = np.exp(G[-1])
    Khat = k * dec[:, None]

    dVn = P.T @ dO + Khat @ dS_C
    dS0 = (gam[:, None] * qs).T @ dO + gC * dS_C - W.T @ dVn

    dG = np.zeros(C)
    # output, inter-chunk part: O += gamma * (Qs S0)
    dQ_inter = gam[:, None] * (dO @ S0.T)
    dG += np.sum(qs * dQ_inter, axis=1)
    # output, intra-chunk part: O += (QK * Gamma) V_new
    M = (dO @ Vn.T) * Gam
    dQs = dQ_inter + M @ k
    dK = M.T @ qs
    ZP = M * QK
    dG += ZP.sum(axis=1) - ZP.sum(axis=0)
    # state: S_C = gamma_C S0 + Khat^T V_new
    VdS = Vn @ dS_C.T                      # [C, dk] = d(Khat)
    dK += dec[:, None] * VdS
    z = np.sum(k * dec[:, None] * VdS, axis=1)
    dG[-1] += gC * np.sum(S0 * dS_C) + z.sum()
    dG -= z
    # V_new = U - W S0
    dW = -dVn @ S0.T
    dU = dVn
    Kt = gam[:, None] * k
    dV = Tm.T @ dU
    dbeta = None
    if beta is not None:
        dKt = Tm.T @ dW
        dK += gam[:, None] * dKt
        dG += gam * np.sum(k * dKt, axis=1)
        dT = dW @ Kt.T + dU @ v.T
        dbeta = np.sum(dT * Linv, axis=0)
        dLinv = dT * beta[None, :]
        dA = np.tril(-Linv.T @ dLinv @ Linv.T, -1)
        KK = k @ k.T
        dbeta = dbeta + np.sum(dA * Gam * KK, axis=1)
        Z = dA * beta[:, None] * Gam
        dK += (Z + Z.T) @ k
        ZA = Z * KK
        dG += ZA.sum(axis=1) - ZA.sum(axis=0)
    dg = np.cumsum(dG[::-1])[::-1]
    inter = {"V_new": Vn, "dV_new": dVn, "S0": S0, "dS_C": dS_C, "W": W, "U": pre["U"]}
    return scale * dQs, dK, dV, dg, dbeta, dS0, inter


def gdn_fwd(q, k, v, g, beta, S_in=None, scale=1.0, C=64):
    """Chunkwise forward over [B,H,T,.] arrays; ragged tails are zero-padded
    (k = q = v = 0, g = 0, beta = 0 is an exact identity step)."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    qp, kp, vp = (_pad(x, C, 2) for x in (q, k, v))
    gp = _pad(g, C, 2)
    bp = None if beta is None else _pad(beta, C, 2)
    Tp = qp.shape[2]
    o = np.zeros((B, H, Tp, dv))
    S_out = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S_in is None else np.array(S_in[b, h], dtype=np.float64)
            for c0 in range(0, Tp, C):
                sl = slice(c0, c0 + C)
                o_c, S, _ = chunk_fwd(qp[b, h, sl], kp[b, h, sl], vp[b, h, sl], gp[b, h, sl],
                                      None if bp is None else bp[b, h, sl], S, scale)
                o[b, h, sl] = o_c
            S_out[b, h] = S
    return o[:, :, :T], S_out


def gdn_bwd(q, k, v, g, beta, S_in, dO, dS_out=None, scale=1.0, C=64):
    """Chunkwise backward: recompute the chunk-entry states forward, then the
    reverse chain of state gradients, then per-chunk gradients."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    qp, kp, vp, dOp = (_pad(x, C, 2) for x in (q, k, v, dO))
    gp = _pad(g, C, 2)
    bp = None if beta is None else _pad(beta, C, 2)
    Tp = qp.shape[2]
    out = {"dq": np.zeros((B, H, Tp, dk)), "dk": np.zeros((B, H, Tp, dk)),
           "dv": np.zeros((B, H, Tp, dv)), "dg": np.zeros((B, H, Tp)),
           "dbeta": None if beta is None else np.zeros((B, H, Tp)),
           "dS_in": np.zeros((B, H, dk, dv))}
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S_in is None else np.array(S_in[b, h], dtype=np.float64)
            states = []
            for c0 in range(0, Tp, C):
                sl = slice(c0, c0 + C)
                states.append(S)
                _, S, _ = chunk_fwd(qp[b, h, sl], kp[b, h, sl], vp[b, h, sl], gp[b, h, sl],
                                    None if bp is None else bp[b, h, sl], S, scale)
            dS = np.zeros((dk, dv)) if dS_out is None else np.array(dS_out[b, h], dtype=np.float64)
            for ci in range(len(states) - 1, -1, -1):
                c0 = ci * C
                sl = slice(c0, c0 + C)
                dq_, dk_, dv_, dg_, db_, dS, _ = chunk_bwd(
                    qp[b, h, sl], kp[b, h, sl], vp[b, h, sl], gp[b, h, sl],
                    None if bp is None else bp[b, h, sl], states[ci], dOp[b, h, sl], dS, scale)
                out["dq"][b, h, sl] = dq_
                out["dk"][b, h, sl] = dk_
                out["dv"][b, h, sl] = dv_
                out["dg"][b, h, sl] = dg_
                if db_ is not None:
                    out["dbeta"][b, h, sl] = db_
            out["dS_in"][b, h] = dS
    for name in ("dq", "dk", "dv", "dg"):
        out[name] = out[name][:, :, :T]
    if out["dbeta"] is not None:
        out["dbeta"] = out["dbeta"][:, :, :T]
    return out
