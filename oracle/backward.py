"""Backward pass of the gated delta rule with a fake-quantized state, fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The GatedDeltaNet/KDA state QAT pages simulate the state quantization in
training and differentiate through it with the straight-through estimator
(the QDQ is the identity in the backward pass; PR #2497 What section, state
QAT with fake quantization).  Forward, per (sequence, head) and token t
(H = S^T, [d_k, d_v]; the same steps as :func:`oracle.recurrence`):

    alpha = exp(g_t)                      (scalar, or one per key for KDA)
    Ht    = diag(alpha) H_{t-1}
    a     = Ht^T k_t,   u = beta_t (v_t - a)
    Hn    = Ht + k_t u^T
    o_t   = scale Hn^T q_t                (scale = 1 / sqrt(d_k))
    H_t   = QDQ(Hn) at a chunk boundary, else Hn

Reverse, with dH the gradient of the loss with respect to H_t (at the end:
``dstate_out``) and the QDQ passed straight through:

    dHn   = dH + scale q_t do_t^T;         dq_t = scale Hn do_t
    du    = dHn^T k_t;                     dk_t = dHn u
    dbeta = du . (v_t - a);  dv_t = beta du;  da = -beta du
    dHt   = dHn + k_t da^T;                dk_t += Ht da
    dalpha_i = sum_j H_{t-1}[i, j] dHt[i, j]   (summed over i for a scalar gate)
    dg_t  = alpha * dalpha;                dH_{t-1} = diag(alpha) dHt

Pins (tests/test_oracle_backward.py): central finite differences of the C
token recurrence with QDQ off; with QDQ on, finite differences of the forward
whose QDQ residuals QDQ(Hn) - Hn are frozen at their unperturbed values (its
exact derivative is the straight-through gradient); closed forms.  The
chunk-level pass at the end of this file is pinned to the token pass.
"""

from __future__ import annotations

import numpy as np

from . import CHUNK, _f64, qdq as _qdq


def _prep(q, k, v, g, beta, state_in, cu_seqlens, per_key_gate):
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    d_k, d_v = q.shape[-1], v.shape[-1]
    H = v.shape[-2]
    q = q.reshape(-1, H, d_k)
    k = k.reshape(-1, H, d_k)
    v = v.reshape(-1, H, d_v)
    beta = beta.reshape(-1, H)
    g = g.reshape((-1, H, d_k) if per_key_gate else (-1, H))
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    n_seq = cu.size - 1
    st = _f64(state_in)
    st = (np.zeros((n_seq, H, d_k, d_v)) if st is None else st.reshape(n_seq, H, d_k, d_v))
    return q, k, v, g, beta, st, cu


def _alpha(g_t, d_k, per_key_gate):
    return np.exp(g_t) if per_key_gate else np.full(d_k, np.exp(g_t))


def _boundary(t, L, every):
    return (t + 1) % every == 0 or t == L - 1


def forward(q, k, v, g, beta, state_in, cu_seqlens, *, per_key_gate: bool,
            qdq: str = "none", boundary_every: int = CHUNK, residuals=None,
            record: bool = False):
    """fp64 forward in Python (pinned to the C recurrence by the tests).

    ``residuals``: None (apply the QDQ), or a dict {(s, h, t): R} of frozen
    QDQ residuals added instead at the boundaries.  With ``record`` also
    returns the residuals this run applied and the per-token pre-token states.
    Returns ``(o, state_out[, residuals, states])``."""
    q, k, v, g, beta, st, cu = _prep(q, k, v, g, beta, state_in, cu_seqlens, per_key_gate)
    n_seq, H, d_k, d_v = st.shape
    scale = 1.0 / np.sqrt(d_k)
    o = np.zeros((q.shape[0], H, d_v))
    s_out = np.zeros_like(st)
    res_out, states = {}, {}
    for s in range(n_seq):
        for h in range(H):
            Hm = st[s, h].copy()
            t0, L = int(cu[s]), int(cu[s + 1] - cu[s])
            for t in range(L):
                tok = t0 + t
                if record:
                    states[(s, h, t)] = Hm.copy()
                al = _alpha(g[tok, h], d_k, per_key_gate)
                Ht = al[:, None] * Hm
                a = Ht.T @ k[tok, h]
                u = beta[tok, h] * (v[tok, h] - a)
                Hn = Ht + np.outer(k[tok, h], u)
                o[tok, h] = scale * (Hn.T @ q[tok, h])
                if _boundary(t, L, boundary_every) and qdq != "none":
                    if residuals is None:
                        R = _qdq(Hn.astype(np.float32), qdq)[0].astype(np.float64) - Hn
                    else:
                        R = residuals[(s, h, t)]
                    res_out[(s, h, t)] = R
                    Hn = Hn + R
                Hm = Hn
            s_out[s, h] = Hm
    if record:
        return o, s_out, res_out, states
    return o, s_out


def backward(q, k, v, g, beta, state_in, cu_seqlens, do, dstate_out, *,
             per_key_gate: bool, qdq: str = "none", boundary_every: int = CHUNK):
    """Gradients of <o, do> + <state_out, dstate_out> with the QDQ passed
    straight through.  Returns ``dq, dk, dv, dg, dbeta, dstate_in`` shaped
    like q, k, v, g, beta ([total_T, H, ...]) and [n_seq, H, d_k, d_v]."""
    _, _, _, states = forward(q, k, v, g, beta, state_in, cu_seqlens,
                              per_key_gate=per_key_gate, qdq=qdq,
                              boundary_every=boundary_every, record=True)
    q, k, v, g, beta, st, cu = _prep(q, k, v, g, beta, state_in, cu_seqlens, per_key_gate)
    n_seq, H, d_k, d_v = st.shape
    scale = 1.0 / np.sqrt(d_k)
    do = _f64(do).reshape(-1, H, d_v)
    dso = (np.zeros_like(st) if dstate_out is None
           else _f64(dstate_out).reshape(n_seq, H, d_k, d_v))
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg, dbeta = np.zeros_like(g), np.zeros_like(beta)
    dst = np.zeros_like(st)
    for s in range(n_seq):
        for h in range(H):
            dH = dso[s, h].copy()
            t0, L = int(cu[s]), int(cu[s + 1] - cu[s])
            for t in range(L - 1, -1, -1):
                tok = t0 + t
                Hp = states[(s, h, t)]
                al = _alpha(g[tok, h], d_k, per_key_gate)
                kt, qt, vt, bt = k[tok, h], q[tok, h], v[tok, h], beta[tok, h]
                Ht = al[:, None] * Hp
                a = Ht.T @ kt
                u = bt * (vt - a)
                Hn = Ht + np.outer(kt, u)
                # (a boundary's QDQ is the identity here: dH reaches Hn as is)
                dHn = dH + scale * np.outer(qt, do[tok, h])
                dq[tok, h] = scale * (Hn @ do[tok, h])
                du = dHn.T @ kt
                dkt = dHn @ u
                dbeta[tok, h] = du @ (vt - a)
                dv[tok, h] = bt * du
                da = -bt * du
                dHt = dHn + np.outer(kt, da)
                dkt = dkt + Ht @ da
                dk[tok, h] = dkt
                dal = np.sum(Hp * dHt, axis=1)
                if per_key_gate:
                    dg[tok, h] = al * dal
                else:
                    dg[tok, h] = al[0] * dal.sum()
                dH = al[:, None] * dHt
            dst[s, h] = dH
    return dq, dk, dv, dg, dbeta, dst


# ----------------------------------------------------------------------------
# Chunk-level reverse pass
#
# The adjoint of the chunked WY form (:func:`oracle.chunked.chunk_step`), one
# 64-token chunk at a time from the chunk-start states of the forward: the
# shape a chunked kernel computes.  The pages fix only the forward steps and
# the straight-through QDQ; this is the exact derivative of those steps,
# taken through each product in reverse order, and its pin is equality with
# :func:`backward` (itself pinned by finite differences).  With G the
# within-chunk cumulative log gate ([n, d_k]; a scalar gate broadcast over
# the keys), D[r, i, c] = exp(G[r, c] - G[i, c]), gamma = exp(G),
# E = exp(G[n-1] - G), and the forward's A, T, W, U, V_new, A_qk:
#
#   dV_new = scale A_qk^T dO + (K * E) dH_n
#   dH_0   = scale (Q * gamma)^T dO + diag(gamma_n) dH_n - W^T dV_new
#   dA_qk  = lower(scale dO V_new^T),       dU = dV_new,  dW = -dV_new H_0^T
#   dT     = dW (beta K gamma)^T + dU (beta V)^T
#   dA     = strict_lower(-T^T dT T^T)
#
# then the products A = strict_lower(beta K K^T * D), A_qk = lower(Q K^T * D),
# W = T beta (K * gamma), U = T beta V, O and H_n give dq, dk, dv, dbeta and
# dG, and dg_t = sum_{r >= t} dG_r (summed over the keys for a scalar gate).
# ----------------------------------------------------------------------------

def chunk_backward_step(Q, K, V, g, beta, H0, dO, dHn, *, scale: float):
    """Reverse of one chunk (per-key gate form, fp64).  ``g`` is [n, d_k]
    (broadcast a scalar gate before the call).  Returns
    ``dQ, dK, dV, dg [n, d_k], dbeta [n], dH0``."""
    n, d_k = K.shape
    G = np.cumsum(g, axis=0)
    gamma = np.exp(G)
    D = np.exp(G[:, None, :] - G[None, :, :])          # [n, n, d_k]
    E = np.exp(G[n - 1][None, :] - G)                   # [n, d_k]
    low_strict = np.tril(np.ones((n, n)), k=-1)
    low = np.tril(np.ones((n, n)))
    # forward quantities
    KK = np.einsum("rc,ic,ric->ri", K, K, D)
    A = low_strict * (beta[:, None] * KK)
    T = np.linalg.inv(np.eye(n) + A)
    BKg = beta[:, None] * (K * gamma)
    BV = beta[:, None] * V
    W = T @ BKg
    U = T @ BV
    Vn = U - W @ H0
    QK = np.einsum("rc,ic,ric->ri", Q, K, D)
    Aqk = low * QK
    # outputs and the state
    dVn = scale * (Aqk.T @ dO) + (K * E) @ dHn
    dH0 = scale * ((Q * gamma).T @ dO) + gamma[n - 1][:, None] * dHn - W.T @ dVn
    dAqk = low * (scale * (dO @ Vn.T))
    dQg = scale * (dO @ H0.T)                           # d(Q * gamma)
    dKe = Vn @ dHn.T                                    # d(K * E)
    dQ = dQg * gamma
    dK = dKe * E
    dgam = dQg * Q
    dG = np.zeros_like(G)
    dEK = dKe * K * E                                   # d/dG of E terms
    dG -= dEK
    dG[n - 1] += dEK.sum(axis=0)
    dG[n - 1] += np.sum(H0 * dHn, axis=1) * gamma[n - 1]
    # V_new = U - W H0
    dU = dVn
    dW = -dVn @ H0.T
    # W = T (beta K gamma), U = T (beta V)
    dT = dW @ BKg.T + dU @ BV.T
    dBKg = T.T @ dW
    dBV = T.T @ dU
    dbeta = np.sum(dBKg * K * gamma, axis=1) + np.sum(dBV * V, axis=1)
    dK += beta[:, None] * dBKg * gamma
    dgam += beta[:, None] * dBKg * K
    dV = beta[:, None] * dBV
    # T = (I + A)^-1
    dA = low_strict * (-(T.T @ dT @ T.T))
    # A = strict_lower(beta K K^T * D)
    dbeta += np.sum(dA * KK, axis=1)
    dKK = beta[:, None] * dA
    dK += np.einsum("ri,ic,ric->rc", dKK, K, D) + np.einsum("ri,rc,ric->ic", dKK, K, D)
    dD = np.einsum("ri,rc,ic->ric", dKK, K, K)
    # A_qk = lower(Q K^T * D)
    dQ += np.einsum("ri,ic,ric->rc", dAqk, K, D)
    dK += np.einsum("ri,rc,ric->ic", dAqk, Q, D)
    dD += np.einsum("ri,rc,ic->ric", dAqk, Q, K)
    # D[r, i] = exp(G_r - G_i), gamma = exp(G)
    dDD = dD * D
    dG += dDD.sum(axis=1) - dDD.sum(axis=0)
    dG += dgam * gamma
    # G = cumsum(g)
    dg = np.cumsum(dG[::-1], axis=0)[::-1]
    return dQ, dK, dV, dg, dbeta, dH0


def chunked_backward(q, k, v, g, beta, state_in, cu_seqlens, do, dstate_out, *,
                     per_key_gate: bool, qdq: str = "none", chunk: int = CHUNK,
                     record: bool = False):
    """Chunk-level reverse pass, same arguments and returns as
    :func:`backward` (QDQ at every chunk end, passed straight through).  The
    chunk-start states come from the token forward.  With ``record`` also
    returns ``{(s, h, c): dH}``, the gradient with respect to each chunk's
    end state."""
    _, _, _, states = forward(q, k, v, g, beta, state_in, cu_seqlens,
                              per_key_gate=per_key_gate, qdq=qdq,
                              boundary_every=chunk, record=True)
    q, k, v, g, beta, st, cu = _prep(q, k, v, g, beta, state_in, cu_seqlens, per_key_gate)
    n_seq, H, d_k, d_v = st.shape
    scale = 1.0 / np.sqrt(d_k)
    do = _f64(do).reshape(-1, H, d_v)
    dso = (np.zeros_like(st) if dstate_out is None
           else _f64(dstate_out).reshape(n_seq, H, d_k, d_v))
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    dg, dbeta = np.zeros_like(g), np.zeros_like(beta)
    dst = np.zeros_like(st)
    dH_end = {}
    for s in range(n_seq):
        for h in range(H):
            dH = dso[s, h].copy()
            t0, L = int(cu[s]), int(cu[s + 1] - cu[s])
            starts = list(range(0, L, chunk))
            for ci in range(len(starts) - 1, -1, -1):
                c0 = starts[ci]
                c1 = min(c0 + chunk, L)
                a, b = t0 + c0, t0 + c1
                gc = g[a:b, h] if per_key_gate else g[a:b, h][:, None] * np.ones((1, d_k))
                dH_end[(s, h, ci)] = dH.copy()
                dQ, dK, dV, dgc, dbc, dH = chunk_backward_step(
                    q[a:b, h], k[a:b, h], v[a:b, h], gc, beta[a:b, h],
                    states[(s, h, c0)], do[a:b, h], dH, scale=scale)
                dq[a:b, h], dk[a:b, h], dv[a:b, h] = dQ, dK, dV
                dg[a:b, h] = dgc if per_key_gate else dgc.sum(axis=1)
                dbeta[a:b, h] = dbc
            dst[s, h] = dH
    if record:
        return dq, dk, dv, dg, dbeta, dst, dH_end
    return dq, dk, dv, dg, dbeta, dst


def chunk_state_gradient(Q, K, V, g, beta, H0, dO, dHn, *, scale: float):
    """The sequential part of :func:`chunk_backward_step` alone: the gradient
    with respect to the chunk-start state,
    dH0 = diag(gamma_n) dHn - W^T (K * E) dHn + scale ((Q * gamma)^T - W^T A_qk^T) dO,
    whose bracketed term and W, K * E, A_qk do not depend on dHn."""
    n, d_k = K.shape
    G = np.cumsum(g, axis=0)
    gamma = np.exp(G)
    D = np.exp(G[:, None, :] - G[None, :, :])
    E = np.exp(G[n - 1][None, :] - G)
    A = np.tril(beta[:, None] * np.einsum("rc,ic,ric->ri", K, K, D), k=-1)
    T = np.linalg.inv(np.eye(n) + A)
    W = T @ (beta[:, None] * (K * gamma))
    Aqk = np.tril(np.einsum("rc,ic,ric->ri", Q, K, D))
    bracket = scale * ((Q * gamma).T @ dO - W.T @ (Aqk.T @ dO))
    return gamma[n - 1][:, None] * dHn - W.T @ ((K * E) @ dHn) + bracket
