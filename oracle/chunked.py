"""Chunked WY form of the gated delta rule in fp64 (second oracle mode).

TEST INFRASTRUCTURE ONLY (see the package docstring).

For one (sequence, head) and one chunk of n <= 64 tokens starting from state
H0 (H = S^T, [d_k, d_v]), with G_r = sum_{i<=r} g_i the within-chunk
cumulative log gate (scalar for GDN, d_k-vector for KDA) and gamma_r =
exp(G_r), the steps follow the prefix description of the GatedDeltaNet state
QAT pages ("64-token chunks", "WY-transformed W", exact triangular solve as
the default) and the WY decomposition of the delta rule:

  A[r, i]   = beta_r * sum_c k[r,c] k[i,c] exp(G[r,c] - G[i,c])   (i < r), else 0
  T         = (I + A)^-1                  exact forward substitution
  W         = T diag(beta) (K * gamma)    rows of K scaled per channel
  U         = T diag(beta) V
  V_new     = U - W H0
  A_qk[r,i] = sum_c q[r,c] k[i,c] exp(G[r,c] - G[i,c])            (i <= r)
  O         = scale * ((Q * gamma) H0 + A_qk V_new)
  H_n       = diag(gamma_n) H0 + (K * gamma_n / gamma_i)^T V_new

and the state QDQ at the chunk end.  Equality with the token recurrence (QDQ
off) is the pin of this algebra.

Optionally (``w_qdq="fp8_row"``) the WY-transformed W itself is fake-quantized
before it is used, the pages' second, independent QDQ site (PR #2497 "GDN
state/W QAT foundation", What and Usage sections: dynamic FP8 E4M3 on W, the
quantizer keeping the batch, token and head axes): one scale per row of W
(per token and head), amax over the key axis, scale = amax / 448 with a
zero guard, all in fp32 like the state codec (:func:`w_row_qdq`).
"""

from __future__ import annotations

import numpy as np

from . import CHUNK, _f64, dense_cu_seqlens, e4m3 as _e4m3, qdq as _qdq


def w_row_qdq(W):
    """Dynamic FP8 E4M3 QDQ of W [n, d_k], one scale per row: in fp32,
    s = amax / 448 over the row (IEEE division), code = E4M3(fl32(w / s))
    (nearest, ties to even, saturating), y = fl32(code * s); an all-zero row
    stays zero.  Returns (y, codes, scales [n, 1]) as fp32."""
    Wf = np.asarray(W, dtype=np.float32)
    amax = np.abs(Wf).max(axis=-1, keepdims=True)
    s = (amax / np.float32(448.0)).astype(np.float32)
    safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)
    codes = _e4m3((Wf / safe).astype(np.float32))
    y = (codes * safe).astype(np.float32)
    y = np.where(amax > 0, y, np.float32(0.0)).astype(np.float32)
    return y, codes, s


def forward_substitution(A: np.ndarray) -> np.ndarray:
    """T = (I + A)^-1 for strictly lower-triangular A, row by row:
    T_r = e_r - sum_{i<r} A[r, i] T_i."""
    n = A.shape[0]
    T = np.zeros_like(A)
    for r in range(n):
        T[r, r] = 1.0
        for i in range(r):
            T[r, :] -= A[r, i] * T[i, :]
    return T


def neumann_inverse(A: np.ndarray, degree: int) -> np.ndarray:
    """Approximate (I + A)^-1 by the truncated Neumann series
    sum_{n=0}^{degree} (-A)^n (the approximate-inverse solve of the
    experimental GDN/KDA approximate-inverse PR)."""
    n = A.shape[0]
    P = np.eye(n)
    S = np.eye(n)
    for _ in range(degree):
        P = -A @ P
        S = S + P
    return S


def chunk_step(Q, K, V, g, beta, H0, *, per_key_gate: bool, scale: float,
               solve="exact", w_qdq: str = "none"):
    """One chunk: returns (O [n, d_v], H_n [d_k, d_v]) in fp64."""
    n = K.shape[0]
    if per_key_gate:
        G = np.cumsum(g, axis=0)                 # [n, d_k]
    else:
        G = np.cumsum(g, axis=0)[:, None] * np.ones((1, K.shape[1]))
    gamma = np.exp(G)
    # pairwise decays exp(G[r,c] - G[i,c]) for every (r, i, c)
    D = np.exp(G[:, None, :] - G[None, :, :])    # [n, n, d_k]
    KK = np.einsum("rc,ic,ric->ri", K, K, D)
    A = np.tril(beta[:, None] * KK, k=-1)
    if solve == "exact":
        T = forward_substitution(A)
    else:
        T = neumann_inverse(A, int(solve[1]))
    W = T @ (beta[:, None] * (K * gamma))
    if w_qdq == "fp8_row":
        W = w_row_qdq(W)[0].astype(np.float64)
    U = T @ (beta[:, None] * V)
    V_new = U - W @ H0
    Aqk = np.tril(np.einsum("rc,ic,ric->ri", Q, K, D))
    O = scale * ((Q * gamma) @ H0 + Aqk @ V_new)
    decay_to_end = np.exp(G[n - 1][None, :] - G)  # [n, d_k]
    Hn = gamma[n - 1][:, None] * H0 + (K * decay_to_end).T @ V_new
    return O, Hn


def chunked_wy(q, k, v, g, beta, state_in, cu_seqlens, *, per_key_gate: bool,
               qdq: str = "none", chunk: int = CHUNK, solve="exact",
               w_qdq: str = "none"):
    """Chunked prefix over packed sequences (same layout as
    :func:`oracle.recurrence`).  QDQ (if any) runs after every chunk."""
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
    scale = 1.0 / np.sqrt(d_k)
    o = np.zeros((q.shape[0], H, d_v))
    s_out = np.zeros((n_seq, H, d_k, d_v))
    for s in range(n_seq):
        for h in range(H):
            Hs = (st.reshape(n_seq, H, d_k, d_v)[s, h].copy() if st is not None
                  else np.zeros((d_k, d_v)))
            for c0 in range(cu[s], cu[s + 1], chunk):
                c1 = min(c0 + chunk, cu[s + 1])
                O, Hs = chunk_step(q[c0:c1, h], k[c0:c1, h], v[c0:c1, h],
                                   g[c0:c1, h], beta[c0:c1, h], Hs,
                                   per_key_gate=per_key_gate, scale=scale,
                                   solve=solve, w_qdq=w_qdq)
                o[c0:c1, h] = O
                if qdq != "none":
                    Hs = _qdq(Hs.astype(np.float32), qdq)[0].astype(np.float64)
            s_out[s, h] = Hs
    return o, s_out


def chunked_dense(inp: dict, case, **kw):
    cu = inp["cu_seqlens"]
    if cu is None:
        cu = dense_cu_seqlens(case.n_seq, case.T)
    return chunked_wy(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                      inp["state_in"], cu, per_key_gate=case.gate == "per_key",
                      **kw)
