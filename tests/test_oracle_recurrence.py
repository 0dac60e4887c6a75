"""Pins of the oracle's recurrence and of its chunked WY mode (CPU only).

The token recurrence is the decode rule of the GatedDeltaNet / KDA state-QAT
pages (S_t = S_{t-1} diag(alpha_t); u_t = beta_t (v_t - S_t k_t);
S_t += u_t k_t^T; o_t = S_t q_t / sqrt(d_k)); the prefix uses 64-token chunks
in the WY form with an exact triangular solve (PR #2497 What section, PR
#2507 What section); the state QDQ runs at every chunk boundary and after
every decode token.

Pins (each chosen so that a dropped term, a wrong sign or index, or a
transposed operand fails at least one):
 * hand-worked two-token examples, GDN and KDA (tests/golden/hand_worked.json);
 * beta = 0: the state only decays, H_T = diag(exp(sum g)) H_0 (rows = keys);
 * alpha = 1, beta = 0: constant state, o_t = H_0^T q_t / sqrt(d_k);
 * delta-rule retrieval: unit k_t and beta_t = 1 give H_t^T k_t = v_t, so
   q_t = k_t yields o_t = v_t / sqrt(d_k);
 * orthonormal keys, alpha = beta = 1 (d_k != d_v): the closed form
   H_T = H_0 + sum_i k_i (v_i - H_0^T k_i)^T;
 * the chunked WY form equals the token recurrence (QDQ off) for lengths
   1, 63, 64, 65, 200 (GDN and KDA);
 * the forward substitution against 2x2 / 4x4 closed forms and numpy's
   inverse, and the degree-63 Neumann series equals the exact inverse of
   I + A for strictly lower A (nilpotent);
 * QDQ placement: the QDQ run equals the no-QDQ recurrence composed with the
   codec at each 64-token boundary counted from each sequence's start (and
   after every token for decode); outputs use the pre-QDQ state.
"""

import json
import os

import numpy as np
import pytest

import gdn_synth as gs
import oracle
from oracle import chunked

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                   "hand_worked.json")))


def _run(q, k, v, g, beta, state, lengths, per_key, qdq="none", every=64):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return oracle.recurrence(q, k, v, g, beta, state, cu, per_key_gate=per_key,
                             qdq=qdq, boundary_every=every)


def _rand(rng, T, H, d_k, d_v, per_key, unit_keys=True):
    q = rng.standard_normal((T, H, d_k))
    k = rng.standard_normal((T, H, d_k))
    if unit_keys:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, d_v))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    g = -np.log1p(np.exp(-(rng.standard_normal((T, H, d_k) if per_key else (T, H)) + 3)))
    return q, k, v, g, beta


@pytest.mark.parametrize("name,per_key", [("gdn_two_tokens", False),
                                          ("kda_two_tokens", True)])
def test_golden_hand_worked(name, per_key):
    e = GOLD[name]
    f = lambda key: np.array(e[key], dtype=np.float64)
    q, k, v = f("q")[:, None], f("k")[:, None], f("v")[:, None]
    g = f("g")[:, None]
    beta = f("beta")[:, None]
    st = f("state_in")[None, None] if "state_in" in e else None
    o, s = _run(q, k, v, g, beta, st, [2], per_key)
    np.testing.assert_allclose(o[:, 0] * np.sqrt(2), f("o_times_sqrt2"), rtol=0, atol=1e-14)
    np.testing.assert_allclose(s[0, 0], f("state_out"), rtol=0, atol=1e-14)


@pytest.mark.parametrize("per_key", [False, True])
def test_beta_zero_only_decays(per_key):
    rng = np.random.default_rng(11)
    T, H, dk, dv = 70, 2, 64, 128
    q, k, v, g, beta = _rand(rng, T, H, dk, dv, per_key)
    beta[:] = 0.0
    H0 = rng.standard_normal((1, H, dk, dv))
    o, s = _run(q, k, v, g, beta, H0, [T], per_key)
    G = np.cumsum(g, axis=0)                     # [T, H] or [T, H, dk]
    for h in range(H):
        gam = np.exp(G[:, h]) if per_key else np.exp(G[:, h])[:, None] * np.ones(dk)
        np.testing.assert_allclose(s[0, h], gam[-1][:, None] * H0[0, h], rtol=1e-12)
        for t in (0, 33, T - 1):
            exp_o = (gam[t][:, None] * H0[0, h]).T @ q[t, h] / np.sqrt(dk)
            np.testing.assert_allclose(o[t, h], exp_o, rtol=1e-11, atol=1e-14)


def test_identity_gate_zero_beta_constant():
    rng = np.random.default_rng(12)
    T, H, dk, dv = 40, 3, 128, 64
    q, k, v, g, beta = _rand(rng, T, H, dk, dv, False)
    g[:] = 0.0
    beta[:] = 0.0
    H0 = rng.standard_normal((1, H, dk, dv))
    o, s = _run(q, k, v, g, beta, H0, [T], False)
    np.testing.assert_array_equal(s, H0)
    exp_o = np.einsum("hkv,thk->thv", H0[0], q) / np.sqrt(dk)
    np.testing.assert_allclose(o, exp_o, rtol=1e-13, atol=1e-15)


@pytest.mark.parametrize("per_key", [False, True])
def test_delta_rule_retrieval(per_key):
    """beta = 1, unit key: the update writes v_t exactly under k_t."""
    rng = np.random.default_rng(13)
    T, H, dk, dv = 50, 2, 64, 128
    q, k, v, g, beta = _rand(rng, T, H, dk, dv, per_key)
    beta[:] = 1.0
    q = k.copy()
    H0 = rng.standard_normal((1, H, dk, dv)) * 0.3
    o, s = _run(q, k, v, g, beta, H0, [T], per_key)
    np.testing.assert_allclose(o * np.sqrt(dk), v, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s[0].transpose(0, 2, 1) @ k[-1][:, :, None],
                               v[-1][:, :, None], atol=1e-12)


def test_orthonormal_keys_closed_form():
    rng = np.random.default_rng(14)
    T, H, dk, dv = 48, 1, 64, 128
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    k = Qm[:, :T].T[:, None, :]                  # T orthonormal keys
    q = rng.standard_normal((T, H, dk))
    v = rng.standard_normal((T, H, dv))
    g = np.zeros((T, H))
    beta = np.ones((T, H))
    H0 = rng.standard_normal((1, H, dk, dv))
    o, s = _run(q, k, v, g, beta, H0, [T], False)
    expect = H0[0, 0].copy()
    for i in range(T):
        expect += np.outer(k[i, 0], v[i, 0] - H0[0, 0].T @ k[i, 0])
    np.testing.assert_allclose(s[0, 0], expect, rtol=0, atol=1e-12)


@pytest.mark.parametrize("per_key", [False, True])
def test_chunked_wy_equals_token_recurrence(per_key):
    rng = np.random.default_rng(15)
    lengths = [1, 63, 64, 65, 200]
    T, H, dk, dv = sum(lengths), 2, 64, 128
    q, k, v, g, beta = _rand(rng, T, H, dk, dv, per_key)
    H0 = rng.standard_normal((len(lengths), H, dk, dv)) * 0.05
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    o1, s1 = oracle.recurrence(q, k, v, g, beta, H0, cu, per_key_gate=per_key)
    o2, s2 = chunked.chunked_wy(q, k, v, g, beta, H0, cu, per_key_gate=per_key)
    assert np.abs(o1 - o2).max() <= 1e-12 * np.abs(o1).max()
    assert np.abs(s1 - s2).max() <= 1e-12 * np.abs(s1).max()


def test_forward_substitution_small_closed_forms():
    A2 = np.array([[0.0, 0.0], [0.7, 0.0]])
    np.testing.assert_array_equal(chunked.forward_substitution(A2),
                                  np.array([[1.0, 0.0], [-0.7, 1.0]]))
    a, b, c = 0.5, -0.25, 2.0
    A3 = np.array([[0, 0, 0], [a, 0, 0], [b, c, 0]], dtype=np.float64)
    # (I + A)^-1 for unit lower 3x3 by cofactors: [[1,0,0],[-a,1,0],[ac-b,-c,1]]
    np.testing.assert_allclose(chunked.forward_substitution(A3),
                               np.array([[1, 0, 0], [-a, 1, 0], [a * c - b, -c, 1]]),
                               rtol=0, atol=1e-15)
    rng = np.random.default_rng(16)
    A4 = np.tril(rng.standard_normal((4, 4)), -1)
    np.testing.assert_allclose(chunked.forward_substitution(A4),
                               np.linalg.inv(np.eye(4) + A4), rtol=1e-13, atol=1e-14)


def test_solve_identities_64():
    rng = np.random.default_rng(17)
    K = rng.standard_normal((64, 128))
    K /= np.linalg.norm(K, axis=1, keepdims=True)
    beta = 1 / (1 + np.exp(-rng.standard_normal(64)))
    A = np.tril(beta[:, None] * (K @ K.T), -1)
    T = chunked.forward_substitution(A)
    np.testing.assert_allclose(T @ (np.eye(64) + A), np.eye(64), atol=1e-12)
    # strictly lower A is nilpotent: the degree-63 Neumann series is exact
    np.testing.assert_allclose(chunked.neumann_inverse(A, 63), T, atol=1e-12)
    # a low degree is only an approximation
    assert np.abs(chunked.neumann_inverse(A, 3) - T).max() > 1e-6


@pytest.mark.parametrize("degree", [1, 3, 7, 15, 31])
def test_neumann_residual_identity(degree):
    """(I + A) sum_{n<=d} (-A)^n = I - (-A)^(d+1): a dropped or extra term, a
    sign slip or an off-by-one degree breaks it.  The right side comes from
    numpy's matrix power, not from the oracle's series."""
    rng = np.random.default_rng(40 + degree)
    A = np.tril(rng.standard_normal((64, 64)) * 0.15, -1)
    Td = chunked.neumann_inverse(A, degree)
    rhs = np.eye(64) - np.linalg.matrix_power(-A, degree + 1)
    np.testing.assert_allclose((np.eye(64) + A) @ Td, rhs, rtol=0, atol=1e-12)


@pytest.mark.parametrize("m", [1, 2, 3, 4, 5, 6])
def test_neumann_product_form(m):
    """For degree 2^m - 1 the series factors as prod_{i<m} (I + X^(2^i)),
    X = -A (the GPU evaluates this form)."""
    rng = np.random.default_rng(60 + m)
    A = np.tril(rng.standard_normal((64, 64)) * 0.15, -1)
    X = -A
    P = np.eye(64)
    for i in range(m):
        P = P @ (np.eye(64) + np.linalg.matrix_power(X, 2 ** i))
    np.testing.assert_allclose(chunked.neumann_inverse(A, 2 ** m - 1), P, rtol=0, atol=1e-12)


@pytest.mark.parametrize("degree", [3, 7])
def test_neumann_exact_on_short_chunks(degree):
    """A chunk of n tokens has an n x n strictly lower A, so A^n = 0: the
    degree-d series is the exact inverse whenever n <= d + 1.  Sequences of
    n <= d + 1 tokens give the exact chunked result (and the token
    recurrence); a full 64-token chunk does not."""
    rng = np.random.default_rng(70 + degree)
    lengths = [1, degree, degree + 1, 64]
    T, H, dk, dv = sum(lengths), 2, 32, 16
    q, k, v, g, beta = _rand(rng, T, H, dk, dv, True)
    H0 = rng.standard_normal((len(lengths), H, dk, dv)) * 0.05
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    o_e, s_e = chunked.chunked_wy(q, k, v, g, beta, H0, cu, per_key_gate=True)
    o_n, s_n = chunked.chunked_wy(q, k, v, g, beta, H0, cu, per_key_gate=True,
                                  solve=("neumann", degree))
    o_r, _ = _run(q, k, v, g, beta, H0, lengths, True)
    np.testing.assert_allclose(o_e, o_r, rtol=0, atol=1e-12)
    short = slice(0, int(cu[3]))
    np.testing.assert_allclose(o_n[short], o_e[short], rtol=0, atol=1e-12)
    np.testing.assert_allclose(s_n[:3], s_e[:3], rtol=0, atol=1e-12)
    assert np.abs(o_n[int(cu[3]):] - o_e[int(cu[3]):]).max() > 1e-9
    assert np.abs(s_n[3] - s_e[3]).max() > 1e-9


@pytest.mark.parametrize("mode", ["int8_g32", "fp8_tile64"])
def test_qdq_placement_prefill(mode):
    rng = np.random.default_rng(18)
    lengths = [150, 64, 30]
    T, H, dk, dv = sum(lengths), 2, 64, 128
    q, k, v, g, beta = _rand(rng, T, H, dk, dv, False)
    H0 = rng.standard_normal((len(lengths), H, dk, dv)) * 0.05
    o_q, s_q = _run(q, k, v, g, beta, H0, lengths, False, qdq=mode)
    o_n, _ = _run(q, k, v, g, beta, H0, lengths, False)
    starts = np.concatenate([[0], np.cumsum(lengths)])
    for si, L in enumerate(lengths):
        st = H0[si:si + 1]                       # the incoming state is not QDQ'd
        for c0 in range(0, L, 64):
            c1 = min(c0 + 64, L)
            sl = slice(starts[si] + c0, starts[si] + c1)
            o_c, s_c = _run(q[sl], k[sl], v[sl], g[sl], beta[sl], st,
                            [c1 - c0], False)
            np.testing.assert_allclose(o_q[sl], o_c, rtol=0, atol=1e-12)
            st = oracle.qdq(s_c.astype(np.float32), mode)[0].astype(np.float64)
        np.testing.assert_array_equal(s_q[si], st[0])
    # outputs of the first chunk come before any QDQ
    np.testing.assert_array_equal(o_q[:64], o_n[:64])


def test_qdq_placement_decode():
    rng = np.random.default_rng(19)
    S, N, H, dk, dv = 5, 2, 2, 64, 64
    dq, dk_, dv_, dg, db = (np.moveaxis(x.reshape(N, S, H, -1) if x.ndim == 3 else
                                        x.reshape(N, S, H), 0, 1)
                            for x in _rand(rng, N * S, H, dk, dv, False))
    dg = dg.reshape(S, N, H)
    db = db.reshape(S, N, H)
    H0 = rng.standard_normal((N, H, dk, dv)) * 0.05
    o, s = oracle.decode(dq, dk_, dv_, dg, db, H0, per_key_gate=False, qdq="int8_g32")
    st = H0
    for t in range(S):
        cu = np.arange(N + 1, dtype=np.int32)
        o_t, s_t = oracle.recurrence(dq[t], dk_[t], dv_[t], dg[t], db[t], st, cu,
                                     per_key_gate=False)
        np.testing.assert_allclose(o[t], o_t, rtol=0, atol=1e-12)
        st = oracle.qdq(s_t.astype(np.float32), "int8_g32")[0].astype(np.float64)
    np.testing.assert_array_equal(s, st)


def test_generator_inputs_run_tiny():
    """The tiny workload (fp32, INT8 g32) runs end to end through the oracle;
    the returned state is on the INT8 grid."""
    case = gs.CONFIGS["tiny"]
    inp = gs.generate(case)
    o, s, codes, scales = oracle.prefill(inp, case, want_codes=True)
    assert np.all(np.isfinite(o))
    rebuilt = (codes.reshape(1, 2, 64, 2, 32) *
               scales.reshape(1, 2, 64, 2, 1)).reshape(s.shape).astype(np.float32)
    np.testing.assert_array_equal(s.astype(np.float32), rebuilt)


# ---------------------------------------------------------------- W QDQ ----
# The optional FP8 QDQ of the WY-transformed W (one dynamic scale per row of
# W, i.e. per token and head, over the key axis; PR #2497 "GDN state/W QAT
# foundation", What and Usage sections).

def _w_rows(seed=3):
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((64, 128)) * np.exp2(rng.integers(-30, 20, (64, 1)))
    W[5] = 0.0                      # an all-zero row
    W[9] = 0.0
    W[9, 17] = -3.25                # a row with one nonzero element
    return W.astype(np.float32)


def test_w_row_qdq_grid_and_per_row_scale():
    """Every value is code * s_row with code on the E4M3 grid; the row's
    largest magnitude maps to exactly +-448 (so the scale is the row's own,
    not a column's or the tensor's); a zero row stays zero; idempotent."""
    import torch
    from test_oracle_codecs import e4m3_value_set
    W = _w_rows()
    y, codes, s = chunked.w_row_qdq(W)
    grid = e4m3_value_set()
    assert set(np.unique(codes).astype(np.float64)) <= grid
    nz = np.abs(W).max(axis=1) > 0
    np.testing.assert_array_equal(np.abs(codes[nz]).max(axis=1), 448.0)
    assert not y[~nz].any() and not codes[~nz].any()
    np.testing.assert_array_equal(y[nz], (codes[nz] * s[nz]).astype(np.float32))
    # the code rounding against the library's float8 cast of the same quotients
    q = (W[nz] / s[nz]).astype(np.float32)
    lib = torch.from_numpy(q).to(torch.float8_e4m3fn).float().numpy()
    np.testing.assert_array_equal(codes[nz], lib)
    y2 = chunked.w_row_qdq(y)[0]
    np.testing.assert_array_equal(y2, y)


def test_w_row_qdq_matches_the_tile_codec_row_by_row():
    """Each row on its own in column 0 of an otherwise zero [128 x 64] FP8
    tile goes through the C state codec (an independent implementation of
    the same scale and rounding) to the same values."""
    W = _w_rows(4)
    y = chunked.w_row_qdq(W)[0]
    tiles = np.zeros((W.shape[0], 128, 64), np.float32)
    tiles[:, :, 0] = W
    ref = oracle.qdq(tiles, "fp8_tile64")[0][:, :, 0]
    np.testing.assert_array_equal(y, ref)


def test_w_qdq_leaves_beta_zero_chunks_alone():
    """beta = 0 makes W = 0 (zero rows): the W QDQ changes nothing."""
    case = gs.Case("wq0", n_seq=1, H=2, d_k=64, d_v=64, T=100, dtype="f32",
                   qdq="fp8_tile64", state="normal", seed=131)
    inp = gs.generate(case)
    inp["beta"] = np.zeros_like(inp["beta"])
    a = chunked.chunked_dense(inp, case, qdq="fp8_tile64")
    b = chunked.chunked_dense(inp, case, qdq="fp8_tile64", w_qdq="fp8_row")
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_w_qdq_on_one_hot_keys_is_the_identity_within_an_ulp():
    """Mutually orthogonal one-hot keys give A = 0, T = I and W rows
    beta_t gamma_t e_t: a one-element row keeps its value up to the fp32
    rounding of its scale, so the chunk's result moves by at most a few
    ulp - whereas a QDQ applied to U, V or K (dense rows) moves it by the
    FP8 step."""
    import torch
    n, d = 40, 64
    q = torch.randn((1, n, 1, d), generator=torch.Generator().manual_seed(5))
    k = torch.zeros((1, n, 1, d))
    k[0, np.arange(n), 0, np.arange(n)] = 1.0
    v = torch.randn((1, n, 1, d), generator=torch.Generator().manual_seed(6))
    g = torch.full((1, n, 1), -0.05)
    beta = torch.full((1, n, 1), 0.7)
    st = torch.randn((1, 1, d, d), generator=torch.Generator().manual_seed(7)) * 0.1
    cu = np.array([0, n])
    a = chunked.chunked_wy(q, k, v, g, beta, st, cu, per_key_gate=False)
    b = chunked.chunked_wy(q, k, v, g, beta, st, cu, per_key_gate=False, w_qdq="fp8_row")
    assert np.abs(b[0] - a[0]).max() <= 1e-6 * np.abs(a[0]).max()
    assert np.abs(b[1] - a[1]).max() <= 1e-6 * np.abs(a[1]).max()
