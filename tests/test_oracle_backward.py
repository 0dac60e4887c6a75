"""Pins of the fp64 backward oracle (oracle/backward.py), no GPU.

* its Python forward equals the C token recurrence (QDQ off and on);
* QDQ off: central finite differences of the C recurrence match the
  gradients of <o, Wo> + <state_out, Ws> for every input;
* QDQ on: finite differences of the forward whose QDQ residuals are frozen at
  their unperturbed values (so its exact derivative is the straight-through
  gradient) match the backward's gradients;
* closed forms at beta = 0, g = 0 (the state stays H0);
* the chunk-level reverse pass (the adjoint of the chunked WY form, chunk by
  chunk from the forward's chunk-start states) equals the token reverse pass,
  and its sequential part run alone (the state-gradient chain) gives the same
  chunk-end state gradients.
"""

import numpy as np
import pytest

import oracle
from oracle import backward as bw


def _case(rng, lengths, H, d_k, d_v, per_key, state=True):
    T = sum(lengths)
    q = rng.standard_normal((T, H, d_k))
    k = rng.standard_normal((T, H, d_k))
    q /= np.linalg.norm(q, axis=-1, keepdims=True)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, d_v))
    beta = 1 / (1 + np.exp(-rng.standard_normal((T, H))))
    g = -np.log1p(np.exp(-(rng.standard_normal((T, H, d_k) if per_key else (T, H)) + 3)))
    st = rng.standard_normal((len(lengths), H, d_k, d_v)) * 0.3 if state else None
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return dict(q=q, k=k, v=v, g=g, beta=beta, state_in=st), cu


def _loss(o, s, Wo, Ws):
    return float(np.sum(o * Wo) + np.sum(s * Ws))


@pytest.mark.parametrize("per_key", [False, True])
@pytest.mark.parametrize("mode", ["none", "int8_g32", "fp8_tile64"])
def test_python_forward_matches_c_recurrence(per_key, mode):
    rng = np.random.default_rng(90)
    x, cu = _case(rng, [5, 70, 1], 2, 16, 64, per_key)
    o_c, s_c = oracle.recurrence(*x.values(), cu, per_key_gate=per_key, qdq=mode)
    o_p, s_p = bw.forward(*x.values(), cu, per_key_gate=per_key, qdq=mode)
    np.testing.assert_allclose(o_p, o_c, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s_p, s_c, rtol=0, atol=1e-12)


@pytest.mark.parametrize("per_key", [False, True])
def test_backward_matches_finite_differences_qdq_off(per_key):
    rng = np.random.default_rng(91)
    x, cu = _case(rng, [5, 9], 2, 8, 6, per_key)
    o, s = oracle.recurrence(*x.values(), cu, per_key_gate=per_key)
    Wo, Ws = rng.standard_normal(o.shape), rng.standard_normal(s.shape)
    grads = bw.backward(*x.values(), cu, Wo, Ws, per_key_gate=per_key)
    eps = 1e-6
    for name, gr in zip(("q", "k", "v", "g", "beta", "state_in"), grads):
        D = rng.standard_normal(x[name].shape)
        xp, xm = dict(x), dict(x)
        xp[name] = x[name] + eps * D
        xm[name] = x[name] - eps * D
        fd = (_loss(*oracle.recurrence(*xp.values(), cu, per_key_gate=per_key), Wo, Ws)
              - _loss(*oracle.recurrence(*xm.values(), cu, per_key_gate=per_key), Wo, Ws)) / (2 * eps)
        ad = float(np.sum(gr.reshape(D.shape) * D))
        assert abs(fd - ad) <= 1e-6 * max(1.0, abs(ad)), (name, fd, ad)


@pytest.mark.parametrize("per_key", [False, True])
@pytest.mark.parametrize("mode", ["int8_g32", "fp8_tile64"])
def test_backward_is_straight_through(per_key, mode):
    """With QDQ on, the gradient is that of the forward with the QDQ's
    residuals held fixed: the straight-through estimator."""
    rng = np.random.default_rng(92)
    x, cu = _case(rng, [5, 9], 2, 8, 64, per_key)
    every = 4
    o, s, res, _ = bw.forward(*x.values(), cu, per_key_gate=per_key, qdq=mode,
                              boundary_every=every, record=True)
    assert any(np.abs(r).max() > 0 for r in res.values())   # the QDQ does act
    Wo, Ws = rng.standard_normal(o.shape), rng.standard_normal(s.shape)
    grads = bw.backward(*x.values(), cu, Wo, Ws, per_key_gate=per_key, qdq=mode,
                        boundary_every=every)
    eps = 1e-6

    def frozen(xx):
        return bw.forward(*xx.values(), cu, per_key_gate=per_key, qdq=mode,
                          boundary_every=every, residuals=res)

    for name, gr in zip(("q", "k", "v", "g", "beta", "state_in"), grads):
        D = rng.standard_normal(x[name].shape)
        xp, xm = dict(x), dict(x)
        xp[name] = x[name] + eps * D
        xm[name] = x[name] - eps * D
        fd = (_loss(*frozen(xp), Wo, Ws) - _loss(*frozen(xm), Wo, Ws)) / (2 * eps)
        ad = float(np.sum(gr.reshape(D.shape) * D))
        assert abs(fd - ad) <= 1e-6 * max(1.0, abs(ad)), (name, fd, ad)


def test_backward_closed_forms_constant_state():
    """beta = 0, g = 0: H_t = H0, o_t = scale H0^T q_t.  Then dq_t = scale H0
    do_t, dk = dv = 0, dstate_in = Ws + scale sum_t q_t do_t^T, and with
    dH_t = Ws + scale sum_{t' > t} q_t' do_t'^T (+ this token's term):
    dg_t = <H0, dH_t + scale q_t do_t^T>, dbeta_t = (dH^T k_t) . (v_t - H0^T k_t)."""
    rng = np.random.default_rng(93)
    x, cu = _case(rng, [7], 1, 8, 6, False)
    x["beta"] = np.zeros_like(x["beta"])
    x["g"] = np.zeros_like(x["g"])
    o, s = oracle.recurrence(*x.values(), cu, per_key_gate=False)
    Wo, Ws = rng.standard_normal(o.shape), rng.standard_normal(s.shape)
    dq, dk, dv, dg, dbeta, dst = bw.backward(*x.values(), cu, Wo, Ws, per_key_gate=False)
    H0 = x["state_in"][0, 0]
    sc = 1 / np.sqrt(8)
    q, k, v, do = x["q"][:, 0], x["k"][:, 0], x["v"][:, 0], Wo[:, 0]
    np.testing.assert_allclose(dq[:, 0], sc * do @ H0.T, rtol=0, atol=1e-13)
    np.testing.assert_array_equal(dk, 0.0)
    np.testing.assert_array_equal(dv, 0.0)
    np.testing.assert_allclose(dst[0, 0], Ws[0, 0] + sc * q.T @ do, rtol=0, atol=1e-12)
    for t in range(7):
        dHn = Ws[0, 0] + sc * q[t:].T @ do[t:]
        np.testing.assert_allclose(dg[t, 0], np.sum(H0 * dHn), rtol=0, atol=1e-12)
        np.testing.assert_allclose(dbeta[t, 0], (dHn.T @ k[t]) @ (v[t] - H0.T @ k[t]),
                                   rtol=0, atol=1e-12)


@pytest.mark.parametrize("per_key", [False, True])
@pytest.mark.parametrize("mode", ["none", "int8_g32", "fp8_tile64"])
def test_chunked_backward_matches_token_backward(per_key, mode):
    """Ragged sequences (a chunk plus a tail, two chunks plus a tail, one
    short sequence), a random initial state, d_o and d_state_out: every
    gradient of the chunk-level pass equals the token pass's to rounding,
    the gradient at the last chunk's end is d_state_out, and the pass's
    d_state_in is the one it carries out of the first chunk."""
    rng = np.random.default_rng(95 + 2 * per_key + (mode != "none"))
    x, cu = _case(rng, [70, 130, 9], 2, 16, 64, per_key)
    o, s = oracle.recurrence(*x.values(), cu, per_key_gate=per_key, qdq=mode)
    Wo, Ws = rng.standard_normal(o.shape), rng.standard_normal(s.shape)
    ref = bw.backward(*x.values(), cu, Wo, Ws, per_key_gate=per_key, qdq=mode)
    got = bw.chunked_backward(*x.values(), cu, Wo, Ws, per_key_gate=per_key, qdq=mode,
                              record=True)
    for name, a, b in zip(["dq", "dk", "dv", "dg", "dbeta", "dstate_in"], ref, got):
        err = np.abs(a - b).max() / np.abs(a).max()
        assert err < 1e-12, f"{name}: relative difference {err:.2e}"
    dH_end = got[6]
    for s_i, L in enumerate([70, 130, 9]):
        last = (L - 1) // 64
        for h in range(2):
            np.testing.assert_array_equal(dH_end[(s_i, h, last)], Ws[s_i, h])


@pytest.mark.parametrize("per_key", [False, True])
def test_state_gradient_chain_alone(per_key):
    """The sequential part of the chunk adjoint run by itself from the end
    (dH_n of the last chunk = d_state_out) reproduces the chunk-end state
    gradients the full chunk-level pass records, and d_state_in."""
    rng = np.random.default_rng(97 + per_key)
    lengths = [150, 64]
    x, cu = _case(rng, lengths, 1, 16, 64, per_key)
    o, s = oracle.recurrence(*x.values(), cu, per_key_gate=per_key, qdq="int8_g32")
    Wo, Ws = rng.standard_normal(o.shape), rng.standard_normal(s.shape)
    got = bw.chunked_backward(*x.values(), cu, Wo, Ws, per_key_gate=per_key, qdq="int8_g32",
                              record=True)
    dH_end, dst = got[6], got[5]
    _, _, _, states = bw.forward(*x.values(), cu, per_key_gate=per_key, qdq="int8_g32",
                                 record=True)
    scale = 1 / np.sqrt(16)
    for s_i, L in enumerate(lengths):
        t0 = int(cu[s_i])
        dH = Ws[s_i, 0].copy()
        for ci in range((L - 1) // 64, -1, -1):
            np.testing.assert_allclose(dH, dH_end[(s_i, 0, ci)], rtol=1e-12, atol=1e-12)
            a, b = t0 + 64 * ci, t0 + min(64 * ci + 64, L)
            gc = x["g"][a:b, 0] if per_key else x["g"][a:b, 0][:, None] * np.ones((1, 16))
            dH = bw.chunk_state_gradient(x["q"][a:b, 0], x["k"][a:b, 0], x["v"][a:b, 0], gc,
                                         x["beta"][a:b, 0], states[(s_i, 0, 64 * ci)],
                                         Wo[a:b, 0], dH, scale=scale)
        np.testing.assert_allclose(dH, dst[s_i, 0], rtol=1e-12, atol=1e-12)
