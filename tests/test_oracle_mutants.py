"""Planted mistakes in the oracle must fail its pins (CPU only).

The oracle's pins (``test_oracle_codecs.py``, ``test_oracle_recurrence.py``)
claim that a plausible mistake anywhere in it (a dropped term, a wrong sign,
index or operand, a wrong codec constant or rounding rule, a misplaced
boundary) fails at least one of them.  This file checks the claim: each case
plants one such mistake in a copy of the oracle, runs the pins against the
copy, and requires that some pin fails.

* C token recurrence and codecs: a copy of ``gdn_oracle.c`` with one textual
  change is compiled with the oracle's own flags into a temporary library and
  swapped in for the duration of the case;
* fp64 chunked WY form and fp64 backward: a copy of ``oracle/chunked.py`` or
  ``oracle/backward.py`` with one textual change is loaded as a module and
  swapped in for the pin module's reference to it.

The oracle itself is never modified on disk; every case restores it.
"""

import os
import types

import pytest

import oracle
import test_oracle_backward as bwd
import test_oracle_codecs as codecs
import test_oracle_recurrence as rec

# every case ends in seconds; the bound turns a stuck case into a failure
pytestmark = pytest.mark.timeout(300)

# (name, original text, planted text).  Each original occurs exactly once.
C_MUTANTS = [
    ("decay dropped", "Hm[(size_t)i * d_v + j] *= alpha[i];",
     "Hm[(size_t)i * d_v + j] *= 1.0;"),
    ("gate sign", "alpha[i] = exp(per_key_gate ? g[tok * d_k + i] : g[tok]);",
     "alpha[i] = exp(-(per_key_gate ? g[tok * d_k + i] : g[tok]));"),
    ("per-key gate index", "alpha[i] = exp(per_key_gate ? g[tok * d_k + i] : g[tok]);",
     "alpha[i] = exp(per_key_gate ? g[tok * d_k] : g[tok]);"),
    ("delta sign", "u[j] = bt * (vt[j] - a[j]);", "u[j] = bt * (vt[j] + a[j]);"),
    ("beta dropped", "u[j] = bt * (vt[j] - a[j]);", "u[j] = (vt[j] - a[j]);"),
    ("retrieval reads q", "a[j] += Hm[(size_t)i * d_v + j] * kt[i];",
     "a[j] += Hm[(size_t)i * d_v + j] * qt[i];"),
    ("update writes q", "Hm[(size_t)i * d_v + j] += kt[i] * u[j];",
     "Hm[(size_t)i * d_v + j] += qt[i] * u[j];"),
    ("output reads k", "ot[j] += Hm[(size_t)i * d_v + j] * qt[i];",
     "ot[j] += Hm[(size_t)i * d_v + j] * kt[i];"),
    ("output scale dropped", "for (int j = 0; j < d_v; ++j) ot[j] *= scale;",
     "for (int j = 0; j < d_v; ++j) ot[j] *= 1.0;"),
    ("boundary off by one", "int boundary = ((t + 1) % boundary_every == 0) || (t == L - 1);",
     "int boundary = (t % boundary_every == 0) || (t == L - 1);"),
    ("partial last chunk not quantized",
     "int boundary = ((t + 1) % boundary_every == 0) || (t == L - 1);",
     "int boundary = ((t + 1) % boundary_every == 0);"),
    ("FP8 scale constant", "float s = m / 448.0f;", "float s = m / 240.0f;"),
    ("FP8 tile width", "qdq_fp8_tile(X + s * (size_t)d_k * d_v, d_k, d_v, 64,",
     "qdq_fp8_tile(X + s * (size_t)d_k * d_v, d_k, d_v, 32,"),
    ("FP8 ties away from zero", "double n = nearbyint(a / quantum);",
     "double n = floor(a / quantum + 0.5);"),
    ("FP8 subnormal range", "double quantum = (binade < -6) ? ldexp(1.0, -9) : ldexp(1.0, binade - 3);",
     "double quantum = (binade < -7) ? ldexp(1.0, -9) : ldexp(1.0, binade - 3);"),
    ("FP8 no saturation", "r = 448.0;\n    } else {", "r = a;\n    } else {"),
    ("INT8 scale constant", "float s = m / 127.0f;", "float s = m / 128.0f;"),
    ("INT8 ties away from zero", "float c = rintf(t);", "float c = roundf(t);"),
    ("INT8 group along keys", "idx[e] = axis == 1 ? (size_t)line * d_v + pos",
     "idx[e] = axis != 1 ? (size_t)line * d_v + pos"),
]

PY_MUTANTS = [
    ("A keeps its diagonal", "A = np.tril(beta[:, None] * KK, k=-1)",
     "A = np.tril(beta[:, None] * KK, k=0)"),
    ("A without beta", "A = np.tril(beta[:, None] * KK, k=-1)", "A = np.tril(KK, k=-1)"),
    ("W without the gate", "W = T @ (beta[:, None] * (K * gamma))",
     "W = T @ (beta[:, None] * K)"),
    ("U without beta", "U = T @ (beta[:, None] * V)", "U = T @ V"),
    ("V_new sign", "V_new = U - W @ H0", "V_new = U + W @ H0"),
    ("A_qk strict", 'Aqk = np.tril(np.einsum("rc,ic,ric->ri", Q, K, D))',
     'Aqk = np.tril(np.einsum("rc,ic,ric->ri", Q, K, D), k=-1)'),
    ("A_qk transposed decay", 'Aqk = np.tril(np.einsum("rc,ic,ric->ri", Q, K, D))',
     'Aqk = np.tril(np.einsum("rc,ic,irc->ri", Q, K, D))'),
    ("output gate dropped", "O = scale * ((Q * gamma) @ H0 + Aqk @ V_new)",
     "O = scale * (Q @ H0 + Aqk @ V_new)"),
    ("output intra-chunk term dropped", "O = scale * ((Q * gamma) @ H0 + Aqk @ V_new)",
     "O = scale * ((Q * gamma) @ H0)"),
    ("carry decay sign", "decay_to_end = np.exp(G[n - 1][None, :] - G)",
     "decay_to_end = np.exp(G - G[n - 1][None, :])"),
    ("carry without state decay", "Hn = gamma[n - 1][:, None] * H0 +", "Hn = H0 +"),
    ("substitution sign", "T[r, :] -= A[r, i] * T[i, :]", "T[r, :] += A[r, i] * T[i, :]"),
    ("substitution transposed", "T[r, :] -= A[r, i] * T[i, :]", "T[r, :] -= A[i, r] * T[i, :]"),
    ("W QDQ per column", "amax = np.abs(Wf).max(axis=-1, keepdims=True)",
     "amax = np.abs(Wf).max(axis=0, keepdims=True)"),
    ("W QDQ scale constant", "s = (amax / np.float32(448.0)).astype(np.float32)",
     "s = (amax / np.float32(240.0)).astype(np.float32)"),
    ("W QDQ on U instead of W", "    U = T @ (beta[:, None] * V)\n",
     "    U = T @ (beta[:, None] * V)\n    if w_qdq == \"fp8_row\":\n        U = w_row_qdq(U)[0].astype(np.float64)\n"),
    ("W QDQ without the zero guard",
     "safe = np.where(s > 0, s, np.float32(1.0)).astype(np.float32)", "safe = s"),
    ("Neumann sign", "P = -A @ P", "P = A @ P"),
    ("Neumann one term short", "for _ in range(degree):", "for _ in range(degree - 1):"),
]

BWD_MUTANTS = [
    ("dq without the scale", "dq[tok, h] = scale * (Hn @ do[tok, h])",
     "dq[tok, h] = Hn @ do[tok, h]"),
    ("dq from the pre-update state", "dq[tok, h] = scale * (Hn @ do[tok, h])",
     "dq[tok, h] = scale * (Ht @ do[tok, h])"),
    ("output adjoint dropped", "dHn = dH + scale * np.outer(qt, do[tok, h])", "dHn = dH"),
    ("dbeta sign", "dbeta[tok, h] = du @ (vt - a)", "dbeta[tok, h] = du @ (vt + a)"),
    ("dv without beta", "dv[tok, h] = bt * du", "dv[tok, h] = du"),
    ("retrieval adjoint sign", "da = -bt * du", "da = bt * du"),
    ("dk misses the retrieval path", "dkt = dkt + Ht @ da", "dkt = dkt"),
    ("gate adjoint from the decayed state", "dal = np.sum(Hp * dHt, axis=1)",
     "dal = np.sum(Ht * dHt, axis=1)"),
    ("scalar gate adjoint without alpha", "dg[tok, h] = al[0] * dal.sum()",
     "dg[tok, h] = dal.sum()"),
    ("state adjoint not decayed", "dH = al[:, None] * dHt", "dH = dHt"),
    ("reverse pass off the quantized trajectory",
     "per_key_gate=per_key_gate, qdq=qdq,\n                              boundary_every=boundary_every, record=True)",
     "per_key_gate=per_key_gate, qdq=\"none\",\n                              boundary_every=boundary_every, record=True)"),
    ("forward misses the partial last chunk", "return (t + 1) % every == 0 or t == L - 1",
     "return (t + 1) % every == 0"),
    ("chunk: state adjoint without the chunk decay",
     "+ gamma[n - 1][:, None] * dHn - W.T @ dVn", "+ dHn - W.T @ dVn"),
    ("chunk: solve adjoint untransposed", "dA = low_strict * (-(T.T @ dT @ T.T))",
     "dA = low_strict * (-(T @ dT @ T))"),
    ("chunk: gate gradient not summed back", "dg = np.cumsum(dG[::-1], axis=0)[::-1]",
     "dg = dG"),
    ("chunk: end-decay adjoint sign", "dG -= dEK", "dG += dEK"),
    ("chunk: A_qk adjoint above the diagonal", "dAqk = low * (scale * (dO @ Vn.T))",
     "dAqk = scale * (dO @ Vn.T)"),
    ("chunk: dbeta misses the A term", "dbeta += np.sum(dA * KK, axis=1)", "dbeta += 0.0"),
]

BWD_PINS = [
    ("closed forms", bwd.test_backward_closed_forms_constant_state),
    ("python forward = C (gdn, int8)",
     lambda: bwd.test_python_forward_matches_c_recurrence(False, "int8_g32")),
    ("python forward = C (kda, fp8)",
     lambda: bwd.test_python_forward_matches_c_recurrence(True, "fp8_tile64")),
    ("finite differences (gdn)", lambda: bwd.test_backward_matches_finite_differences_qdq_off(False)),
    ("finite differences (kda)", lambda: bwd.test_backward_matches_finite_differences_qdq_off(True)),
    ("straight through (gdn, fp8)", lambda: bwd.test_backward_is_straight_through(False, "fp8_tile64")),
    ("straight through (kda, int8)", lambda: bwd.test_backward_is_straight_through(True, "int8_g32")),
    ("chunked = token (gdn, int8)",
     lambda: bwd.test_chunked_backward_matches_token_backward(False, "int8_g32")),
    ("chunked = token (kda, none)",
     lambda: bwd.test_chunked_backward_matches_token_backward(True, "none")),
]

# The pins, cheapest first: a case stops at the first one that fails.
PINS = [
    ("golden fp8 tile", codecs.test_golden_fp8_tile),
    ("golden int8 group", codecs.test_golden_int8_group),
    ("e4m3 saturates", codecs.test_e4m3_saturates),
    ("e4m3 value set", codecs.test_e4m3_value_set_matches_library),
    ("e4m3 vs library cast", codecs.test_e4m3_rounding_matches_library_cast),
    ("int8 vs torch ops", codecs.test_int8_matches_torch_ops),
    ("fp8 vs torch ops", codecs.test_fp8_matches_torch_ops),
    ("int8 group axis", codecs.test_int8_group_axis),
    ("fp8 tile independence", codecs.test_fp8_tile_independence),
    ("golden gdn", lambda: rec.test_golden_hand_worked("gdn_two_tokens", False)),
    ("golden kda", lambda: rec.test_golden_hand_worked("kda_two_tokens", True)),
    ("beta 0 decays (gdn)", lambda: rec.test_beta_zero_only_decays(False)),
    ("beta 0 decays (kda)", lambda: rec.test_beta_zero_only_decays(True)),
    ("constant state", rec.test_identity_gate_zero_beta_constant),
    ("retrieval (gdn)", lambda: rec.test_delta_rule_retrieval(False)),
    ("retrieval (kda)", lambda: rec.test_delta_rule_retrieval(True)),
    ("orthonormal keys", rec.test_orthonormal_keys_closed_form),
    ("substitution closed forms", rec.test_forward_substitution_small_closed_forms),
    ("solve identities", rec.test_solve_identities_64),
    ("neumann residual", lambda: rec.test_neumann_residual_identity(7)),
    ("neumann product form", lambda: rec.test_neumann_product_form(3)),
    ("neumann short chunks", lambda: rec.test_neumann_exact_on_short_chunks(3)),
    ("chunked = token (gdn)", lambda: rec.test_chunked_wy_equals_token_recurrence(False)),
    ("chunked = token (kda)", lambda: rec.test_chunked_wy_equals_token_recurrence(True)),
    ("qdq placement int8", lambda: rec.test_qdq_placement_prefill("int8_g32")),
    ("qdq placement fp8", lambda: rec.test_qdq_placement_prefill("fp8_tile64")),
    ("qdq placement decode", rec.test_qdq_placement_decode),
    ("w qdq grid and row scale", rec.test_w_row_qdq_grid_and_per_row_scale),
    ("w qdq = tile codec per row", rec.test_w_row_qdq_matches_the_tile_codec_row_by_row),
    ("w qdq beta 0", rec.test_w_qdq_leaves_beta_zero_chunks_alone),
    ("w qdq one-hot keys", rec.test_w_qdq_on_one_hot_keys_is_the_identity_within_an_ulp),
]


def first_failing_pin(pins=None):
    for name, pin in PINS if pins is None else pins:
        try:
            pin()
        except Exception:  # an assertion, or arithmetic the mistake broke
            return name
    return None


def _plant(text, old, new, what):
    assert text.count(old) == 1, f"{what}: the original text must occur once: {old!r}"
    return text.replace(old, new)


def test_pins_pass_on_the_oracle_itself():
    assert first_failing_pin() is None
    assert first_failing_pin(BWD_PINS) is None


@pytest.mark.parametrize("name,old,new", C_MUTANTS, ids=[m[0] for m in C_MUTANTS])
def test_planted_c_mistake_fails_a_pin(name, old, new, tmp_path, monkeypatch):
    src = open(oracle._SRC).read()
    path = tmp_path / "mutant.c"
    path.write_text(_plant(src, old, new, name))
    lib = oracle.build(force=True, src=str(path), out=str(tmp_path / "libmutant.so"))
    monkeypatch.setattr(oracle, "_lib", oracle.bind(lib))
    assert first_failing_pin() is not None, f"no pin fails with the mistake '{name}'"


@pytest.mark.parametrize("name,old,new", PY_MUTANTS, ids=[m[0] for m in PY_MUTANTS])
def test_planted_chunked_mistake_fails_a_pin(name, old, new, monkeypatch):
    path = os.path.join(os.path.dirname(oracle.__file__), "chunked.py")
    src = _plant(open(path).read(), old, new, name)
    mod = types.ModuleType("oracle.chunked_mutant")
    mod.__package__ = "oracle"
    mod.__file__ = path
    exec(compile(src, path + " (mutant)", "exec"), mod.__dict__)
    monkeypatch.setattr(rec, "chunked", mod)
    assert first_failing_pin() is not None, f"no pin fails with the mistake '{name}'"


@pytest.mark.parametrize("name,old,new", BWD_MUTANTS, ids=[m[0] for m in BWD_MUTANTS])
def test_planted_backward_mistake_fails_a_pin(name, old, new, monkeypatch):
    path = os.path.join(os.path.dirname(oracle.__file__), "backward.py")
    src = _plant(open(path).read(), old, new, name)
    mod = types.ModuleType("oracle.backward_mutant")
    mod.__package__ = "oracle"
    mod.__file__ = path
    exec(compile(src, path + " (mutant)", "exec"), mod.__dict__)
    monkeypatch.setattr(bwd, "bw", mod)
    assert first_failing_pin(BWD_PINS) is not None, f"no pin fails with the mistake '{name}'"
