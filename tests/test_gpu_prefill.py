"""GPU parity of gdn_prefill (through the C ABI) against the CPU oracle.

* codec alone: one token with g = 0, beta = 0 leaves the state unchanged
  before the final QDQ, so state_out must equal the oracle's codec of
  state_in bit for bit;
* free-running, QDQ off: packed lengths 1, 63, 64, 65, 200 and a dense
  batch; GDN and KDA; bf16 and fp32; d_k, d_v in {64, 128};
* teacher-forced, QDQ on: the GPU run split into one call per chunk agrees
  with the single call, and the oracle restarted from the GPU's state at
  every chunk boundary matches outputs and codes;
* the five workloads: the tiny one in full, reduced copies of the others,
  and the full-size prefill workloads in the benchmark's launch
  configuration: 16 sampled (sequence, head) units each, free-running over
  their whole sequences and teacher-forced on 8 or more chunks per unit;
  the packed workload's 32-token decode tail for every (sequence, head);
* INT8 groups of 16, 32 and 64 on the tensor-core kernels over several
  chunks from random states;
* edge cases: empty sequences, an all-empty packed batch, a malformed
  cu_seqlens reported through gdn_last_error, state_out aliasing state_in.

Every test runs three times: under the automatic schedule choice and with
the single-CTA and the CTA-pair tensor-core kernels forced.
"""

import dataclasses

import numpy as np
import pytest
import torch

import gdn_synth as gs
import oracle
from parity import (TOL, assert_flip_budget, assert_rows_close, check_codes,
                    per_unit_rel_err, rel_err)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=["auto", "single", "pair", "wy"])
def schedule(request, monkeypatch):
    """Every case under the library's own choice of tensor-core schedule and
    under each schedule forced: one CTA per (sequence, head)
    (GDN_PREFILL_CTA_PAIR=0), the delta-form CTA pair (GDN_PREFILL_CTA_PAIR=1),
    or the WY-form pair (GDN_PREFILL_CTA_PAIR=1, GDN_PREFILL_WY=1: FP8 tiles;
    other codecs keep the delta-form pair).  Cases off the tensor-core path
    (fp32, KDA gates, d = 64) run the same kernel in all four."""
    monkeypatch.delenv("GDN_PREFILL_WY", raising=False)
    if request.param == "auto":
        monkeypatch.delenv("GDN_PREFILL_CTA_PAIR", raising=False)
    elif request.param == "single":
        monkeypatch.setenv("GDN_PREFILL_CTA_PAIR", "0")
    else:
        monkeypatch.setenv("GDN_PREFILL_CTA_PAIR", "1")
        if request.param == "wy":
            monkeypatch.setenv("GDN_PREFILL_WY", "1")
    return request.param


def dev(x):
    return None if x is None else x.cuda()


def run_gpu(cuda_lib, inp, case, state_in="inp"):
    st = inp["state_in"] if state_in == "inp" else state_in
    o, s = cuda_lib.gdn_prefill(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["g"]),
                                dev(inp["beta"]), dev(st), dev(inp["cu_seqlens"]), qdq=case.qdq)
    torch.cuda.synchronize()
    cuda_lib.check_last_error(where="gdn_prefill")
    return o.float().cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("mode", ["int8_g32", "int8_g16", "int8_g64", "fp8_tile64"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64)])
def test_prefill_codec_bit_exact(cuda_lib, mode, dtype, dk, dv):
    case = gs.Case("codec", n_seq=3, H=4, d_k=dk, d_v=dv, T=1, dtype=dtype, qdq=mode,
                   state="normal", seed=51)
    inp = gs.generate(case)
    st = inp["state_in"].clone()
    st[0, 1, :, :64] = 0.0
    st[2, 3, 9, :] *= 30.0
    inp["state_in"] = st
    inp["g"] = torch.zeros_like(inp["g"])
    inp["beta"] = torch.zeros_like(inp["beta"])
    _, s = run_gpu(cuda_lib, inp, case)
    np.testing.assert_array_equal(s, oracle.qdq(st.numpy(), mode)[0])


@pytest.mark.parametrize("gate", ["scalar", "per_key"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_prefill_free_running_no_qdq_packed(cuda_lib, gate, dtype, dk, dv):
    case = gs.Case("packed", n_seq=5, H=2, d_k=dk, d_v=dv, lengths=(1, 63, 64, 65, 200),
                   dtype=dtype, gate=gate, qdq="none", state="normal", seed=61)
    inp = gs.generate(case)
    o, s = run_gpu(cuda_lib, inp, case)
    o_ref, s_ref = oracle.prefill(inp, case)
    assert rel_err(o, o_ref.reshape(o.shape)) <= TOL[dtype]
    assert_rows_close(o, o_ref, dtype, "free-running packed o")
    assert per_unit_rel_err(s, s_ref, axes=(-2, -1)) <= TOL[dtype]


@pytest.mark.parametrize("gate", ["scalar", "per_key"])
def test_prefill_free_running_no_qdq_dense(cuda_lib, gate):
    case = gs.Case("dense", n_seq=3, H=4, d_k=128, d_v=128, T=130, dtype="bf16", gate=gate,
                   qdq="none", state="zero", seed=62)
    inp = gs.generate(case)
    o, s = run_gpu(cuda_lib, inp, case)
    o_ref, s_ref = oracle.prefill(inp, case)
    assert rel_err(o, o_ref.reshape(o.shape)) <= TOL["bf16"]
    assert_rows_close(o, o_ref, "bf16", "free-running dense o")
    assert per_unit_rel_err(s, s_ref, axes=(-2, -1)) <= TOL["bf16"]


def teacher_forced_chunks(cuda_lib, case, label):
    """Run each sequence chunk by chunk on the GPU (state handed from call to
    call), check that this equals the single call bit for bit, and compare
    each chunk with the oracle restarted from the GPU's chunk-start state."""
    inp = gs.generate(case)
    o_full, s_full = run_gpu(cuda_lib, inp, case)
    per_key = case.gate == "per_key"
    lengths = inp["lengths"]
    starts = np.concatenate([[0], np.cumsum(lengths)])
    q, k, v, g, beta = (inp[x].reshape((-1,) + inp[x].shape[2:]) for x in ("q", "k", "v", "g", "beta"))
    H, dk, dv = case.H, case.d_k, case.d_v
    stats, worst_o = [], 0.0
    for si, L in enumerate(lengths):
        st = (inp["state_in"][si:si + 1].clone() if inp["state_in"] is not None
              else torch.zeros((1, H, dk, dv)))
        for c0 in range(0, L, 64):
            c1 = min(c0 + 64, L)
            sl = slice(int(starts[si] + c0), int(starts[si] + c1))
            sub = {"q": q[sl][None], "k": k[sl][None], "v": v[sl][None], "g": g[sl][None],
                   "beta": beta[sl][None], "state_in": st, "cu_seqlens": None}
            sub_case = gs.Case("chunk", n_seq=1, H=H, d_k=dk, d_v=dv, T=c1 - c0,
                               dtype=case.dtype, gate=case.gate, qdq=case.qdq)
            o_c, s_c = run_gpu(cuda_lib, sub, sub_case)
            cu = np.array([0, c1 - c0], dtype=np.int32)
            o_r, s_r, codes, scales = oracle.recurrence(
                sub["q"], sub["k"], sub["v"], sub["g"], sub["beta"], st, cu,
                per_key_gate=per_key, qdq=case.qdq, want_codes=True)
            worst_o = max(worst_o, rel_err(o_c[0], o_r))
            assert_rows_close(o_c[0], o_r, case.dtype, f"{label} seq {si} chunk {c0 // 64}")
            if case.qdq != "none":
                stats.append(check_codes(s_c, s_r, codes, scales, case.qdq,
                                         label=f"{label} seq {si} chunk {c0 // 64}"))
            # one call per chunk agrees with the single call: bit for bit on the
            # CUDA-core kernel; the tensor-core kernel feeds an FP8 state as
            # exact codes inside one call but as hi/lo splits when a call
            # starts from it, so there the two may differ in the last bits
            ref_o = o_full.reshape((-1, H, dv))[sl]
            if case.dtype == "f32" or case.gate == "per_key":
                np.testing.assert_array_equal(o_c[0], ref_o)
            else:
                assert rel_err(o_c[0], ref_o) <= TOL[case.dtype]
            st = torch.from_numpy(s_c)
        if case.dtype == "f32" or case.gate == "per_key":
            np.testing.assert_array_equal(st.numpy()[0], s_full[si])
        else:
            assert rel_err(st.numpy()[0], s_full[si]) <= TOL[case.dtype]
    assert worst_o <= TOL[case.dtype], (label, worst_o)
    return assert_flip_budget(stats, label) if stats else None


def test_prefill_tiny_config(cuda_lib):
    case = gs.CONFIGS["tiny"]
    teacher_forced_chunks(cuda_lib, case, "tiny prefill")
    inp = gs.generate(case)
    o, s = run_gpu(cuda_lib, inp, case)
    o_ref, s_ref = oracle.prefill(inp, case)
    assert rel_err(o, o_ref.reshape(o.shape)) <= TOL["f32"]


@pytest.mark.parametrize("base,over", [
    ("gdn_prefill", dict(n_seq=2, H=3, T=300)),
    ("kda_prefill", dict(n_seq=1, H=3, T=300)),
    ("varlen", dict(n_seq=6, H=2, varlen_max=300)),
    ("gdn_prefill", dict(n_seq=2, H=2, T=200, qdq="int8_g32", dtype="f32")),
    ("kda_prefill", dict(n_seq=2, H=2, T=150, qdq="fp8_tile64", state="normal")),
])
def test_prefill_teacher_forced(cuda_lib, base, over):
    case = gs.small_case(base, seed=71, **over)
    teacher_forced_chunks(cuda_lib, case, f"{base} {over}")


_TENSORS = ("q", "k", "v", "g", "beta")


def _flat(inp):
    return {x: inp[x].reshape((-1,) + inp[x].shape[2:]) for x in _TENSORS}


def _unit_batch(inp, units, ranges):
    """Oracle inputs for (sequence, head) units over token ranges [a, b) of
    their sequences: every unit becomes one packed sequence of one head."""
    starts = np.concatenate([[0], np.cumsum(inp["lengths"])])
    flat = _flat(inp)
    parts = {x: [] for x in _TENSORS}
    cu = [0]
    for (si, h), (a, b) in zip(units, ranges):
        sl = slice(int(starts[si] + a), int(starts[si] + b))
        for x in _TENSORS:
            parts[x].append(flat[x][sl][:, h:h + 1])
        cu.append(cu[-1] + (b - a))
    return {x: torch.cat(parts[x]) for x in _TENSORS}, np.array(cu, dtype=np.int32)


def _unit_states(S, units, dk, dv):
    """[n_units, 1, d_k, d_v] states of the units from [n_seq, H, ...] (None: zero)."""
    if S is None:
        return torch.zeros((len(units), 1, dk, dv))
    S = torch.as_tensor(S)
    return torch.stack([S[si, h:h + 1] for (si, h) in units])


def _truncated(inp, case, lens):
    """The workload cut to the first lens[s] tokens of every sequence: a
    dense batch when the case is dense and the cut uniform (the layout the
    benchmark runs), otherwise a packed batch of the same sequences."""
    if inp["cu_seqlens"] is None and len(set(lens)) == 1:
        sub = {x: inp[x][:, :lens[0]].contiguous() for x in _TENSORS}
        sub.update(state_in=inp["state_in"], cu_seqlens=None, lengths=list(lens))
        return sub, dataclasses.replace(case, T=int(lens[0]))
    starts = np.concatenate([[0], np.cumsum(inp["lengths"])])
    flat = _flat(inp)
    sub = {x: torch.cat([flat[x][int(starts[si]):int(starts[si] + n)]
                         for si, n in enumerate(lens)])[None] for x in _TENSORS}
    cu = torch.zeros(len(lens) + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(torch.tensor(lens, dtype=torch.int64), 0).to(torch.int32)
    sub.update(state_in=inp["state_in"], cu_seqlens=cu, lengths=list(lens))
    return sub, dataclasses.replace(case, lengths=tuple(int(n) for n in lens), varlen_max=0, T=0)


def _check_full_workload(cuda_lib, case, units, n_tf_chunks=8):
    """The whole workload in one call, as the benchmark launches it, then:

    * free-running: the oracle over every sampled (sequence, head) unit's
      whole sequence, from the same initial state; o and the final state
      norm-wise per unit;
    * teacher-forced: for each sampled unit, ``n_tf_chunks`` chunks spread
      over its sequence (first, second and last included).  The GPU's state
      at the start of chunk c is the final state of the same workload cut
      to its first 64 c tokens per sequence (the same kernel computes the
      same chunks bit for bit), and the state after it that of the cut at
      64 (c + 1); the oracle restarted from the former over chunk c must
      give the latter's codes (one-step flips within the budget) and the
      single call's outputs of that chunk (norm-wise and per element)."""
    inp = gs.generate(case)
    o, s = run_gpu(cuda_lib, inp, case)
    lengths = [int(x) for x in inp["lengths"]]
    starts = np.concatenate([[0], np.cumsum(lengths)])
    H, dk, dv = case.H, case.d_k, case.d_v
    per_key = case.gate == "per_key"
    o_flat = o.reshape((-1, H, dv))
    tol = TOL[case.dtype]

    # free-running, all sampled units in one oracle call
    batch, cu = _unit_batch(inp, units, [(0, lengths[si]) for si, _ in units])
    o_r, s_r = oracle.recurrence(*(batch[x] for x in _TENSORS),
                                 _unit_states(inp["state_in"], units, dk, dv), cu,
                                 per_key_gate=per_key, qdq=case.qdq)
    for i, (si, h) in enumerate(units):
        o_u = o_flat[int(starts[si]):int(starts[si + 1]), h]
        assert rel_err(o_u, o_r[cu[i]:cu[i + 1], 0]) <= tol, ("o", si, h)
        assert rel_err(s[si, h], s_r[i, 0]) <= tol, ("state", si, h)

    # teacher-forced, n_tf_chunks chunk positions per sequence
    n_ch = [(L + 63) // 64 for L in lengths]
    pos = [sorted({0, min(1, n - 1)} | {round(j * (n - 1) / (n_tf_chunks - 1))
                                        for j in range(n_tf_chunks)}) if n else []
           for n in n_ch]
    n_pos = max(len(p) for p in pos)
    stats, checked = [], 0
    for j in range(n_pos):
        c_of = [p[j] if j < len(p) else (p[-1] if p else 0) for p in pos]
        before = [min(64 * c, L) for c, L in zip(c_of, lengths)]
        after = [min(64 * (c + 1), L) for c, L in zip(c_of, lengths)]
        if max(before) == 0:
            S0 = (inp["state_in"].numpy() if inp["state_in"] is not None
                  else np.zeros((case.n_seq, H, dk, dv), np.float32))
        else:
            sub, sc = _truncated(inp, case, before)
            _, S0 = run_gpu(cuda_lib, sub, sc)
        sub, sc = _truncated(inp, case, after)
        _, S1 = run_gpu(cuda_lib, sub, sc)
        live = [(si, h) for (si, h) in units if after[si] > before[si]]
        batch, cu = _unit_batch(inp, live, [(before[si], after[si]) for si, _ in live])
        o_t, s_t, codes, scales = oracle.recurrence(
            *(batch[x] for x in _TENSORS), _unit_states(S0, live, dk, dv), cu,
            per_key_gate=per_key, qdq=case.qdq, want_codes=True)
        for i, (si, h) in enumerate(live):
            sl = slice(int(starts[si] + before[si]), int(starts[si] + after[si]))
            ref = o_t[cu[i]:cu[i + 1], 0]
            assert rel_err(o_flat[sl, h], ref) <= tol, ("tf o", si, h, c_of[si])
            assert_rows_close(o_flat[sl, h], ref, case.dtype, f"tf o {si} {h} {c_of[si]}")
        if case.qdq != "none":
            got = np.stack([S1[si, h:h + 1] for (si, h) in live])
            stats.append(check_codes(got, s_t, codes, scales, case.qdq,
                                     label=f"{case.name} position {j}"))
        checked += len(live)
    assert checked >= n_tf_chunks * len(units)
    return assert_flip_budget(stats, case.name) if stats else None


def test_full_gdn_prefill_workload(cuda_lib):
    """B=4, H=16, T=4096, FP8 tiles: 16 of the 64 units, 9 chunks each."""
    case = gs.CONFIGS["gdn_prefill"]
    units = [(si, h) for si in range(4) for h in (0, 5, 10, 15)]
    _check_full_workload(cuda_lib, case, units)


def test_full_kda_prefill_workload(cuda_lib):
    """B=2, H=32, T=8192, per-key gates, INT8 g32: 16 of the 64 units."""
    case = gs.CONFIGS["kda_prefill"]
    units = [(si, h) for si in range(2) for h in range(0, 32, 4)]
    _check_full_workload(cuda_lib, case, units)


def _varlen_units(lengths, n=16):
    """n units of distinct sequences with at least 9 chunks, spread over
    the length range and the heads."""
    order = [int(i) for i in np.argsort(lengths) if lengths[i] > 8 * 64]
    pick = [order[round(j * (len(order) - 1) / (n - 1))] for j in range(n)]
    assert len(set(pick)) == n
    return [(si, (3 * j) % 16) for j, si in enumerate(pick)]


def test_full_varlen_workload(cuda_lib):
    """64 packed sequences of U{1..4096} tokens, H=16, random states, FP8
    tiles (1,024 units): 16 units, 8 or more chunks each."""
    case = gs.small_case("varlen", decode_steps=0)
    assert case.n_seq == 64
    lengths = gs.generate(case)["lengths"]
    _check_full_workload(cuda_lib, case, _varlen_units(lengths))


def test_full_varlen_workload_decode_tail(cuda_lib, schedule):
    """The packed workload end to end: the packed prefill of all 64
    sequences, then 32 decode tokens for every sequence (FP8 tiles, the
    prefill's codec) starting from the GPU's own prefill states; every
    decode step of every (sequence, head) is compared with the oracle
    restarted from the GPU's state before it (outputs of all 1,024 units;
    codes within the one-step / 1e-4 budget for a window of 256 units that
    rotates over all of them every 4 steps).  Run under the automatic
    schedule and the WY-form pair (the decode kernel is the same in all)."""
    if schedule not in ("auto", "wy"):
        pytest.skip("the decode tail is the same kernel under every prefill schedule")
    case = gs.CONFIGS["varlen"]
    assert case.decode_steps == 32
    inp = gs.generate(case)
    _, st = run_gpu(cuda_lib, inp, case)
    S = torch.from_numpy(st).cuda()
    stats, worst_o = [], 0.0
    for t in range(case.decode_steps):
        prev = S.cpu().numpy().copy()
        o = cuda_lib.gdn_decode(dev(inp["dec_q"][t]), dev(inp["dec_k"][t]), dev(inp["dec_v"][t]),
                                dev(inp["dec_g"][t]), dev(inp["dec_beta"][t]), S, qdq=case.qdq)
        torch.cuda.synchronize()
        sl = slice(t, t + 1)
        o_ref, s_ref, codes, scales = oracle.decode(
            inp["dec_q"][sl], inp["dec_k"][sl], inp["dec_v"][sl], inp["dec_g"][sl],
            inp["dec_beta"][sl], prev, per_key_gate=False, qdq=case.qdq, want_codes=True)
        o_g = o.float().cpu().numpy()
        worst_o = max(worst_o, rel_err(o_g, o_ref[0]))
        assert_rows_close(o_g, o_ref[0], "bf16", f"decode tail step {t}")
        # units (sequence, head) flattened; 256 of the 1,024 per step
        win = (256 * t + np.arange(256)) % (case.n_seq * case.H)
        si, hi = win // case.H, win % case.H
        S_h = S.cpu().numpy()
        stats.append(check_codes(S_h[si, hi][:, None], s_ref[si, hi][:, None],
                                 codes[si, hi][:, None], scales[si, hi][:, None], case.qdq,
                                 label=f"decode tail step {t}"))
    assert worst_o <= TOL["bf16"], worst_o
    assert_flip_budget(stats, "varlen decode tail")


def test_long_single_sequence(cuda_lib):
    """One sequence of 16384 tokens (256 chunks), one head."""
    case = gs.Case("long", n_seq=1, H=1, d_k=128, d_v=128, T=16384, dtype="bf16",
                   gate="scalar", qdq="fp8_tile64", state="normal", seed=81)
    _check_full_workload(cuda_lib, case, units=[(0, 0)], n_tf_chunks=12)


@pytest.mark.parametrize("mode", ["int8_g32", "int8_g16", "int8_g64"])
def test_prefill_int8_tensor_cores_multichunk(cuda_lib, mode):
    """bf16 GDN at d = 128 takes the tensor-core kernels for every codec: INT8
    groups of 32, 16 and 64 over 6 chunks (a partial last one) from random
    initial states (whose hi/lo split path an INT8 state keeps), free-running
    against the oracle and teacher-forced chunk by chunk."""
    case = gs.Case("int8tc", n_seq=2, H=3, d_k=128, d_v=128, T=5 * 64 + 21, dtype="bf16",
                   gate="scalar", qdq=mode, state="normal", seed=95)
    inp = gs.generate(case)
    o, s = run_gpu(cuda_lib, inp, case)
    o_ref, s_ref = oracle.prefill(inp, case)
    assert rel_err(o, o_ref.reshape(o.shape)) <= TOL["bf16"]
    assert per_unit_rel_err(s, s_ref, axes=(-2, -1)) <= TOL["bf16"]
    teacher_forced_chunks(cuda_lib, case, f"int8 tensor cores {mode}")


def test_empty_sequences_and_alias(cuda_lib):
    """Zero-length sequences keep their state unquantized; state_out may
    alias state_in."""
    case = gs.Case("empty", n_seq=4, H=2, d_k=64, d_v=64, lengths=(0, 70, 0, 5), dtype="bf16",
                   qdq="int8_g32", state="normal", seed=91)
    inp = gs.generate(case)
    o_ref, s_ref = oracle.prefill(inp, case)
    S = inp["state_in"].clone().cuda()
    o = torch.empty(inp["v"].shape, dtype=torch.bfloat16, device="cuda")
    cuda_lib.gdn_prefill_into(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["g"]),
                              dev(inp["beta"]), S, dev(inp["cu_seqlens"]), o, S, qdq=case.qdq)
    torch.cuda.synchronize()
    cuda_lib.check_last_error(where="alias")
    s = S.cpu().numpy()
    np.testing.assert_array_equal(s[0], inp["state_in"][0].numpy())
    np.testing.assert_array_equal(s[2], inp["state_in"][2].numpy())
    assert rel_err(o.float().cpu().numpy(), o_ref.reshape(o.shape)) <= TOL["bf16"]


def test_all_empty_packed_batch(cuda_lib):
    st = torch.randn((3, 2, 64, 64), device="cuda") * 0.05
    out = torch.full_like(st, 7.0)
    cu = torch.zeros(4, dtype=torch.int32, device="cuda")
    e = torch.empty((1, 0, 2, 64), dtype=torch.bfloat16, device="cuda")
    g = torch.empty((1, 0, 2), device="cuda")
    cuda_lib.gdn_prefill_into(e, e, e, g, g, st, cu, e, out, qdq="fp8_tile64")
    torch.cuda.synchronize()
    cuda_lib.check_last_error(where="all empty")
    assert torch.equal(out, st)


def test_malformed_cu_seqlens_reported(cuda_lib):
    case = gs.Case("bad", n_seq=3, H=2, d_k=64, d_v=64, lengths=(40, 40, 40), dtype="bf16",
                   qdq="none", seed=92)
    inp = gs.generate(case)
    bad = torch.tensor([0, 50, 30, 120], dtype=torch.int32)  # not non-decreasing
    with pytest.raises(cuda_lib.GdnError) as ei:
        cuda_lib.gdn_prefill(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["g"]),
                             dev(inp["beta"]), None, bad.cuda(), qdq="none")
        torch.cuda.synchronize()
        cuda_lib.check_last_error(where="bad cu_seqlens")
    assert ei.value.status == 1
    # the error word is cleared by the read
    assert cuda_lib.gdn_last_error() == 0


@pytest.mark.parametrize("n_seq", [40, 300])
@pytest.mark.parametrize("dtype,dk", [("bf16", 128), ("f32", 64)])
def test_packed_order_many_sequences(cuda_lib, n_seq, dtype, dk):
    """Packed batches are processed longest first when they have at most 256
    sequences (each CTA ranks the lengths) and in index order beyond; either
    way every (sequence, head) lands in its own place.  Lengths repeat, so
    the rank's tie-break by index is exercised."""
    rng = np.random.default_rng(1000 + n_seq)
    lengths = tuple(int(x) for x in rng.choice([1, 7, 64, 65, 130], size=n_seq))
    case = gs.Case("many", n_seq=n_seq, H=2, d_k=dk, d_v=dk, lengths=lengths, dtype=dtype,
                   qdq="none", state="normal", seed=93)
    inp = gs.generate(case)
    o, s = run_gpu(cuda_lib, inp, case)
    o_ref, s_ref = oracle.prefill(inp, case)
    assert rel_err(o, o_ref.reshape(o.shape)) <= TOL[dtype]
    assert per_unit_rel_err(s, s_ref, axes=(-2, -1)) <= TOL[dtype]


def test_schedule_is_the_one_forced(cuda_lib, schedule):
    """The forced schedules are the ones launched; the automatic choice takes
    a pair while every unit gets one in a wave (the WY-form pair for FP8
    tiles), one CTA per unit beyond."""
    pick = cuda_lib.gdn_prefill_schedule
    if schedule == "pair":
        assert pick(4, 16, 128, 128) == "tc_cta_pair"
        assert pick(4, 16, 128, 128, qdq="int8_g32") == "tc_cta_pair"
    elif schedule == "wy":
        assert pick(4, 16, 128, 128) == "tc_wy_pair"
        assert pick(64, 16, 128, 128) == "tc_wy_pair"
        assert pick(4, 16, 128, 128, qdq="int8_g32") == "tc_cta_pair"
    elif schedule == "single":
        assert pick(4, 16, 128, 128) == "tc_one_cta"
    else:
        assert pick(4, 16, 128, 128) == "tc_cta_pair"
        assert pick(4, 16, 128, 128, qdq="none") == "tc_cta_pair"
        assert pick(64, 16, 128, 128) == "tc_one_cta"
    assert pick(4, 16, 128, 128, dtype=torch.float32) == "cuda_cores"
    assert pick(4, 16, 128, 128, gate="per_key", qdq="int8_g32") == "cuda_cores"
