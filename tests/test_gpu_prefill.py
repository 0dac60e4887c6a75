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
  configuration compared on sampled (sequence, head) units;
* edge cases: empty sequences, an all-empty packed batch, a malformed
  cu_seqlens reported through gdn_last_error, state_out aliasing state_in.

Every test runs three times: under the automatic schedule choice and with
the single-CTA and the CTA-pair tensor-core kernels forced.
"""

import numpy as np
import pytest
import torch

import gdn_synth as gs
import oracle
from parity import TOL, assert_flip_budget, check_codes, per_unit_rel_err, rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, params=["auto", "single", "pair"])
def schedule(request, monkeypatch):
    """Every case under the library's own choice of tensor-core schedule and
    under each schedule forced (GDN_PREFILL_CTA_PAIR): one CTA per
    (sequence, head), or a CTA pair.  Cases off the tensor-core path (fp32,
    KDA gates, d = 64) run the same kernel in all three."""
    if request.param == "auto":
        monkeypatch.delenv("GDN_PREFILL_CTA_PAIR", raising=False)
    else:
        monkeypatch.setenv("GDN_PREFILL_CTA_PAIR", "1" if request.param == "pair" else "0")
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
    assert per_unit_rel_err(s, s_ref, axes=(-2, -1)) <= TOL[dtype]


@pytest.mark.parametrize("gate", ["scalar", "per_key"])
def test_prefill_free_running_no_qdq_dense(cuda_lib, gate):
    case = gs.Case("dense", n_seq=3, H=4, d_k=128, d_v=128, T=130, dtype="bf16", gate=gate,
                   qdq="none", state="zero", seed=62)
    inp = gs.generate(case)
    o, s = run_gpu(cuda_lib, inp, case)
    o_ref, s_ref = oracle.prefill(inp, case)
    assert rel_err(o, o_ref.reshape(o.shape)) <= TOL["bf16"]
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


def _sampled_units(cuda_lib, case, units, tf_units):
    """Full workload on the GPU; free-running comparison on `units`
    (seq, head) pairs and a teacher-forced last chunk on `tf_units`."""
    inp = gs.generate(case)
    o, s = run_gpu(cuda_lib, inp, case)
    lengths = inp["lengths"]
    starts = np.concatenate([[0], np.cumsum(lengths)])
    H, dv = case.H, case.d_v
    per_key = case.gate == "per_key"
    flat = {x: inp[x].reshape((-1,) + inp[x].shape[2:]) for x in ("q", "k", "v", "g", "beta")}
    o_flat = o.reshape((-1, H, dv))
    stats = []
    for (si, h) in units:
        sl = slice(int(starts[si]), int(starts[si + 1]))
        st = None if inp["state_in"] is None else inp["state_in"][si:si + 1, h:h + 1]
        cu = np.array([0, lengths[si]], dtype=np.int32)
        args = [flat[x][sl][:, h:h + 1] for x in ("q", "k", "v", "g", "beta")]
        o_r, s_r = oracle.recurrence(*args, st, cu, per_key_gate=per_key, qdq=case.qdq)
        assert rel_err(o_flat[sl, h], o_r[:, 0]) <= TOL[case.dtype], (si, h)
        assert rel_err(s[si, h], s_r[0, 0]) <= TOL[case.dtype], (si, h)
    for si in tf_units:
        L = lengths[si]
        if L <= 64:
            continue
        cut = ((L - 1) // 64) * 64
        sl = slice(int(starts[si]), int(starts[si] + cut))
        sub = {x: flat[x][sl][None] for x in ("q", "k", "v", "g", "beta")}
        sub["state_in"] = None if inp["state_in"] is None else inp["state_in"][si:si + 1]
        sub["cu_seqlens"] = None
        _, s_mid = run_gpu(cuda_lib, sub, gs.Case("p", n_seq=1, H=H, d_k=case.d_k, d_v=dv, T=cut,
                                                  dtype=case.dtype, gate=case.gate, qdq=case.qdq))
        sl2 = slice(int(starts[si] + cut), int(starts[si + 1]))
        args = [flat[x][sl2] for x in ("q", "k", "v", "g", "beta")]
        cu = np.array([0, L - cut], dtype=np.int32)
        o_r, s_r, codes, scales = oracle.recurrence(*args, s_mid, cu, per_key_gate=per_key,
                                                    qdq=case.qdq, want_codes=True)
        assert rel_err(o_flat[sl2], o_r) <= TOL[case.dtype]
        stats.append(check_codes(s[si:si + 1], s_r, codes, scales, case.qdq,
                                 label=f"{case.name} seq {si} last chunk"))
    return assert_flip_budget(stats, case.name)


def test_full_gdn_prefill_workload(cuda_lib):
    case = gs.CONFIGS["gdn_prefill"]
    _sampled_units(cuda_lib, case, units=[(0, 0), (1, 7), (2, 15), (3, 3)], tf_units=[0, 3])


def test_full_kda_prefill_workload(cuda_lib):
    case = gs.CONFIGS["kda_prefill"]
    _sampled_units(cuda_lib, case, units=[(0, 0), (1, 31), (0, 17)], tf_units=[1])


def test_full_varlen_workload(cuda_lib):
    case = gs.CONFIGS["varlen"]
    inp_len = gs.generate(gs.small_case("varlen", decode_steps=0))["lengths"]
    order = np.argsort(inp_len)
    units = [(int(order[0]), 0), (int(order[-1]), 15), (int(order[31]), 5), (int(order[-2]), 9)]
    _sampled_units(cuda_lib, gs.small_case("varlen", decode_steps=0), units=units,
                   tf_units=[int(order[-1]), int(order[40])])
    assert case.n_seq == 64


def test_long_single_sequence(cuda_lib):
    """One sequence of 16384 tokens (256 chunks), one head."""
    case = gs.Case("long", n_seq=1, H=1, d_k=128, d_v=128, T=16384, dtype="bf16",
                   gate="scalar", qdq="fp8_tile64", state="normal", seed=81)
    _sampled_units(cuda_lib, case, units=[(0, 0)], tf_units=[0])


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
    the pair while every unit gets one in a wave, one CTA per unit beyond."""
    pick = cuda_lib.gdn_prefill_schedule
    if schedule == "pair":
        assert pick(4, 16, 128, 128) == "tc_cta_pair"
    elif schedule == "single":
        assert pick(4, 16, 128, 128) == "tc_one_cta"
    else:
        assert pick(4, 16, 128, 128) == "tc_cta_pair"
        assert pick(64, 16, 128, 128) == "tc_one_cta"
    assert pick(4, 16, 128, 128, dtype=torch.float32) == "cuda_cores"
    assert pick(4, 16, 128, 128, gate="per_key") == "cuda_cores"

