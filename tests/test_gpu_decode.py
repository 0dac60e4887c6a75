"""GPU parity of gdn_decode (through the C ABI) against the CPU oracle.

* codec alone: with g = 0 and beta = 0 the pre-QDQ state equals the input
  state exactly, so the GPU's output state must equal the oracle's codec of
  the same fp32 state bit for bit (every codec, both dtypes, all d_k/d_v);
* teacher-forced steps: the oracle advances the GPU's own previous state by
  one token; outputs within the float tolerance, QDQ codes within the
  one-step / 1e-4 budget (tiny fp32 config, serving-decode shapes, KDA);
* free-running without QDQ: 24 steps within the float tolerance;
* the full serving-decode shapes (256 sequences x 32 heads, d = 128, INT8
  g32): two teacher-forced steps, compared on a quarter of the sequences;
  and the benchmark's whole run, 512 tokens of all 256 sequences, on 8
  sampled sequences (every head): teacher-forced at every one of the 512
  steps, and free-running against the oracle's own chain (a looser bound:
  see FREE_RUNNING_DECODE_CHAIN_TOL).
"""

import numpy as np
import pytest
import torch

import gdn_synth as gs
import oracle
from parity import TOL, assert_flip_budget, assert_rows_close, check_codes, rel_err

pytestmark = pytest.mark.gpu


def dev(x):
    return None if x is None else x.cuda()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("mode", ["int8_g32", "int8_g16", "int8_g64", "fp8_tile64"])
def test_decode_codec_bit_exact(cuda_lib, mode, dk, dv, dtype):
    case = gs.Case("codec", n_seq=3, H=4, d_k=dk, d_v=dv, dtype=dtype, qdq=mode,
                   state="normal", decode_steps=1, seed=11)
    inp = gs.generate(case)
    st = inp["state_in"].clone()
    st[1, 2, :, :64] = 0.0            # a zero FP8 tile / zero INT8 groups
    st[2, 0, 5, :] *= 40.0            # one large key row
    g = torch.zeros_like(inp["dec_g"][0])
    beta = torch.zeros_like(inp["dec_beta"][0])
    S = st.cuda()
    o = cuda_lib.gdn_decode(dev(inp["dec_q"][0]), dev(inp["dec_k"][0]), dev(inp["dec_v"][0]),
                            g.cuda(), beta.cuda(), S, qdq=mode)
    torch.cuda.synchronize()
    expect = oracle.qdq(st.numpy(), mode)[0]
    np.testing.assert_array_equal(S.cpu().numpy(), expect)
    # the output is still scale * H^T q of the (unchanged) state
    ref = np.einsum("nhkv,nhk->nhv", st.double().numpy(),
                    inp["dec_q"][0].double().numpy()) / np.sqrt(dk)
    assert rel_err(o.float().cpu().numpy(), ref) <= TOL[dtype]


def _teacher_forced(cuda_lib, case, S0: torch.Tensor, steps: int, label: str):
    """Advance the GPU state `steps` tokens; after each, restart the oracle
    from the GPU's previous state and compare."""
    inp = gs.generate(case)
    per_key = case.gate == "per_key"
    S = S0.clone().cuda()
    stats, worst_o = [], 0.0
    for t in range(steps):
        prev = S.cpu().numpy().copy()
        o = cuda_lib.gdn_decode(dev(inp["dec_q"][t]), dev(inp["dec_k"][t]), dev(inp["dec_v"][t]),
                                dev(inp["dec_g"][t]), dev(inp["dec_beta"][t]), S, qdq=case.qdq)
        torch.cuda.synchronize()
        sl = slice(t, t + 1)
        o_ref, s_ref, codes, scales = oracle.decode(
            inp["dec_q"][sl], inp["dec_k"][sl], inp["dec_v"][sl], inp["dec_g"][sl],
            inp["dec_beta"][sl], prev, per_key_gate=per_key, qdq=case.qdq, want_codes=True)
        worst_o = max(worst_o, rel_err(o.float().cpu().numpy(), o_ref[0]))
        assert_rows_close(o.float().cpu().numpy(), o_ref[0], case.dtype, f"{label} step {t}")
        stats.append(check_codes(S.cpu().numpy(), s_ref, codes, scales, case.qdq,
                                 label=f"{label} step {t}"))
    assert worst_o <= TOL[case.dtype], (label, worst_o)
    return assert_flip_budget(stats, label)


def test_decode_tiny_config(cuda_lib):
    """Tiny workload: 64-token prefill (fp32, d = 64, INT8 g32) then 64
    decode tokens, teacher-forced from the GPU's own prefill state."""
    case = gs.CONFIGS["tiny"]
    inp = gs.generate(case)
    o, st = cuda_lib.gdn_prefill(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["g"]),
                                 dev(inp["beta"]), None, None, qdq=case.qdq)
    torch.cuda.synchronize()
    _teacher_forced(cuda_lib, case, st.cpu(), case.decode_steps, "tiny decode")


@pytest.mark.parametrize("gate,mode,dtype", [
    ("scalar", "int8_g32", "bf16"), ("scalar", "fp8_tile64", "bf16"),
    ("per_key", "int8_g32", "bf16"), ("per_key", "fp8_tile64", "f32"),
    ("scalar", "int8_g16", "f32"), ("scalar", "int8_g64", "bf16")])
def test_decode_teacher_forced(cuda_lib, gate, mode, dtype):
    case = gs.small_case("serving_decode", n_seq=8, H=4, decode_steps=12, gate=gate, qdq=mode,
                         dtype=dtype, seed=21)
    st = gs.generate(case)["state_in"]
    _teacher_forced(cuda_lib, case, st, case.decode_steps, f"decode {gate} {mode} {dtype}")


@pytest.mark.parametrize("gate", ["scalar", "per_key"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_free_running_no_qdq(cuda_lib, gate, dtype):
    case = gs.small_case("serving_decode", n_seq=4, H=3, decode_steps=24, gate=gate, qdq="none",
                         dtype=dtype, seed=31)
    inp = gs.generate(case)
    S = inp["state_in"].clone().cuda()
    outs = []
    for t in range(case.decode_steps):
        outs.append(cuda_lib.gdn_decode(dev(inp["dec_q"][t]), dev(inp["dec_k"][t]),
                                        dev(inp["dec_v"][t]), dev(inp["dec_g"][t]),
                                        dev(inp["dec_beta"][t]), S, qdq="none"))
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.decode(inp["dec_q"], inp["dec_k"], inp["dec_v"], inp["dec_g"],
                                 inp["dec_beta"], inp["state_in"], per_key_gate=gate == "per_key",
                                 qdq="none")
    o = torch.stack(outs).float().cpu().numpy()
    assert rel_err(o, o_ref) <= TOL[dtype]
    assert rel_err(S.cpu().numpy(), s_ref) <= TOL[dtype]


def test_decode_full_serving_shape(cuda_lib):
    """256 sequences x 32 heads, d = 128, INT8 g32 (the serving-decode
    workload's shapes and distributions, two tokens), compared on sequences
    0..63."""
    case = gs.small_case("serving_decode", decode_steps=2)
    inp = gs.generate(case)
    S = inp["state_in"].clone().cuda()
    stats = []
    for t in range(2):
        prev = S[:64].cpu().numpy().copy()
        o = cuda_lib.gdn_decode(dev(inp["dec_q"][t]), dev(inp["dec_k"][t]), dev(inp["dec_v"][t]),
                                dev(inp["dec_g"][t]), dev(inp["dec_beta"][t]), S, qdq=case.qdq)
        torch.cuda.synchronize()
        sl = (slice(t, t + 1), slice(0, 64))
        o_ref, s_ref, codes, scales = oracle.decode(
            inp["dec_q"][sl], inp["dec_k"][sl], inp["dec_v"][sl], inp["dec_g"][sl],
            inp["dec_beta"][sl], prev, per_key_gate=False, qdq=case.qdq, want_codes=True)
        assert rel_err(o[:64].float().cpu().numpy(), o_ref[0]) <= TOL["bf16"]
        assert_rows_close(o[:64].float().cpu().numpy(), o_ref[0], "bf16", f"full decode {t}")
        stats.append(check_codes(S[:64].cpu().numpy(), s_ref, codes, scales, case.qdq,
                                 label=f"full decode step {t}"))
    assert_flip_budget(stats, "full serving decode")


# Free-running over the 512-token chain, the QDQ after every token turns
# last-bit differences into one-step code flips that persist: an fp32
# evaluation of the same recurrence with the oracle's own codec departs
# from the fp64 oracle by up to 1.2e-2 per token step (measured on two of
# these sequences), so no fp32 implementation meets 2e-3 there.  The run
# is therefore held to the teacher-forced bar at every step, and its
# free-running distance only to 3e-2, which catches a wrong recurrence.
FREE_RUNNING_DECODE_CHAIN_TOL = 3e-2


def test_decode_full_serving_run(cuda_lib):
    """The serving-decode workload as the benchmark runs it: 512 consecutive
    single-token calls over all 256 sequences x 32 heads (INT8 g32 after
    every token).  On 8 sequences spread over the batch: every one of the
    512 steps teacher-forced (the oracle advances the GPU's own previous
    state; every head's outputs, and the codes of a rotating window of 8
    heads, within the bar), and the whole free-running chain against the
    oracle's own 512-token chain."""
    case = gs.CONFIGS["serving_decode"]
    assert case.decode_steps == 512
    inp = gs.generate(case)
    S = inp["state_in"].clone().cuda()
    dq, dk, dv = (inp[x].cuda() for x in ("dec_q", "dec_k", "dec_v"))
    dg, db = inp["dec_g"].cuda(), inp["dec_beta"].cuda()
    o = torch.empty(dv.shape, dtype=dq.dtype, device="cuda")
    seqs = [0, 37, 73, 110, 146, 183, 219, 255]
    stats, worst_tf = [], 0.0
    for t in range(case.decode_steps):
        prev = S[seqs].cpu().numpy()
        cuda_lib.gdn_decode_into(dq[t], dk[t], dv[t], dg[t], db[t], S, o[t], qdq=case.qdq)
        sl = (slice(t, t + 1), seqs)
        o_ref, s_ref, codes, scales = oracle.decode(
            inp["dec_q"][sl], inp["dec_k"][sl], inp["dec_v"][sl], inp["dec_g"][sl],
            inp["dec_beta"][sl], prev, per_key_gate=False, qdq=case.qdq, want_codes=True)
        o_g = o[t, seqs].float().cpu().numpy()
        worst_tf = max(worst_tf, rel_err(o_g, o_ref[0]))
        assert_rows_close(o_g, o_ref[0], "bf16", f"serving run step {t}")
        # codes of 8 of the 32 heads per step, a window that rotates over
        # the heads (all heads every 4 steps), to keep the check fast
        hs = [(8 * t + i) % case.H for i in range(8)]
        stats.append(check_codes(S[seqs][:, hs].cpu().numpy(), s_ref[:, hs], codes[:, hs],
                                 scales[:, hs], case.qdq, label=f"serving run step {t}"))
    cuda_lib.check_last_error(where="serving decode run")
    assert worst_tf <= TOL["bf16"], worst_tf
    assert_flip_budget(stats, "serving decode, 512 steps")

    sl = (slice(None), seqs)
    o_ref, s_ref = oracle.decode(inp["dec_q"][sl], inp["dec_k"][sl], inp["dec_v"][sl],
                                 inp["dec_g"][sl], inp["dec_beta"][sl], inp["state_in"][seqs],
                                 per_key_gate=False, qdq=case.qdq)
    o_g = o[:, seqs].float().cpu().numpy()
    worst_step = max(rel_err(o_g[t], o_ref[t]) for t in range(case.decode_steps))
    assert worst_step <= FREE_RUNNING_DECODE_CHAIN_TOL, worst_step
    s_g = S[seqs].cpu().numpy()
    worst_unit = max(rel_err(s_g[i, h], s_ref[i, h]) for i in range(len(seqs))
                     for h in range(case.H))
    assert worst_unit <= FREE_RUNNING_DECODE_CHAIN_TOL, worst_unit


def test_decode_single_head_edge(cuda_lib):
    """n_seq = 1, H = 1, d_k = 64, d_v = 128 with a zero initial state: the
    first token writes beta * v under k."""
    case = gs.Case("edge", n_seq=1, H=1, d_k=64, d_v=128, dtype="f32", qdq="none",
                   state="zero", decode_steps=1, seed=41)
    inp = gs.generate(case)
    S = torch.zeros((1, 1, 64, 128), device="cuda")
    o = cuda_lib.gdn_decode(dev(inp["dec_q"][0]), dev(inp["dec_k"][0]), dev(inp["dec_v"][0]),
                            dev(inp["dec_g"][0]), dev(inp["dec_beta"][0]), S, qdq="none")
    torch.cuda.synchronize()
    k = inp["dec_k"][0, 0, 0].double().numpy()
    v = inp["dec_v"][0, 0, 0].double().numpy()
    b = float(inp["dec_beta"][0, 0, 0])
    np.testing.assert_allclose(S[0, 0].cpu().double().numpy(), np.outer(k, b * v),
                               rtol=1e-5, atol=1e-7)


@pytest.mark.parametrize("mode", ["int8_g32", "int8_g16", "fp8_tile64"])
@pytest.mark.parametrize("lo_exp", [-140, -90])
def test_decode_codec_bit_exact_wide_range(cuda_lib, mode, lo_exp):
    """4 M state values whose groups span 2^lo_exp .. 2^60 in magnitude: the
    codec (scale, quotient, rounding, dequantization) is bit-exact against
    the oracle's IEEE fp32 codec everywhere.  From 2^-140 most warps hold a
    scale below 2^-100 and take the pre-scaled quotient; from 2^-90 none
    does and every warp divides directly."""
    gen = torch.Generator().manual_seed(123)
    N, H, dk, dv = 16, 16, 128, 128
    st = torch.randn((N, H, dk, dv), generator=gen)
    expo = torch.randint(lo_exp, 60, (N, H, dk, dv // 32), generator=gen).float()
    st = (st * torch.exp2(expo).repeat_interleave(32, dim=-1)).float()
    q = torch.randn((N, H, dk), generator=gen).to(torch.bfloat16)
    v = torch.randn((N, H, dv), generator=gen).to(torch.bfloat16)
    S = st.cuda()
    cuda_lib.gdn_decode(q.cuda(), q.cuda(), v.cuda(), torch.zeros((N, H), device="cuda"),
                        torch.zeros((N, H), device="cuda"), S, qdq=mode)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(S.cpu().numpy(), oracle.qdq(st.numpy(), mode)[0])
