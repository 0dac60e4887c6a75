"""GPU parity of gdn_prefill_w_qdq (the FP8 QDQ of the WY-transformed W, one
scale per row of W, on top of the FP8 tile state QDQ) against the fp64
chunked oracle with the same W codec (``oracle.chunked``, w_qdq="fp8_row").

* free-running: dense (zero and random initial states) and packed sequences
  with partial last chunks; outputs norm-wise and per element, states per
  (sequence, head); the W codec must matter (the oracle's states without it
  are far further away than the GPU's are from the oracle's with it);
* teacher-forced chunk by chunk: the oracle restarted from the GPU's own
  state at every boundary gives the state codes within the one-step / 1e-4
  budget;
* the GDN prefill workload (B=4, H=16, T=4096) on 16 sampled units;
* w_qdq="none" through the same entry point is gdn_prefill bit for bit.

Outputs are compared norm-wise only, also chunk by chunk: the two sides form
W in different arithmetic (fp32 tensor-core products against fp64), so a W
element within an ulp of an E4M3 rounding boundary can take the
neighbouring code on one side - the one-step code difference the parity bar
admits - and such a flip moves a whole row of V_new, hence single outputs
by up to about 1 % of their row.
"""

import numpy as np
import pytest
import torch

import gdn_synth as gs
import oracle
from oracle import chunked
from parity import TOL, assert_flip_budget, check_codes, per_unit_rel_err, rel_err

pytestmark = pytest.mark.gpu


def _dev(inp):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}


def _gpu(cuda_lib, inp, qdq="fp8_tile64", w_qdq="fp8_row"):
    d = _dev(inp)
    o, s = cuda_lib.gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state_in"],
                                d["cu_seqlens"], qdq=qdq, w_qdq=w_qdq)
    torch.cuda.synchronize()
    cuda_lib.check_last_error(where="gdn_prefill_w_qdq")
    return o.float().cpu().numpy(), s.cpu().numpy()


@pytest.mark.parametrize("kind", ["dense_zero", "dense_random", "packed"])
def test_w_qdq_free_running(cuda_lib, kind):
    if kind == "packed":
        case = gs.Case("wq", n_seq=5, H=2, d_k=128, d_v=128, lengths=(1, 63, 64, 65, 200),
                       dtype="bf16", qdq="fp8_tile64", state="normal", seed=141)
    else:
        case = gs.Case("wq", n_seq=2, H=3, d_k=128, d_v=128, T=5 * 64 + 17, dtype="bf16",
                       qdq="fp8_tile64", state="zero" if kind == "dense_zero" else "normal",
                       seed=142)
    inp = gs.generate(case)
    o, s = _gpu(cuda_lib, inp)
    o_ref, s_ref = chunked.chunked_dense(inp, case, qdq="fp8_tile64", w_qdq="fp8_row")
    e_o = rel_err(o, o_ref.reshape(o.shape))
    assert e_o <= TOL["bf16"], e_o
    assert per_unit_rel_err(s, s_ref, axes=(-2, -1)) <= TOL["bf16"]
    # the W codec is really applied: without it the oracle's states are much
    # further away (its effect on the bf16 outputs, about 1e-3, is below their
    # rounding; on the fp32 states it is about 1e-2)
    _, s_nw = chunked.chunked_dense(inp, case, qdq="fp8_tile64")
    assert rel_err(s, s_nw) > 5 * rel_err(s, s_ref)


def test_w_qdq_teacher_forced_chunks(cuda_lib):
    """One call per chunk (state handed over), each compared with the oracle's
    chunk restarted from the GPU's chunk-start state."""
    case = gs.Case("wqtf", n_seq=1, H=4, d_k=128, d_v=128, T=6 * 64 + 9, dtype="bf16",
                   qdq="fp8_tile64", state="normal", seed=143)
    inp = gs.generate(case)
    H = case.H
    st = inp["state_in"].clone()
    stats, worst = [], 0.0
    for c0 in range(0, case.T, 64):
        c1 = min(c0 + 64, case.T)
        sub = {x: inp[x][:, c0:c1].contiguous() for x in ("q", "k", "v", "g", "beta")}
        sub.update(state_in=st, cu_seqlens=None)
        o_g, s_g = _gpu(cuda_lib, sub)
        scale = 1.0 / np.sqrt(case.d_k)
        pre = np.zeros((1, H, 128, 128))
        o_r = np.zeros((c1 - c0, H, 128))
        for h in range(H):
            args = [oracle._f64(sub[x][0, :, h]) for x in ("q", "k", "v", "g", "beta")]
            o_r[:, h], pre[0, h] = chunked.chunk_step(*args, st[0, h].double().numpy(),
                                                      per_key_gate=False, scale=scale,
                                                      w_qdq="fp8_row")
        y, codes, scales = oracle.qdq(pre.astype(np.float32), "fp8_tile64")
        worst = max(worst, rel_err(o_g[0], o_r))
        stats.append(check_codes(s_g, y, codes, scales, "fp8_tile64",
                                 label=f"w qdq chunk {c0 // 64}"))
        st = torch.from_numpy(s_g)
    assert worst <= TOL["bf16"], worst
    assert_flip_budget(stats, "w qdq teacher-forced")


def test_w_qdq_full_gdn_workload(cuda_lib):
    """B=4, H=16, T=4096 with both QDQ sites: 16 sampled units free-running
    against the chunked oracle."""
    case = gs.CONFIGS["gdn_prefill"]
    inp = gs.generate(case)
    o, s = _gpu(cuda_lib, inp)
    scale = 1.0 / np.sqrt(case.d_k)
    for (si, h) in [(si, h) for si in range(4) for h in (0, 5, 10, 15)]:
        args = [oracle._f64(inp[x][si, :, h]) for x in ("q", "k", "v", "g", "beta")]
        Hs = np.zeros((128, 128))
        o_r = np.zeros((case.T, 128))
        for c0 in range(0, case.T, 64):
            sl = slice(c0, c0 + 64)
            o_r[sl], Hs = chunked.chunk_step(*(a[sl] for a in args), Hs, per_key_gate=False,
                                             scale=scale, w_qdq="fp8_row")
            Hs = oracle.qdq(Hs.astype(np.float32), "fp8_tile64")[0].astype(np.float64)
        assert rel_err(o[si, :, h], o_r) <= TOL["bf16"], (si, h)
        assert rel_err(s[si, h], Hs) <= TOL["bf16"], (si, h)


def test_w_qdq_none_is_gdn_prefill(cuda_lib):
    case = gs.Case("wqn", n_seq=2, H=2, d_k=128, d_v=128, T=200, dtype="bf16",
                   qdq="fp8_tile64", state="normal", seed=144)
    inp = gs.generate(case)
    a = _gpu(cuda_lib, inp, w_qdq="none")
    d = _dev(inp)
    o, s = cuda_lib.gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state_in"], None,
                                qdq="fp8_tile64")
    torch.cuda.synchronize()
    np.testing.assert_array_equal(a[0], o.float().cpu().numpy())
    np.testing.assert_array_equal(a[1], s.cpu().numpy())
