"""GPU parity of gdn_prefill_neumann (the approximate triangular solve)
against the oracle's chunked form with the same Neumann degree.

* free-running, QDQ off: every supported degree, bf16 and fp32, GDN and KDA
  gates, d_k, d_v in {64, 128}, packed lengths 1, 63, 64, 65, 200;
* degree 63 is exact on every chunk (strictly lower A is nilpotent): it
  agrees with gdn_prefill; degree 1 does not;
* QDQ on: one call per chunk, each compared with the oracle restarted from
  the GPU's chunk-start state, codes within the flip budget.
"""

import numpy as np
import pytest
import torch

import gdn_synth as gs
import oracle
from oracle import chunked
from parity import TOL, assert_flip_budget, check_codes, per_unit_rel_err, rel_err

pytestmark = pytest.mark.gpu

DEGREES = [1, 3, 7, 15, 31, 63]


def dev(x):
    return None if x is None else x.cuda()


def run_gpu(cuda_lib, inp, case, degree):
    o, s = cuda_lib.gdn_prefill(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]), dev(inp["g"]),
                                dev(inp["beta"]), dev(inp["state_in"]), dev(inp["cu_seqlens"]),
                                qdq=case.qdq, neumann_degree=degree)
    torch.cuda.synchronize()
    cuda_lib.check_last_error(where="gdn_prefill_neumann")
    return o.float().cpu().numpy(), s.cpu().numpy()


def oracle_neumann(inp, case, degree, qdq="none"):
    return chunked.chunked_wy(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                              inp["state_in"], inp["cu_seqlens"].numpy(),
                              per_key_gate=case.gate == "per_key", qdq=qdq,
                              solve=("neumann", degree))


@pytest.mark.parametrize("degree", DEGREES)
@pytest.mark.parametrize("gate", ["scalar", "per_key"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (128, 64)])
def test_neumann_free_running(cuda_lib, degree, gate, dtype, dk, dv):
    case = gs.Case("neu", n_seq=5, H=2, d_k=dk, d_v=dv, lengths=(1, 63, 64, 65, 200),
                   dtype=dtype, gate=gate, qdq="none", state="normal", seed=81)
    inp = gs.generate(case)
    o, s = run_gpu(cuda_lib, inp, case, degree)
    o_ref, s_ref = oracle_neumann(inp, case, degree)
    assert rel_err(o, o_ref.reshape(o.shape)) <= TOL[dtype]
    assert per_unit_rel_err(s, s_ref, axes=(-2, -1)) <= TOL[dtype]


@pytest.mark.parametrize("dtype,gate,dk", [("bf16", "scalar", 128), ("f32", "per_key", 64),
                                           ("bf16", "per_key", 128)])
def test_neumann_degree_63_is_exact_degree_1_is_not(cuda_lib, dtype, gate, dk):
    case = gs.Case("neu63", n_seq=3, H=2, d_k=dk, d_v=dk, lengths=(64, 130, 7), dtype=dtype,
                   gate=gate, qdq="none", state="normal", seed=82)
    inp = gs.generate(case)
    o63, s63 = run_gpu(cuda_lib, inp, case, 63)
    o_ex, s_ex = cuda_lib.gdn_prefill(dev(inp["q"]), dev(inp["k"]), dev(inp["v"]),
                                      dev(inp["g"]), dev(inp["beta"]), dev(inp["state_in"]),
                                      dev(inp["cu_seqlens"]), qdq="none")
    o_ex, s_ex = o_ex.float().cpu().numpy(), s_ex.cpu().numpy()
    assert rel_err(o63, o_ex) <= TOL[dtype]
    assert rel_err(s63, s_ex) <= TOL[dtype]
    o1, _ = run_gpu(cuda_lib, inp, case, 1)
    assert rel_err(o1, o_ex) > 3 * TOL[dtype]


@pytest.mark.parametrize("mode,degree,dtype,gate", [("int8_g32", 3, "f32", "scalar"),
                                                    ("fp8_tile64", 7, "f32", "per_key"),
                                                    ("int8_g32", 15, "bf16", "per_key"),
                                                    ("fp8_tile64", 31, "bf16", "scalar")])
def test_neumann_teacher_forced_qdq(cuda_lib, mode, degree, dtype, gate):
    """Each chunk as its own call from the previous call's state: outputs
    against the oracle from the same start state, and the QDQ'd state against
    the oracle's codec of its pre-QDQ state."""
    case = gs.Case("neuq", n_seq=2, H=2, d_k=128, d_v=128, lengths=(150, 64), dtype=dtype,
                   gate=gate, qdq=mode, state="normal", seed=83)
    inp = gs.generate(case)
    lengths = inp["lengths"]
    starts = np.concatenate([[0], np.cumsum(lengths)])
    flat = {x: inp[x].reshape((-1,) + inp[x].shape[2:]) for x in ("q", "k", "v", "g", "beta")}
    stats, worst_o = [], 0.0
    for si, L in enumerate(lengths):
        st = inp["state_in"][si:si + 1].clone()
        for c0 in range(0, L, 64):
            c1 = min(c0 + 64, L)
            sl = slice(int(starts[si] + c0), int(starts[si] + c1))
            sub = {x: flat[x][sl][None] for x in flat}
            sub["state_in"], sub["cu_seqlens"] = st, torch.tensor([0, c1 - c0], dtype=torch.int32)
            sub_case = gs.Case("chunk", n_seq=1, H=case.H, d_k=128, d_v=128, T=c1 - c0,
                               dtype=dtype, gate=gate, qdq=mode)
            o_c, s_c = run_gpu(cuda_lib, sub, sub_case, degree)
            o_r, s_pre = oracle_neumann(sub, sub_case, degree, qdq="none")
            worst_o = max(worst_o, rel_err(o_c, o_r.reshape(o_c.shape)))
            y_ref, codes, scales = oracle.qdq(s_pre.astype(np.float32), mode)
            stats.append(check_codes(s_c, y_ref, codes, scales, mode,
                                     label=f"{mode} d={degree} seq {si} chunk {c0 // 64}"))
            st = torch.from_numpy(s_c)
    assert worst_o <= TOL[dtype]
    assert_flip_budget(stats, f"neumann {mode} {degree}")
