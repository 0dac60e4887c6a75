"""The tensor-core prefill kernels' bounded waits, made to run out on purpose.

Every wait of those kernels (for a TMA load, an MMA commit, the CTA pair's
hand-off) is bounded; on a timeout the CTA records GDN_ERR_TIMEOUT in the
library's error word, lets its in-flight copies and MMAs finish (again
bounded), frees its TMEM and exits - it never hangs or traps (the method's
pages ask for explicit failure, never a silent fallback: PR #2507
"Experimental GDN/KDA approximate-inverse QAT", What section).  With
GDN_WAIT_LIMIT_NS=0 every wait that is not already complete gives up at
once, which drives each kernel down that path on an ordinary input.  The
call must report GDN_ERR_TIMEOUT through gdn_last_error(), and the next
ordinary call in the same process must match the oracle (the context is
still usable and the error word was cleared by the read).
"""

import numpy as np
import pytest
import torch

import gdn_synth as gs
import oracle
from parity import TOL, per_unit_rel_err, rel_err

pytestmark = pytest.mark.gpu

GDN_ERR_TIMEOUT = 4


@pytest.mark.parametrize("schedule,qdq", [("single", "fp8_tile64"), ("pair", "fp8_tile64"),
                                          ("wy", "fp8_tile64"), ("single", "int8_g32"),
                                          ("pair", "int8_g32")])
def test_wait_timeout_is_reported_and_the_context_stays_usable(cuda_lib, monkeypatch, schedule,
                                                               qdq):
    monkeypatch.delenv("GDN_PREFILL_WY", raising=False)
    monkeypatch.setenv("GDN_PREFILL_CTA_PAIR", "0" if schedule == "single" else "1")
    if schedule == "wy":
        monkeypatch.setenv("GDN_PREFILL_WY", "1")
    expect = {"single": "tc_one_cta", "pair": "tc_cta_pair", "wy": "tc_wy_pair"}[schedule]
    case = gs.Case("timeout", n_seq=2, H=2, d_k=128, d_v=128, T=3 * 64 + 5, dtype="bf16",
                   qdq=qdq, state="normal", seed=97)
    assert cuda_lib.gdn_prefill_schedule(case.n_seq, case.H, 128, 128, qdq=qdq) == expect
    inp = gs.generate(case)
    d = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in inp.items()}
    assert cuda_lib.gdn_last_error() == 0

    monkeypatch.setenv("GDN_WAIT_LIMIT_NS", "0")
    cuda_lib.gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state_in"], None, qdq=qdq)
    torch.cuda.synchronize()
    assert cuda_lib.gdn_last_error() == GDN_ERR_TIMEOUT
    assert cuda_lib.gdn_last_error() == 0  # the read cleared it

    monkeypatch.delenv("GDN_WAIT_LIMIT_NS")
    o, s = cuda_lib.gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state_in"], None,
                                qdq=qdq)
    torch.cuda.synchronize()
    cuda_lib.check_last_error(where="after the timeout")
    o_ref, s_ref = oracle.prefill(inp, case)
    assert rel_err(o.float().cpu().numpy(), o_ref.reshape(o.shape)) <= TOL["bf16"]
    assert per_unit_rel_err(s.cpu().numpy(), s_ref, axes=(-2, -1)) <= TOL["bf16"]
