"""gdn_prefill_backward_static (workspace in the library's static device
array) against gdn_prefill_backward (caller workspace): the same gradients,
bit for bit, on two consecutive calls with different inputs and QDQ modes.
The file sorts last so that it also runs after every other test; it passes
alone as well."""

import pytest
import torch

import gdn_synth as gs

pytestmark = pytest.mark.gpu


def _args(case, seed):
    inp = gs.generate(case)
    gen = torch.Generator().manual_seed(seed)
    d_o = torch.randn(inp["v"].shape, generator=gen).to(inp["q"].dtype)
    dso = torch.randn((case.n_seq, case.H, case.d_k, case.d_v), generator=gen)
    dev = lambda x: None if x is None else x.cuda()
    return ([dev(inp[x]) for x in ("q", "k", "v", "g", "beta")] + [dev(d_o)],
            dict(state_in=dev(inp["state_in"]), cu_seqlens=dev(inp["cu_seqlens"]),
                 dstate_out=dev(dso), qdq=case.qdq))


def test_static_workspace_matches_caller_workspace(cuda_lib):
    cases = [gs.Case("na1", n_seq=2, H=2, d_k=128, d_v=128, T=130, dtype="bf16", gate="scalar",
                     qdq="fp8_tile64", state="normal", seed=121),
             gs.Case("na2", n_seq=3, H=2, d_k=64, d_v=128, lengths=(70, 1, 64), dtype="f32",
                     gate="per_key", qdq="int8_g32", state="normal", seed=122)]
    for i, case in enumerate(cases):          # two consecutive calls of each entry point
        pos, kw = _args(case, 130 + i)
        ref = cuda_lib.gdn_prefill_backward(*pos, **kw)
        got = cuda_lib.gdn_prefill_backward_static(*pos, **kw)
        torch.cuda.synchronize()
        assert cuda_lib.gdn_last_error() == 0
        for a, b in zip(ref, got):
            assert torch.equal(a, b)
