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


def test_static_workspace_call_allocates_nothing(cuda_lib):
    """The reason the static entry point exists: with every output made by
    the caller beforehand, a call reserves no device memory at all - the
    free device memory the driver reports, torch's allocated bytes and its
    allocation count are the same before and after a second call (the first
    one may still load the kernel's module)."""
    import ctypes

    case = gs.Case("na3", n_seq=2, H=2, d_k=128, d_v=128, T=200, dtype="bf16", gate="scalar",
                   qdq="int8_g32", state="normal", seed=123)
    (q, k, v, g, beta, d_o), kw = _args(case, 140)
    f32 = dict(dtype=torch.float32, device="cuda")
    outs = [torch.empty(q.shape, **f32), torch.empty(q.shape, **f32), torch.empty(v.shape, **f32),
            torch.empty(g.shape, **f32), torch.empty(beta.shape, **f32),
            torch.empty((case.n_seq, case.H, case.d_k, case.d_v), **f32)]
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        s = cuda_lib.lib.gdn_prefill_backward_static(
            P(q), P(k), P(v), P(g), P(beta), P(kw["state_in"]), None, case.n_seq, case.T,
            case.H, case.d_k, case.d_v, 0, 0, cuda_lib.GDN_QDQ[case.qdq], P(d_o),
            P(kw["dstate_out"]), *[P(t) for t in outs], stream)
        assert s == 0, s

    call()
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    alloc0 = torch.cuda.memory_allocated()
    n0 = torch.cuda.memory_stats().get("allocation.all.allocated", 0)
    call()
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.memory_stats().get("allocation.all.allocated", 0) == n0
    assert cuda_lib.gdn_last_error() == 0
    ref = cuda_lib.gdn_prefill_backward(q, k, v, g, beta, d_o, **kw)
    torch.cuda.synchronize()
    for a, b in zip(ref, outs):
        assert torch.equal(a, b)
