"""The seeded input recipe shared by the oracle and the CUDA path (CPU).

``gdn_synth`` holds none of the method's arithmetic; it only draws inputs.
These checks pin it to the stated recipe and workload shapes:

* the five workloads carry the benchmark description's shapes, dtypes, gate
  kinds, codecs, initial states and decode lengths;
* q and k are unit rows over d_k (before the cast), v ~ N(0, 1),
  beta = sigmoid(N(0, 1)) in (0, 1), g = log sigmoid(N(3, 1)) < 0, random
  states N(0, 0.05^2), packed lengths in [1, 4096] with int32 cu_seqlens;
* a seed gives the same inputs every time, another seed other inputs.
"""

import numpy as np
import torch

import gdn_synth as gs


def test_workload_shapes():
    c = gs.CONFIGS
    t = c["tiny"]
    assert (t.n_seq, t.H, t.d_k, t.d_v, t.T, t.dtype, t.qdq, t.state, t.decode_steps) == \
        (1, 2, 64, 64, 64, "f32", "int8_g32", "zero", 64)
    g = c["gdn_prefill"]
    assert (g.n_seq, g.H, g.d_k, g.d_v, g.T, g.dtype, g.gate, g.qdq, g.state) == \
        (4, 16, 128, 128, 4096, "bf16", "scalar", "fp8_tile64", "zero")
    k = c["kda_prefill"]
    assert (k.n_seq, k.H, k.d_k, k.d_v, k.T, k.dtype, k.gate, k.qdq, k.state) == \
        (2, 32, 128, 128, 8192, "bf16", "per_key", "int8_g32", "zero")
    s = c["serving_decode"]
    assert (s.n_seq, s.H, s.d_k, s.d_v, s.dtype, s.qdq, s.state, s.state_std, s.decode_steps) == \
        (256, 32, 128, 128, "bf16", "int8_g32", "normal", 0.05, 512)
    v = c["varlen"]
    assert (v.n_seq, v.H, v.varlen_max, v.dtype, v.qdq, v.state, v.decode_steps) == \
        (64, 16, 4096, "bf16", "fp8_tile64", "normal", 32)
    assert [c[n].seed for n in ("tiny", "gdn_prefill", "kda_prefill", "serving_decode",
                                "varlen")] == [1000, 1001, 1002, 1003, 1004]


def test_distributions_dense_and_decode():
    case = gs.small_case("kda_prefill", n_seq=2, H=4, T=512, dtype="f32", state="normal",
                         decode_steps=8)
    inp = gs.generate(case)
    assert inp["cu_seqlens"] is None and inp["q"].shape == (2, 512, 4, 128)
    for name in ("q", "k", "dec_q", "dec_k"):
        n = inp[name].double().norm(dim=-1)
        assert torch.allclose(n, torch.ones_like(n), atol=1e-6), name
    v = inp["v"].double()
    assert abs(v.mean().item()) < 0.02 and abs(v.std().item() - 1) < 0.02
    b = inp["beta"]
    assert b.dtype == torch.float32 and (b > 0).all() and (b < 1).all()
    assert abs(b.mean().item() - 0.5) < 0.02
    g = inp["g"]
    assert g.dtype == torch.float32 and g.shape == (2, 512, 4, 128) and (g < 0).all()
    # log sigmoid(x) for x ~ N(3, 1): the median is log sigmoid(3)
    assert abs(g.median().item() - float(np.log(1 / (1 + np.exp(-3.0))))) < 2e-3
    st = inp["state_in"]
    assert st.shape == (2, 4, 128, 128) and abs(st.std().item() - 0.05) < 1e-3
    assert inp["dec_g"].shape == (8, 2, 4, 128) and inp["dec_v"].shape == (8, 2, 4, 128)


def test_bf16_cast_of_unit_rows():
    inp = gs.generate(gs.small_case("gdn_prefill", n_seq=1, H=2, T=256))
    assert inp["q"].dtype == torch.bfloat16 and inp["g"].shape == (1, 256, 2)
    n = inp["k"].double().norm(dim=-1)
    assert (n - 1).abs().max().item() < 1e-2     # bf16 rounding of unit rows
    assert inp["state_in"] is None


def test_packed_lengths():
    # the varlen workload's lengths, with one head to keep the draw small
    inp = gs.generate(gs.small_case("varlen", H=1, decode_steps=0))
    L = inp["lengths"]
    cu = inp["cu_seqlens"]
    assert len(L) == 64 and min(L) >= 1 and max(L) <= 4096
    assert cu.dtype == torch.int32 and cu[0] == 0 and cu[-1] == sum(L)
    assert torch.equal(cu[1:] - cu[:-1], torch.tensor(L, dtype=torch.int32))
    assert inp["q"].shape == (1, sum(L), 1, 128)


def test_seeds_are_deterministic():
    a = gs.generate(gs.small_case("gdn_prefill", n_seq=1, H=2, T=128))
    b = gs.generate(gs.small_case("gdn_prefill", n_seq=1, H=2, T=128))
    c = gs.generate(gs.small_case("gdn_prefill", n_seq=1, H=2, T=128, seed=7))
    for name in ("q", "k", "v", "g", "beta"):
        assert torch.equal(a[name], b[name]), name
        assert not torch.equal(a[name], c[name]), name
