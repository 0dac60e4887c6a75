"""Packed state storage (codes + scales) on the GPU.

* gdn_state_pack applies the oracle's QDQ codec bit for bit: the same codes
  (int8 integers, E4M3 values decoded here from the format's definition) and
  the same scales, and gdn_state_unpack gives the oracle's dequantized state;
* gdn_decode_packed is bit-identical to gdn_decode on the fp32 state it
  dequantizes to, step after step (outputs and states), for every codec,
  dtype, gate kind and state shape, and at the serving workload's size.
"""

import numpy as np
import pytest
import torch

import gdn_synth as gs
import oracle

pytestmark = pytest.mark.gpu

MODES = ["fp8_tile64", "int8_g16", "int8_g32", "int8_g64"]


def e4m3_value(byte: np.ndarray) -> np.ndarray:
    """E4M3 (bias 7, 3 mantissa bits, subnormals, no infinities) byte -> value."""
    b = byte.astype(np.int64)
    s = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    return s * val


def code_values(codes: torch.Tensor, mode: str) -> np.ndarray:
    c = codes.cpu().numpy()
    if mode == "fp8_tile64":
        return e4m3_value(c)
    return c.view(np.int8).astype(np.float64)


def make_states(N, H, d_k, d_v, seed):
    """N(0, 0.05^2) states with a zero tile, a zero row and tiny magnitudes."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn((N, H, d_k, d_v), generator=g) * 0.05
    x[0, 0, :, :64] = 0.0                       # a zero FP8 tile / zero INT8 groups
    x[0, H - 1, 3, :] = 0.0                     # a zero row
    x[N - 1, 0] *= 2.0 ** -110                  # scales below 2^-100: prescaled path
    x[N - 1, H - 1, :, :16] *= 1e4              # large magnitudes
    return x


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dims", [(128, 128), (64, 64), (128, 64)])
def test_pack_matches_oracle_codec(cuda_lib, mode, dims):
    sqr = cuda_lib
    d_k, d_v = dims
    x = make_states(3, 2, d_k, d_v, seed=11)
    ps = sqr.gdn_state_pack(x.cuda(), mode)
    back = sqr.gdn_state_unpack(ps)
    torch.cuda.synchronize()
    y_ref, codes_ref, scales_ref = oracle.qdq(x.numpy(), mode)
    assert np.array_equal(ps.scales.cpu().numpy().view(np.uint32),
                          scales_ref.astype(np.float32).view(np.uint32))
    assert np.array_equal(code_values(ps.codes, mode), codes_ref.astype(np.float64))
    # unpack = code * scale = the oracle's QDQ values, bit for bit (zeros by value)
    got = back.cpu().numpy()
    assert np.array_equal(got, y_ref.astype(np.float32))


def decode_inputs(N, H, d_k, d_v, dtype, gate, steps, seed):
    g = torch.Generator().manual_seed(seed)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = []
    for _ in range(steps):
        q = torch.nn.functional.normalize(torch.randn((N, H, d_k), generator=g), dim=-1).to(dt)
        k = torch.nn.functional.normalize(torch.randn((N, H, d_k), generator=g), dim=-1).to(dt)
        v = torch.randn((N, H, d_v), generator=g).to(dt)
        beta = torch.sigmoid(torch.randn((N, H), generator=g))
        gshape = (N, H) if gate == "scalar" else (N, H, d_k)
        gg = torch.nn.functional.logsigmoid(torch.randn(gshape, generator=g) + 3.0)
        out.append([t.cuda() for t in (q, k, v, gg, beta)])
    return out


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("dtype,gate,dims", [("bf16", "scalar", (128, 128)),
                                             ("f32", "scalar", (64, 64)),
                                             ("bf16", "per_key", (128, 64)),
                                             ("f32", "per_key", (64, 128))])
def test_decode_packed_bit_identical(cuda_lib, mode, dtype, gate, dims):
    sqr = cuda_lib
    d_k, d_v = dims
    N, H, steps = 5, 3, 6
    x = make_states(N, H, d_k, d_v, seed=21).cuda()
    ps = sqr.gdn_state_pack(x, mode)
    state = sqr.gdn_state_unpack(ps)        # the fp32 storage of the same QDQ'd state
    for q, k, v, g, beta in decode_inputs(N, H, d_k, d_v, dtype, gate, steps, seed=22):
        o32 = sqr.gdn_decode(q, k, v, g, beta, state, qdq=mode)
        opk = sqr.gdn_decode_packed(q, k, v, g, beta, ps)
        assert torch.equal(o32, opk)
    torch.cuda.synchronize()
    assert sqr.gdn_last_error() == 0
    assert torch.equal(sqr.gdn_state_unpack(ps), state)


def test_decode_packed_serving_shape(cuda_lib):
    """The serving workload's shape (256 sequences x 32 heads, d = 128, bf16,
    INT8 group 32) from its synthetic initial state: packed and fp32 storage
    agree bit for bit over 4 tokens."""
    sqr = cuda_lib
    case = gs.small_case("serving_decode", decode_steps=4)
    inp = gs.generate(case)
    ps = sqr.gdn_state_pack(inp["state_in"].cuda(), case.qdq)
    state = sqr.gdn_state_unpack(ps)
    for t in range(4):
        args = [inp[k][t].cuda() for k in ("dec_q", "dec_k", "dec_v", "dec_g", "dec_beta")]
        o32 = sqr.gdn_decode(*args, state, qdq=case.qdq)
        opk = sqr.gdn_decode_packed(*args, ps)
        assert torch.equal(o32, opk)
    torch.cuda.synchronize()
    assert torch.equal(sqr.gdn_state_unpack(ps), state)


def test_packed_empty_batch(cuda_lib):
    sqr = cuda_lib
    ps = sqr.packed_state_empty(0, 2, 128, 128, "int8_g32", "cuda")
    e = torch.empty((0, 2, 128), device="cuda", dtype=torch.bfloat16)
    o = sqr.gdn_decode_packed(e, e, e, torch.empty((0, 2), device="cuda"),
                              torch.empty((0, 2), device="cuda"), ps)
    assert o.shape == (0, 2, 128)


@pytest.mark.parametrize("mode", ["fp8_tile64", "int8_g32"])
def test_decode_packed_unaligned_storage(cuda_lib, mode):
    """Codes and scales at 4-byte (not 16-byte) offsets, the alignment the
    C ABI accepts: results stay bit-identical to the fp32 storage and no byte
    outside the codes is written."""
    sqr = cuda_lib
    N, H, d_k, d_v = 7, 5, 128, 128
    x = make_states(N, H, d_k, d_v, seed=31).cuda()
    ps = sqr.gdn_state_pack(x, mode)
    state = sqr.gdn_state_unpack(ps)
    cbuf = torch.zeros(ps.codes.numel() + 16, dtype=torch.uint8, device="cuda")
    sbuf = torch.zeros(ps.scales.numel() + 4, dtype=torch.float32, device="cuda")
    codes = cbuf[4:4 + ps.codes.numel()].view(ps.codes.shape)
    scales = sbuf[1:1 + ps.scales.numel()].view(ps.scales.shape)
    assert codes.data_ptr() % 16 == 4 and scales.data_ptr() % 16 == 4
    codes.copy_(ps.codes)
    scales.copy_(ps.scales)
    pu = sqr.PackedState(codes, scales, mode)
    for q, k, v, g, beta in decode_inputs(N, H, d_k, d_v, "bf16", "scalar", 3, seed=32):
        o32 = sqr.gdn_decode(q, k, v, g, beta, state, qdq=mode)
        opk = sqr.gdn_decode_packed(q, k, v, g, beta, pu)
        assert torch.equal(o32, opk)
    torch.cuda.synchronize()
    assert torch.equal(sqr.gdn_state_unpack(pu), state)
    assert torch.equal(cbuf[:4], torch.zeros(4, dtype=torch.uint8, device="cuda"))
    assert torch.equal(cbuf[4 + ps.codes.numel():], torch.zeros(12, dtype=torch.uint8, device="cuda"))
