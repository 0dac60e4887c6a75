"""Pins of the oracle's QDQ codecs (CPU only).

The codecs follow the state-QAT pages: dynamic FP8 E4M3 with one scale per
(full key x 64 value columns) tile, scale = amax / 448 with a zero guard
(PR #2497, What section); dynamic INT8 with groups of 32 along the last axis,
scale = amax / 127, round half to even, clamp (PR #2519 commit notes).

Pins, none of which re-types the oracle's own code:
 * hand-worked values (tests/golden/hand_worked.json);
 * the E4M3FN value set enumerated from the bit-level definition, and the
   rounding compared with PyTorch's float8_e4m3fn cast (a library routine);
 * the INT8 codec compared with PyTorch CPU division / torch.round /
   clamp on the same fp32 inputs;
 * invariants: codes on the grid, amax element maps to +-127 / +-448, zero
   tile/group maps to zero, idempotence, tile/group independence.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                   "hand_worked.json")))


def e4m3_value_set():
    """All finite E4M3FN values from the definition: sign, 4-bit exponent
    (bias 7), 3-bit mantissa; exponent field 0 is subnormal (m * 2^-9);
    the pattern S.1111.111 is NaN and there are no infinities."""
    vals = set()
    for s in (1.0, -1.0):
        for e in range(16):
            for m in range(8):
                if e == 15 and m == 7:
                    continue
                if e == 0:
                    v = m * 2.0 ** -9
                else:
                    v = (1.0 + m / 8.0) * 2.0 ** (e - 7)
                vals.add(s * v)
    return vals


def test_e4m3_value_set_matches_library():
    ours = e4m3_value_set()
    lib = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float()
    lib = set(float(x) for x in lib if not torch.isnan(x))
    assert ours == lib
    assert max(ours) == 448.0 and min(x for x in ours if x > 0) == 2.0 ** -9
    assert len({abs(x) for x in ours}) == 127  # 0 and 126 positive values


def test_e4m3_rounding_matches_library_cast():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * 30,
        rng.uniform(-448, 448, 200000).astype(np.float32),
        (rng.standard_normal(100000) * 1e-3).astype(np.float32),
        # exact midpoints between neighbouring grid values (ties)
        np.array(sorted(e4m3_value_set()), dtype=np.float64),
    ]).astype(np.float32)
    vs = np.array(sorted(e4m3_value_set()))
    mids = ((vs[1:] + vs[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids])
    ours = oracle.e4m3(x)
    lib = torch.from_numpy(x).to(torch.float8_e4m3fn).float().numpy()
    np.testing.assert_array_equal(ours, lib)
    assert set(np.unique(ours).astype(np.float64)) <= e4m3_value_set()


def test_e4m3_saturates():
    x = np.array([448.0, 449.0, 463.9, 464.0, 500.0, 1e6, 3e38], np.float32)
    np.testing.assert_array_equal(oracle.e4m3(x), np.full(7, 448.0, np.float32))
    np.testing.assert_array_equal(oracle.e4m3(-x), np.full(7, -448.0, np.float32))


def test_golden_fp8_tile():
    g = GOLD["fp8_tile"]
    X = np.zeros((128, 64), np.float32)
    X[3, :8] = g["x"]
    Y, codes, scales = oracle.qdq(X, "fp8_tile64")
    assert scales[0] == 1.0
    np.testing.assert_array_equal(Y[3, :8], np.array(g["y"], np.float32))
    assert np.all(Y[np.arange(128) != 3] == 0)


def test_golden_int8_group():
    g = GOLD["int8_group"]
    X = np.zeros((64, 64), np.float32)
    X[5, 32:40] = g["x"]
    Y, codes, scales = oracle.qdq(X, "int8_g32")
    assert scales[5, 1] == 1.0
    np.testing.assert_array_equal(codes[5, 32:40], np.array(g["codes"], np.float32))
    np.testing.assert_array_equal(Y[5, 32:40], np.array(g["y"], np.float32))


def _states(seed, shape=(3, 128, 128), std=0.05):
    rng = np.random.default_rng(seed)
    X = (rng.standard_normal(shape) * std).astype(np.float32)
    X[1, :, 64:] = 0.0          # a zero FP8 tile / zero INT8 groups
    X[2, 7, :] *= 50.0          # one large row
    return X


def test_int8_matches_torch_ops():
    X = _states(1)
    Y, codes, scales = oracle.qdq(X, "int8_g32")
    t = torch.from_numpy(X).reshape(3, 128, 4, 32)
    amax = t.abs().amax(-1, keepdim=True)
    s = amax / 127.0
    safe = torch.where(amax == 0, torch.ones_like(s), s)
    c = torch.round(t / safe).clamp(-127, 127)
    y = torch.where(amax == 0, torch.zeros_like(t), c * safe)
    np.testing.assert_array_equal(Y, y.reshape(3, 128, 128).numpy())
    np.testing.assert_array_equal(scales, s.reshape(3, 128, 4).numpy())


def test_fp8_matches_torch_ops():
    X = _states(2)
    Y, codes, scales = oracle.qdq(X, "fp8_tile64")
    t = torch.from_numpy(X).reshape(3, 128, 2, 64)
    amax = t.abs().amax(dim=(1, 3), keepdim=True)
    s = amax / 448.0
    safe = torch.where(amax == 0, torch.ones_like(s), s)
    c = (t / safe).to(torch.float8_e4m3fn).float()
    y = torch.where(amax == 0, torch.zeros_like(t), c * safe)
    np.testing.assert_array_equal(Y, y.reshape(3, 128, 128).numpy())
    np.testing.assert_array_equal(scales, s.reshape(3, 2).numpy())


@pytest.mark.parametrize("mode", ["int8_g32", "fp8_tile64", "int8_g16", "int8_g64"])
def test_codec_invariants(mode):
    X = _states(3)
    Y, codes, scales = oracle.qdq(X, mode)
    if mode.startswith("int8"):
        assert np.all(codes == np.round(codes)) and np.abs(codes).max() <= 127
        grp = int(mode[-2:])
        g = np.abs(X).reshape(3, 128, 128 // grp, grp)
        cg = np.abs(codes).reshape(3, 128, 128 // grp, grp)
        nz = g.max(-1) > 0
        # the amax element of every nonzero group codes to exactly 127
        assert np.all(cg.max(-1)[nz] == 127)
        assert np.all(cg.max(-1)[~nz] == 0)
    else:
        assert set(np.unique(codes).astype(np.float64)) <= e4m3_value_set()
        t = np.abs(codes).reshape(3, 128, 2, 64)
        assert t.max(axis=(1, 3))[0, 0] == 448.0
        assert np.all(t.max(axis=(1, 3))[1] == [448.0, 0.0])
    # zero tile / groups stay zero; the large row does not leak to other tiles
    assert np.all(Y[1, :, 64:] == 0)
    # idempotence: QDQ(QDQ(x)) == QDQ(x)
    Y2, _, _ = oracle.qdq(Y, mode)
    np.testing.assert_array_equal(Y2, Y)


def test_fp8_tile_independence():
    X = _states(4)
    Y, _, s0 = oracle.qdq(X, "fp8_tile64")
    X2 = X.copy()
    X2[0, 100, 70] = 9.0        # only the second tile of state 0 changes
    Y2, _, s1 = oracle.qdq(X2, "fp8_tile64")
    np.testing.assert_array_equal(Y2[0, :, :64], Y[0, :, :64])
    np.testing.assert_array_equal(Y2[1:], Y[1:])
    assert s1[0, 1] != s0[0, 1] and s1[0, 0] == s0[0, 0]


def test_int8_group_axis():
    X = _states(5)
    X2 = X.copy()
    X2[0, 9, 40] = 3.0          # one group along the value axis of row 9
    Y, _, _ = oracle.qdq(X, "int8_g32")
    Y2, _, _ = oracle.qdq(X2, "int8_g32")
    diff = np.argwhere(Y2 != Y)
    assert set(map(tuple, diff[:, :2])) == {(0, 9)}
    assert diff[:, 2].min() >= 32 and diff[:, 2].max() < 64
    # the other reading (groups along the key axis) changes a column group
    Yk, _, _ = oracle.qdq(X, "int8_g32", axis=0)
    Yk2, _, _ = oracle.qdq(X2, "int8_g32", axis=0)
    diff = np.argwhere(Yk2 != Yk)
    assert set(diff[:, 2]) == {40} and diff[:, 1].min() >= 0 and diff[:, 1].max() < 32
