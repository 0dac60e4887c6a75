"""The parity checker itself (``tests/parity.py``), on crafted cases (CPU).

The GPU parity tests accept a teacher-forced QDQ state when its codes equal
the oracle's except for at most 1e-4 of the elements, each exactly one
quantization step away, and when equal codes carry equal values up to the
scale's last bits.  These cases pin that checker: it must accept the
oracle's own state and a one-step flip (in INT8, across an FP8 binade, out
of an FP8 zero), and refuse a two-step flip, an equal code whose value
drifts, a value off the code grid, and more flips than the budget allows.
"""

import numpy as np
import pytest

import oracle
from parity import assert_flip_budget, check_codes, code_steps, per_unit_rel_err, rel_err


def _ref(mode, seed=0, shape=(2, 64, 128)):
    rng = np.random.default_rng(seed)
    X = (rng.standard_normal(shape) * 0.05).astype(np.float32)
    Y, codes, scales = oracle.qdq(X, mode)
    return Y, codes, scales


def _scale_of(scales, mode, i, r, c):
    if mode == "fp8_tile64":
        return float(scales[i, c // 64])
    return float(scales[i, r, c // int(mode[-2:])])


@pytest.mark.parametrize("mode", ["int8_g32", "fp8_tile64"])
def test_identical_state_passes(mode):
    Y, codes, scales = _ref(mode)
    st = check_codes(Y, Y, codes, scales, mode)
    assert st["flips"] == 0 and st["max_step"] == 0 and st["bit_equal_frac"] == 1.0


def test_int8_one_step_flip_is_counted_and_accepted():
    Y, codes, scales = _ref("int8_g32")
    G = Y.copy()
    r, c = 5, 40
    assert abs(codes[0, r, c]) < 127
    G[0, r, c] = np.float32((codes[0, r, c] + 1) * _scale_of(scales, "int8_g32", 0, r, c))
    steps = code_steps(G, codes, scales, "int8_g32")
    assert steps[0, r, c] == 1 and np.count_nonzero(steps) == 1
    st = check_codes(G, Y, codes, scales, "int8_g32")
    assert st["flips"] == 1 and st["max_step"] == 1


def test_int8_two_step_flip_is_refused():
    Y, codes, scales = _ref("int8_g32")
    G = Y.copy()
    r, c = 5, 40
    G[0, r, c] = np.float32((codes[0, r, c] - 2) * _scale_of(scales, "int8_g32", 0, r, c))
    with pytest.raises(AssertionError, match="more than one step"):
        check_codes(G, Y, codes, scales, "int8_g32")


def test_fp8_one_step_across_a_binade_and_out_of_zero():
    Y, codes, scales = _ref("fp8_tile64")
    G = Y.copy()
    s = _scale_of(scales, "fp8_tile64", 1, 0, 70)
    # code 1.875 * 2^-3 -> its upper neighbour 2^-2 is one step (a new binade)
    codes = codes.copy()
    codes[1, 3, 70] = 1.875 * 2.0 ** -3
    Y[1, 3, 70] = np.float32(codes[1, 3, 70] * s)
    G[1, 3, 70] = np.float32(2.0 ** -2 * s)
    # code 0 -> the smallest subnormal 2^-9, negative side
    codes[1, 4, 71] = 0.0
    Y[1, 4, 71] = 0.0
    G[1, 4, 71] = np.float32(-(2.0 ** -9) * s)
    steps = code_steps(G, codes, scales, "fp8_tile64")
    assert steps[1, 3, 70] == 1 and steps[1, 4, 71] == -1
    assert np.count_nonzero(steps) == 2
    st = check_codes(G, Y, codes, scales, "fp8_tile64")
    assert st["flips"] == 2 and st["max_step"] == 1


def test_equal_code_with_drifting_value_is_refused():
    Y, codes, scales = _ref("fp8_tile64")
    G = Y.copy()
    i, r, c = 0, 10, 5
    assert codes[i, r, c] != 0
    G[i, r, c] = np.float32(Y[i, r, c] * (1 + 1e-4))  # same code, value off by 1e-4
    with pytest.raises(AssertionError, match="equal codes"):
        check_codes(G, Y, codes, scales, "fp8_tile64")
    # within the scale tolerance (a last-bits scale difference) it passes
    G[i, r, c] = np.float32(Y[i, r, c] * (1 + 2e-7))
    check_codes(G, Y, codes, scales, "fp8_tile64")


@pytest.mark.parametrize("mode", ["int8_g32", "fp8_tile64"])
def test_off_grid_value_is_refused(mode):
    Y, codes, scales = _ref(mode)
    G = Y.copy()
    s = _scale_of(scales, mode, 0, 2, 3)
    assert codes[0, 2, 3] != 0
    if mode.startswith("int8"):
        G[0, 2, 3] = np.float32(G[0, 2, 3] + 0.3 * s)     # a third of a step
    else:
        # 1 % off: ten times the checker's relative grid tolerance, well
        # inside half an E4M3 spacing (1/16 to 1/8 of the value)
        G[0, 2, 3] = np.float32(G[0, 2, 3] * 1.01)
    with pytest.raises(AssertionError, match="grid"):
        code_steps(G, codes, scales, mode)


def test_flip_budget():
    ok = [{"elements": 20_000, "flips": 2, "bit_equal_frac": 1.0, "max_step": 1.0}]
    assert assert_flip_budget(ok)["flip_frac"] == 1e-4
    bad = [{"elements": 20_000, "flips": 3, "bit_equal_frac": 1.0, "max_step": 1.0}]
    with pytest.raises(AssertionError, match="too many"):
        assert_flip_budget(bad)


def test_relative_errors():
    ref = np.array([[3.0, 4.0], [0.0, 1.0]])
    assert rel_err(ref, ref) == 0.0
    assert rel_err(ref * 1.01, ref) == pytest.approx(0.01)
    x = ref.copy()
    x[1, 1] = 1.1                                   # unit 1 off by 10 %, unit 0 exact
    assert per_unit_rel_err(x, ref, axes=(1,)) == pytest.approx(0.1)
    assert rel_err(np.zeros(2), np.zeros(2)) == 0.0


def test_element_guard_catches_one_corrupted_element_the_norm_misses():
    """One element of a 4096 x 128 bf16-sized output off by 20 % of its row's
    largest value moves the norm-wise error by about 2e-4 (under the 2e-3
    bar) but fails the element-level guard; bf16 rounding of every element
    (at most 2^-8 of the row's largest value) passes both."""
    from parity import TOL, assert_rows_close
    rng = np.random.default_rng(5)
    ref = rng.standard_normal((4096, 128))
    x = ref.astype(np.float32).astype(np.float64)
    # round to bf16 (8-bit significands, nearest even) through the bit pattern
    b = ref.astype(np.float32).view(np.uint32)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    x = b.view(np.float32).astype(np.float64)
    assert rel_err(x, ref) <= TOL["bf16"]
    assert assert_rows_close(x, ref, "bf16") <= 2.0 ** -8
    bad = x.copy()
    bad[1234, 17] += 0.2 * np.abs(ref[1234]).max()
    assert rel_err(bad, ref) <= TOL["bf16"]
    with pytest.raises(AssertionError):
        assert_rows_close(bad, ref, "bf16")


def test_element_guard_on_rows_of_zeros():
    """A row whose reference is zero is measured against 1e-6 of the tensor's
    largest magnitude: a stray value there fails, an exact zero passes."""
    from parity import assert_rows_close
    ref = np.zeros((3, 8))
    ref[0] = 1.0
    x = ref.copy()
    assert assert_rows_close(x, ref, "f32") == 0.0
    x[2, 3] = 1e-3
    with pytest.raises(AssertionError):
        assert_rows_close(x, ref, "f32")
