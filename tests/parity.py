"""Parity helpers: compare the CUDA path's results with the oracle's.

Criteria (the method's stated bar, read as follows where it is literal
about bits that the fp32 GPU arithmetic cannot reproduce from an fp64
trajectory):

* codec alone (identical fp32 input on both sides): bit-equal;
* teacher-forced (the oracle restarts every chunk / decode step from the
  GPU's own state): outputs within the float tolerance, norm-wise and
  element by element (``assert_rows_close``); the QDQ'd state compared code
  by code - at most 1e-4 of the elements may differ, each by exactly one
  quantization step.  A tile's (group's) scale is amax / 448 (/ 127), and
  the two sides' pre-QDQ amax differ in their last bits (fp32 chains against
  an fp64 trajectory), so the scales are compared to ``scale_rtol`` = 1e-5
  relative; an element whose code is equal then differs by exactly its
  code times that scale difference.  The fraction of bit-equal elements is
  reported, not asserted: one ulp of amax changes every value of the tile;
* free-running: norm-wise relative error within the float tolerance (and,
  with the QDQ off, element by element as well).
"""

from __future__ import annotations

import numpy as np

TOL = {"bf16": 2e-3, "f32": 1e-5}
MAX_FLIP_FRAC = 1e-4
# Element-level bound beside the norm-wise one, relative to the largest
# magnitude of the element's row (one token and head of o): bf16 storage
# alone moves an element by up to 2^-8 of the row's largest value (half an
# ulp of an 8-bit significand at the row's top binade), so 4 * 2^-9 = 2^-7
# leaves as much again for the arithmetic.  fp32 rows: ten times the
# norm-wise bar.
ELEM_TOL = {"bf16": 4 * 2.0 ** -9, "f32": 1e-4}


def rel_err(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (den if den > 0 else 1.0))


def per_unit_rel_err(x, ref, axes) -> float:
    """Largest norm-wise relative error over the units (e.g. (seq, head))."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    num = np.sqrt(((x - ref) ** 2).sum(axis=axes))
    den = np.sqrt((ref ** 2).sum(axis=axes))
    den = np.where(den > 0, den, 1.0)
    return float((num / den).max())


def assert_rows_close(x, ref, dtype: str, label: str = "") -> float:
    """Every element within ELEM_TOL[dtype] of its last-axis row's largest
    reference magnitude (rows whose reference is all but zero are measured
    against 1e-6 of the tensor's largest magnitude).  Returns the worst
    ratio |x - ref| / row scale."""
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64).reshape(x.shape)
    row = np.abs(ref).max(axis=-1, keepdims=True)
    floor = 1e-6 * (float(np.abs(ref).max()) if ref.size else 0.0)
    den = np.maximum(row, max(floor, 1e-30))
    worst = float((np.abs(x - ref) / den).max()) if x.size else 0.0
    assert worst <= ELEM_TOL[dtype], f"{label}: element error {worst:.3e} of its row's scale"
    return worst


def _e4m3_grid() -> np.ndarray:
    vals = set()
    for e in range(16):
        for m in range(8):
            if e == 15 and m == 7:
                continue
            v = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
            vals.add(v)
            vals.add(-v)
    return np.array(sorted(vals))


_GRID = _e4m3_grid()


def _expand_scales(scales, mode: str, shape):
    """Per-element oracle scale for states of `shape` [..., d_k, d_v]."""
    d_k, d_v = shape[-2:]
    lead = shape[:-2]
    if mode == "fp8_tile64":
        s = scales.reshape(lead + (1, d_v // 64, 1))
        return np.broadcast_to(s, lead + (d_k, d_v // 64, 64)).reshape(shape)
    grp = int(mode[-2:])
    s = scales.reshape(lead + (d_k, d_v // grp, 1))
    return np.broadcast_to(s, lead + (d_k, d_v // grp, grp)).reshape(shape)


def code_steps(y_gpu, codes_ref, scales_ref, mode: str):
    """Signed number of quantization steps between the GPU's dequantized
    state and the oracle's codes, measured on the oracle's scale grid."""
    y = np.asarray(y_gpu, dtype=np.float64)
    s = _expand_scales(np.asarray(scales_ref, dtype=np.float64), mode, y.shape)
    safe = np.where(s > 0, s, 1.0)
    t = np.where(s > 0, y / safe, y)
    c = np.asarray(codes_ref, dtype=np.float64)
    if mode.startswith("int8"):
        ci = np.rint(t)
        assert np.abs(t - ci).max() < 1e-3, "GPU state is not on the oracle's INT8 grid"
        return ci - c
    idx_gpu = np.clip(np.searchsorted(_GRID, t), 1, len(_GRID) - 1)
    lo, hi = _GRID[idx_gpu - 1], _GRID[idx_gpu]
    idx_gpu = np.where(np.abs(t - lo) <= np.abs(t - hi), idx_gpu - 1, idx_gpu)
    snapped = _GRID[idx_gpu]
    assert np.all(np.abs(t - snapped) <= 1e-3 * np.maximum(np.abs(snapped), 2.0 ** -9)), \
        "GPU state is not on the oracle's E4M3 grid"
    idx_ref = np.searchsorted(_GRID, c)      # the grid holds a single zero
    return (idx_gpu - idx_ref).astype(np.float64)


def check_codes(y_gpu, y_ref, codes_ref, scales_ref, mode: str, *, label: str = "",
                scale_rtol: float = 1e-5) -> dict:
    """Teacher-forced QDQ state comparison; asserts the bar and returns stats.

    Codes: at most one step apart (the 1e-4 budget is checked over a whole
    run by ``assert_flip_budget``).  Scales: an element with equal codes is
    code * s on both sides, so its relative difference is exactly the
    relative difference of the two scales of its tile or group; asserting
    it within ``scale_rtol`` for every such element bounds every scale of
    the state to that.  Zero-coded elements are exact zeros on both sides."""
    steps = code_steps(y_gpu, codes_ref, scales_ref, mode)
    n = steps.size
    flips = int(np.count_nonzero(steps))
    max_step = float(np.abs(steps).max()) if n else 0.0
    y = np.asarray(y_gpu, dtype=np.float32)
    r = np.asarray(y_ref, dtype=np.float32)
    same = steps == 0
    bit_equal = int(np.count_nonzero((y == r) & same))
    dev = np.abs(y.astype(np.float64) - r.astype(np.float64))
    tol = scale_rtol * np.abs(r.astype(np.float64))
    worst = float((dev[same] / np.maximum(np.abs(r[same]), 1e-30)).max()) if same.any() else 0.0
    stats = {"elements": n, "flips": flips, "flip_frac": flips / max(n, 1),
             "max_step": max_step, "bit_equal_frac": bit_equal / max(n, 1),
             "equal_code_max_rel": worst}
    assert np.all(dev[same] <= tol[same]), f"{label}: equal codes but values differ: {stats}"
    assert max_step <= 1.0, f"{label}: a code differs by more than one step: {stats}"
    return stats


def assert_flip_budget(stats_list, label: str = "") -> dict:
    """Aggregate teacher-forced comparisons (all boundaries of a run) and
    assert that at most 1e-4 of the compared state elements flipped."""
    n = sum(s["elements"] for s in stats_list)
    flips = sum(s["flips"] for s in stats_list)
    total = {"elements": n, "flips": flips, "flip_frac": flips / max(n, 1),
             "max_step": max((s["max_step"] for s in stats_list), default=0.0),
             "bit_equal_frac": sum(s["bit_equal_frac"] * s["elements"] for s in stats_list) / max(n, 1)}
    assert flips <= MAX_FLIP_FRAC * n, f"{label}: too many one-step code differences: {total}"
    return total
