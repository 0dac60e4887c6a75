"""CPU oracle for the gated delta rule with a fake-quantized (QDQ) state.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the benchmark's CPU-baseline leg may import this package; the product path
(``state_quantized_recurrence_b200``) never does, and the two share no code.

Modes:

* :func:`recurrence` - the definition: the fp64 token-by-token gated delta
  rule with the fp32 QDQ codecs at chunk boundaries / after decode tokens,
  in plain C (``gdn_oracle.c``), OpenMP over independent (sequence, head).
* :func:`oracle.chunked.chunked_wy` - the 64-token chunked WY form in fp64
  numpy, used to pin the chunked algebra against the token recurrence (and,
  with ``solve=("neumann", d)``, the approximate solve).
* :func:`oracle.backward.backward` - the fp64 reverse pass of the token
  recurrence with the state QDQ passed straight through;
  :func:`oracle.backward.chunked_backward` - the same gradients chunk by
  chunk (the adjoint of the chunked WY form), pinned to the token pass, and
  :func:`oracle.backward.chunk_state_gradient`, its sequential part alone.

Pins: every function here is checked by ``tests/test_oracle_*.py`` against
closed forms, invariants, special cases and library routines (see the
tests' docstrings); ``tests/test_oracle_mutants.py`` plants single mistakes
in copies of the C recurrence, the codecs, the chunked form and the backward
and requires each to fail a pin.  Nothing stored or computed here comes from the CUDA path.
"""

from __future__ import annotations

import ctypes
import hashlib
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

QDQ_NONE, QDQ_FP8_TILE, QDQ_INT8_GROUP = 0, 1, 2
_QDQ_NAMES = {"none": QDQ_NONE, "fp8_tile64": QDQ_FP8_TILE,
              "int8_g32": QDQ_INT8_GROUP, "int8_g16": QDQ_INT8_GROUP,
              "int8_g64": QDQ_INT8_GROUP}
_QDQ_GROUP = {"int8_g32": 32, "int8_g16": 16, "int8_g64": 64}

CHUNK = 64


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile ``liboracle.so`` with gcc (no fast-math, no FP contraction).
    ``src``/``out`` let the tests compile a copy with a planted mistake."""
    cmd = ["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", "-fno-finite-math-only",
           "-o", out + ".tmp", src, "-lm"]
    # staleness by content (flags + source), not modification times
    h = hashlib.sha256(" ".join(cmd[:-4]).encode())
    with open(src, "rb") as f:
        h.update(f.read())
    digest, stamp = h.hexdigest(), out + ".sha256"
    if not force and os.path.exists(out) and os.path.exists(stamp):
        with open(stamp) as f:
            if f.read().strip() == digest:
                return out
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    with open(stamp, "w") as f:
        f.write(digest + "\n")
    return out


_lib = None


def _load():
    global _lib
    if _lib is None:
        _lib = bind(build())
    return _lib


def bind(path: str):
    """Load a compiled oracle library and declare its entry points."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    lib.or_e4m3_rne_satfinite.argtypes = [ctypes.c_float]
    lib.or_e4m3_rne_satfinite.restype = ctypes.c_float
    lib.or_e4m3_array.argtypes = [P, P, ctypes.c_long]
    lib.or_e4m3_array.restype = None
    lib.or_qdq.argtypes = [P, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                           ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
    lib.or_qdq.restype = ctypes.c_int
    lib.or_gdn_recurrence.argtypes = [P] * 7 + [ctypes.c_int] * 9 + [P] * 4 + [ctypes.c_int]
    lib.or_gdn_recurrence.restype = ctypes.c_int
    lib.or_max_threads.argtypes = []
    lib.or_max_threads.restype = ctypes.c_int
    return lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def max_threads() -> int:
    return int(_load().or_max_threads())


def qdq_mode_of(name: str):
    """(mode, group) for a codec name such as 'fp8_tile64' or 'int8_g32'."""
    return _QDQ_NAMES[name], _QDQ_GROUP.get(name, 32)


def e4m3(x) -> np.ndarray:
    """Round fp32 values to E4M3FN (nearest, ties to even, saturate at 448)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty_like(x)
    _load().or_e4m3_array(_ptr(x), _ptr(out), x.size)
    return out


def qdq(X, mode: str, axis: int = 1):
    """Fake-quantize fp32 states ``X[..., d_k, d_v]``.

    Returns ``(Y, codes, scales)``: the dequantized fp32 states, the code of
    each element (INT8 integer or E4M3 value, as fp32) and the scales (FP8:
    ``[..., d_v // 64]``; INT8 axis 1: ``[..., d_k, d_v // group]``).
    """
    X = np.array(X, dtype=np.float32, order="C", copy=True)
    d_k, d_v = X.shape[-2:]
    count = X.size // (d_k * d_v)
    m, grp = qdq_mode_of(mode)
    if m == QDQ_NONE:
        return X, None, None
    codes = np.empty_like(X)
    if m == QDQ_FP8_TILE:
        scales = np.empty(X.shape[:-2] + (d_v // 64,), dtype=np.float32)
    elif axis == 1:
        scales = np.empty(X.shape[:-2] + (d_k, d_v // grp), dtype=np.float32)
    else:
        scales = np.empty(X.shape[:-2] + (d_k // grp, d_v), dtype=np.float32)
    rc = _load().or_qdq(_ptr(X), count, d_k, d_v, m, grp, axis, _ptr(codes),
                        _ptr(scales))
    if rc != 0:
        raise ValueError("oracle qdq: bad arguments")
    return X, codes, scales


def _f64(t) -> np.ndarray:
    if t is None:
        return None
    if hasattr(t, "detach"):
        t = t.detach().cpu().double().numpy()
    return np.ascontiguousarray(t, dtype=np.float64)


def recurrence(q, k, v, g, beta, state_in, cu_seqlens, *, per_key_gate: bool,
               qdq: str = "none", boundary_every: int = CHUNK,
               qdq_axis: int = 1, n_threads: int = 0, want_codes: bool = False):
    """fp64 token recurrence over packed sequences.

    ``q, k``: [total_T, H, d_k]; ``v``: [total_T, H, d_v]; ``g``: [total_T, H]
    or [total_T, H, d_k] (natural-log gates); ``beta``: [total_T, H];
    ``state_in``: [n_seq, H, d_k, d_v] or None; ``cu_seqlens``: int [n_seq+1].
    Any leading dims are flattened into total_T.  Returns ``(o, state_out)``
    in fp64 (plus ``codes, scales`` of the last QDQ when ``want_codes``).
    """
    q, k, v, g, beta = (_f64(x) for x in (q, k, v, g, beta))
    d_k, d_v = q.shape[-1], v.shape[-1]
    H = v.shape[-2]
    q = q.reshape(-1, H, d_k)
    k = k.reshape(-1, H, d_k)
    v = v.reshape(-1, H, d_v)
    beta = beta.reshape(-1, H)
    g = g.reshape((-1, H, d_k) if per_key_gate else (-1, H))
    cu = np.ascontiguousarray(np.asarray(cu_seqlens), dtype=np.int32)
    n_seq = cu.size - 1
    st = _f64(state_in)
    if st is not None:
        st = st.reshape(n_seq, H, d_k, d_v)
    m, grp = qdq_mode_of(qdq)
    o = np.zeros((q.shape[0], H, d_v), dtype=np.float64)
    s_out = np.zeros((n_seq, H, d_k, d_v), dtype=np.float64)
    codes = scales = None
    if want_codes and m != QDQ_NONE:
        codes = np.zeros((n_seq, H, d_k, d_v), dtype=np.float32)
        nsc = d_v // 64 if m == QDQ_FP8_TILE else d_k * d_v // grp
        scales = np.zeros((n_seq, H, nsc), dtype=np.float32)
    rc = _load().or_gdn_recurrence(
        _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(st), _ptr(cu),
        n_seq, H, d_k, d_v, int(per_key_gate), m, grp, qdq_axis,
        boundary_every, _ptr(o), _ptr(s_out), _ptr(codes), _ptr(scales),
        n_threads)
    if rc != 0:
        raise ValueError("oracle recurrence: bad arguments")
    if want_codes:
        return o, s_out, codes, scales
    return o, s_out


def dense_cu_seqlens(n_seq: int, T: int) -> np.ndarray:
    return (np.arange(n_seq + 1, dtype=np.int64) * T).astype(np.int32)


def prefill(inp: dict, case, **kw):
    """Oracle prefix over a generated case (dense or packed)."""
    cu = inp["cu_seqlens"]
    if cu is None:
        cu = dense_cu_seqlens(case.n_seq, case.T)
    return recurrence(inp["q"], inp["k"], inp["v"], inp["g"], inp["beta"],
                      inp["state_in"], cu, per_key_gate=case.gate == "per_key",
                      qdq=case.qdq, boundary_every=CHUNK, **kw)


def decode(dq, dk, dv, dg, dbeta, state_in, *, per_key_gate: bool, qdq: str,
           **kw):
    """Oracle decode over ``S`` steps of one token per sequence.

    Inputs are ``[S, N, H, d]`` (``dg``: [S, N, H] or [S, N, H, d_k]); the
    state QDQ follows every token.  Returns ``o`` [S, N, H, d_v] and the
    final state [N, H, d_k, d_v].
    """
    dq, dk, dv, dg, dbeta = (_f64(x) for x in (dq, dk, dv, dg, dbeta))
    S, N, H = dq.shape[:3]
    perm = lambda a: np.ascontiguousarray(np.swapaxes(a, 0, 1)).reshape(
        (N * S,) + a.shape[2:])
    cu = dense_cu_seqlens(N, S)
    res = recurrence(perm(dq), perm(dk), perm(dv), perm(dg), perm(dbeta),
                     state_in, cu, per_key_gate=per_key_gate, qdq=qdq,
                     boundary_every=1, **kw)
    o = np.swapaxes(res[0].reshape(N, S, H, -1), 0, 1)
    return (o,) + tuple(res[1:])
