"""ctypes binding of ``libgdn_qdq.so`` (argument marshalling only)."""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libgdn_qdq.so")

GDN_STATUS = {0: "GDN_OK", 1: "GDN_ERR_INVALID_ARG", 2: "GDN_ERR_UNSUPPORTED",
              3: "GDN_ERR_CUDA", 4: "GDN_ERR_TIMEOUT"}
GDN_QDQ = {"none": 0, "fp8_tile64": 1, "int8_g32": 2, "int8_g16": 3, "int8_g64": 4}
GDN_W_QDQ = {"none": 0, "fp8_row": 1}
GDN_DTYPE = {torch.bfloat16: 0, torch.float32: 1}
GDN_GATE = {"scalar": 0, "per_key": 1}


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {GDN_STATUS.get(self.status, self.status)}")


def _load() -> ctypes.CDLL:
    if not os.path.exists(library_path):
        raise ImportError(
            f"CUDA library {library_path} is missing; build it with "
            "`python state_quantized_recurrence_b200/build.py` (there is no fallback)")
    L = ctypes.CDLL(library_path)
    P, I = ctypes.c_void_p, ctypes.c_int
    L.gdn_prefill.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, P, P]
    L.gdn_prefill.restype = I
    L.gdn_prefill_neumann.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, P, P, P]
    L.gdn_prefill_neumann.restype = I
    L.gdn_prefill_w_qdq.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, P, P, P]
    L.gdn_prefill_w_qdq.restype = I
    L.gdn_prefill_backward_workspace_bytes.argtypes = [I, I, I, I, I, I]
    L.gdn_prefill_backward_workspace_bytes.restype = ctypes.c_size_t
    L.gdn_prefill_backward.argtypes = ([P] * 7 + [I] * 8 + [P, P, P, ctypes.c_size_t]
                                       + [P] * 6 + [P])
    L.gdn_prefill_backward.restype = I
    L.gdn_prefill_backward_static.argtypes = [P] * 7 + [I] * 8 + [P, P] + [P] * 6 + [P]
    L.gdn_prefill_backward_static.restype = I
    L.gdn_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, P, P]
    L.gdn_decode.restype = I
    L.gdn_decode_packed.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P]
    L.gdn_decode_packed.restype = I
    L.gdn_state_pack.argtypes = [P, P, P, I, I, I, I, I, P]
    L.gdn_state_pack.restype = I
    L.gdn_state_unpack.argtypes = [P, P, P, I, I, I, I, I, P]
    L.gdn_state_unpack.restype = I
    L.gdn_last_error.argtypes = [P]
    L.gdn_last_error.restype = I
    L.gdn_status_string.argtypes = [I]
    L.gdn_status_string.restype = ctypes.c_char_p
    L.gdn_version.argtypes = []
    L.gdn_version.restype = I
    L.gdn_prefill_schedule.argtypes = [I, I, I, I, I, I, I]
    L.gdn_prefill_schedule.restype = I
    return L


lib = _load()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device=None) -> ctypes.c_void_p:
    """The given stream, else the current stream of ``device`` (default: the
    current device)."""
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _need(cond: bool, msg: str):
    if not cond:
        raise ValueError(msg)


def _check_dev(*ts) -> torch.device:
    """Every tensor a contiguous CUDA tensor on one device; returns it.  The
    library launches on the current device, so each call below makes this
    device current around the C call (and takes its current stream)."""
    dev = None
    for t in ts:
        if t is not None:
            _need(t.is_cuda and t.is_contiguous(), "tensors must be contiguous CUDA tensors")
            if dev is None:
                dev = t.device
            _need(t.device == dev, f"tensors on different devices ({dev} and {t.device})")
    return dev


GDN_PREFILL_KERNEL = {0: "cuda_cores", 1: "tc_one_cta", 2: "tc_cta_pair", 3: "tc_wy_pair"}


def gdn_prefill_schedule(n_seq: int, H: int, d_k: int, d_v: int, dtype=torch.bfloat16,
                         gate: str = "scalar", qdq: str = "fp8_tile64") -> str:
    """Which prefill kernel gdn_prefill launches for these shapes and this
    codec on the current device: "cuda_cores", "tc_one_cta", "tc_cta_pair"
    or "tc_wy_pair"."""
    _need(dtype in GDN_DTYPE and gate in GDN_GATE and qdq in GDN_QDQ,
          "unsupported dtype, gate kind or codec")
    r = int(lib.gdn_prefill_schedule(int(n_seq), int(H), int(d_k), int(d_v), GDN_DTYPE[dtype],
                                     GDN_GATE[gate], GDN_QDQ[qdq]))
    _need(r >= 0, "shapes gdn_prefill does not support")
    return GDN_PREFILL_KERNEL[r]


def gdn_last_error(stream=None, device=None) -> int:
    """Synchronize the stream (default: the current stream of ``device``, or
    of the current device) and return (and clear) that device's error
    status."""
    if device is None:
        device = stream.device if stream is not None else torch.cuda.current_device()
    with torch.cuda.device(device):
        return int(lib.gdn_last_error(_stream(stream, device)))


def check_last_error(stream=None, where: str = "gdn", device=None) -> None:
    s = gdn_last_error(stream, device)
    if s != 0:
        raise GdnError(s, where)


def _gate_kind(g: torch.Tensor, lead: int) -> str:
    return "per_key" if g.dim() == lead + 1 else "scalar"


def gdn_prefill_into(q, k, v, g, beta, state_in, cu_seqlens, o, state_out,
                     qdq: str = "fp8_tile64", stream=None,
                     neumann_degree: Optional[int] = None, w_qdq: str = "none") -> None:
    """Chunked prefix writing into preallocated ``o`` and ``state_out``.

    Dense: q, k [B, T, H, d_k], v/o [B, T, H, d_v]; packed (cu_seqlens int32
    [n_seq + 1]): [1, T_total, H, d].  g: fp32 [.., H] or [.., H, d_k];
    beta fp32 [.., H]; states fp32 [n_seq, H, d_k, d_v].  ``neumann_degree``
    (1, 3, 7, 15, 31 or 63) selects the approximate solve
    (gdn_prefill_neumann); None the exact one.  ``w_qdq="fp8_row"`` adds the
    FP8 QDQ of the WY-transformed W, one scale per row (gdn_prefill_w_qdq).
    """
    _need(w_qdq in GDN_W_QDQ, "w_qdq must be 'none' or 'fp8_row'")
    _need(w_qdq == "none" or neumann_degree is None,
          "the W codec is not offered with the Neumann solve")
    dev = _check_dev(q, k, v, g, beta, state_in, cu_seqlens, o, state_out)
    _need(q.dim() == 4 and k.shape == q.shape and v.dim() == 4, "q, k, v must be [B, T, H, d]")
    B, T, H, d_k = q.shape
    d_v = v.shape[-1]
    _need(v.shape[:3] == q.shape[:3] and o.shape == v.shape, "v/o shapes do not match q")
    _need(q.dtype in GDN_DTYPE and k.dtype == q.dtype and v.dtype == q.dtype and o.dtype == q.dtype,
          "q, k, v, o must share dtype bf16 or fp32")
    _need(g.dtype == torch.float32 and beta.dtype == torch.float32, "g and beta must be fp32")
    _need(beta.shape == q.shape[:3], "beta must be [B, T, H]")
    gk = _gate_kind(g, 3)
    _need(g.shape == (q.shape[:3] if gk == "scalar" else q.shape), "g must be [B,T,H] or [B,T,H,d_k]")
    if cu_seqlens is not None:
        _need(B == 1 and cu_seqlens.dtype == torch.int32 and cu_seqlens.dim() == 1,
              "packed layout needs B == 1 and int32 cu_seqlens")
        n_seq, T_arg = cu_seqlens.numel() - 1, T
    else:
        n_seq, T_arg = B, T
    _need(state_out.shape == (n_seq, H, d_k, d_v) and state_out.dtype == torch.float32,
          "state_out must be fp32 [n_seq, H, d_k, d_v]")
    if state_in is not None:
        _need(state_in.shape == state_out.shape and state_in.dtype == torch.float32,
              "state_in must be fp32 [n_seq, H, d_k, d_v]")
    args = (_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in), _ptr(cu_seqlens),
            n_seq, T_arg, H, d_k, d_v, GDN_DTYPE[q.dtype], GDN_GATE[gk], GDN_QDQ[qdq])
    with torch.cuda.device(dev):
        tail = (_ptr(o), _ptr(state_out), _stream(stream, dev))
        if w_qdq != "none":
            s, where = lib.gdn_prefill_w_qdq(*args, GDN_W_QDQ[w_qdq], *tail), "gdn_prefill_w_qdq"
        elif neumann_degree is None:
            s, where = lib.gdn_prefill(*args, *tail), "gdn_prefill"
        else:
            s, where = (lib.gdn_prefill_neumann(*args, int(neumann_degree), *tail),
                        "gdn_prefill_neumann")
    if s != 0:
        raise GdnError(s, where)


def gdn_prefill_backward(q, k, v, g, beta, d_o, state_in=None, cu_seqlens=None,
                         dstate_out=None, qdq: str = "fp8_tile64", workspace=None,
                         stream=None):
    """Gradients of ``gdn_prefill(q, k, v, g, beta, state_in, cu_seqlens, qdq)``
    for the upstream gradients ``d_o`` (o's shape and dtype) and
    ``dstate_out`` (fp32, or None), with the state QDQ passed straight
    through.  Returns fp32 ``(dq, dk, dv, dg, dbeta, dstate_in)``.
    ``workspace``: a CUDA uint8 tensor of at least
    gdn_prefill_backward_workspace_bytes(...) bytes, or None to allocate one."""
    dev = _check_dev(q, k, v, g, beta, d_o, state_in, cu_seqlens, dstate_out, workspace)
    _need(q.dim() == 4 and k.shape == q.shape and v.dim() == 4, "q, k, v must be [B, T, H, d]")
    B, T, H, d_k = q.shape
    d_v = v.shape[-1]
    _need(q.dtype in GDN_DTYPE and k.dtype == q.dtype and v.dtype == q.dtype
          and d_o.dtype == q.dtype and d_o.shape == v.shape, "d_o must be shaped like o, q's dtype")
    _need(g.dtype == torch.float32 and beta.dtype == torch.float32 and beta.shape == q.shape[:3],
          "g, beta must be fp32; beta [B, T, H]")
    gk = _gate_kind(g, 3)
    _need(g.shape == (q.shape[:3] if gk == "scalar" else q.shape), "g must be [B,T,H] or [B,T,H,d_k]")
    if cu_seqlens is not None:
        _need(B == 1 and cu_seqlens.dtype == torch.int32 and cu_seqlens.dim() == 1,
              "packed layout needs B == 1 and int32 cu_seqlens")
        n_seq, T_arg = cu_seqlens.numel() - 1, T
    else:
        n_seq, T_arg = B, T
    sshape = (n_seq, H, d_k, d_v)
    for t in (state_in, dstate_out):
        _need(t is None or (t.shape == sshape and t.dtype == torch.float32),
              "states must be fp32 [n_seq, H, d_k, d_v]")
    need = int(lib.gdn_prefill_backward_workspace_bytes(n_seq, T_arg, H, d_k, d_v,
                                                        int(cu_seqlens is not None)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    f32 = dict(dtype=torch.float32, device=q.device)
    dq, dk = torch.empty(q.shape, **f32), torch.empty(q.shape, **f32)
    dv = torch.empty(v.shape, **f32)
    dg, dbeta = torch.empty(g.shape, **f32), torch.empty(beta.shape, **f32)
    dstate_in = torch.empty(sshape, **f32)
    with torch.cuda.device(dev):
        s = lib.gdn_prefill_backward(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in), _ptr(cu_seqlens), n_seq,
            T_arg, H, d_k, d_v, GDN_DTYPE[q.dtype], GDN_GATE[gk], GDN_QDQ[qdq], _ptr(d_o),
            _ptr(dstate_out), _ptr(workspace), workspace.numel(), _ptr(dq), _ptr(dk), _ptr(dv),
            _ptr(dg), _ptr(dbeta), _ptr(dstate_in), _stream(stream, dev))
    if s != 0:
        raise GdnError(s, "gdn_prefill_backward")
    return dq, dk, dv, dg, dbeta, dstate_in


def gdn_prefill_backward_static(q, k, v, g, beta, d_o, state_in=None, cu_seqlens=None,
                                dstate_out=None, qdq: str = "fp8_tile64", stream=None):
    """gdn_prefill_backward with the workspace taken from the library's
    static device array (64 MiB; larger problems raise GDN_ERR_UNSUPPORTED).
    Calls that overlap on one device share that array: order them.  Returns
    fp32 ``(dq, dk, dv, dg, dbeta, dstate_in)`` (allocated here with torch)."""
    dev = _check_dev(q, k, v, g, beta, d_o, state_in, cu_seqlens, dstate_out)
    _need(q.dim() == 4 and k.shape == q.shape and v.dim() == 4, "q, k, v must be [B, T, H, d]")
    B, T, H, d_k = q.shape
    d_v = v.shape[-1]
    _need(q.dtype in GDN_DTYPE and k.dtype == q.dtype and v.dtype == q.dtype
          and d_o.dtype == q.dtype and d_o.shape == v.shape, "d_o must be shaped like o, q's dtype")
    _need(g.dtype == torch.float32 and beta.dtype == torch.float32 and beta.shape == q.shape[:3],
          "g, beta must be fp32; beta [B, T, H]")
    gk = _gate_kind(g, 3)
    _need(g.shape == (q.shape[:3] if gk == "scalar" else q.shape), "g must be [B,T,H] or [B,T,H,d_k]")
    if cu_seqlens is not None:
        _need(B == 1 and cu_seqlens.dtype == torch.int32 and cu_seqlens.dim() == 1,
              "packed layout needs B == 1 and int32 cu_seqlens")
        n_seq, T_arg = cu_seqlens.numel() - 1, T
    else:
        n_seq, T_arg = B, T
    sshape = (n_seq, H, d_k, d_v)
    for t in (state_in, dstate_out):
        _need(t is None or (t.shape == sshape and t.dtype == torch.float32),
              "states must be fp32 [n_seq, H, d_k, d_v]")
    f32 = dict(dtype=torch.float32, device=q.device)
    dq, dk = torch.empty(q.shape, **f32), torch.empty(q.shape, **f32)
    dv = torch.empty(v.shape, **f32)
    dg, dbeta = torch.empty(g.shape, **f32), torch.empty(beta.shape, **f32)
    dstate_in = torch.empty(sshape, **f32)
    with torch.cuda.device(dev):
        s = lib.gdn_prefill_backward_static(
            _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state_in), _ptr(cu_seqlens), n_seq,
            T_arg, H, d_k, d_v, GDN_DTYPE[q.dtype], GDN_GATE[gk], GDN_QDQ[qdq], _ptr(d_o),
            _ptr(dstate_out), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dbeta), _ptr(dstate_in),
            _stream(stream, dev))
    if s != 0:
        raise GdnError(s, "gdn_prefill_backward_static")
    return dq, dk, dv, dg, dbeta, dstate_in


def gdn_prefill(q, k, v, g, beta, state_in=None, cu_seqlens=None, qdq: str = "fp8_tile64",
                stream=None, neumann_degree: Optional[int] = None, w_qdq: str = "none"):
    """Chunked prefix; returns ``(o, state_out)`` (allocated with torch).
    ``neumann_degree`` (1, 3, 7, 15, 31 or 63) replaces the exact triangular
    solve of every chunk by the truncated Neumann series of that degree
    (``gdn_prefill_neumann``); None keeps the exact solve (``gdn_prefill``)."""
    n_seq = q.shape[0] if cu_seqlens is None else cu_seqlens.numel() - 1
    o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    state_out = torch.empty((n_seq, q.shape[2], q.shape[3], v.shape[3]), dtype=torch.float32,
                            device=q.device)
    gdn_prefill_into(q, k, v, g, beta, state_in, cu_seqlens, o, state_out, qdq, stream,
                     neumann_degree, w_qdq)
    return o, state_out


def gdn_decode_into(q, k, v, g, beta, state, o, qdq: str = "int8_g32", stream=None) -> None:
    """One decode token per sequence: q, k [N, H, d_k], v/o [N, H, d_v],
    g [N, H] or [N, H, d_k], beta [N, H]; ``state`` [N, H, d_k, d_v] fp32 is
    advanced and QDQ'd in place."""
    dev = _check_dev(q, k, v, g, beta, state, o)
    _need(q.dim() == 3 and k.shape == q.shape and v.dim() == 3 and o.shape == v.shape,
          "q, k [N, H, d_k]; v, o [N, H, d_v]")
    N, H, d_k = q.shape
    d_v = v.shape[-1]
    _need(q.dtype in GDN_DTYPE and k.dtype == q.dtype and v.dtype == q.dtype and o.dtype == q.dtype,
          "q, k, v, o must share dtype bf16 or fp32")
    _need(g.dtype == torch.float32 and beta.dtype == torch.float32 and beta.shape == (N, H),
          "g, beta must be fp32; beta [N, H]")
    gk = _gate_kind(g, 2)
    _need(g.shape == ((N, H) if gk == "scalar" else (N, H, d_k)), "g must be [N,H] or [N,H,d_k]")
    _need(state.shape == (N, H, d_k, d_v) and state.dtype == torch.float32,
          "state must be fp32 [N, H, d_k, d_v]")
    with torch.cuda.device(dev):
        s = lib.gdn_decode(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(state), N, H, d_k,
                           d_v, GDN_DTYPE[q.dtype], GDN_GATE[gk], GDN_QDQ[qdq], _ptr(o),
                           _stream(stream, dev))
    if s != 0:
        raise GdnError(s, "gdn_decode")


def gdn_decode(q, k, v, g, beta, state, qdq: str = "int8_g32", stream=None):
    o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    gdn_decode_into(q, k, v, g, beta, state, o, qdq, stream)
    return o


# ------------------------------------------------------------ packed states
class PackedState:
    """A batch of QDQ states stored as codes + scales (see gdn_qdq.h):
    ``codes`` uint8 [N, H, d_k, d_v] (int8 codes or E4M3 bytes), ``scales``
    fp32 [N, H, d_k, d_v / G] (INT8 group G) or [N, H, d_v / 64] (FP8 tile)."""

    def __init__(self, codes: torch.Tensor, scales: torch.Tensor, qdq: str):
        self.codes, self.scales, self.qdq = codes, scales, qdq

    @property
    def shape(self):
        return tuple(self.codes.shape)


def _scales_shape(N, H, d_k, d_v, qdq: str):
    _need(qdq in GDN_QDQ and qdq != "none", "packed states need an FP8 or INT8 qdq mode")
    if qdq == "fp8_tile64":
        return (N, H, d_v // 64)
    return (N, H, d_k, d_v // int(qdq.split("_g")[1]))


def packed_state_empty(N, H, d_k, d_v, qdq: str, device) -> PackedState:
    return PackedState(torch.empty((N, H, d_k, d_v), dtype=torch.uint8, device=device),
                       torch.empty(_scales_shape(N, H, d_k, d_v, qdq), dtype=torch.float32,
                                   device=device), qdq)


def gdn_state_pack(state: torch.Tensor, qdq: str, out: Optional[PackedState] = None,
                   stream=None) -> PackedState:
    """Codes and scales of QDQ(state) for fp32 ``state`` [N, H, d_k, d_v]."""
    _need(state.dim() == 4 and state.dtype == torch.float32, "state must be fp32 [N, H, d_k, d_v]")
    N, H, d_k, d_v = state.shape
    ps = out if out is not None else packed_state_empty(N, H, d_k, d_v, qdq, state.device)
    dev = _check_dev(state, ps.codes, ps.scales)
    _need(ps.shape == tuple(state.shape) and ps.qdq == qdq, "packed state shape / mode mismatch")
    with torch.cuda.device(dev):
        s = lib.gdn_state_pack(_ptr(state), _ptr(ps.codes), _ptr(ps.scales), N, H, d_k, d_v,
                               GDN_QDQ[qdq], _stream(stream, dev))
    if s != 0:
        raise GdnError(s, "gdn_state_pack")
    return ps


def gdn_state_unpack(ps: PackedState, out: Optional[torch.Tensor] = None, stream=None):
    """fp32 [N, H, d_k, d_v] = code * scale."""
    N, H, d_k, d_v = ps.shape
    st = out if out is not None else torch.empty((N, H, d_k, d_v), dtype=torch.float32,
                                                 device=ps.codes.device)
    dev = _check_dev(st, ps.codes, ps.scales)
    with torch.cuda.device(dev):
        s = lib.gdn_state_unpack(_ptr(ps.codes), _ptr(ps.scales), _ptr(st), N, H, d_k, d_v,
                                 GDN_QDQ[ps.qdq], _stream(stream, dev))
    if s != 0:
        raise GdnError(s, "gdn_state_unpack")
    return st


def gdn_decode_packed_into(q, k, v, g, beta, ps: PackedState, o, stream=None) -> None:
    """gdn_decode_into with the state stored packed (updated in place)."""
    dev = _check_dev(q, k, v, g, beta, ps.codes, ps.scales, o)
    _need(q.dim() == 3 and k.shape == q.shape and v.dim() == 3 and o.shape == v.shape,
          "q, k [N, H, d_k]; v, o [N, H, d_v]")
    N, H, d_k = q.shape
    d_v = v.shape[-1]
    _need(q.dtype in GDN_DTYPE and k.dtype == q.dtype and v.dtype == q.dtype and o.dtype == q.dtype,
          "q, k, v, o must share dtype bf16 or fp32")
    _need(g.dtype == torch.float32 and beta.dtype == torch.float32 and beta.shape == (N, H),
          "g, beta must be fp32; beta [N, H]")
    gk = _gate_kind(g, 2)
    _need(g.shape == ((N, H) if gk == "scalar" else (N, H, d_k)), "g must be [N,H] or [N,H,d_k]")
    _need(ps.shape == (N, H, d_k, d_v) and ps.codes.dtype == torch.uint8 and
          tuple(ps.scales.shape) == _scales_shape(N, H, d_k, d_v, ps.qdq),
          "packed state does not match the call")
    with torch.cuda.device(dev):
        s = lib.gdn_decode_packed(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(ps.codes),
                                  _ptr(ps.scales), N, H, d_k, d_v, GDN_DTYPE[q.dtype], GDN_GATE[gk],
                                  GDN_QDQ[ps.qdq], _ptr(o), _stream(stream, dev))
    if s != 0:
        raise GdnError(s, "gdn_decode_packed")


def gdn_decode_packed(q, k, v, g, beta, ps: PackedState, stream=None):
    o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    gdn_decode_packed_into(q, k, v, g, beta, ps, o, stream)
    return o
