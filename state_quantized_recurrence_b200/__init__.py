"""B200 (sm_100a) gated delta rule with a fake-quantized recurrent state.

Thin Python binding over the C ABI in ``include/gdn_qdq.h``: it only checks
and marshals arguments (device pointers, sizes, the current CUDA stream);
every step of the computation runs in the library's CUDA kernels.  There is
no CPU or PyTorch fallback - importing this package fails if the compiled
library is missing.

    o, state = gdn_prefill(q, k, v, g, beta, state_in=None, cu_seqlens=None,
                           qdq="fp8_tile64")
    o, state = gdn_prefill(..., neumann_degree=7)   # approximate solve, 2^m - 1
    o, state = gdn_prefill(..., w_qdq="fp8_row")    # + FP8 QDQ of W, a scale per row
    gdn_prefill_schedule(n_seq, H, d_k, d_v)        # which prefill kernel runs
    o = gdn_decode(q, k, v, g, beta, state, qdq="int8_g32")   # state in place
    dq, dk, dv, dg, dbeta, dstate_in = gdn_prefill_backward(q, k, v, g, beta, d_o, ...)

Packed state storage (codes + scales instead of fp32 QDQ values):

    ps = gdn_state_pack(state, qdq="int8_g32")
    o = gdn_decode_packed(q, k, v, g, beta, ps)                # ps in place
    state = gdn_state_unpack(ps)
"""

from __future__ import annotations

from ._binding import (  # noqa: F401
    GDN_DTYPE, GDN_GATE, GDN_QDQ, GDN_STATUS, GDN_W_QDQ, GdnError, check_last_error,
    PackedState, gdn_decode, gdn_decode_into, gdn_decode_packed, gdn_decode_packed_into,
    gdn_last_error, gdn_prefill, gdn_prefill_backward, gdn_prefill_backward_static,
    gdn_prefill_into, gdn_prefill_schedule,
    gdn_state_pack, gdn_state_unpack, lib, library_path, packed_state_empty,
)

__all__ = [
    "gdn_prefill", "gdn_prefill_into", "gdn_prefill_backward", "gdn_prefill_backward_static",
    "gdn_prefill_schedule",
    "gdn_decode", "gdn_decode_into",
    "gdn_decode_packed", "gdn_decode_packed_into", "gdn_state_pack", "gdn_state_unpack",
    "PackedState", "packed_state_empty",
    "gdn_last_error", "check_last_error", "GdnError", "library_path", "lib",
    "GDN_QDQ", "GDN_W_QDQ", "GDN_DTYPE", "GDN_GATE", "GDN_STATUS",
]
