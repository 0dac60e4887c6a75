"""B200 (sm_100a) gated delta rule with a fake-quantized recurrent state.

Thin Python binding over the C ABI in ``include/gdn_qdq.h``: it only checks
and marshals arguments (device pointers, sizes, the current CUDA stream);
every step of the computation runs in the library's CUDA kernels.  There is
no CPU or PyTorch fallback - importing this package fails if the compiled
library is missing.

    o, state = gdn_prefill(q, k, v, g, beta, state_in=None, cu_seqlens=None,
                           qdq="fp8_tile64")
    o = gdn_decode(q, k, v, g, beta, state, qdq="int8_g32")   # state in place
"""

from __future__ import annotations

from ._binding import (  # noqa: F401
    GDN_DTYPE, GDN_GATE, GDN_QDQ, GDN_STATUS, GdnError, check_last_error,
    gdn_decode, gdn_decode_into, gdn_last_error, gdn_prefill, gdn_prefill_into,
    lib, library_path,
)

__all__ = [
    "gdn_prefill", "gdn_prefill_into", "gdn_decode", "gdn_decode_into",
    "gdn_last_error", "check_last_error", "GdnError", "library_path", "lib",
    "GDN_QDQ", "GDN_DTYPE", "GDN_GATE", "GDN_STATUS",
]
