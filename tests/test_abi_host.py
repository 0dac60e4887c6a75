"""Host-only checks of the C ABI (no GPU needed, nothing is launched).

* the library loads and exports, unmangled, every function that
  include/*.h declares;
* argument errors are caught on the host with the documented status codes
  before any CUDA call (bad sizes, unsupported d_k / d_v / dtype / gate /
  codec, null or misaligned pointers);
* an empty batch (n_seq == 0) is a successful no-op.
"""

import ctypes
import glob
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIB = os.path.join(ROOT, "state_quantized_recurrence_b200", "libgdn_qdq.so")

OK, INVALID, UNSUPPORTED = 0, 1, 2
BF16, F32 = 0, 1


@pytest.fixture(scope="module")
def lib():
    import importlib.util  # the build script by path: the package import needs the library
    spec = importlib.util.spec_from_file_location(
        "state_quantized_recurrence_b200_build",
        os.path.join(ROOT, "state_quantized_recurrence_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    build.build()
    L = ctypes.CDLL(LIB)
    P, I = ctypes.c_void_p, ctypes.c_int
    L.gdn_prefill.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, P, P]
    L.gdn_prefill.restype = I
    L.gdn_prefill_neumann.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, P, P, P]
    L.gdn_prefill_neumann.restype = I
    L.gdn_prefill_w_qdq.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, P, P, P]
    L.gdn_prefill_w_qdq.restype = I
    L.gdn_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, I, P, P]
    L.gdn_decode.restype = I
    L.gdn_decode_packed.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P]
    L.gdn_decode_packed.restype = I
    for f in (L.gdn_state_pack, L.gdn_state_unpack):
        f.argtypes = [P, P, P, I, I, I, I, I, P]
        f.restype = I
    L.gdn_status_string.argtypes = [I]
    L.gdn_status_string.restype = ctypes.c_char_p
    return L


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w \*]*?\b(gdn_\w+)\s*\(", src, flags=re.M):
            names.add(m.group(1))
    return names


def test_header_symbols_exported(lib):
    names = declared_functions()
    assert {"gdn_prefill", "gdn_decode", "gdn_last_error", "gdn_status_string"} <= names
    out = subprocess.run(["nm", "-D", "--defined-only", LIB], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n), n


def test_status_strings(lib):
    assert lib.gdn_status_string(0) == b"GDN_OK"
    assert lib.gdn_status_string(4) == b"GDN_ERR_TIMEOUT"
    assert lib.gdn_status_string(99) == b"GDN_ERR_UNKNOWN"


A = 0x10000  # a 16-byte aligned stand-in address; never dereferenced


def pf(lib, **kw):
    a = dict(q=A, k=A, v=A, g=A, beta=A, state_in=None, cu=None, n_seq=2, T=64, H=4, d_k=128,
             d_v=128, dt=BF16, gk=0, qdq=1, o=A, state_out=A, stream=None)
    a.update(kw)
    return lib.gdn_prefill(a["q"], a["k"], a["v"], a["g"], a["beta"], a["state_in"], a["cu"],
                           a["n_seq"], a["T"], a["H"], a["d_k"], a["d_v"], a["dt"], a["gk"],
                           a["qdq"], a["o"], a["state_out"], a["stream"])


def pn(lib, degree=3, **kw):
    a = dict(q=A, k=A, v=A, g=A, beta=A, state_in=None, cu=None, n_seq=2, T=64, H=4, d_k=128,
             d_v=128, dt=BF16, gk=0, qdq=1, o=A, state_out=A, stream=None)
    a.update(kw)
    return lib.gdn_prefill_neumann(a["q"], a["k"], a["v"], a["g"], a["beta"], a["state_in"],
                                   a["cu"], a["n_seq"], a["T"], a["H"], a["d_k"], a["d_v"],
                                   a["dt"], a["gk"], a["qdq"], degree, a["o"], a["state_out"],
                                   a["stream"])


def pw(lib, w_qdq=1, **kw):
    a = dict(q=A, k=A, v=A, g=A, beta=A, state_in=None, cu=None, n_seq=2, T=64, H=4, d_k=128,
             d_v=128, dt=BF16, gk=0, qdq=1, o=A, state_out=A, stream=None)
    a.update(kw)
    return lib.gdn_prefill_w_qdq(a["q"], a["k"], a["v"], a["g"], a["beta"], a["state_in"],
                                 a["cu"], a["n_seq"], a["T"], a["H"], a["d_k"], a["d_v"],
                                 a["dt"], a["gk"], a["qdq"], w_qdq, a["o"], a["state_out"],
                                 a["stream"])


def dc(lib, **kw):
    a = dict(q=A, k=A, v=A, g=A, beta=A, state=A, n_seq=2, H=4, d_k=128, d_v=128, dt=BF16, gk=0,
             qdq=2, o=A, stream=None)
    a.update(kw)
    return lib.gdn_decode(a["q"], a["k"], a["v"], a["g"], a["beta"], a["state"], a["n_seq"],
                          a["H"], a["d_k"], a["d_v"], a["dt"], a["gk"], a["qdq"], a["o"],
                          a["stream"])


def dp(lib, **kw):
    a = dict(q=A, k=A, v=A, g=A, beta=A, codes=A, scales=A, n_seq=2, H=4, d_k=128, d_v=128,
             dt=BF16, gk=0, qdq=2, o=A, stream=None)
    a.update(kw)
    return lib.gdn_decode_packed(a["q"], a["k"], a["v"], a["g"], a["beta"], a["codes"],
                                 a["scales"], a["n_seq"], a["H"], a["d_k"], a["d_v"], a["dt"],
                                 a["gk"], a["qdq"], a["o"], a["stream"])


def cv(lib, unpack=False, **kw):
    a = dict(state=A, codes=A, scales=A, n=2, H=4, d_k=128, d_v=128, qdq=2, stream=None)
    a.update(kw)
    if unpack:
        return lib.gdn_state_unpack(a["codes"], a["scales"], a["state"], a["n"], a["H"],
                                    a["d_k"], a["d_v"], a["qdq"], a["stream"])
    return lib.gdn_state_pack(a["state"], a["codes"], a["scales"], a["n"], a["H"], a["d_k"],
                              a["d_v"], a["qdq"], a["stream"])


@pytest.mark.parametrize("call", [pf, pn, pw, dc, dp])
def test_validation_errors(lib, call):
    assert call(lib, n_seq=-1) == INVALID
    assert call(lib, H=0) == INVALID
    assert call(lib, d_k=96) == UNSUPPORTED
    assert call(lib, d_v=32) == UNSUPPORTED
    assert call(lib, d_k=256) == UNSUPPORTED
    assert call(lib, dt=7) == UNSUPPORTED
    assert call(lib, gk=3) == UNSUPPORTED
    assert call(lib, qdq=9) == UNSUPPORTED
    assert call(lib, q=None) == INVALID
    assert call(lib, beta=None) == INVALID
    assert call(lib, o=None) == INVALID
    assert call(lib, k=A + 8) == INVALID          # q/k/v/o need 16-byte alignment
    assert call(lib, g=A + 2) == INVALID          # g/beta need 4-byte alignment
    assert call(lib, n_seq=0) == OK               # empty batch: no work, no launch


def test_prefill_specific_errors(lib):
    assert pf(lib, T=-1) == INVALID
    assert pf(lib, state_out=None) == INVALID
    assert pf(lib, state_out=A + 4) == INVALID
    assert pf(lib, state_in=A + 4) == INVALID
    assert pf(lib, cu=A + 2) == INVALID


def test_w_qdq_unsupported_combinations(lib):
    """The FP8 QDQ of W runs on the WY-form pair only: bf16, scalar gates,
    d = 128, FP8 state tiles; anything else is refused before a launch (an
    unknown W codec too)."""
    assert pw(lib, w_qdq=2) == UNSUPPORTED
    assert pw(lib, dt=F32) == UNSUPPORTED
    assert pw(lib, gk=1) == UNSUPPORTED
    assert pw(lib, d_k=64, d_v=64) == UNSUPPORTED
    assert pw(lib, qdq=2) == UNSUPPORTED            # INT8 state
    assert pw(lib, qdq=0) == UNSUPPORTED            # no state QDQ
    assert pw(lib, n_seq=0) == OK
    assert pw(lib, w_qdq=0, n_seq=0) == OK


@pytest.mark.parametrize("degree", [-1, 0, 2, 4, 5, 30, 64, 127])
def test_neumann_degree_rejected(lib, degree):
    """Only 2^m - 1 for m = 1..6: any other degree is refused before a
    launch, never rounded to a supported one."""
    assert pn(lib, degree=degree) == INVALID
    assert pn(lib, degree=degree, n_seq=0) == INVALID


def bw(lib, ws_bytes=None, **kw):
    import ctypes as C
    lib.gdn_prefill_backward_workspace_bytes.argtypes = [C.c_int] * 6
    lib.gdn_prefill_backward_workspace_bytes.restype = C.c_size_t
    P, I = C.c_void_p, C.c_int
    lib.gdn_prefill_backward.argtypes = [P] * 7 + [I] * 8 + [P, P, P, C.c_size_t] + [P] * 7
    lib.gdn_prefill_backward.restype = I
    a = dict(q=A, k=A, v=A, g=A, beta=A, state_in=None, cu=None, n_seq=2, T=64, H=4, d_k=128,
             d_v=128, dt=BF16, gk=0, qdq=1, d_o=A, dso=None, ws=A, dq=A, dk=A, dv=A, dg=A,
             dbeta=A, dsi=A, stream=None)
    a.update(kw)
    need = lib.gdn_prefill_backward_workspace_bytes(a["n_seq"], a["T"], a["H"], a["d_k"],
                                                    a["d_v"], int(a["cu"] is not None))
    return lib.gdn_prefill_backward(
        a["q"], a["k"], a["v"], a["g"], a["beta"], a["state_in"], a["cu"], a["n_seq"], a["T"],
        a["H"], a["d_k"], a["d_v"], a["dt"], a["gk"], a["qdq"], a["d_o"], a["dso"], a["ws"],
        need if ws_bytes is None else ws_bytes, a["dq"], a["dk"], a["dv"], a["dg"], a["dbeta"],
        a["dsi"], a["stream"])


def test_backward_workspace_and_errors(lib):
    """Workspace size formula (chunk-start states per slot and value tile,
    plus one chunk of token states per CTA) and the checks made before any
    launch."""
    lib.gdn_prefill_backward_workspace_bytes.argtypes = [ctypes.c_int] * 6
    lib.gdn_prefill_backward_workspace_bytes.restype = ctypes.c_size_t
    tile = 128 * 64 * 4
    # dense: 2 sequences x ceil(100 / 64) = 4 slots, 4 heads, 2 tiles; 16 CTAs
    assert lib.gdn_prefill_backward_workspace_bytes(2, 100, 4, 128, 128, 0) == \
        tile * (4 * 4 * 2 + 16 * 64)
    # packed: n_seq + T / 64 slots
    assert lib.gdn_prefill_backward_workspace_bytes(3, 200, 1, 128, 64, 1) == \
        tile * ((3 + 3) * 1 * 1 + 3 * 64)
    assert lib.gdn_prefill_backward_workspace_bytes(2, 64, 4, 96, 128, 0) == 0
    assert bw(lib, ws_bytes=1) == INVALID            # workspace too small
    assert bw(lib, ws=None) == INVALID
    assert bw(lib, ws=A + 4) == INVALID              # 16-byte alignment
    assert bw(lib, dsi=None) == INVALID
    assert bw(lib, dq=None) == INVALID
    assert bw(lib, d_o=None) == INVALID
    assert bw(lib, d_k=96) == UNSUPPORTED
    assert bw(lib, n_seq=0) == OK


def test_backward_static_rejects_oversize(lib):
    """A problem whose workspace exceeds the 64 MiB static array is refused
    before the device is touched."""
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.gdn_prefill_backward_static.argtypes = [P] * 7 + [I] * 8 + [P, P] + [P] * 7
    lib.gdn_prefill_backward_static.restype = I
    lib.gdn_prefill_backward_workspace_bytes.argtypes = [I] * 6
    lib.gdn_prefill_backward_workspace_bytes.restype = ctypes.c_size_t
    assert lib.gdn_prefill_backward_workspace_bytes(4, 4096, 16, 128, 128, 0) > 64 << 20
    assert lib.gdn_prefill_backward_static(A, A, A, A, A, None, None, 4, 4096, 16, 128, 128, BF16,
                                           0, 1, A, None, A, A, A, A, A, A, None) == UNSUPPORTED


def test_decode_specific_errors(lib):
    assert dc(lib, state=None) == INVALID
    assert dc(lib, state=A + 4) == INVALID


def test_packed_state_errors(lib):
    assert dp(lib, qdq=0) == UNSUPPORTED          # packing needs a quantizing codec
    assert dp(lib, codes=None) == INVALID
    assert dp(lib, scales=None) == INVALID
    assert dp(lib, codes=A + 2) == INVALID        # codes and scales: 4-byte aligned
    assert dp(lib, scales=A + 1) == INVALID
    for unpack in (False, True):
        assert cv(lib, unpack, qdq=0) == UNSUPPORTED
        assert cv(lib, unpack, qdq=9) == UNSUPPORTED
        assert cv(lib, unpack, d_k=96) == UNSUPPORTED
        assert cv(lib, unpack, d_v=32) == UNSUPPORTED
        assert cv(lib, unpack, H=0) == INVALID
        assert cv(lib, unpack, n=-1) == INVALID
        assert cv(lib, unpack, state=None) == INVALID
        assert cv(lib, unpack, state=A + 4) == INVALID  # fp32 state: 16-byte aligned
        assert cv(lib, unpack, codes=A + 2) == INVALID
        assert cv(lib, unpack, scales=None) == INVALID
        assert cv(lib, unpack, n=0) == OK             # empty batch: no work, no launch


def test_binding_refuses_missing_library(tmp_path, monkeypatch):
    """The binding fails loudly (ImportError) when the CUDA library is absent."""
    import importlib
    import state_quantized_recurrence_b200._binding as b
    monkeypatch.setattr(b, "library_path", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        b._load()
    importlib.reload(b)


def test_prefill_schedule_host_cases(lib):
    """Shapes off the tensor-core path choose the CUDA-core kernel without
    touching a device; shapes gdn_prefill rejects give -1."""
    I = ctypes.c_int
    lib.gdn_prefill_schedule.argtypes = [I] * 7
    lib.gdn_prefill_schedule.restype = I
    assert lib.gdn_prefill_schedule(2, 4, 128, 128, 1, 0, 1) == 0   # fp32
    assert lib.gdn_prefill_schedule(2, 4, 128, 128, 0, 1, 2) == 0   # KDA gates
    assert lib.gdn_prefill_schedule(2, 4, 64, 64, 0, 0, 1) == 0     # d = 64
    assert lib.gdn_prefill_schedule(2, 4, 96, 128, 0, 0, 1) == -1
    assert lib.gdn_prefill_schedule(2, 0, 128, 128, 0, 0, 1) == -1
    assert lib.gdn_prefill_schedule(2, 4, 128, 128, 7, 0, 1) == -1
    assert lib.gdn_prefill_schedule(2, 4, 128, 128, 1, 0, 9) == -1   # no such codec
