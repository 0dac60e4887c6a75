"""Host-only checks that both builds decide staleness by content.

A copy of the source tree to another machine need not keep modification
times (some keep whole seconds only), so a library must be rebuilt exactly
when its flags or sources differ from those it was built from, whatever the
files' times say.  Nothing is compiled here except a two-line C file.
"""

import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _build_module():
    spec = importlib.util.spec_from_file_location(
        "state_quantized_recurrence_b200_build_stamp",
        os.path.join(ROOT, "state_quantized_recurrence_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_cuda_library_stale_by_content(tmp_path, monkeypatch):
    b = _build_module()
    src = tmp_path / "kernel.cuh"
    src.write_text("// one\n")
    lib = tmp_path / "lib.so"
    lib.write_bytes(b"\0")
    monkeypatch.setattr(b, "_sources", lambda: [str(src)])
    monkeypatch.setattr(b, "ROOT", str(tmp_path))
    monkeypatch.setattr(b, "LIB", str(lib))
    monkeypatch.setattr(b, "STAMP", str(lib) + ".sha256")
    assert not b.up_to_date()  # no stamp yet
    (tmp_path / "lib.so.sha256").write_text(b.source_digest() + "\n")
    assert b.up_to_date()
    # a source newer than the library but unchanged: still up to date
    os.utime(src, (os.path.getmtime(lib) + 100,) * 2)
    assert b.up_to_date()
    # changed contents with the library's own modification time: stale
    t = os.path.getmtime(lib)
    src.write_text("// two\n")
    os.utime(src, (t - 100, t - 100))
    assert not b.up_to_date()
    # a changed flag is a change too
    (tmp_path / "lib.so.sha256").write_text(b.source_digest() + "\n")
    assert b.up_to_date()
    monkeypatch.setattr(b, "NVCC_FLAGS", b.NVCC_FLAGS + ["-DEXTRA"])
    assert not b.up_to_date()


def test_oracle_stale_by_content(tmp_path):
    import oracle
    src = tmp_path / "f.c"
    src.write_text("int f(void) { return 1; }\n")
    out = str(tmp_path / "libf.so")
    oracle.build(src=str(src), out=out)
    first = os.path.getmtime(out)
    stamp = open(out + ".sha256").read()
    # same contents, newer source time: no rebuild
    os.utime(src, (first + 100, first + 100))
    oracle.build(src=str(src), out=out)
    assert open(out + ".sha256").read() == stamp
    # new contents, older source time: rebuilt
    src.write_text("int f(void) { return 2; }\n")
    os.utime(src, (first - 100, first - 100))
    oracle.build(src=str(src), out=out)
    assert open(out + ".sha256").read() != stamp
    import ctypes
    assert ctypes.CDLL(out).f() == 2


if __name__ == "__main__":
    pytest.main([__file__, "-q"])
