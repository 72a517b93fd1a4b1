"""The C ABI library loads on a machine without a GPU, exports every symbol the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from gated_delta_rule_122_b200 import build as kbuild
from gated_delta_rule_122_b200 import kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

OK, ERR_NULL, ERR_SHAPE, ERR_DTYPE, ERR_ALIGN, ERR_UNSUP, ERR_WS, ERR_LAUNCH, ERR_TIMEOUT, ERR_ALIAS = range(10)


@pytest.fixture(scope="module")
def lib():
    kbuild.build()
    return kda.library()


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert sorted(kda.EXPORTED_SYMBOLS) == _declared_functions()


def test_library_exports_every_declared_symbol(lib):
    for name in _declared_functions():
        assert hasattr(lib, name), name
    raw = ctypes.CDLL(kda.library_path())
    for name in _declared_functions():
        getattr(raw, name)


def test_status_strings(lib):
    assert kda.status_string(OK) == "ok"
    for code in range(1, 10):
        assert kda.status_string(code) not in ("ok", "unknown status")
    assert kda.version() >= 100


def _fwd(lib, q=0x10000, k=0x20000, v=0x30000, a=0x40000, b=0x50000, s0=None, o=0x60000,
         s1=None, B=1, T=4, H=1, dk=16, dv=16, qkv=0, gate=0, out=0, ws=0x90000, wsb=16):
    return lib.kda_forward(q, k, v, a, b, s0, o, s1, B, T, H, dk, dv, 1.0, qkv, gate, out, ws, wsb,
                           None)


def test_forward_rejects_bad_arguments_before_launch(lib):
    assert _fwd(lib, q=None) == ERR_NULL
    assert _fwd(lib, T=-1) == ERR_SHAPE
    assert _fwd(lib, dk=48) == ERR_UNSUP
    assert _fwd(lib, dv=256) == ERR_UNSUP
    assert _fwd(lib, qkv=7) == ERR_DTYPE
    assert _fwd(lib, k=0x20008) == ERR_ALIGN
    assert _fwd(lib, o=0x10000 + 64) == ERR_ALIAS          # o overlaps q
    assert _fwd(lib, B=0) == OK                             # nothing to do, nothing launched
    assert _fwd(lib, H=0, ws=None) == OK
    assert _fwd(lib, ws=None) == ERR_WS
    assert _fwd(lib, wsb=8) == ERR_WS
    assert _fwd(lib, ws=0x90008) == ERR_ALIGN


def test_sequential_and_decode_reject_bad_arguments(lib):
    f = lib.kda_forward_sequential
    assert f(None, 1, 1, 1, 1, None, 1, None, 1, 4, 1, 16, 16, 1.0, 0, 0, 0, None) == ERR_NULL
    assert f(16, 32, 48, 64, 80, None, 96, None, 1, 4, 1, 20, 16, 1.0, 0, 0, 0, None) == ERR_UNSUP
    d = lib.kda_decode_step
    assert d(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, None, 0x60000, 2, 2, 16, 16, 1.0,
             0, 0, 0, None) == ERR_NULL
    assert d(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x70000, 0x70000 + 16, 2, 2, 16, 16, 1.0,
             0, 0, 0, None) == ERR_ALIAS                    # o inside the state
    assert d(0x10000, 0x20000, 0x30000, 0x40000, 0x50002, 0x70000, 0x60000, 2, 2, 16, 16, 1.0,
             0, 0, 0, None) == ERR_ALIGN                    # fp32 beta, 2-byte offset
    assert d(0x10000, 0x20000, 0x30000, 0x40008, 0x50004, 0x70000, 0x60000, 2, 2, 16, 16, 1.0,
             0, 0, 0, None) == ERR_ALIGN                    # alpha rows need 16 bytes


def test_workspace_query(lib):
    assert lib.kda_forward_workspace_bytes(2, 8192, 64, 128, 128) == 16
    assert lib.kda_workspace_status(None, None) == ERR_NULL
    assert lib.kda_workspace_status(0x90004, None) == ERR_ALIGN


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(kda, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(kda, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        kda.library()
