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
    for code in range(1, 11):
        assert kda.status_string(code) not in ("ok", "unknown status")
    assert kda.version() >= 100


def _fwd(lib, q=0x10000, k=0x20000, v=0x30000, a=0x40000, b=0x50000, s0=None, o=0x60000,
         s1=None, B=1, T=4, H=1, dk=16, dv=16, qkv=0, gate=0, out=0, ws=0x90000, wsb=16):
    return lib.kda_forward(q, k, v, a, b, s0, o, s1, B, T, H, dk, dv, 1.0, qkv, gate, out, ws, wsb,
                           None)


def test_forward_rejects_bad_arguments_before_launch(lib):
    assert _fwd(lib, q=None) == ERR_NULL
    assert _fwd(lib, T=-1) == ERR_SHAPE
    assert _fwd(lib, dk=40) == ERR_UNSUP                   # not a multiple of 16
    assert _fwd(lib, dk=144) == ERR_UNSUP                  # above 128
    assert _fwd(lib, dv=256) == ERR_UNSUP
    assert _fwd(lib, qkv=7) == ERR_DTYPE
    assert _fwd(lib, k=0x20008) == ERR_ALIGN
    assert _fwd(lib, o=0x10000 + 64) == ERR_ALIAS          # o overlaps q
    assert _fwd(lib, B=0) == OK                             # nothing to do, nothing launched
    assert _fwd(lib, H=0, ws=None) == OK
    assert _fwd(lib, ws=None) == ERR_WS
    assert _fwd(lib, wsb=8) == ERR_WS
    assert _fwd(lib, ws=0x90008) == ERR_ALIGN


@pytest.mark.parametrize("d", [16, 32, 48, 64, 80, 96, 112, 128])
def test_every_multiple_of_16_head_size_is_accepted(lib, d):
    # B = 0: the checks run, nothing is launched
    assert _fwd(lib, dk=d, dv=d, B=0) == OK
    assert _fwd(lib, dk=d, dv=16, B=0) == OK and _fwd(lib, dk=16, dv=d, B=0) == OK
    assert lib.kda_forward_sequential(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, None, 0x60000, None,
                                      0, 4, 1, d, d, 1.0, 0, 0, 0, None) == OK
    assert lib.kda_decode_step(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x70000, 0x60000, 0, 2, d, d, 1.0,
                               0, 0, 0, None) == OK


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


# ---- the further entry points: host-side rejections (nothing reaches the device) ----------

def test_gdn2_rejects_bad_arguments(lib):
    def g(q=0x10000, e=0x70000, w=0x80000, o=0x60000, dk=16, ws=0x90000):
        return lib.kda_forward_gdn2(q, 0x20000, 0x30000, 0x40000, e, w, None, o, None, 1, 4, 1, dk, 16, 1.0,
                                    0, 0, 0, ws, 16, None)
    assert g(q=None) == ERR_NULL
    assert g(w=None) == ERR_NULL
    assert g(e=0x70004) == ERR_ALIGN
    assert g(o=0x80000 + 64) == ERR_ALIAS                   # o overlaps the write gate
    assert g(dk=40) == ERR_UNSUP
    assert g(ws=None) == ERR_WS
    d = lib.kda_decode_step_gdn2
    assert d(0x10000, 0x20000, 0x30000, 0x40000, 0x70000, None, 0xA0000, 0x60000, 2, 1, 16, 16, 1.0,
             0, 0, 0, None) == ERR_NULL


def test_raw_and_scalar_gate_reject_bad_arguments(lib):
    r = lib.kda_forward_raw
    assert r(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, None, 0x60000, None, 1, 4, 1, 56, 16, 1.0,
             0, 0, 0, 0x90000, 16, None) == ERR_UNSUP
    assert r(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, None, 0x60000, None, 1, 4, 1, 16, 16, 1.0,
             0, 0, 0, None, 0, None) == ERR_WS
    s = lib.kda_forward_scalar_gate
    # a per-head gate needs only its element alignment: fp32 at a 2-byte offset is rejected
    assert s(0x10000, 0x20000, 0x30000, 0x40002, 0x50000, None, 0x60000, None, 1, 4, 1, 16, 16, 1.0,
             0, 0, 0, 0x90000, 16, None) == ERR_ALIGN
    assert lib.kda_decode_step_raw(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, None, 0x60000, 2, 1, 16, 16,
                                   1.0, 0, 0, 0, None) == ERR_NULL


def test_varlen_rejects_bad_arguments(lib):
    def v(N=2, cu=0xB0000, T=8, dk=16):
        return lib.kda_forward_varlen(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, cu, None, 0x60000, None,
                                      N, T, 1, dk, 16, 1.0, 0, 0, 0, 0x90000, 16, None)
    assert v(N=-1) == ERR_SHAPE
    assert v(cu=None) == ERR_NULL
    assert v(cu=0xB0002) == ERR_ALIGN
    assert v(dk=40) == ERR_UNSUP


def test_decode_tokens_rejects_bad_arguments(lib):
    def d(state=0xA0000, slots=None, num_slots=4, o=0x60000, N=2, T=3, status=None, dk=16):
        return lib.kda_decode_tokens(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, state, slots, num_slots, 1,
                                     None, o, N, T, 1, dk, 16, 1.0, 0, 0, 0, status, None)
    assert d(num_slots=1) == ERR_SHAPE                      # identity slots need num_slots >= N
    assert d(num_slots=-1, slots=0xC0000) == ERR_SHAPE
    assert d(state=0xA0004) == ERR_ALIGN
    assert d(slots=0xC0002) == ERR_ALIGN
    assert d(status=0x90004) == ERR_ALIGN
    assert d(state=None) == ERR_NULL
    assert d(o=0xA0000 + 256) == ERR_ALIAS                  # o inside the state pool
    assert d(dk=40) == ERR_UNSUP
    assert d(N=0) == OK                                     # nothing to do, nothing launched


def test_state_copy_rejects_bad_arguments(lib):
    def c(src=0x10000, si=None, ss=4, dst=0x80000, di=None, ds=4, count=2, H=1, dk=16, status=None):
        return lib.kda_state_copy(src, si, ss, dst, di, ds, count, H, dk, 16, status, None)
    assert c(count=-1) == ERR_SHAPE
    assert c(dk=40) == ERR_UNSUP
    assert c(count=5) == ERR_SHAPE                          # identity index past the source pool
    assert c(count=5, si=0xC0000, ds=4) == ERR_SHAPE        # identity index past the destination pool
    assert c(src=0x10008) == ERR_ALIGN
    assert c(si=0xC0002) == ERR_ALIGN
    assert c(src=None) == ERR_NULL
    assert c(count=0) == OK and c(H=0) == OK                # nothing to copy, nothing launched


def test_selftest_rejects_bad_arguments(lib):
    assert lib.kda_selftest_bounded_wait(0, 1000, None, None) == ERR_NULL
    assert lib.kda_selftest_bounded_wait(0, 1000, 0x90004, None) == ERR_ALIGN
    assert lib.kda_selftest_bounded_wait(0, 0, 0x90000, None) == ERR_SHAPE
    assert lib.kda_selftest_bounded_wait(0, 2000001, 0x90000, None) == ERR_SHAPE


def test_host_path_rejects_bad_arguments(lib):
    def f(kind=0, q=0x10000, dk=16, B=1, T=4, ws=0x100000, wsb=1 << 20):
        return lib.kda_forward_host(kind, q, 0x20000, 0x30000, 0x40000, 0x50000, None, 0x60000, None, B, T, 1, dk, 16,
                                    1.0, 0, 0, 0, ws, wsb, None)
    assert f(kind=3) == ERR_SHAPE
    assert f(q=None) == ERR_NULL
    assert f(dk=40) == ERR_UNSUP
    assert f(ws=None) == ERR_WS
    assert f(wsb=64) == ERR_WS
    assert f(ws=0x100010) == ERR_ALIGN                      # the workspace needs 256-byte alignment
    assert f(B=0) == OK
    need = lib.kda_forward_host_workspace_bytes(2, 8192, 64, 128, 128, 1, 1, 0, 0)
    # two slots of 1024-token segments and the carried state, plus the status word
    seg = 2 * 1024 * 64 * (3 * 256 + 256 + 2 + 512)
    assert need >= 2 * seg + 2 * 64 * 128 * 128 * 4
    d = lib.kda_decode_step_host
    assert d(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, None, 0x60000, 2, 1, 16, 16, 1.0, 0, 0, 0,
             0x100000, 1 << 20, None) == ERR_NULL
    assert d(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, 0x70000, 0x60000, 2, 1, 16, 16, 1.0, 0, 0, 0,
             None, 0, None) == ERR_WS


def test_varlen_raw_and_gdn2_reject_bad_arguments(lib):
    def r(N=2, cu=0xB0000, dk=16, ws=0x90000):
        return lib.kda_forward_varlen_raw(0x10000, 0x20000, 0x30000, 0x40000, 0x50000, cu, None, 0x60000, None,
                                          N, 8, 1, dk, 16, 1.0, 0, 0, 0, ws, 16, None)
    assert r(N=-1) == ERR_SHAPE
    assert r(cu=None) == ERR_NULL
    assert r(dk=40) == ERR_UNSUP
    assert r(ws=None) == ERR_WS
    assert r(N=0) == OK

    def g(w=0x70000, e=0x50000, o=0x60000, cu=0xB0000):
        return lib.kda_forward_varlen_gdn2(0x10000, 0x20000, 0x30000, 0x40000, e, w, cu, None, o, None,
                                           2, 8, 1, 16, 16, 1.0, 0, 0, 0, 0x90000, 16, None)
    assert g(w=None) == ERR_NULL
    assert g(e=0x50004) == ERR_ALIGN                        # the erase gate needs 16-byte rows
    assert g(o=0x70000 + 64) == ERR_ALIAS                   # o overlaps the write gate
    assert g(cu=None) == ERR_NULL


def test_schedule_setting_round_trip_and_rejection(lib):
    """The process-wide prefill schedule: every known value round-trips, an unknown one
    returns KDA_ERR_VALUE (10) and leaves the setting as it was."""
    prev = lib.kda_get_schedule()
    try:
        for value in (1, 2, 0):
            assert lib.kda_set_schedule(value) == OK
            assert lib.kda_get_schedule() == value
        assert lib.kda_set_schedule(3) == 10 and lib.kda_get_schedule() == 0
        assert lib.kda_set_schedule(-1) == 10 and lib.kda_get_schedule() == 0
        with kda.schedule("scan"):
            assert kda.get_schedule() == "scan"
        assert kda.get_schedule() == "auto"
        with pytest.raises(ValueError):
            kda.set_schedule("fastest")
    finally:
        lib.kda_set_schedule(prev)


def test_schedule_context_restores_after_an_exception(lib):
    prev = kda.get_schedule()
    try:
        kda.set_schedule("scan")
        with pytest.raises(RuntimeError):
            with kda.schedule("chunked"):
                assert kda.get_schedule() == "chunked"
                raise RuntimeError("inside the block")
        assert kda.get_schedule() == "scan"
    finally:
        kda.set_schedule(prev)
