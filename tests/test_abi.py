"""The C-ABI library loads, exports every symbol include/h2o.h declares, and
validates arguments -- all without a GPU (no call here reaches a kernel)."""
import ctypes
import os
import re
import subprocess

import pytest

from h2o_kv_cache_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "h2o.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(h2o_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for must in ("h2o_create", "h2o_prefill", "h2o_step", "h2o_read_state", "h2o_destroy",
                 "h2o_last_error"):
        assert must in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(h2o_\w+)", out))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, f"declared but not exported: {missing}"
    # and the binding covers exactly the declared calls
    assert sorted(_lib.SIGNATURES) == declared_functions()


def _create(M=64, R=8, Hq=4, Hkv=2, d=64, dtype=_lib.H2O_F32):
    h = ctypes.c_void_p()
    rc = _lib.lib.h2o_create(M, R, Hq, Hkv, d, dtype, ctypes.byref(h))
    return rc, h


@pytest.mark.parametrize("args,code", [
    (dict(M=0), _lib.H2O_EINVAL),
    (dict(R=64), _lib.H2O_EINVAL),          # R >= M
    (dict(R=-1), _lib.H2O_EINVAL),
    (dict(Hq=6, Hkv=4), _lib.H2O_EINVAL),   # Hq % Hkv
    (dict(d=96), _lib.H2O_EINVAL),
    (dict(dtype=7), _lib.H2O_EINVAL),
])
def test_create_rejects_bad_arguments(args, code):
    rc, h = _create(**args)
    assert rc == code and not h.value
    assert len(_lib.lib.h2o_last_error(None)) > 0


def test_create_destroy_and_state_errors():
    rc, h = _create()
    assert rc == _lib.H2O_OK and h.value
    arr = (ctypes.c_int64 * 5)()
    assert _lib.lib.h2o_info(h, arr) == _lib.H2O_OK
    assert list(arr) == [0, 0, 0, 0, 0]
    dummy = ctypes.c_void_p(16)
    # step / read_state before prefill: H2O_ESTATE, decided on the host
    assert _lib.lib.h2o_step(h, dummy, dummy, dummy, dummy, 8, None) == _lib.H2O_ESTATE
    assert b"before h2o_prefill" in _lib.lib.h2o_last_error(h)
    assert _lib.lib.h2o_read_state(h, None, None, None, None) == _lib.H2O_ESTATE
    # prefill longer than the cache: H2O_ESHAPE before any allocation
    assert _lib.lib.h2o_prefill(h, dummy, dummy, dummy, None, 1, 65, None) == _lib.H2O_ESHAPE
    assert _lib.lib.h2o_prefill(h, None, dummy, dummy, None, 1, 8, None) == _lib.H2O_EINVAL
    assert _lib.lib.h2o_last_timings(h, None, 0) == _lib.H2O_ESTATE
    assert _lib.lib.h2o_destroy(h) == _lib.H2O_OK
    assert _lib.lib.h2o_destroy(None) == _lib.H2O_OK


def test_null_handle_calls_fail_cleanly():
    dummy = ctypes.c_void_p(16)
    assert _lib.lib.h2o_step(None, dummy, dummy, dummy, dummy, 1, None) == _lib.H2O_EINVAL
    assert _lib.lib.h2o_prefill(None, dummy, dummy, dummy, None, 1, 1, None) == _lib.H2O_EINVAL
    assert _lib.lib.h2o_info(None, None) == _lib.H2O_EINVAL


def test_select_rejects_bad_sizes():
    dummy = ctypes.c_void_p(16)
    assert _lib.lib.h2o_select(dummy, dummy, 0, 8, 10, 1, 2, dummy, None) == _lib.H2O_EINVAL
    assert _lib.lib.h2o_select(dummy, dummy, 1, 8, 10, 1, 9, dummy, None) == _lib.H2O_EINVAL
    assert _lib.lib.h2o_select(None, dummy, 1, 8, 10, 1, 2, dummy, None) == _lib.H2O_EINVAL
    # need == 0 is a no-op that touches no memory
    assert _lib.lib.h2o_select(dummy, dummy, 1, 8, 10, 1, 0, None, None) == _lib.H2O_OK


def test_injected_allocation_failure_is_reported(monkeypatch):
    # H2O_FAULT=alloc makes every device allocation of the library fail; it is
    # made on the host, before any CUDA call, so no GPU is needed to see it
    monkeypatch.setenv("H2O_FAULT", "alloc")
    rc, h = _create()
    assert rc == _lib.H2O_OK
    dummy = ctypes.c_void_p(16)
    assert _lib.lib.h2o_prefill(h, dummy, dummy, dummy, None, 1, 8, None) == _lib.H2O_ENOMEM
    assert b"alloc" in _lib.lib.h2o_last_error(h)
    # nothing stays allocated, the handle is still not prefilled
    assert _lib.lib.h2o_step(h, dummy, dummy, dummy, dummy, 8, None) == _lib.H2O_ESTATE
    assert _lib.lib.h2o_prefill(h, dummy, dummy, dummy, None, 1, 8, None) == _lib.H2O_ENOMEM
    assert _lib.lib.h2o_destroy(h) == _lib.H2O_OK


def test_create_policy_rejects_unknown_policies():
    h = ctypes.c_void_p()
    assert _lib.lib.h2o_create_policy(64, 8, 4, 2, 64, _lib.H2O_F32, 7, ctypes.byref(h)) == _lib.H2O_EINVAL
    assert not h.value and b"policy" in _lib.lib.h2o_last_error(None)
    for pol in (_lib.H2O_POLICY_H2O, _lib.H2O_POLICY_LR):
        assert _lib.lib.h2o_create_policy(64, 8, 4, 2, 64, _lib.H2O_F32, pol, ctypes.byref(h)) == _lib.H2O_OK
        assert _lib.lib.h2o_destroy(h) == _lib.H2O_OK
