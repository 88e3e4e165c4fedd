"""Host-side checks of the C-ABI library (no GPU needed): it loads, exports
every entry point ``include/h2o.h`` declares, and rejects bad arguments
before touching the device."""
import ctypes
import os
import re

import pytest

from h2o_kv_cache_step_b200 import _lib
from h2o_kv_cache_step_b200._lib import lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "h2o.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(h2o_[a-z_0-9]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from h2o_kv_cache_step_b200 import build
    build.build()
    return lib()


def test_header_symbols_exported(L):
    names = header_functions()
    assert len(names) >= 15
    bound = {n for n, _, _ in _lib.SIGNATURES}
    for n in names:
        assert hasattr(L, n), f"{n} declared in h2o.h but not exported"
        assert n in bound, f"{n} has no ctypes signature in the binding"
    assert bound == set(names)


def test_version(L):
    assert b"sm_100a" in L.h2o_version()


@pytest.mark.parametrize("args,code", [
    ((1, 6, 4, 128, 64, 0, 64), _lib.H2O_ERR_ARG),          # Hq % Hkv != 0
    ((1, 4, 2, 96, 64, 0, 64), _lib.H2O_ERR_UNSUPPORTED),   # d not in {64, 128}
    ((0, 4, 2, 128, 64, 0, 64), _lib.H2O_ERR_ARG),          # B < 1
    ((1, 4, 2, 128, 0, 0, 64), _lib.H2O_ERR_ARG),           # C < 1
    ((1, 4, 2, 128, 64, 7, 64), _lib.H2O_ERR_ARG),          # unknown dtype
    ((1, 4, 2, 128, 64, 0, 0), _lib.H2O_ERR_ARG),           # max_T < 1
])
def test_create_rejects_bad_shapes(L, args, code):
    h = ctypes.c_void_p()
    rc = L.h2o_create_ex(*args, ctypes.byref(h))
    assert rc == code
    assert not h.value
    assert L.h2o_last_error(None)


def test_null_context_is_an_argument_error(L):
    assert L.h2o_step(None, None, None, None, None, 4, None) == _lib.H2O_ERR_ARG
    assert L.h2o_destroy(None) == _lib.H2O_OK
    assert L.h2o_counters(None, None, None) == _lib.H2O_ERR_ARG
    assert L.h2o_sync_check(None, None) == _lib.H2O_ERR_ARG


def test_create_without_gpu_fails_cleanly(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    h = ctypes.c_void_p()
    rc = L.h2o_create(1, 4, 2, 128, 64, ctypes.byref(h))
    assert rc in (_lib.H2O_ERR_CUDA, _lib.H2O_ERR_OOM)
    assert not h.value
    assert b"cuda" in L.h2o_last_error(None).lower()


def test_new_entry_points_reject_a_null_context(L):
    assert L.h2o_set_policy(None, _lib.H2O_POLICY_SUM) == _lib.H2O_ERR_ARG
    assert L.h2o_host_sync(None) == _lib.H2O_ERR_ARG
    assert L.h2o_step_host_async(None, None, None, None, None, 4, None) == _lib.H2O_ERR_ARG
    assert L.h2o_last_error(None)


def test_policy_constants_match_the_header():
    src = open(os.path.join(ROOT, "include", "h2o.h")).read()
    m = re.search(r"enum h2o_policy \{\s*H2O_POLICY_SUM = (\d+),\s*H2O_POLICY_NORMALIZED = (\d+),"
                  r"\s*H2O_POLICY_INSERT_ALWAYS = (\d+)\s*\}", src)
    assert m, "enum h2o_policy not found in h2o.h"
    assert tuple(int(x) for x in m.groups()) == (_lib.H2O_POLICY_SUM, _lib.H2O_POLICY_NORMALIZED,
                                                 _lib.H2O_POLICY_INSERT_ALWAYS)
