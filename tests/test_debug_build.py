"""The FA_DEBUG build (libfa_debug.so): same entry points as libfa.so, device-side index checks compiled in.

CPU: it builds, loads without a GPU, exports every symbol include/fa.h declares and reports itself as the debug
build (the release library does not).  GPU: every kernel family runs through it on small cases in a child process
and matches the oracle with no index check failing, the bounds self-test is caught there (FA_ERR_BOUNDS, site 99),
and in the release library the same self-test records nothing (checks compiled out).
"""
import ctypes
import json
import os
import subprocess
import sys

import pytest

from exact_io_aware_48_b200 import _lib, build

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
from test_abi import declared_functions  # noqa: E402


@pytest.fixture(scope="module")
def debug_lib():
    build.build()
    lib = ctypes.CDLL(_lib.DEBUG_LIB_PATH)
    lib.fa_debug_build.restype = ctypes.c_int
    return lib


def test_debug_library_exports_every_declared_symbol(debug_lib):
    for n in declared_functions():
        assert hasattr(debug_lib, n), n


def test_debug_flag_differs_between_builds(debug_lib):
    assert debug_lib.fa_debug_build() == 1
    assert _lib.load().fa_debug_build() == 0


def test_bounds_status_string():
    assert _lib.fa_status_string(_lib.FA_ERR_BOUNDS) == "FA_ERR_BOUNDS"


@pytest.mark.gpu
def test_release_build_records_no_bounds_error():
    assert _lib.fa_selftest_bounds(None) == 0
    assert _lib.fa_last_device_status(None) == 0
    assert _lib.fa_last_bounds_site(None) == 0


@pytest.mark.gpu
def test_debug_build_parity_and_bounds_selftest():
    env = dict(os.environ, FA_LIB_PATH=_lib.DEBUG_LIB_PATH)
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_cases.py")], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    assert res["debug_build"] == 1
    assert res["selftest"] == {"status": _lib.FA_ERR_BOUNDS, "site": 99}
    cases = [k for k in res if isinstance(res[k], dict) and "err" in res[k]]
    assert len(cases) == 7
    for k in cases:
        assert res[k]["status"] == 0 and res[k]["site"] == 0, k


@pytest.mark.gpu
def test_debug_build_full_size_workloads_pass_every_index_check():
    env = dict(os.environ, FA_LIB_PATH=_lib.DEBUG_LIB_PATH)
    r = subprocess.run([sys.executable, os.path.join(HERE, "debug_cases.py"), "--full"], env=env,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stdout[-3000:] + r.stderr[-3000:]
    res = json.loads(r.stdout.strip().splitlines()[-1])
    full = [k for k in res if k.startswith("full_")]
    assert len(full) >= 8
    for k in full:
        assert res[k] == {"status": 0, "site": 0}, k

