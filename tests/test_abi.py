"""CPU-side checks of the C ABI: libfa.so builds, loads without a GPU, exports every symbol include/fa.h declares,
and rejects bad arguments on the host before touching CUDA."""
import os
import re

import pytest

from exact_io_aware_48_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "fa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree(lib):
    names = declared_functions()
    assert len(names) >= 12
    assert set(names) == set(_lib.SIGNATURES)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert lib.fa_version() == 10300
    assert _lib.fa_status_string(0) == "FA_OK"
    assert _lib.fa_status_string(4) == "FA_ERR_TIMEOUT"
    assert _lib.fa_status_string(99) == "FA_UNKNOWN_STATUS"


def test_workspace_queries(lib):
    assert _lib.fa_blocksparse_workspace_size(0) == 0
    nT = 512
    assert _lib.fa_blocksparse_workspace_size(65536) >= 2 * (nT + 1) * 4 + 2 * nT * nT * 4
    base = _lib.fa_bwd_workspace_size(1, 16, 4096, 128, False)
    assert base >= 16 * 4096 * 128 * 4 + 2 * 16 * 4096 * 4
    assert _lib.fa_bwd_workspace_size(1, 16, 4096, 128, True) > base
    assert _lib.fa_bwd_workspace_size(1, 16, 4096, 96, False) > 0  # 96 runs on the 128 kernel
    assert _lib.fa_bwd_workspace_size(1, 16, 4096, 48, False) == 0


A = 1 << 12  # an aligned fake address: only used for calls that must fail validation before any CUDA call


@pytest.mark.parametrize("args,expect", [
    (dict(q=None), _lib.FA_ERR_INVALID_ARG),
    (dict(q=A + 2), _lib.FA_ERR_INVALID_ARG),
    (dict(d=48), _lib.FA_ERR_UNSUPPORTED),
    (dict(d=192), _lib.FA_ERR_UNSUPPORTED),
    (dict(d=512), _lib.FA_ERR_UNSUPPORTED),
    (dict(N=0), _lib.FA_ERR_INVALID_ARG),
    (dict(N=(1 << 20) + 1), _lib.FA_ERR_INVALID_ARG),
    (dict(B=0), _lib.FA_ERR_INVALID_ARG),
    (dict(scale=0.0), _lib.FA_ERR_INVALID_ARG),
    (dict(scale=-1.0), _lib.FA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), _lib.FA_ERR_INVALID_ARG),
    (dict(dtype=7), _lib.FA_ERR_INVALID_ARG),
    (dict(o=None), _lib.FA_ERR_INVALID_ARG),
])
def test_fwd_argument_errors(lib, args, expect):
    a = dict(q=A, k=A, v=A, o=A, lse=A, B=1, H=1, N=128, d=64, scale=0.125, causal=0, key_lens=None, dtype=0)
    a.update(args)
    rc = _lib.fa_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["N"], a["d"], a["scale"],
                     a["causal"], a["key_lens"], a["dtype"], 0)
    assert rc == expect


def test_bwd_and_blocksparse_argument_errors(lib):
    # missing workspace is reported as a workspace error, missing mask/outputs as invalid arguments
    rc = _lib.fa_bwd(A, A, A, A, A, A, A, A, A, 1, 1, 128, 64, 0.125, 0, None, None, None, 0, 0, 0)
    assert rc == _lib.FA_ERR_WORKSPACE
    rc = _lib.fa_bwd(A, A, A, A, A, A, None, A, A, 1, 1, 128, 64, 0.125, 0, None, None, A, 1 << 30, 0, 0)
    assert rc == _lib.FA_ERR_INVALID_ARG
    rc = _lib.fa_bwd(A, A, A, A, A, A, A, A, A, 1, 1, 128, 64, 0.125, 0, None, None, A, 16, 0, 0)
    assert rc == _lib.FA_ERR_WORKSPACE
    rc = _lib.fa_fwd_blocksparse(A, A, A, A, A, 1, 1, 128, 64, 0.125, 0, None, None, A, 1 << 20, 0, 0)
    assert rc == _lib.FA_ERR_INVALID_ARG
    rc = _lib.fa_fwd_blocksparse(A, A, A, A, A, 1, 1, 128, 64, 0.125, 0, None, A, A + 16, 1 << 20, 0, 0)
    assert rc == _lib.FA_ERR_WORKSPACE
    assert _lib.fa_blockmask_lists(A, 0, A, A, A, A, 0) == _lib.FA_ERR_INVALID_ARG
    assert _lib.fa_blockmask_lists(A, 8193, A, A, A, A, 0) == _lib.FA_ERR_INVALID_ARG


def test_head_dims_checked_before_any_cuda_call(lib):
    # d = 256 runs forward and backward; other head dims are refused before any CUDA call
    rc = _lib.fa_bwd(A, A, A, A, A, A, A, A, A, 1, 1, 128, 192, 0.0625, 0, None, None, A, 1 << 30, 0, 0)
    assert rc == _lib.FA_ERR_UNSUPPORTED
    assert _lib.fa_bwd_workspace_size(1, 2, 1024, 256, False) >= 2 * 1024 * 256 * 4
    assert _lib.fa_bwd_varlen_workspace_size(1, 2, 1024, 256) > 0
    assert _lib.fa_bwd_workspace_size(1, 2, 1024, 192, False) == 0
    assert _lib.fa_fwd_splitkv_workspace_size(1, 2, 1, 4096, 256, 0) > 0


def test_budget_and_selftest_argument_errors(lib):
    assert _lib.fa_set_wait_budget_ns(10) == _lib.FA_ERR_INVALID_ARG
    assert _lib.fa_selftest_wait_timeout(10, 0) == _lib.FA_ERR_INVALID_ARG
    assert _lib.fa_selftest_wait_timeout(2_000_000_000, 0) == _lib.FA_ERR_INVALID_ARG


def test_noalloc_reports_the_same_status_as_fa_bwd(lib):
    # fa_bwd_noalloc runs fa_bwd's argument checks first, so a bad argument gets the same status from both; only a
    # valid problem too large for the fixed array gets FA_ERR_WORKSPACE.  No CUDA call is reached in these cases.
    big = dict(B=8, H=64, N=1024, d=128)  # needs ~260 MiB of scratch
    cases = [
        (dict(q=None, **big), _lib.FA_ERR_INVALID_ARG),
        (dict(dq=A + 8, **big), _lib.FA_ERR_INVALID_ARG),
        (dict(B=8, H=64, N=(1 << 20) + 1, d=48), _lib.FA_ERR_INVALID_ARG),
        (dict(B=8, H=64, N=1024, d=48), _lib.FA_ERR_UNSUPPORTED),
        (dict(B=1 << 20, H=1 << 12, N=1024, d=64), _lib.FA_ERR_INVALID_ARG),  # B*H*N*d far beyond 2^34
        (dict(scale=0.0, **big), _lib.FA_ERR_INVALID_ARG),
        (big, _lib.FA_ERR_WORKSPACE),
    ]
    for args, expect in cases:
        a = dict(q=A, dq=A, B=1, H=1, N=128, d=64, scale=0.125)
        a.update(args)
        rc = _lib.fa_bwd_noalloc(a["q"], A, A, A, A, A, a["dq"], A, A, a["B"], a["H"], a["N"], a["d"], a["scale"], 0,
                                 None, None, 0, 0)
        assert rc == expect, (args, rc)
        if expect != _lib.FA_ERR_WORKSPACE:  # fa_bwd reports the same (with a workspace far too small)
            rc2 = _lib.fa_bwd(a["q"], A, A, A, A, A, a["dq"], A, A, a["B"], a["H"], a["N"], a["d"], a["scale"], 0,
                              None, None, A, 16, 0, 0)
            assert rc2 == expect, (args, rc2)
    assert _lib.fa_bwd_workspace_size(1 << 20, 1 << 12, 1024, 64, False) == 0  # no int overflow in B*H
