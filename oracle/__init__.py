"""fp64 CPU oracle for exact softmax attention (forward, backward, block-mask index lists).

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the benchmark's CPU-baseline leg are the
only callers.  The CUDA library never imports, links or runs anything here, and nothing here imports the CUDA
library; the two sides meet only through seeded inputs made by ``exact_io_aware_48_b200.inputs``.

The arithmetic lives in ``attn_oracle.c`` (plain loops, fp64, OpenMP over independent heads or rows).  This module
compiles it with gcc on first use and marshals numpy arrays in and out.  Every function follows the definitions
cited in the C file's header: standard attention softmax(scale * Q K^T + mask) V (FlashAttention review page,
"Method" and claim C2; explainer page, "standard attention"), its analytic gradients (review page, claim C7,
read as the calculus of that definition) and the online-softmax recurrence (explainer page, "online softmax").

Parity pins: every function here is pinned by tests/test_oracle_pins.py against closed forms, invariants, a
library routine (scipy.special.logsumexp) and central finite differences; none is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i32p = ctypes.POINTER(ctypes.c_int32)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u8p = ctypes.POINTER(ctypes.c_uint8)


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP).  Returns the path."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        # -fno-fast-math keeps IEEE semantics (inf handling, no reassociation) for the reference arithmetic.
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC,
                               "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _bind(path: str):
    """Open a compiled oracle library and declare its C signatures."""
    lib = ctypes.CDLL(path)
    common = [_dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
              ctypes.c_int, _i32p, _u8p, ctypes.c_int]
    lib.oracle_fwd.argtypes = common + [_dp, _dp]
    lib.oracle_fwd_rows.argtypes = common + [ctypes.c_int, _i64p, _i64p, _dp, _dp]
    lib.oracle_fwd_online.argtypes = common + [ctypes.c_int, ctypes.c_int, ctypes.c_int, _dp, _dp]
    common_bwd = [_dp, _dp, _dp, _dp] + common[3:]
    lib.oracle_bwd.argtypes = common_bwd + [_dp, _dp, _dp, _dp, _dp]
    lib.oracle_bwd_rows.argtypes = common_bwd + [ctypes.c_int, _i64p, _i64p, _dp]
    lib.oracle_bwd_keys.argtypes = common_bwd + [ctypes.c_int, _i64p, _i64p, _dp, _dp]
    lib.oracle_blockmask_csr.argtypes = [_u8p, ctypes.c_int, _i32p, _i32p]
    lib.oracle_blockmask_csr.restype = ctypes.c_int64
    lib.oracle_blockmask_csc.argtypes = [_u8p, ctypes.c_int, _i32p, _i32p]
    lib.oracle_blockmask_csc.restype = ctypes.c_int64
    lib.oracle_num_threads.restype = ctypes.c_int
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(build())
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle uses (OMP_NUM_THREADS, else all host cores)."""
    return int(_load().oracle_num_threads())


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a, t):
    return None if a is None else a.ctypes.data_as(t)


def _problem(q, k, v, scale, causal, key_lens, block_mask, tile):
    q, k, v = _f64(q), _f64(k), _f64(v)
    if q.ndim != 4 or q.shape != k.shape or q.shape != v.shape:
        raise ValueError("q, k, v must all be [B, H, N, d]")
    B, H, N, d = q.shape
    kl = None if key_lens is None else np.ascontiguousarray(key_lens, dtype=np.int32)
    bm = None if block_mask is None else np.ascontiguousarray(block_mask, dtype=np.uint8)
    if kl is not None and kl.shape != (B,):
        raise ValueError("key_lens must be [B]")
    if bm is not None:
        nT = -(-N // tile)
        if bm.shape != (nT, nT):
            raise ValueError(f"block_mask must be [{nT}, {nT}] for tile {tile}")
    args = [_ptr(q, _dp), _ptr(k, _dp), _ptr(v, _dp), B, H, N, d, float(scale), int(bool(causal)),
            _ptr(kl, _i32p), _ptr(bm, _u8p), int(tile)]
    return (q, k, v, kl, bm), args, (B, H, N, d)


def attn_fwd(q, k, v, scale, causal=False, key_lens=None, block_mask=None, tile=128):
    """Two-pass standard attention. Returns (O [B,H,N,d], LSE [B,H,N]) in fp64."""
    keep, args, (B, H, N, d) = _problem(q, k, v, scale, causal, key_lens, block_mask, tile)
    o = np.empty((B, H, N, d))
    lse = np.empty((B, H, N))
    _load().oracle_fwd(*args, _ptr(o, _dp), _ptr(lse, _dp))
    return o, lse


def attn_fwd_rows(q, k, v, scale, sel_bh, sel_r, causal=False, key_lens=None, block_mask=None, tile=128):
    """Forward for selected (flattened head, row) pairs. Returns (O [n,d], LSE [n])."""
    keep, args, (B, H, N, d) = _problem(q, k, v, scale, causal, key_lens, block_mask, tile)
    sb = np.ascontiguousarray(sel_bh, dtype=np.int64)
    sr = np.ascontiguousarray(sel_r, dtype=np.int64)
    n = sb.shape[0]
    o = np.empty((n, d))
    lse = np.empty((n,))
    _load().oracle_fwd_rows(*args, n, _ptr(sb, _i64p), _ptr(sr, _i64p), _ptr(o, _dp), _ptr(lse, _dp))
    return o, lse


def attn_fwd_online(q, k, v, scale, tile_q, tile_k, kv_outer, causal=False, key_lens=None, block_mask=None,
                    tile=128):
    """Online-softmax tiled forward (any tile sizes, either loop order). Returns (O, LSE)."""
    keep, args, (B, H, N, d) = _problem(q, k, v, scale, causal, key_lens, block_mask, tile)
    o = np.empty((B, H, N, d))
    lse = np.empty((B, H, N))
    _load().oracle_fwd_online(*args, int(tile_q), int(tile_k), int(bool(kv_outer)), _ptr(o, _dp), _ptr(lse, _dp))
    return o, lse


def attn_bwd(q, k, v, do, scale, causal=False, key_lens=None, block_mask=None, tile=128):
    """Analytic gradients of sum(O * dO). Returns (dQ, dK, dV, O, LSE)."""
    keep, args, (B, H, N, d) = _problem(q, k, v, scale, causal, key_lens, block_mask, tile)
    do = _f64(do)
    if do.shape != (B, H, N, d):
        raise ValueError("dO must match q")
    dq, dk, dv, o = (np.empty((B, H, N, d)) for _ in range(4))
    lse = np.empty((B, H, N))
    _load().oracle_bwd(*args[:3], _ptr(do, _dp), *args[3:], _ptr(dq, _dp), _ptr(dk, _dp), _ptr(dv, _dp),
                       _ptr(o, _dp), _ptr(lse, _dp))
    return dq, dk, dv, o, lse


def attn_bwd_rows(q, k, v, do, scale, sel_bh, sel_r, causal=False, key_lens=None, block_mask=None, tile=128):
    """dQ rows for selected (head, row) pairs. Returns dQ [n, d]."""
    keep, args, (B, H, N, d) = _problem(q, k, v, scale, causal, key_lens, block_mask, tile)
    do = _f64(do)
    sb = np.ascontiguousarray(sel_bh, dtype=np.int64)
    sr = np.ascontiguousarray(sel_r, dtype=np.int64)
    n = sb.shape[0]
    dq = np.empty((n, d))
    _load().oracle_bwd_rows(*args[:3], _ptr(do, _dp), *args[3:], n, _ptr(sb, _i64p), _ptr(sr, _i64p),
                            _ptr(dq, _dp))
    return dq


def attn_bwd_keys(q, k, v, do, scale, sel_bh, sel_c, causal=False, key_lens=None, block_mask=None, tile=128):
    """dK and dV rows for selected (head, key) pairs. Returns (dK [n, d], dV [n, d])."""
    keep, args, (B, H, N, d) = _problem(q, k, v, scale, causal, key_lens, block_mask, tile)
    do = _f64(do)
    sb = np.ascontiguousarray(sel_bh, dtype=np.int64)
    sc = np.ascontiguousarray(sel_c, dtype=np.int64)
    n = sb.shape[0]
    dk = np.empty((n, d))
    dv = np.empty((n, d))
    _load().oracle_bwd_keys(*args[:3], _ptr(do, _dp), *args[3:], n, _ptr(sb, _i64p), _ptr(sc, _i64p),
                            _ptr(dk, _dp), _ptr(dv, _dp))
    return dk, dv


def blockmask_csr(mask):
    """CSR of a square 0/1 tile mask: (row_ptr [nT+1] int32, col_idx [nnz] int32), ascending columns."""
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    nT = m.shape[0]
    row_ptr = np.empty(nT + 1, dtype=np.int32)
    col_idx = np.empty(max(int(m.astype(bool).sum()), 1), dtype=np.int32)
    nnz = _load().oracle_blockmask_csr(_ptr(m, _u8p), nT, _ptr(row_ptr, _i32p), _ptr(col_idx, _i32p))
    return row_ptr, col_idx[:nnz]


def blockmask_csc(mask):
    """CSC of a square 0/1 tile mask: (col_ptr [nT+1] int32, row_idx [nnz] int32), ascending rows."""
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    nT = m.shape[0]
    col_ptr = np.empty(nT + 1, dtype=np.int32)
    row_idx = np.empty(max(int(m.astype(bool).sum()), 1), dtype=np.int32)
    nnz = _load().oracle_blockmask_csc(_ptr(m, _u8p), nT, _ptr(col_ptr, _i32p), _ptr(row_idx, _i32p))
    return col_ptr, row_idx[:nnz]
