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
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
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


def set_num_threads(n: int) -> None:
    """Use n OpenMP threads from now on (n >= 1)."""
    _load().oracle_set_num_threads(int(n))


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


def _varlen_slices(cu_q, cu_k):
    cu_q = np.asarray(cu_q, dtype=np.int64)
    cu_k = np.asarray(cu_k, dtype=np.int64)
    if cu_q.shape != cu_k.shape or cu_q.ndim != 1 or cu_q.size < 2:
        raise ValueError("cu_seqlens_q and cu_seqlens_k must be 1-D of the same length B+1 >= 2")
    for b in range(cu_q.size - 1):
        yield int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])


def _pad_seq(x, a, e, n):
    """Tokens a..e-1 of a [total, H, d] array as a [1, H, n, d] problem, zero rows after e-a."""
    t = np.zeros((1, x.shape[1], n, x.shape[2]))
    t[0, :, :e - a] = x[a:e].transpose(1, 0, 2)
    return t


def attn_fwd_varlen(q, k, v, cu_q, cu_k, scale, causal=False):
    """Packed variable-length batch (q [total_q,H,d], k, v [total_k,H,d]): sequence b is standard attention of its
    own queries cu_q[b]..cu_q[b+1]-1 against its own keys cu_k[b]..cu_k[b+1]-1, causal meaning key c <= query r
    within the sequence.  Each sequence is run through attn_fwd zero-padded to n = max(len_q, len_k) rows with
    key_lens = [len_k]; the padded query rows are dropped.  Returns (O [total_q,H,d], LSE [H,total_q]) in fp64."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    total_q, H, d = q.shape
    o = np.zeros((total_q, H, d))
    lse = np.full((H, total_q), -np.inf)
    for a, e, ak, ek in _varlen_slices(cu_q, cu_k):
        lq, lk = e - a, ek - ak
        if lq <= 0:
            continue
        n = max(lq, lk)
        ob, lb = attn_fwd(_pad_seq(q, a, e, n), _pad_seq(k, ak, ek, n), _pad_seq(v, ak, ek, n), scale, causal=causal,
                          key_lens=np.array([lk], dtype=np.int32))
        o[a:e] = ob[0, :, :lq].transpose(1, 0, 2)
        lse[:, a:e] = lb[0, :, :lq]
    return o, lse


def attn_bwd_varlen(q, k, v, do, cu_q, cu_k, scale, causal=False):
    """Gradients of sum(O * dO) for attn_fwd_varlen, per sequence through attn_bwd (padded query rows carry dO = 0,
    so they add nothing).  Returns (dQ [total_q,H,d], dK, dV [total_k,H,d], O, LSE [H,total_q])."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    total_q, H, d = q.shape
    total_k = k.shape[0]
    dq = np.zeros((total_q, H, d))
    dk = np.zeros((total_k, H, d))
    dv = np.zeros((total_k, H, d))
    o = np.zeros((total_q, H, d))
    lse = np.full((H, total_q), -np.inf)
    for a, e, ak, ek in _varlen_slices(cu_q, cu_k):
        lq, lk = e - a, ek - ak
        if lq <= 0 and lk <= 0:
            continue
        n = max(lq, lk, 1)
        gq, gk, gv, ob, lb = attn_bwd(_pad_seq(q, a, e, n), _pad_seq(k, ak, ek, n), _pad_seq(v, ak, ek, n),
                                      _pad_seq(do, a, e, n), scale, causal=causal,
                                      key_lens=np.array([lk], dtype=np.int32))
        dq[a:e] = gq[0, :, :lq].transpose(1, 0, 2)
        dk[ak:ek] = gk[0, :, :lk].transpose(1, 0, 2)
        dv[ak:ek] = gv[0, :, :lk].transpose(1, 0, 2)
        o[a:e] = ob[0, :, :lq].transpose(1, 0, 2)
        lse[:, a:e] = lb[0, :, :lq]
    return dq, dk, dv, o, lse


def attn_fwd_decode(q, k, v, scale, causal=False, key_lens=None):
    """Attention of Nq new queries per (b, h) against Nk cached keys/values (q [B,H,Nq,d], k, v [B,H,Nk,d]): the
    queries are the last Nq positions of their sequence, so with len = key_lens[b] (else Nk) key c is visible from
    query r iff c < len and (causal) c <= r + len - Nq.  Softmax of scale * q k^T over the visible keys, written
    out directly in numpy (fp64).  Returns (O [B,H,Nq,d], LSE [B,H,Nq]); a row with no visible key has O = 0 and
    LSE = -inf."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    o = np.zeros((B, H, Nq, d))
    lse = np.full((B, H, Nq), -np.inf)
    r = np.arange(Nq)[:, None]
    c = np.arange(Nk)[None, :]
    for b in range(B):
        n = Nk if key_lens is None else int(min(max(int(key_lens[b]), 0), Nk))
        vis = c < n
        if causal:
            vis = vis & (c <= r + n - Nq)
        for h in range(H):
            s = scale * (q[b, h] @ k[b, h].T)
            s = np.where(vis, s, -np.inf)
            m = s.max(axis=1, keepdims=True)
            ok = np.isfinite(m[:, 0])
            e = np.where(vis, np.exp(s - np.where(np.isfinite(m), m, 0.0)), 0.0)
            l = e.sum(axis=1)
            o[b, h, ok] = (e[ok] @ v[b, h]) / l[ok, None]
            lse[b, h, ok] = m[ok, 0] + np.log(l[ok])
    return o, lse


def attn_bwd_head_masks(q, k, v, do, scale, masks, causal=False, key_lens=None, tile=128):
    """Per-head block masks (masks [H, nT, nT]): head h is attn_bwd of that head's slice with mask masks[h].
    Returns (dQ, dK, dV, O, LSE) like attn_bwd."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    outs = [attn_bwd(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], do[:, h:h + 1], scale, causal=causal,
                     key_lens=key_lens, block_mask=np.asarray(masks[h], dtype=np.uint8), tile=tile)
            for h in range(q.shape[1])]
    return tuple(np.concatenate([o[i] for o in outs], axis=1) for i in range(5))


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
