"""ctypes binding of libfa.so: one Python function per C entry point, with the same names and arguments.

Argument marshalling only: pointers may be given as ints or as torch tensors (their data_ptr() is passed), the
stream as an int handle, a torch.cuda.Stream or None (current torch stream).  Every step of the computation runs
in the library's CUDA kernels; there is no fallback.  If libfa.so is missing or cannot be loaded, every call
raises RuntimeError.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
RELEASE_LIB_PATH = os.path.join(_HERE, "libfa.so")
DEBUG_LIB_PATH = os.path.join(_HERE, "libfa_debug.so")  # FA_DEBUG=1 build: device-side index checks
# FA_LIB_PATH (a debug knob) selects another build of the same library, e.g. DEBUG_LIB_PATH
LIB_PATH = os.environ.get("FA_LIB_PATH") or RELEASE_LIB_PATH

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_CUDA, FA_ERR_TIMEOUT, FA_ERR_WORKSPACE, FA_ERR_BOUNDS = range(7)
FA_BF16, FA_FP16 = 0, 1

# C signatures, exactly as declared in include/fa.h
_P, _I, _F, _SZ, _U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint64
SIGNATURES = {
    "fa_version": ([], _I),
    "fa_status_string": ([_I], ctypes.c_char_p),
    "fa_last_error_string": ([], ctypes.c_char_p),
    "fa_fwd": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _I, _P], _I),
    "fa_blocksparse_workspace_size": ([_I], _SZ),
    "fa_fwd_blocksparse": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _P, _P, _SZ, _I, _P], _I),
    "fa_bwd_workspace_size": ([_I, _I, _I, _I, _I], _SZ),
    "fa_bwd": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _P, _P, _SZ, _I, _P], _I),
    "fa_blockmask_lists": ([_P, _I, _P, _P, _P, _P, _P], _I),
    "fa_last_device_status": ([_P], _I),
    "fa_set_wait_budget_ns": ([_U64], _I),
    "fa_selftest_wait_timeout": ([_U64, _P], _I),
    "fa_set_kernel_events": ([_I, _P, _P], _I),
    "fa_selftest_exp2": ([_P, _P, _P, _I, _P], _I),
    "fa_debug_build": ([], _I),
    "fa_last_bounds_site": ([_P], _I),
    "fa_selftest_bounds": ([_P], _I),
    "fa_set_fwd_tiles_per_cta": ([_I], _I),
    "fa_bwd_noalloc": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _P, _I, _P], _I),
    "fa_fwd_varlen": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _I, _P], _I),
    "fa_bwd_varlen_workspace_size": ([_I, _I, _I, _I], _SZ),
    "fa_fwd_splitkv_workspace_size": ([_I, _I, _I, _I, _I, _I], _SZ),
    "fa_blocksparse_heads_workspace_size": ([_I, _I], _SZ),
    "fa_fwd_blocksparse_heads": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _P, _P, _SZ, _I, _P], _I),
    "fa_bwd_blocksparse_heads_workspace_size": ([_I, _I, _I, _I], _SZ),
    "fa_bwd_blocksparse_heads": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P, _P, _P, _SZ, _I,
                                  _P], _I),
    "fa_fwd_splitkv": ([_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _I, _P, _I, _P, _SZ, _I, _P], _I),
    "fa_bwd_varlen": ([_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I, _P, _SZ, _I,
                       _P], _I),
}
FA_NOALLOC_SCRATCH_BYTES = 32 << 20
FA_KERNEL_FWD, FA_KERNEL_BWD_MAIN = 0, 1

_lib = None


def load(path: str = LIB_PATH):
    """Load libfa.so once and declare its signatures.  Raises RuntimeError if it cannot be loaded."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"libfa.so not found at {path}: build it with `python -m exact_io_aware_48_b200.build`")
        try:
            lib = ctypes.CDLL(path)
        except OSError as e:  # pragma: no cover - environment dependent
            raise RuntimeError(f"cannot load libfa.so: {e}") from e
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def fa_version() -> int:
    return load().fa_version()


def fa_status_string(status: int) -> str:
    return load().fa_status_string(status).decode()


def fa_last_error_string() -> str:
    return load().fa_last_error_string().decode()


def fa_fwd(q, k, v, o, lse, B, H, N, d, softmax_scale, causal, key_lens, dtype, stream=None) -> int:
    return load().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, softmax_scale, int(causal),
                         _ptr(key_lens), dtype, _stream(stream))


def fa_blocksparse_workspace_size(N) -> int:
    return load().fa_blocksparse_workspace_size(N)


def fa_fwd_blocksparse(q, k, v, o, lse, B, H, N, d, softmax_scale, causal, key_lens, block_mask, workspace,
                       workspace_bytes, dtype, stream=None) -> int:
    return load().fa_fwd_blocksparse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, softmax_scale,
                                     int(causal), _ptr(key_lens), _ptr(block_mask), _ptr(workspace),
                                     workspace_bytes, dtype, _stream(stream))


def fa_bwd_workspace_size(B, H, N, d, has_block_mask) -> int:
    return load().fa_bwd_workspace_size(B, H, N, d, int(bool(has_block_mask)))


def fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, softmax_scale, causal, key_lens, block_mask, workspace,
           workspace_bytes, dtype, stream=None) -> int:
    return load().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                         B, H, N, d, softmax_scale, int(causal), _ptr(key_lens), _ptr(block_mask), _ptr(workspace),
                         workspace_bytes, dtype, _stream(stream))


def fa_blockmask_lists(mask, nT, row_ptr, col_idx, col_ptr, row_idx, stream=None) -> int:
    return load().fa_blockmask_lists(_ptr(mask), nT, _ptr(row_ptr), _ptr(col_idx), _ptr(col_ptr), _ptr(row_idx),
                                     _stream(stream))


def fa_last_device_status(stream=None) -> int:
    return load().fa_last_device_status(_stream(stream))


def fa_set_wait_budget_ns(budget_ns) -> int:
    return load().fa_set_wait_budget_ns(int(budget_ns))


def fa_selftest_wait_timeout(budget_ns, stream=None) -> int:
    return load().fa_selftest_wait_timeout(int(budget_ns), _stream(stream))


def fa_set_kernel_events(kernel, start_event, stop_event) -> int:
    """Events are torch.cuda.Event (their cuda_event handle is passed), raw int handles, or None."""
    def h(e):
        if e is None:
            return None
        handle = e if isinstance(e, int) else e.cuda_event
        if not handle:
            raise ValueError("CUDA event not created yet (torch creates events on their first record())")
        return handle
    return load().fa_set_kernel_events(kernel, h(start_event), h(stop_event))


def fa_bwd_noalloc(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, softmax_scale, causal, key_lens, block_mask,
                   dtype, stream=None) -> int:
    """fa_bwd with the library's fixed device scratch instead of a caller workspace (allocates nothing)."""
    return load().fa_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                 _ptr(dv), B, H, N, d, softmax_scale, int(causal), _ptr(key_lens), _ptr(block_mask),
                                 dtype, _stream(stream))


def fa_selftest_exp2(x, out_fma, out_mufu, n, stream=None) -> int:
    return load().fa_selftest_exp2(_ptr(x), _ptr(out_fma), _ptr(out_mufu), n, _stream(stream))


def fa_debug_build() -> int:
    return load().fa_debug_build()


def fa_last_bounds_site(stream=None) -> int:
    return load().fa_last_bounds_site(_stream(stream))


def fa_selftest_bounds(stream=None) -> int:
    return load().fa_selftest_bounds(_stream(stream))


def fa_set_fwd_tiles_per_cta(tiles) -> int:
    return load().fa_set_fwd_tiles_per_cta(int(tiles))


def fa_fwd_varlen(q, k, v, o, lse, cu_q, cu_k, B, H, max_q, max_k, total_q, total_k, d, softmax_scale, causal, dtype,
                  stream=None) -> int:
    return load().fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(cu_q), _ptr(cu_k), B, H, max_q,
                                max_k, total_q, total_k, d, softmax_scale, int(causal), dtype, _stream(stream))


def fa_bwd_varlen_workspace_size(B, H, max_q, d) -> int:
    return load().fa_bwd_varlen_workspace_size(B, H, max_q, d)


def fa_bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, cu_q, cu_k, B, H, max_q, max_k, total_q, total_k, d,
                  softmax_scale, causal, workspace, workspace_bytes, dtype, stream=None) -> int:
    return load().fa_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk),
                                _ptr(dv), _ptr(cu_q), _ptr(cu_k), B, H, max_q, max_k, total_q, total_k, d,
                                softmax_scale, int(causal), _ptr(workspace), workspace_bytes, dtype, _stream(stream))


def fa_fwd_splitkv_workspace_size(B, H, Nq, Nk, d, num_splits) -> int:
    return load().fa_fwd_splitkv_workspace_size(B, H, Nq, Nk, d, num_splits)


def fa_fwd_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, softmax_scale, causal, key_lens, num_splits, workspace,
                   workspace_bytes, dtype, stream=None) -> int:
    return load().fa_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, Nq, Nk, d, softmax_scale,
                                 int(causal), _ptr(key_lens), num_splits, _ptr(workspace), workspace_bytes, dtype,
                                 _stream(stream))


def fa_blocksparse_heads_workspace_size(H, N) -> int:
    return load().fa_blocksparse_heads_workspace_size(H, N)


def fa_fwd_blocksparse_heads(q, k, v, o, lse, B, H, N, d, softmax_scale, causal, key_lens, block_masks, workspace,
                             workspace_bytes, dtype, stream=None) -> int:
    return load().fa_fwd_blocksparse_heads(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), B, H, N, d, softmax_scale,
                                           int(causal), _ptr(key_lens), _ptr(block_masks), _ptr(workspace),
                                           workspace_bytes, dtype, _stream(stream))


def fa_bwd_blocksparse_heads_workspace_size(B, H, N, d) -> int:
    return load().fa_bwd_blocksparse_heads_workspace_size(B, H, N, d)


def fa_bwd_blocksparse_heads(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, softmax_scale, causal, key_lens,
                             block_masks, workspace, workspace_bytes, dtype, stream=None) -> int:
    return load().fa_bwd_blocksparse_heads(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq),
                                           _ptr(dk), _ptr(dv), B, H, N, d, softmax_scale, int(causal), _ptr(key_lens),
                                           _ptr(block_masks), _ptr(workspace), workspace_bytes, dtype,
                                           _stream(stream))
