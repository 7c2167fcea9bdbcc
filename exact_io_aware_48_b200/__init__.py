"""exact_io_aware_48_b200: exact IO-aware attention (FlashAttention-style tiling) for NVIDIA B200 (sm_100a).

The computation lives in libfa.so (hand-written CUDA kernels behind the C ABI of include/fa.h); this package is
its thin Python face.  ``_lib`` mirrors the C entry points one to one; the helpers below only allocate outputs
and workspace with torch (device memory and streams), call the library and turn a non-zero status into an
exception.  There is no CPU or library fallback: without a CUDA device and a loadable libfa.so every call raises.
"""
from __future__ import annotations

import math

from . import _lib
from ._lib import (FA_BF16, FA_FP16, FA_OK, FA_ERR_CUDA, FA_ERR_INVALID_ARG, FA_ERR_TIMEOUT, FA_ERR_UNSUPPORTED,
                   FA_ERR_WORKSPACE)

__all__ = ["attention", "attention_varlen", "attention_fwd", "attention_bwd", "attention_fwd_varlen", "attention_bwd_varlen",
           "attention_fwd_splitkv", "blockmask_lists", "FAError", "FA_BF16", "FA_FP16"]


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        detail = _lib.fa_last_error_string() if status == FA_ERR_CUDA else ""
        super().__init__(f"{where}: {_lib.fa_status_string(status)}{(' (' + detail + ')') if detail else ''}")
        self.status = status


def _check(rc: int, where: str):
    if rc != FA_OK:
        raise FAError(rc, where)


def _dtype_code(t):
    import torch
    if t.dtype == torch.bfloat16:
        return FA_BF16
    if t.dtype == torch.float16:
        return FA_FP16
    raise TypeError(f"q/k/v must be bfloat16 or float16, got {t.dtype}")


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise RuntimeError("exact_io_aware_48_b200 runs on CUDA tensors only (no CPU fallback)")


def attention_fwd(q, k, v, causal=False, softmax_scale=None, key_lens=None, block_mask=None, stream=None):
    """O, LSE = exact attention of [B, H, N, d] CUDA tensors (bf16 or fp16).

    key_lens: optional int32 CUDA tensor [B]; block_mask: optional uint8 CUDA tensor [nT, nT] (128x128 tiles,
    shared by all heads) or [H, nT, nT] (one mask per head).
    Returns O (same dtype) and LSE (fp32, natural log) [B, H, N].
    """
    import torch
    _require_cuda(q, k, v, key_lens, block_mask)
    B, H, N, d = q.shape
    scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    dt = _dtype_code(q)
    if block_mask is None:
        _check(_lib.fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, key_lens, dt, stream), "fa_fwd")
    elif block_mask.dim() == 3:  # one mask per head
        ws_bytes = _lib.fa_blocksparse_heads_workspace_size(H, N)
        ws = torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
        _check(_lib.fa_fwd_blocksparse_heads(q, k, v, o, lse, B, H, N, d, scale, causal, key_lens, block_mask, ws,
                                             ws_bytes, dt, stream), "fa_fwd_blocksparse_heads")
    else:
        ws_bytes = _lib.fa_blocksparse_workspace_size(N)
        ws = torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
        _check(_lib.fa_fwd_blocksparse(q, k, v, o, lse, B, H, N, d, scale, causal, key_lens, block_mask, ws,
                                       ws_bytes, dt, stream), "fa_fwd_blocksparse")
    return o, lse


def attention_bwd(q, k, v, o, dout, lse, causal=False, softmax_scale=None, key_lens=None, block_mask=None,
                  stream=None):
    """dQ, dK, dV of sum(O * dout) for the attention computed by attention_fwd with the same arguments."""
    import torch
    _require_cuda(q, k, v, o, dout, lse, key_lens, block_mask)
    B, H, N, d = q.shape
    scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(d)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    if block_mask is not None and block_mask.dim() == 3:  # one mask per head
        ws_bytes = _lib.fa_bwd_blocksparse_heads_workspace_size(B, H, N, d)
        ws = torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
        _check(_lib.fa_bwd_blocksparse_heads(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, key_lens,
                                             block_mask, ws, ws_bytes, _dtype_code(q), stream),
               "fa_bwd_blocksparse_heads")
        return dq, dk, dv
    ws_bytes = _lib.fa_bwd_workspace_size(B, H, N, d, block_mask is not None)
    ws = torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
    _check(_lib.fa_bwd(q, k, v, o, dout, lse, dq, dk, dv, B, H, N, d, scale, causal, key_lens, block_mask, ws,
                       ws_bytes, _dtype_code(q), stream), "fa_bwd")
    return dq, dk, dv


_AUTOGRAD_FN = None


def _autograd_fn():
    """torch.autograd.Functions over attention_fwd / attention_bwd and their packed variants (built on first use, so
    importing this package does not import torch)."""
    global _AUTOGRAD_FN
    if _AUTOGRAD_FN is None:
        import torch

        class _Attention(torch.autograd.Function):
            @staticmethod
            def forward(ctx, q, k, v, causal, softmax_scale, key_lens, block_mask):
                o, lse = attention_fwd(q, k, v, causal=causal, softmax_scale=softmax_scale, key_lens=key_lens,
                                       block_mask=block_mask)
                ctx.save_for_backward(q, k, v, o, lse)
                ctx.args = (causal, softmax_scale, key_lens, block_mask)
                return o

            @staticmethod
            def backward(ctx, dout):
                q, k, v, o, lse = ctx.saved_tensors
                causal, softmax_scale, key_lens, block_mask = ctx.args
                dq, dk, dv = attention_bwd(q, k, v, o, dout.contiguous(), lse, causal=causal,
                                           softmax_scale=softmax_scale, key_lens=key_lens, block_mask=block_mask)
                return dq, dk, dv, None, None, None, None

        class _AttentionVarlen(torch.autograd.Function):
            @staticmethod
            def forward(ctx, q, k, v, cu_q, cu_k, max_q, max_k, causal, softmax_scale):
                o, lse = attention_fwd_varlen(q, k, v, cu_q, cu_k, max_q, max_k, causal=causal,
                                              softmax_scale=softmax_scale)
                ctx.save_for_backward(q, k, v, o, lse, cu_q, cu_k)
                ctx.args = (max_q, max_k, causal, softmax_scale)
                return o

            @staticmethod
            def backward(ctx, dout):
                q, k, v, o, lse, cu_q, cu_k = ctx.saved_tensors
                max_q, max_k, causal, softmax_scale = ctx.args
                dq, dk, dv = attention_bwd_varlen(q, k, v, o, dout.contiguous(), lse, cu_q, cu_k, max_q, max_k,
                                                  causal=causal, softmax_scale=softmax_scale)
                return dq, dk, dv, None, None, None, None, None, None

        _AUTOGRAD_FN = (_Attention, _AttentionVarlen)
    return _AUTOGRAD_FN


def attention(q, k, v, causal=False, softmax_scale=None, key_lens=None, block_mask=None):
    """O = exact attention of [B, H, N, d] CUDA tensors (bf16 or fp16), differentiable through torch autograd: the
    forward saves O and the per-row logsumexp, and the backward of the graph calls the library's backward (the
    score and probability tiles are recomputed, never stored).  Arguments as for attention_fwd; q, k, v must be
    contiguous."""
    return _autograd_fn()[0].apply(q, k, v, causal, softmax_scale, key_lens, block_mask)


def attention_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal=False,
                     softmax_scale=None):
    """O of a packed variable-length batch (arguments as for attention_fwd_varlen), differentiable through torch
    autograd like attention()."""
    return _autograd_fn()[1].apply(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal,
                                   softmax_scale)


def blockmask_lists(mask, stream=None):
    """Device CSR/CSC lists of a [nT, nT] uint8 CUDA mask: (row_ptr, col_idx, col_ptr, row_idx), int32, with
    col_idx/row_idx cut to the number of kept tiles."""
    import torch
    _require_cuda(mask)
    nT = mask.shape[0]
    dev = mask.device
    row_ptr = torch.empty(nT + 1, device=dev, dtype=torch.int32)
    col_ptr = torch.empty(nT + 1, device=dev, dtype=torch.int32)
    col_idx = torch.empty(nT * nT, device=dev, dtype=torch.int32)
    row_idx = torch.empty(nT * nT, device=dev, dtype=torch.int32)
    _check(_lib.fa_blockmask_lists(mask.contiguous(), nT, row_ptr, col_idx, col_ptr, row_idx, stream),
           "fa_blockmask_lists")
    nnz = int(row_ptr[-1].item())
    return row_ptr, col_idx[:nnz], col_ptr, row_idx[:nnz]


def last_device_status(stream=None) -> int:
    """Synchronise and return (then clear) the device status word: FA_OK or FA_ERR_TIMEOUT."""
    return _lib.fa_last_device_status(stream)


def attention_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, causal=False,
                         softmax_scale=None, stream=None):
    """O, LSE of a packed variable-length batch: q [total_q, H, d], k, v [total_k, H, d] CUDA tensors (bf16 or
    fp16), cu_seqlens_* int32 CUDA tensors [B+1].  Returns O [total_q, H, d] and LSE [H, total_q] (fp32)."""
    import torch
    _require_cuda(q, k, v, cu_seqlens_q, cu_seqlens_k)
    total_q, H, d = q.shape
    total_k = k.shape[0]
    B = cu_seqlens_q.numel() - 1
    scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty((H, total_q), device=q.device, dtype=torch.float32)
    _check(_lib.fa_fwd_varlen(q, k, v, o, lse, cu_seqlens_q, cu_seqlens_k, B, H, max_seqlen_q, max_seqlen_k, total_q,
                              total_k, d, scale, causal, _dtype_code(q), stream), "fa_fwd_varlen")
    return o, lse


def attention_bwd_varlen(q, k, v, o, dout, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                         causal=False, softmax_scale=None, stream=None):
    """dQ, dK, dV of sum(O * dout) for attention_fwd_varlen with the same arguments."""
    import torch
    _require_cuda(q, k, v, o, dout, lse, cu_seqlens_q, cu_seqlens_k)
    total_q, H, d = q.shape
    total_k = k.shape[0]
    B = cu_seqlens_q.numel() - 1
    scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(d)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws_bytes = _lib.fa_bwd_varlen_workspace_size(B, H, max_seqlen_q, d)
    ws = torch.empty(ws_bytes, device=q.device, dtype=torch.uint8)
    _check(_lib.fa_bwd_varlen(q, k, v, o, dout, lse, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, B, H, max_seqlen_q,
                              max_seqlen_k, total_q, total_k, d, scale, causal, ws, ws_bytes, _dtype_code(q), stream),
           "fa_bwd_varlen")
    return dq, dk, dv


def attention_fwd_splitkv(q, k, v, causal=False, softmax_scale=None, key_lens=None, num_splits=0, stream=None):
    """O, LSE for decoding: q [B, H, Nq, d] are the last Nq positions of sequences whose keys/values k, v are
    [B, H, Nk, d] (key_lens: optional int32 [B], valid cache entries).  Causal aligns the queries with the end of
    the keys.  The keys are split into num_splits ranges (0 = automatic) processed in parallel."""
    import torch
    _require_cuda(q, k, v, key_lens)
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(d)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), device=q.device, dtype=torch.float32)
    ws_bytes = _lib.fa_fwd_splitkv_workspace_size(B, H, Nq, Nk, d, num_splits)
    ws = torch.empty(max(ws_bytes, 1), device=q.device, dtype=torch.uint8)
    _check(_lib.fa_fwd_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, scale, causal, key_lens, num_splits, ws, ws_bytes,
                               _dtype_code(q), stream), "fa_fwd_splitkv")
    return o, lse

