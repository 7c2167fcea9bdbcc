"""Second, independently written fp64 statement of standard attention and its gradients (numpy, dense).

TEST INFRASTRUCTURE ONLY.  Used on tiny problems to cross-check the loop-based C oracle with a differently
structured computation (dense einsum with an explicit boolean mask, scipy's logsumexp).  Definitions as in
attn_oracle.c: FlashAttention review page "Method" / claim C2 (exact standard attention) and claim C7
(gradients of the same function, read as the calculus of softmax attention).
"""
from __future__ import annotations

import numpy as np
from scipy.special import logsumexp


def element_mask(B, N, causal=False, key_lens=None, block_mask=None, tile=128):
    """Boolean [B, N, N] visibility (query row, key column)."""
    r = np.arange(N)[:, None]
    c = np.arange(N)[None, :]
    m = np.ones((B, N, N), dtype=bool)
    if causal:
        m &= (c <= r)[None]
    if key_lens is not None:
        m &= c[None] < np.asarray(key_lens)[:, None, None]
    if block_mask is not None:
        bm = np.asarray(block_mask).astype(bool)
        m &= bm[(r // tile), (c // tile)][None]
    return m


def attn_np(q, k, v, scale, mask):
    """O, LSE, P for [B,H,N,d] inputs and a [B,N,N] boolean mask."""
    s = scale * np.einsum("bhrd,bhcd->bhrc", q, k)
    s = np.where(mask[:, None], s, -np.inf)
    with np.errstate(invalid="ignore"):
        lse = logsumexp(s, axis=-1)
        p = np.where(np.isfinite(lse)[..., None], np.exp(s - lse[..., None]), 0.0)
    o = np.einsum("bhrc,bhcd->bhrd", p, v)
    return o, lse, p


def attn_grads_np(q, k, v, do, scale, mask):
    o, lse, p = attn_np(q, k, v, scale, mask)
    D = np.sum(do * o, axis=-1)
    dv = np.einsum("bhrc,bhrd->bhcd", p, do)
    dp = np.einsum("bhrd,bhcd->bhrc", do, v)
    ds = p * (dp - D[..., None])
    dq = scale * np.einsum("bhrc,bhcd->bhrd", ds, k)
    dk = scale * np.einsum("bhrc,bhrd->bhcd", ds, q)
    return dq, dk, dv, o, lse
