"""Forward parity on the GPU: libfa.so through the C ABI vs the fp64 oracle, element by element.

Tolerance: O and LSE max-abs error <= 1e-2 (bf16/fp16 inputs, fp32 accumulation).  Sizes span several 128-row tiles
and ragged tails; the workload shapes run at full size (full oracle where it finishes in seconds, else 256 seeded
sampled query rows).
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_48_b200 import inputs
from parity import assert_lse_close, assert_o_close, f64, gpu_fwd, log_errors

pytestmark = pytest.mark.gpu


def make(B, H, N, d, dtype, seed):
    shape = (B, H, N, d)
    return [inputs.gaussian(shape, seed * 10 + t, dtype) for t in range(3)]


SMALL = [
    # B, H, N, d, dtype, causal, key_lens
    (1, 2, 128, 64, "bf16", False, None),
    (1, 2, 256, 64, "bf16", True, None),
    (2, 3, 1, 64, "bf16", False, None),
    (2, 2, 5, 128, "fp16", True, None),
    (1, 2, 127, 64, "bf16", True, None),
    (2, 2, 129, 128, "bf16", False, None),
    (1, 3, 300, 64, "fp16", False, None),
    (2, 2, 333, 128, "bf16", True, None),
    (2, 2, 700, 64, "bf16", True, None),
    (3, 2, 640, 128, "fp16", False, [640, 1, 257]),
    (3, 2, 500, 64, "bf16", True, [500, 129, 3]),
    (2, 1, 384, 128, "bf16", False, [0, 384]),
]


@pytest.mark.parametrize("B,H,N,d,dtype,causal,kl", SMALL)
def test_fwd_small_cases(B, H, N, d, dtype, causal, kl):
    q, k, v = make(B, H, N, d, dtype, N + d)
    scale = 1.0 / np.sqrt(d)
    o, lse = gpu_fwd(q, k, v, causal, scale, key_lens=kl)
    o_ref, lse_ref = oracle.attn_fwd(f64(q), f64(k), f64(v), scale, causal=causal,
                                     key_lens=None if kl is None else np.array(kl, np.int32))
    eo = assert_o_close(o.double().numpy(), o_ref)
    el = assert_lse_close(lse.numpy(), lse_ref)
    log_errors(f"fwd_small B{B} H{H} N{N} d{d} {dtype} causal={causal} kl={kl}", o=eo, lse=el)


def test_fwd_large_scores_rescale_path():
    # scaled-up inputs make the running max move often (exercises the lazy O rescale)
    B, H, N, d = 1, 2, 1024, 64
    q, k, v = make(B, H, N, d, "bf16", 5)
    q = (q.float() * 4).to(torch.bfloat16)
    scale = 1.0 / np.sqrt(d)
    for causal in (False, True):
        o, lse = gpu_fwd(q, k, v, causal, scale)
        o_ref, lse_ref = oracle.attn_fwd(f64(q), f64(k), f64(v), scale, causal=causal)
        eo = assert_o_close(o.double().numpy(), o_ref)
        el = assert_lse_close(lse.numpy(), lse_ref)
        log_errors(f"fwd_peaky causal={causal}", o=eo, lse=el)


@pytest.mark.parametrize("name", ["tiny", "gpt2", "bert"])
def test_fwd_workloads_full(name):
    w = inputs.workloads()[name]
    q, k, v, _ = w.tensors()
    kl = w.key_lens_array()
    o, lse = gpu_fwd(q, k, v, w.causal, w.scale, key_lens=kl)
    o_ref, lse_ref = oracle.attn_fwd(f64(q), f64(k), f64(v), w.scale, causal=w.causal, key_lens=kl)
    eo = assert_o_close(o.double().numpy(), o_ref)
    el = assert_lse_close(lse.numpy(), lse_ref)
    log_errors(f"fwd_{name}", o=eo, lse=el)


@pytest.mark.parametrize("name", ["lc4k", "lc8k", "lc16k"])
def test_fwd_long_context_sampled_rows(name):
    w = inputs.workloads()[name]
    q, k, v, _ = w.tensors()
    o, lse = gpu_fwd(q, k, v, w.causal, w.scale)
    sb, sr = inputs.sample_rows(w.seed + 500, w.B * w.H, w.N, 256)
    o_ref, lse_ref = oracle.attn_fwd_rows(f64(q), f64(k), f64(v), w.scale, sb, sr, causal=w.causal)
    o_s = o.reshape(-1, w.N, w.d)[sb, sr].double().numpy()
    lse_s = lse.reshape(-1, w.N)[sb, sr].numpy()
    eo = assert_o_close(o_s, o_ref)
    el = assert_lse_close(lse_s, lse_ref)
    log_errors(f"fwd_{name}_sampled", o=eo, lse=el)
    # properties that hold at any size: finite everywhere, LSE >= the diagonal score (causal), O rows bounded by V
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


@pytest.fixture
def one_tile_ctas():
    from exact_io_aware_48_b200 import _lib
    assert _lib.fa_set_fwd_tiles_per_cta(1) == 0
    yield
    assert _lib.fa_set_fwd_tiles_per_cta(0) == 0


@pytest.mark.parametrize("B,H,N,d,dtype,causal,kl", [SMALL[i] for i in (1, 3, 5, 7, 9, 10, 11)])
def test_fwd_one_tile_ctas(one_tile_ctas, B, H, N, d, dtype, causal, kl):
    # the variant with one Q tile per CTA (two CTAs per SM) computes the same attention
    q, k, v = make(B, H, N, d, dtype, N + d)
    scale = 1.0 / np.sqrt(d)
    o, lse = gpu_fwd(q, k, v, causal, scale, key_lens=kl)
    o_ref, lse_ref = oracle.attn_fwd(f64(q), f64(k), f64(v), scale, causal=causal,
                                     key_lens=None if kl is None else np.array(kl, np.int32))
    eo = assert_o_close(o.double().numpy(), o_ref)
    el = assert_lse_close(lse.numpy(), lse_ref)
    log_errors(f"fwd_1tile B{B} H{H} N{N} d{d} {dtype} causal={causal} kl={kl}", o=eo, lse=el)


def test_fwd_one_tile_ctas_blocksparse(one_tile_ctas):
    B, H, N, d = 1, 2, 896, 128
    q, k, v = make(B, H, N, d, "bf16", 77)
    nT = 7
    mask = (np.random.default_rng(5).random((nT, nT)) < 0.5).astype(np.uint8)
    mask[np.arange(nT), np.arange(nT)] = 1
    scale = 1.0 / np.sqrt(d)
    o, lse = gpu_fwd(q, k, v, True, scale, block_mask=mask)
    o_ref, lse_ref = oracle.attn_fwd(f64(q), f64(k), f64(v), scale, causal=True, block_mask=mask, tile=128)
    assert_o_close(o.double().numpy(), o_ref)
    assert_lse_close(lse.numpy(), lse_ref)
