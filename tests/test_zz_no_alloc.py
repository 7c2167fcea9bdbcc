"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory while they run.

Who needs it: code hosted inside a framework or plugin host that owns all GPU memory and forbids allocation during
execution, and latency-sensitive loops that cannot pay for cudaMalloc's implicit device synchronisation.  Such a
caller passes its own inputs and outputs; the library takes the backward's scratch from a fixed 32 MiB device array.

These tests call the entry point through the C ABI and check, on two calls in a row (the array keeps the previous
call's contents), that its gradients equal those of fa_bwd with a caller-provided workspace within the gradient
tolerance used everywhere else (max-abs <= 5e-2 * max |gradient|), and that both match the fp64 oracle within that
tolerance.  The cases cover a block mask with key lengths (the tile lists sit inside the fixed array) and a large
call followed by a smaller one of another shape (the second must not see the first one's leftovers).  The file sorts
last so that a run stopping at the first failure has already run every other test; it also passes on its own in a
fresh process.
"""
import numpy as np
import pytest
import torch

import oracle
import exact_io_aware_48_b200 as fa
from exact_io_aware_48_b200 import _lib, inputs
from parity import assert_grad_close, f64

pytestmark = pytest.mark.gpu


def _case(B, H, N, d, dtype, seed):
    return [inputs.gaussian((B, H, N, d), seed * 10 + t, dtype) for t in range(4)]


def _run_and_check(B, H, N, d, dtype, causal, kl=None, mask=None, seed=0, calls=2):
    q, k, v, do = _case(B, H, N, d, dtype, seed)
    scale = 1.0 / np.sqrt(d)
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    kld = None if kl is None else torch.as_tensor(kl, dtype=torch.int32).cuda()
    mkd = None if mask is None else torch.as_tensor(mask, dtype=torch.uint8).cuda()
    o, lse = fa.attention_fwd(qd, kd, vd, causal=causal, softmax_scale=scale, key_lens=kld, block_mask=mkd)
    ref = fa.attention_bwd(qd, kd, vd, o, dod, lse, causal=causal, softmax_scale=scale, key_lens=kld, block_mask=mkd)
    orc = oracle.attn_bwd(f64(q), f64(k), f64(v), f64(do), scale, causal=causal,
                          key_lens=None if kl is None else np.asarray(kl, np.int32), block_mask=mask, tile=128)
    dt = _lib.FA_BF16 if dtype == "bf16" else _lib.FA_FP16
    for _ in range(calls):
        dq, dk, dv = (torch.full_like(qd, float("nan")) for _ in range(3))
        rc = _lib.fa_bwd_noalloc(qd, kd, vd, o, dod, lse, dq, dk, dv, B, H, N, d, scale, causal, kld, mkd, dt)
        assert rc == _lib.FA_OK, _lib.fa_status_string(rc)
        assert fa.last_device_status() == _lib.FA_OK
        for got, want, r, name in zip((dq, dk, dv), ref, orc[:3], ("dQ", "dK", "dV")):
            g = got.double().cpu().numpy()
            assert_grad_close(g, want.double().cpu().numpy(), name + " vs fa_bwd")
            assert_grad_close(g, r, name + " vs oracle")


@pytest.mark.parametrize("B,H,N,d,dtype,causal", [
    (1, 2, 256, 64, "bf16", False),   # the tiny workload shape
    (2, 3, 333, 128, "fp16", True),   # ragged tail, causal, d = 128
])
def test_noalloc_matches_workspace_backward_twice(B, H, N, d, dtype, causal):
    _run_and_check(B, H, N, d, dtype, causal, seed=N + d)


def test_noalloc_block_mask_and_key_lens():
    N = 700
    nT = -(-N // 128)
    mask = (np.random.default_rng(11).random((nT, nT)) < 0.5).astype(np.uint8)
    mask[np.arange(nT), np.arange(nT)] = 1
    _run_and_check(2, 2, N, 64, "bf16", True, kl=[700, 300], mask=mask, seed=5)


def test_noalloc_large_then_small():
    # a call near the GPT-2 shape's scratch size (B4 H12 N1024 d64: ~12.4 MiB), then a smaller call of another
    # shape, head dim and mask: the second call must rebuild everything it reads from the shared array
    _run_and_check(4, 12, 1024, 64, "bf16", True, seed=21, calls=1)
    nT = 3
    mask = np.tril(np.ones((nT, nT), np.uint8))
    _run_and_check(1, 3, 300, 128, "fp16", False, kl=[257], mask=mask, seed=22, calls=2)


def test_noalloc_rejects_problems_larger_than_the_array():
    # B*H = 512, N = 1024, d = 128 needs ~260 MiB of scratch: refused on the host, nothing launched
    need = _lib.fa_bwd_workspace_size(8, 64, 1024, 128, False)
    assert need > _lib.FA_NOALLOC_SCRATCH_BYTES
    x = torch.empty(16, device="cuda", dtype=torch.bfloat16)
    rc = _lib.fa_bwd_noalloc(x, x, x, x, x, x, x, x, x, 8, 64, 1024, 128, 0.1, 0, None, None, _lib.FA_BF16)
    assert rc == _lib.FA_ERR_WORKSPACE
