"""fa_bwd_noalloc: the backward for callers that cannot allocate device memory while they run.

Who needs it: code hosted inside a framework or plugin host that owns all GPU memory and forbids allocation during
execution, and latency-sensitive loops that cannot pay for cudaMalloc's implicit device synchronisation.  Such a
caller passes its own inputs and outputs; the library takes the backward's scratch from a fixed 32 MiB device array.

These tests call the entry point through the C ABI and check, on two calls in a row (the array keeps the previous
call's contents), that its gradients equal those of fa_bwd with a caller-provided workspace within the gradient
tolerance used everywhere else (max-abs <= 5e-2 * max |gradient|).  The file sorts last so that a run stopping at
the first failure has already run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import exact_io_aware_48_b200 as fa
from exact_io_aware_48_b200 import _lib, inputs
from parity import assert_grad_close

pytestmark = pytest.mark.gpu


def _inputs(B, H, N, d, dtype, seed):
    q, k, v, do = [inputs.gaussian((B, H, N, d), seed * 10 + t, dtype).cuda() for t in range(4)]
    return q, k, v, do


@pytest.mark.parametrize("B,H,N,d,dtype,causal", [
    (1, 2, 256, 64, "bf16", False),   # the tiny workload shape
    (2, 3, 333, 128, "fp16", True),   # ragged tail, causal, d = 128
])
def test_noalloc_matches_workspace_backward_twice(B, H, N, d, dtype, causal):
    q, k, v, do = _inputs(B, H, N, d, dtype, N + d)
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.attention_fwd(q, k, v, causal=causal, softmax_scale=scale)
    ref = fa.attention_bwd(q, k, v, o, do, lse, causal=causal, softmax_scale=scale)
    dt = _lib.FA_BF16 if dtype == "bf16" else _lib.FA_FP16
    for _ in range(2):
        dq, dk, dv = (torch.full_like(q, float("nan")) for _ in range(3))
        rc = _lib.fa_bwd_noalloc(q, k, v, o, do, lse, dq, dk, dv, B, H, N, d, scale, causal, None, None, dt)
        assert rc == _lib.FA_OK, _lib.fa_status_string(rc)
        assert fa.last_device_status() == _lib.FA_OK
        for got, want, name in zip((dq, dk, dv), ref, ("dQ", "dK", "dV")):
            assert_grad_close(got.double().cpu().numpy(), want.double().cpu().numpy(), name)


def test_noalloc_rejects_problems_larger_than_the_array():
    # B*H = 512, N = 1024, d = 128 needs ~260 MiB of scratch: refused on the host, nothing launched
    need = _lib.fa_bwd_workspace_size(8, 64, 1024, 128, False)
    assert need > _lib.FA_NOALLOC_SCRATCH_BYTES
    x = torch.empty(16, device="cuda", dtype=torch.bfloat16)
    rc = _lib.fa_bwd_noalloc(x, x, x, x, x, x, x, x, x, 8, 64, 1024, 128, 0.1, 0, None, None, _lib.FA_BF16)
    assert rc == _lib.FA_ERR_WORKSPACE
