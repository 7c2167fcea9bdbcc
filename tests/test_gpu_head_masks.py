"""Per-head block masks on the GPU (fa_fwd_blocksparse_heads / fa_bwd_blocksparse_heads through the C ABI) vs the
fp64 oracle: each head its own 128x128 tile mask (dense, band, random, one with an empty row), causal or not,
d = 64 and 128.  Tolerances as for the shared-mask tests."""
import numpy as np
import pytest

import oracle
from exact_io_aware_48_b200 import inputs
from parity import assert_grad_close, assert_lse_close, assert_o_close, f64, gpu_fwd_bwd, log_errors

pytestmark = pytest.mark.gpu


def masks(H, nT, seed):
    rng = np.random.default_rng(seed)
    out = []
    for h in range(H):
        if h % 4 == 0:
            m = np.ones((nT, nT), np.uint8)
        elif h % 4 == 1:
            m = inputs.band_mask(nT).astype(np.uint8)
        elif h % 4 == 2:
            m = (rng.random((nT, nT)) < 0.35).astype(np.uint8)
        else:
            m = np.tril(np.ones((nT, nT), np.uint8))
            m[1] = 0  # a row of tiles with nothing kept
        out.append(m)
    return np.stack(out)


@pytest.mark.parametrize("B,H,N,d,dtype,causal", [(1, 4, 600, 64, "bf16", False), (2, 4, 512, 128, "fp16", True),
                                                  (1, 3, 1000, 128, "bf16", False)])
def test_head_masks_fwd_bwd(B, H, N, d, dtype, causal):
    nT = -(-N // 128)
    m = masks(H, nT, 700 + N)
    q, k, v, do = [inputs.gaussian((B, H, N, d), 710 + t, dtype) for t in range(4)]
    scale = 1.0 / np.sqrt(d)
    o, lse, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, causal, scale, block_mask=m)
    rdq, rdk, rdv, ro, rl = oracle.attn_bwd_head_masks(f64(q), f64(k), f64(v), f64(do), scale, m, causal=causal)
    eo = assert_o_close(o.double().numpy(), ro)
    el = assert_lse_close(lse.numpy(), rl)
    eq = assert_grad_close(dq.double().numpy(), rdq, "dQ")
    ek = assert_grad_close(dk.double().numpy(), rdk, "dK")
    ev = assert_grad_close(dv.double().numpy(), rdv, "dV")
    log_errors(f"head masks B{B} H{H} N{N} d{d} {dtype} causal={causal}", O=eo, LSE=el, dQ=eq, dK=ek, dV=ev)
