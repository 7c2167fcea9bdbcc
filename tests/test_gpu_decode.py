"""Split-K/V decode forward on the GPU (fa_fwd_splitkv through the C ABI) vs the fp64 decode oracle.

A few queries per (b, h) against a long key/value cache, the queries aligned with the end of each sequence's keys.
Cases: 1, 4 and 130 queries; caches of 1000-16384 keys with and without per-sequence lengths; causal or not;
d = 64 and 128; bf16 and fp16; automatic and explicit split counts.  Tolerance as for the forward: O and LSE
max-abs <= 1e-2.  The result must not depend on the number of splits beyond rounding.
"""
import numpy as np
import pytest
import torch

import oracle
import exact_io_aware_48_b200 as fa
from exact_io_aware_48_b200 import inputs
from parity import assert_lse_close, assert_o_close, f64, log_errors

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, Nq, Nk, d, dtype, causal, key_lens, splits
    (4, 8, 1, 4096, 128, "bf16", True, None, 0),
    (2, 4, 4, 16384, 128, "bf16", True, [16384, 9000], 0),
    (3, 2, 1, 1000, 64, "fp16", False, [1000, 1, 517], 0),
    (2, 2, 130, 3000, 64, "bf16", True, None, 5),
    (1, 4, 7, 2049, 128, "fp16", False, None, 32),
    (2, 2, 16, 5, 64, "bf16", True, [5, 2], 0),
]


@pytest.mark.parametrize("B,H,Nq,Nk,d,dtype,causal,kl,splits", CASES)
def test_decode_matches_oracle(B, H, Nq, Nk, d, dtype, causal, kl, splits):
    q = inputs.gaussian((B, H, Nq, d), 400 + Nq, dtype)
    k = inputs.gaussian((B, H, Nk, d), 401, dtype)
    v = inputs.gaussian((B, H, Nk, d), 402, dtype)
    scale = 1.0 / np.sqrt(d)
    kld = None if kl is None else torch.as_tensor(np.array(kl, np.int32)).cuda()
    o, lse = fa.attention_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=causal, softmax_scale=scale, key_lens=kld,
                                      num_splits=splits)
    assert fa.last_device_status() == 0
    ro, rl = oracle.attn_fwd_decode(f64(q), f64(k), f64(v), scale, causal=causal,
                                    key_lens=None if kl is None else np.array(kl))
    eo = assert_o_close(o.cpu().double().numpy(), ro)
    el = assert_lse_close(lse.cpu().numpy(), rl)
    log_errors(f"decode B{B} H{H} Nq{Nq} Nk{Nk} d{d} {dtype} causal={causal} kl={kl} splits={splits}", O=eo, LSE=el)


def test_decode_split_count_does_not_change_the_result():
    B, H, Nq, Nk, d = 2, 4, 3, 8192, 128
    q, k, v = [inputs.gaussian(s, 410 + t, "bf16").cuda() for t, s in
               enumerate([(B, H, Nq, d), (B, H, Nk, d), (B, H, Nk, d)])]
    outs = [fa.attention_fwd_splitkv(q, k, v, causal=True, num_splits=n) for n in (1, 3, 32)]
    for o, lse in outs[1:]:
        torch.testing.assert_close(o.float(), outs[0][0].float(), rtol=0, atol=8e-3)
        torch.testing.assert_close(lse, outs[0][1], rtol=0, atol=1e-4)


def test_decode_one_split_equals_the_forward_when_queries_fill_the_cache():
    """Nq = Nk: the decode alignment is the forward's, so one split gives fa_fwd's result."""
    B, H, N, d = 1, 2, 300, 64
    q, k, v = [inputs.gaussian((B, H, N, d), 420 + t, "bf16").cuda() for t in range(3)]
    o, lse = fa.attention_fwd(q, k, v, causal=True)
    od, ld = fa.attention_fwd_splitkv(q, k, v, causal=True, num_splits=1)
    torch.testing.assert_close(od.float(), o.float(), rtol=0, atol=8e-3)
    torch.testing.assert_close(ld, lse, rtol=0, atol=1e-4)
