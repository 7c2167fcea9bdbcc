"""fa.attention through torch autograd: the gradients that loss.backward() leaves in q, k, v are those of the
library's backward called directly, and they match the fp64 oracle at the usual tolerances (O max-abs <= 1e-2;
dQ, dK, dV max-abs <= 5e-2 of the oracle's largest magnitude).  The upstream gradient is the 16-bit dO that autograd
hands the attention node, and the oracle gets exactly those values."""
import math

import numpy as np
import pytest
import torch

import oracle
import exact_io_aware_48_b200 as fa
from exact_io_aware_48_b200 import inputs
from parity import assert_grad_close, assert_o_close, f64

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, N, d, dtype, causal, key_lens, block-mask density
    (1, 2, 300, 64, "bf16", True, None, None),
    (2, 2, 257, 128, "fp16", False, [257, 40], None),
    (1, 2, 640, 64, "bf16", False, None, 0.5),
]


@pytest.mark.parametrize("B,H,N,d,dtype,causal,kl,density", CASES)
def test_autograd_matches_direct_backward_and_oracle(B, H, N, d, dtype, causal, kl, density):
    q, k, v = [inputs.gaussian((B, H, N, d), 600 + t, dtype).cuda().requires_grad_() for t in range(3)]
    g = inputs.gaussian((B, H, N, d), 610, "bf16").cuda().float()  # weights of the loss
    klt = None if kl is None else torch.tensor(kl, dtype=torch.int32, device="cuda")
    mask = None
    if density is not None:
        nT = (N + 127) // 128
        mask = (np.random.default_rng(11).random((nT, nT)) < density).astype(np.uint8)
        np.fill_diagonal(mask, 1)
    bm = None if mask is None else torch.as_tensor(mask).cuda()

    o = fa.attention(q, k, v, causal=causal, key_lens=klt, block_mask=bm)
    (o.float() * g).sum().backward()
    assert fa.last_device_status() == 0
    do = g.to(o.dtype)  # the gradient autograd passes to the attention node (cast to O's dtype)

    with torch.no_grad():
        o2, lse = fa.attention_fwd(q, k, v, causal=causal, key_lens=klt, block_mask=bm)
        dq, dk, dv = fa.attention_bwd(q, k, v, o2, do, lse, causal=causal, key_lens=klt, block_mask=bm)
    assert torch.equal(o.detach(), o2)
    assert torch.equal(k.grad, dk) and torch.equal(v.grad, dv)
    ulp = 2.0 ** (-7 if dtype == "bf16" else -10)
    assert float((q.grad.float() - dq.float()).abs().max()) <= ulp * max(float(dq.float().abs().max()), 1e-3)

    scale = 1.0 / math.sqrt(d)
    rq, rk, rv, ro, _ = oracle.attn_bwd(f64(q.detach().cpu()), f64(k.detach().cpu()), f64(v.detach().cpu()),
                                        f64(do.cpu()), scale, causal=causal,
                                        key_lens=None if kl is None else np.asarray(kl, np.int32), block_mask=mask)
    assert_o_close(o.detach().cpu().double().numpy(), ro)
    for got, ref, name in ((q.grad, rq, "dQ"), (k.grad, rk, "dK"), (v.grad, rv, "dV")):
        assert_grad_close(got.cpu().double().numpy(), ref, name)


def test_autograd_varlen_matches_oracle():
    lens = [130, 1, 257]
    cq = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    H, d, total = 2, 64, int(cq[-1])
    q, k, v = [inputs.gaussian((total, H, d), 620 + t, "bf16").cuda().requires_grad_() for t in range(3)]
    g = inputs.gaussian((total, H, d), 630, "bf16").cuda().float()
    cqd = torch.as_tensor(cq).cuda()
    o = fa.attention_varlen(q, k, v, cqd, cqd, max(lens), max(lens), causal=True)
    (o.float() * g).sum().backward()
    assert fa.last_device_status() == 0
    do = g.to(o.dtype)
    scale = 1.0 / math.sqrt(d)
    rq, rk, rv, ro, _ = oracle.attn_bwd_varlen(f64(q.detach().cpu()), f64(k.detach().cpu()), f64(v.detach().cpu()),
                                               f64(do.cpu()), cq, cq, scale, causal=True)
    assert_o_close(o.detach().cpu().double().numpy(), ro)
    for got, ref, name in ((q.grad, rq, "dQ"), (k.grad, rk, "dK"), (v.grad, rv, "dV")):
        assert_grad_close(got.cpu().double().numpy(), ref, name)

