"""Head dims 32 and 96 on the GPU (they run on the 64 / 128 kernels; TMA zero-fills the columns past the tensor's
own) vs the fp64 oracle: dense forward and backward with causal masks and key lengths, a block mask, a packed
variable-length batch and the split-K/V decode path.  Tolerances as for d = 64 / 128: O, LSE max-abs <= 1e-2,
gradients max-abs <= 5e-2 * max |gradient|."""
import numpy as np
import pytest
import torch

import oracle
import exact_io_aware_48_b200 as fa
from exact_io_aware_48_b200 import inputs
from parity import assert_grad_close, assert_lse_close, assert_o_close, f64, gpu_fwd_bwd, log_errors

pytestmark = pytest.mark.gpu

DENSE = [
    # B, H, N, d, dtype, causal, key_lens
    (1, 2, 300, 32, "bf16", True, None),
    (2, 2, 333, 96, "fp16", False, [333, 150]),
    (2, 2, 640, 96, "bf16", True, None),
    (3, 1, 129, 32, "fp16", False, [1, 129, 64]),
]


@pytest.mark.parametrize("B,H,N,d,dtype,causal,kl", DENSE)
def test_headdim_dense_fwd_bwd(B, H, N, d, dtype, causal, kl):
    q, k, v, do = [inputs.gaussian((B, H, N, d), 600 + d + t, dtype) for t in range(4)]
    scale = 1.0 / np.sqrt(d)
    o, lse, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, causal, scale, key_lens=kl)
    kla = None if kl is None else np.array(kl, np.int32)
    rdq, rdk, rdv, ro, rl = oracle.attn_bwd(f64(q), f64(k), f64(v), f64(do), scale, causal=causal, key_lens=kla)
    eo = assert_o_close(o.double().numpy(), ro)
    el = assert_lse_close(lse.numpy(), rl)
    eq = assert_grad_close(dq.double().numpy(), rdq, "dQ")
    ek = assert_grad_close(dk.double().numpy(), rdk, "dK")
    ev = assert_grad_close(dv.double().numpy(), rdv, "dV")
    log_errors(f"headdim B{B} H{H} N{N} d{d} {dtype} causal={causal} kl={kl}", O=eo, LSE=el, dQ=eq, dK=ek, dV=ev)


def test_headdim_96_block_mask():
    B, H, N, d = 1, 2, 512, 96
    q, k, v, do = [inputs.gaussian((B, H, N, d), 640 + t, "bf16") for t in range(4)]
    mask = np.array([[1, 0, 0, 0], [1, 1, 0, 0], [0, 1, 1, 0], [1, 0, 1, 1]], np.uint8)
    o, lse, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, False, 0.1, block_mask=mask)
    rdq, rdk, rdv, ro, rl = oracle.attn_bwd(f64(q), f64(k), f64(v), f64(do), 0.1, block_mask=mask)
    assert_o_close(o.double().numpy(), ro)
    assert_lse_close(lse.numpy(), rl)
    for got, ref, name in ((dq, rdq, "dQ"), (dk, rdk, "dK"), (dv, rdv, "dV")):
        assert_grad_close(got.double().numpy(), ref, name)


def test_headdim_32_packed_and_96_decode():
    lens = [200, 1, 129]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    H, d = 2, 32
    q, k, v, do = [inputs.gaussian((int(cu[-1]), H, d), 650 + t, "bf16") for t in range(4)]
    cud = torch.as_tensor(cu).cuda()
    o, lse = fa.attention_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cud, cud, 200, 200, causal=True)
    dq, dk, dv = fa.attention_bwd_varlen(q.cuda(), k.cuda(), v.cuda(), o, do.cuda(), lse, cud, cud, 200, 200,
                                         causal=True)
    assert fa.last_device_status() == 0
    scale = 1.0 / np.sqrt(d)
    rdq, rdk, rdv, ro, rl = oracle.attn_bwd_varlen(f64(q), f64(k), f64(v), f64(do), cu, cu, scale, causal=True)
    assert_o_close(o.cpu().double().numpy(), ro)
    assert_lse_close(lse.cpu().numpy(), rl)
    for got, ref, name in ((dq, rdq, "dQ"), (dk, rdk, "dK"), (dv, rdv, "dV")):
        assert_grad_close(got.cpu().double().numpy(), ref, name)
    # decode at d = 96: 3 queries against 5000 cached keys with lengths
    B, H, Nq, Nk, d = 2, 2, 3, 5000, 96
    q = inputs.gaussian((B, H, Nq, d), 660, "fp16")
    k = inputs.gaussian((B, H, Nk, d), 661, "fp16")
    v = inputs.gaussian((B, H, Nk, d), 662, "fp16")
    kl = np.array([5000, 777], np.int32)
    o, lse = fa.attention_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=True,
                                      key_lens=torch.as_tensor(kl).cuda())
    assert fa.last_device_status() == 0
    ro, rl = oracle.attn_fwd_decode(f64(q), f64(k), f64(v), 1.0 / np.sqrt(d), causal=True, key_lens=kl)
    assert_o_close(o.cpu().double().numpy(), ro)
    assert_lse_close(lse.cpu().numpy(), rl)
