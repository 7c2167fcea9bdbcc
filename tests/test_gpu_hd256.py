"""Head dim 256 on the GPU vs the fp64 oracle.

Forward (fwd256_kernel, one Q tile per CTA with two score buffers): dense with causal masks, key lengths (0
included), ragged tiles, more units than SMs, shared and per-head block masks, a packed variable-length batch and the
split-K/V decode path.  Backward (bwd256_kernel, two passes over halves of the head dim, every operand streamed in
16 KB boxes): the same mask kinds, packed batches and runs of more units than SMs.  Tolerances as for the other head
dims: O and LSE max-abs <= 1e-2, dQ/dK/dV max-abs <= 5e-2 of the oracle's largest gradient magnitude."""
import numpy as np
import pytest
import torch

import oracle
import exact_io_aware_48_b200 as fa
from exact_io_aware_48_b200 import _lib, inputs
from parity import assert_grad_close, assert_lse_close, assert_o_close, f64, gpu_fwd, gpu_fwd_bwd, log_errors

pytestmark = pytest.mark.gpu

D = 256

DENSE = [
    # B, H, N, dtype, causal, key_lens
    (1, 2, 300, "bf16", True, None),
    (2, 2, 640, "fp16", False, [640, 200]),
    (1, 3, 1000, "bf16", True, None),
    (3, 1, 129, "bf16", False, [1, 129, 0]),
    (2, 16, 1200, "bf16", True, None),        # 320 units: several per CTA
    (2, 64, 256, "fp16", False, [0, 256]),    # runs of units with no visible key
]


@pytest.mark.parametrize("B,H,N,dtype,causal,kl", DENSE)
def test_d256_dense_fwd(B, H, N, dtype, causal, kl):
    q, k, v = [inputs.gaussian((B, H, N, D), 700 + N + t, dtype) for t in range(3)]
    scale = 1.0 / np.sqrt(D)
    o, lse = gpu_fwd(q, k, v, causal, scale, key_lens=kl)
    kla = None if kl is None else np.array(kl, np.int32)
    ro, rl = oracle.attn_fwd(f64(q), f64(k), f64(v), scale, causal=causal, key_lens=kla)
    eo = assert_o_close(o.double().numpy(), ro)
    el = assert_lse_close(lse.numpy(), rl)
    log_errors(f"d256 B{B} H{H} N{N} {dtype} causal={causal} kl={kl}", O=eo, LSE=el)


def test_d256_repeatable():
    q, k, v = [inputs.gaussian((1, 4, 900, D), 760 + t, "bf16") for t in range(3)]
    a = gpu_fwd(q, k, v, True, 0.0625)
    b = gpu_fwd(q, k, v, True, 0.0625)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_d256_block_masks():
    B, H, N = 1, 2, 640
    q, k, v = [inputs.gaussian((B, H, N, D), 770 + t, "bf16") for t in range(3)]
    nT = 5
    shared = np.tril(np.ones((nT, nT), np.uint8))
    shared[3, 1] = 0
    shared[4, 4] = 0
    o, lse = gpu_fwd(q, k, v, False, 0.07, block_mask=shared)
    ro, rl = oracle.attn_fwd(f64(q), f64(k), f64(v), 0.07, block_mask=shared)
    assert_o_close(o.double().numpy(), ro)
    assert_lse_close(lse.numpy(), rl)
    heads = np.stack([shared, (np.arange(nT)[:, None] + np.arange(nT)[None, :]) % 2 == 0]).astype(np.uint8)
    o, lse = gpu_fwd(q, k, v, True, 0.07, block_mask=heads)
    for h in range(H):
        ro, rl = oracle.attn_fwd(f64(q[:, h:h + 1]), f64(k[:, h:h + 1]), f64(v[:, h:h + 1]), 0.07, causal=True,
                                 block_mask=heads[h])
        assert_o_close(o[:, h:h + 1].double().numpy(), ro)
        assert_lse_close(lse[:, h:h + 1].numpy(), rl)


def test_d256_packed_varlen():
    lens = [200, 1, 129, 384]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    H = 2
    q, k, v = [inputs.gaussian((int(cu[-1]), H, D), 780 + t, "bf16") for t in range(3)]
    cud = torch.as_tensor(cu).cuda()
    o, lse = fa.attention_fwd_varlen(q.cuda(), k.cuda(), v.cuda(), cud, cud, 384, 384, causal=True)
    assert fa.last_device_status() == 0
    ro, rl = oracle.attn_fwd_varlen(f64(q), f64(k), f64(v), cu, cu, 1.0 / np.sqrt(D), causal=True)
    eo = assert_o_close(o.cpu().double().numpy(), ro)
    el = assert_lse_close(lse.cpu().numpy(), rl)
    log_errors("d256 varlen", O=eo, LSE=el)


@pytest.mark.parametrize("splits", [0, 3])
def test_d256_decode(splits):
    B, H, Nq, Nk = 2, 2, 3, 5000
    q = inputs.gaussian((B, H, Nq, D), 790, "fp16")
    k = inputs.gaussian((B, H, Nk, D), 791, "fp16")
    v = inputs.gaussian((B, H, Nk, D), 792, "fp16")
    kl = np.array([5000, 777], np.int32)
    o, lse = fa.attention_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=True,
                                      key_lens=torch.as_tensor(kl).cuda(), num_splits=splits)
    assert fa.last_device_status() == 0
    ro, rl = oracle.attn_fwd_decode(f64(q), f64(k), f64(v), 1.0 / np.sqrt(D), causal=True, key_lens=kl)
    eo = assert_o_close(o.cpu().double().numpy(), ro)
    el = assert_lse_close(lse.cpu().numpy(), rl)
    log_errors(f"d256 decode splits={splits}", O=eo, LSE=el)


BWD = [
    # B, H, N, dtype, causal, key_lens
    (1, 2, 128, "bf16", False, None),
    (1, 2, 300, "bf16", True, None),
    (2, 2, 640, "fp16", False, [640, 200]),
    (3, 1, 129, "bf16", True, [1, 129, 0]),
    (2, 8, 1200, "bf16", True, None),          # 320 units (key tile x half x head): several per CTA
    (2, 16, 256, "fp16", False, [0, 256]),     # runs of units with no visible query
]


@pytest.mark.parametrize("B,H,N,dtype,causal,kl", BWD)
def test_d256_backward(B, H, N, dtype, causal, kl):
    q, k, v, do = [inputs.gaussian((B, H, N, D), 720 + N + t, dtype) for t in range(4)]
    scale = 1.0 / np.sqrt(D)
    kla = None if kl is None else np.array(kl, np.int32)
    o, lse, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, causal, scale, key_lens=kla)
    rq, rk, rv, ro, rl = oracle.attn_bwd(f64(q), f64(k), f64(v), f64(do), scale, causal=causal, key_lens=kla)
    eo = assert_o_close(o.double().numpy(), ro)
    el = assert_lse_close(lse.numpy(), rl)
    e = [assert_grad_close(g.double().numpy(), r, n) for g, r, n in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV"))]
    log_errors(f"d256 bwd B{B} H{H} N{N} {dtype} causal={causal} kl={kl}", O=eo, LSE=el, dQ=e[0], dK=e[1], dV=e[2])
    if kl is not None:  # keys beyond the length get exactly zero gradient
        for b in range(B):
            assert torch.all(dk[b, :, kl[b]:] == 0) and torch.all(dv[b, :, kl[b]:] == 0)


def test_d256_backward_block_masks():
    B, H, N = 1, 2, 640
    q, k, v, do = [inputs.gaussian((B, H, N, D), 740 + t, "bf16") for t in range(4)]
    nT = 5
    shared = np.tril(np.ones((nT, nT), np.uint8))
    shared[3, 1] = 0
    shared[4, 4] = 0
    o, lse, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, True, 0.07, block_mask=shared)
    rq, rk, rv, ro, rl = oracle.attn_bwd(f64(q), f64(k), f64(v), f64(do), 0.07, causal=True, block_mask=shared)
    for g, r, n in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV")):
        assert_grad_close(g.double().numpy(), r, n)
    heads = np.stack([shared, (np.arange(nT)[:, None] + np.arange(nT)[None, :]) % 2 == 0]).astype(np.uint8)
    o, lse, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, False, 0.07, block_mask=heads)
    rq, rk, rv, ro, rl = oracle.attn_bwd_head_masks(f64(q), f64(k), f64(v), f64(do), 0.07, heads)
    for g, r, n in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV")):
        assert_grad_close(g.double().numpy(), r, n)


def test_d256_backward_packed_varlen():
    lens = [200, 1, 129, 384]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    H = 2
    q, k, v, do = [inputs.gaussian((int(cu[-1]), H, D), 750 + t, "bf16") for t in range(4)]
    cud = torch.as_tensor(cu).cuda()
    qd, kd, vd, dod = (t.cuda() for t in (q, k, v, do))
    o, lse = fa.attention_fwd_varlen(qd, kd, vd, cud, cud, 384, 384, causal=True)
    dq, dk, dv = fa.attention_bwd_varlen(qd, kd, vd, o, dod, lse, cud, cud, 384, 384, causal=True)
    assert fa.last_device_status() == 0
    rq, rk, rv, ro, rl = oracle.attn_bwd_varlen(f64(q), f64(k), f64(v), f64(do), cu, cu, 1.0 / np.sqrt(D),
                                                causal=True)
    e = [assert_grad_close(g.cpu().double().numpy(), r, n) for g, r, n in ((dq, rq, "dQ"), (dk, rk, "dK"),
                                                                           (dv, rv, "dV"))]
    log_errors("d256 bwd varlen", dQ=e[0], dK=e[1], dV=e[2])


def test_d256_backward_repeatable():
    # every gradient is a sum in a fixed order except dQ (fp32 reductions in L2 in arrival order)
    q, k, v, do = [inputs.gaussian((1, 4, 900, D), 760 + t, "bf16") for t in range(4)]
    a = gpu_fwd_bwd(q, k, v, do, True, 0.0625)
    b = gpu_fwd_bwd(q, k, v, do, True, 0.0625)
    for x, y in zip(a[:2] + a[3:], b[:2] + b[3:]):
        assert torch.equal(x, y)
    assert torch.allclose(a[2].float(), b[2].float(), rtol=0, atol=2e-2 * float(a[2].float().abs().max()))


def test_d256_workload_sampled():
    # B1 H16 N8192 d256 causal at full size: O, LSE and dQ of 1024 seeded rows, dK and dV of 128 seeded keys in each
    # of two seeded heads against the oracle; each tolerance scale is the oracle's largest sampled magnitude
    from parity import sampled_keys
    w = inputs.workloads()["lc8k_d256"]
    q, k, v, do = w.tensors()
    o, lse, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, w.causal, w.scale)
    qf, kf, vf, dof = f64(q), f64(k), f64(v), f64(do)
    sb, sr = inputs.sample_rows(w.seed + 600, w.B * w.H, w.N, 1024)
    ro, rl = oracle.attn_fwd_rows(qf, kf, vf, w.scale, sb, sr, causal=w.causal)
    eo = assert_o_close(o.reshape(-1, w.N, D)[sb, sr].double().numpy(), ro)
    el = assert_lse_close(lse.reshape(-1, w.N)[sb, sr].numpy(), rl)
    rq = oracle.attn_bwd_rows(qf, kf, vf, dof, w.scale, sb, sr, causal=w.causal)
    kb, kc = sampled_keys(w.seed + 700, w.B * w.H, w.N, heads=2, per_head=128)
    rk, rv = oracle.attn_bwd_keys(qf, kf, vf, dof, w.scale, kb, kc, causal=w.causal)
    e_q = assert_grad_close(dq.reshape(-1, w.N, D)[sb, sr].double().numpy(), rq, "dQ")
    e_k = assert_grad_close(dk.reshape(-1, w.N, D)[kb, kc].double().numpy(), rk, "dK")
    e_v = assert_grad_close(dv.reshape(-1, w.N, D)[kb, kc].double().numpy(), rv, "dV")
    log_errors("d256 lc8k sampled", O=eo, LSE=el, dQ=e_q, dK=e_k, dV=e_v)
