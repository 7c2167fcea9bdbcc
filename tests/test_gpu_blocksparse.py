"""Block-sparse path on the GPU: device tile lists equal the CPU oracle's exactly; forward and backward under a
128x128 tile mask match the fp64 oracle (same tolerances as the dense path)."""
import numpy as np
import pytest
import torch

import oracle
import exact_io_aware_48_b200 as fa
from exact_io_aware_48_b200 import inputs
from parity import (assert_grad_close, assert_lse_close, assert_o_close, f64, gpu_fwd, gpu_fwd_bwd, log_errors,
                    sampled_keys)

pytestmark = pytest.mark.gpu


def lists_equal(mask):
    rp, ci, cp, ri = fa.blockmask_lists(torch.as_tensor(mask, dtype=torch.uint8).cuda())
    erp, eci = oracle.blockmask_csr(mask)
    ecp, eri = oracle.blockmask_csc(mask)
    assert np.array_equal(rp.cpu().numpy(), erp) and np.array_equal(ci.cpu().numpy(), eci)
    assert np.array_equal(cp.cpu().numpy(), ecp) and np.array_equal(ri.cpu().numpy(), eri)


def test_lists_workload_mask_exact():
    w = inputs.workloads()["bs64k"]
    m = w.block_mask()
    lists_equal(m)
    assert 10000 < int(m.sum()) < 12500


@pytest.mark.parametrize("nT", [1, 2, 7, 64, 333, 1500])
def test_lists_random_masks_exact(nT):
    rng = np.random.default_rng(nT)
    for p in (0.0, 0.03, 0.5, 1.0):
        lists_equal((rng.random((nT, nT)) < p).astype(np.uint8))


CASES = [
    # N, d, dtype, causal, key_lens, density
    (640, 64, "fp16", False, None, 0.4),
    (640, 128, "bf16", True, None, 0.5),
    (1000, 64, "bf16", False, [1000, 300], 0.3),
    (896, 128, "fp16", True, [896, 500], 0.6),
    (384, 64, "bf16", False, None, 0.0),
]


@pytest.mark.parametrize("N,d,dtype,causal,kl,density", CASES)
def test_blocksparse_fwd_bwd_small(N, d, dtype, causal, kl, density):
    B = 1 if kl is None else len(kl)
    H = 2
    q, k, v, do = [inputs.gaussian((B, H, N, d), 40 + t, dtype) for t in range(4)]
    nT = -(-N // 128)
    mask = (np.random.default_rng(N + d).random((nT, nT)) < density).astype(np.uint8)
    if density > 0:
        mask[np.arange(nT), np.arange(nT)] = 1
        mask[nT - 1, 0] = 1
    kla = None if kl is None else np.array(kl, np.int32)
    scale = 1.0 / np.sqrt(d)
    o, lse, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, causal, scale, key_lens=kla, block_mask=mask)
    rq, rk, rv, ro, rl = oracle.attn_bwd(f64(q), f64(k), f64(v), f64(do), scale, causal=causal, key_lens=kla,
                                         block_mask=mask, tile=128)
    eo = assert_o_close(o.double().numpy(), ro)
    el = assert_lse_close(lse.numpy(), rl)
    e = [assert_grad_close(g.double().numpy(), r, n) for g, r, n in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV"))]
    log_errors(f"bs_small N{N} d{d} {dtype} causal={causal} kl={kl} p={density}", o=eo, lse=el, dq=e[0], dk=e[1],
               dv=e[2])


def test_blocksparse_workload_sampled():
    # B1 H8 N65536 d64 fp16 under the band + butterfly + 2% random tile mask.  The oracle computes sampled elements:
    # O, LSE and dQ of 1024 seeded (head, query) rows, dK and dV of 256 seeded keys in each of two seeded heads.
    # Each tolerance scale is the largest magnitude among the oracle's sampled values (never the GPU's).
    w = inputs.workloads()["bs64k"]
    q, k, v, do = w.tensors()
    mask = w.block_mask()
    o, lse, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, w.causal, w.scale, block_mask=mask)
    qf, kf, vf, dof = f64(q), f64(k), f64(v), f64(do)
    sb, sr = inputs.sample_rows(w.seed + 800, w.B * w.H, w.N, 1024)
    ro, rl = oracle.attn_fwd_rows(qf, kf, vf, w.scale, sb, sr, block_mask=mask, tile=128)
    eo = assert_o_close(o.reshape(-1, w.N, w.d)[sb, sr].double().numpy(), ro)
    el = assert_lse_close(lse.reshape(-1, w.N)[sb, sr].numpy(), rl)
    rq = oracle.attn_bwd_rows(qf, kf, vf, dof, w.scale, sb, sr, block_mask=mask, tile=128)
    eq = assert_grad_close(dq.reshape(-1, w.N, w.d)[sb, sr].double().numpy(), rq, "dQ")
    kb, kc = sampled_keys(w.seed + 900, w.B * w.H, w.N, heads=2, per_head=256)
    rk, rv = oracle.attn_bwd_keys(qf, kf, vf, dof, w.scale, kb, kc, block_mask=mask, tile=128)
    ek = assert_grad_close(dk.reshape(-1, w.N, w.d)[kb, kc].double().numpy(), rk, "dK")
    ev = assert_grad_close(dv.reshape(-1, w.N, w.d)[kb, kc].double().numpy(), rv, "dV")
    log_errors("bs64k_sampled", o=eo, lse=el, dq=eq, dk=ek, dv=ev)
