"""Backward parity on the GPU: dQ, dK, dV from libfa.so through the C ABI vs the fp64 oracle.

Tolerance: per tensor, max-abs error <= 5e-2 * max |gradient| (bf16/fp16 inputs, fp32 accumulation).  Small cases
span several tiles with ragged tails; the workload shapes run at full size (full oracle where it finishes in
seconds; long sequences: 256 sampled query rows for dQ and sampled keys of one head for dK/dV, plus invariants
that hold at any size).
"""
import numpy as np
import pytest
import torch

import oracle
from exact_io_aware_48_b200 import inputs
from parity import assert_grad_close, assert_lse_close, assert_o_close, f64, gpu_fwd_bwd, log_errors

pytestmark = pytest.mark.gpu


def make(B, H, N, d, dtype, seed):
    return [inputs.gaussian((B, H, N, d), seed * 10 + t, dtype) for t in range(4)]


SMALL = [
    (1, 2, 128, 64, "bf16", False, None),
    (1, 2, 256, 128, "bf16", True, None),
    (2, 2, 1, 64, "bf16", True, None),
    (2, 2, 5, 128, "fp16", False, None),
    (1, 2, 127, 64, "bf16", True, None),
    (2, 2, 129, 128, "fp16", True, None),
    (1, 3, 300, 64, "bf16", False, None),
    (2, 2, 333, 128, "bf16", True, None),
    (2, 2, 700, 64, "fp16", True, None),
    (3, 2, 640, 128, "bf16", False, [640, 1, 257]),
    (3, 2, 500, 64, "bf16", True, [500, 129, 3]),
    (2, 1, 384, 128, "bf16", False, [0, 384]),
]


@pytest.mark.parametrize("B,H,N,d,dtype,causal,kl", SMALL)
def test_bwd_small_cases(B, H, N, d, dtype, causal, kl):
    q, k, v, do = make(B, H, N, d, dtype, N + 3 * d)
    scale = 1.0 / np.sqrt(d)
    kla = None if kl is None else np.array(kl, np.int32)
    o, lse, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, causal, scale, key_lens=kla)
    rq, rk, rv, ro, rl = oracle.attn_bwd(f64(q), f64(k), f64(v), f64(do), scale, causal=causal, key_lens=kla)
    assert_o_close(o.double().numpy(), ro)
    assert_lse_close(lse.numpy(), rl)
    e = [assert_grad_close(g.double().numpy(), r, n) for g, r, n in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV"))]
    log_errors(f"bwd_small B{B} H{H} N{N} d{d} {dtype} causal={causal} kl={kl}", dq=e[0], dk=e[1], dv=e[2])


@pytest.mark.parametrize("name", ["tiny", "gpt2", "bert"])
def test_bwd_workloads_full(name):
    w = inputs.workloads()[name]
    q, k, v, do = w.tensors()
    kl = w.key_lens_array()
    o, lse, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, w.causal, w.scale, key_lens=kl)
    rq, rk, rv, ro, rl = oracle.attn_bwd(f64(q), f64(k), f64(v), f64(do), w.scale, causal=w.causal, key_lens=kl)
    e = [assert_grad_close(g.double().numpy(), r, n) for g, r, n in ((dq, rq, "dQ"), (dk, rk, "dK"), (dv, rv, "dV"))]
    log_errors(f"bwd_{name}", dq=e[0], dk=e[1], dv=e[2])
    if kl is not None:  # keys beyond the length get exactly zero gradient
        for b in range(w.B):
            assert torch.all(dk[b, :, kl[b]:] == 0) and torch.all(dv[b, :, kl[b]:] == 0)


def check_invariants(dq, dk, dv, do, lse):
    # sum_c dK_c = 0 and sum_c dV_c = sum of dO over rows with a visible key, per head (algebra of softmax)
    dk64, dv64 = dk.double(), dv.double()
    do64 = do.double() * torch.isfinite(lse).double()[..., None]
    ref = do64.sum(dim=2)
    assert torch.max(torch.abs(dv64.sum(dim=2) - ref)) <= 2e-2 * (1 + torch.max(torch.abs(ref)))
    assert torch.max(torch.abs(dk64.sum(dim=2))) <= 2e-2 * (1 + dk64.abs().sum(dim=2).max())


@pytest.mark.parametrize("name", ["lc4k", "lc8k", "lc16k"])
def test_bwd_long_context_sampled(name):
    w = inputs.workloads()[name]
    q, k, v, do = w.tensors()
    o, lse, dq, dk, dv = gpu_fwd_bwd(q, k, v, do, w.causal, w.scale)
    qf, kf, vf, dof = f64(q), f64(k), f64(v), f64(do)
    sb, sr = inputs.sample_rows(w.seed + 600, w.B * w.H, w.N, 256)
    rq = oracle.attn_bwd_rows(qf, kf, vf, dof, w.scale, sb, sr, causal=w.causal)
    # dK/dV: 128 sampled keys of one head (the oracle needs that head's full forward)
    head = int(sb[0])
    kb, kc = inputs.sample_rows(w.seed + 700, 1, w.N, 128)
    kb = np.full_like(kc, head)
    rk, rv = oracle.attn_bwd_keys(qf, kf, vf, dof, w.scale, kb, kc, causal=w.causal)
    # the tolerance scale is the largest gradient magnitude of the whole tensor (GPU value, within tolerance)
    e_q = _sampled_close(dq.reshape(-1, w.N, w.d)[sb, sr], rq, dq, "dQ")
    e_k = _sampled_close(dk.reshape(-1, w.N, w.d)[kb, kc], rk, dk, "dK")
    e_v = _sampled_close(dv.reshape(-1, w.N, w.d)[kb, kc], rv, dv, "dV")
    log_errors(f"bwd_{name}_sampled", dq=e_q, dk=e_k, dv=e_v)
    check_invariants(dq, dk, dv, do, lse)


def _sampled_close(got, ref, full, name):
    got = got.double().numpy()
    assert np.all(np.isfinite(got)), name
    scale = max(float(np.max(np.abs(ref))), float(full.float().abs().max()))
    err = float(np.max(np.abs(got - ref)))
    assert err <= 5e-2 * scale, f"{name}: {err:.3e} > 5e-2 * {scale:.3e}"
    return err / scale
