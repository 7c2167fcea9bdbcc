"""Helpers for GPU-vs-oracle parity tests (test infrastructure).

Inputs come from exact_io_aware_48_b200.inputs (seeded); the GPU side runs through the C ABI (via the package's
thin binding), the oracle side through oracle/ in fp64 on the exact same 16-bit values.
"""
import json
import os

import numpy as np
import torch

import oracle
import exact_io_aware_48_b200 as fa
from exact_io_aware_48_b200 import inputs

O_TOL = 1e-2          # O and LSE: max-abs error
GRAD_REL_TOL = 5e-2   # dQ, dK, dV: max-abs error relative to the largest gradient magnitude of that tensor
GRAD_ZERO_FLOOR = 1e-3  # floor of that magnitude for an identically-zero exact gradient


def to_dev(*ts):
    return [None if t is None else t.cuda() for t in ts]


def gpu_fwd(q, k, v, causal, scale, key_lens=None, block_mask=None):
    kl = None if key_lens is None else torch.as_tensor(key_lens, dtype=torch.int32).cuda()
    bm = None if block_mask is None else torch.as_tensor(block_mask, dtype=torch.uint8).cuda()
    qd, kd, vd = to_dev(q, k, v)
    o, lse = fa.attention_fwd(qd, kd, vd, causal=causal, softmax_scale=scale, key_lens=kl, block_mask=bm)
    assert fa.last_device_status() == 0
    return o.cpu(), lse.cpu()


def gpu_fwd_bwd(q, k, v, do, causal, scale, key_lens=None, block_mask=None):
    kl = None if key_lens is None else torch.as_tensor(key_lens, dtype=torch.int32).cuda()
    bm = None if block_mask is None else torch.as_tensor(block_mask, dtype=torch.uint8).cuda()
    qd, kd, vd, dod = to_dev(q, k, v, do)
    o, lse = fa.attention_fwd(qd, kd, vd, causal=causal, softmax_scale=scale, key_lens=kl, block_mask=bm)
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, dod, lse, causal=causal, softmax_scale=scale, key_lens=kl,
                                  block_mask=bm)
    assert fa.last_device_status() == 0
    return o.cpu(), lse.cpu(), dq.cpu(), dk.cpu(), dv.cpu()


def f64(t):
    return inputs.to_f64(t)


def assert_lse_close(got, ref, tol=O_TOL):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    np.testing.assert_array_equal(np.isneginf(got), np.isneginf(ref))
    fin = np.isfinite(ref)
    assert np.all(np.isfinite(got[fin]))
    err = np.max(np.abs(got[fin] - ref[fin])) if fin.any() else 0.0
    assert err <= tol, f"LSE max-abs error {err:.3e} > {tol}"
    return err


def assert_o_close(got, ref, tol=O_TOL):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got))
    err = float(np.max(np.abs(got - ref))) if got.size else 0.0
    assert err <= tol, f"O max-abs error {err:.3e} > {tol}"
    return err


def assert_grad_close(got, ref, name, tol=GRAD_REL_TOL):
    got = np.asarray(got, dtype=np.float64)
    assert np.all(np.isfinite(got)), name
    # Relative bound; when the exact gradient is identically zero (e.g. one visible key: dS = P (dP - D) = 0 in exact
    # arithmetic) the largest magnitude is floored at GRAD_ZERO_FLOOR so rounding of O into D is not an error.
    scale = max(float(np.max(np.abs(ref))) if ref.size else 0.0, GRAD_ZERO_FLOOR)
    err = float(np.max(np.abs(got - ref))) if got.size else 0.0
    assert err <= tol * scale, f"{name}: max-abs error {err:.3e} > {tol} * {scale:.3e}"
    return err / scale


def sampled_keys(seed, BH, N, heads, per_head):
    """`per_head` distinct seeded keys in each of `heads` distinct seeded heads: (head index, key index) arrays."""
    hb, _ = inputs.sample_rows(seed, BH, 1, heads)
    kb, kc = [], []
    for t, h in enumerate(hb.tolist()):
        _, c = inputs.sample_rows(seed + 1 + t, 1, N, per_head)
        kb.append(np.full_like(c, h))
        kc.append(c)
    return np.concatenate(kb), np.concatenate(kc)


def log_errors(name, **errs):
    """Append measured parity errors (for margins) to $FA_PARITY_LOG if set."""
    path = os.environ.get("FA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": name, **{k: float(v) for k, v in errs.items()}}) + "\n")
