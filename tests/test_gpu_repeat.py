"""Repeatability: a race between warps shows up as run-to-run differences.  O, LSE, dK and dV are accumulated in a
fixed order on chip, so repeated runs on the same inputs must agree bit for bit; dQ is summed across CTAs by fp32 L2
reductions in no fixed order, so its fp32 sums agree to rounding and its 16-bit output may differ by one unit in the
last place: at most 2^-7 (bf16) or 2^-10 (fp16) of the largest magnitude."""
import numpy as np
import pytest
import torch

import exact_io_aware_48_b200 as fa
from exact_io_aware_48_b200 import inputs

pytestmark = pytest.mark.gpu

CASES = [
    (2, 3, 333, 128, "fp16", True, None),
    (2, 2, 700, 64, "bf16", False, None),
    (1, 4, 1024, 128, "bf16", True, None),
    (3, 2, 500, 64, "fp16", True, [500, 129, 3]),
]


@pytest.mark.parametrize("B,H,N,d,dtype,causal,kl", CASES)
def test_runs_repeat_exactly(B, H, N, d, dtype, causal, kl):
    q, k, v, do = [inputs.gaussian((B, H, N, d), 70 + t, dtype).cuda() for t in range(4)]
    klt = None if kl is None else torch.tensor(kl, dtype=torch.int32, device="cuda")
    runs = []
    for _ in range(5):
        o, lse = fa.attention_fwd(q, k, v, causal=causal, key_lens=klt)
        dq, dk, dv = fa.attention_bwd(q, k, v, o, do, lse, causal=causal, key_lens=klt)
        runs.append([t.clone() for t in (o, lse, dq, dk, dv)])
    assert fa.last_device_status() == 0
    base = runs[0]
    for r in runs[1:]:
        for name, a, b in zip(("O", "LSE", "dK", "dV"), (base[0], base[1], base[3], base[4]), (r[0], r[1], r[3], r[4])):
            assert torch.equal(a, b), f"{name} differs between runs"
        scale = float(base[2].float().abs().max())
        ulp = 2.0 ** (-7 if dtype == "bf16" else -10)
        assert float((base[2].float() - r[2].float()).abs().max()) <= ulp * max(scale, 1e-3), "dQ drifts"
