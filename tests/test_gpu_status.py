"""Device-side failure detection without a GPU fault: a kernel waits on an mbarrier that nothing arrives on, its
bounded wait gives up, records FA_ERR_TIMEOUT in the status word and returns; the host reads and clears it."""
import pytest
import torch

import exact_io_aware_48_b200 as fa
from exact_io_aware_48_b200 import _lib

pytestmark = pytest.mark.gpu


def test_wait_timeout_is_reported_and_cleared():
    assert fa.last_device_status() == _lib.FA_OK
    assert _lib.fa_selftest_wait_timeout(1_000_000) == _lib.FA_OK  # 1 ms budget
    assert fa.last_device_status() == _lib.FA_ERR_TIMEOUT
    assert fa.last_device_status() == _lib.FA_OK  # cleared by the read
    # the context is still usable afterwards
    q = torch.randn(1, 1, 128, 64, device="cuda", dtype=torch.bfloat16)
    o, lse = fa.attention_fwd(q, q, q)
    assert fa.last_device_status() == _lib.FA_OK
    assert torch.isfinite(o.float()).all()


def test_cpu_tensors_are_rejected():
    q = torch.zeros(1, 1, 128, 64, dtype=torch.bfloat16)
    with pytest.raises(RuntimeError):
        fa.attention_fwd(q, q, q)


def test_fma_pipe_exp2_accuracy():
    # the forward exponentiates part of P with a range-reduced cubic; its relative error must stay far below the
    # bf16/fp16 rounding of P (checked against fp64 exp2 and next to the hardware ex2.approx)
    x = torch.cat([torch.linspace(-124.9, 10.0, 200001), torch.tensor([-125.5, -200.0, float("-inf"), 0.0, -1.0])])
    xd = x.cuda()
    a, b = torch.empty_like(xd), torch.empty_like(xd)
    assert _lib.fa_selftest_exp2(xd, a, b, xd.numel()) == _lib.FA_OK
    torch.cuda.synchronize()
    ref = torch.exp2(x.double())
    fin = x > -125.0
    rel = ((a.cpu().double() - ref).abs() / ref)[fin]
    assert float(rel.max()) < 1e-4
    assert torch.all(a.cpu()[~fin] == 0.0)
    relm = ((b.cpu().double() - ref).abs() / ref)[fin & (x > -120)]
    assert float(relm.max()) < 1e-5  # hardware reference is close to exact; the polynomial is within 1e-4
