"""CUDA-graph capture: forward + backward captured once through the package API (every call is stream-ordered; the
tensor maps are encoded on the host at capture and travel as kernel parameters) and replayed.  A replay must give
the eager results on the same inputs, and on new inputs copied into the captured input buffers it must give the
eager results for those.  Comparison as in the repeatability test: O, LSE, dK, dV bit for bit; dQ (fp32 L2
reductions in no fixed order) to one unit in the last place of its largest magnitude."""
import numpy as np
import pytest
import torch

import exact_io_aware_48_b200 as fa
from exact_io_aware_48_b200 import inputs

pytestmark = pytest.mark.gpu

CASES = [
    # B, H, N, d, dtype, causal, key_lens, block-mask density
    (1, 2, 640, 128, "bf16", True, None, None),
    (2, 2, 333, 64, "fp16", False, [333, 100], None),
    (1, 2, 700, 64, "bf16", False, None, 0.5),
    (1, 2, 300, 256, "bf16", True, None, None),
]


def same(a, b, dtype):
    names = ("O", "LSE", "dQ", "dK", "dV")
    for i, (x, y) in enumerate(zip(a, b)):
        if names[i] == "dQ":
            scale = float(x.float().abs().max())
            ulp = 2.0 ** (-7 if dtype == "bf16" else -10)
            assert float((x.float() - y.float()).abs().max()) <= ulp * max(scale, 1e-3), "dQ"
        else:
            assert torch.equal(x, y), names[i]


@pytest.mark.parametrize("B,H,N,d,dtype,causal,kl,density", CASES)
def test_graph_replay_matches_eager(B, H, N, d, dtype, causal, kl, density):
    q, k, v, do = [inputs.gaussian((B, H, N, d), 90 + t, dtype).cuda() for t in range(4)]
    klt = None if kl is None else torch.tensor(kl, dtype=torch.int32, device="cuda")
    bm = None
    if density is not None:
        nT = (N + 127) // 128
        m = (np.random.default_rng(7).random((nT, nT)) < density).astype(np.uint8)
        np.fill_diagonal(m, 1)
        bm = torch.as_tensor(m).cuda()

    def run():
        o, lse = fa.attention_fwd(q, k, v, causal=causal, key_lens=klt, block_mask=bm)
        dq, dk, dv = fa.attention_bwd(q, k, v, o, do, lse, causal=causal, key_lens=klt, block_mask=bm)
        return o, lse, dq, dk, dv

    eager = [t.clone() for t in run()]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up outside the capture (first-launch attributes, allocator pools)
        for _ in range(2):
            run()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        outs = run()
    g.replay()
    torch.cuda.synchronize()
    assert fa.last_device_status() == 0
    same(eager, outs, dtype)

    # new inputs in the captured buffers: the replay follows them
    for t, seed in ((q, 190), (k, 191), (v, 192), (do, 193)):
        t.copy_(inputs.gaussian((B, H, N, d), seed, dtype).cuda())
    eager2 = [t.clone() for t in run()]
    g.replay()
    torch.cuda.synchronize()
    assert fa.last_device_status() == 0
    same(eager2, outs, dtype)
    assert not torch.equal(eager[0], eager2[0])  # the inputs really changed
    del g
