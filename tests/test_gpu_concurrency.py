"""Concurrent use: two different problems (different head dims, masks and shapes) run at the same time on two
streams, launched interleaved from one host thread and from two host threads (ctypes releases the interpreter lock
during each call).  Each stream's results must equal the same problem run alone: O, LSE, dK, dV bit for bit, dQ to
one unit in the last place of its largest magnitude (its fp32 L2 reductions have no fixed order)."""
import threading

import pytest
import torch

import exact_io_aware_48_b200 as fa
from exact_io_aware_48_b200 import inputs

pytestmark = pytest.mark.gpu

PROBLEMS = [
    # B, H, N, d, dtype, causal, key_lens
    (1, 4, 1000, 128, "bf16", True, None),
    (2, 3, 700, 64, "fp16", False, [700, 129]),
]


def make(i):
    B, H, N, d, dtype, causal, kl = PROBLEMS[i]
    t = [inputs.gaussian((B, H, N, d), 300 + 10 * i + j, dtype).cuda() for j in range(4)]
    klt = None if kl is None else torch.tensor(kl, dtype=torch.int32, device="cuda")
    return t, causal, klt, dtype


def run(prob, stream):
    (q, k, v, do), causal, klt, _ = prob
    o, lse = fa.attention_fwd(q, k, v, causal=causal, key_lens=klt, stream=stream)
    dq, dk, dv = fa.attention_bwd(q, k, v, o, do, lse, causal=causal, key_lens=klt, stream=stream)
    return o, lse, dq, dk, dv


def same(a, b, dtype):
    for name, x, y in zip(("O", "LSE", "dQ", "dK", "dV"), a, b):
        if name == "dQ":
            ulp = 2.0 ** (-7 if dtype == "bf16" else -10)
            assert float((x.float() - y.float()).abs().max()) <= ulp * max(float(x.float().abs().max()), 1e-3)
        else:
            assert torch.equal(x, y), name


def reference(probs):
    refs = []
    for p in probs:
        out = run(p, None)
        torch.cuda.synchronize()
        refs.append([t.clone() for t in out])
    return refs


def test_two_streams_one_thread():
    probs = [make(0), make(1)]
    refs = reference(probs)
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    results = [[], []]
    for _ in range(4):
        for i in (0, 1):
            with torch.cuda.stream(streams[i]):
                results[i].append(run(probs[i], streams[i]))
    torch.cuda.synchronize()
    assert fa.last_device_status() == 0
    for i in (0, 1):
        for r in results[i]:
            same(refs[i], r, probs[i][3])


def test_two_host_threads():
    probs = [make(0), make(1)]
    refs = reference(probs)
    results = [[], []]
    errors = []

    def worker(i):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                for _ in range(4):
                    out = run(probs[i], s)
                    s.synchronize()
                    results[i].append([t.clone() for t in out])
        except Exception as e:  # surfaced in the main thread
            errors.append(repr(e))

    threads = [threading.Thread(target=worker, args=(i,)) for i in (0, 1)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=300)
    assert not errors, errors
    assert all(len(r) == 4 for r in results)
    assert fa.last_device_status() == 0
    for i in (0, 1):
        for r in results[i]:
            same(refs[i], r, probs[i][3])
