"""Parity cases for the debug build (test infrastructure), run in a child process whose FA_LIB_PATH selects
libfa_debug.so.  Every kernel family with index checks runs once on a small case and is compared with the fp64
oracle at the tolerances of the main parity tests; after each case the device status word and the bounds-site word
must be clear (no index check failed on valid inputs).  Finally the bounds self-test must be caught: status
FA_ERR_BOUNDS, site 99.  Prints one JSON object on the last line of stdout.

    FA_LIB_PATH=.../libfa_debug.so python tests/debug_cases.py [--full]

With --full it instead runs one forward + backward of every benchmark workload at full size through the debug
library and checks only that no index check failed.
"""
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import oracle  # noqa: E402
import exact_io_aware_48_b200 as fa  # noqa: E402
from exact_io_aware_48_b200 import _lib, inputs  # noqa: E402
from parity import assert_grad_close, assert_lse_close, assert_o_close, f64  # noqa: E402


def clear(name, out):
    st = _lib.fa_last_device_status(None)
    site = _lib.fa_last_bounds_site(None)
    out[name] = {"status": st, "site": site}
    assert st == 0 and site == 0, (name, st, site)


def dense(name, B, H, N, d, dtype, causal, out, key_lens=None, block_mask=None):
    q, k, v, do = [inputs.gaussian((B, H, N, d), 700 + t, dtype) for t in range(4)]
    scale = 1.0 / np.sqrt(d)
    kl = None if key_lens is None else torch.as_tensor(np.array(key_lens, np.int32)).cuda()
    bm = None if block_mask is None else torch.as_tensor(block_mask, dtype=torch.uint8).cuda()
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.attention_fwd(qd, kd, vd, causal=causal, softmax_scale=scale, key_lens=kl, block_mask=bm)
    dq, dk, dv = fa.attention_bwd(qd, kd, vd, o, dod, lse, causal=causal, softmax_scale=scale, key_lens=kl,
                                  block_mask=bm)
    torch.cuda.synchronize()
    clear(name, out)
    rdq, rdk, rdv, ro, rl = oracle.attn_bwd(f64(q), f64(k), f64(v), f64(do), scale, causal=causal,
                                            key_lens=key_lens, block_mask=block_mask)
    out[name]["err"] = [assert_o_close(o.cpu().double().numpy(), ro), assert_lse_close(lse.cpu().numpy(), rl),
                        assert_grad_close(dq.cpu().double().numpy(), rdq, "dQ"),
                        assert_grad_close(dk.cpu().double().numpy(), rdk, "dK"),
                        assert_grad_close(dv.cpu().double().numpy(), rdv, "dV")]


def varlen(out):
    lens = [130, 1, 257]
    cq = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    H, d, total = 2, 128, int(cq[-1])
    q, k, v, do = [inputs.gaussian((total, H, d), 720 + t, "bf16") for t in range(4)]
    scale = 1.0 / np.sqrt(d)
    cqd = torch.as_tensor(cq).cuda()
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = fa.attention_fwd_varlen(qd, kd, vd, cqd, cqd, max(lens), max(lens), causal=True, softmax_scale=scale)
    dq, dk, dv = fa.attention_bwd_varlen(qd, kd, vd, o, dod, lse, cqd, cqd, max(lens), max(lens), causal=True,
                                         softmax_scale=scale)
    torch.cuda.synchronize()
    clear("varlen", out)
    rdq, rdk, rdv, ro, rl = oracle.attn_bwd_varlen(f64(q), f64(k), f64(v), f64(do), cq, cq, scale, causal=True)
    out["varlen"]["err"] = [assert_o_close(o.cpu().double().numpy(), ro), assert_lse_close(lse.cpu().numpy(), rl),
                            assert_grad_close(dq.cpu().double().numpy(), rdq, "dQ"),
                            assert_grad_close(dk.cpu().double().numpy(), rdk, "dK"),
                            assert_grad_close(dv.cpu().double().numpy(), rdv, "dV")]


def decode(out):
    B, H, Nq, Nk, d = 2, 2, 4, 3000, 128
    q = inputs.gaussian((B, H, Nq, d), 730, "bf16")
    k = inputs.gaussian((B, H, Nk, d), 731, "bf16")
    v = inputs.gaussian((B, H, Nk, d), 732, "bf16")
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.attention_fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=True, softmax_scale=scale, num_splits=5)
    torch.cuda.synchronize()
    clear("decode", out)
    ro, rl = oracle.attn_fwd_decode(f64(q), f64(k), f64(v), scale, causal=True)
    out["decode"]["err"] = [assert_o_close(o.cpu().double().numpy(), ro), assert_lse_close(lse.cpu().numpy(), rl)]


def full_size(out):
    """One forward + backward of every benchmark workload (full size): only the status words are checked here;
    the values at these sizes are compared with the oracle by the sampled parity tests."""
    import bench
    st = torch.cuda.Stream()
    for name, w in inputs.workloads().items():
        p = bench.Problem(w)
        p.step(st)
        st.synchronize()
        clear("full_" + name, out)
        del p
        torch.cuda.empty_cache()


def main():
    torch.cuda.set_device(0)
    if "--full" in sys.argv:
        out = {"debug_build": _lib.fa_debug_build()}
        assert out["debug_build"] == 1, "FA_LIB_PATH must select libfa_debug.so"
        clear("start", out)
        full_size(out)
        print(json.dumps(out))
        return
    out = {"debug_build": _lib.fa_debug_build(), "lib": os.path.basename(_lib.LIB_PATH)}
    assert out["debug_build"] == 1, "FA_LIB_PATH must select libfa_debug.so"
    clear("start", out)
    dense("d64_causal", 1, 2, 333, 64, "bf16", True, out)
    dense("d128_keylens", 2, 2, 1000, 128, "fp16", False, out, key_lens=[1000, 129])
    dense("d96", 1, 2, 200, 96, "bf16", True, out)
    dense("d256_causal", 1, 2, 300, 256, "bf16", True, out)
    rng = np.random.default_rng(5)
    mask = (rng.random((5, 5)) < 0.5).astype(np.uint8)
    np.fill_diagonal(mask, 1)
    dense("blocksparse_d64", 1, 2, 640, 64, "fp16", False, out, block_mask=mask)
    varlen(out)
    decode(out)
    # the check itself: the self-test's out-of-range index is caught and its store skipped
    assert _lib.fa_selftest_bounds(None) == 0
    st = _lib.fa_last_device_status(None)
    site = _lib.fa_last_bounds_site(None)
    out["selftest"] = {"status": st, "site": site}
    assert st == _lib.FA_ERR_BOUNDS and site == 99, out["selftest"]
    clear("after_selftest", out)  # both words were cleared by the reads
    print(json.dumps(out))


if __name__ == "__main__":
    main()
