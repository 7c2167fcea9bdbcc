"""Pins for the fp64 oracle: each check ties the oracle to something other than itself.

Sources of truth used here (no stored value comes from the CUDA path):
* closed forms: the hand-derived 2x2 example (tests/golden/hand_2x2.json), uniform scores, key length 1,
  identity V (which makes O equal P), constant V;
* a library routine: scipy.special.logsumexp / softmax on single rows;
* the online-softmax recurrence of the explainer page (its "online softmax" section) against the two-pass
  definition, in both loop orders of the slide deck's "Executable shape" slide;
* masking special cases (explainer page, block-sparse section): all-ones mask == dense, causal == the
  equivalent element mask, invisible tiles' K/V do not matter;
* calculus: central finite differences of sum(O * dO) for dQ, dK, dV (review page, claim C7: the backward is
  the gradient of the same exact attention), plus the algebraic invariants sum_c dK_c = 0 and
  sum_c dV_c = sum of dO over non-empty rows;
* a hand-enumerated tile mask with its CSR/CSC lists (tests/golden/mask_nT8.json).
"""
import json
import math
import os

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

import oracle
from oracle import check_np
from exact_io_aware_48_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def qkv(B, H, N, d, seed=0):
    return rnd((B, H, N, d), seed), rnd((B, H, N, d), seed + 1), rnd((B, H, N, d), seed + 2)


# ----------------------------------------------------------------------------------------------- closed forms
@pytest.mark.parametrize("causal", [False, True])
def test_hand_2x2_golden(causal):
    g = json.load(open(os.path.join(GOLDEN, "hand_2x2.json")))
    q = np.array(g["q"])[None, None]
    k = np.array(g["k"])[None, None]
    v = np.array(g["v"])[None, None]
    o, lse = oracle.attn_fwd(q, k, v, g["scale"], causal=causal)
    ref = g["causal" if causal else "noncausal"]
    np.testing.assert_allclose(o[0, 0], ref["O"], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse[0, 0], ref["LSE"], rtol=0, atol=1e-14)


def test_identity_v_exposes_probabilities():
    # V = [I | 0] makes O_r = P_r: rows sum to one and equal scipy's softmax of the scaled scores.
    B, H, N, d = 1, 2, 6, 8
    q, k, _ = qkv(B, H, N, d, 10)
    v = np.zeros((B, H, N, d))
    v[..., :N] = np.eye(N)
    s = 0.37
    o, lse = oracle.attn_fwd(q, k, v, s)
    P = o[..., :N]
    np.testing.assert_allclose(P.sum(-1), 1.0, atol=1e-12)
    scores = s * np.einsum("bhrd,bhcd->bhrc", q, k)
    np.testing.assert_allclose(P, softmax(scores, axis=-1), atol=1e-13)
    np.testing.assert_allclose(lse, logsumexp(scores, axis=-1), atol=1e-12)
    # with a causal mask the rows of P still sum to one and vanish above the diagonal
    o, _ = oracle.attn_fwd(q, k, v, s, causal=True)
    P = o[..., :N]
    np.testing.assert_allclose(P.sum(-1), 1.0, atol=1e-12)
    assert np.all(P[..., np.triu_indices(N, 1)[0], np.triu_indices(N, 1)[1]] == 0.0)


def test_single_rows_match_scipy():
    B, H, N, d = 2, 1, 9, 5
    q, k, v = qkv(B, H, N, d, 20)
    kl = np.array([9, 4], dtype=np.int32)
    o, lse = oracle.attn_fwd(q, k, v, 0.5, key_lens=kl)
    for b in range(B):
        for r in range(N):
            sc = 0.5 * k[b, 0, : kl[b]] @ q[b, 0, r]
            assert abs(lse[b, 0, r] - logsumexp(sc)) < 1e-12
            np.testing.assert_allclose(o[b, 0, r], softmax(sc) @ v[b, 0, : kl[b]], atol=1e-12)


def test_constant_v_gives_constant_o():
    B, H, N, d = 2, 2, 11, 4
    q, k, _ = qkv(B, H, N, d, 30)
    row = np.array([0.25, -1.5, 3.0, 7.0])
    v = np.broadcast_to(row, (B, H, N, d)).copy()
    for kw in ({}, {"causal": True}, {"key_lens": np.array([3, 11], np.int32)}):
        o, _ = oracle.attn_fwd(q, k, v, 0.9, **kw)
        np.testing.assert_allclose(o, np.broadcast_to(row, o.shape), atol=1e-13)


def test_uniform_scores_give_mean_and_log_count():
    B, H, N, d = 1, 1, 7, 3
    _, k, v = qkv(B, H, N, d, 40)
    q = np.zeros((B, H, N, d))
    o, lse = oracle.attn_fwd(q, k, v, 1.0, causal=True)
    for r in range(N):
        np.testing.assert_allclose(o[0, 0, r], v[0, 0, : r + 1].mean(0), atol=1e-14)
        assert abs(lse[0, 0, r] - math.log(r + 1)) < 1e-14


def test_key_length_one_and_causal_first_row():
    B, H, N, d = 2, 3, 8, 4
    q, k, v = qkv(B, H, N, d, 50)
    o, lse = oracle.attn_fwd(q, k, v, 0.7, key_lens=np.array([1, 1], np.int32))
    np.testing.assert_array_equal(o, np.broadcast_to(v[:, :, :1], o.shape))
    np.testing.assert_allclose(lse, 0.7 * np.einsum("bhrd,bhd->bhr", q, k[:, :, 0]), atol=1e-14)
    o, lse = oracle.attn_fwd(q, k, v, 0.7, causal=True)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0])


def test_empty_rows():
    B, H, N, d = 2, 2, 6, 4
    q, k, v = qkv(B, H, N, d, 60)
    do = rnd((B, H, N, d), 61)
    kl = np.array([0, 6], np.int32)
    o, lse = oracle.attn_fwd(q, k, v, 0.5, key_lens=kl)
    assert np.all(o[0] == 0.0) and np.all(np.isneginf(lse[0]))
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, do, 0.5, key_lens=kl)
    assert np.all(dq[0] == 0) and np.all(dk[0] == 0) and np.all(dv[0] == 0)
    # an all-zero block-mask row empties those query rows only
    bm = np.ones((3, 3), np.uint8)
    bm[1] = 0
    o, lse = oracle.attn_fwd(q, k, v, 0.5, block_mask=bm, tile=2)
    assert np.all(o[:, :, 2:4] == 0.0) and np.all(np.isneginf(lse[:, :, 2:4]))
    assert np.all(np.isfinite(lse[:, :, :2]))


# ------------------------------------------------------------------------------------- online == two-pass
@pytest.mark.parametrize("kv_outer", [False, True])
@pytest.mark.parametrize("tq,tk", [(1, 1), (3, 5), (4, 4), (7, 16), (64, 64)])
def test_online_equals_two_pass(kv_outer, tq, tk):
    B, H, N, d = 2, 2, 23, 6
    q, k, v = qkv(B, H, N, d, 70)
    q *= 3.0  # spread scores so the running max moves often
    kl = np.array([23, 9], np.int32)
    bm = (np.random.default_rng(3).random((6, 6)) < 0.6).astype(np.uint8)
    for kw in ({}, {"causal": True}, {"key_lens": kl}, {"block_mask": bm, "tile": 4},
               {"causal": True, "key_lens": kl, "block_mask": bm, "tile": 4}):
        o1, l1 = oracle.attn_fwd(q, k, v, 0.6, **kw)
        o2, l2 = oracle.attn_fwd_online(q, k, v, 0.6, tq, tk, kv_outer, **kw)
        np.testing.assert_allclose(o2, o1, atol=1e-12)
        np.testing.assert_array_equal(np.isneginf(l1), np.isneginf(l2))
        fin = np.isfinite(l1)
        np.testing.assert_allclose(l2[fin], l1[fin], atol=1e-12)


# ------------------------------------------------------------------------------------------ mask special cases
def test_all_ones_block_mask_is_dense():
    B, H, N, d = 1, 2, 20, 5
    q, k, v = qkv(B, H, N, d, 80)
    o1, l1 = oracle.attn_fwd(q, k, v, 0.4)
    o2, l2 = oracle.attn_fwd(q, k, v, 0.4, block_mask=np.ones((5, 5), np.uint8), tile=4)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_causal_and_key_lens_equal_element_masks():
    B, H, N, d = 1, 2, 13, 4
    q, k, v = qkv(B, H, N, d, 90)
    tri = np.tril(np.ones((N, N), np.uint8))
    o1, l1 = oracle.attn_fwd(q, k, v, 0.8, causal=True)
    o2, l2 = oracle.attn_fwd(q, k, v, 0.8, block_mask=tri, tile=1)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    kl = np.zeros((N, N), np.uint8)
    kl[:, :5] = 1
    o1, l1 = oracle.attn_fwd(q, k, v, 0.8, key_lens=np.array([5], np.int32))
    o2, l2 = oracle.attn_fwd(q, k, v, 0.8, block_mask=kl, tile=1)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)


def test_invisible_tiles_contribute_nothing():
    # tile column 2 (keys 8..11) is masked for every row, so garbage K/V there cannot change anything
    B, H, N, d = 1, 2, 16, 4
    q, k, v = qkv(B, H, N, d, 100)
    do = rnd((B, H, N, d), 101)
    bm = np.ones((4, 4), np.uint8)
    bm[:, 2] = 0
    bm[0, 3] = 0
    o1, l1 = oracle.attn_fwd(q, k, v, 0.5, block_mask=bm, tile=4)
    g1 = oracle.attn_bwd(q, k, v, do, 0.5, block_mask=bm, tile=4)
    k2, v2 = k.copy(), v.copy()
    k2[:, :, 8:12] = 1e6 * rnd((B, H, 4, d), 102)
    v2[:, :, 8:12] = -1e6
    o2, l2 = oracle.attn_fwd(q, k2, v2, 0.5, block_mask=bm, tile=4)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(l1, l2)
    g2 = oracle.attn_bwd(q, k2, v2, do, 0.5, block_mask=bm, tile=4)
    np.testing.assert_array_equal(g1[0], g2[0])
    assert np.all(g2[1][:, :, 8:12] == 0) and np.all(g2[2][:, :, 8:12] == 0)


# ----------------------------------------------------------------------------------------------- gradients
def _loss(q, k, v, do, scale, kw):
    o, _ = oracle.attn_fwd(q, k, v, scale, **kw)
    return float(np.sum(o * do))


FD_CASES = [
    (5, 4, {}),
    (16, 8, {"causal": True}),
    (16, 8, {"key_lens": np.array([11], np.int32)}),
    (16, 8, {"block_mask": np.array([[1, 0, 1, 1], [1, 1, 0, 0], [0, 1, 1, 0], [1, 1, 1, 1]], np.uint8), "tile": 4}),
]


@pytest.mark.parametrize("N,d,kw", FD_CASES)
def test_gradients_match_central_differences(N, d, kw):
    B, H = 1, 1
    q, k, v = qkv(B, H, N, d, 110 + N + d)
    do = rnd((B, H, N, d), 120)
    s = 1.0 / math.sqrt(d)
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, do, s, **kw)
    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v}
            args_m = {"q": q, "k": k, "v": v}
            args_p[name], args_m[name] = xp, xm
            fd[idx] = (_loss(args_p["q"], args_p["k"], args_p["v"], do, s, kw)
                       - _loss(args_m["q"], args_m["k"], args_m["v"], do, s, kw)) / (2 * h)
        err = np.max(np.abs(fd - g)) / max(np.max(np.abs(g)), 1e-30)
        assert err <= 1e-6, (name, err)


def test_gradient_invariants():
    B, H, N, d = 2, 2, 37, 8
    q, k, v = qkv(B, H, N, d, 130)
    do = rnd((B, H, N, d), 131)
    kl = np.array([37, 20], np.int32)
    for kw in ({}, {"causal": True}, {"key_lens": kl}):
        dq, dk, dv, o, lse = oracle.attn_bwd(q, k, v, do, 0.35, **kw)
        np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-11)
        nonempty = np.isfinite(lse)[..., None]
        np.testing.assert_allclose(dv.sum(axis=2), (do * nonempty).sum(axis=2), atol=1e-11)
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, do, 0.35, key_lens=kl)
    assert np.all(dk[1, :, 20:] == 0) and np.all(dv[1, :, 20:] == 0)


def test_matches_numpy_statement():
    B, H, N, d = 2, 2, 19, 8
    q, k, v = qkv(B, H, N, d, 140)
    do = rnd((B, H, N, d), 141)
    kl = np.array([19, 7], np.int32)
    bm = np.array([[1, 0, 1, 1, 0], [1, 1, 0, 1, 1], [0, 0, 1, 1, 0], [1, 1, 1, 1, 1], [0, 1, 0, 1, 1]], np.uint8)
    for kw in ({}, {"causal": True}, {"key_lens": kl}, {"block_mask": bm, "tile": 4},
               {"causal": True, "key_lens": kl, "block_mask": bm, "tile": 4}):
        mask = check_np.element_mask(B, N, **kw)
        ref = check_np.attn_grads_np(q, k, v, do, 0.3, mask)
        got = oracle.attn_bwd(q, k, v, do, 0.3, **kw)
        for a, b in zip(got[:4], ref[:4]):
            np.testing.assert_allclose(a, b, atol=1e-12)
        np.testing.assert_array_equal(np.isneginf(got[4]), np.isneginf(ref[4]))


# -------------------------------------------------------------------------------- sampled variants == full
def test_sampled_rows_and_keys_equal_full():
    B, H, N, d = 2, 3, 29, 8
    q, k, v = qkv(B, H, N, d, 150)
    do = rnd((B, H, N, d), 151)
    kl = np.array([29, 13], np.int32)
    for kw in ({"causal": True}, {"key_lens": kl}):
        dq, dk, dv, o, lse = oracle.attn_bwd(q, k, v, do, 0.4, **kw)
        sb, sr = inputs.sample_rows(5, B * H, N, 40)
        o_s, l_s = oracle.attn_fwd_rows(q, k, v, 0.4, sb, sr, **kw)
        np.testing.assert_allclose(o_s, o.reshape(-1, N, d)[sb, sr], atol=1e-13)
        np.testing.assert_allclose(l_s, lse.reshape(-1, N)[sb, sr], atol=1e-13)
        dq_s = oracle.attn_bwd_rows(q, k, v, do, 0.4, sb, sr, **kw)
        np.testing.assert_allclose(dq_s, dq.reshape(-1, N, d)[sb, sr], atol=1e-12)
        dk_s, dv_s = oracle.attn_bwd_keys(q, k, v, do, 0.4, sb, sr, **kw)
        np.testing.assert_allclose(dk_s, dk.reshape(-1, N, d)[sb, sr], atol=1e-12)
        np.testing.assert_allclose(dv_s, dv.reshape(-1, N, d)[sb, sr], atol=1e-12)


# ------------------------------------------------------------------------------------------ block-mask lists
def test_mask_recipe_and_lists_golden():
    g = json.load(open(os.path.join(GOLDEN, "mask_nT8.json")))
    m = inputs.band_mask(8) | inputs.butterfly_mask(8)
    assert [list(np.nonzero(r)[0]) for r in m] == g["rows"]
    row_ptr, col_idx = oracle.blockmask_csr(m)
    assert row_ptr.tolist() == g["row_ptr"]
    assert col_idx.tolist() == [c for r in g["rows"] for c in r]
    col_ptr, row_idx = oracle.blockmask_csc(m)
    assert col_ptr.tolist() == g["col_ptr"]
    assert row_idx.tolist() == [r for c in g["cols"] for r in c]


def test_lists_match_brute_force_random_masks():
    rng = np.random.default_rng(7)
    for nT in (1, 2, 5, 33):
        m = (rng.random((nT, nT)) < 0.3).astype(np.uint8)
        row_ptr, col_idx = oracle.blockmask_csr(m)
        col_ptr, row_idx = oracle.blockmask_csc(m)
        for i in range(nT):
            assert col_idx[row_ptr[i]:row_ptr[i + 1]].tolist() == [j for j in range(nT) if m[i, j]]
        for j in range(nT):
            assert row_idx[col_ptr[j]:col_ptr[j + 1]].tolist() == [i for i in range(nT) if m[i, j]]
    empty = np.zeros((4, 4), np.uint8)
    rp, ci = oracle.blockmask_csr(empty)
    assert rp.tolist() == [0] * 5 and ci.size == 0


# ----------------------------------------------------------------------------------------------- packed batches
# The packed variable-length oracle composes the pinned dense oracle with per-sequence slicing and padding; these
# pins check the composition against the dense batch it must reduce to, against reordering and independence of
# the sequences, against calculus (finite differences of a cross-length case) and the per-sequence invariants.
def _packed(x):
    """[B, H, N, d] -> packed [B*N, H, d] with cu = 0, N, 2N, ..."""
    B, H, N, d = x.shape
    return x.transpose(0, 2, 1, 3).reshape(B * N, H, d)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equal_lengths_equal_dense_batch(causal):
    B, H, N, d = 3, 2, 11, 4
    q, k, v = qkv(B, H, N, d, 160)
    do = rnd((B, H, N, d), 161)
    cu = np.arange(B + 1, dtype=np.int32) * N
    o, lse = oracle.attn_fwd(q, k, v, 0.4, causal=causal)
    ov, lv = oracle.attn_fwd_varlen(_packed(q), _packed(k), _packed(v), cu, cu, 0.4, causal=causal)
    np.testing.assert_allclose(ov, _packed(o), rtol=0, atol=1e-13)
    np.testing.assert_allclose(lv, lse.transpose(1, 0, 2).reshape(H, B * N), rtol=0, atol=1e-13)
    dq, dk, dv, _, _ = oracle.attn_bwd(q, k, v, do, 0.4, causal=causal)
    gq, gk, gv, _, _ = oracle.attn_bwd_varlen(_packed(q), _packed(k), _packed(v), _packed(do), cu, cu, 0.4,
                                              causal=causal)
    for a, b in ((gq, dq), (gk, dk), (gv, dv)):
        np.testing.assert_allclose(a, _packed(b), rtol=0, atol=1e-13)


def test_varlen_sequences_are_independent_and_order_free():
    H, d = 2, 4
    lq, lk = [5, 0, 9, 3], [7, 4, 9, 1]
    cq, ck = np.concatenate([[0], np.cumsum(lq)]), np.concatenate([[0], np.cumsum(lk)])
    q, k, v = rnd((cq[-1], H, d), 170), rnd((ck[-1], H, d), 171), rnd((ck[-1], H, d), 172)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cq, ck, 0.5)
    # each sequence alone gives the same rows
    for b in range(4):
        if lq[b] == 0:
            continue
        ob, lb = oracle.attn_fwd_varlen(q[cq[b]:cq[b + 1]], k[ck[b]:ck[b + 1]], v[ck[b]:ck[b + 1]],
                                        [0, lq[b]], [0, lk[b]], 0.5)
        np.testing.assert_allclose(ob, o[cq[b]:cq[b + 1]], rtol=0, atol=1e-14)
        np.testing.assert_allclose(lb, lse[:, cq[b]:cq[b + 1]], rtol=0, atol=1e-14)
    # reversing the sequence order reverses the blocks
    perm = [3, 2, 1, 0]
    q2 = np.concatenate([q[cq[b]:cq[b + 1]] for b in perm])
    k2 = np.concatenate([k[ck[b]:ck[b + 1]] for b in perm])
    v2 = np.concatenate([v[ck[b]:ck[b + 1]] for b in perm])
    cq2 = np.concatenate([[0], np.cumsum([lq[b] for b in perm])])
    ck2 = np.concatenate([[0], np.cumsum([lk[b] for b in perm])])
    o2, _ = oracle.attn_fwd_varlen(q2, k2, v2, cq2, ck2, 0.5)
    np.testing.assert_allclose(o2, np.concatenate([o[cq[b]:cq[b + 1]] for b in perm]), rtol=0, atol=1e-14)


def test_varlen_empty_key_sequence_and_key_count_one():
    H, d = 1, 3
    q, k, v = rnd((4, H, d), 180), rnd((3, H, d), 181), rnd((3, H, d), 182)
    # sequence 0: 2 queries, 0 keys -> O = 0, LSE = -inf; sequence 1: 2 queries, 3 keys, causal -> query 0 sees key 0
    o, lse = oracle.attn_fwd_varlen(q, k, v, [0, 2, 4], [0, 0, 3], 1.0, causal=True)
    assert np.all(o[:2] == 0) and np.all(np.isneginf(lse[:, :2]))
    np.testing.assert_allclose(o[2], v[0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse[:, 2], np.sum(q[2] * k[0], axis=-1), atol=1e-15)  # one visible key: LSE = scale*q.k


def test_varlen_cross_lengths_match_central_differences():
    H, d = 1, 3
    lq, lk = [3, 4], [5, 2]
    cq, ck = np.array([0, 3, 7]), np.array([0, 5, 7])
    q, k, v = rnd((7, H, d), 190), rnd((7, H, d), 191), rnd((7, H, d), 192)
    do = rnd((7, H, d), 193)
    s = 0.7
    for causal in (False, True):
        dq, dk, dv, _, _ = oracle.attn_bwd_varlen(q, k, v, do, cq, ck, s, causal=causal)

        def loss(qq, kk, vv):
            o, _ = oracle.attn_fwd_varlen(qq, kk, vv, cq, ck, s, causal=causal)
            return float(np.sum(o * do))

        h = 1e-6
        for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
            fd = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                xp, xm = x.copy(), x.copy()
                xp[idx] += h
                xm[idx] -= h
                a = {"q": q, "k": k, "v": v}
                m = dict(a)
                a[name], m[name] = xp, xm
                fd[idx] = (loss(a["q"], a["k"], a["v"]) - loss(m["q"], m["k"], m["v"])) / (2 * h)
            err = np.max(np.abs(fd - g)) / max(np.max(np.abs(g)), 1e-30)
            assert err <= 1e-6, (causal, name, err)


def test_varlen_gradient_invariants_per_sequence():
    H, d = 2, 5
    lq, lk = [6, 13, 1], [9, 13, 4]
    cq, ck = np.concatenate([[0], np.cumsum(lq)]), np.concatenate([[0], np.cumsum(lk)])
    q, k, v = rnd((cq[-1], H, d), 200), rnd((ck[-1], H, d), 201), rnd((ck[-1], H, d), 202)
    do = rnd((cq[-1], H, d), 203)
    dq, dk, dv, o, lse = oracle.attn_bwd_varlen(q, k, v, do, cq, ck, 0.45, causal=True)
    for b in range(3):
        ks, qs = slice(ck[b], ck[b + 1]), slice(cq[b], cq[b + 1])
        np.testing.assert_allclose(dk[ks].sum(axis=0), 0.0, atol=1e-11)
        nonempty = np.isfinite(lse[:, qs]).T[..., None]
        np.testing.assert_allclose(dv[ks].sum(axis=0), (do[qs] * nonempty).sum(axis=0), atol=1e-11)


# ----------------------------------------------------------------------------------------------- decode
# The decode oracle (numpy statement, queries aligned with the end of the keys) is pinned against the C oracle:
# with as many queries as keys it is the ordinary attention; with fewer, its rows are the last rows of an ordinary
# causal attention over the full sequence; key lengths truncate the cache; queries with no visible key are empty.
@pytest.mark.parametrize("causal", [False, True])
def test_decode_full_length_is_ordinary_attention(causal):
    q, k, v = qkv(2, 2, 23, 8, 210)
    o, lse = oracle.attn_fwd(q, k, v, 0.3, causal=causal)
    od, ld = oracle.attn_fwd_decode(q, k, v, 0.3, causal=causal)
    np.testing.assert_allclose(od, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(ld, lse, rtol=0, atol=1e-12)


@pytest.mark.parametrize("nq", [1, 4, 19])
def test_decode_rows_are_last_rows_of_causal_attention(nq):
    B, H, N, d = 2, 2, 37, 8
    qf, k, v = qkv(B, H, N, d, 220)
    o, lse = oracle.attn_fwd(qf, k, v, 0.4, causal=True)
    od, ld = oracle.attn_fwd_decode(qf[:, :, N - nq:], k, v, 0.4, causal=True)
    np.testing.assert_allclose(od, o[:, :, N - nq:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(ld, lse[:, :, N - nq:], rtol=0, atol=1e-12)
    if nq == 1:  # the last query sees every key either way
        on, ln = oracle.attn_fwd_decode(qf[:, :, N - 1:], k, v, 0.4, causal=False)
        np.testing.assert_allclose(on, od, rtol=0, atol=1e-14)


def test_decode_key_lengths_truncate_the_cache_and_empty_queries():
    B, H, Nq, Nk, d = 2, 1, 5, 30, 4
    q, k, v = rnd((B, H, Nq, d), 230), rnd((B, H, Nk, d), 231), rnd((B, H, Nk, d), 232)
    kl = np.array([17, 3], np.int32)
    o, lse = oracle.attn_fwd_decode(q, k, v, 0.5, causal=True, key_lens=kl)
    for b in range(B):
        n = int(kl[b])
        ob, lb = oracle.attn_fwd_decode(q[b:b + 1], k[b:b + 1, :, :n], v[b:b + 1, :, :n], 0.5, causal=True)
        np.testing.assert_allclose(o[b:b + 1], ob, rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[b:b + 1], lb, rtol=0, atol=1e-14)
    # sequence 1 has 3 keys for 5 queries: queries 0 and 1 see nothing (c <= r + 3 - 5 < 0), query 2 sees key 0
    assert np.all(o[1, :, :2] == 0) and np.all(np.isneginf(lse[1, :, :2]))
    np.testing.assert_allclose(o[1, :, 2], v[1, :, 0], rtol=0, atol=1e-15)


# ----------------------------------------------------------------------------------------------- per-head masks
def test_head_masks_all_equal_give_the_shared_mask_result():
    B, H, N, d = 2, 3, 16, 4
    q, k, v = qkv(B, H, N, d, 240)
    do = rnd((B, H, N, d), 241)
    m = np.array([[1, 0, 1, 1], [1, 1, 0, 0], [0, 1, 1, 0], [1, 1, 1, 1]], np.uint8)
    shared = oracle.attn_bwd(q, k, v, do, 0.5, block_mask=m, tile=4)
    per = oracle.attn_bwd_head_masks(q, k, v, do, 0.5, np.stack([m] * H), tile=4)
    for a, b in zip(per, shared):
        np.testing.assert_allclose(a, b, rtol=0, atol=1e-14)


def test_head_masks_differ_per_head():
    B, H, N, d = 1, 2, 16, 4
    q, k, v = qkv(B, H, N, d, 250)
    do = rnd((B, H, N, d), 251)
    ones = np.ones((4, 4), np.uint8)
    band = np.eye(4, dtype=np.uint8)
    dq, dk, dv, o, lse = oracle.attn_bwd_head_masks(q, k, v, do, 0.5, np.stack([ones, band]), tile=4)
    od, _ = oracle.attn_fwd(q[:, :1], k[:, :1], v[:, :1], 0.5)  # head 0: all tiles kept = dense
    np.testing.assert_allclose(o[:, :1], od, rtol=0, atol=1e-14)
    ob, _ = oracle.attn_fwd(q[:, 1:], k[:, 1:], v[:, 1:], 0.5, block_mask=band, tile=4)
    np.testing.assert_allclose(o[:, 1:], ob, rtol=0, atol=1e-14)
