"""Pins of the oracle's block-summary (CSA-style) index against facts that do
not come from the oracle itself: a hand-worked example, the m = 1 special case
(the token path, pinned on its own in test_oracle_pins.py), invariants of a sum
of keys, a brute-force selection written differently (lexsort instead of a
comparison sort, set algebra instead of a membership mask), and the closed
form of dense softmax attention when every block is selected.

The index follows the DeepSeek DSA->CSA/HCA page (section CSA: m history
tokens become one summary entry, top-k runs over the summaries; section on the
compressed versus the state cache: tokens of an incomplete block wait in the
state cache).  A wrong block boundary, a dropped tail, a top-k over the
incomplete block, a tie broken towards the higher block or a summary taken
from one token instead of the block fails at least one test here.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

from oracle import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _grid(rng, shape):
    return np.clip(np.round(rng.standard_normal(shape) * 64.0), -256, 256) / 64.0


def test_blocks_worked_example():
    with open(os.path.join(GOLD, "hadamard4_blocks_example.json")) as f:
        g = json.load(f)
    R = np.array(g["R"], dtype=np.int8)
    K = np.array(g["K"], dtype=np.float64)[None, None]  # [1,1,7,4]
    V = np.array(g["V"], dtype=np.float64)[None, None]
    q = np.array(g["q"], dtype=np.float64)[None]         # [1,2,4]
    L = O.Layout(B=1, Hkv=1, d=4, bits=4, n_cap=7)
    seq = np.array([7], dtype=np.int32)
    for m, case in g["blocks"].items():
        m = int(m)
        bc = O.encode_blocks(L, K, seq, m, R, nb_cap=4)
        nb = 7 // m
        assert bc[0, 0, :nb, 0].tolist() == case["codes"]
        assert np.all(bc[0, 0, nb:] == 0)
        bs, _ = O.block_scores(L, 2, q, bc, seq, m, R)
        assert bs[0, 0, :nb].tolist() == case["scores"]
        assert np.isnan(bs[0, 0, nb:]).all()
        for c in case["select_cases"]:
            idx, cnt = O.select_blocks(bs, seq, m, c["topk_blocks"], c["sink"], c["window"], cap=7)
            assert idx[0, 0, :cnt[0, 0]].tolist() == c["sel"], (m, c)
            assert np.all(idx[0, 0, cnt[0, 0]:] == -1)
    bc = O.encode_blocks(L, K, seq, 2, R, nb_cap=4)
    bs, _ = O.block_scores(L, 2, q, bc, seq, 2, R)
    idx, cnt = O.select_blocks(bs, seq, 2, 1, 0, 1, cap=7)
    out, lse = O.attend(L, 2, q, K, V, idx, cnt)
    a = g["attend_m2_k1_over_0_1_6"]
    w = np.exp(a["head0_logits"])
    want0 = (w[0] * V[0, 0, 0] + w[1] * V[0, 0, 1] + w[2] * V[0, 0, 6]) / w.sum()
    np.testing.assert_allclose(out[0, 0], want0, rtol=1e-14, atol=1e-14)
    assert lse[0, 0] == pytest.approx(math.log(w.sum()), rel=1e-14)
    np.testing.assert_allclose(out[0, 1], a["head1_out"], rtol=1e-14)
    assert lse[0, 1] == pytest.approx(math.log(3.0), rel=1e-14)


@pytest.mark.parametrize("paged", [False, True])
def test_blocks_of_one_token_are_the_token_path(paged):
    # m = 1: every token is a complete block, the tail is empty, so the codes,
    # the scores and the selection must be those of the (separately pinned)
    # token path
    rng = np.random.default_rng(11)
    B, Hkv, G, d, bits, ps = 2, 2, 2, 64, 64, 32
    seq = np.array([150, 77], dtype=np.int32)
    R = O.hyperplanes(5, bits, d)
    if paged:
        pages = 5
        P = B * pages + 1
        pt = (rng.permutation(P)[:B * pages]).reshape(B, pages).astype(np.int32)
        K = _grid(rng, (P, ps, Hkv, d))
        L = O.Layout(B, Hkv, d, bits, page_table=pt, page=ps)
        cap = pages * ps
    else:
        cap = 160
        K = _grid(rng, (B, Hkv, cap, d))
        L = O.Layout(B, Hkv, d, bits, n_cap=cap)
    q = _grid(rng, (B, Hkv * G, d))
    codes = O.encode(L, K, seq, R)
    bc = O.encode_blocks(L, K, seq, 1, R, nb_cap=cap)
    sc, _ = O.scores(L, Hkv * G, q, codes, seq, R)
    bs, _ = O.block_scores(L, Hkv * G, q, bc, seq, 1, R)
    for b in range(B):
        n = int(seq[b])
        for h in range(Hkv):
            tok = codes[b, h, :n] if not paged else np.stack(
                [codes[pt[b, t // ps], h, t % ps] for t in range(n)])
            assert np.array_equal(bc[b, h, :n], tok)
            assert np.array_equal(bs[b, h, :n], sc[b, h, :n])
    for k, s, w in [(10, 0, 0), (7, 4, 16), (500, 2, 3)]:
        i1, c1 = O.select(sc, seq, k, s, w, cap=k + s + w)
        i2, c2 = O.select_blocks(bs, seq, 1, k, s, w, cap=k + s + w)
        assert np.array_equal(c1, c2) and np.array_equal(i1, i2)


def test_block_code_invariants():
    rng = np.random.default_rng(12)
    d, bits, m = 128, 128, 4
    R = O.hyperplanes(9, bits, d)
    nb = 6
    K = _grid(rng, (1, 1, nb * m, d))
    # block 1: four copies of one key (its code); block 2: a key and its
    # negation twice (sum 0, every projection ties, all bits 1)
    K[0, 0, 4:8] = K[0, 0, 4]
    K[0, 0, 8:12] = np.stack([K[0, 0, 8], -K[0, 0, 8], K[0, 0, 9], -K[0, 0, 9]])
    L = O.Layout(1, 1, d, bits, n_cap=nb * m)
    seq = np.array([nb * m], dtype=np.int32)
    bc = O.encode_blocks(L, K, seq, m, R, nb_cap=nb)
    codes = O.encode(L, K, seq, R)
    assert np.array_equal(bc[0, 0, 1], codes[0, 0, 4])
    assert np.all(bc[0, 0, 2] == np.uint64(2**64 - 1))
    # order inside a block does not matter; order of blocks does
    perm = np.concatenate([rng.permutation(m) + m * i for i in range(nb)])
    bp = O.encode_blocks(L, K[:, :, perm], seq, m, R, nb_cap=nb)
    assert np.array_equal(bp, bc)
    # the summary is the code of the summed key, computed here by integer matmul
    ks = (K[0, 0] * 64).astype(np.int64).reshape(nb, m, d).sum(axis=1)
    dots = ks @ R.T.astype(np.int64)                      # [nb, bits]
    bits_ = (dots >= 0).astype(np.uint64)
    w0 = (bits_[:, :64] << np.arange(64, dtype=np.uint64)).sum(axis=1, dtype=np.uint64)
    w1 = (bits_[:, 64:] << np.arange(64, dtype=np.uint64)).sum(axis=1, dtype=np.uint64)
    assert np.array_equal(bc[0, 0, :, 0], w0) and np.array_equal(bc[0, 0, :, 1], w1)
    # a prefix length that is not a multiple of m encodes only complete blocks
    short = O.encode_blocks(L, K, np.array([4 * m + 3], dtype=np.int32), m, R, nb_cap=nb)
    assert np.array_equal(short[0, 0, :4], bc[0, 0, :4]) and np.all(short[0, 0, 4:] == 0)


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_select_blocks_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    B, Hkv, m = 3, 2, [2, 4, 8, 16][seed]
    seq = rng.integers(0, 200, size=B).astype(np.int32)
    seq[0] = 7 * m + m - 1  # a full tail
    nb_cap = 200 // m + 1
    # few distinct scores: many ties
    bs = rng.integers(-3, 4, size=(B, Hkv, nb_cap)).astype(np.float64)
    kb, S, W = 3, int(rng.integers(0, 5)), int(rng.integers(m - 1, 3 * m))
    cap = kb * m + S + W + m
    idx, cnt = O.select_blocks(bs, seq, m, kb, S, W, cap)
    for b in range(B):
        n = int(seq[b])
        nb = n // m
        for h in range(Hkv):
            order = np.lexsort((np.arange(nb), -bs[b, h, :nb]))  # score desc, then index asc
            top = set(order[:kb].tolist())
            want = set()
            for i in top:
                want |= set(range(i * m, (i + 1) * m))
            want |= set(range(min(S, n))) | set(range(max(0, n - W), n)) | set(range(nb * m, n))
            got = idx[b, h, :cnt[b, h]].tolist()
            assert got == sorted(want)
            assert np.all(idx[b, h, cnt[b, h]:] == -1)


def test_select_blocks_zero_query_takes_lowest_blocks():
    # q = 0: every block scores 0, so the lowest block indices win the ties
    rng = np.random.default_rng(13)
    d, bits, m = 64, 64, 4
    R = O.hyperplanes(3, bits, d)
    n = 61
    K = _grid(rng, (1, 1, 64, d))
    L = O.Layout(1, 1, d, bits, n_cap=64)
    seq = np.array([n], dtype=np.int32)
    bc = O.encode_blocks(L, K, seq, m, R, nb_cap=16)
    bs, bound = O.block_scores(L, 2, np.zeros((1, 2, d)), bc, seq, m, R)
    assert bound == 0.0 and np.all(bs[0, 0, :15] == 0.0)
    idx, cnt = O.select_blocks(bs, seq, m, 2, 0, 3, cap=16)
    assert idx[0, 0, :cnt[0, 0]].tolist() == list(range(8)) + [58, 59, 60]


def test_blocks_full_selection_is_dense_attention():
    rng = np.random.default_rng(14)
    B, Hkv, G, d, bits, m = 2, 2, 4, 64, 64, 8
    n_cap = 100
    seq = np.array([100, 45], dtype=np.int32)
    K = _grid(rng, (B, Hkv, n_cap, d))
    V = _grid(rng, (B, Hkv, n_cap, d))
    q = _grid(rng, (B, Hkv * G, d))
    R = O.hyperplanes(4, bits, d)
    L = O.Layout(B, Hkv, d, bits, n_cap=n_cap)
    bc = O.encode_blocks(L, K, seq, m, R, nb_cap=n_cap // m)
    r = O.decode_step_blocks(L, Hkv * G, q, K, V, bc, seq, R, m, topk_blocks=1000, sink=0, window=m - 1,
                             cap=n_cap)
    for b in range(B):
        n = int(seq[b])
        assert np.all(r["sel_cnt"][b] == n)
        for hq in range(Hkv * G):
            h = hq // G
            logits = K[b, h, :n] @ q[b, hq] / math.sqrt(d)
            p = scipy.special.softmax(logits)
            np.testing.assert_allclose(r["out"][b, hq], p @ V[b, h, :n], rtol=1e-12, atol=1e-12)
            assert r["lse"][b, hq] == pytest.approx(scipy.special.logsumexp(logits), rel=1e-12)
