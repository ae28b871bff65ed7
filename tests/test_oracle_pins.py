"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each test ties one oracle function to something external: a published
known-answer vector, a hand-worked example, a closed form, a textbook special
case computed by a library routine, an invariant, or brute force written
differently.  Chosen so that a dropped term, a flipped sign, a transposed
operand, a wrong bit position or a wrong GQA grouping fails at least one.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

from oracle import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- generator
def test_splitmix64_known_answers():
    # Published splitmix64 test vectors (Vigna's reference C code and the
    # widely used seed-1234567 sequence).
    assert O.splitmix64_nth(0, 1) == 0xE220A8397B1DCDAF
    want = [6457827717110365317, 3203168211198807973, 9817491932198370423,
            4593380528125082431, 16408922859458223821]
    assert [O.splitmix64_nth(1234567, n) for n in range(1, 6)] == want


def test_hyperplanes_counter_layout_and_balance():
    R = O.hyperplanes(0x5EEDDA5B, 128, 128)
    assert R.shape == (128, 128) and set(np.unique(R)) == {-1, 1}
    # element (j, i) is output number j*d + i + 1 of the stream
    for j, i in [(0, 0), (3, 7), (127, 127), (64, 1)]:
        top = O.splitmix64_nth(0x5EEDDA5B, j * 128 + i + 1) >> 63
        assert R[j, i] == (-1 if top else 1)
    # Rademacher: mean 0, std of mean = 1/128; rows pairwise near-orthogonal
    assert abs(R.mean()) < 5 / 128
    G = R.astype(np.int64) @ R.T.astype(np.int64)
    off = G[~np.eye(128, dtype=bool)]
    assert np.all(np.diag(G) == 128) and np.abs(off).max() < 6 * math.sqrt(128)


# ---------------------------------------------------------------- worked example
def _gold():
    with open(os.path.join(GOLD, "hadamard4_example.json")) as f:
        return json.load(f)


def test_worked_example_all_steps():
    g = _gold()
    R = np.array(g["R"], dtype=np.int8)
    K = np.array(g["K"], dtype=np.float64)[None, None]        # [1,1,6,4]
    V = np.array(g["V"], dtype=np.float64)[None, None]
    q = np.array(g["q"], dtype=np.float64)[None]               # [1,2,4]
    L = O.Layout(B=1, Hkv=1, d=4, bits=4, n_cap=6)
    seq = np.array([6], dtype=np.int32)
    codes = O.encode(L, K, seq, R)
    assert codes[0, 0, :, 0].tolist() == g["codes"]
    sc, bound = O.scores(L, 2, q, codes, seq, R)
    assert sc[0, 0].tolist() == g["scores"]
    assert bound == pytest.approx(4.0)
    for case in g["select_cases"]:
        idx, cnt = O.select(sc, seq, case["topk"], case["sink"], case["window"])
        assert idx[0, 0, : cnt[0, 0]].tolist() == case["sel"]
        assert np.all(idx[0, 0, cnt[0, 0]:] == -1)
    idx, cnt = O.select(sc, seq, 2, 0, 0)
    out, lse = O.attend(L, 2, q, K, V, idx, cnt)
    l0, l5 = g["attend_head0_over_0_5"]["logits"]
    p0 = 1.0 / (1.0 + math.exp(l5 - l0))
    want = p0 * V[0, 0, 0] + (1 - p0) * V[0, 0, 5]
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-14, atol=1e-14)
    assert lse[0, 0] == pytest.approx(math.log(math.exp(l0) + math.exp(l5)), rel=1e-14)


# ---------------------------------------------------------------- encode
def _grid(rng, shape):
    return np.clip(np.round(64 * rng.standard_normal(shape)), -256, 256) / 64 + 0.0


def test_encode_hyperplane_aligned_keys_bit_positions():
    # key = c * R_j gives dot_j = c*d > 0 (bit j set); key = -c * R_j gives
    # dot_j = -c*d < 0 (bit j clear).  Checks orientation of R and that bit j
    # sits in word j/64 at position j%64.
    bits, d = 128, 64
    R = O.hyperplanes(99, bits, d)
    L = O.Layout(B=1, Hkv=1, d=d, bits=bits, n_cap=2 * bits)
    K = np.concatenate([0.5 * R, -0.5 * R]).astype(np.float64)[None, None]
    codes = O.encode(L, K, np.array([2 * bits], np.int32), R)[0, 0]
    for j in range(bits):
        assert (int(codes[j, j // 64]) >> (j % 64)) & 1 == 1
        assert (int(codes[bits + j, j // 64]) >> (j % 64)) & 1 == 0


def test_encode_zero_key_ties_to_one_and_antipodal_complement():
    bits, d = 64, 128
    R = O.hyperplanes(5, bits, d)
    rng = np.random.default_rng(0)
    k = _grid(rng, (1, d))
    K = np.concatenate([np.zeros((1, d)), k, -k])[None, None]
    L = O.Layout(B=1, Hkv=1, d=d, bits=bits, n_cap=3)
    c = O.encode(L, K, np.array([3], np.int32), R)[0, 0, :, 0]
    assert int(c[0]) == (1 << 64) - 1                       # all dots are 0 -> all ones
    dots = R.astype(np.float64) @ k[0]
    nz = np.flatnonzero(dots != 0)
    for j in map(int, nz):                                  # -k flips every nonzero bit
        assert ((int(c[1]) >> j) & 1) != ((int(c[2]) >> j) & 1)


def test_encode_matches_matmul_brute_force_and_paged_permutation():
    rng = np.random.default_rng(1)
    B, Hkv, d, bits, N = 2, 3, 64, 128, 200
    R = O.hyperplanes(7, bits, d)
    K = _grid(rng, (B, Hkv, N, d))
    seq = np.array([N, 137], np.int32)
    L = O.Layout(B, Hkv, d, bits, n_cap=N)
    codes = O.encode(L, K, seq, R)
    sgn = (np.einsum("bhtd,jd->bhtj", K, R.astype(np.float64)) >= 0)
    for b in range(B):
        for h in range(Hkv):
            n = seq[b]
            packed = np.packbits(sgn[b, h, :n], axis=-1, bitorder="little").view(np.uint64)
            assert np.array_equal(codes[b, h, :n], packed)
    # the same keys stored in shuffled 64-token pages give the same codes
    ps = 64
    pages = [(N + ps - 1) // ps] * B
    P = sum(pages)
    perm = rng.permutation(P).astype(np.int32)
    pt = perm.reshape(B, -1)
    Kp = np.zeros((P, ps, Hkv, d))
    for b in range(B):
        for t in range(N):
            Kp[pt[b, t // ps], t % ps, :, :] = K[b, :, t, :]
    Lp = O.Layout(B, Hkv, d, bits, page_table=pt, page=ps)
    cp = O.encode(Lp, Kp, seq, R)
    for b in range(B):
        for t in range(seq[b]):
            assert np.array_equal(cp[pt[b, t // ps], :, t % ps], codes[b, :, t])


def test_encode_simhash_collision_rate():
    # Charikar: for sign random projections P[bit(x) = bit(y)] = 1 - theta/pi.
    rng = np.random.default_rng(2)
    d, bits, n = 128, 128, 400
    R = O.hyperplanes(11, bits, d)
    x = rng.standard_normal((n, d))
    z = rng.standard_normal((n, d))
    z -= (np.sum(z * x, 1, keepdims=True) / np.sum(x * x, 1, keepdims=True)) * x
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    z /= np.linalg.norm(z, axis=1, keepdims=True)
    theta = np.pi / 3
    y = math.cos(theta) * x + math.sin(theta) * z
    K = np.concatenate([x, y])[None, None]
    L = O.Layout(1, 1, d, bits, n_cap=2 * n)
    c = O.encode(L, K, np.array([2 * n], np.int32), R)[0, 0]
    eq = 0
    for i in range(n):
        for w in range(2):
            eq += 64 - bin(int(c[i, w]) ^ int(c[n + i, w])).count("1")
    rate = eq / (n * bits)
    assert abs(rate - (1 - theta / math.pi)) < 0.02


def test_append_equals_one_shot_encode():
    rng = np.random.default_rng(3)
    B, Hkv, d, bits, N0, steps = 2, 2, 64, 64, 50, 5
    R = O.hyperplanes(13, bits, d)
    cap = N0 + steps
    Kfull = _grid(rng, (B, Hkv, cap, d))
    Vfull = _grid(rng, (B, Hkv, cap, d))
    L = O.Layout(B, Hkv, d, bits, n_cap=cap)
    K = np.zeros_like(Kfull); V = np.zeros_like(Vfull)
    K[:, :, :N0] = Kfull[:, :, :N0]; V[:, :, :N0] = Vfull[:, :, :N0]
    seq = np.array([N0, N0], np.int32)
    codes = O.encode(L, K, seq, R)
    for s in range(steps):
        O.append(L, K, V, codes, seq, Kfull[:, :, N0 + s], Vfull[:, :, N0 + s], R)
    assert seq.tolist() == [cap, cap]
    assert np.array_equal(K, Kfull) and np.array_equal(V, Vfull)
    assert np.array_equal(codes, O.encode(L, Kfull, seq, R))


# ---------------------------------------------------------------- score
def _setup_scores(seed, B=2, Hq=8, Hkv=2, d=64, bits=128, N=300):
    rng = np.random.default_rng(seed)
    R = O.hyperplanes(seed + 100, bits, d)
    K = _grid(rng, (B, Hkv, N, d))
    q = _grid(rng, (B, Hq, d))
    seq = np.array([N, N - 77][:B], np.int32)
    L = O.Layout(B, Hkv, d, bits, n_cap=N)
    codes = O.encode(L, K, seq, R)
    return rng, R, K, q, seq, L, codes


def _bits(codes_row, bits):
    out = np.zeros(bits, dtype=np.int64)
    for j in range(bits):
        out[j] = (int(codes_row[j // 64]) >> (j % 64)) & 1
    return out


def test_score_closed_form_and_back_projection():
    B, Hq, Hkv, d, bits = 2, 8, 2, 64, 128
    rng, R, K, q, seq, L, codes = _setup_scores(20, B, Hq, Hkv, d, bits)
    sc, bound = O.scores(L, Hq, q, codes, seq, R)
    G = Hq // Hkv
    Rf = R.astype(np.float64)
    for b in range(B):
        for h in range(Hkv):
            qg = q[b, h * G:(h + 1) * G]
            Qp = (Rf @ qg.T).sum(axis=1)                     # summed projections
            for t in range(0, seq[b], 13):
                bt = _bits(codes[b, h, t], bits)
                closed = 2 * Qp[bt == 1].sum() - Qp.sum()    # 2*sum_{bit=1} qp - sum qp
                u = Rf.T @ (2 * bt - 1)                      # back-projected sign code
                back = float((qg @ u).sum())
                assert sc[b, h, t] == closed == back
    assert np.all(np.abs(sc[~np.isnan(sc)]) <= bound)


def test_score_gqa_is_sum_of_single_head_scores():
    B, Hq, Hkv, d, bits = 1, 8, 2, 64, 64
    rng, R, K, q, seq, L, codes = _setup_scores(21, B, Hq, Hkv, d, bits)
    sc, _ = O.scores(L, Hq, q, codes, seq, R)
    G = Hq // Hkv
    for h in range(Hkv):
        acc = np.zeros(seq[0])
        for g in range(G):
            Lh = O.Layout(1, 1, d, bits, n_cap=L.n_cap)
            s1, _ = O.scores(Lh, 1, q[:, h * G + g][:, None], codes[:, h:h + 1], seq, R)
            acc += s1[0, 0, :seq[0]]
        assert np.array_equal(sc[0, h, :seq[0]], acc)


def test_score_extreme_codes():
    # all-ones code scores +sum Qp, all-zeros code scores -sum Qp
    d, bits, Hq = 64, 64, 2
    R = O.hyperplanes(3, bits, d)
    rng = np.random.default_rng(4)
    q = _grid(rng, (1, Hq, d))
    codes = np.array([[[[np.uint64(2**64 - 1)], [np.uint64(0)]]]], dtype=np.uint64)
    L = O.Layout(1, 1, d, bits, n_cap=2)
    sc, _ = O.scores(L, Hq, q, codes, np.array([2], np.int32), R)
    Qp = (R.astype(np.float64) @ q[0].T).sum()
    assert sc[0, 0, 0] == Qp and sc[0, 0, 1] == -Qp


# ---------------------------------------------------------------- select
def _brute_select(s, n, k, S, W):
    order = sorted(range(n), key=lambda t: (-s[t], t))
    sel = set(order[:k]) | set(range(min(S, n))) | set(range(max(0, n - W), n))
    return sorted(sel)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_select_exhaustive_with_ties(seed):
    rng = np.random.default_rng(seed)
    B, Hkv, N = 2, 3, 180
    s = rng.integers(-6, 7, size=(B, Hkv, N)).astype(np.float64)   # many ties
    seq = np.array([N, 97], np.int32)
    for k, S, W in [(10, 4, 16), (1, 0, 0), (64, 0, 5), (500, 4, 16), (3, 200, 0), (7, 0, 300)]:
        idx, cnt = O.select(s, seq, k, S, W, cap=k + S + W)
        for b in range(B):
            for h in range(Hkv):
                n = int(seq[b])
                want = _brute_select(s[b, h], n, k, S, W)
                got = idx[b, h, :cnt[b, h]].tolist()
                assert got == want
                assert got == sorted(set(got))
                assert set(range(min(S, n))) <= set(got)
                assert set(range(max(0, n - W), n)) <= set(got)
                assert max(min(k, n), min(n, S + W)) <= len(got) <= min(n, k + S + W)


def test_select_all_equal_takes_lowest_indices():
    s = np.zeros((1, 1, 50))
    idx, cnt = O.select(s, np.array([50], np.int32), 5, 0, 0)
    assert idx[0, 0, :cnt[0, 0]].tolist() == [0, 1, 2, 3, 4]


# ---------------------------------------------------------------- attend
def test_attend_full_selection_equals_dense_softmax_attention():
    rng = np.random.default_rng(30)
    B, Hq, Hkv, d, N = 2, 6, 2, 64, 90
    K = _grid(rng, (B, Hkv, N, d)); V = _grid(rng, (B, Hkv, N, d)); q = _grid(rng, (B, Hq, d))
    seq = np.array([N, 61], np.int32)
    L = O.Layout(B, Hkv, d, 64, n_cap=N)
    idx = np.full((B, Hkv, N), -1, np.int32)
    cnt = np.zeros((B, Hkv), np.int32)
    for b in range(B):
        idx[b, :, :seq[b]] = np.arange(seq[b])
        cnt[b] = seq[b]
    out, lse = O.attend(L, Hq, q, K, V, idx, cnt)
    G = Hq // Hkv
    for b in range(B):
        n = seq[b]
        kk = torch.tensor(K[b, :, :n]).repeat_interleave(G, 0)        # [Hq,n,d]
        vv = torch.tensor(V[b, :, :n]).repeat_interleave(G, 0)
        qq = torch.tensor(q[b]).unsqueeze(1)                          # [Hq,1,d]
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv).squeeze(1).numpy()
        np.testing.assert_allclose(out[b], ref, rtol=1e-12, atol=1e-12)
        logits = np.einsum("hd,hnd->hn", q[b], kk.numpy()) / math.sqrt(d)
        np.testing.assert_allclose(lse[b], scipy.special.logsumexp(logits, axis=1), rtol=1e-13)


def test_attend_special_cases():
    rng = np.random.default_rng(31)
    d, N = 64, 40
    K = _grid(rng, (1, 1, N, d)); V = _grid(rng, (1, 1, N, d)); q = _grid(rng, (1, 1, d))
    L = O.Layout(1, 1, d, 64, n_cap=N)
    # one selected token: out = V_t, lse = its logit
    idx = np.array([[[17]]], np.int32); cnt = np.array([[1]], np.int32)
    out, lse = O.attend(L, 1, q, K, V, idx, cnt)
    assert np.array_equal(out[0, 0], V[0, 0, 17])
    assert lse[0, 0] == pytest.approx(float(q[0, 0] @ K[0, 0, 17]) / 8.0, rel=1e-15)
    # identical keys: uniform weights, out = mean of V, lse = logit + ln n
    K2 = np.repeat(K[:, :, :1], N, axis=2)
    sel = np.array([[[1, 5, 9, 30]]], np.int32); c4 = np.array([[4]], np.int32)
    out, lse = O.attend(L, 1, q, K2, V, sel, c4)
    np.testing.assert_allclose(out[0, 0], V[0, 0, [1, 5, 9, 30]].mean(0), rtol=1e-14, atol=1e-15)
    assert lse[0, 0] == pytest.approx(float(q[0, 0] @ K[0, 0, 0]) / 8.0 + math.log(4), rel=1e-14)


def test_attend_paged_equals_dense():
    rng = np.random.default_rng(32)
    B, Hq, Hkv, d, N, ps = 2, 4, 2, 64, 150, 64
    K = _grid(rng, (B, Hkv, N, d)); V = _grid(rng, (B, Hkv, N, d)); q = _grid(rng, (B, Hq, d))
    pages = (N + ps - 1) // ps
    pt = rng.permutation(B * pages).astype(np.int32).reshape(B, pages)
    Kp = np.zeros((B * pages, ps, Hkv, d)); Vp = np.zeros_like(Kp)
    for b in range(B):
        for t in range(N):
            Kp[pt[b, t // ps], t % ps] = K[b, :, t]
            Vp[pt[b, t // ps], t % ps] = V[b, :, t]
    idx = np.sort(rng.choice(N, size=(B, Hkv, 30), replace=True), axis=-1).astype(np.int32)
    cnt = np.full((B, Hkv), 30, np.int32)
    o1, l1 = O.attend(O.Layout(B, Hkv, d, 64, n_cap=N), Hq, q, K, V, idx, cnt)
    o2, l2 = O.attend(O.Layout(B, Hkv, d, 64, page_table=pt, page=ps), Hq, q, Kp, Vp, idx, cnt)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_select_with_full_topk_makes_step_dense():
    # k >= N: the method reduces to full attention (DSA page: attention on all candidates)
    _, R, K, q, seq, L, codes = _setup_scores(40, B=1, Hq=4, Hkv=1, d=64, bits=64, N=120)
    V = _grid(np.random.default_rng(41), K.shape)
    r = O.decode_step(L, 4, q, K, V, codes, seq, R, topk=10_000, sink=0, window=0)
    assert r["sel_cnt"][0, 0] == seq[0]
    n = seq[0]
    kk = torch.tensor(K[0, 0, :n]); vv = torch.tensor(V[0, 0, :n])
    ref = torch.softmax(torch.tensor(q[0]) @ kk.T / 8.0, dim=-1) @ vv
    np.testing.assert_allclose(r["out"][0], ref.numpy(), rtol=1e-12, atol=1e-12)
