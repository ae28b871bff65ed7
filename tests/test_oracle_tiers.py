"""Pins of the oracle's precision tiers (FP8 E4M3 pages; Spherical KV page,
section 2.2 RDR, tier-homogeneous pages; DASH-KV page, section
"技术架构：动态混合精度机制").

The pages fix the idea (critical tokens in full precision, the others in a
cheaper tier, one tier per page) but not the number format; the format is the
OCP 8-bit floating-point E4M3 ("FN") encoding, so the codec is pinned against
torch's own float8_e4m3fn conversion (an independent implementation) over
every bf16 value in range, and against hand-worked ties.  The scale exponent
and the page controller are pinned by brute force from their definitions.
"""
import math

import numpy as np
import pytest
import torch

from oracle import oracle as O


def _torch_e4m3_bytes(v: torch.Tensor) -> np.ndarray:
    return v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_value_matches_torch_for_every_code():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    mine = O.e4m3_table()
    nan = np.isnan(ref)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.isnan(mine[nan]).all()
    assert np.array_equal(mine[~nan], ref[~nan])
    # the format's landmarks
    assert mine[0x7E] == 448.0 and mine[0x08] == 2.0 ** -6 and mine[0x01] == 2.0 ** -9
    assert mine[0x38] == 1.0 and mine[0xB8] == -1.0


def test_e4m3_encode_matches_torch_on_every_bf16_in_range():
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    v = bits.view(torch.bfloat16).to(torch.float32)
    keep = torch.isfinite(v) & (v.abs() <= 448.0)
    v = v[keep]
    ref = _torch_e4m3_bytes(v)
    mine = np.array([O.e4m3_encode(float(x)) for x in v.tolist()], dtype=np.uint8)
    bad = np.nonzero(mine != ref)[0]
    assert bad.size == 0, [(float(v[i]), int(mine[i]), int(ref[i])) for i in bad[:8]]


@pytest.mark.parametrize("v, code", [
    (1.0625, 0x38),    # halfway between 1 (m = 0) and 1.125 (m = 1): even -> 1
    (1.1875, 0x3A),    # halfway between 1.125 (m = 1) and 1.25 (m = 2): even -> 1.25
    (17.0, 0x58),      # binade [16, 32) (exponent field 11) has quantum 2: 17 is a tie -> 16 (m = 0)
    (19.0, 0x5A),      # tie between 18 (m = 1) and 20 (m = 2) -> 20
    (2.0 ** -10, 0x00),  # half the smallest subnormal: tie -> 0
    (3 * 2.0 ** -10, 0x02),  # tie between 1 and 2 subnormal quanta -> 2
    (-0.0, 0x80),
    (432.0, 0x7E),     # tie between 416 (m = 5) and 448 (m = 6) -> 448
    (424.0, 0x7D),     # below the tie -> 416
])
def test_e4m3_encode_ties(v, code):
    assert O.e4m3_encode(v) == code


def _brute_exponent(amax: float) -> int:
    if amax == 0.0:
        return 0
    s = -200
    while math.ldexp(amax, s + 1) <= 448.0 and s < 127:
        s += 1
    return s


def test_tier_exponent_is_the_largest_fitting_power():
    rng = np.random.default_rng(3)
    cases = [0.0, 448.0, 448.0 * (1 + 2 ** -20), 447.9, 4.0, 1.0, 0.875, 0.876, 2.0 ** -133, 3.3e38, 1e-30]
    cases += list(np.exp(rng.uniform(-60, 60, 200)))
    for a in cases:
        row = np.array([0.25 * a, -a, 0.0])
        assert O.tier_exponent(row) == _brute_exponent(a), a


def test_tier_row_roundtrip_error_bound():
    rng = np.random.default_rng(5)
    for _ in range(50):
        x = rng.standard_normal(128) * np.exp(rng.uniform(-8, 8))
        x = torch.tensor(x).to(torch.bfloat16).double().numpy()
        codes, s = O.tier_quantize_row(x)
        xt = O.e4m3_table()[codes] * 2.0 ** -s
        # codes are torch's E4M3 of x * 2^s
        assert np.array_equal(codes, _torch_e4m3_bytes(torch.tensor(np.ldexp(x, s), dtype=torch.float32)))
        assert np.abs(x).max() * 2.0 ** s <= 448.0
        # relative 2^-4 in the normal range, 2^-10 2^-s absolute below it
        err = np.abs(xt - x)
        assert (err <= np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** (-10 - s))).all()


def _paged_case(seed=7, B=3, Hkv=2, d=16, page=4, lens=(23, 9, 30)):
    rng = np.random.default_rng(seed)
    pages_per = [(n + page - 1) // page for n in lens]
    P = sum(pages_per) + 2
    perm = rng.permutation(P)
    pt = np.full((B, max(pages_per)), -1, dtype=np.int32)
    o = 0
    for b in range(B):
        pt[b, :pages_per[b]] = perm[o:o + pages_per[b]]
        o += pages_per[b]
    grid = lambda a: np.clip(np.round(a * 64), -256, 256) / 64
    K = grid(rng.standard_normal((P, page, Hkv, d)))
    V = grid(rng.standard_normal((P, page, Hkv, d)))
    return O.Layout(B, Hkv, d, 64, page_table=pt, page=page), K, V, np.array(lens, dtype=np.int32), P


def test_demote_pages_follows_the_controller_definition():
    L, K, V, lens, P = _paged_case()
    S, W, page = 2, 5, L.page
    tier, k8, v8, ex = O.tier_arrays(P, page, L.Hkv, L.d)
    protect = np.zeros(P, dtype=np.uint8)
    protect[L.page_table[2, 3]] = 1  # a middle page of sequence 2
    tier[L.page_table[0, 2]] = 1     # already demoted: left as is
    n = O.demote_pages(L, K, V, lens, S, W, tier, k8, v8, ex, protect)
    expect = set()
    for b, N in enumerate(lens):
        for p in range(L.max_pages):
            phys = L.page_table[b, p]
            if phys < 0:
                continue
            toks = range(p * page, (p + 1) * page)
            if all(S <= t < N - W for t in toks) and not protect[phys] and not (b == 0 and p == 2):
                expect.add(int(phys))
    # hand check of sequence 0 (N = 23): middle [2, 18) holds pages 1..3 whole
    assert {int(L.page_table[0, p]) for p in (1, 3)} <= expect
    assert int(L.page_table[0, 0]) not in expect and int(L.page_table[0, 4]) not in expect
    assert n == len(expect)
    assert set(np.nonzero(tier)[0].tolist()) == expect | {int(L.page_table[0, 2])}
    for p in range(P):
        if p in expect:
            for slot in range(page):
                for h in range(L.Hkv):
                    for X, C, j in ((K, k8, 0), (V, v8, 1)):
                        x = X[p, slot, h]
                        s = _brute_exponent(float(np.abs(x).max()))
                        assert ex[p, slot, h, j] == s
                        ref = _torch_e4m3_bytes(torch.tensor(np.ldexp(x, s), dtype=torch.float32))
                        assert np.array_equal(C[p, slot, h], ref)
        else:
            assert not k8[p].any() and not v8[p].any() and not ex[p].any()
    # a second pass demotes nothing new
    assert O.demote_pages(L, K, V, lens, S, W, tier, k8, v8, ex, protect) == 0


def test_attend_tiered_equals_plain_attention_when_fp8_is_exact():
    # rows whose 64x values are integers of magnitude <= 16 (and amax 4 or
    # less: s >= 6) are exact in E4M3 after scaling, so the tiered attention
    # must equal the plain one bit for bit
    L, K, V, lens, P = _paged_case(seed=11)
    rng = np.random.default_rng(2)
    K = rng.integers(-16, 17, K.shape) / 64.0
    V = rng.integers(-16, 17, V.shape) / 64.0
    tier, k8, v8, ex = O.tier_arrays(P, L.page, L.Hkv, L.d)
    assert O.demote_pages(L, K, V, lens, 1, 3, tier, k8, v8, ex) > 0
    Kd, Vd = O.dequantized(K, V, tier, k8, v8, ex)
    assert np.array_equal(Kd, K) and np.array_equal(Vd, V)
    Hq = 2 * L.Hkv
    q = rng.integers(-64, 65, (L.B, Hq, L.d)) / 64.0
    cap = 40
    idx = np.full((L.B, L.Hkv, cap), -1, dtype=np.int32)
    cnt = np.zeros((L.B, L.Hkv), dtype=np.int32)
    for b, N in enumerate(lens):
        for h in range(L.Hkv):
            sel = np.sort(rng.choice(N, size=min(N, 12), replace=False))
            idx[b, h, :sel.size] = sel
            cnt[b, h] = sel.size
    o1, l1 = O.attend(L, Hq, q, K, V, idx, cnt)
    o2, l2 = O.attend_tiered(L, Hq, q, K, V, tier, k8, v8, ex, idx, cnt)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_attend_tiered_reads_dequantized_rows():
    # grid rows up to 4 in magnitude are not all exact in E4M3: the tiered
    # output differs from the plain one, by the rounding of the rows only
    L, K, V, lens, P = _paged_case(seed=13)
    rng = np.random.default_rng(4)
    tier, k8, v8, ex = O.tier_arrays(P, L.page, L.Hkv, L.d)
    O.demote_pages(L, K, V, lens, 1, 3, tier, k8, v8, ex)
    Hq = L.Hkv
    q = np.clip(np.round(rng.standard_normal((L.B, Hq, L.d)) * 64), -256, 256) / 64
    idx = np.full((L.B, L.Hkv, 8), -1, dtype=np.int32)
    cnt = np.zeros((L.B, L.Hkv), dtype=np.int32)
    for b, N in enumerate(lens):
        for h in range(L.Hkv):
            idx[b, h, :4] = [4, 5, 6, 7]  # page 1 of every sequence (in the middle for all three)
            cnt[b, h] = 4
    o1, l1 = O.attend(L, Hq, q, K, V, idx, cnt)
    o2, l2 = O.attend_tiered(L, Hq, q, K, V, tier, k8, v8, ex, idx, cnt)
    Kd, Vd = O.dequantized(K, V, tier, k8, v8, ex)
    o3, l3 = O.attend(L, Hq, q, Kd, Vd, idx, cnt)
    assert np.array_equal(o2, o3) and np.array_equal(l2, l3)
    assert not np.array_equal(o1, o2)
    assert np.allclose(o1, o2, atol=0.5) and np.allclose(l1, l2, atol=2.0)
