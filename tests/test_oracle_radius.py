"""Pins of the oracle's radius-scaled scores (Spherical KV page, section 2.1
ADA: a quantized key radius beside the angle code scales the estimated
logit) against facts that do not come from the oracle itself: a hand-worked
example, the integer form of the quantizer on the 1/64 grid (isqrt instead of
an fp32 square root), and invariants of a norm-preserving change of the keys.
A wrong step, a missing half-step, a radius taken from the query or a scale
applied before the fp32 rounding of the score fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _grid(rng, shape):
    return np.clip(np.round(rng.standard_normal(shape) * 64.0), -256, 256) / 64.0


def test_radius_worked_example():
    with open(os.path.join(GOLD, "hadamard4_radius_example.json")) as f:
        g = json.load(f)
    R = np.array(g["R"], dtype=np.int8)
    K = np.array(g["K"], dtype=np.float64)[None, None]
    q = np.array(g["q"], dtype=np.float64)[None]
    L = O.Layout(B=1, Hkv=1, d=4, bits=4, n_cap=6)
    seq = np.array([6], dtype=np.int32)
    codes = O.encode(L, K, seq, R)
    assert codes[0, 0, :, 0].tolist() == g["codes"]
    rc = O.radius_codes(L, K, seq)
    assert rc[0, 0].tolist() == g["radius_codes"]
    sc, _ = O.scores(L, 2, q, codes, seq, R)
    assert sc[0, 0].tolist() == g["unscaled"]
    ss = O.radius_scale(L, sc, seq, rc)
    assert ss[0, 0].tolist() == g["scaled"]
    for c in g["select_cases"]:
        idx, cnt = O.select(ss, seq, c["topk"], c["sink"], c["window"])
        assert idx[0, 0, :cnt[0, 0]].tolist() == c["sel"]
        idx, cnt = O.select(sc, seq, c["topk"], c["sink"], c["window"])
        assert idx[0, 0, :cnt[0, 0]].tolist() == c["unscaled_sel"]


def test_radius_code_values_and_clip():
    assert O.radius_code([0.0] * 8) == 0
    assert O.radius_code([0.25, 0.0]) == 1                # 4 * 0.25 = 1 exactly
    assert O.radius_code([3.0, 0.0, 0.0, 0.0]) == 12
    assert O.radius_code([0.5] * 4) == 4                  # norm 1
    assert O.radius_code([-4.0] * 128) == math.floor(4 * 4 * math.sqrt(128))  # largest grid norm, 181
    assert O.radius_code([100.0] * 4) == 255              # beyond the range: clipped
    assert [O.radius_value(c) for c in (0, 1, 12, 255)] == [0.125, 0.375, 3.125, 63.875]


def _squares_summing_to(target: int, d: int) -> np.ndarray:
    """d integers in [0, 256] whose squares sum to target (greedy; target at
    most about 100 * 256^2, so the greedy tail fits in the dims left)."""
    m = np.zeros(d)
    rest, i = target, 0
    while rest:
        v = min(256, math.isqrt(rest))
        m[i] = v
        rest -= v * v
        i += 1
    assert i <= d
    return m


def test_radius_code_equals_integer_isqrt_on_the_grid():
    # on the grid k_i = m_i / 64: 4 |k| = sqrt(S) / 16 with S = sum m_i^2, so
    # the code is isqrt(S) // 16 -- including every S just below a step
    rng = np.random.default_rng(21)
    d = 128
    cases = [np.clip(np.round(rng.standard_normal(d) * 64.0 * s), -256, 256) for s in (0.01, 0.3, 1, 2, 4, 8)
             for _ in range(200)]
    for n in range(1, 161):  # S = 256 n^2 - 1 sits just below the n-th step
        cases.append(_squares_summing_to(256 * n * n - 1, d))
    for m in cases:
        S = int(np.sum(m.astype(np.int64) ** 2))
        assert O.radius_code(m / 64.0) == min(255, math.isqrt(S) // 16), S


def test_equal_norms_leave_the_selection_unchanged():
    # permutations and sign flips of one grid key keep its norm (so every key
    # has the same radius code): scaling by one positive r~ keeps the order
    rng = np.random.default_rng(22)
    B, Hkv, G, d, bits, n = 1, 2, 4, 64, 64, 300
    base = _grid(rng, d)
    K = np.empty((B, Hkv, n, d))
    for h in range(Hkv):
        for t in range(n):
            K[0, h, t] = base[rng.permutation(d)] * rng.choice([-1.0, 1.0], size=d)
    R = O.hyperplanes(7, bits, d)
    L = O.Layout(B, Hkv, d, bits, n_cap=n)
    seq = np.array([n], dtype=np.int32)
    codes = O.encode(L, K, seq, R)
    rc = O.radius_codes(L, K, seq)
    assert len(np.unique(rc)) == 1
    q = _grid(rng, (B, Hkv * G, d))
    sc, _ = O.scores(L, Hkv * G, q, codes, seq, R)
    ss = O.radius_scale(L, sc, seq, rc)
    for k in (1, 17, 100, 299):
        a = O.select(sc, seq, k, 3, 5)
        b = O.select(ss, seq, k, 3, 5)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_scaling_a_key_keeps_its_code_and_scales_its_radius():
    rng = np.random.default_rng(23)
    d, bits = 128, 128
    R = O.hyperplanes(8, bits, d)
    K = np.clip(_grid(rng, (1, 1, 64, d)), -2, 2)
    K2 = K * 2.0  # still on the grid
    L = O.Layout(1, 1, d, bits, n_cap=64)
    seq = np.array([64], dtype=np.int32)
    assert np.array_equal(O.encode(L, K, seq, R), O.encode(L, K2, seq, R))
    r1 = O.radius_codes(L, K, seq).astype(int)
    r2 = O.radius_codes(L, K2, seq).astype(int)
    assert np.all((r2 == 2 * r1) | (r2 == 2 * r1 + 1))  # floor(2x) from floor(x)


def test_radius_paged_equals_dense():
    rng = np.random.default_rng(24)
    B, Hkv, d, ps, pages = 2, 2, 64, 32, 4
    P = B * pages
    pt = rng.permutation(P).reshape(B, pages).astype(np.int32)
    Kp = _grid(rng, (P, ps, Hkv, d))
    seq = np.array([100, 57], dtype=np.int32)
    Kd = np.zeros((B, Hkv, pages * ps, d))
    for b in range(B):
        for t in range(pages * ps):
            Kd[b, :, t] = Kp[pt[b, t // ps], t % ps]
    Lp = O.Layout(B, Hkv, d, 64, page_table=pt, page=ps)
    Ld = O.Layout(B, Hkv, d, 64, n_cap=pages * ps)
    rp = O.radius_codes(Lp, Kp, seq)
    rd = O.radius_codes(Ld, Kd, seq)
    for b in range(B):
        for t in range(int(seq[b])):
            assert np.array_equal(rp[pt[b, t // ps], :, t % ps], rd[b, :, t])
