"""Precision tiers of pages (Spherical KV page, section 2.2 RDR,
tier-homogeneous pages; DASH-KV page, section "技术架构：动态混合精度机制")
on the GPU against the oracle, through the C ABI.

Every step the GPU appends the step's key, runs the tier controller
(dashkv_demote_pages), selects and decodes with FP8 rows for the demoted pages
(dashkv_sparse_decode_tiered); the oracle does the same from its own copy of
the cache.  Tier bytes, FP8 codes and scale exponents must be bit-identical,
the selection too, and the outputs within the attention tolerance of the
oracle's attention over the dequantized rows.
"""
import ctypes

import numpy as np
import pytest
import torch

from hash_indexed_top_b200 import dashkv as dk
from hash_indexed_top_b200 import workloads as W
from oracle import oracle as O

from pipeline import DeviceRun, OracleRun, assert_exact_scoring, within_tol

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from hash_indexed_top_b200 import build
    build.build()


def _protect_mask(num_pages: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return (rng.random(num_pages) < 0.2).astype(np.uint8)


def run_tier_parity(cfg: W.Config, steps: int, window_decode: bool = True, protect: bool = True) -> None:
    w = W.make_workload(cfg, device="cpu", steps=steps)
    g = DeviceRun(cfg, w.to("cuda"), window=window_decode)
    o = OracleRun(cfg, w)
    P = int(w.K.shape[0])
    pm = _protect_mask(P, cfg.seed) if protect else None
    gpm = torch.from_numpy(pm).cuda() if protect else None
    tiers = dk.PageTiers.empty_for(g.cache)
    ot, ok8, ov8, oex = O.tier_arrays(P, cfg.page_size, cfg.Hkv, cfg.d)
    g.encode()
    demoted = 0
    try:
        for s in range(steps):
            g.append(s)
            o.append(s)
            g.eng.demote_pages(g.cache, tiers, g.seq, gpm)
            demoted += O.demote_pages(o.L, o.K, o.V, o.seq, cfg.sink, cfg.window, ot, ok8, ov8, oex, pm)
            q = w.q[s]
            b = g.buf
            g.eng.select(g.cache, q.cuda(), g.seq, b["sel_idx"], b["sel_cnt"], g.scores)
            g.eng.sparse_decode_tiered(g.cache, tiers, q.cuda(), b["sel_idx"], b["sel_cnt"], b["out"], b["lse"],
                                       seq_lens=g.seq if window_decode else None)
            assert g.error() == 0
            what = f"{cfg.name} step {s}"
            assert np.array_equal(tiers.tier.cpu().numpy(), ot), f"{what}: tier bytes differ"
            assert np.array_equal(tiers.exps.cpu().numpy(), oex), f"{what}: exponents differ"
            for name, a, e in (("k8", tiers.k8, ok8), ("v8", tiers.v8, ov8)):
                a = a.cpu().numpy()
                assert np.array_equal(a, e), f"{what}: {name} differs at {np.argwhere(a != e)[:4].tolist()}"
            r = o.step(q)
            assert_exact_scoring(r["bound"], what)
            assert np.array_equal(b["sel_cnt"].cpu().numpy(), r["sel_cnt"]), f"{what}: sel_cnt differ"
            assert np.array_equal(b["sel_idx"].cpu().numpy(), r["sel_idx"]), f"{what}: sel_idx differ"
            ro, rl = O.attend_tiered(o.L, cfg.Hq, q.double().numpy(), o.K, o.V, ot, ok8, ov8, oex, r["sel_idx"],
                                     r["sel_cnt"])
            out = b["out"].cpu().double().numpy()
            lse = b["lse"].cpu().double().numpy()
            assert within_tol(out, ro).all(), f"{what}: out max err {np.nanmax(np.abs(out - ro)):.3e}"
            assert within_tol(lse, rl).all(), f"{what}: lse max err {np.nanmax(np.abs(lse - rl)):.3e}"
        # the case is only a test of the FP8 path if pages were demoted and selected
        assert demoted > 0 and ot.any()
    finally:
        g.close()


CASES = {
    # pages of 32 tokens and a 40-token window: pages leave the window during
    # the run and are demoted on the way
    "g4_b64_d128": (W.CONFIGS["ragged_paged"].scaled(name="t_g4", B=3, N=2500, n_min=300, topk=200, sink=3,
                                                     window=40, page_size=32, steps=40), 40),
    "g8_b128_d128": (W.CONFIGS["c1m"].scaled(name="t_g8", B=2, N=3000, topk=256, window=64, page_size=32,
                                             steps=8), 8),
    "g1_b32_d64": (W.Config("t_g1", B=2, Hq=4, Hkv=4, d=64, N=1800, bits=32, topk=100, sink=0, window=33,
                            steps=6, needles=4, page_size=32, n_min=500, seed=311), 6),
    "g2_b64_d64": (W.Config("t_g2", B=3, Hq=8, Hkv=4, d=64, N=1500, bits=64, topk=64, sink=5, window=70,
                            steps=3, needles=4, page_size=64, seed=313), 3),
}


@pytest.mark.parametrize("window_decode", [True, False])
@pytest.mark.parametrize("name", list(CASES))
def test_tiers_match_oracle(name, window_decode):
    cfg, steps = CASES[name]
    run_tier_parity(cfg, steps, window_decode=window_decode)


def test_tiers_without_protection():
    cfg, _ = CASES["g4_b64_d128"]
    run_tier_parity(cfg.scaled(name="t_g4_noprot", steps=3), 3, protect=False)


def test_tiered_decode_without_demoted_pages_is_the_plain_decode():
    cfg, _ = CASES["g8_b128_d128"]
    w = W.make_workload(cfg, device="cuda", steps=1)
    g = DeviceRun(cfg, w)
    try:
        g.encode()
        g.append(0)
        tiers = dk.PageTiers.empty_for(g.cache)
        b = g.buf
        g.eng.select(g.cache, w.q[0], g.seq, b["sel_idx"], b["sel_cnt"], g.scores)
        g.eng.sparse_decode(g.cache, w.q[0], b["sel_idx"], b["sel_cnt"], b["out"], b["lse"], seq_lens=g.seq)
        out0, lse0 = b["out"].clone(), b["lse"].clone()
        g.eng.sparse_decode_tiered(g.cache, tiers, w.q[0], b["sel_idx"], b["sel_cnt"], b["out"], b["lse"],
                                   seq_lens=g.seq)
        assert g.error() == 0
        assert torch.allclose(out0, b["out"], rtol=1e-6, atol=1e-6)
        assert torch.allclose(lse0, b["lse"], rtol=1e-6, atol=1e-6)
    finally:
        g.close()


def test_tier_calls_reject_dense_caches_and_bad_views():
    cfg = W.Config("t_dense", B=1, Hq=4, Hkv=1, d=128, N=512, bits=64, topk=32, sink=2, window=16, steps=1,
                   needles=0, seed=5)
    w = W.make_workload(cfg, device="cuda", steps=1)
    g = DeviceRun(cfg, w)
    try:
        z = torch.zeros(64, dtype=torch.uint8, device="cuda")
        tv = dk.TierView(z.data_ptr(), z.data_ptr(), z.data_ptr(), z.data_ptr())
        v = g.cache.view()
        L = dk.lib()
        assert L.dashkv_demote_pages(g.eng._ctx, ctypes.byref(v), ctypes.byref(tv), g.seq.data_ptr(), None,
                                     None) == 2
        assert L.dashkv_demote_pages(g.eng._ctx, ctypes.byref(v), None, g.seq.data_ptr(), None, None) == 1
        bad = dk.TierView(z.data_ptr(), z.data_ptr() + 1, z.data_ptr(), z.data_ptr())
        pcfg = CASES["g2_b64_d64"][0]
        pw = W.make_workload(pcfg, device="cuda", steps=1)
        pg = DeviceRun(pcfg, pw)
        try:
            pv = pg.cache.view()
            assert L.dashkv_demote_pages(pg.eng._ctx, ctypes.byref(pv), ctypes.byref(bad), pg.seq.data_ptr(), None,
                                         None) == 1
        finally:
            pg.close()
    finally:
        g.close()


def test_demote_reports_a_page_id_beyond_the_pool():
    # the view declares 4 pages fewer than the buffers hold and one page-table
    # entry points into that margin: the controller must skip it and report it
    # (were the check missing, the access would still land inside the buffers)
    cfg, _ = CASES["g2_b64_d64"]
    w = W.make_workload(cfg, device="cuda", steps=1)
    g = DeviceRun(cfg, w)
    try:
        g.encode()
        P = int(w.K.shape[0])
        tiers = dk.PageTiers.empty_for(g.cache)  # arrays for all P allocated pages
        pt = w.page_table.clone()
        pt[0, 1] = P - 2
        view = g.cache.view()
        view.page_table = pt.data_ptr()
        view.num_pages = P - 4
        t = tiers.view()
        st = dk.lib().dashkv_demote_pages(g.eng._ctx, ctypes.byref(view), ctypes.byref(t), g.seq.data_ptr(), None,
                                          None)
        assert st == 0
        assert g.eng.get_error() == 6
        tier = tiers.tier.cpu()
        assert int(tier[P - 2]) == 0  # beyond the declared pool: skipped
        assert int(tier[:P - 4].sum()) > 0  # the pages inside it were demoted as usual
    finally:
        g.close()


def _pair_pages(w: W.Workload, b: int, n: int) -> np.ndarray:
    ps = w.cfg.page_size
    return w.page_table[b, :(n + ps - 1) // ps].long().cpu().numpy()


def test_full_size_ragged_paged_tiers_on_sampled_pairs():
    # the ragged paged workload at full size: controller at prefill and after
    # the step's append, then selection and the tiered decode; the first and
    # last (sequence, kv head) pairs against the oracle on the pair's own pages
    cfg = W.CONFIGS["ragged_paged"]
    dev = torch.device("cuda")
    w = W.make_workload(cfg, device=dev, steps=1)
    eng = dk.DashKV(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.bits, cfg.topk, cfg.sink, cfg.window, cfg.page_size,
                    W.HYPERPLANE_SEED)
    try:
        cache = dk.KVCache(w.K, w.V, dk.KVCache.empty_codes_like(w.K, cfg.bits, True), w.page_table)
        tiers = dk.PageTiers.empty_for(cache)
        seq = w.seq_lens.clone()
        eng.encode_keys(cache, seq)
        eng.demote_pages(cache, tiers, seq)
        eng.append_keys(cache, w.k_new[0], w.v_new[0], seq)
        eng.demote_pages(cache, tiers, seq)
        buf = eng.alloc_step(dev)
        ws = eng.workspace(cache.capacity, dev)
        eng.select(cache, w.q[0], seq, buf["sel_idx"], buf["sel_cnt"], None, ws)
        eng.sparse_decode_tiered(cache, tiers, w.q[0], buf["sel_idx"], buf["sel_cnt"], buf["out"], buf["lse"], ws,
                                 seq_lens=seq)
        torch.cuda.synchronize()
        assert eng.get_error() == 0
        R = O.hyperplanes(W.HYPERPLANE_SEED, cfg.bits, cfg.d)
        G, ps = cfg.G, cfg.page_size
        for b, h in [(0, 0), (cfg.B - 1, cfg.Hkv - 1)]:
            n = int(seq[b])
            pages = _pair_pages(w, b, n)
            npg = pages.size
            # the pair's own paged cache: local page i = physical page pages[i], head h only
            K = w.K[pages][:, :, h:h + 1].double().cpu().numpy()
            V = w.V[pages][:, :, h:h + 1].double().cpu().numpy()
            L = O.Layout(1, 1, cfg.d, cfg.bits, page_table=np.arange(npg, dtype=np.int32).reshape(1, npg), page=ps)
            sl = np.array([n], dtype=np.int32)
            oc = O.encode(L, K, sl, R)
            ot, ok8, ov8, oex = O.tier_arrays(npg, ps, 1, cfg.d)
            O.demote_pages(L, K, V, sl, cfg.sink, cfg.window, ot, ok8, ov8, oex)
            what = f"ragged_paged ({b},{h})"
            assert np.array_equal(tiers.tier[pages].cpu().numpy(), ot), f"{what}: tier bytes differ"
            assert ot.sum() > npg // 2, f"{what}: most pages should be demoted"
            assert np.array_equal(tiers.exps[pages][:, :, h:h + 1].cpu().numpy(), oex), f"{what}: exponents differ"
            assert np.array_equal(tiers.k8[pages][:, :, h:h + 1].cpu().numpy(), ok8), f"{what}: k8 differs"
            assert np.array_equal(tiers.v8[pages][:, :, h:h + 1].cpu().numpy(), ov8), f"{what}: v8 differs"
            q = w.q[0][b, h * G:(h + 1) * G].double().cpu().numpy().reshape(1, G, cfg.d)
            r = O.decode_step(L, G, q, K, V, oc, sl, R, cfg.topk, cfg.sink, cfg.window)
            assert_exact_scoring(r["bound"], what)
            assert int(buf["sel_cnt"][b, h]) == int(r["sel_cnt"][0, 0]), f"{what}: sel_cnt"
            assert np.array_equal(buf["sel_idx"][b, h].cpu().numpy(), r["sel_idx"][0, 0]), f"{what}: selection"
            ro, rl = O.attend_tiered(L, G, q, K, V, ot, ok8, ov8, oex, r["sel_idx"], r["sel_cnt"])
            out = buf["out"][b, h * G:(h + 1) * G].double().cpu().numpy()
            lse = buf["lse"][b, h * G:(h + 1) * G].double().cpu().numpy()
            assert within_tol(out, ro[0]).all(), f"{what}: out err {np.abs(out - ro[0]).max()}"
            assert within_tol(lse, rl[0]).all(), f"{what}: lse err {np.abs(lse - rl[0]).max()}"
    finally:
        eng.close()
