"""Full-size parity: every configured long-context workload at its full size.

test_full_size_decode_steps_every_pair runs the configured number of decode
steps exactly as the benchmark times them -- each step one
dashkv_decode_step call captured in a CUDA graph and replayed -- and checks
every (sequence, kv head) pair of every step against the oracle: selection
(bit for bit), attention output and lse of the pair's query heads (within
tolerance), and at the end the pair's codes, cached keys and values.  The
oracle starts from its own encode of a copy of the prefilled cache taken
before the GPU ran and appends the step inputs itself (no GPU value enters
it); pairs are checked one at a time so host memory holds one pair.

test_full_size_select_scores_on_sampled_pairs checks the selection call with
its scores output (fp32 scores bit for bit) on the first and last pair, and
the block-summary workloads are checked the same way, summaries and block
scores included."""
import numpy as np
import pytest
import torch

from hash_indexed_top_b200 import dashkv as dk
from hash_indexed_top_b200 import workloads as W
from oracle import oracle as O

from pipeline import assert_exact_scoring, within_tol

pytestmark = pytest.mark.gpu

FULL = ["c32k", "c128k", "ragged_paged", "c1m"]


def _pair_rows(x: torch.Tensor, w: W.Workload, b: int, h: int, n: int) -> torch.Tensor:
    """Rows [0, n) of kv head h of sequence b: [n, ...] (dense or through the page table)."""
    if not w.paged:
        return x[b, h, :n]
    ps = w.cfg.page_size
    t = torch.arange(n, device=x.device)
    pages = w.page_table[b].long()[t // ps]
    return x[pages, t % ps, h]


def _pair_codes(codes: torch.Tensor, w: W.Workload, b: int, h: int, n: int) -> torch.Tensor:
    if not w.paged:
        return codes[b, h, :n]
    ps = w.cfg.page_size
    t = torch.arange(n, device=codes.device)
    pages = w.page_table[b].long()[t // ps]
    return codes[pages, h, t % ps]


@pytest.mark.parametrize("name", FULL)
def test_full_size_decode_steps_every_pair(name):
    cfg = W.CONFIGS[name]
    steps = cfg.steps
    dev = torch.device("cuda")
    w = W.make_workload(cfg, device=dev, steps=steps)
    K0, V0 = w.K.clone(), w.V.clone()  # the prefilled cache, for the oracle
    eng = dk.DashKV(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.bits, cfg.topk, cfg.sink, cfg.window,
                    cfg.page_size if w.paged else 0, W.HYPERPLANE_SEED)
    rec = []
    try:
        cache = dk.KVCache(w.K, w.V, dk.KVCache.empty_codes_like(w.K, cfg.bits, w.paged), w.page_table)
        seq = w.seq_lens.clone()
        eng.encode_keys(cache, seq)
        buf = eng.alloc_step(dev)
        ws = eng.workspace(cache.capacity, dev)
        torch.cuda.synchronize()
        for s in range(steps):  # one captured graph per step, as the benchmark replays them
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                eng.decode_step(cache, w.q[s], w.k_new[s], w.v_new[s], seq, buf["sel_idx"], buf["sel_cnt"],
                                buf["out"], buf["lse"], ws)
            g.replay()
            torch.cuda.synchronize()
            rec.append({k: v.cpu() for k, v in buf.items()})
            del g
        assert eng.get_error() == 0
        gcodes = dk.canonical_codes(cache.codes, cfg.bits)
        R = O.hyperplanes(W.HYPERPLANE_SEED, cfg.bits, cfg.d)
        G = cfg.G
        assert torch.equal(seq.cpu(), w.seq_lens.cpu() + steps)
        for b in range(cfg.B):
            n0 = int(w.seq_lens[b])
            for h in range(cfg.Hkv):
                cap = n0 + steps
                L = O.Layout(1, 1, cfg.d, cfg.bits, n_cap=cap)
                K = np.zeros((1, 1, cap, cfg.d))
                V = np.zeros((1, 1, cap, cfg.d))
                K[0, 0, :n0] = _pair_rows(K0, w, b, h, n0).double().cpu().numpy()
                V[0, 0, :n0] = _pair_rows(V0, w, b, h, n0).double().cpu().numpy()
                sl = np.array([n0], dtype=np.int32)
                oc = O.encode(L, K, sl, R)
                for s in range(steps):
                    O.append(L, K, V, oc, sl, w.k_new[s][b:b + 1, h:h + 1].double().cpu().numpy(),
                             w.v_new[s][b:b + 1, h:h + 1].double().cpu().numpy(), R)
                    q = w.q[s][b, h * G:(h + 1) * G].double().cpu().numpy().reshape(1, G, cfg.d)
                    r = O.decode_step(L, G, q, K, V, oc, sl, R, cfg.topk, cfg.sink, cfg.window)
                    what = f"{name} step {s} ({b},{h})"
                    assert_exact_scoring(r["bound"], what)
                    got = rec[s]
                    assert int(got["sel_cnt"][b, h]) == int(r["sel_cnt"][0, 0]), f"{what}: sel_cnt"
                    assert np.array_equal(got["sel_idx"][b, h].numpy(), r["sel_idx"][0, 0]), f"{what}: selection"
                    out = got["out"][b, h * G:(h + 1) * G].double().numpy()
                    lse = got["lse"][b, h * G:(h + 1) * G].double().numpy()
                    assert within_tol(out, r["out"][0]).all(), f"{what}: out err {np.abs(out - r['out'][0]).max()}"
                    assert within_tol(lse, r["lse"][0]).all(), f"{what}: lse err {np.abs(lse - r['lse'][0]).max()}"
                n = int(sl[0])
                gc = _pair_codes(gcodes, w, b, h, n).cpu().numpy().view(np.uint64)
                assert np.array_equal(gc, oc[0, 0, :n]), f"{name} ({b},{h}): codes differ"
                assert np.array_equal(_pair_rows(w.K, w, b, h, n).double().cpu().numpy(), K[0, 0, :n]), \
                    f"{name} ({b},{h}): cached keys differ"
                assert np.array_equal(_pair_rows(w.V, w, b, h, n).double().cpu().numpy(), V[0, 0, :n]), \
                    f"{name} ({b},{h}): cached values differ"
    finally:
        eng.close()


@pytest.mark.parametrize("name", FULL)
def test_full_size_select_scores_on_sampled_pairs(name):
    cfg = W.CONFIGS[name]
    dev = torch.device("cuda")
    w = W.make_workload(cfg, device=dev, steps=1)
    eng = dk.DashKV(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.bits, cfg.topk, cfg.sink, cfg.window,
                    cfg.page_size if w.paged else 0, W.HYPERPLANE_SEED)
    try:
        cache = dk.KVCache(w.K, w.V, dk.KVCache.empty_codes_like(w.K, cfg.bits, w.paged), w.page_table)
        seq = w.seq_lens.clone()
        eng.encode_keys(cache, seq)
        eng.append_keys(cache, w.k_new[0], w.v_new[0], seq)
        buf = eng.alloc_step(dev)
        scores = torch.full((cfg.B, cfg.Hkv, cache.capacity), float("nan"), device=dev)
        ws = eng.workspace(cache.capacity, dev)
        eng.select(cache, w.q[0], seq, buf["sel_idx"], buf["sel_cnt"], scores, ws)
        eng.sparse_decode(cache, w.q[0], buf["sel_idx"], buf["sel_cnt"], buf["out"], buf["lse"], ws, seq_lens=seq)
        torch.cuda.synchronize()
        assert eng.get_error() == 0
        gcodes = dk.canonical_codes(cache.codes, cfg.bits)
        R = O.hyperplanes(W.HYPERPLANE_SEED, cfg.bits, cfg.d)
        G = cfg.G
        for b, h in [(0, 0), (cfg.B - 1, cfg.Hkv - 1)]:
            n = int(seq[b])
            K = _pair_rows(w.K, w, b, h, n).double().cpu().numpy().reshape(1, 1, n, cfg.d)
            V = _pair_rows(w.V, w, b, h, n).double().cpu().numpy().reshape(1, 1, n, cfg.d)
            L = O.Layout(1, 1, cfg.d, cfg.bits, n_cap=n)
            sl = np.array([n], dtype=np.int32)
            oc = O.encode(L, K, sl, R)
            gc = _pair_codes(gcodes, w, b, h, n).cpu().numpy().view(np.uint64)
            assert np.array_equal(gc, oc[0, 0]), f"{name} ({b},{h}): codes differ at {np.argwhere(gc != oc[0, 0])[:3]}"
            q = w.q[0][b, h * G:(h + 1) * G].double().cpu().numpy().reshape(1, G, cfg.d)
            r = O.decode_step(L, G, q, K, V, oc, sl, R, cfg.topk, cfg.sink, cfg.window)
            assert_exact_scoring(r["bound"], f"{name} ({b},{h})")
            gs = scores[b, h, :n].cpu().numpy()
            es = r["scores"][0, 0, :n].astype(np.float32)
            assert np.array_equal(gs.view(np.uint32), es.view(np.uint32)), \
                f"{name} ({b},{h}): scores differ at {np.argwhere(gs != es)[:3].ravel()}"
            cnt = int(buf["sel_cnt"][b, h])
            assert cnt == int(r["sel_cnt"][0, 0]), f"{name} ({b},{h}): sel_cnt {cnt} vs {int(r['sel_cnt'][0, 0])}"
            assert np.array_equal(buf["sel_idx"][b, h].cpu().numpy(), r["sel_idx"][0, 0]), \
                f"{name} ({b},{h}): selection differs"
            out = buf["out"][b, h * G:(h + 1) * G].double().cpu().numpy()
            lse = buf["lse"][b, h * G:(h + 1) * G].double().cpu().numpy()
            assert within_tol(out, r["out"][0]).all(), f"{name} ({b},{h}): out err {np.abs(out - r['out'][0]).max()}"
            assert within_tol(lse, r["lse"][0]).all(), f"{name} ({b},{h}): lse err {np.abs(lse - r['lse'][0]).max()}"
    finally:
        eng.close()


BLOCK_FULL = ["c128k_blocks4", "c1m_blocks4"]


@pytest.mark.parametrize("name", BLOCK_FULL)
def test_full_size_block_step_on_sampled_pairs(name):
    # one step through block summaries as the benchmark runs it (append,
    # summary update, block selection, decode given the lengths); the oracle
    # encodes the pair's summaries from its keys
    cfg = W.CONFIGS[name]
    m = cfg.block
    dev = torch.device("cuda")
    w = W.make_workload(cfg, device=dev, steps=1)
    eng = dk.DashKV(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.bits, cfg.topk, cfg.sink, cfg.window,
                    cfg.page_size if w.paged else 0, W.HYPERPLANE_SEED)
    try:
        cache = dk.KVCache(w.K, w.V, dk.KVCache.empty_codes_like(w.K, cfg.bits, w.paged), w.page_table)
        seq = w.seq_lens.clone()
        eng.encode_keys(cache, seq)
        index = dk.BlockIndex.empty_for(cache, cfg.B, cfg.bits, m)
        eng.encode_blocks(cache, index, seq)
        eng.append_keys(cache, w.k_new[0], w.v_new[0], seq)
        eng.append_blocks(cache, index, seq)
        buf = eng.alloc_step(dev)
        bsc = torch.full((cfg.B, cfg.Hkv, index.capacity), float("nan"), device=dev)
        ws = eng.workspace(cache.capacity, dev)
        eng.select_blocks(cache, index, w.q[0], seq, buf["sel_idx"], buf["sel_cnt"], bsc, ws)
        eng.sparse_decode(cache, w.q[0], buf["sel_idx"], buf["sel_cnt"], buf["out"], buf["lse"], ws, seq_lens=seq)
        torch.cuda.synchronize()
        assert eng.get_error() == 0
        gcodes = dk.canonical_codes(index.codes, cfg.bits)
        R = O.hyperplanes(W.HYPERPLANE_SEED, cfg.bits, cfg.d)
        G = cfg.G
        for b, h in [(0, 0), (cfg.B - 1, cfg.Hkv - 1)]:
            n = int(seq[b])
            nb = n // m
            K = _pair_rows(w.K, w, b, h, n).double().cpu().numpy().reshape(1, 1, n, cfg.d)
            V = _pair_rows(w.V, w, b, h, n).double().cpu().numpy().reshape(1, 1, n, cfg.d)
            L = O.Layout(1, 1, cfg.d, cfg.bits, n_cap=n)
            sl = np.array([n], dtype=np.int32)
            oc = O.encode_blocks(L, K, sl, m, R, nb_cap=max(1, nb))
            gc = gcodes[b, h, :nb].cpu().numpy().view(np.uint64)
            assert np.array_equal(gc, oc[0, 0, :nb]), f"{name} ({b},{h}): summaries differ"
            q = w.q[0][b, h * G:(h + 1) * G].double().cpu().numpy().reshape(1, G, cfg.d)
            r = O.decode_step_blocks(L, G, q, K, V, oc, sl, R, m, cfg.topk // m, cfg.sink, cfg.window,
                                     cap=cfg.sel_cap)
            gs = bsc[b, h, :nb].cpu().numpy()
            es = r["block_scores"][0, 0, :nb].astype(np.float32)
            assert np.array_equal(gs.view(np.uint32), es.view(np.uint32)), f"{name} ({b},{h}): block scores differ"
            assert int(buf["sel_cnt"][b, h]) == int(r["sel_cnt"][0, 0])
            assert np.array_equal(buf["sel_idx"][b, h].cpu().numpy(), r["sel_idx"][0, 0]), \
                f"{name} ({b},{h}): selection differs"
            out = buf["out"][b, h * G:(h + 1) * G].double().cpu().numpy()
            lse = buf["lse"][b, h * G:(h + 1) * G].double().cpu().numpy()
            assert within_tol(out, r["out"][0]).all(), f"{name} ({b},{h}): out err {np.abs(out - r['out'][0]).max()}"
            assert within_tol(lse, r["lse"][0]).all(), f"{name} ({b},{h}): lse err {np.abs(lse - r['lse'][0]).max()}"
    finally:
        eng.close()
