"""Block summaries (CSA-style two-level index) on the GPU against the oracle,
through the C ABI.

Every step: the GPU appends the step's key, updates the summary of a block the
append completed (dashkv_append_blocks), selects through the summaries and
decodes; the oracle re-encodes every summary of its cache from scratch and
runs its block-score / block-select / attend.  Summary codes, block scores and
the token lists must be bit-identical, outputs within the attention tolerance.
Step counts are chosen so that appends complete blocks.
"""
import numpy as np
import pytest
import torch

from hash_indexed_top_b200 import dashkv as dk
from hash_indexed_top_b200 import workloads as W
from oracle import oracle as O

from pipeline import DeviceRun, OracleRun, within_tol

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def built():
    from hash_indexed_top_b200 import build
    build.build()


def run_block_parity(cfg: W.Config, steps: int, window_decode: bool = True, two_kernel: bool = False,
                     mutate=None) -> list:
    m = cfg.block
    w = W.make_workload(cfg, device="cpu", steps=steps)
    if mutate is not None:
        w = mutate(w)
    g = DeviceRun(cfg, w.to("cuda"), two_kernel=two_kernel, window=window_decode)
    o = OracleRun(cfg, w)
    index = dk.BlockIndex.empty_for(g.cache, cfg.B, cfg.bits, m)
    nb_cap = index.capacity
    g.encode()
    g.eng.encode_blocks(g.cache, index, g.seq)
    counts = []
    try:
        for s in range(steps):
            g.append(s)
            g.eng.append_blocks(g.cache, index, g.seq)
            o.append(s)
            q = w.q[s]
            bsc = torch.full((cfg.B, cfg.Hkv, nb_cap), float("nan"), device="cuda")
            b = g.buf
            g.eng.select_blocks(g.cache, index, q.cuda(), g.seq, b["sel_idx"], b["sel_cnt"], bsc)
            g.eng.sparse_decode(g.cache, q.cuda(), b["sel_idx"], b["sel_cnt"], b["out"], b["lse"],
                                seq_lens=g.seq if window_decode else None)
            assert g.error() == 0
            what = f"{cfg.name} m={m} step {s}"
            oc = O.encode_blocks(o.L, o.K, o.seq, m, o.R, nb_cap)
            gc = dk.canonical_codes(index.codes, cfg.bits).cpu().numpy().view(np.uint64)
            assert np.array_equal(gc, oc), f"{what}: summaries differ at {np.argwhere(gc != oc)[:5].tolist()}"
            assert np.array_equal(g.seq.cpu().numpy(), o.seq)
            r = O.decode_step_blocks(o.L, cfg.Hq, q.double().numpy(), o.K, o.V, oc, o.seq, o.R, m, cfg.topk // m,
                                     cfg.sink, cfg.window, cap=cfg.sel_cap)
            gs = bsc.cpu().numpy()
            es = r["block_scores"].astype(np.float32)
            for bb in range(cfg.B):
                nb = int(o.seq[bb]) // m
                assert np.array_equal(gs[bb, :, :nb].view(np.uint32), es[bb, :, :nb].view(np.uint32)), \
                    f"{what}: block scores differ (b={bb})"
            gn = b["sel_cnt"].cpu().numpy()
            assert np.array_equal(gn, r["sel_cnt"]), f"{what}: sel_cnt {gn.ravel()[:8]} vs {r['sel_cnt'].ravel()[:8]}"
            assert np.array_equal(b["sel_idx"].cpu().numpy(), r["sel_idx"]), f"{what}: sel_idx differ"
            out = b["out"].cpu().double().numpy()
            lse = b["lse"].cpu().double().numpy()
            assert within_tol(out, r["out"]).all(), f"{what}: out max err {np.nanmax(np.abs(out - r['out'])):.3e}"
            assert within_tol(lse, r["lse"]).all(), f"{what}: lse max err {np.nanmax(np.abs(lse - r['lse'])):.3e}"
            counts.append(gn.copy())
    finally:
        g.close()
    return counts


CASES = {
    # (config, steps): lengths and steps put block boundaries inside the run
    "c128k_small_m4": (W.CONFIGS["c128k"].scaled(name="c128k_small_m4", B=2, N=6001, topk=512, steps=4, block=4),
                       4),
    "c32k_small_m8": (W.CONFIGS["c32k"].scaled(name="c32k_small_m8", N=4003, topk=256, window=16, steps=6, block=8),
                      6),
    "ragged_paged_m16": (W.CONFIGS["ragged_paged"].scaled(name="ragged_paged_m16", B=5, N=5000, n_min=700, topk=320,
                                                          window=40, steps=3, block=16), 3),
    "c1m_small_m4": (W.CONFIGS["c1m"].scaled(name="c1m_small_m4", N=20001, topk=1024, steps=3, block=4), 3),
    "d64_b32_m2": (W.Config("d64_b32_m2", B=3, Hq=8, Hkv=4, d=64, N=3333, bits=32, topk=100, sink=2, window=5,
                            steps=3, needles=4, seed=91, block=2), 3),
    "g1_b64_paged32_m64": (W.Config("g1_b64_paged32_m64", B=2, Hq=2, Hkv=2, d=128, N=1500, n_min=100, bits=64,
                                    topk=256, sink=0, window=63, steps=2, needles=2, page_size=32, seed=92,
                                    block=64), 2),
}

PATHS = {"fused": dict(two_kernel=False, window_decode=True),
         "fused_list_decode": dict(two_kernel=False, window_decode=False),
         "two_kernel": dict(two_kernel=True, window_decode=True)}


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("name", list(CASES))
def test_block_parity(name, path):
    cfg, steps = CASES[name]
    assert len(run_block_parity(cfg, steps, **PATHS[path])) == steps


def test_blocks_of_one_token_equal_the_token_selection():
    # m = 1: the block path must give the token path's list, on the same device state
    cfg = W.CONFIGS["c32k"].scaled(name="m1", N=3000, topk=200, steps=1, block=1)
    w = W.make_workload(cfg, device="cpu", steps=1).to("cuda")
    g = DeviceRun(cfg, w)
    index = dk.BlockIndex.empty_for(g.cache, cfg.B, cfg.bits, 1)
    g.encode()
    g.eng.encode_blocks(g.cache, index, g.seq)
    g.append(0)
    g.eng.append_blocks(g.cache, index, g.seq)
    assert torch.equal(index.codes[:, :, :int(g.seq.max())], g.cache.codes[:, :, :int(g.seq.max())])
    b = g.buf
    g.eng.select(g.cache, w.q[0], g.seq, b["sel_idx"], b["sel_cnt"])
    tok = (b["sel_idx"].clone(), b["sel_cnt"].clone())
    g.eng.select_blocks(g.cache, index, w.q[0], g.seq, b["sel_idx"], b["sel_cnt"])
    assert g.error() == 0
    assert torch.equal(tok[1], b["sel_cnt"]) and torch.equal(tok[0], b["sel_idx"])
    g.close()


@pytest.mark.parametrize("path", list(PATHS))
def test_blocks_edge_lengths(path):
    # lengths 0, below one block, exactly one block, and around the sinks / window
    cfg = W.Config("blk_edges", B=6, Hq=4, Hkv=2, d=64, N=40, bits=64, topk=8, sink=3, window=7,
                   steps=1, needles=0, seed=93, block=8)

    def mutate(w):
        w.seq_lens[:] = torch.tensor([0, 5, 7, 15, 31, 39], dtype=torch.int32)
        return w
    run_block_parity(cfg, 1, mutate=mutate, **PATHS[path])


@pytest.mark.parametrize("path", list(PATHS))
def test_blocks_topk_covers_everything_is_dense(path):
    cfg = W.Config("blk_all", B=2, Hq=8, Hkv=2, d=128, N=700, n_min=300, bits=128, topk=4096, sink=4, window=16,
                   steps=2, needles=2, seed=94, block=16)
    counts = run_block_parity(cfg, 2, **PATHS[path])
    assert counts[-1].min() > 0


@pytest.mark.parametrize("path", list(PATHS))
def test_blocks_zero_query_ties_to_lowest_blocks(path):
    cfg = W.Config("blk_zeroq", B=1, Hq=4, Hkv=1, d=128, N=9002, bits=128, topk=700, sink=3, window=5,
                   steps=2, needles=0, seed=95, block=4)

    def mutate(w):
        w.q.zero_()
        return w
    run_block_parity(cfg, 2, mutate=mutate, **PATHS[path])


def test_select_blocks_rejects_a_window_shorter_than_a_block():
    cfg = W.Config("blk_bad", B=1, Hq=4, Hkv=1, d=64, N=100, bits=64, topk=16, sink=0, window=2, steps=0,
                   needles=0, seed=96)
    w = W.make_workload(cfg, device="cpu", steps=0).to("cuda")
    g = DeviceRun(cfg, w)
    index = dk.BlockIndex.empty_for(g.cache, cfg.B, cfg.bits, 4)  # window 2 < m - 1 = 3
    b = g.buf
    b["sel_cnt"].fill_(-7)
    q = torch.zeros((1, 4, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(dk.DashKVError) as e:
        g.eng.select_blocks(g.cache, index, q, g.seq, b["sel_idx"], b["sel_cnt"])
    assert e.value.status == 2  # DASHKV_ERR_UNSUPPORTED, nothing launched
    torch.cuda.synchronize()
    assert int(b["sel_cnt"][0, 0]) == -7
    bad = dk.BlockIndex(index.codes, 3)  # not a power of two
    with pytest.raises(dk.DashKVError) as e:
        g.eng.encode_blocks(g.cache, bad, g.seq)
    assert e.value.status == 1
    g.close()
