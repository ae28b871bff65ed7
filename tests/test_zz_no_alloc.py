"""dashkv_select_static: the allocation-free selection (library-owned static
device scratch) against dashkv_select with a caller workspace.

Collected last on purpose: the static scratch lives for the whole process,
so these checks must hold both alone and after every other test has used the
library.  Two steps in a row (append, then both selections) also check that
each call leaves the scratch ready for the next; a sequence of problems with
different capacities and batch shapes checks that a call whose scratch layout
differs from the previous one's does not read counters the previous call left
in its rows (both selection paths: the two-kernel path reads histogram and
arrival words that must start at zero).
"""
import pytest
import torch

from hash_indexed_top_b200 import dashkv as dk
from hash_indexed_top_b200 import workloads as W

STATIC_SCRATCH_BYTES = 24 << 20  # the limit stated in include/dashkv.h

CASES = {
    "dense_b64": W.Config("ns_dense", B=1, Hq=32, Hkv=8, d=128, N=6001, bits=64, topk=300, sink=4, window=64,
                          steps=2, needles=8, seed=4101),
    "paged_b128": W.Config("ns_paged", B=3, Hq=16, Hkv=4, d=64, N=5000, n_min=900, bits=128, topk=200, sink=4,
                           window=32, steps=2, needles=4, page_size=64, seed=4102),
}


def _engine(cfg, w, two_kernel=False):
    eng = dk.DashKV(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.bits, cfg.topk, cfg.sink, cfg.window,
                    cfg.page_size if w.paged else 0, W.HYPERPLANE_SEED, two_kernel_select=two_kernel)
    codes = dk.KVCache.empty_codes_like(w.K, cfg.bits, w.paged)
    return eng, dk.KVCache(w.K, w.V, codes, w.page_table)


@pytest.mark.gpu
@pytest.mark.parametrize("two_kernel", [False, True], ids=["fused", "two_kernel"])
@pytest.mark.parametrize("name", list(CASES))
def test_static_select_matches_workspace_select(name, two_kernel):
    cfg = CASES[name]
    dev = torch.device("cuda")
    w = W.make_workload(cfg, device=dev, steps=cfg.steps)
    eng, cache = _engine(cfg, w, two_kernel)
    try:
        assert eng.workspace_size(cache.capacity) <= STATIC_SCRATCH_BYTES
        seq = w.seq_lens.clone()
        eng.encode_keys(cache, seq)
        cap_sel = cfg.topk + cfg.sink + cfg.window
        for s in range(cfg.steps):  # two calls of each entry point in a row
            eng.append_keys(cache, w.k_new[s], w.v_new[s], seq)
            out = {}
            for kind in ("workspace", "static"):
                idx = torch.full((cfg.B, cfg.Hkv, cap_sel), -7, dtype=torch.int32, device=dev)
                cnt = torch.full((cfg.B, cfg.Hkv), -7, dtype=torch.int32, device=dev)
                sc = torch.full((cfg.B, cfg.Hkv, cache.capacity), float("nan"), device=dev)
                if kind == "workspace":
                    eng.select(cache, w.q[s], seq, idx, cnt, sc)
                else:
                    eng.select_static(cache, w.q[s], seq, idx, cnt, sc)
                torch.cuda.synchronize()
                assert eng.get_error() == 0
                out[kind] = (idx.cpu(), cnt.cpu(), sc.cpu())
            (ia, ca, sa), (ib, cb, sb) = out["workspace"], out["static"]
            assert torch.equal(ca, cb)
            assert torch.equal(ia, ib)
            assert torch.equal(torch.nan_to_num(sa, nan=-1e30), torch.nan_to_num(sb, nan=-1e30))
            assert int(cb.min()) > 0
    finally:
        eng.close()


# Problems whose scratch layouts differ (capacity and B * Hkv), run in this
# order in one process: large, small, large again.
LAYOUTS = [
    W.Config("ns_large", B=2, Hq=16, Hkv=8, d=64, N=9000, bits=64, topk=400, sink=4, window=64, steps=1,
             needles=4, seed=4201),
    W.Config("ns_small", B=1, Hq=8, Hkv=2, d=128, N=3000, bits=128, topk=150, sink=2, window=16, steps=1,
             needles=4, seed=4202),
    W.Config("ns_large2", B=2, Hq=16, Hkv=8, d=64, N=9000, bits=64, topk=400, sink=4, window=64, steps=1,
             needles=4, seed=4203),
]


@pytest.mark.gpu
@pytest.mark.parametrize("two_kernel", [False, True], ids=["fused", "two_kernel"])
def test_static_select_across_layout_changes(two_kernel):
    dev = torch.device("cuda")
    for cfg in LAYOUTS:
        w = W.make_workload(cfg, device=dev, steps=1)
        eng, cache = _engine(cfg, w, two_kernel)
        try:
            seq = w.seq_lens.clone()
            eng.encode_keys(cache, seq)
            eng.append_keys(cache, w.k_new[0], w.v_new[0], seq)
            cap_sel = cfg.topk + cfg.sink + cfg.window
            res = {}
            for kind in ("static", "fresh"):
                idx = torch.full((cfg.B, cfg.Hkv, cap_sel), -7, dtype=torch.int32, device=dev)
                cnt = torch.full((cfg.B, cfg.Hkv), -7, dtype=torch.int32, device=dev)
                if kind == "static":
                    eng.select_static(cache, w.q[0], seq, idx, cnt)
                else:  # a freshly zeroed caller workspace
                    ws = torch.zeros(eng.workspace_size(cache.capacity), dtype=torch.uint8, device=dev)
                    eng.select(cache, w.q[0], seq, idx, cnt, None, ws)
                torch.cuda.synchronize()
                assert eng.get_error() == 0
                res[kind] = (idx.cpu(), cnt.cpu())
            assert torch.equal(res["static"][1], res["fresh"][1]), cfg.name
            assert torch.equal(res["static"][0], res["fresh"][0]), cfg.name
            assert int(res["static"][1].min()) > 0
        finally:
            eng.close()


@pytest.mark.gpu
def test_static_select_rejects_inputs_beyond_the_limit():
    # a paged view whose capacity (max_pages * page_size) needs more than the
    # scratch holds; every table entry points at one of four real pages
    B, Hq, Hkv, d, bits, ps = 2, 8, 8, 64, 64, 64
    dev = torch.device("cuda")
    eng = dk.DashKV(B, Hq, Hkv, d, bits, 64, 4, 16, ps, W.HYPERPLANE_SEED)
    try:
        max_pages = 4096
        K = torch.zeros((4, ps, Hkv, d), dtype=torch.bfloat16, device=dev)
        V = torch.zeros_like(K)
        codes = dk.KVCache.empty_codes_like(K, bits, True)
        pt = (torch.arange(B * max_pages, dtype=torch.int32, device=dev) % 4).reshape(B, max_pages)
        cache = dk.KVCache(K, V, codes, pt)
        assert eng.workspace_size(cache.capacity) > STATIC_SCRATCH_BYTES
        seq = torch.full((B,), 100, dtype=torch.int32, device=dev)
        q = torch.zeros((B, Hq, d), dtype=torch.bfloat16, device=dev)
        idx = torch.full((B, Hkv, 64 + 4 + 16), -7, dtype=torch.int32, device=dev)
        cnt = torch.full((B, Hkv), -7, dtype=torch.int32, device=dev)
        with pytest.raises(dk.DashKVError) as e:
            eng.select_static(cache, q, seq, idx, cnt)
        assert e.value.status == 3  # DASHKV_ERR_WORKSPACE
        torch.cuda.synchronize()
        assert int(cnt.min()) == -7 and int(idx.min()) == -7  # nothing was launched
        assert eng.get_error() == 0
    finally:
        eng.close()
