"""GPU path vs the CPU oracle on seeded workloads, through the C ABI.

Sizes are small enough for the oracle to finish in seconds but span several
scorer / selector CTAs, warps and ragged tails; the shapes are the pages'
long-context decode shapes scaled down (GQA 4:1 and 8:1, d = 64 / 128,
b = 32 / 64 / 128, dense and paged layouts)."""
import numpy as np
import pytest
import torch

from hash_indexed_top_b200 import workloads as W

from pipeline import run_parity

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": (W.CONFIGS["tiny"], 8),
    "c32k_small": (W.CONFIGS["c32k"].scaled(name="c32k_small", N=4001, topk=256, steps=3), 3),
    "c128k_small": (W.CONFIGS["c128k"].scaled(name="c128k_small", B=2, N=6000, topk=512, steps=2), 2),
    "ragged_paged_small": (W.CONFIGS["ragged_paged"].scaled(name="ragged_paged_small", B=5, N=5000, n_min=700,
                                                            topk=300, steps=2), 2),
    "c1m_small": (W.CONFIGS["c1m"].scaled(name="c1m_small", N=20000, topk=1024, steps=1), 1),
    "d64_b128": (W.Config("d64_b128", B=3, Hq=8, Hkv=4, d=64, N=3333, bits=128, topk=100, sink=2, window=40,
                          steps=2, needles=4, seed=77), 2),
    "g1_b64_paged32": (W.Config("g1_b64_paged32", B=2, Hq=2, Hkv=2, d=128, N=1500, n_min=100, bits=64, topk=64,
                                sink=0, window=0, steps=2, needles=2, page_size=32, seed=78), 2),
    "g2_b32": (W.Config("g2_b32", B=2, Hq=4, Hkv=2, d=128, N=2500, bits=32, topk=200, sink=8, window=8,
                        steps=2, needles=2, seed=79), 2),
}


@pytest.fixture(scope="module", autouse=True)
def built():
    from hash_indexed_top_b200 import build
    build.build()


# selection path x decode mode: the clustered selection with the decode's
# window CTAs (lengths given), the same selection with a plain list decode, the
# two-kernel selection, and the whole step as one clustered launch
# (dashkv_decode_step: append, selection and attention in one kernel)
PATHS = {"fused": dict(two_kernel=False, window=True), "fused_list_decode": dict(two_kernel=False, window=False),
         "two_kernel": dict(two_kernel=True, window=True), "step": dict(fused_step=True)}
# the paths whose select and decode can run without an append before them
SPLIT_PATHS = {k: v for k, v in PATHS.items() if k != "step"}


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("name", list(CASES))
def test_parity(name, path):
    cfg, steps = CASES[name]
    diags = run_parity(cfg, steps, **PATHS[path])
    assert len(diags) == steps


@pytest.mark.parametrize("path", list(PATHS))
def test_topk_covers_everything_is_dense_attention(path):
    cfg = W.Config("allk", B=2, Hq=8, Hkv=2, d=128, N=700, n_min=300, bits=64, topk=5000, sink=4, window=16,
                   steps=1, needles=2, seed=80)
    run_parity(cfg, 1, **PATHS[path])


@pytest.mark.parametrize("path", list(PATHS))
def test_sinks_and_window_overlap_short_sequences(path):
    cfg = W.Config("overlap", B=4, Hq=4, Hkv=1, d=64, N=60, n_min=1, bits=32, topk=5, sink=20, window=50,
                   steps=2, needles=0, seed=81)
    run_parity(cfg, 2, **PATHS[path])


@pytest.mark.parametrize("path", list(PATHS))
def test_zero_query_all_scores_tie(path):
    # q = 0 makes every score 0: one histogram bin holds every token, so the
    # exact threshold comes from the radix path and ties go to the lowest ids.
    cfg = W.Config("zeroq", B=1, Hq=4, Hkv=1, d=128, N=9000, bits=128, topk=700, sink=3, window=5,
                   steps=1, needles=0, seed=82)

    def mutate(w):
        w.q.zero_()
        return w
    run_parity(cfg, 1, mutate=mutate, **PATHS[path])


@pytest.mark.parametrize("path", list(PATHS))
def test_repeated_keys_heavy_ties(path):
    # only 3 distinct keys: huge tie groups at the threshold, in small-bin and radix regimes
    cfg = W.Config("ties", B=2, Hq=8, Hkv=2, d=128, N=5000, bits=64, topk=1500, sink=0, window=0,
                   steps=1, needles=0, seed=83)

    def mutate(w):
        pat = w.K[:, :, :3].clone()
        idx = torch.arange(w.K.shape[2]) % 3
        w.K[:] = pat[:, :, idx]
        return w
    run_parity(cfg, 1, mutate=mutate, **PATHS[path])


@pytest.mark.parametrize("path", list(SPLIT_PATHS))
def test_empty_sequence_selects_nothing(path):
    cfg = W.Config("empty", B=3, Hq=4, Hkv=2, d=64, N=200, bits=64, topk=10, sink=2, window=2,
                   steps=0, needles=0, seed=84)
    w = W.make_workload(cfg, steps=0)
    w.seq_lens[1] = 0
    from pipeline import DeviceRun, OracleRun, compare_step
    g = DeviceRun(cfg, w.to("cuda"), **PATHS[path])
    o = OracleRun(cfg, w)
    g.encode()
    q = torch.zeros((cfg.B, cfg.Hq, cfg.d), dtype=torch.bfloat16)
    q[:] = W.grid(torch.randn(q.shape, generator=torch.Generator().manual_seed(5)))
    g.select_decode(q.cuda())
    r = o.step(q)
    assert g.error() == 0
    compare_step(g, o, r, "empty")
    assert (g.buf["sel_cnt"][1] == 0).all()
    assert torch.isneginf(g.buf["lse"][1]).all() and (g.buf["out"][1] == 0).all()
    g.close()


@pytest.mark.parametrize("path", list(SPLIT_PATHS))
def test_repeat_calls_are_deterministic_and_leave_workspace_clean(path):
    cfg, _ = CASES["c128k_small"]
    w = W.make_workload(cfg, steps=1).to("cuda")
    from pipeline import DeviceRun
    g = DeviceRun(cfg, w, **PATHS[path])
    g.encode()
    g.append(0)
    outs = []
    for _ in range(3):
        g.select_decode(w.q[0])
        outs.append({k: v.clone() for k, v in g.buf.items()})
    assert g.error() == 0
    for o in outs[1:]:
        for k in ("sel_idx", "sel_cnt", "out", "lse"):
            assert torch.equal(o[k], outs[0][k]), k
    g.close()


def test_needle_recall_reported():
    # quality number, not a parity gate: planted needles close to the query
    cfg = W.CONFIGS["c32k"].scaled(name="recall", N=16384, steps=1)
    w = W.make_workload(cfg, steps=1).to("cuda")
    from pipeline import DeviceRun
    g = DeviceRun(cfg, w)
    g.encode()
    g.append(0)
    g.select_decode(w.q[0])
    sel = g.buf["sel_idx"].cpu()
    pos = w.needle_pos.cpu()
    hit = tot = 0
    for b in range(cfg.B):
        for h in range(cfg.Hkv):
            s = set(sel[b, h].tolist())
            for p in pos[b, h].tolist():
                if p >= 0:
                    tot += 1
                    hit += p in s
    g.close()
    print(f"needle recall {hit}/{tot}")
    assert tot > 0 and hit / tot > 0.5
