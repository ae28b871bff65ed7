"""Radius-scaled scores (Spherical KV page, section 2.1 ADA) on the GPU
against the oracle, through the C ABI.

Every step the GPU appends the step's key and its radius code
(dashkv_append_radius), selects on s' = r~ s and decodes; the oracle encodes
every radius code from its keys.  Radius codes, scaled scores and the token
lists must be bit-identical, outputs within the attention tolerance.
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


def run_radius_parity(cfg: W.Config, steps: int, window_decode: bool = True, mutate=None) -> None:
    w = W.make_workload(cfg, device="cpu", steps=steps)
    if mutate is not None:
        w = mutate(w)
    g = DeviceRun(cfg, w.to("cuda"), window=window_decode)
    o = OracleRun(cfg, w)
    radius = dk.KVCache.empty_radius_like(g.cache.k, g.cache.paged)
    g.encode()
    g.eng.encode_radius(g.cache, radius, g.seq)
    try:
        for s in range(steps):
            g.append(s)
            g.eng.append_radius(g.cache, radius, g.seq)
            o.append(s)
            q = w.q[s]
            b = g.buf
            g.eng.select_radius(g.cache, radius, q.cuda(), g.seq, b["sel_idx"], b["sel_cnt"], g.scores)
            g.eng.sparse_decode(g.cache, q.cuda(), b["sel_idx"], b["sel_cnt"], b["out"], b["lse"],
                                seq_lens=g.seq if window_decode else None)
            assert g.error() == 0
            what = f"{cfg.name} step {s}"
            orc = O.radius_codes(o.L, o.K, o.seq)
            grc = radius.cpu().numpy()
            assert np.array_equal(grc, orc), f"{what}: radius codes differ at {np.argwhere(grc != orc)[:5].tolist()}"
            r = O.decode_step_radius(o.L, cfg.Hq, q.double().numpy(), o.K, o.V, o.codes, orc, o.seq, o.R, cfg.topk,
                                     cfg.sink, cfg.window)
            gs = g.scores.cpu().numpy()
            es = r["scores"].astype(np.float32)
            for bb in range(cfg.B):
                n = int(o.seq[bb])
                assert np.array_equal(gs[bb, :, :n].view(np.uint32), es[bb, :, :n].view(np.uint32)), \
                    f"{what}: scaled scores differ (b={bb})"
            assert np.array_equal(b["sel_cnt"].cpu().numpy(), r["sel_cnt"]), f"{what}: sel_cnt differ"
            assert np.array_equal(b["sel_idx"].cpu().numpy(), r["sel_idx"]), f"{what}: sel_idx differ"
            out = b["out"].cpu().double().numpy()
            lse = b["lse"].cpu().double().numpy()
            assert within_tol(out, r["out"]).all(), f"{what}: out max err {np.nanmax(np.abs(out - r['out'])):.3e}"
            assert within_tol(lse, r["lse"]).all(), f"{what}: lse max err {np.nanmax(np.abs(lse - r['lse'])):.3e}"
    finally:
        g.close()


CASES = {
    "c128k_small": (W.CONFIGS["c128k"].scaled(name="r_c128k_small", B=2, N=6000, topk=512, steps=2), 2),
    "ragged_paged_small": (W.CONFIGS["ragged_paged"].scaled(name="r_ragged_paged_small", B=5, N=5000, n_min=700,
                                                            topk=300, steps=2), 2),
    "d64_b32": (W.Config("r_d64_b32", B=3, Hq=8, Hkv=4, d=64, N=3333, bits=32, topk=100, sink=2, window=40,
                         steps=2, needles=4, seed=97), 2),
}


@pytest.mark.parametrize("window_decode", [True, False])
@pytest.mark.parametrize("name", list(CASES))
def test_radius_parity(name, window_decode):
    cfg, steps = CASES[name]
    run_radius_parity(cfg, steps, window_decode)


def test_radius_zero_and_scaled_keys():
    # zero keys (code 0) and keys scaled by 2 and 4 (same sign code, larger
    # radius): ties in the code score broken by the radius
    cfg = W.Config("r_scaled", B=1, Hq=4, Hkv=1, d=128, N=4000, bits=64, topk=300, sink=3, window=5, steps=1,
                   needles=0, seed=98)

    def mutate(w):
        w.K[:, :, 0:500] = 0
        w.K[:, :, 1000:1500] = torch.clamp(w.K[:, :, 1000:1500].float() * 2, -4, 4).to(torch.bfloat16)
        w.K[:, :, 2000:2500] = torch.clamp(w.K[:, :, 2000:2500].float() * 4, -4, 4).to(torch.bfloat16)
        return w
    run_radius_parity(cfg, 1, mutate=mutate)
