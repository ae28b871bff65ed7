"""Test harness: run the same seeded workload through the CUDA library (via
its C ABI binding) and through the CPU oracle, and compare.

Bars: codes, scores and selected indices bit-identical; attention outputs and
log-sum-exp within |err| <= 1e-3 + 8e-3 |ref| per element.
"""
from __future__ import annotations

import numpy as np
import torch

from hash_indexed_top_b200 import dashkv as dk
from hash_indexed_top_b200 import workloads as W
from oracle import oracle as O

ATOL, RTOL = 1e-3, 8e-3
# Scores are compared bit for bit because on 1/64-grid inputs every partial sum
# of the fp32 scorer is a multiple of 1/64 bounded by A = sum_j |Qp_j| (the
# oracle's `bound`); fp32 holds all of them exactly while 64 A < 2^24.
EXACT_BOUND = 2.0 ** 18


def assert_exact_scoring(bound: float, what: str = "") -> None:
    assert bound < EXACT_BOUND, f"{what}: score bound {bound} breaks the exactness precondition (< 2^18)"


class DeviceRun:
    """The device side of a parity run.  fused_step: each step is one
    dashkv_decode_step call (append + select + attention in one launch, no
    scores output); otherwise append_keys, select (with its scores) and
    sparse_decode, given the lengths (window) or the plain list."""

    def __init__(self, cfg: W.Config, w: W.Workload, seed: int = W.HYPERPLANE_SEED, two_kernel: bool = False,
                 window: bool = True, fused_step: bool = False):
        self.cfg, self.w = cfg, w
        self.window = window  # decode given the lengths (window CTAs) or the plain list
        self.fused_step = fused_step
        self.pending = None   # fused step: the step whose append is still to run
        dev = w.K.device
        self.eng = dk.DashKV(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.bits, cfg.topk, cfg.sink, cfg.window,
                             cfg.page_size if w.paged else 0, seed, two_kernel_select=two_kernel)
        codes = dk.KVCache.empty_codes_like(w.K, cfg.bits, w.paged)
        self.cache = dk.KVCache(w.K, w.V, codes, w.page_table)
        self.seq = w.seq_lens.clone()
        self.buf = self.eng.alloc_step(dev)
        self.scores = torch.full((cfg.B, cfg.Hkv, self.cache.capacity), float("nan"), device=dev)

    def encode(self):
        self.eng.encode_keys(self.cache, self.seq)

    def append(self, s: int):
        if self.fused_step:
            self.pending = s
            return
        self.eng.append_keys(self.cache, self.w.k_new[s], self.w.v_new[s], self.seq)

    @property
    def has_scores(self) -> bool:
        return not self.fused_step

    def select_decode(self, q: torch.Tensor):
        b = self.buf
        if self.fused_step:
            assert self.pending is not None, "the fused step appends: call append(s) first"
            s, self.pending = self.pending, None
            self.eng.decode_step(self.cache, q, self.w.k_new[s], self.w.v_new[s], self.seq, b["sel_idx"],
                                 b["sel_cnt"], b["out"], b["lse"])
            return
        self.eng.select(self.cache, q, self.seq, b["sel_idx"], b["sel_cnt"], self.scores)
        self.eng.sparse_decode(self.cache, q, b["sel_idx"], b["sel_cnt"], b["out"], b["lse"],
                               seq_lens=self.seq if self.window else None)

    def error(self) -> int:
        return self.eng.get_error()

    def close(self):
        self.eng.close()


class OracleRun:
    """Oracle state over the full cache (small workloads)."""

    def __init__(self, cfg: W.Config, w: W.Workload, seed: int = W.HYPERPLANE_SEED):
        self.cfg = cfg
        self.R = O.hyperplanes(seed, cfg.bits, cfg.d)
        if w.paged:
            self.L = O.Layout(cfg.B, cfg.Hkv, cfg.d, cfg.bits, page_table=w.page_table.cpu().numpy(),
                              page=cfg.page_size)
        else:
            self.L = O.Layout(cfg.B, cfg.Hkv, cfg.d, cfg.bits, n_cap=w.n_cap)
        self.K = w.K.cpu().double().numpy().copy()
        self.V = w.V.cpu().double().numpy().copy()
        self.seq = w.seq_lens.cpu().numpy().astype(np.int32).copy()
        self.codes = O.encode(self.L, self.K, self.seq, self.R)
        self.w = w

    def append(self, s: int):
        O.append(self.L, self.K, self.V, self.codes, self.seq, self.w.k_new[s].cpu().double().numpy(),
                 self.w.v_new[s].cpu().double().numpy(), self.R)

    def step(self, q: torch.Tensor) -> dict:
        return O.decode_step(self.L, self.cfg.Hq, q.cpu().double().numpy(), self.K, self.V, self.codes,
                             self.seq, self.R, self.cfg.topk, self.cfg.sink, self.cfg.window)


def within_tol(got: np.ndarray, ref: np.ndarray) -> np.ndarray:
    both_inf = np.isneginf(got) & np.isneginf(ref)
    with np.errstate(invalid="ignore"):
        err = np.abs(got - ref)
    return both_inf | (err <= ATOL + RTOL * np.abs(ref))


def compare_step(g: DeviceRun, o: OracleRun, r: dict, what: str = "") -> dict:
    """Assert parity of one step; returns a few diagnostics."""
    assert_exact_scoring(r["bound"], what)
    gc = dk.canonical_codes(g.cache.codes, o.cfg.bits).cpu().numpy().view(np.uint64)
    assert np.array_equal(gc, o.codes), f"{what}: codes differ at {np.argwhere(gc != o.codes)[:5].tolist()}"
    assert np.array_equal(g.seq.cpu().numpy(), o.seq), f"{what}: seq_lens differ"
    if g.fused_step:  # the step wrote the appended rows itself
        assert np.array_equal(g.cache.k.cpu().double().numpy(), o.K), f"{what}: cached keys differ"
        assert np.array_equal(g.cache.v.cpu().double().numpy(), o.V), f"{what}: cached values differ"
    if g.has_scores:
        gs = g.scores.cpu().numpy()
        os_ = r["scores"].astype(np.float32)
        for b in range(o.cfg.B):
            n = int(o.seq[b])
            a, e = gs[b, :, :n], os_[b, :, :n]
            assert np.array_equal(a.view(np.uint32), e.view(np.uint32)), \
                f"{what}: scores differ (b={b}) at {np.argwhere(a != e)[:5].tolist()}"
    gi = g.buf["sel_idx"].cpu().numpy()
    gn = g.buf["sel_cnt"].cpu().numpy()
    assert np.array_equal(gn, r["sel_cnt"]), f"{what}: sel_cnt {gn.ravel()[:8]} vs {r['sel_cnt'].ravel()[:8]}"
    assert np.array_equal(gi, r["sel_idx"]), f"{what}: sel_idx differ"
    out = g.buf["out"].cpu().double().numpy()
    lse = g.buf["lse"].cpu().double().numpy()
    ok = within_tol(out, r["out"])
    assert ok.all(), f"{what}: out max err {np.nanmax(np.abs(out - r['out'])):.3e}"
    okl = within_tol(lse, r["lse"])
    assert okl.all(), f"{what}: lse max err {np.nanmax(np.abs(lse - r['lse'])):.3e}"
    fin = np.isfinite(r["out"])
    return dict(max_err=float(np.abs(out - r["out"])[fin].max()) if fin.any() else 0.0)


def run_parity(cfg: W.Config, steps: int, device="cuda", w: W.Workload | None = None, mutate=None,
               two_kernel: bool = False, window: bool = True, fused_step: bool = False) -> list:
    """Encode, then `steps` x (append, select, decode) on GPU and oracle, comparing every step."""
    if w is None:
        w = W.make_workload(cfg, device="cpu", steps=steps)
    if mutate is not None:
        w = mutate(w)
    g = DeviceRun(cfg, w.to(device), two_kernel=two_kernel, window=window, fused_step=fused_step)
    o = OracleRun(cfg, w)
    g.encode()
    diags = []
    try:
        for s in range(steps):
            g.append(s)
            o.append(s)
            q = w.q[s]
            g.select_decode(q.to(device))
            r = o.step(q)
            assert g.error() == 0
            diags.append(compare_step(g, o, r, f"{cfg.name} step {s}"))
    finally:
        g.close()
    return diags
