"""Seeded synthetic decode workloads (inputs only; no step of the method).

Both the CUDA path and the CPU oracle are fed from here; this module holds
none of the method's arithmetic (no hashing, scoring, selection or
attention).  Everything is drawn from a seeded ``torch.Generator`` on the
requested device.

Value recipe (the 1/64 grid): every K, V and Q element is
``round(64 * x) / 64`` clipped to [-4, 4] and stored as bf16, which holds
these values exactly; ``-0`` is canonicalised to ``+0``.  On this grid every
partial sum of the scorer and the encoder is an exact multiple of 1/64, so
fp32 sums do not depend on their order.

Planted needles: per (sequence, KV head) a few cache positions drawn
uniformly (distinct) from [S, N0 - W) hold ``grid(q_base + 0.25 z)``, where
``q_base`` is the continuous Gaussian base query of the group's first query
head; each decode step's queries are ``grid(q_base + 0.25 z_step)``, so the
needles stay relevant across steps.  Appended keys and values are fresh grid
Gaussians.

Workload shapes are those of long-context decode (32K-1M cached tokens, GQA
32:8 and 64:8, head dim 128), standing in for the LongBench / PG-19 /
needle-in-a-haystack evaluations the pages report, which are not available
here.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

HYPERPLANE_SEED = 0x5EEDDA5B


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    N: int                 # cached tokens per sequence (ragged: upper bound)
    bits: int
    topk: int
    sink: int
    window: int
    steps: int
    needles: int
    page_size: int = 0     # 0 = dense layout
    n_min: int = 0         # ragged: lower bound of the length draw (0 = fixed N)
    seed: int = 1234
    block: int = 0         # > 0: select through summaries of blocks of this many tokens
    radius: bool = False   # select on radius-scaled scores (8-bit key-norm codes)
    tiers: bool = False    # paged: pages between the sinks and the window held as FP8 rows

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def sel_cap(self) -> int:
        return self.topk + self.sink + self.window

    def scaled(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": Config("tiny", B=1, Hq=4, Hkv=1, d=64, N=1024, bits=32, topk=64, sink=4, window=16,
                   steps=8, needles=4, seed=1234),
    "c32k": Config("c32k", B=1, Hq=32, Hkv=8, d=128, N=32768, bits=64, topk=1024, sink=4, window=128,
                   steps=64, needles=16, seed=1235),
    "c128k": Config("c128k", B=4, Hq=32, Hkv=8, d=128, N=131072, bits=128, topk=2048, sink=4, window=512,
                    steps=32, needles=32, seed=1236),
    "ragged_paged": Config("ragged_paged", B=16, Hq=32, Hkv=8, d=128, N=65536, n_min=8192, bits=64,
                           topk=1024, sink=4, window=256, steps=16, needles=16, page_size=64, seed=1237),
    "c1m": Config("c1m", B=1, Hq=64, Hkv=8, d=128, N=1048576, bits=128, topk=4096, sink=4, window=1024,
                  steps=16, needles=64, seed=1238),
}
# the same workloads selected through block summaries of 4 tokens (the
# compression ratio of the DeepSeek DSA->CSA/HCA page's CSA example): the
# top topk / 4 blocks give the same top-k token budget
CONFIGS["c128k_blocks4"] = CONFIGS["c128k"].scaled(name="c128k_blocks4", block=4)
CONFIGS["c1m_blocks4"] = CONFIGS["c1m"].scaled(name="c1m_blocks4", block=4)
# the 128K workload selected on radius-scaled scores
CONFIGS["c128k_radius"] = CONFIGS["c128k"].scaled(name="c128k_radius", radius=True)
# the ragged paged workload with every page between the sinks and the window
# demoted to FP8 rows (the pages' mixed-precision KV store)
CONFIGS["ragged_paged_fp8"] = CONFIGS["ragged_paged"].scaled(name="ragged_paged_fp8", tiers=True)
# the 1M-token workload's shape at half the length: a case small enough for
# multi-pass profiler captures of the same kernels
CONFIGS["c512k"] = CONFIGS["c1m"].scaled(name="c512k", N=524288)


def grid(x: torch.Tensor) -> torch.Tensor:
    """round(64 x)/64 clipped to [-4, 4], as bf16 (exact), with -0 -> +0."""
    y = torch.clamp(torch.round(x * 64.0), -256.0, 256.0) / 64.0
    return (y + 0.0).to(torch.bfloat16)


def _randn(shape, gen, device, chunk=1 << 26):
    """Gaussian draw in bounded-size chunks (keeps fp32 temporaries small)."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        flat[s:e] = grid(torch.randn(e - s, generator=gen, device=device))
    return out


@dataclasses.dataclass
class Workload:
    cfg: Config
    seq_lens: torch.Tensor          # [B] int32, lengths before the first decode step
    n_cap: int                      # dense: rows per (b, h); paged: 0
    K: torch.Tensor                 # dense [B,Hkv,n_cap,d] / paged [P,page,Hkv,d] bf16
    V: torch.Tensor
    page_table: Optional[torch.Tensor]  # [B, max_pages] int32 (paged) or None
    num_pages: int
    q: torch.Tensor                 # [steps, B, Hq, d] bf16
    k_new: torch.Tensor             # [steps, B, Hkv, d] bf16
    v_new: torch.Tensor             # [steps, B, Hkv, d] bf16
    needle_pos: torch.Tensor        # [B, Hkv, needles] int64 (positions; -1 unused)

    @property
    def paged(self) -> bool:
        return self.page_table is not None

    def to(self, device) -> "Workload":
        f = lambda t: None if t is None else t.to(device)
        return dataclasses.replace(self, seq_lens=f(self.seq_lens), K=f(self.K), V=f(self.V),
                                   page_table=f(self.page_table), q=f(self.q), k_new=f(self.k_new),
                                   v_new=f(self.v_new), needle_pos=f(self.needle_pos))


def make_workload(cfg: Config, device="cpu", steps: Optional[int] = None, extra_cap: int = 0) -> Workload:
    """Draw a workload.  Capacity covers ``steps`` appends (+ ``extra_cap``)."""
    steps = cfg.steps if steps is None else steps
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(cfg.seed)
    cpu_gen = torch.Generator()
    cpu_gen.manual_seed(cfg.seed + 7919)

    B, Hkv, Hq, d = cfg.B, cfg.Hkv, cfg.Hq, cfg.d
    if cfg.n_min:
        lens = torch.randint(cfg.n_min, cfg.N + 1, (B,), generator=cpu_gen, dtype=torch.int64)
    else:
        lens = torch.full((B,), cfg.N, dtype=torch.int64)
    cap_tokens = lens + steps + extra_cap

    if cfg.page_size:
        ps = cfg.page_size
        pages_per = (cap_tokens + ps - 1) // ps
        num_pages = int(pages_per.sum())
        max_pages = int(pages_per.max())
        perm = torch.randperm(num_pages, generator=cpu_gen).to(torch.int32)
        pt = torch.full((B, max_pages), -1, dtype=torch.int32)
        o = 0
        for b in range(B):
            n = int(pages_per[b])
            pt[b, :n] = perm[o:o + n]
            o += n
        K = _randn((num_pages, ps, Hkv, d), gen, dev)
        V = _randn((num_pages, ps, Hkv, d), gen, dev)
        n_cap = 0
        page_table = pt.to(dev)
    else:
        n_cap = int(cap_tokens.max())
        K = _randn((B, Hkv, n_cap, d), gen, dev)
        V = _randn((B, Hkv, n_cap, d), gen, dev)
        page_table = None
        num_pages = 0

    q_base = torch.randn((B, Hq, d), generator=gen, device=dev)
    q = torch.stack([grid(q_base + 0.25 * torch.randn((B, Hq, d), generator=gen, device=dev))
                     for _ in range(steps)]) if steps else torch.empty((0, B, Hq, d), dtype=torch.bfloat16, device=dev)
    k_new = _randn((steps, B, Hkv, d), gen, dev)
    v_new = _randn((steps, B, Hkv, d), gen, dev)

    # planted needles: keys close to the group's base query
    nn = cfg.needles
    pos = torch.full((B, Hkv, nn), -1, dtype=torch.int64)
    for b in range(B):
        lo, hi = cfg.sink, int(lens[b]) - cfg.window
        if hi - lo < nn or nn == 0:
            continue
        for h in range(Hkv):
            p = torch.randperm(hi - lo, generator=cpu_gen)[:nn] + lo
            pos[b, h] = p
            kv = grid(q_base[b, h * cfg.G].unsqueeze(0) + 0.25 * torch.randn((nn, d), generator=gen, device=dev))
            pd = p.to(dev)
            if cfg.page_size:
                ps = cfg.page_size
                phys = page_table[b].to(torch.int64)[pd // ps]
                K[phys, pd % ps, h] = kv
            else:
                K[b, h, pd] = kv
    return Workload(cfg=cfg, seq_lens=lens.to(torch.int32).to(dev), n_cap=n_cap, K=K, V=V,
                    page_table=page_table, num_pages=num_pages, q=q, k_new=k_new, v_new=v_new,
                    needle_pos=pos.to(dev))


class L2Flush:
    """Cold-cache state between timed steps: write a buffer of twice the L2
    size (evicting everything cached), then read a second, clean buffer of the
    same size so that L2 holds only clean lines and no write-back of the flush
    data lands inside the next timed step."""

    def __init__(self, device, l2_bytes: int = 126 * 1024 * 1024):
        n = int(2 * l2_bytes) // 4
        self.dirty = torch.empty(n, dtype=torch.int32, device=device)
        self.clean = torch.zeros(n, dtype=torch.int32, device=device)
        self.sink = torch.empty((), dtype=torch.int64, device=device)

    def __call__(self, i: int = 0) -> None:
        self.dirty.fill_(i)
        torch.sum(self.clean, dim=0, out=self.sink)
