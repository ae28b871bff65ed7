"""Decode-step benchmark: append -> hash-score + top-k select -> sparse attention.

One step = one decode query per sequence of the batch: append the new key /
value (with its code), score every cached key from its code, select top-k +
sinks + window, attend over the selection.  Default workload: B=4 sequences of
128K cached tokens, Hq=32, Hkv=8, d=128, 128-bit codes, k=2048, S=4, W=512
(synthetic 1/64-grid Gaussian K/V/Q with planted needles).

L2 is flushed (a 2 x L2 buffer is written) before every timed step; each step
is timed with CUDA events on the launching stream.  Multi-GPU: one replica per
rank (weak scaling, no data-path collective); NCCL only for the barrier and
the max-over-ranks of the timings.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl dashkv|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hash_indexed_top_b200 import workloads as W  # noqa: E402

METRIC = "sparse-decode queries/s at 128K ctx; achieved HBM GB/s vs ~8 TB/s peak"
SPEC_HBM_GBS = 8000.0


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), source="measured")
    return dict(hbm_gbs=6650.0, source="fallback")


def _strip_comments(src: str) -> str:
    """C/C++ source without comments and with whitespace collapsed (string
    literals are kept as they are)."""
    out, i, n = [], 0, len(src)
    while i < n:
        c = src[i]
        if c == '"':
            j = i + 1
            while j < n and src[j] != '"':
                j += 2 if src[j] == "\\" else 1
            out.append(src[i:j + 1])
            i = j + 1
        elif src.startswith("//", i):
            j = src.find("\n", i)
            i = n if j < 0 else j
        elif src.startswith("/*", i):
            j = src.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_sources_sha() -> str:
    """sha256 over the library's CUDA sources (name and code without comments
    or layout, sorted by name): it changes when the kernels do, not when only
    their comments do."""
    d = os.path.join(ROOT, "hash_indexed_top_b200", "csrc")
    h = hashlib.sha256()
    for n in sorted(os.listdir(d)):
        if n.endswith((".cu", ".cuh")):
            h.update(n.encode())
            with open(os.path.join(d, n), encoding="utf-8") as f:
                h.update(_strip_comments(f.read()).encode())
    return h.hexdigest()


def recorded_traffic(workload: str, kernel: str, algorithmic_bytes: float = 0.0):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from a
    committed ncu summary under profiles/ -- a text file with the lines
    ``workload: <name>``, ``kernel sources sha256: <sha>`` and
    ``traffic_per_launch <kernel> <bytes>`` -- or None when there is no summary
    for this workload taken from the kernel sources built now (the counters
    would be stale).  `algorithmic_bytes` is unused; it documents what the
    figure is compared with."""
    del algorithmic_bytes
    d = os.path.join(ROOT, "profiles")
    if not os.path.isdir(d):
        return None
    sha_now = kernel_sources_sha()
    for name in sorted(os.listdir(d)):
        if not name.endswith(".txt"):
            continue
        wl, sha, traffic = None, None, {}
        with open(os.path.join(d, name)) as f:
            for ln in f:
                if ln.startswith("workload:"):
                    wl = ln.split(":", 1)[1].strip()
                elif ln.startswith("kernel sources sha256:"):
                    sha = ln.split(":", 1)[1].strip()
                elif ln.startswith("traffic_per_launch "):
                    parts = ln.split()
                    traffic[parts[1]] = int(parts[2])
        if wl == workload and sha == sha_now and kernel in traffic:
            return traffic[kernel]
    return None


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while timing."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self) -> dict:
        if self.proc is None or not self.path:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------- dist
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if (args.impl == "dashkv" and torch.cuda.is_available()) else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    elif torch.cuda.is_available() and args.impl == "dashkv":
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- oracle leg
def oracle_block_update(L, K: np.ndarray, bcodes: np.ndarray, n: int, m: int, R) -> None:
    """After an oracle append that made sequence 0 n tokens long: when n is a
    multiple of m, encode the summary of the block the append completed (the
    oracle's whole-cache summary encode applied to that block's m rows)."""
    from oracle import oracle as O
    if n == 0 or n % m:
        return
    Lb = O.Layout(1, L.Hkv, L.d, L.bits, n_cap=m)
    last = np.ascontiguousarray(K[:, :, n - m:n])
    bcodes[:, :, n // m - 1] = O.encode_blocks(Lb, last, np.array([m], np.int32), m, R, 1)[:, :, 0]


def oracle_sample(cfg: W.Config, n_steps: int, seq_index: int = 0) -> dict:
    """Time the CPU oracle's decode step (score + select + attend; with block
    summaries: block score + block select + attend) on one sequence of the
    workload (all its KV / query heads), after one untimed oracle encode of that
    sequence's cache.  Appends (and the summary of a block an append completes)
    are untimed too."""
    from oracle import oracle as O
    # one sequence of the workload's longest length, dense (a paged workload's
    # page permutation changes nothing in the oracle's arithmetic)
    one = cfg.scaled(B=1, steps=n_steps + 1, page_size=0, n_min=0)
    w = W.make_workload(one, device="cpu", steps=n_steps + 1)
    R = O.hyperplanes(W.HYPERPLANE_SEED, cfg.bits, cfg.d)
    L = O.Layout(1, cfg.Hkv, cfg.d, cfg.bits, n_cap=w.n_cap)
    K = w.K.double().numpy()
    V = w.V.double().numpy()
    seq = w.seq_lens.numpy().astype(np.int32).copy()
    codes = O.encode(L, K, seq, R)
    m = cfg.block
    if m:
        nb_cap = w.n_cap // m
        bcodes = O.encode_blocks(L, K, seq, m, R, nb_cap)

    def append(s):
        O.append(L, K, V, codes, seq, w.k_new[s].double().numpy(), w.v_new[s].double().numpy(), R)
        if m:
            oracle_block_update(L, K, bcodes, int(seq[0]), m, R)
        if cfg.tiers:  # the appended row into the paged copy too (its page is in the window: bf16)
            t = int(seq[0]) - 1
            Kp[t // cfg.page_size, t % cfg.page_size] = K[0, :, t]
            Vp[t // cfg.page_size, t % cfg.page_size] = V[0, :, t]
        if cfg.radius:  # the appended token's radius code
            n = int(seq[0])
            rc[:, :, n - 1] = O.radius_codes(O.Layout(1, cfg.Hkv, cfg.d, cfg.bits, n_cap=1),
                                             np.ascontiguousarray(K[:, :, n - 1:n]), np.array([1], np.int32))[:, :, 0]

    rc = O.radius_codes(L, K, seq) if cfg.radius else None
    if cfg.tiers:  # the same sequence as a paged cache, its middle pages demoted (untimed)
        ps = cfg.page_size
        npg = (w.n_cap + ps - 1) // ps
        Lp = O.Layout(1, cfg.Hkv, cfg.d, cfg.bits, page_table=np.arange(npg, dtype=np.int32).reshape(1, npg), page=ps)
        Kp = np.zeros((npg * ps, cfg.Hkv, cfg.d))
        Vp = np.zeros((npg * ps, cfg.Hkv, cfg.d))
        Kp[:w.n_cap] = K[0].transpose(1, 0, 2)
        Vp[:w.n_cap] = V[0].transpose(1, 0, 2)
        Kp = Kp.reshape(npg, ps, cfg.Hkv, cfg.d)
        Vp = Vp.reshape(npg, ps, cfg.Hkv, cfg.d)
        tarr = O.tier_arrays(npg, ps, cfg.Hkv, cfg.d)
        O.demote_pages(Lp, Kp, Vp, seq, cfg.sink, cfg.window, *tarr)

    def decode(s):
        q = w.q[s].double().numpy()
        if cfg.tiers:
            sc, _ = O.scores(L, cfg.Hq, q, codes, seq, R)
            idx, cnt = O.select(sc, seq, cfg.topk, cfg.sink, cfg.window)
            O.attend_tiered(Lp, cfg.Hq, q, Kp, Vp, *tarr, idx, cnt)
        elif cfg.radius:
            O.decode_step_radius(L, cfg.Hq, q, K, V, codes, rc, seq, R, cfg.topk, cfg.sink, cfg.window)
        elif m:
            O.decode_step_blocks(L, cfg.Hq, q, K, V, bcodes, seq, R, m, cfg.topk // m, cfg.sink, cfg.window,
                                 cap=cfg.sel_cap)
        else:
            O.decode_step(L, cfg.Hq, q, K, V, codes, seq, R, cfg.topk, cfg.sink, cfg.window)

    times = []
    for s in range(n_steps):
        append(s)
        t0 = time.perf_counter()
        decode(s)
        times.append(time.perf_counter() - t0)
    cores = O.get_threads()
    # one more step on a single thread, for reference
    append(n_steps)
    O.set_threads(1)
    t0 = time.perf_counter()
    decode(n_steps)
    one_thread_s = time.perf_counter() - t0
    O.set_threads(cores)
    how = f", blocks of {m}" if m else (", radius-scaled scores" if cfg.radius else "")
    if cfg.tiers:
        how = ", middle pages as FP8 rows (attention reads them dequantized; appended rows stay bf16)"
    return dict(times=times, cores=cores, one_thread_s=one_thread_s,
                sample=f"sequence {seq_index} of {cfg.B} (N={cfg.N}, all {cfg.Hkv} KV / {cfg.Hq} query heads{how}), "
                       f"{n_steps} decode steps, oracle encode untimed")


def run_reference(args, cfg, world, rank):
    if rank != 0:
        return
    warm = max(0, args.warmup)
    r = oracle_sample(cfg, warm + args.steps)
    t = r["times"][warm:]
    value = len(t) / sum(t)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sum(t) / len(t),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "B": cfg.B, "N": cfg.N, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d": cfg.d,
                   "bits": cfg.bits, "topk": cfg.topk, "sink": cfg.sink, "window": cfg.window,
                   "block": cfg.block or None, "per_step_sample": "one sequence's decode query"},
        "cpu_baseline": {"value": value, "unit": "queries/s", "cores": r["cores"], "kind": "oracle",
                         "sample": r["sample"], "one_thread_value": 1.0 / r["one_thread_s"]},
        "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU leg
def run_dashkv(args, cfg, world, rank, local):
    from hash_indexed_top_b200 import build
    from hash_indexed_top_b200 import dashkv as dk
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: the dashkv arm needs a CUDA device")
    build.build()
    dev = torch.device("cuda", local)
    total = args.warmup + args.steps + args.e2e_steps
    # capacity also covers the extra replays of the timed graphs that keep the
    # clock sampler busy (each replay appends one token per sequence)
    w = W.make_workload(cfg, device=dev, steps=total + args.trace_steps,
                        extra_cap=args.steps * (args.clock_reps + 1))
    eng = dk.DashKV(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.bits, cfg.topk, cfg.sink, cfg.window,
                    cfg.page_size if w.paged else 0, W.HYPERPLANE_SEED,
                    two_kernel_select=args.two_kernel_select)
    codes = dk.KVCache.empty_codes_like(w.K, cfg.bits, w.paged)
    cache = dk.KVCache(w.K, w.V, codes, w.page_table)
    seq = w.seq_lens.clone()
    ws = eng.workspace(cache.capacity, dev)
    buf = eng.alloc_step(dev)
    flush = W.L2Flush(dev)
    stream = torch.cuda.current_stream(dev)
    eng.encode_keys(cache, seq)
    index = radius = None
    if cfg.block:  # block summaries of the prefilled cache (untimed, like the key codes)
        index = dk.BlockIndex.empty_for(cache, cfg.B, cfg.bits, cfg.block)
        eng.encode_blocks(cache, index, seq)
    if cfg.radius:  # radius codes of the prefilled cache (untimed)
        radius = dk.KVCache.empty_radius_like(w.K, w.paged)
        eng.encode_radius(cache, radius, seq)
    tiers = demote = None
    if cfg.tiers:  # the controller over the prefilled cache: middle pages to FP8 rows
        tiers = dk.PageTiers.empty_for(cache)
        eng.demote_pages(cache, tiers, seq)  # (loads the kernel; repeated below, timed)
        torch.cuda.synchronize(dev)
        tiers.tier.zero_()
        flush(0)
        e_dem = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        e_dem[0].record(stream)
        eng.demote_pages(cache, tiers, seq)
        e_dem[1].record(stream)
        torch.cuda.synchronize(dev)
        n_pages = int(tiers.tier.sum())
        rows = n_pages * cfg.page_size * cfg.Hkv
        dem_ms = e_dem[0].elapsed_time(e_dem[1])
        demote = {"ms": dem_ms, "pages": n_pages, "of_pages": int(tiers.tier.numel()),
                  "bytes": rows * (2 * cfg.d * 2 + 2 * cfg.d + 2),
                  "gbs": rows * (2 * cfg.d * 2 + 2 * cfg.d + 2) / (dem_ms * 1e-3) / 1e9,
                  "timing": "one full controller pass over the prefilled cache, L2 flushed before it; a decode loop "
                            "runs it again when a page leaves the window (once per page of steps)"}
    torch.cuda.synchronize(dev)
    assert eng.get_error() == 0
    # the prefill encode, timed on its own (a second, identical call: cold L2, kernel already loaded)
    flush(0)
    e_enc = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    e_enc[0].record(stream)
    eng.encode_keys(cache, seq)
    e_enc[1].record(stream)
    torch.cuda.synchronize(dev)
    assert eng.get_error() == 0
    enc_ms = e_enc[0].elapsed_time(e_enc[1])
    enc_keys = int(seq.sum()) * cfg.Hkv
    # the encode is b d signed adds per key-head (R is +-1): its roof is one fp32
    # add per lane per clock
    add_peak = torch.cuda.get_device_properties(dev).multi_processor_count * 128 * 1.965e9  # fp32 adds/s
    adds_per_s = cfg.bits * cfg.d * enc_keys / (enc_ms * 1e-3)
    encode = {"ms": enc_ms, "key_heads": enc_keys, "key_heads_per_s": enc_keys / (enc_ms * 1e-3),
              "alu_tadds_per_s": adds_per_s / 1e12,
              "alu_frac": adds_per_s / add_peak,
              "peak": "fp32 add lanes: SMs x 128 x 1.965 GHz (one signed add per key element and hyperplane)",
              "bytes": enc_keys * (cfg.d * 2 + cfg.bits // 8), "timing": "one call, L2 flushed before it"}

    # One CUDA graph per step (append -> select -> decode on that step's inputs);
    # capture runs nothing.  The timed graphs carry no trace events (an event
    # between two kernels would stop the next one from launching early); a
    # second set with trace events around every kernel gives the per-kernel
    # durations, replayed right after the timed steps.
    K = args.steps
    T = min(K, args.trace_steps)
    n_sel_kernels = eng.select_kernels(cache.capacity)
    sel_names = ["select_fused"] if n_sel_kernels == 1 else ["score_hist", "collect_select"]
    # --path step: the whole step as one clustered launch (dashkv_decode_step),
    # for token selection on the clustered path; otherwise the separate calls
    # (append, select, sparse decode), captured into one graph with
    # programmatic dependent launches between them
    fused = args.path == "step" and not (cfg.block or cfg.radius or cfg.tiers or n_sel_kernels != 1)
    # the kernels of one step, in launch order, and the calls that launch them
    if fused:
        calls = [("decode_step", ["decode_step"])]
        dom = "decode_step"
    else:
        dom = sel_names[0]  # the kernel that streams the codes (of the tokens, or of the block summaries)
        calls = [("append_keys", ["append_keys"])]
        if cfg.block:
            calls += [("append_blocks", ["append_blocks"]), ("select_blocks", sel_names + ["expand_blocks"])]
        elif cfg.radius:
            calls += [("append_radius", ["append_radius"]), ("select_radius", sel_names)]
        else:
            calls += [("select", sel_names)]
        calls += [("sparse_decode_tiered" if cfg.tiers else "sparse_decode", ["sparse_decode"])]
    kernels = [k for _, ks in calls for k in ks]
    n_graph = args.warmup + K + T

    def step(q, kn, vn, out, lse, e=None):
        """Enqueue one decode step; with events e, trace pair 1 + j around kernel j."""
        j = 1
        for name, ks in calls:
            if e is not None:
                eng.set_trace(e[2 * j:2 * (j + len(ks))])
            if name == "decode_step":
                eng.decode_step(cache, q, kn, vn, seq, buf["sel_idx"], buf["sel_cnt"], out, lse, ws)
            elif name == "append_keys":
                eng.append_keys(cache, kn, vn, seq)
            elif name == "append_blocks":
                eng.append_blocks(cache, index, seq)
            elif name == "select_blocks":
                eng.select_blocks(cache, index, q, seq, buf["sel_idx"], buf["sel_cnt"], None, ws)
            elif name == "append_radius":
                eng.append_radius(cache, radius, seq)
            elif name == "select_radius":
                eng.select_radius(cache, radius, q, seq, buf["sel_idx"], buf["sel_cnt"], None, ws)
            elif name == "select":
                eng.select(cache, q, seq, buf["sel_idx"], buf["sel_cnt"], None, ws)
            elif name == "sparse_decode_tiered":
                eng.sparse_decode_tiered(cache, tiers, q, buf["sel_idx"], buf["sel_cnt"], out, lse, ws, seq_lens=seq)
            else:
                eng.sparse_decode(cache, q, buf["sel_idx"], buf["sel_cnt"], out, lse, ws, seq_lens=seq)
            j += len(ks)
        if e is not None:
            eng.set_trace(None)

    def capture(s, e=None):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(w.q[s], w.k_new[s], w.v_new[s], buf["out"], buf["lse"], e)
        return g

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 + 2 * len(kernels))] for _ in range(n_graph)]
    for e in ev:  # materialise the CUDA events (torch creates them on first record)
        for x in e:
            x.record(stream)
    torch.cuda.synchronize(dev)
    graphs = [capture(s) for s in range(args.warmup + K)]
    traced = [capture(args.warmup + K + i, ev[args.warmup + K + i]) for i in range(T)]

    for s in range(args.warmup):
        flush(s)
        graphs[s].replay()
    torch.cuda.synchronize(dev)
    assert eng.get_error() == 0

    # ---- device-timed steps
    n_before = seq.clone()
    barrier(world)
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        wall0 = time.perf_counter()
        for rep in range(args.clock_reps):
            for i in range(K):
                s = args.warmup + i
                flush(i)
                ev[s][0].record(stream)
                graphs[s].replay()
                ev[s][1].record(stream)
            torch.cuda.synchronize(dev)
            if rep == 0:
                step_ms = [ev[args.warmup + i][0].elapsed_time(ev[args.warmup + i][1]) for i in range(K)]
                wall = time.perf_counter() - wall0
                # traced replays: per-kernel durations on the same workload
                for i in range(T):
                    flush(i)
                    traced[i].replay()
                torch.cuda.synchronize(dev)
                tb = args.warmup + K
                kern = {k: [ev[tb + i][2 + 2 * j].elapsed_time(ev[tb + i][3 + 2 * j]) for i in range(T)]
                        for j, k in enumerate(kernels)}
    # back-to-back replays of the same steps without the L2 flush (warm; reported
    # for reference only, labelled as such)
    for i in range(K):
        s = args.warmup + i
        ev[s][0].record(stream)
        graphs[s].replay()
        ev[s][1].record(stream)
    torch.cuda.synchronize(dev)
    warm_ms = sum(ev[args.warmup + i][0].elapsed_time(ev[args.warmup + i][1]) for i in range(K)) / K
    warm_ms = max_over_ranks(warm_ms, world)  # every rank takes part in the collective
    barrier(world)
    assert eng.get_error() == 0
    del graphs, traced
    sum_ms = max_over_ranks(sum(step_ms), world)
    ms_per_step = sum_ms / K
    value = world * cfg.B * K / (sum_ms / 1e3)

    # ---- algorithmic bytes (codes of every cached key -- or of every complete
    # block -- + selected K/V rows + q in / out)
    lens_mid = n_before.double() + 1 + (K - 1) / 2.0  # mean cache length over the timed steps
    scanned = lens_mid / cfg.block if cfg.block else lens_mid  # codes the scan reads per sequence
    code_bytes = float(scanned.sum()) * cfg.Hkv * cfg.bits / 8
    sel_rows = float(buf["sel_cnt"].sum())
    kv_bytes = sel_rows * 2 * cfg.d * 2
    fp8_rows = None
    if tiers is not None:  # rows of FP8 pages: 2 d code bytes + 2 exponents; every row: its page's tier byte
        idx = buf["sel_idx"].long()
        valid = torch.arange(idx.shape[-1], device=dev)[None, None, :] < buf["sel_cnt"][..., None]
        phys = w.page_table.long()[torch.arange(cfg.B, device=dev)[:, None, None], idx.clamp(min=0) // cfg.page_size]
        fp8_rows = float(((tiers.tier.long()[phys] == 1) & valid).sum())
        kv_bytes = (sel_rows - fp8_rows) * 2 * cfg.d * 2 + fp8_rows * (2 * cfg.d + 2) + sel_rows
    qo_bytes = cfg.B * cfg.Hq * cfg.d * (2 + 4)
    step_bytes = code_bytes + kv_bytes + qo_bytes
    peaks = measured_peaks()
    kms = {k: statistics.mean(v) for k, v in kern.items()}
    # the roofline kernel: the fused step kernel moves every byte of the step;
    # on the split path the selection kernel moves the codes
    dom_bytes = step_bytes if fused else code_bytes
    dom_gbs = dom_bytes / (kms[dom] * 1e-3) / 1e9
    kernel_gbs = {dom: dom_gbs}
    if "sparse_decode" in kms:
        kernel_gbs["sparse_decode"] = kv_bytes / (kms["sparse_decode"] * 1e-3) / 1e9
    step_gbs = step_bytes / (ms_per_step * 1e-3) / 1e9

    # ---- end to end through the C ABI with host buffers (pinned), copies timed.
    # The way a decode loop drives the library: each step's inputs packed in one
    # pinned buffer (q | k_new | v_new, one H2D copy), the three calls captured
    # once as a CUDA graph on fixed device buffers (the kernels read the lengths
    # on the device, so one graph serves every step), out | lse in one buffer
    # (one D2H copy).
    E = args.e2e_steps
    e2e = None
    if E > 0:
        nq, nk = w.q[0].numel(), w.k_new[0].numel()
        no, nl = buf["out"].numel(), buf["lse"].numel()
        hin = torch.empty((E, nq + 2 * nk), dtype=torch.bfloat16).pin_memory()
        for i in range(E):
            s = args.warmup + K + T + i
            hin[i, :nq] = w.q[s].reshape(-1).cpu()
            hin[i, nq:nq + nk] = w.k_new[s].reshape(-1).cpu()
            hin[i, nq + nk:] = w.v_new[s].reshape(-1).cpu()
        hout = torch.empty(no + nl, dtype=torch.float32).pin_memory()
        din = torch.empty(nq + 2 * nk, dtype=torch.bfloat16, device=dev)
        dout = torch.empty(no + nl, dtype=torch.float32, device=dev)
        dq = din[:nq].view(w.q[0].shape)
        dkn = din[nq:nq + nk].view(w.k_new[0].shape)
        dvn = din[nq + nk:].view(w.v_new[0].shape)
        out_v = dout[:no].view(buf["out"].shape)
        lse_v = dout[no:].view(buf["lse"].shape)
        din.copy_(hin[0], non_blocking=True)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(dq, dkn, dvn, out_v, lse_v)
        g.replay()  # upload the graph (one more appended token; the capacity covers it)
        torch.cuda.synchronize(dev)
        eev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(E)]
        barrier(world)
        for i in range(E):
            flush(i)
            eev[i][0].record(stream)
            din.copy_(hin[i], non_blocking=True)
            g.replay()
            hout.copy_(dout, non_blocking=True)
            eev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        barrier(world)
        assert eng.get_error() == 0
        del g
        e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in eev), world)
        e2e = {"value": world * cfg.B * E / (e_ms / 1e3), "unit": "queries/s",
               "h2d_bytes_per_step": hin[0].numel() * hin.element_size(),
               "d2h_bytes_per_step": hout.numel() * hout.element_size(), "steps": E,
               "how": "per step: one pinned H2D copy of (q | k_new | v_new), a CUDA graph of the step's calls "
                      f"({', '.join(n for n, _ in calls)}), one D2H copy of (out | lse); L2 flushed before each step"}

    cpu = None
    if rank == 0 and world == 1 and args.cpu_steps > 0:
        r = oracle_sample(cfg, args.cpu_steps)
        cpu = {"value": len(r["times"]) / sum(r["times"]), "unit": "queries/s", "cores": r["cores"],
               "kind": "oracle", "sample": r["sample"], "one_thread_value": 1.0 / r["one_thread_s"]}

    clk = clocks.summary()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "N": cfg.N, "Hq": cfg.Hq, "Hkv": cfg.Hkv, "d": cfg.d,
                       "bits": cfg.bits, "topk": cfg.topk, "sink": cfg.sink, "window": cfg.window,
                       "block": cfg.block or None, "radius": cfg.radius or None,
                       "tiers": "pages between the sinks and the window as FP8 E4M3 rows" if cfg.tiers else None,
                       "layout": "paged" if w.paged else "dense", "l2": "flushed before every step: 2 x L2 write, then 2 x L2 clean read (no pending write-backs)",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "hbm", "kernel": dom, "achieved": dom_gbs,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": dom_gbs / peaks["hbm_gbs"],
                         "peak_source": peaks["source"], "frac_of_8tbs": dom_gbs / SPEC_HBM_GBS,
                         "algorithmic_bytes_per_launch": dom_bytes,
                         "traffic": recorded_traffic(cfg.name, dom, dom_bytes)},
            "step_roofline": {"algorithmic_bytes": step_bytes, "achieved_gbs": step_gbs,
                              "frac": step_gbs / peaks["hbm_gbs"], "frac_of_8tbs": step_gbs / SPEC_HBM_GBS,
                              "code_bytes": code_bytes, "selected_kv_bytes": kv_bytes, "q_out_bytes": qo_bytes},
            "kernels_ms": kms,
            "kernel_gbs": kernel_gbs,
            "per_head_queries_per_s": value * cfg.Hq,
            "warm_ms_per_step": warm_ms,
            "encode": encode,
            "demote": demote,
            "fp8_selected_rows": fp8_rows,
            "codes_scanned_per_s": float(scanned.sum()) * cfg.Hkv / (ms_per_step * 1e-3),
            "selected_kv_bytes_per_s": kv_bytes / (ms_per_step * 1e-3),
            "e2e": e2e, "cpu_baseline": cpu, "gpu_launches": len(kernels) * K, "clocks": clk,
            "timing": f"one CUDA graph per step ({', '.join(n for n, _ in calls)}; programmatic dependent launches); events around each replay; kernels_ms from separately traced replays",
            "wall_s_timed_region": wall,
        }
        print(json.dumps(line), flush=True)
    eng.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["dashkv", "reference"], default="dashkv")
    ap.add_argument("--config", default="c128k", choices=sorted(W.CONFIGS))
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-steps", type=int, default=2)
    ap.add_argument("--two-kernel-select", action="store_true",
                    help="use the two-kernel selection path (and the separate calls)")
    ap.add_argument("--path", choices=["calls", "step"], default="calls",
                    help="calls: append_keys + select + sparse_decode, one graph per step (the faster path "
                         "at every configured workload); step: the one-launch dashkv_decode_step")
    ap.add_argument("--trace-steps", type=int, default=10,
                    help="extra traced steps for the per-kernel durations")
    ap.add_argument("--clock-reps", type=int, default=20,
                    help="replays of the timed steps while clocks are sampled (only the first is reported)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    cfg = W.CONFIGS[args.config]
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, cfg, world, rank)
        else:
            run_dashkv(args, cfg, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
