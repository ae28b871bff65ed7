"""Host logic of bench.py that needs no GPU: the DRAM-traffic figure of the
roofline object is taken from the committed ncu summary only while the
kernel code it was measured on is unchanged (comments may change)."""
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_strip_comments_keeps_code_and_string_literals():
    src = 'int a = 1; // one\n/* block\n comment */ const char *p = "x//y/*z*/";\nint  b;'
    assert bench._strip_comments(src) == 'int a = 1; const char *p = "x//y/*z*/"; int b;'


def test_recorded_traffic_follows_the_kernel_code(tmp_path, monkeypatch):
    shutil.copytree(os.path.join(ROOT, "hash_indexed_top_b200", "csrc"), tmp_path / "hash_indexed_top_b200" / "csrc")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    summary = tmp_path / "profiles" / "decode_step_c128k.txt"
    assert bench.recorded_traffic("c128k", "decode_step") is None  # no summary, no figure
    summary.write_text("workload: c128k\n"
                       f"kernel sources sha256: {bench.kernel_sources_sha()}\n"
                       "traffic_per_launch decode_step 123456\n")
    assert bench.recorded_traffic("c128k", "decode_step") == 123456  # taken from these kernels
    assert bench.recorded_traffic("c1m", "decode_step") is None  # another workload
    assert bench.recorded_traffic("c128k", "score_hist") is None  # not measured
    src = tmp_path / "hash_indexed_top_b200" / "csrc" / "step.cuh"
    src.write_text("// a comment-only change\n" + src.read_text())
    assert bench.recorded_traffic("c128k", "decode_step") == 123456  # comments do not make the counters stale
    src.write_text(src.read_text() + "\nstatic int changed_code = 1;\n")
    assert bench.recorded_traffic("c128k", "decode_step") is None  # a code change does


def test_oracle_block_update_matches_a_whole_cache_encode():
    # the bench's CPU-baseline leg keeps block summaries up to date one append
    # at a time; after every step they must equal a from-scratch encode
    import numpy as np
    from hash_indexed_top_b200 import workloads as W
    from oracle import oracle as O
    cfg = W.CONFIGS["tiny"].scaled(name="tiny_b8", N=101, block=8)
    steps = 20
    w = W.make_workload(cfg, device="cpu", steps=steps)
    R = O.hyperplanes(W.HYPERPLANE_SEED, cfg.bits, cfg.d)
    L = O.Layout(1, cfg.Hkv, cfg.d, cfg.bits, n_cap=w.n_cap)
    K = w.K.double().numpy().copy()
    V = w.V.double().numpy().copy()
    seq = w.seq_lens.numpy().astype(np.int32).copy()
    codes = O.encode(L, K, seq, R)
    nb_cap = w.n_cap // cfg.block
    bcodes = O.encode_blocks(L, K, seq, cfg.block, R, nb_cap)
    completed = 0
    for s in range(steps):
        O.append(L, K, V, codes, seq, w.k_new[s].double().numpy(), w.v_new[s].double().numpy(), R)
        bench.oracle_block_update(L, K, bcodes, int(seq[0]), cfg.block, R)
        completed += int(seq[0]) % cfg.block == 0
        assert np.array_equal(bcodes, O.encode_blocks(L, K, seq, cfg.block, R, nb_cap)), s
    assert completed >= 2


def test_oracle_sample_runs_paged_and_tiered_workloads_as_one_dense_sequence():
    # the CPU baseline times one sequence of the workload at its longest
    # length, dense; the tiered workload demotes its middle pages first
    from hash_indexed_top_b200 import workloads as W
    for name in ("ragged_paged", "ragged_paged_fp8"):
        cfg = W.CONFIGS[name].scaled(N=3000, n_min=500, topk=128, window=64)
        r = bench.oracle_sample(cfg, 2)
        assert len(r["times"]) == 2 and all(t > 0 for t in r["times"])
        assert "N=3000" in r["sample"]
        assert ("FP8" in r["sample"]) == (name == "ragged_paged_fp8")
