"""The device error word on the GPU: problems only the device can see -- a
sequence length beyond the cache capacity, a page id outside the pages the
view declares -- are reported by dashkv_get_error, the affected tokens are
skipped, and the rest of the result stays the oracle's.

No case here can fault: every buffer is allocated larger than the view
declares, so a token the checks failed to skip would still read valid memory
(and show up as a parity failure, not a fault)."""
import numpy as np
import pytest
import torch

from hash_indexed_top_b200 import dashkv as dk
from hash_indexed_top_b200 import workloads as W
from oracle import oracle as O

from pipeline import within_tol

pytestmark = pytest.mark.gpu

ERR_CAPACITY, ERR_DEVICE = 4, 6


class DeclaredCache(dk.KVCache):
    """A cache whose view declares fewer physical pages than its tensors hold."""

    def __init__(self, k, v, codes, page_table, num_pages_declared):
        super().__init__(k, v, codes, page_table)
        self.num_pages_declared = num_pages_declared

    def view(self) -> dk.KVView:
        v = super().view()
        v.num_pages = self.num_pages_declared
        return v


def _oracle_pair(cfg, K, V, n, b, h, q, R):
    """Oracle step for pair (b, h) over its first n cached rows (dense [B,Hkv,cap,d] numpy)."""
    L = O.Layout(1, 1, cfg.d, cfg.bits, n_cap=max(n, 1))
    sl = np.array([n], dtype=np.int32)
    Kp = np.ascontiguousarray(K[b:b + 1, h:h + 1, :max(n, 1)])
    Vp = np.ascontiguousarray(V[b:b + 1, h:h + 1, :max(n, 1)])
    codes = O.encode(L, Kp, sl, R)
    G = cfg.G
    return O.decode_step(L, G, q[b, h * G:(h + 1) * G].reshape(1, G, cfg.d), Kp, Vp, codes, sl, R, cfg.topk,
                         cfg.sink, cfg.window)


@pytest.mark.parametrize("path", ["fused", "two_kernel", "step"])
def test_length_beyond_capacity_is_reported_and_clamped(path):
    cfg = W.Config("cap", B=2, Hq=4, Hkv=2, d=64, N=900, bits=64, topk=50, sink=2, window=8, steps=1,
                   needles=2, seed=91)
    dev = torch.device("cuda")
    w = W.make_workload(cfg, device="cpu", steps=1)
    n_cap = w.n_cap
    # the cache tensors are views of the front of larger buffers
    extra = 64
    kbig = torch.zeros((cfg.B * cfg.Hkv * n_cap + extra) * cfg.d, dtype=torch.bfloat16, device=dev)
    vbig = torch.zeros_like(kbig)
    cbig = torch.zeros((cfg.B * cfg.Hkv * n_cap + extra) * 1, dtype=torch.int64, device=dev)
    K = kbig[:cfg.B * cfg.Hkv * n_cap * cfg.d].view(cfg.B, cfg.Hkv, n_cap, cfg.d)
    V = vbig[:cfg.B * cfg.Hkv * n_cap * cfg.d].view(cfg.B, cfg.Hkv, n_cap, cfg.d)
    K.copy_(w.K)
    V.copy_(w.V)
    codes = cbig[:cfg.B * cfg.Hkv * n_cap].view(cfg.B, cfg.Hkv, n_cap, 1)
    eng = dk.DashKV(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.bits, cfg.topk, cfg.sink, cfg.window, 0,
                    W.HYPERPLANE_SEED, two_kernel_select=path == "two_kernel")
    try:
        cache = dk.KVCache(K, V, codes)
        seq_ok = torch.tensor([n_cap, 600], dtype=torch.int32, device=dev)
        eng.encode_keys(cache, seq_ok)  # every row the view holds
        assert eng.get_error() == 0
        seq = torch.tensor([n_cap + 7, 600], dtype=torch.int32, device=dev)  # sequence 0 outgrew its cache
        buf = eng.alloc_step(dev)
        q = w.q[0].to(dev)
        if path == "step":
            eng.decode_step(cache, q, w.k_new[0].to(dev), w.v_new[0].to(dev), seq, buf["sel_idx"],
                            buf["sel_cnt"], buf["out"], buf["lse"])
        else:
            eng.select(cache, q, seq, buf["sel_idx"], buf["sel_cnt"])
            eng.sparse_decode(cache, q, buf["sel_idx"], buf["sel_cnt"], buf["out"], buf["lse"], seq_lens=seq)
        assert eng.get_error() == ERR_CAPACITY
        assert eng.get_error() == 0  # read and cleared
        # the oracle's cache: the workload's rows, plus the step's append where one happened
        Kh = w.K.double().numpy().copy()
        Vh = w.V.double().numpy().copy()
        if path == "step":  # the append to sequence 0 was refused; sequence 1's went in
            assert seq.tolist() == [n_cap + 7, 601]
            Kh[1, :, 600] = w.k_new[0][1].double().numpy()
            Vh[1, :, 600] = w.v_new[0][1].double().numpy()
        R = O.hyperplanes(W.HYPERPLANE_SEED, cfg.bits, cfg.d)
        qh = q.cpu().double().numpy()
        for b, n in ((0, n_cap), (1, int(seq[1]))):  # sequence 0 is taken at its capacity
            for h in range(cfg.Hkv):
                r = _oracle_pair(cfg, Kh, Vh, n, b, h, qh, R)
                assert int(buf["sel_cnt"][b, h]) == int(r["sel_cnt"][0, 0]), (b, h)
                assert np.array_equal(buf["sel_idx"][b, h].cpu().numpy(), r["sel_idx"][0, 0]), (b, h)
                G = cfg.G
                out = buf["out"][b, h * G:(h + 1) * G].cpu().double().numpy()
                assert within_tol(out, r["out"][0]).all(), (b, h)
    finally:
        eng.close()


@pytest.mark.parametrize("path", ["fused", "two_kernel", "step"])
def test_page_id_out_of_declared_range_is_reported(path):
    cfg = W.Config("page", B=2, Hq=4, Hkv=2, d=64, N=700, bits=64, topk=40, sink=2, window=8, steps=1,
                   needles=2, page_size=64, seed=92)
    dev = torch.device("cuda")
    w = W.make_workload(cfg, device="cpu", steps=1)
    P = w.num_pages
    spare = 3  # physical pages beyond the declared ones
    ps = cfg.page_size
    K = torch.zeros((P + spare, ps, cfg.Hkv, cfg.d), dtype=torch.bfloat16, device=dev)
    V = torch.zeros_like(K)
    K[:P] = w.K.to(dev)
    V[:P] = w.V.to(dev)
    codes = torch.zeros((P + spare, cfg.Hkv, ps, 1), dtype=torch.int64, device=dev)
    pt = w.page_table.clone()
    bad_slot = 2
    pt[1, bad_slot] = P + 1  # sequence 1: one page outside the declared range (valid memory)
    pt = pt.to(dev)
    eng = dk.DashKV(cfg.B, cfg.Hq, cfg.Hkv, cfg.d, cfg.bits, cfg.topk, cfg.sink, cfg.window, ps,
                    W.HYPERPLANE_SEED, two_kernel_select=path == "two_kernel")
    try:
        good = DeclaredCache(K, V, codes, w.page_table.to(dev), P)
        seq = w.seq_lens.to(dev).clone()
        eng.encode_keys(good, seq)
        assert eng.get_error() == 0
        cache = DeclaredCache(K, V, codes, pt, P)
        buf = eng.alloc_step(dev)
        q = w.q[0].to(dev)
        if path == "step":
            eng.decode_step(cache, q, w.k_new[0].to(dev), w.v_new[0].to(dev), seq, buf["sel_idx"],
                            buf["sel_cnt"], buf["out"], buf["lse"])
        else:
            eng.select(cache, q, seq, buf["sel_idx"], buf["sel_cnt"])
            eng.sparse_decode(cache, q, buf["sel_idx"], buf["sel_cnt"], buf["out"], buf["lse"], seq_lens=seq)
        assert eng.get_error() == ERR_DEVICE
        assert eng.get_error() == 0
        # sequence 0 never touches the bad page: its results are the oracle's,
        # on the workload's rows (plus the step's appended row)
        n_before = int(w.seq_lens[0])
        n0 = int(seq[0])
        assert n0 == n_before + (1 if path == "step" else 0)
        Kd = np.zeros((1, cfg.Hkv, n0, cfg.d))
        Vd = np.zeros((1, cfg.Hkv, n0, cfg.d))
        t = np.arange(n_before)
        phys = w.page_table[0].numpy()[t // ps]
        Kc, Vc = w.K.double().numpy(), w.V.double().numpy()
        for h in range(cfg.Hkv):
            Kd[0, h, :n_before] = Kc[phys, t % ps, h]
            Vd[0, h, :n_before] = Vc[phys, t % ps, h]
        if path == "step":
            Kd[0, :, n_before] = w.k_new[0][0].double().numpy()
            Vd[0, :, n_before] = w.v_new[0][0].double().numpy()
        R = O.hyperplanes(W.HYPERPLANE_SEED, cfg.bits, cfg.d)
        qh = q.cpu().double().numpy()
        for h in range(cfg.Hkv):
            r = _oracle_pair(cfg, Kd, Vd, n0, 0, h, qh, R)
            assert int(buf["sel_cnt"][0, h]) == int(r["sel_cnt"][0, 0]), h
            assert np.array_equal(buf["sel_idx"][0, h].cpu().numpy(), r["sel_idx"][0, 0]), h
            G = cfg.G
            out = buf["out"][0, h * G:(h + 1) * G].cpu().double().numpy()
            assert within_tol(out, r["out"][0]).all(), h
    finally:
        eng.close()
