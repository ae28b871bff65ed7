"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point its header declares, validates configurations before it
touches a device, and its hyperplane generator agrees with the oracle's
independently written one."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest
import torch

from hash_indexed_top_b200 import build as B
from hash_indexed_top_b200 import dashkv as dk
from oracle import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()


def header_functions():
    src = open(os.path.join(ROOT, "include", "dashkv.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dashkv_[a-z_]+)\s*\(", src)))


def test_header_declares_the_four_calls():
    fns = header_functions()
    for f in ("dashkv_encode_keys", "dashkv_append_keys", "dashkv_select", "dashkv_sparse_decode"):
        assert f in fns


def test_library_exports_every_declared_symbol():
    fns = header_functions()
    assert set(fns) == set(dk.SYMBOLS)
    L = dk.lib()
    for f in fns:
        assert getattr(L, f) is not None
    out = subprocess.run(["nm", "-D", "--defined-only", dk.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(dashkv_\w+)", out))
    assert set(fns) <= exported


def test_status_strings():
    L = dk.lib()
    for code, text in dk.STATUS.items():
        assert L.dashkv_status_str(code).decode() == text


@pytest.mark.parametrize("seed,bits,d", [(0x5EEDDA5B, 128, 128), (1, 64, 128), (7, 32, 64), (2**63 + 5, 128, 64)])
def test_library_hyperplanes_match_oracle(seed, bits, d):
    a = dk.hyperplanes(seed, bits, d).numpy()
    b = O.hyperplanes(seed, bits, d)
    assert np.array_equal(a, b)


def _cfg(**kw):
    base = dict(batch=1, num_q_heads=4, num_kv_heads=1, head_dim=64, bits=32, topk=8, sink=0, window=0,
                page_size=0, flags=0, seed=1)
    base.update(kw)
    return dk.Config(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=96), 2), (dict(bits=48), 2), (dict(bits=256), 2), (dict(num_q_heads=12, num_kv_heads=1), 2),
    (dict(num_q_heads=6, num_kv_heads=4), 1), (dict(topk=0), 1), (dict(sink=-1), 1), (dict(page_size=48), 2),
    (dict(batch=0), 1), (dict(flags=6), 1), (dict(num_q_heads=64, num_kv_heads=64), 2),
    (dict(page_size=1056), 2), (dict(window=-1), 1), (dict(topk=2**30, sink=2**29, window=2**29), 1),
])
def test_create_rejects_bad_configs(kw, status):
    h = ctypes.c_void_p()
    cfg = _cfg(**kw)
    assert dk.lib().dashkv_create(ctypes.byref(cfg), ctypes.byref(h)) == status
    assert not h.value


@pytest.mark.skipif(torch.cuda.is_available(), reason="host without a GPU only")
def test_create_without_device_reports_no_device():
    h = ctypes.c_void_p()
    cfg = _cfg()
    assert dk.lib().dashkv_create(ctypes.byref(cfg), ctypes.byref(h)) == 7
    with pytest.raises(RuntimeError):
        dk.DashKV(1, 4, 1, 64, 32, 8, 0, 0)


@pytest.mark.parametrize("bits", [32, 64, 128])
def test_canonical_codes_undoes_the_storage_rotation(bits):
    # stored byte p of token t holds code byte (p + t mod T) mod T
    T, W = bits // 8, max(1, bits // 64)
    rng = np.random.default_rng(bits)
    orig = rng.integers(0, 256, size=(2, 3, 70, W * 8), dtype=np.uint8)
    orig[..., T:] = 0
    stored = np.zeros_like(orig)
    for t in range(70):
        for p in range(T):
            stored[:, :, t, p] = orig[:, :, t, (p + t % T) % T]
    st = torch.from_numpy(stored.copy()).view(torch.int64).reshape(2, 3, 70, W)
    back = dk.canonical_codes(st, bits).view(torch.uint8).reshape(2, 3, 70, W * 8).numpy()
    assert np.array_equal(back, orig)


def test_block_view_layout_and_index_shapes():
    # dashkv_block_view: { uint64_t *codes; int64_t nb_cap; int32_t block; int32_t reserved; }
    assert ctypes.sizeof(dk.BlockView) == 24
    assert [dk.BlockView.codes.offset, dk.BlockView.nb_cap.offset, dk.BlockView.block.offset,
            dk.BlockView.reserved.offset] == [0, 8, 16, 20]
    # summaries for every complete block the cache holds: dense and paged
    K = torch.zeros((3, 2, 1001, 64), dtype=torch.bfloat16)
    dense = dk.KVCache(K, K, dk.KVCache.empty_codes_like(K, 128, False))
    idx = dk.BlockIndex.empty_for(dense, 3, 128, 8)
    assert tuple(idx.codes.shape) == (3, 2, 125, 2) and idx.capacity == 125
    v = idx.view()
    assert v.nb_cap == 125 and v.block == 8 and v.reserved == 0
    Kp = torch.zeros((10, 64, 4, 128), dtype=torch.bfloat16)
    pt = torch.zeros((2, 7), dtype=torch.int32)
    paged = dk.KVCache(Kp, Kp, dk.KVCache.empty_codes_like(Kp, 64, True), pt)
    idx = dk.BlockIndex.empty_for(paged, 2, 64, 16)
    assert tuple(idx.codes.shape) == (2, 4, 7 * 64 // 16, 1)


def test_tier_view_layout_and_page_tier_shapes():
    # dashkv_tier_view: { uint8_t *tier; uint8_t *k8; uint8_t *v8; int8_t *exps; }
    assert ctypes.sizeof(dk.TierView) == 32
    assert [dk.TierView.tier.offset, dk.TierView.k8.offset, dk.TierView.v8.offset,
            dk.TierView.exps.offset] == [0, 8, 16, 24]
    Kp = torch.zeros((10, 64, 4, 128), dtype=torch.bfloat16)
    pt = torch.zeros((2, 7), dtype=torch.int32)
    paged = dk.KVCache(Kp, Kp, dk.KVCache.empty_codes_like(Kp, 64, True), pt)
    t = dk.PageTiers.empty_for(paged)
    assert tuple(t.tier.shape) == (10,) and t.tier.dtype == torch.uint8
    assert tuple(t.k8.shape) == (10, 64, 4, 128) and tuple(t.v8.shape) == (10, 64, 4, 128)
    assert tuple(t.exps.shape) == (10, 64, 4, 2) and t.exps.dtype == torch.int8
    assert not t.tier.any() and t.view().tier == t.tier.data_ptr()
    K = torch.zeros((3, 2, 100, 64), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        dk.PageTiers.empty_for(dk.KVCache(K, K, dk.KVCache.empty_codes_like(K, 64, False)))
