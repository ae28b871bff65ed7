"""NumPy front end of the CPU oracle (``dashkv_oracle.c``).

Test infrastructure only: the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use this module; the product library never
imports it.  Every function takes and returns NumPy arrays; floating-point
inputs are widened to float64 before they reach the C code, so bf16 values
arrive exactly.

The steps follow the pages' method (see the C file's header for the exact
definitions and the passages they come from): sign-random-projection key
codes, a full-precision query scored against those codes, exact top-k with
sinks and a recent window, then exact softmax attention over the selected
tokens only.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dashkv_oracle.c")
_LIB = os.path.join(_HERE, "libdashkv_oracle.so")


def build(force: bool = False) -> str:
    """Compile the C oracle in place (gcc, OpenMP) and return the .so path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-std=c11", "-Wall", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I, I64, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64
        L.dko_splitmix64_nth.argtypes = [U64, U64]
        L.dko_splitmix64_nth.restype = U64
        L.dko_hyperplanes.argtypes = [U64, I, I, P]
        L.dko_encode.argtypes = [I, I, I, I, I64, P, I, I, P, P, P, P]
        L.dko_append.argtypes = [I, I, I, I, I64, P, I, I, P, P, P, P, P, P, P]
        L.dko_scores.argtypes = [I, I, I, I, I, I64, P, I, I, P, P, P, P, P]
        L.dko_scores.restype = ctypes.c_double
        L.dko_select.argtypes = [I, I, I64, P, P, I, I, I, P, P, I]
        L.dko_select.restype = I
        L.dko_attend.argtypes = [I, I, I, I, I64, P, I, I, P, P, P, P, P, I, P, P]
        L.dko_encode_blocks.argtypes = [I, I, I, I, I64, P, I, I, P, P, I, P, I64, P]
        L.dko_select_blocks.argtypes = [I, I, I64, P, I, P, I, I, I, P, P, I]
        L.dko_select_blocks.restype = I
        L.dko_radius_code.argtypes = [P, I]
        L.dko_radius_code.restype = ctypes.c_uint8
        L.dko_radius_value.argtypes = [ctypes.c_uint8]
        L.dko_radius_value.restype = ctypes.c_double
        L.dko_radius_codes.argtypes = [I, I, I, I64, P, I, I, P, P, P]
        L.dko_radius_scale.argtypes = [I, I, I64, P, I, I, P, P, P, P]
        L.dko_e4m3_value.argtypes = [ctypes.c_uint8]
        L.dko_e4m3_value.restype = ctypes.c_double
        L.dko_e4m3_encode.argtypes = [ctypes.c_double]
        L.dko_e4m3_encode.restype = ctypes.c_uint8
        L.dko_tier_exponent.argtypes = [P, I]
        L.dko_tier_exponent.restype = I
        L.dko_tier_quantize_row.argtypes = [P, I, P, P]
        L.dko_demote_pages.argtypes = [I, I, I, I, P, I, P, P, P, I, I, P, P, P, P, P]
        L.dko_demote_pages.restype = I
        L.dko_set_threads.argtypes = [I]
        L.dko_get_threads.restype = I
        _lib = L
    return _lib


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def set_threads(n: int) -> None:
    lib().dko_set_threads(int(n))


def get_threads() -> int:
    return int(lib().dko_get_threads())


def splitmix64_nth(seed: int, n: int) -> int:
    return int(lib().dko_splitmix64_nth(seed & (2**64 - 1), n))


def hyperplanes(seed: int, bits: int, d: int) -> np.ndarray:
    """R[j][i] in {+1, -1}, shape [bits, d], int8."""
    R = np.empty((bits, d), dtype=np.int8)
    lib().dko_hyperplanes(seed & (2**64 - 1), bits, d, _p(R))
    return R


class Layout:
    """Dense ([B,Hkv,n_cap,d]) or paged ([P,page,Hkv,d] + page table) KV layout."""

    def __init__(self, B, Hkv, d, bits, n_cap=0, page_table=None, page=0):
        self.B, self.Hkv, self.d, self.bits = int(B), int(Hkv), int(d), int(bits)
        self.n_cap = int(n_cap)
        self.page = int(page)
        self.page_table = None if page_table is None else _i32(page_table)
        self.max_pages = 0 if page_table is None else int(self.page_table.shape[1])
        self.w64 = max(1, self.bits // 64)

    def args(self):
        return (self.B, self.Hkv, self.d, self.bits, self.n_cap,
                _p(self.page_table), self.max_pages, self.page)


def encode(layout: Layout, K, seq_lens, R, codes: np.ndarray | None = None) -> np.ndarray:
    """Codes for tokens [0, seq_lens[b]) in the layout's code shape (uint64)."""
    K = _f64(K)
    seq = _i32(seq_lens)
    R = np.ascontiguousarray(R, dtype=np.int8)
    if codes is None:
        if layout.page:
            P = K.shape[0]
            codes = np.zeros((P, layout.Hkv, layout.page, layout.w64), dtype=np.uint64)
        else:
            codes = np.zeros((layout.B, layout.Hkv, layout.n_cap, layout.w64), dtype=np.uint64)
    lib().dko_encode(*layout.args(), _p(K), _p(seq), _p(R), _p(codes))
    return codes


def append(layout: Layout, K: np.ndarray, V: np.ndarray, codes: np.ndarray, seq_lens: np.ndarray,
           k_new, v_new, R) -> None:
    """In-place append of one token per (b, kv head); K, V float64, seq_lens int32."""
    assert K.dtype == np.float64 and V.dtype == np.float64 and seq_lens.dtype == np.int32
    lib().dko_append(*layout.args(), _p(K), _p(V), _p(codes), _p(seq_lens),
                     _p(_f64(k_new)), _p(_f64(v_new)), _p(np.ascontiguousarray(R, dtype=np.int8)))


def scores(layout: Layout, Hq, q, codes, seq_lens, R):
    """(scores [B,Hkv,n_cap] float64 (NaN beyond seq_len), bound on |s|)."""
    n_cap = layout.n_cap if not layout.page else layout.max_pages * layout.page
    out = np.full((layout.B, layout.Hkv, n_cap), np.nan)
    # the C side uses n_cap as the scores row length (and, dense, as the KV row count)
    B, Hkv, d, bits, _, pt, mp, page = layout.args()
    bound = lib().dko_scores(B, int(Hq), Hkv, d, bits, n_cap, pt, mp, page,
                             _p(_f64(q)), _p(np.ascontiguousarray(codes, dtype=np.uint64)),
                             _p(_i32(seq_lens)), _p(np.ascontiguousarray(R, dtype=np.int8)), _p(out))
    return out, float(bound)


def select(scores_arr, seq_lens, topk, sink, window, cap=None):
    """(sel_idx [B,Hkv,cap] int32 ascending, -1 padded; sel_cnt [B,Hkv] int32)."""
    s = _f64(scores_arr)
    B, Hkv, n_cap = s.shape
    cap = int(cap if cap is not None else topk + sink + window)
    idx = np.empty((B, Hkv, cap), dtype=np.int32)
    cnt = np.empty((B, Hkv), dtype=np.int32)
    rc = lib().dko_select(B, Hkv, n_cap, _p(_i32(seq_lens)), _p(s), int(topk), int(sink),
                          int(window), _p(idx), _p(cnt), cap)
    if rc != 0:
        raise ValueError("selection larger than cap")
    return idx, cnt


def attend(layout: Layout, Hq, q, K, V, sel_idx, sel_cnt):
    """(out [B,Hq,d] float64, lse [B,Hq] float64)."""
    sel_idx = _i32(sel_idx)
    cap = sel_idx.shape[-1]
    out = np.empty((layout.B, int(Hq), layout.d))
    lse = np.empty((layout.B, int(Hq)))
    B, Hkv, d, _, n_cap, pt, mp, page = layout.args()
    lib().dko_attend(B, int(Hq), Hkv, d, n_cap, pt, mp, page, _p(_f64(q)), _p(_f64(K)), _p(_f64(V)),
                     _p(sel_idx), _p(_i32(sel_cnt)), cap, _p(out), _p(lse))
    return out, lse


def decode_step(layout: Layout, Hq, q, K, V, codes, seq_lens, R, topk, sink, window):
    """Score -> select -> attend for one decode query batch (no append)."""
    sc, bound = scores(layout, Hq, q, codes, seq_lens, R)
    idx, cnt = select(sc, seq_lens, topk, sink, window)
    out, lse = attend(layout, Hq, q, K, V, idx, cnt)
    return dict(scores=sc, bound=bound, sel_idx=idx, sel_cnt=cnt, out=out, lse=lse)


# ---------------------------------------------------------------- block summaries
# CSA-style two-level index (DeepSeek DSA->CSA/HCA page, CSA section and the
# section on the compressed versus the state cache): the summary of each
# complete block of m tokens is the code of the block's summed key, the top
# blocks are selected by the same asymmetric score, and attention runs exactly
# over their tokens, the sinks, the window and the incomplete tail.

def block_capacity(n_cap: int, block: int) -> int:
    """Blocks a cache of n_cap tokens can hold (complete blocks only)."""
    return int(n_cap) // int(block)


def encode_blocks(layout: Layout, K, seq_lens, block: int, R, nb_cap: int) -> np.ndarray:
    """Summary codes [B, Hkv, nb_cap, W64] (uint64, canonical bit order) of the
    complete blocks [0, seq_lens[b] // block); other entries 0."""
    codes = np.zeros((layout.B, layout.Hkv, int(nb_cap), layout.w64), dtype=np.uint64)
    lib().dko_encode_blocks(*layout.args(), _p(_f64(K)), _p(_i32(seq_lens)), int(block),
                            _p(np.ascontiguousarray(R, dtype=np.int8)), int(nb_cap), _p(codes))
    return codes


def block_scores(layout: Layout, Hq, q, block_codes, seq_lens, block: int, R):
    """(scores [B, Hkv, nb_cap] float64 of the complete blocks (NaN beyond), bound):
    the asymmetric score of each block's summary code."""
    nb_cap = int(block_codes.shape[2])
    L = Layout(layout.B, layout.Hkv, layout.d, layout.bits, n_cap=nb_cap)
    return scores(L, Hq, q, block_codes, _i32(seq_lens) // int(block), R)


def select_blocks(bscores, seq_lens, block: int, topk_blocks: int, sink: int, window: int, cap: int):
    """(sel_idx [B, Hkv, cap] int32 ascending token ids, -1 padded; sel_cnt [B, Hkv])."""
    s = _f64(bscores)
    B, Hkv, nb_cap = s.shape
    idx = np.empty((B, Hkv, int(cap)), dtype=np.int32)
    cnt = np.empty((B, Hkv), dtype=np.int32)
    rc = lib().dko_select_blocks(B, Hkv, nb_cap, _p(_i32(seq_lens)), int(block), _p(s), int(topk_blocks),
                                 int(sink), int(window), _p(idx), _p(cnt), int(cap))
    if rc != 0:
        raise ValueError("selection larger than cap")
    return idx, cnt


def decode_step_blocks(layout: Layout, Hq, q, K, V, block_codes, seq_lens, R, block, topk_blocks, sink, window,
                       cap):
    """Block score -> block select -> exact attention for one decode query batch."""
    bs, bound = block_scores(layout, Hq, q, block_codes, seq_lens, block, R)
    idx, cnt = select_blocks(bs, seq_lens, block, topk_blocks, sink, window, cap)
    out, lse = attend(layout, Hq, q, K, V, idx, cnt)
    return dict(block_scores=bs, bound=bound, sel_idx=idx, sel_cnt=cnt, out=out, lse=lse)


# ---------------------------------------------------------------- radius scaling
# Spherical KV page, section 2.1 ADA: a quantized key radius r~ beside the
# angle code, logits estimated as |q| r~ f_b(codes).  Here s'_t = r~_t s_t (the
# constant |q| does not change the ranking); 8-bit radius codes, step 1/4.

def radius_code(k) -> int:
    """c = min(255, floor(4 sqrtf(sum k_i^2))) (fp32 sum, i ascending)."""
    k = _f64(k)
    return int(lib().dko_radius_code(_p(k), int(k.shape[-1])))


def radius_value(c: int) -> float:
    """r~ = (c + 1/2) / 4."""
    return float(lib().dko_radius_value(int(c)))


def radius_codes(layout: Layout, K, seq_lens) -> np.ndarray:
    """uint8 radius codes of tokens [0, seq_lens[b]): dense [B, Hkv, n_cap],
    paged [P, Hkv, page] (zero elsewhere)."""
    K = _f64(K)
    if layout.page:
        rc = np.zeros((K.shape[0], layout.Hkv, layout.page), dtype=np.uint8)
    else:
        rc = np.zeros((layout.B, layout.Hkv, layout.n_cap), dtype=np.uint8)
    lib().dko_radius_codes(layout.B, layout.Hkv, layout.d, layout.n_cap, _p(layout.page_table), layout.max_pages,
                           layout.page, _p(K), _p(_i32(seq_lens)), _p(rc))
    return rc


def radius_scale(layout: Layout, scores_arr, seq_lens, rc) -> np.ndarray:
    """s' = fp32(r~_t * fp32(s_t)) for t < seq_lens[b] (NaN elsewhere), float64."""
    s = _f64(scores_arr)
    out = np.full_like(s, np.nan)
    B, Hkv, n_cap = s.shape
    lib().dko_radius_scale(B, Hkv, n_cap, _p(layout.page_table), layout.max_pages, layout.page,
                           _p(_i32(seq_lens)), _p(np.ascontiguousarray(rc, dtype=np.uint8)), _p(s), _p(out))
    return out


def decode_step_radius(layout: Layout, Hq, q, K, V, codes, rc, seq_lens, R, topk, sink, window):
    """Score -> radius scale -> select -> attend for one decode query batch."""
    sc, bound = scores(layout, Hq, q, codes, seq_lens, R)
    ss = radius_scale(layout, sc, seq_lens, rc)
    idx, cnt = select(ss, seq_lens, topk, sink, window)
    out, lse = attend(layout, Hq, q, K, V, idx, cnt)
    return dict(scores=ss, unscaled=sc, bound=bound, sel_idx=idx, sel_cnt=cnt, out=out, lse=lse)


# ---------------------------------------------------------------- precision tiers
# Tier-homogeneous pages (Spherical KV page, section 2.2 RDR; DASH-KV page,
# section "技术架构：动态混合精度机制"): pages whose tokens all lie between the
# sinks and the window are demoted to FP8 E4M3 rows with a power-of-two scale
# per (token, kv head) row; attention reads those rows dequantized.  The C
# file's section on precision tiers has the exact definitions.

def e4m3_value(c: int) -> float:
    """Value of an FP8 E4M3 (FN) code (NaN for the two NaN codes)."""
    return float(lib().dko_e4m3_value(int(c) & 0xFF))


def e4m3_encode(v: float) -> int:
    """Nearest E4M3 code of v, ties to even (|v| <= 448)."""
    return int(lib().dko_e4m3_encode(float(v)))


def tier_exponent(x) -> int:
    """s = the largest integer with max|x| * 2^s <= 448, capped at 127 (0 for a zero row)."""
    x = _f64(x)
    return int(lib().dko_tier_exponent(_p(x), int(x.shape[-1])))


def tier_quantize_row(x):
    """(codes uint8 [d], s) of one row."""
    x = _f64(x)
    codes = np.empty(x.shape[-1], dtype=np.uint8)
    s = np.zeros(1, dtype=np.int8)
    lib().dko_tier_quantize_row(_p(x), int(x.shape[-1]), _p(codes), _p(s))
    return codes, int(s[0])


def tier_arrays(num_pages: int, page: int, Hkv: int, d: int):
    """Zeroed (tier [P], k8 [P,page,Hkv,d], v8, exps [P,page,Hkv,2]) arrays."""
    return (np.zeros(num_pages, dtype=np.uint8), np.zeros((num_pages, page, Hkv, d), dtype=np.uint8),
            np.zeros((num_pages, page, Hkv, d), dtype=np.uint8), np.zeros((num_pages, page, Hkv, 2), dtype=np.int8))


def demote_pages(layout: Layout, K, V, seq_lens, sink: int, window: int, tier, k8, v8, exps, protect=None) -> int:
    """The page controller on a paged layout; updates tier / k8 / v8 / exps in
    place and returns the number of pages demoted."""
    assert layout.page > 0, "tiers are defined on paged layouts"
    for a, dt in ((tier, np.uint8), (k8, np.uint8), (v8, np.uint8), (exps, np.int8)):
        assert a.dtype == dt and a.flags.c_contiguous
    pr = None if protect is None else np.ascontiguousarray(protect, dtype=np.uint8)
    return int(lib().dko_demote_pages(layout.B, layout.Hkv, layout.d, layout.page, _p(layout.page_table),
                                      layout.max_pages, _p(_f64(K)), _p(_f64(V)), _p(_i32(seq_lens)), int(sink),
                                      int(window), _p(pr), _p(tier), _p(k8), _p(v8), _p(exps)))


def e4m3_table() -> np.ndarray:
    """Values of all 256 codes (float64)."""
    return np.array([e4m3_value(c) for c in range(256)])


def dequantized(K, V, tier, k8, v8, exps):
    """K / V as attention reads them: rows of tier-1 pages replaced by
    value(c) * 2^-s, the others unchanged (paged layout, float64)."""
    K = _f64(K).copy()
    V = _f64(V).copy()
    tab = e4m3_table()
    for p in np.nonzero(np.asarray(tier) == 1)[0]:
        K[p] = tab[k8[p]] * np.ldexp(1.0, -exps[p][..., 0:1].astype(np.int64))
        V[p] = tab[v8[p]] * np.ldexp(1.0, -exps[p][..., 1:2].astype(np.int64))
    return K, V


def attend_tiered(layout: Layout, Hq, q, K, V, tier, k8, v8, exps, sel_idx, sel_cnt):
    """Exact attention over the selection with tier-1 rows dequantized."""
    Kd, Vd = dequantized(K, V, tier, k8, v8, exps)
    return attend(layout, Hq, q, Kd, Vd, sel_idx, sel_cnt)
