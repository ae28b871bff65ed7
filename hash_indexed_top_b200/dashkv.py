"""Python binding of ``libdashkv.so`` (C ABI in ``include/dashkv.h``).

Argument marshalling only: every stage of the decode step runs in the
library's CUDA kernels.  PyTorch provides device memory and streams; tensors
are passed to the C calls as raw pointers.  There is no CPU fallback -- if the
shared library is missing or no CUDA device is present, the calls raise.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdashkv.so")

STATUS = {
    0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "workspace missing or too small",
    4: "sequence length beyond cache capacity", 5: "CUDA error", 6: "page id out of range", 7: "no CUDA device",
    8: "a bounded wait in a kernel gave up",
}

FLAG_TWO_KERNEL_SELECT = 1

SYMBOLS = ("dashkv_create", "dashkv_destroy", "dashkv_workspace_size", "dashkv_encode_keys",
           "dashkv_append_keys", "dashkv_select", "dashkv_sparse_decode", "dashkv_get_error",
           "dashkv_hyperplanes", "dashkv_set_trace", "dashkv_select_kernels", "dashkv_status_str",
           "dashkv_select_static", "dashkv_encode_blocks", "dashkv_append_blocks", "dashkv_select_blocks",
           "dashkv_encode_radius", "dashkv_append_radius", "dashkv_select_radius", "dashkv_decode_step",
           "dashkv_demote_pages", "dashkv_sparse_decode_tiered")


class DashKVError(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call}: {STATUS.get(status, status)} (status {status})")
        self.status = status


class Config(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("bits", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("sink", ctypes.c_int32), ("window", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("flags", ctypes.c_int32), ("seed", ctypes.c_uint64)]


class KVView(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("codes", ctypes.c_void_p),
                ("n_cap", ctypes.c_int64), ("page_table", ctypes.c_void_p), ("max_pages", ctypes.c_int32),
                ("num_pages", ctypes.c_int32)]


class TierView(ctypes.Structure):
    _fields_ = [("tier", ctypes.c_void_p), ("k8", ctypes.c_void_p), ("v8", ctypes.c_void_p),
                ("exps", ctypes.c_void_p)]


class BlockView(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("nb_cap", ctypes.c_int64), ("block", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libdashkv.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with hash_indexed_top_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, I32, U64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint64, ctypes.c_size_t
        L.dashkv_create.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(P)]
        L.dashkv_create.restype = ctypes.c_int
        L.dashkv_destroy.argtypes = [P]
        L.dashkv_destroy.restype = None
        L.dashkv_workspace_size.argtypes = [P, ctypes.c_int64]
        L.dashkv_workspace_size.restype = SZ
        L.dashkv_encode_keys.argtypes = [P, ctypes.POINTER(KVView), P, P]
        L.dashkv_append_keys.argtypes = [P, ctypes.POINTER(KVView), P, P, P, P]
        L.dashkv_select.argtypes = [P, ctypes.POINTER(KVView), P, P, P, P, P, P, SZ, P]
        L.dashkv_sparse_decode.argtypes = [P, ctypes.POINTER(KVView), P, P, P, P, P, P, P, SZ, P]
        L.dashkv_select_static.argtypes = [P, ctypes.POINTER(KVView), P, P, P, P, P, P]
        L.dashkv_decode_step.argtypes = [P, ctypes.POINTER(KVView), P, P, P, P, P, P, P, P, P, SZ, P]
        L.dashkv_encode_blocks.argtypes = [P, ctypes.POINTER(KVView), ctypes.POINTER(BlockView), P, P]
        L.dashkv_append_blocks.argtypes = [P, ctypes.POINTER(KVView), ctypes.POINTER(BlockView), P, P]
        L.dashkv_select_blocks.argtypes = [P, ctypes.POINTER(KVView), ctypes.POINTER(BlockView), P, P, P, P, P, P,
                                           SZ, P]
        L.dashkv_encode_radius.argtypes = [P, ctypes.POINTER(KVView), P, P, P]
        L.dashkv_append_radius.argtypes = [P, ctypes.POINTER(KVView), P, P, P]
        L.dashkv_select_radius.argtypes = [P, ctypes.POINTER(KVView), P, P, P, P, P, P, P, SZ, P]
        L.dashkv_demote_pages.argtypes = [P, ctypes.POINTER(KVView), ctypes.POINTER(TierView), P, P, P]
        L.dashkv_sparse_decode_tiered.argtypes = [P, ctypes.POINTER(KVView), ctypes.POINTER(TierView), P, P, P, P,
                                                  P, P, P, SZ, P]
        L.dashkv_get_error.argtypes = [P]
        L.dashkv_hyperplanes.argtypes = [U64, I32, I32, P]
        L.dashkv_set_trace.argtypes = [P, P, I32]
        L.dashkv_select_kernels.argtypes = [P, ctypes.c_int64]
        L.dashkv_select_kernels.restype = I32
        L.dashkv_status_str.argtypes = [ctypes.c_int]
        L.dashkv_status_str.restype = ctypes.c_char_p
        for f in ("dashkv_encode_keys", "dashkv_append_keys", "dashkv_select", "dashkv_sparse_decode", "dashkv_decode_step",
                  "dashkv_get_error", "dashkv_hyperplanes", "dashkv_set_trace", "dashkv_select_static",
                  "dashkv_encode_blocks", "dashkv_append_blocks", "dashkv_select_blocks",
                  "dashkv_encode_radius", "dashkv_append_radius", "dashkv_select_radius", "dashkv_decode_step",
           "dashkv_demote_pages", "dashkv_sparse_decode_tiered"):
            getattr(L, f).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(call: str, status: int) -> None:
    if status != 0:
        raise DashKVError(call, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream: Optional[torch.cuda.Stream]):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def canonical_codes(codes: torch.Tensor, bits: int) -> torch.Tensor:
    """Undo the storage rotation of key codes (host or device tensor, int64).

    The library stores token t's code with its T = bits/8 bytes rotated by
    t mod T (stored byte p = code byte (p + t mod T) mod T); the token position
    is the second-to-last axis in both layouts (dense [B,Hkv,n_cap,W], paged
    [P,Hkv,page,W], page a multiple of 32).  Returns the codes with hyperplane j
    at word j/64, bit j%64."""
    T = bits // 8
    W = codes.shape[-1]
    n = codes.shape[-2]
    b = codes.contiguous().view(torch.uint8).reshape(*codes.shape[:-1], W * 8)
    rho = torch.arange(n, device=codes.device) % T
    src = (torch.arange(T, device=codes.device)[None, :] - rho[:, None]) % T  # original c <- stored (c - rho) mod T
    idx = src.expand(*b.shape[:-1], T)
    orig = torch.gather(b[..., :T], -1, idx)
    full = torch.zeros_like(b)
    full[..., :T] = orig
    return full.reshape(*codes.shape[:-1], W * 8).view(torch.int64).reshape(codes.shape)


def hyperplanes(seed: int, bits: int, d: int) -> torch.Tensor:
    """The +-1 hyperplanes [bits, d] (int8, host) a context with this seed uses."""
    out = torch.empty((bits, d), dtype=torch.int8)
    _check("dashkv_hyperplanes", lib().dashkv_hyperplanes(seed & (2**64 - 1), bits, d, _ptr(out)))
    return out


@dataclasses.dataclass
class KVCache:
    """Device tensors of one cache.  Dense: k, v [B,Hkv,n_cap,d] bf16, codes
    [B,Hkv,n_cap,W] int64.  Paged: k, v [P,page,Hkv,d], codes [P,Hkv,page,W],
    page_table [B,max_pages] int32."""
    k: torch.Tensor
    v: torch.Tensor
    codes: torch.Tensor
    page_table: Optional[torch.Tensor] = None

    @property
    def paged(self) -> bool:
        return self.page_table is not None

    @property
    def page_size(self) -> int:
        return int(self.k.shape[1]) if self.paged else 0

    @property
    def capacity(self) -> int:
        return int(self.page_table.shape[1]) * self.page_size if self.paged else int(self.k.shape[2])

    def view(self) -> KVView:
        if self.paged:
            return KVView(self.k.data_ptr(), self.v.data_ptr(), self.codes.data_ptr(), 0,
                          self.page_table.data_ptr(), int(self.page_table.shape[1]), int(self.k.shape[0]))
        return KVView(self.k.data_ptr(), self.v.data_ptr(), self.codes.data_ptr(), int(self.k.shape[2]),
                      None, 0, 0)

    @staticmethod
    def empty_radius_like(k: torch.Tensor, paged: bool) -> torch.Tensor:
        """Zeroed uint8 radius codes: dense [B,Hkv,n_cap], paged [P,Hkv,page]."""
        if paged:
            P, ps, Hkv, _ = k.shape
            return torch.zeros((P, Hkv, ps), dtype=torch.uint8, device=k.device)
        B, Hkv, n_cap, _ = k.shape
        return torch.zeros((B, Hkv, n_cap), dtype=torch.uint8, device=k.device)

    @staticmethod
    def empty_codes_like(k: torch.Tensor, bits: int, paged: bool) -> torch.Tensor:
        W = max(1, bits // 64)
        if paged:
            P, ps, Hkv, _ = k.shape
            return torch.zeros((P, Hkv, ps, W), dtype=torch.int64, device=k.device)
        B, Hkv, n_cap, _ = k.shape
        return torch.zeros((B, Hkv, n_cap, W), dtype=torch.int64, device=k.device)


@dataclasses.dataclass
class BlockIndex:
    """Summary codes of the complete blocks of `block` tokens of a cache:
    codes [B, Hkv, nb_cap, W] int64 on the device (block i at index i, stored
    like token codes; canonical_codes() undoes the rotation)."""
    codes: torch.Tensor
    block: int

    @property
    def capacity(self) -> int:
        return int(self.codes.shape[2])

    def view(self) -> BlockView:
        return BlockView(self.codes.data_ptr(), self.capacity, int(self.block), 0)

    @staticmethod
    def empty_for(cache: KVCache, batch: int, bits: int, block: int) -> "BlockIndex":
        """Zeroed codes for every complete block the cache can hold."""
        Hkv = int(cache.k.shape[2] if cache.paged else cache.k.shape[1])
        nb_cap = max(1, cache.capacity // int(block))
        W = max(1, bits // 64)
        return BlockIndex(torch.zeros((batch, Hkv, nb_cap, W), dtype=torch.int64, device=cache.k.device), int(block))


@dataclasses.dataclass
class PageTiers:
    """Precision tiers of a paged cache's pages: tier [P] uint8 (0 = bf16
    rows, 1 = FP8 rows), k8 / v8 [P, page, Hkv, d] uint8 (FP8 E4M3 codes) and
    exps [P, page, Hkv, 2] int8 (the rows' power-of-two scale exponents)."""
    tier: torch.Tensor
    k8: torch.Tensor
    v8: torch.Tensor
    exps: torch.Tensor

    def view(self) -> TierView:
        return TierView(self.tier.data_ptr(), self.k8.data_ptr(), self.v8.data_ptr(), self.exps.data_ptr())

    @staticmethod
    def empty_for(cache: "KVCache") -> "PageTiers":
        """Every page tier 0 (zeroed arrays shaped like the cache's pages)."""
        if not cache.paged:
            raise ValueError("precision tiers are defined on paged caches")
        P, page, Hkv, d = cache.k.shape
        dev = cache.k.device
        return PageTiers(torch.zeros(P, dtype=torch.uint8, device=dev),
                         torch.zeros((P, page, Hkv, d), dtype=torch.uint8, device=dev),
                         torch.zeros((P, page, Hkv, d), dtype=torch.uint8, device=dev),
                         torch.zeros((P, page, Hkv, 2), dtype=torch.int8, device=dev))


class DashKV:
    """One problem configuration (shapes, bits, k, S, W, layout, seed)."""

    def __init__(self, batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int, bits: int, topk: int,
                 sink: int, window: int, page_size: int = 0, seed: int = 0x5EEDDA5B,
                 two_kernel_select: bool = False):
        if not torch.cuda.is_available():
            raise RuntimeError("hash_indexed_top_b200 needs a CUDA device (B200, sm_100a)")
        flags = FLAG_TWO_KERNEL_SELECT if two_kernel_select else 0
        self.cfg = Config(batch, num_q_heads, num_kv_heads, head_dim, bits, topk, sink, window, page_size, flags,
                          seed & (2**64 - 1))
        self.sel_cap = topk + sink + window
        h = ctypes.c_void_p()
        _check("dashkv_create", lib().dashkv_create(ctypes.byref(self.cfg), ctypes.byref(h)))
        self._ctx = h
        self._ws = None

    def close(self) -> None:
        if self._ctx:
            lib().dashkv_destroy(self._ctx)
            self._ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ---- workspace
    def workspace_size(self, max_tokens: int) -> int:
        return int(lib().dashkv_workspace_size(self._ctx, int(max_tokens)))

    def workspace(self, max_tokens: int, device=None) -> torch.Tensor:
        """A zero-filled workspace (kept and reused while it is large enough)."""
        need = self.workspace_size(max_tokens)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.zeros(need, dtype=torch.uint8, device=device or torch.cuda.current_device())
        return self._ws

    # ---- the four calls
    def encode_keys(self, cache: KVCache, seq_lens: torch.Tensor, stream=None) -> None:
        v = cache.view()
        _check("dashkv_encode_keys", lib().dashkv_encode_keys(self._ctx, ctypes.byref(v), _ptr(seq_lens),
                                                              _stream(stream)))

    def append_keys(self, cache: KVCache, k_new: torch.Tensor, v_new: torch.Tensor, seq_lens: torch.Tensor,
                    stream=None) -> None:
        v = cache.view()
        _check("dashkv_append_keys", lib().dashkv_append_keys(self._ctx, ctypes.byref(v), _ptr(k_new),
                                                              _ptr(v_new), _ptr(seq_lens), _stream(stream)))

    def select(self, cache: KVCache, q: torch.Tensor, seq_lens: torch.Tensor, sel_idx: torch.Tensor,
               sel_cnt: torch.Tensor, scores: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               stream=None) -> None:
        ws = workspace if workspace is not None else self.workspace(cache.capacity, q.device)
        v = cache.view()
        _check("dashkv_select", lib().dashkv_select(self._ctx, ctypes.byref(v), _ptr(q), _ptr(seq_lens),
                                                    _ptr(sel_idx), _ptr(sel_cnt), _ptr(scores), _ptr(ws),
                                                    ws.numel(), _stream(stream)))

    def select_static(self, cache: KVCache, q: torch.Tensor, seq_lens: torch.Tensor, sel_idx: torch.Tensor,
                      sel_cnt: torch.Tensor, scores: Optional[torch.Tensor] = None, stream=None) -> None:
        """dashkv_select on the library's fixed 24 MiB device scratch: for callers
        that may not allocate device memory (e.g. inside CUDA graph capture,
        where cudaMalloc is not allowed).  The first call on a device must not be
        captured; overlapping calls on one device race (one shared scratch)."""
        v = cache.view()
        _check("dashkv_select_static", lib().dashkv_select_static(self._ctx, ctypes.byref(v), _ptr(q),
                                                                  _ptr(seq_lens), _ptr(sel_idx), _ptr(sel_cnt),
                                                                  _ptr(scores), _stream(stream)))

    def sparse_decode(self, cache: KVCache, q: torch.Tensor, sel_idx: torch.Tensor, sel_cnt: torch.Tensor,
                      out: torch.Tensor, lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                      stream=None, seq_lens: Optional[torch.Tensor] = None) -> None:
        """seq_lens (optional): the lengths sel_idx was selected for; given, the
        sinks and the window are attended from the token range by CTAs that do
        not wait for the selection."""
        ws = workspace if workspace is not None else self.workspace(cache.capacity, q.device)
        v = cache.view()
        _check("dashkv_sparse_decode", lib().dashkv_sparse_decode(self._ctx, ctypes.byref(v), _ptr(q),
                                                                  _ptr(seq_lens), _ptr(sel_idx), _ptr(sel_cnt),
                                                                  _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                                                  _stream(stream)))

    def demote_pages(self, cache: KVCache, tiers: PageTiers, seq_lens: torch.Tensor,
                     protect: Optional[torch.Tensor] = None, stream=None) -> None:
        """Move every page that holds no sink and no window token (and is not
        protected) to the FP8 tier."""
        v, t = cache.view(), tiers.view()
        _check("dashkv_demote_pages", lib().dashkv_demote_pages(self._ctx, ctypes.byref(v), ctypes.byref(t),
                                                                _ptr(seq_lens), _ptr(protect), _stream(stream)))

    def sparse_decode_tiered(self, cache: KVCache, tiers: PageTiers, q: torch.Tensor, sel_idx: torch.Tensor,
                             sel_cnt: torch.Tensor, out: torch.Tensor, lse: Optional[torch.Tensor] = None,
                             workspace: Optional[torch.Tensor] = None, stream=None,
                             seq_lens: Optional[torch.Tensor] = None) -> None:
        """sparse_decode with the rows of FP8-tier pages read from `tiers`."""
        ws = workspace if workspace is not None else self.workspace(cache.capacity, q.device)
        v, t = cache.view(), tiers.view()
        _check("dashkv_sparse_decode_tiered",
               lib().dashkv_sparse_decode_tiered(self._ctx, ctypes.byref(v), ctypes.byref(t), _ptr(q),
                                                 _ptr(seq_lens), _ptr(sel_idx), _ptr(sel_cnt), _ptr(out), _ptr(lse),
                                                 _ptr(ws), ws.numel(), _stream(stream)))

    def decode_step(self, cache: KVCache, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                    seq_lens: torch.Tensor, sel_idx: torch.Tensor, sel_cnt: torch.Tensor, out: torch.Tensor,
                    lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                    stream=None) -> None:
        """append_keys + select + sparse_decode (given the lengths) in one launch."""
        ws = workspace if workspace is not None else self.workspace(cache.capacity, q.device)
        v = cache.view()
        _check("dashkv_decode_step", lib().dashkv_decode_step(self._ctx, ctypes.byref(v), _ptr(q), _ptr(k_new),
                                                              _ptr(v_new), _ptr(seq_lens), _ptr(sel_idx),
                                                              _ptr(sel_cnt), _ptr(out), _ptr(lse), _ptr(ws),
                                                              ws.numel(), _stream(stream)))

    # ---- block summaries (CSA-style two-level index)
    def encode_blocks(self, cache: KVCache, index: BlockIndex, seq_lens: torch.Tensor, stream=None) -> None:
        v, bv = cache.view(), index.view()
        _check("dashkv_encode_blocks", lib().dashkv_encode_blocks(self._ctx, ctypes.byref(v), ctypes.byref(bv),
                                                                  _ptr(seq_lens), _stream(stream)))

    def append_blocks(self, cache: KVCache, index: BlockIndex, seq_lens: torch.Tensor, stream=None) -> None:
        """After append_keys: encode the block the append completed, if any."""
        v, bv = cache.view(), index.view()
        _check("dashkv_append_blocks", lib().dashkv_append_blocks(self._ctx, ctypes.byref(v), ctypes.byref(bv),
                                                                  _ptr(seq_lens), _stream(stream)))

    def select_blocks(self, cache: KVCache, index: BlockIndex, q: torch.Tensor, seq_lens: torch.Tensor,
                      sel_idx: torch.Tensor, sel_cnt: torch.Tensor, block_scores: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> None:
        """Top topk // block blocks by summary score, as a token list in select()'s format."""
        ws = workspace if workspace is not None else self.workspace(cache.capacity, q.device)
        v, bv = cache.view(), index.view()
        _check("dashkv_select_blocks", lib().dashkv_select_blocks(self._ctx, ctypes.byref(v), ctypes.byref(bv),
                                                                  _ptr(q), _ptr(seq_lens), _ptr(sel_idx),
                                                                  _ptr(sel_cnt), _ptr(block_scores), _ptr(ws),
                                                                  ws.numel(), _stream(stream)))

    # ---- radius-scaled scores (8-bit key-norm codes)
    def encode_radius(self, cache: KVCache, radius: torch.Tensor, seq_lens: torch.Tensor, stream=None) -> None:
        v = cache.view()
        _check("dashkv_encode_radius", lib().dashkv_encode_radius(self._ctx, ctypes.byref(v), _ptr(seq_lens),
                                                                  _ptr(radius), _stream(stream)))

    def append_radius(self, cache: KVCache, radius: torch.Tensor, seq_lens: torch.Tensor, stream=None) -> None:
        """After append_keys: the radius code of each sequence's newest token."""
        v = cache.view()
        _check("dashkv_append_radius", lib().dashkv_append_radius(self._ctx, ctypes.byref(v), _ptr(seq_lens),
                                                                  _ptr(radius), _stream(stream)))

    def select_radius(self, cache: KVCache, radius: torch.Tensor, q: torch.Tensor, seq_lens: torch.Tensor,
                      sel_idx: torch.Tensor, sel_cnt: torch.Tensor, scores: Optional[torch.Tensor] = None,
                      workspace: Optional[torch.Tensor] = None, stream=None) -> None:
        """select() on the radius-scaled scores r~ s."""
        ws = workspace if workspace is not None else self.workspace(cache.capacity, q.device)
        v = cache.view()
        _check("dashkv_select_radius", lib().dashkv_select_radius(self._ctx, ctypes.byref(v), _ptr(radius), _ptr(q),
                                                                  _ptr(seq_lens), _ptr(sel_idx), _ptr(sel_cnt),
                                                                  _ptr(scores), _ptr(ws), ws.numel(),
                                                                  _stream(stream)))

    def select_kernels(self, max_tokens: int) -> int:
        """1 when dashkv_select runs the fused kernel for this cache size, 2 for score + collect."""
        return int(lib().dashkv_select_kernels(self._ctx, int(max_tokens)))

    def set_trace(self, events: Optional[list] = None) -> None:
        """Record torch.cuda.Event pairs around each kernel of the following calls (None: off)."""
        if events is None:
            self._trace = None
            _check("dashkv_set_trace", lib().dashkv_set_trace(self._ctx, None, 0))
            return
        handles = [e.cuda_event for e in events]
        if not all(handles):
            raise ValueError("set_trace: record each event once first (torch creates CUDA events lazily)")
        arr = (ctypes.c_void_p * len(events))(*handles)
        self._trace = arr  # keep alive while tracing
        _check("dashkv_set_trace", lib().dashkv_set_trace(self._ctx, arr, len(events)))

    def get_error(self, stream=None) -> int:
        """Synchronise the stream; return (and clear) the device error status."""
        return int(lib().dashkv_get_error(_stream(stream)))

    # ---- convenience: output buffers for one step
    def alloc_step(self, device) -> dict:
        B, Hq, Hkv, d = self.cfg.batch, self.cfg.num_q_heads, self.cfg.num_kv_heads, self.cfg.head_dim
        return dict(sel_idx=torch.empty((B, Hkv, self.sel_cap), dtype=torch.int32, device=device),
                    sel_cnt=torch.empty((B, Hkv), dtype=torch.int32, device=device),
                    out=torch.empty((B, Hq, d), dtype=torch.float32, device=device),
                    lse=torch.empty((B, Hq), dtype=torch.float32, device=device))
