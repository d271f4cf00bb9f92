"""Python binding of libqsa.so: argument marshalling only.

Every step of QSA runs in the library's CUDA kernels.  This module checks shapes and
dtypes of torch tensors, allocates output and workspace buffers with torch (the library
itself never allocates), passes raw device pointers and the current CUDA stream through
ctypes, and turns status codes into exceptions.  There is no CPU path: tensors must live
on a CUDA device and the library must load, or the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

import torch

from . import build as _build

NUM_HEADS, NUM_KV_HEADS, HEAD_DIM = 24, 2, 128
IDX_HEADS, IDX_DIM, BLOCK = 16, 64, 4
WS_HEADER_BYTES = 256

STATUS = {0: "QSA_OK", 1: "QSA_ERR_INVALID_ARG", 2: "QSA_ERR_ALIGNMENT", 3: "QSA_ERR_CAPACITY",
          4: "QSA_ERR_WORKSPACE", 5: "QSA_ERR_CUDA", 6: "QSA_ERR_TIMEOUT", 7: "QSA_ERR_DEVICE",
          8: "QSA_ERR_UNSUPPORTED"}

# Names exported by include/qsa.h (checked by the tests).
EXPORTS = ("qsa_status_string", "qsa_version", "qsa_launch_count", "qsa_workspace_init", "qsa_last_device_error",
           "qsa_compress_workspace_size", "qsa_compress", "qsa_index_scores", "qsa_topk",
           "qsa_prefill_workspace_size", "qsa_prefill", "qsa_prefill_select",
           "qsa_sparse_attention", "qsa_append_kv", "qsa_decode_workspace_size", "qsa_decode",
           "qsa_decode_noalloc", "qsa_noalloc_last_device_error", "qsa_append_kv_paged",
           "qsa_decode_paged_workspace_size", "qsa_decode_paged",
           "qsa_decode_shard_workspace_size", "qsa_decode_shard_select", "qsa_merge_candidates",
           "qsa_decode_shard_attend", "qsa_combine_partials", "qsa_gated_deltanet")


class QSAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)}")
        self.code = code


class Params(ctypes.Structure):
    _fields_ = [("topk_blocks", ctypes.c_int32), ("rows_per_tile", ctypes.c_int32),
                ("decode_splits", ctypes.c_int32), ("score_chunk_rows", ctypes.c_int32),
                ("debug_fault", ctypes.c_int32), ("select_mode", ctypes.c_int32)]


class CacheDesc(ctypes.Structure):
    _fields_ = [("k_blocks", ctypes.c_void_p), ("v_blocks", ctypes.c_void_p),
                ("kbar", ctypes.c_void_p), ("kbar_partial", ctypes.c_void_p),
                ("len", ctypes.c_void_p), ("batch", ctypes.c_int32), ("capacity", ctypes.c_int32)]


class PagedCacheDesc(ctypes.Structure):
    _fields_ = [("base", CacheDesc), ("page_table", ctypes.c_void_p),
                ("page_tokens", ctypes.c_int32), ("pool_pages", ctypes.c_int32)]


_lock = threading.Lock()
_lib = None


def load(build_if_needed: bool = True):
    """Load libqsa.so (building it in-tree with nvcc first if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = _build.LIB
        if build_if_needed and _build.is_stale():
            path = _build.build()
        if not os.path.exists(path):
            raise RuntimeError(f"libqsa.so not found at {path}; run block_sparse_attention_40_b200.build")
        lib = ctypes.CDLL(path)
        P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        st = ctypes.c_int
        sig = {
            "qsa_status_string": ([st], ctypes.c_char_p),
            "qsa_version": ([], I32),
            "qsa_launch_count": ([], ctypes.c_uint64),
            "qsa_workspace_init": ([P, SZ, P], st),
            "qsa_last_device_error": ([P, P, P], st),
            "qsa_compress_workspace_size": ([I32], SZ),
            "qsa_compress": ([P, P, P, I32, P, P, SZ, P], st),
            "qsa_index_scores": ([P, P, P, P, P, I32, I64, I64, P, I64, I32, P, SZ, P], st),
            "qsa_topk": ([P, I64, P, I64, I32, I32, P, P, P], st),
            "qsa_prefill_workspace_size": ([P, I32, Params], SZ),
            "qsa_prefill": ([P, P, P, P, P, P, P, P, I32, P, P, SZ, Params, P], st),
            "qsa_prefill_select": ([P, P, P, P, P, I32, P, P, P, SZ, Params, P], st),
            "qsa_sparse_attention": ([P, P, P, P, P, P, P, I32, P, P, SZ, Params, P], st),
            "qsa_append_kv": ([P, P, P, P, I32, P, P, P], st),
            "qsa_decode_workspace_size": ([P, Params], SZ),
            "qsa_decode": ([P, P, P, P, P, P, P, P, P, SZ, Params, P], st),
            "qsa_decode_noalloc": ([P, P, P, P, P, P, P, P, Params, P], st),
            "qsa_noalloc_last_device_error": ([P, P], st),
            "qsa_append_kv_paged": ([P, P, P, P, I32, P, P, P], st),
            "qsa_decode_paged_workspace_size": ([P, Params], SZ),
            "qsa_decode_paged": ([P, P, P, P, P, P, P, P, P, SZ, Params, P], st),
            "qsa_decode_shard_workspace_size": ([P, Params], SZ),
            "qsa_decode_shard_select": ([P, P, P, I32, P, P, P, P, P, P, SZ, Params, P], st),
            "qsa_merge_candidates": ([P, P, P, I32, I32, I32, I32, P, P, P, SZ, P], st),
            "qsa_decode_shard_attend": ([P, P, I32, P, P, P, P, P, P, P, SZ, Params, P], st),
            "qsa_combine_partials": ([P, P, P, I32, I32, P, P], st),
            "qsa_gated_deltanet": ([P, P, P, P, P, P, P, I32, I32, P, P, P], st),
        }
        for name, (args, res) in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
    return _lib


def library_path() -> str:
    return _build.LIB


def _check(fn: str, code: int):
    if code != 0:
        raise QSAError(fn, code)


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t: torch.Tensor, name: str, dtype, shape_tail=None, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the library has no CPU path)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if shape_tail is not None and tuple(t.shape[-len(shape_tail):]) != tuple(shape_tail):
        raise ValueError(f"{name} must end in {shape_tail}, got {tuple(t.shape)}")


def _cu_pair(cu_seqlens, device):
    """(host int32 tensor, device int32 tensor) for the cumulative sequence lengths."""
    if isinstance(cu_seqlens, torch.Tensor) and cu_seqlens.is_cuda:
        h = cu_seqlens.to(torch.int32).cpu().contiguous()
        d = cu_seqlens.to(torch.int32).contiguous()
    else:
        h = torch.as_tensor(cu_seqlens, dtype=torch.int32).contiguous()
        d = h.to(device)
    return h, d


def _params(topk, rows_per_tile=0, decode_splits=0, score_chunk_rows=0, debug_fault=0,
            select_mode=0) -> Params:
    return Params(int(topk), int(rows_per_tile), int(decode_splits), int(score_chunk_rows),
                  int(debug_fault), int(select_mode))


def new_workspace(nbytes: int, device) -> torch.Tensor:
    ws = torch.empty(max(int(nbytes), WS_HEADER_BYTES), dtype=torch.uint8, device=device)
    _check("qsa_workspace_init", load().qsa_workspace_init(_ptr(ws), ws.numel(), _stream(device)))
    return ws


def last_device_error(workspace: torch.Tensor) -> tuple:
    """(status name, site) of the first device-side failure recorded in the workspace."""
    site = ctypes.c_uint32(0)
    code = load().qsa_last_device_error(_ptr(workspace), _stream(workspace.device),
                                        ctypes.byref(site))
    return STATUS.get(code, str(code)), int(site.value)


def status_string(code: int) -> str:
    return load().qsa_status_string(code).decode()


def version() -> int:
    return int(load().qsa_version())


def launch_count() -> int:
    """Kernels launched by libqsa.so so far in this process."""
    return int(load().qsa_launch_count())


# --------------------------------------------------------------------------------------
def prefill_workspace_size(cu_seqlens_host, topk=512, rows_per_tile=0, score_chunk_rows=0,
                           select_mode=0) -> int:
    h = torch.as_tensor(cu_seqlens_host, dtype=torch.int32).contiguous()
    n = load().qsa_prefill_workspace_size(ctypes.c_void_p(h.data_ptr()),
                                          h.numel() - 1,
                                          _params(topk, rows_per_tile, 0, score_chunk_rows,
                                                  0, select_mode))
    if n == 0:
        raise QSAError("qsa_prefill_workspace_size", 1)
    return int(n)


def _prefill_inputs(q, k, v, q_idx, k_idx, w, T):
    if q is not None:
        _need(q, "q", torch.bfloat16, (NUM_HEADS, HEAD_DIM), 3)
        _need(k, "k", torch.bfloat16, (NUM_KV_HEADS, HEAD_DIM), 3)
        _need(v, "v", torch.bfloat16, (NUM_KV_HEADS, HEAD_DIM), 3)
        for n_, t in (("q", q), ("k", k), ("v", v)):
            if t.shape[0] != T:
                raise ValueError(f"{n_} has {t.shape[0]} tokens, cu_seqlens says {T}")
    if q_idx is not None:
        _need(q_idx, "q_idx", torch.bfloat16, (IDX_HEADS, IDX_DIM), 3)
        _need(w, "w", torch.bfloat16, (IDX_HEADS,), 2)
        for n_, t in (("q_idx", q_idx), ("w", w)):
            if t.shape[0] != T:
                raise ValueError(f"{n_} has {t.shape[0]} tokens, cu_seqlens says {T}")
    if k_idx is not None:
        _need(k_idx, "k_idx", torch.bfloat16, (IDX_DIM,), 2)
        if k_idx.shape[0] != T:
            raise ValueError(f"k_idx has {k_idx.shape[0]} tokens, cu_seqlens says {T}")


def compress(k_idx: torch.Tensor, cu_seqlens) -> torch.Tensor:
    """Step a1: packed compressed indexer keys [sum floor(L/4), 64] bf16."""
    dev = k_idx.device
    h, d = _cu_pair(cu_seqlens, dev)
    T = int(h[-1])
    _prefill_inputs(None, None, None, None, k_idx, None, T)
    nb = int(((h[1:] - h[:-1]) // BLOCK).sum())
    kbar = torch.empty((max(nb, 1), IDX_DIM), dtype=torch.bfloat16, device=dev)
    lib = load()
    ws = new_workspace(lib.qsa_compress_workspace_size(h.numel() - 1), dev)
    _check("qsa_compress", lib.qsa_compress(_ptr(k_idx), _ptr(d), ctypes.c_void_p(h.data_ptr()),
                                            h.numel() - 1, _ptr(kbar), _ptr(ws), ws.numel(),
                                            _stream(dev)))
    return kbar[:nb]


def index_scores(q_idx, w, kbar, cu_seqlens, row_begin=None, row_end=None, topk=0,
                 scores=None, ld=None):
    """Step a2: fp32 scores [row_end-row_begin, ld] (entries b >= floor(pos/4) untouched)."""
    dev = q_idx.device
    h, d = _cu_pair(cu_seqlens, dev)
    T = int(h[-1])
    _prefill_inputs(None, None, None, q_idx, None, w, T)
    _need(kbar, "kbar", torch.bfloat16, (IDX_DIM,), 2)
    row_begin = 0 if row_begin is None else int(row_begin)
    row_end = T if row_end is None else int(row_end)
    max_nc = int(((h[1:] - h[:-1]).max() - 1) // BLOCK)
    if ld is None:
        ld = max(4, (max(max_nc, 1) + 3) // 4 * 4)
    if scores is None:
        scores = torch.full((row_end - row_begin, ld), float("nan"), dtype=torch.float32, device=dev)
    _need(scores, "scores", torch.float32)
    lib = load()
    ws = new_workspace(prefill_workspace_size(h, topk if topk > 0 else 512, 1), dev)
    _check("qsa_index_scores",
           lib.qsa_index_scores(_ptr(q_idx), _ptr(w), _ptr(kbar), _ptr(d),
                                ctypes.c_void_p(h.data_ptr()), h.numel() - 1, row_begin, row_end,
                                _ptr(scores), int(ld), int(topk), _ptr(ws), ws.numel(),
                                _stream(dev)))
    return scores


def topk(scores: torch.Tensor, n_c: torch.Tensor, k: int, max_n_c: Optional[int] = None):
    """Step a3 on explicit score rows: (idx [rows, k] int32 ascending -1 padded, cnt [rows])."""
    _need(scores, "scores", torch.float32, ndim=2)
    _need(n_c, "n_c", torch.int32, ndim=1)
    rows, ld = scores.shape
    if max_n_c is None:
        max_n_c = int(n_c.max().item()) if rows else 0
    idx = torch.empty((rows, k), dtype=torch.int32, device=scores.device)
    cnt = torch.empty((rows,), dtype=torch.int32, device=scores.device)
    _check("qsa_topk", load().qsa_topk(_ptr(scores), ld, _ptr(n_c), rows, int(k), int(max_n_c),
                                       _ptr(idx), _ptr(cnt), _stream(scores.device)))
    return idx, cnt


class Prefill:
    """Reusable prefill context: holds the device cu_seqlens and the workspace."""

    def __init__(self, cu_seqlens, device, topk=512, rows_per_tile=0, score_chunk_rows=0,
                 debug_fault=0, select_mode=0):
        self.device = torch.device(device)
        self.h_cu, self.d_cu = _cu_pair(cu_seqlens, self.device)
        self.num_seqs = self.h_cu.numel() - 1
        self.T = int(self.h_cu[-1])
        self.params = _params(topk, rows_per_tile, 0, score_chunk_rows, debug_fault, select_mode)
        self.topk = int(topk)
        self.ws = new_workspace(prefill_workspace_size(self.h_cu, topk, rows_per_tile,
                                                       score_chunk_rows, select_mode),
                                self.device)
        self.lib = load()

    def run(self, q, k, v, q_idx, k_idx, w, out=None):
        _prefill_inputs(q, k, v, q_idx, k_idx, w, self.T)
        if out is None:
            out = torch.empty_like(q)
        _need(out, "out", torch.bfloat16, (NUM_HEADS, HEAD_DIM), 3)
        _check("qsa_prefill", self.lib.qsa_prefill(
            _ptr(q), _ptr(k), _ptr(v), _ptr(q_idx), _ptr(k_idx), _ptr(w), _ptr(self.d_cu),
            ctypes.c_void_p(self.h_cu.data_ptr()), self.num_seqs, _ptr(out), _ptr(self.ws),
            self.ws.numel(), self.params, _stream(self.device)))
        return out

    def select(self, q_idx, k_idx, w, idx=None, cnt=None):
        _prefill_inputs(None, None, None, q_idx, k_idx, w, self.T)
        if idx is None:
            idx = torch.empty((self.T, self.topk), dtype=torch.int32, device=self.device)
            cnt = torch.empty((self.T,), dtype=torch.int32, device=self.device)
        _check("qsa_prefill_select", self.lib.qsa_prefill_select(
            _ptr(q_idx), _ptr(k_idx), _ptr(w), _ptr(self.d_cu),
            ctypes.c_void_p(self.h_cu.data_ptr()), self.num_seqs, _ptr(idx), _ptr(cnt),
            _ptr(self.ws), self.ws.numel(), self.params, _stream(self.device)))
        return idx, cnt

    def attend(self, q, k, v, idx, cnt, out=None):
        _prefill_inputs(q, k, v, None, None, None, self.T)
        _need(idx, "idx", torch.int32, (self.topk,), 2)
        _need(cnt, "cnt", torch.int32, ndim=1)
        if out is None:
            out = torch.empty_like(q)
        _check("qsa_sparse_attention", self.lib.qsa_sparse_attention(
            _ptr(q), _ptr(k), _ptr(v), _ptr(idx), _ptr(cnt), _ptr(self.d_cu),
            ctypes.c_void_p(self.h_cu.data_ptr()), self.num_seqs, _ptr(out), _ptr(self.ws),
            self.ws.numel(), self.params, _stream(self.device)))
        return out

    def device_error(self):
        return last_device_error(self.ws)


def prefill(q, k, v, q_idx, k_idx, w, cu_seqlens, topk=512, rows_per_tile=0, score_chunk_rows=0):
    """QSA prefill (steps a1-a4) over a packed varlen batch; returns out [T, 24, 128] bf16."""
    ctx = Prefill(cu_seqlens, q.device, topk, rows_per_tile, score_chunk_rows)
    return ctx.run(q, k, v, q_idx, k_idx, w)


def prefill_select(q_idx, k_idx, w, cu_seqlens, topk=512):
    ctx = Prefill(cu_seqlens, q_idx.device, topk)
    return ctx.select(q_idx, k_idx, w)


# --------------------------------------------------------------------------------------
class KVCache:
    """Caller-owned decode cache (torch-allocated buffers, blocked layout of include/qsa.h)."""

    _append_fn = "qsa_append_kv"
    _ws_fn = "qsa_decode_workspace_size"
    _decode_fn = "qsa_decode"

    def __init__(self, batch: int, capacity: int, device, zero=True):
        if capacity % BLOCK:
            raise ValueError("capacity must be a multiple of 4")
        alloc = torch.zeros if zero else torch.empty
        self.batch, self.capacity, self.device = int(batch), int(capacity), torch.device(device)
        nb = capacity // BLOCK
        self.k_blocks = alloc((batch, NUM_KV_HEADS, nb, BLOCK, HEAD_DIM), dtype=torch.bfloat16,
                              device=device)
        self.v_blocks = alloc((batch, NUM_KV_HEADS, nb, BLOCK, HEAD_DIM), dtype=torch.bfloat16,
                              device=device)
        self.kbar = alloc((batch, nb, IDX_DIM), dtype=torch.bfloat16, device=device)
        self.kbar_partial = torch.zeros((batch, IDX_DIM), dtype=torch.float32, device=device)
        self.len = torch.zeros((batch,), dtype=torch.int32, device=device)
        self.h_len = [0] * batch          # host mirror of len

    def desc(self) -> CacheDesc:
        return CacheDesc(self.k_blocks.data_ptr(), self.v_blocks.data_ptr(), self.kbar.data_ptr(),
                         self.kbar_partial.data_ptr(), self.len.data_ptr(), self.batch,
                         self.capacity)

    def kbar_rows(self, b: int, n: int) -> torch.Tensor:
        """Compressed keys of blocks 0 .. n-1 of sequence b, [n, 64] (a view or a gather)."""
        return self.kbar[b, :n]

    def kv_rows(self, b: int, g: int, n: int):
        """K and V rows of tokens 0 .. n-1 of sequence b, KV head g: two [n, 128] tensors."""
        return (self.k_blocks[b, g].reshape(-1, HEAD_DIM)[:n],
                self.v_blocks[b, g].reshape(-1, HEAD_DIM)[:n])

    def append(self, k, v, k_idx, counts: Optional[Sequence[int]] = None):
        """Append k, v [B, n, 2, 128] and k_idx [B, n, 64] (counts[b] <= n tokens each)."""
        _need(k, "k", torch.bfloat16, (NUM_KV_HEADS, HEAD_DIM), 4)
        _need(v, "v", torch.bfloat16, (NUM_KV_HEADS, HEAD_DIM), 4)
        _need(k_idx, "k_idx", torch.bfloat16, (IDX_DIM,), 3)
        n = k.shape[1]
        if k.shape[0] != self.batch or v.shape[:2] != k.shape[:2] or k_idx.shape[:2] != k.shape[:2]:
            raise ValueError("append shapes disagree with the cache batch")
        d_counts = None
        if counts is not None:
            counts = [int(c) for c in counts]
            d_counts = torch.tensor(counts, dtype=torch.int32, device=self.device)
        h_len = (ctypes.c_int32 * self.batch)(*self.h_len)
        desc = self.desc()
        name = self._append_fn
        _check(name, getattr(load(), name)(
            ctypes.byref(desc), _ptr(k), _ptr(v), _ptr(k_idx), int(n), _ptr(d_counts), h_len,
            _stream(self.device)))
        for b in range(self.batch):
            self.h_len[b] += n if counts is None else max(0, min(counts[b], n))
        self._keep = d_counts   # keep the counts alive until the copy is enqueued
        return self


class PagedKVCache(KVCache):
    """Caller-owned paged decode cache: sequence b's logical page j (tokens j*page_tokens ..)
    lives in pool page page_table[b, j] (layout of qsa_paged_cache in include/qsa.h)."""

    _append_fn = "qsa_append_kv_paged"
    _ws_fn = "qsa_decode_paged_workspace_size"
    _decode_fn = "qsa_decode_paged"

    def __init__(self, batch: int, capacity: int, page_tokens: int, pool_pages: int,
                 page_table: torch.Tensor, device, zero=True):
        if page_tokens % 512 or capacity % page_tokens:
            raise ValueError("page_tokens must be a multiple of 512 dividing the capacity")
        if (page_table.dtype != torch.int32 or page_table.device != torch.device(device)
                or tuple(page_table.shape) != (batch, capacity // page_tokens)):
            raise ValueError("page_table must be int32 [batch, capacity // page_tokens] on the "
                             "cache's device")
        alloc = torch.zeros if zero else torch.empty
        self.batch, self.capacity, self.device = int(batch), int(capacity), torch.device(device)
        self.page_tokens, self.pool_pages = int(page_tokens), int(pool_pages)
        self.page_table = page_table.contiguous()
        nb = page_tokens // BLOCK
        self.k_blocks = alloc((pool_pages, NUM_KV_HEADS, nb, BLOCK, HEAD_DIM),
                              dtype=torch.bfloat16, device=device)
        self.v_blocks = alloc((pool_pages, NUM_KV_HEADS, nb, BLOCK, HEAD_DIM),
                              dtype=torch.bfloat16, device=device)
        self.kbar = alloc((pool_pages, nb, IDX_DIM), dtype=torch.bfloat16, device=device)
        self.kbar_partial = torch.zeros((batch, IDX_DIM), dtype=torch.float32, device=device)
        self.len = torch.zeros((batch,), dtype=torch.int32, device=device)
        self.h_len = [0] * batch

    def desc(self) -> PagedCacheDesc:
        base = CacheDesc(self.k_blocks.data_ptr(), self.v_blocks.data_ptr(), self.kbar.data_ptr(),
                         self.kbar_partial.data_ptr(), self.len.data_ptr(), self.batch,
                         self.capacity)
        return PagedCacheDesc(base, self.page_table.data_ptr(), self.page_tokens,
                              self.pool_pages)

    def _pages(self, b: int, n_tokens: int):
        return self.page_table[b, :(n_tokens + self.page_tokens - 1) // self.page_tokens].long()

    def kbar_rows(self, b: int, n: int) -> torch.Tensor:
        return self.kbar[self._pages(b, 4 * n)].reshape(-1, IDX_DIM)[:n]

    def kv_rows(self, b: int, g: int, n: int):
        pages = self._pages(b, n)
        return (self.k_blocks[pages, g].reshape(-1, HEAD_DIM)[:n],
                self.v_blocks[pages, g].reshape(-1, HEAD_DIM)[:n])


class Decoder:
    """Reusable decode context for one cache (contiguous or paged): holds the workspace."""

    def __init__(self, cache: KVCache, topk=512, decode_splits=0):
        self.cache = cache
        self.params = _params(topk, 0, decode_splits, 0)
        self.topk = int(topk)
        self.lib = load()
        desc = cache.desc()
        n = getattr(self.lib, cache._ws_fn)(ctypes.byref(desc), self.params)
        if n == 0:
            raise QSAError(cache._ws_fn, 1)
        self.ws = new_workspace(n, cache.device)

    def run(self, q, q_idx, w, out=None, with_selection=False):
        B = self.cache.batch
        _need(q, "q", torch.bfloat16, (NUM_HEADS, HEAD_DIM), 3)
        _need(q_idx, "q_idx", torch.bfloat16, (IDX_HEADS, IDX_DIM), 3)
        _need(w, "w", torch.bfloat16, (IDX_HEADS,), 2)
        if q.shape[0] != B or q_idx.shape[0] != B or w.shape[0] != B:
            raise ValueError("decode inputs must have the cache batch size")
        if out is None:
            out = torch.empty_like(q)
        idx = cnt = None
        if with_selection:
            idx = torch.empty((B, self.topk), dtype=torch.int32, device=q.device)
            cnt = torch.empty((B,), dtype=torch.int32, device=q.device)
        h_len = (ctypes.c_int32 * B)(*self.cache.h_len)
        desc = self.cache.desc()
        name = self.cache._decode_fn
        _check(name, getattr(self.lib, name)(
            _ptr(q), ctypes.byref(desc), _ptr(q_idx), _ptr(w), _ptr(out), h_len, _ptr(idx),
            _ptr(cnt), _ptr(self.ws), self.ws.numel(), self.params, _stream(q.device)))
        return (out, idx, cnt) if with_selection else out

    def device_error(self):
        return last_device_error(self.ws)


def decode_noalloc(cache: KVCache, q, q_idx, w, topk=512, decode_splits=0, out=None):
    """Decode through qsa_decode_noalloc: no workspace is passed; the library uses its own
    fixed device scratch.  Calls must not overlap on the GPU (they share that scratch)."""
    if isinstance(cache, PagedKVCache):
        raise TypeError("qsa_decode_noalloc takes a contiguous cache")
    B = cache.batch
    _need(q, "q", torch.bfloat16, (NUM_HEADS, HEAD_DIM), 3)
    _need(q_idx, "q_idx", torch.bfloat16, (IDX_HEADS, IDX_DIM), 3)
    _need(w, "w", torch.bfloat16, (IDX_HEADS,), 2)
    if out is None:
        out = torch.empty_like(q)
    h_len = (ctypes.c_int32 * B)(*cache.h_len)
    desc = cache.desc()
    _check("qsa_decode_noalloc", load().qsa_decode_noalloc(
        _ptr(q), ctypes.byref(desc), _ptr(q_idx), _ptr(w), _ptr(out), h_len, None, None,
        _params(topk, 0, decode_splits, 0), _stream(q.device)))
    return out


def noalloc_device_error(device) -> tuple:
    """(status name, site) of the last decode_noalloc call, read from the library's own
    scratch (synchronises the current stream of `device`)."""
    site = ctypes.c_uint32(0)
    code = load().qsa_noalloc_last_device_error(_stream(torch.device(device)), ctypes.byref(site))
    return STATUS.get(code, str(code)), int(site.value)


# --------------------------------------------------------------------------------------
class ShardDecoder:
    """Decode over one shard of a context split across caches (see include/qsa.h, context-
    sharded decode): the shard holds tokens [4 * block0, 4 * block0 + capacity) of every
    sequence of the batch, block0 a multiple of 128."""

    def __init__(self, cache: KVCache, block0: int, topk=512):
        if isinstance(cache, PagedKVCache):
            raise TypeError("a shard is a contiguous cache")
        self.cache, self.block0, self.topk = cache, int(block0), int(topk)
        self.params = _params(topk)
        self.lib = load()
        desc = cache.desc()
        n = self.lib.qsa_decode_shard_workspace_size(ctypes.byref(desc), self.params)
        if n == 0:
            raise QSAError("qsa_decode_shard_workspace_size", 1)
        self.ws = new_workspace(n, cache.device)

    def select(self, q_idx, w, glen: torch.Tensor, cand_score=None, cand_idx=None,
               cand_cnt=None):
        """This shard's candidates: (scores [B, topk] fp32, global blocks [B, topk] int32,
        counts [B] int32).  glen: the sequences' whole lengths, int32 [B] on the device."""
        B = self.cache.batch
        _need(q_idx, "q_idx", torch.bfloat16, (IDX_HEADS, IDX_DIM), 3)
        _need(w, "w", torch.bfloat16, (IDX_HEADS,), 2)
        _need(glen, "glen", torch.int32, ndim=1)
        dev = self.cache.device
        if cand_score is None:
            cand_score = torch.empty((B, self.topk), dtype=torch.float32, device=dev)
            cand_idx = torch.empty((B, self.topk), dtype=torch.int32, device=dev)
            cand_cnt = torch.empty((B,), dtype=torch.int32, device=dev)
        h_len = (ctypes.c_int32 * B)(*self.cache.h_len)
        desc = self.cache.desc()
        _check("qsa_decode_shard_select", self.lib.qsa_decode_shard_select(
            _ptr(q_idx), _ptr(w), ctypes.byref(desc), self.block0, _ptr(glen), h_len,
            _ptr(cand_score), _ptr(cand_idx), _ptr(cand_cnt), _ptr(self.ws), self.ws.numel(),
            self.params, _stream(dev)))
        return cand_score, cand_idx, cand_cnt

    def attend(self, q, glen, sel_idx, sel_cnt, part_o=None, part_m=None, part_l=None):
        """This shard's partial softmax: (o [B, 24, 128], m [B, 24], l [B, 24]) fp32."""
        B = self.cache.batch
        _need(q, "q", torch.bfloat16, (NUM_HEADS, HEAD_DIM), 3)
        dev = self.cache.device
        if part_o is None:
            part_o = torch.empty((B, NUM_HEADS, HEAD_DIM), dtype=torch.float32, device=dev)
            part_m = torch.empty((B, NUM_HEADS), dtype=torch.float32, device=dev)
            part_l = torch.empty((B, NUM_HEADS), dtype=torch.float32, device=dev)
        desc = self.cache.desc()
        _check("qsa_decode_shard_attend", self.lib.qsa_decode_shard_attend(
            _ptr(q), ctypes.byref(desc), self.block0, _ptr(glen), _ptr(sel_idx), _ptr(sel_cnt),
            _ptr(part_o), _ptr(part_m), _ptr(part_l), _ptr(self.ws), self.ws.numel(),
            self.params, _stream(dev)))
        return part_o, part_m, part_l

    def device_error(self):
        return last_device_error(self.ws)


def merge_candidates(cand_score, cand_idx, cand_cnt, topk: int, max_blocks: int, sel_idx=None,
                     sel_cnt=None, workspace=None):
    """Stacked shard candidates [R, B, topk] (scores, blocks) and counts [R, B] -> the
    selection (idx [B, topk] ascending -1 padded, cnt [B])."""
    _need(cand_score, "cand_score", torch.float32, ndim=3)
    _need(cand_idx, "cand_idx", torch.int32, ndim=3)
    _need(cand_cnt, "cand_cnt", torch.int32, ndim=2)
    R, B, k = cand_score.shape
    dev = cand_score.device
    if sel_idx is None:
        sel_idx = torch.empty((B, topk), dtype=torch.int32, device=dev)
        sel_cnt = torch.empty((B,), dtype=torch.int32, device=dev)
    ws = workspace if workspace is not None else new_workspace(WS_HEADER_BYTES, dev)
    _check("qsa_merge_candidates", load().qsa_merge_candidates(
        _ptr(cand_score), _ptr(cand_idx), _ptr(cand_cnt), R, B, int(topk), int(max_blocks),
        _ptr(sel_idx), _ptr(sel_cnt), _ptr(ws), ws.numel(), _stream(dev)))
    return sel_idx, sel_cnt


def combine_partials(part_o, part_m, part_l, out=None):
    """Stacked shard partials o [R, B, 24, 128], m and l [R, B, 24] -> out [B, 24, 128] bf16."""
    _need(part_o, "part_o", torch.float32, (NUM_HEADS, HEAD_DIM), 4)
    _need(part_m, "part_m", torch.float32, (NUM_HEADS,), 3)
    _need(part_l, "part_l", torch.float32, (NUM_HEADS,), 3)
    R, B = part_o.shape[:2]
    if out is None:
        out = torch.empty((B, NUM_HEADS, HEAD_DIM), dtype=torch.bfloat16, device=part_o.device)
    _check("qsa_combine_partials", load().qsa_combine_partials(
        _ptr(part_o), _ptr(part_m), _ptr(part_l), R, B, _ptr(out), _stream(part_o.device)))
    return out


def gated_deltanet(q, k, v, log_alpha, beta, cu_seqlens, out=None, with_state=False,
                   d_cu_seqlens=None):
    """The Gated DeltaNet layer over packed sequences: q, k, v bf16 [T, H, 128], log_alpha and
    beta fp32 [T, H] -> out bf16 [T, H, 128] (and the final states fp32 [S, H, 128, 128]).
    d_cu_seqlens: a device copy of cu_seqlens (host) to reuse instead of copying it."""
    dev = q.device
    if d_cu_seqlens is not None:
        h, d = torch.as_tensor(cu_seqlens, dtype=torch.int32).contiguous(), d_cu_seqlens
    else:
        h, d = _cu_pair(cu_seqlens, dev)
    T = int(h[-1])
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, (q.shape[1], 128), 3)
        if t.shape[0] != T:
            raise ValueError(f"{name}: {t.shape[0]} tokens, cu_seqlens says {T}")
    H = q.shape[1]
    for name, t in (("log_alpha", log_alpha), ("beta", beta)):
        _need(t, name, torch.float32, (H,), 2)
        if t.shape[0] != T:
            raise ValueError(f"{name}: {t.shape[0]} tokens, cu_seqlens says {T}")
    if out is None:
        out = torch.empty_like(q)
    S = h.numel() - 1
    state = torch.empty((S, H, 128, 128), dtype=torch.float32, device=dev) if with_state else None
    _check("qsa_gated_deltanet", load().qsa_gated_deltanet(
        _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(d),
        ctypes.c_void_p(h.data_ptr()), S, H, _ptr(out), _ptr(state), _stream(dev)))
    return (out, state) if with_state else out
