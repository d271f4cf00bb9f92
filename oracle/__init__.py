"""CPU oracle for Qwen Sparse Attention (QSA) -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The product library (``block_sparse_attention_40_b200``)
never imports it, and it never imports the product library: the two share no code.

``qsa_oracle.c`` holds the arithmetic (plain C, fp64 after the fp32/bf16 compression
step); this module compiles it with gcc and marshals numpy arrays through ctypes.
``brute.py`` is an independent pure-Python restatement used to pin the C code on tiny
inputs.

Arrays of bf16 values are passed as their raw 16-bit patterns (``numpy.uint16``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qsa_oracle.c")
_LIB = os.path.join(_HERE, "libqsa_oracle.so")
# A prebuilt variant of the oracle (used by the mutation test to plant mistakes).
_LIB_OVERRIDE = os.environ.get("QSA_ORACLE_LIB")
_lock = threading.Lock()
_lib = None

NUM_HEADS, NUM_KV_HEADS, HEAD_DIM = 24, 2, 128
IDX_HEADS, IDX_DIM, BLOCK = 16, 64, 4


def build(force: bool = False) -> str:
    """Compile qsa_oracle.c into libqsa_oracle.so (no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
               "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(_LIB_OVERRIDE if _LIB_OVERRIDE else build())
            P = ctypes.c_void_p
            i64, i32 = ctypes.c_int64, ctypes.c_int32
            lib.qsa_oracle_compress.argtypes = [P, P, i32, P]
            lib.qsa_oracle_compress.restype = None
            lib.qsa_oracle_score_pairs.argtypes = [P, P, P, P, P, P, P, i64, P]
            lib.qsa_oracle_score_pairs.restype = None
            lib.qsa_oracle_rows.argtypes = [P, P, P, P, P, i64, P, P, P, P, P, i32, P, P, P, P,
                                            P, P, i32]
            lib.qsa_oracle_rows.restype = None
            lib.qsa_oracle_constant.argtypes = [i32]
            lib.qsa_oracle_constant.restype = i32
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a, shape_tail):
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    assert a.shape[1:] == tuple(shape_tail), (a.shape, shape_tail)
    return a


def constants() -> dict:
    lib = _load()
    names = ["num_heads", "num_kv_heads", "head_dim", "idx_heads", "idx_dim", "block"]
    return {n: lib.qsa_oracle_constant(i) for i, n in enumerate(names)}


def kbar_offsets(cu_seqlens) -> np.ndarray:
    """Block offset of each sequence in the packed compressed-key array."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    nb = (cu[1:] - cu[:-1]) // BLOCK
    return np.concatenate([[0], np.cumsum(nb)]).astype(np.int64)


def compress(k_idx_bits: np.ndarray, cu_seqlens) -> np.ndarray:
    """Block compression of per-token indexer keys -> packed bf16 bits [sum floor(L/4), 64]."""
    k_idx_bits = _u16(k_idx_bits, (IDX_DIM,))
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    off = kbar_offsets(cu)
    out = np.zeros((int(off[-1]), IDX_DIM), dtype=np.uint16)
    _load().qsa_oracle_compress(_ptr(k_idx_bits), _ptr(cu), len(cu) - 1, _ptr(out))
    return out


def score_pairs(q_idx_rows, w_rows, kbar_bits, cu_seqlens, row_seq, pair_row, pair_block):
    """fp64 indexer scores s(row, block) for explicit pairs."""
    q_idx_rows = _u16(q_idx_rows, (IDX_HEADS, IDX_DIM))
    w_rows = _u16(w_rows, (IDX_HEADS,))
    kbar_bits = _u16(kbar_bits, (IDX_DIM,))
    off = kbar_offsets(cu_seqlens)
    row_seq = np.ascontiguousarray(row_seq, dtype=np.int64)
    pair_row = np.ascontiguousarray(pair_row, dtype=np.int64)
    pair_block = np.ascontiguousarray(pair_block, dtype=np.int64)
    out = np.zeros(len(pair_row), dtype=np.float64)
    _load().qsa_oracle_score_pairs(_ptr(q_idx_rows), _ptr(w_rows), _ptr(kbar_bits), _ptr(off),
                                   _ptr(row_seq), _ptr(pair_row), _ptr(pair_block),
                                   len(pair_row), _ptr(out))
    return out


def rows(*, q_rows, q_idx_rows, w_rows, row_seq, row_pos, k, v, kbar, cu_seqlens, topk,
         forced_idx=None, forced_cnt=None, threads=None):
    """Run the oracle on a list of query rows.

    Returns (idx [n, topk] int32 padded with -1, cnt [n] int32, kth [n] float64,
    out [n, 24, 128] float64 or None).  With ``forced_idx`` the given selection is
    used instead of the oracle's own (idx/cnt/kth are then returned as given / None).
    """
    n = len(row_pos)
    q_idx_rows = _u16(q_idx_rows, (IDX_HEADS, IDX_DIM))
    w_rows = _u16(w_rows, (IDX_HEADS,))
    kbar = _u16(kbar, (IDX_DIM,))
    if q_rows is not None:
        q_rows = _u16(q_rows, (NUM_HEADS, HEAD_DIM))
        k = _u16(k, (NUM_KV_HEADS, HEAD_DIM))
        v = _u16(v, (NUM_KV_HEADS, HEAD_DIM))
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int64)
    off = kbar_offsets(cu)
    row_seq = np.ascontiguousarray(row_seq, dtype=np.int64)
    row_pos = np.ascontiguousarray(row_pos, dtype=np.int64)
    assert len(row_seq) == n
    assert np.all(row_pos >= 0) and np.all(row_pos < (cu[row_seq + 1] - cu[row_seq]))
    idx = np.full((n, topk), -1, dtype=np.int32)
    cnt = np.zeros(n, dtype=np.int32)
    kth = np.zeros(n, dtype=np.float64)
    out = np.zeros((n, NUM_HEADS, HEAD_DIM), dtype=np.float64) if q_rows is not None else None
    if forced_idx is not None:
        forced_idx = np.ascontiguousarray(forced_idx, dtype=np.int32)
        forced_cnt = np.ascontiguousarray(forced_cnt, dtype=np.int32)
        assert forced_idx.shape == (n, topk) and forced_cnt.shape == (n,)
    threads = threads or os.cpu_count() or 1
    _load().qsa_oracle_rows(_ptr(q_rows), _ptr(q_idx_rows), _ptr(w_rows), _ptr(row_seq),
                            _ptr(row_pos), n, _ptr(k), _ptr(v), _ptr(kbar), _ptr(cu), _ptr(off),
                            topk, _ptr(forced_idx), _ptr(forced_cnt), _ptr(idx), _ptr(cnt),
                            _ptr(kth), _ptr(out), int(threads))
    if forced_idx is not None:
        return forced_idx, forced_cnt, None, out
    return idx, cnt, kth, out


def prefill(*, q, k, v, q_idx, k_idx, w, cu_seqlens, topk, row_ids=None, threads=None,
            forced_idx=None, forced_cnt=None):
    """Oracle over a packed varlen prefill batch.

    All tensors are numpy uint16 bf16 bit patterns, token-major:
    q [T,24,128], k/v [T,2,128], q_idx [T,16,64], k_idx [T,64], w [T,16].
    ``row_ids`` (global token indices) selects which rows to evaluate (default: all).
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    T = int(cu[-1])
    if row_ids is None:
        row_ids = np.arange(T, dtype=np.int64)
    row_ids = np.asarray(row_ids, dtype=np.int64)
    row_seq = np.searchsorted(cu, row_ids, side="right") - 1
    row_pos = row_ids - cu[row_seq]
    kbar = compress(k_idx, cu)
    res = rows(q_rows=None if q is None else np.ascontiguousarray(q[row_ids]),
               q_idx_rows=np.ascontiguousarray(q_idx[row_ids]),
               w_rows=np.ascontiguousarray(w[row_ids]), row_seq=row_seq, row_pos=row_pos,
               k=k, v=v, kbar=kbar, cu_seqlens=cu, topk=topk, forced_idx=forced_idx,
               forced_cnt=forced_cnt, threads=threads)
    return res + (kbar,)
