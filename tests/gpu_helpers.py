"""Helpers for the GPU parity tests: run the oracle on the same inputs and compare.

Tolerances (fixed for this library): block selections must match exactly when every score is
exact in fp32 (integer indexer inputs); otherwise a block may be swapped only if its oracle
score lies within 1e-4 (relative) of the k-th selected score.  Outputs (bf16) must match the
oracle (fp64, evaluated on the GPU's own selection) with max |err| <= 2e-2 and relative
L2 error <= 5e-3.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_40_b200 import workloads as W

MAX_ABS = 2e-2
REL_L2 = 5e-3
TIE_BAND = 1e-4

needs_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA device")


def rows_sample(T, n, seed=0, cu=None):
    """Seeded sample of rows: the first and last 8 of every sequence plus uniform draws."""
    rng = np.random.default_rng(seed)
    cu = [0, T] if cu is None else list(cu)
    pick = set()
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        pick.update(range(lo, min(hi, lo + 8)))
        pick.update(range(max(lo, hi - 8), hi))
    if n > len(pick):
        pick.update(rng.integers(0, T, n - len(pick)).tolist())
    return np.array(sorted(pick), dtype=np.int64)


def compare_selection(g_idx, g_cnt, o_idx, o_cnt, o_kth, score_fn, exact=False):
    """g_*/o_*: numpy arrays over the same rows.  score_fn(row_i, blocks) -> oracle scores."""
    assert np.array_equal(g_cnt, o_cnt), "selection counts differ"
    n_swapped = 0
    for i in range(len(g_cnt)):
        c = int(g_cnt[i])
        a, b = g_idx[i, :c], o_idx[i, :c]
        assert np.all(np.diff(a) > 0), f"row {i}: gpu selection not strictly ascending"
        assert np.all(g_idx[i, c:] == -1), f"row {i}: padding not -1"
        if np.array_equal(a, b):
            continue
        assert not exact, f"row {i}: selections differ on exact inputs"
        diff = np.setxor1d(a, b)
        s = score_fn(i, diff)
        kth = o_kth[i]
        assert np.all(np.abs(s - kth) <= TIE_BAND * abs(kth)), (
            f"row {i}: swapped blocks {diff[:8]} with scores {s[:8]} vs k-th {kth}")
        n_swapped += 1
    return n_swapped


def compare_outputs(g_out, o_out):
    g = g_out.to(torch.float64).cpu().numpy() if isinstance(g_out, torch.Tensor) else g_out
    err = np.abs(g - o_out)
    rel = np.linalg.norm(g - o_out) / max(np.linalg.norm(o_out), 1e-30)
    assert np.isfinite(g).all(), "non-finite outputs"
    assert err.max() <= MAX_ABS, f"max abs err {err.max():.3e}"
    assert rel <= REL_L2, f"rel L2 err {rel:.3e}"
    return float(err.max()), float(rel)


def prefill_oracle_check(p: W.Prefill, g_idx, g_cnt, g_out, rows, exact_sel=False, threads=None):
    """Compare GPU prefill results (full tensors) with the oracle on `rows` (global ids)."""
    b = {n: W.bits(getattr(p, n)) for n in ("q", "k", "v", "q_idx", "k_idx", "w")}
    cu = p.cu_seqlens.numpy().astype(np.int64)
    rows = np.asarray(rows, dtype=np.int64)
    o_idx, o_cnt, o_kth, _, kbar = oracle.prefill(q=None, k=b["k"], v=b["v"], q_idx=b["q_idx"],
                                                  k_idx=b["k_idx"], w=b["w"], cu_seqlens=cu,
                                                  topk=p.topk, row_ids=rows, threads=threads)
    gi = g_idx[rows].cpu().numpy() if isinstance(g_idx, torch.Tensor) else g_idx[rows]
    gc = g_cnt[rows].cpu().numpy() if isinstance(g_cnt, torch.Tensor) else g_cnt[rows]
    row_seq = np.searchsorted(cu, rows, side="right") - 1

    def score_fn(i, blocks):
        return oracle.score_pairs(b["q_idx"][rows[i]:rows[i] + 1], b["w"][rows[i]:rows[i] + 1],
                                  kbar, cu, row_seq[i:i + 1], np.zeros(len(blocks), np.int64),
                                  blocks)

    swaps = compare_selection(gi, gc, o_idx, o_cnt, o_kth, score_fn, exact=exact_sel)
    res = {"swapped_rows": swaps}
    if g_out is not None:
        _, _, _, o_out, _ = oracle.prefill(q=b["q"], k=b["k"], v=b["v"], q_idx=b["q_idx"],
                                           k_idx=b["k_idx"], w=b["w"], cu_seqlens=cu, topk=p.topk,
                                           row_ids=rows, forced_idx=gi, forced_cnt=gc,
                                           threads=threads)
        res["max_abs"], res["rel_l2"] = compare_outputs(g_out[rows], o_out)
    return res
