"""Pins of the oracle against closed forms, invariants and library routines.

* dense equivalence: with at most k candidate blocks, QSA is dense causal GQA attention
  (torch scaled_dot_product_attention in fp64, a library routine);
* V == 1 gives outputs of exactly 1 (softmax weights sum to one);
* constant scores (w == 0): the tie-break keeps blocks 0..k-1;
* monotone scores: the k most recent complete blocks, i.e. a sliding window;
* integer indexer inputs: scores equal exact integer arithmetic;
* planted needle blocks are selected by every row that can see them, by a margin.
"""
import numpy as np
import pytest
import torch

import oracle
from block_sparse_attention_40_b200 import workloads as W
from tests.helpers import dense_gqa_reference, prefill_bits


def _run(p, row_ids=None, threads=None):
    b = prefill_bits(p)
    return oracle.prefill(q=b["q"], k=b["k"], v=b["v"], q_idx=b["q_idx"], k_idx=b["k_idx"],
                          w=b["w"], cu_seqlens=b["cu_seqlens"], topk=p.topk, row_ids=row_ids,
                          threads=threads)


def _mask_from_selection(T, idx, cnt):
    m = torch.zeros((T, T), dtype=torch.bool)
    for t in range(T):
        c = t // 4
        for b in idx[t, :cnt[t]]:
            m[t, 4 * b:4 * b + 4] = True
        m[t, 4 * c:t + 1] = True
    return m


def test_dense_equivalence_when_budget_covers_all():
    p = W.custom_prefill([203], topk=64, kind="normal", seed=3)   # n_c <= 50 < 64
    idx, cnt, kth, out, _ = _run(p)
    T = 203
    assert np.all(cnt == np.arange(T) // 4)
    causal = torch.tril(torch.ones((T, T), dtype=torch.bool))
    ref = dense_gqa_reference(p.q, p.k, p.v, causal)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)


def test_dense_equivalence_second_sequence_is_independent():
    p = W.custom_prefill([30, 45], topk=16, kind="normal", seed=4)
    idx, cnt, kth, out, _ = _run(p)
    for s, (lo, hi) in enumerate([(0, 30), (30, 75)]):
        T = hi - lo
        causal = torch.tril(torch.ones((T, T), dtype=torch.bool))
        ref = dense_gqa_reference(p.q[lo:hi], p.k[lo:hi], p.v[lo:hi], causal)
        np.testing.assert_allclose(out[lo:hi], ref.numpy(), rtol=0, atol=1e-12)


def test_values_one_give_one():
    p = W.custom_prefill([157], topk=5, kind="normal", seed=6)
    p.v = torch.ones_like(p.v)
    _, _, _, out, _ = _run(p)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-13)


def test_constant_scores_take_lowest_blocks():
    p = W.custom_prefill([211], topk=7, kind="normal", seed=8)
    p.w = torch.zeros_like(p.w)                                  # every score is 0
    idx, cnt, kth, out, _ = _run(p)
    T = 211
    for t in range(T):
        n_c = t // 4
        want = list(range(min(7, n_c)))
        assert idx[t, :cnt[t]].tolist() == want
    ref = dense_gqa_reference(p.q, p.k, p.v, _mask_from_selection(T, idx, cnt))
    # closed form of the mask: tokens [0, 28) plus the own block, causally
    m = torch.zeros((T, T), dtype=torch.bool)
    for t in range(T):
        m[t, :min(28, 4 * (t // 4))] = True
        m[t, 4 * (t // 4):t + 1] = True
    ref2 = dense_gqa_reference(p.q, p.k, p.v, m)
    np.testing.assert_allclose(out, ref2.numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(ref.numpy(), ref2.numpy(), rtol=0, atol=0)


def test_monotone_scores_give_sliding_window():
    T, k = 180, 6
    p = W.custom_prefill([T], topk=k, kind="normal", seed=10)
    kid = torch.zeros((T, 64))
    kid[:, 0] = (torch.arange(T) // 4 + 1).to(torch.float32)     # block b -> (b+1, 0, ...)
    p.k_idx = kid.to(torch.bfloat16)
    qi = p.q_idx.clone()
    qi[:, :, 0] = 1.0
    p.q_idx = qi
    p.w = (p.w.to(torch.float32) + 0.01).to(torch.bfloat16)     # strictly positive
    idx, cnt, kth, out, _ = _run(p)
    m = torch.zeros((T, T), dtype=torch.bool)
    for t in range(T):
        c = t // 4
        lo = max(0, c - k)
        assert idx[t, :cnt[t]].tolist() == list(range(lo, c))
        m[t, 4 * lo:t + 1] = True
    ref = dense_gqa_reference(p.q, p.k, p.v, m)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)


def test_integer_scores_are_exact():
    p = W.custom_prefill([403], topk=9, kind="int", seed=12)
    b = prefill_bits(p)
    cu = b["cu_seqlens"]
    kbar = oracle.compress(b["k_idx"], cu)
    kbar_f = torch.from_numpy(kbar.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    # exact mean of the four tokens: multiples of 1/4 in [-2, 2], all exact in bf16
    kid = p.k_idx.to(torch.float64)[: 4 * (403 // 4)].reshape(-1, 4, 64)
    assert torch.equal(kbar_f, kid.sum(1) / 4)
    k4 = (kbar_f * 4).to(torch.int64)                                     # integers
    qi = p.q_idx.to(torch.int64)
    w = p.w.to(torch.int64)
    rows = torch.arange(403)
    pr, pb = [], []
    for t in range(0, 403, 7):
        for bb in range(t // 4):
            pr.append(t)
            pb.append(bb)
    pr = np.array(pr)
    pb = np.array(pb)
    s = oracle.score_pairs(b["q_idx"], b["w"], kbar, cu, np.zeros(403, np.int64), pr, pb)
    dots4 = torch.einsum("nhd,nd->nh", qi[pr], k4[pb])                    # 4 * dot, exact
    exact4 = (w[pr] * dots4.clamp(min=0)).sum(1)                          # 4 * score
    assert np.array_equal(s * 4, exact4.numpy().astype(np.float64))
    assert rows.numel() == 403


def test_tiny_needles_always_selected():
    p = W.prefill("tiny")
    assert len(p.needles[0]) == 4
    idx, cnt, kth, out, kbar = _run(p)
    needles = p.needles[0]
    b = prefill_bits(p)
    for t in range(256):
        c = t // 4
        sel = set(idx[t, :cnt[t]].tolist())
        vis = [n for n in needles if n < c]
        assert set(vis) <= sel, (t, vis, sorted(sel))
        if vis and c > len(vis):
            # margin: the weakest visible needle beats the strongest other block
            others = [bb for bb in range(c) if bb not in needles]
            pr = np.full(len(vis) + len(others), 0)
            blocks = np.array(vis + others)
            s = oracle.score_pairs(b["q_idx"][t:t + 1], b["w"][t:t + 1], kbar, b["cu_seqlens"],
                                   np.zeros(1, np.int64), pr, blocks)
            assert s[:len(vis)].min() > s[len(vis):].max()


@pytest.mark.slow
def test_8k_needles_sampled_rows():
    p = W.prefill("8k")
    assert len(p.needles[0]) == 32
    rows = np.unique(np.concatenate([np.arange(8), np.arange(8184, 8192),
                                     np.random.default_rng(0).integers(0, 8192, 120)]))
    idx, cnt, kth, out, kbar = _run(p, row_ids=rows)
    for i, t in enumerate(rows):
        sel = set(idx[i, :cnt[i]].tolist())
        assert {n for n in p.needles[0] if n < t // 4} <= sel


def test_forced_own_selection_reproduces_outputs():
    # Handing the oracle its own selection through the forced path changes nothing: the
    # forced path attends exactly the blocks it is given (the GPU parity tests compare
    # outputs through this path, on the GPU's selection).
    p = W.custom_prefill([97, 66], topk=5, kind="normal", seed=14)
    idx, cnt, _, out, _ = _run(p)
    b = prefill_bits(p)
    _, _, _, out_f, _ = oracle.prefill(q=b["q"], k=b["k"], v=b["v"], q_idx=b["q_idx"],
                                       k_idx=b["k_idx"], w=b["w"], cu_seqlens=b["cu_seqlens"],
                                       topk=p.topk, forced_idx=idx, forced_cnt=cnt)
    assert np.array_equal(out_f, out)


def test_forced_selection_attends_exactly_the_given_blocks():
    # Arbitrary forced selections (seeded random ascending subsets of the candidates, of
    # any size up to k, including empty ones and dense prefixes) give dense attention
    # under the mask those blocks plus the own block make: fp64 SDPA, a library routine.
    T, k = 150, 9
    p = W.custom_prefill([T], topk=k, kind="normal", seed=15)
    rng = np.random.default_rng(15)
    fi = np.full((T, k), -1, dtype=np.int32)
    fc = np.zeros(T, dtype=np.int32)
    for t in range(T):
        n_c = t // 4
        if t % 5 == 0:
            sel = np.arange(min(k, n_c))                       # a dense prefix
        else:
            m = int(rng.integers(0, min(k, n_c) + 1))
            sel = np.sort(rng.choice(n_c, size=m, replace=False)) if m else np.zeros(0, int)
        fi[t, :len(sel)] = sel
        fc[t] = len(sel)
    b = prefill_bits(p)
    _, _, _, out, _ = oracle.prefill(q=b["q"], k=b["k"], v=b["v"], q_idx=b["q_idx"],
                                     k_idx=b["k_idx"], w=b["w"], cu_seqlens=b["cu_seqlens"],
                                     topk=k, forced_idx=fi, forced_cnt=fc)
    ref = dense_gqa_reference(p.q, p.k, p.v, _mask_from_selection(T, fi, fc))
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)
