"""Pin the C oracle against the pure-Python brute force on tiny inputs.

The brute force restates the method independently (rational bf16 rounding, rank
counting instead of sorting, explicit token lists); selections must agree exactly and
outputs to 1e-12.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import brute
from block_sparse_attention_40_b200 import workloads as W
from tests.helpers import prefill_bits, to_lists


def _check(p, rows_attn):
    b = prefill_bits(p)
    cu = b["cu_seqlens"]
    idx, cnt, kth, out, kbar = oracle.prefill(q=b["q"], k=b["k"], v=b["v"], q_idx=b["q_idx"],
                                              k_idx=b["k_idx"], w=b["w"], cu_seqlens=cu,
                                              topk=p.topk)
    off = oracle.kbar_offsets(cu)
    for s in range(len(cu) - 1):
        lo, hi = int(cu[s]), int(cu[s + 1])
        sl = slice(lo, hi)
        res, kbar_b = brute.run_sequence(to_lists(p.q[sl]), to_lists(p.k[sl]), to_lists(p.v[sl]),
                                         to_lists(p.q_idx[sl]), to_lists(p.k_idx[sl]),
                                         to_lists(p.w[sl]), p.topk,
                                         rows=[t for t in range(hi - lo)])
        # compression: identical bf16 values
        kb_c = torch.from_numpy(kbar[off[s]:off[s + 1]].view(np.int16)).view(torch.bfloat16)
        assert kb_c.to(torch.float64).tolist() == kbar_b
        for t, (sel, o) in res.items():
            r = lo + t
            got = idx[r, :cnt[r]].tolist()
            assert got == sel, (s, t, got, sel)
            assert np.all(idx[r, cnt[r]:] == -1)
            if t in rows_attn:
                np.testing.assert_allclose(out[r], np.array(o), rtol=0, atol=1e-12)


@pytest.mark.parametrize("seed", [1, 2])
def test_brute_random(seed):
    # two sequences, lengths not multiples of 4, budget small enough to bind
    p = W.custom_prefill([37, 22], topk=3, kind="normal", seed=seed)
    _check(p, rows_attn={0, 3, 4, 7, 19, 21, 36})


def test_brute_integer_ties():
    # integer indexer inputs produce many exactly tied scores: the tie-break is exercised
    p = W.custom_prefill([41], topk=2, kind="int", seed=5)
    _check(p, rows_attn={5, 40})


def test_brute_needles():
    p = W.custom_prefill([48], topk=2, kind="needle", seed=9, needles_per_seq=2,
                         needle_range=(1, 10))
    _check(p, rows_attn={47})


@pytest.mark.parametrize("seed,kind,topk", [(3, "normal", 3), (4, "normal", 5), (6, "int", 2)])
def test_kth_is_the_boundary_score(seed, kind, topk):
    # The oracle reports, per row, the score of its last kept block: the anchor of the
    # tie band within which a GPU selection may swap blocks.  The brute force finds the
    # same value by rank counting; rows with at most k candidates report -1 (no boundary).
    p = W.custom_prefill([45], topk=topk, kind=kind, seed=seed)
    b = prefill_bits(p)
    idx, cnt, kth, _, _ = oracle.prefill(q=None, k=b["k"], v=b["v"], q_idx=b["q_idx"],
                                         k_idx=b["k_idx"], w=b["w"], cu_seqlens=b["cu_seqlens"],
                                         topk=topk)
    sc = brute.row_scores(to_lists(p.q_idx), to_lists(p.k_idx), to_lists(p.w), range(45))
    bounded = 0
    for t in range(45):
        want = brute.kth_ranked_score(sc[t], topk)
        if want is None:
            assert kth[t] == -1.0, (t, kth[t])
        else:
            assert abs(kth[t] - want) <= 1e-12 * max(1.0, abs(want)), (t, kth[t], want)
            # the boundary is the lowest kept score and no dropped block beats it
            kept = set(idx[t, :cnt[t]].tolist())
            assert min(sc[t][x] for x in kept) == pytest.approx(want, rel=1e-12, abs=1e-12)
            assert all(sc[t][x] <= want + 1e-12 * max(1.0, abs(want))
                       for x in range(len(sc[t])) if x not in kept)
            bounded += 1
    assert bounded >= 20
