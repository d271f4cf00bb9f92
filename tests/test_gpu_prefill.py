"""GPU parity of QSA prefill (steps a1-a4) against the oracle."""
import dataclasses

import numpy as np
import pytest
import torch

import block_sparse_attention_40_b200 as qsa
from block_sparse_attention_40_b200 import workloads as W
from tests.gpu_helpers import needs_gpu, prefill_oracle_check, rows_sample

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda:0"


def _run(p, rows_per_tile=0, chunk=0):
    d = p.to(DEV)
    ctx = qsa.Prefill(p.cu_seqlens, DEV, p.topk, rows_per_tile, chunk)
    idx, cnt = ctx.select(d.q_idx, d.k_idx, d.w)
    out = ctx.run(d.q, d.k, d.v, d.q_idx, d.k_idx, d.w)
    torch.cuda.synchronize()
    assert ctx.device_error() == ("QSA_OK", 0)
    return idx, cnt, out


def test_tiny_full():
    p = W.prefill("tiny")
    idx, cnt, out = _run(p)
    res = prefill_oracle_check(p, idx, cnt, out, np.arange(256))
    assert res["swapped_rows"] <= 2


@pytest.mark.parametrize("rows_per_tile", [1, 3, 8, 10])
def test_rows_per_tile_variants(rows_per_tile):
    p = W.custom_prefill([203, 77], topk=7, kind="normal", seed=rows_per_tile)
    idx, cnt, out = _run(p, rows_per_tile=rows_per_tile)
    prefill_oracle_check(p, idx, cnt, out, np.arange(280))


def test_short_sequences_and_dense_rows():
    # lengths below one block, exactly one block, and rows whose candidates fit the budget
    p = W.custom_prefill([1, 2, 3, 4, 5, 9, 31, 64], topk=512, kind="normal", seed=5)
    idx, cnt, out = _run(p)
    prefill_oracle_check(p, idx, cnt, out, np.arange(int(p.cu_seqlens[-1])))


@pytest.mark.parametrize("case", ["spread", "far_below", "far_above"])
def test_attention_logits_far_from_zero(case):
    # The attention logits q.k/sqrt(128) (log2 units) spread over hundreds of units within a
    # row (q and k times 16, exact in bf16), or all lie about 260 units below or above zero
    # (q = -4 or +4 in every dim, k shifted by +4): the softmax's running reference must move
    # far within a row, and an exponent relative to a stale one would underflow or overflow.
    # The selection comes from the indexer inputs, which stay as drawn.
    p = W.custom_prefill([700, 333], topk=16, kind="normal", seed=11)
    if case == "spread":
        q, k = p.q.float() * 16, p.k.float() * 16
    else:
        q = torch.full_like(p.q, -4.0 if case == "far_below" else 4.0, dtype=torch.float32)
        k = p.k.float() + 4
    p = dataclasses.replace(p, q=q.bfloat16(), k=k.bfloat16())
    idx, cnt, out = _run(p)
    assert torch.isfinite(out.float()).all()
    prefill_oracle_check(p, idx, cnt, out, np.arange(1033))


def test_budget_one_and_chunked_scores():
    p = W.custom_prefill([300, 129], topk=1, kind="normal", seed=6)
    idx, cnt, out = _run(p, chunk=48)
    prefill_oracle_check(p, idx, cnt, out, np.arange(429))


def test_8k_integer_selection_bit_exact():
    p = W.prefill("8k_int")
    d = p.to(DEV)
    ctx = qsa.Prefill(p.cu_seqlens, DEV, p.topk)
    idx, cnt = ctx.select(d.q_idx, d.k_idx, d.w)
    torch.cuda.synchronize()
    prefill_oracle_check(p, idx, cnt, None, np.arange(8192), exact_sel=True)


def test_8k_needles_sampled():
    p = W.prefill("8k")
    idx, cnt, out = _run(p)
    rows = rows_sample(8192, 1024, seed=1)
    prefill_oracle_check(p, idx, cnt, out, rows)
    # needles are always selected by rows that can see them
    needles = p.needles[0]
    ic = idx.cpu().numpy()
    cc = cnt.cpu().numpy()
    for t in range(0, 8192, 3):
        sel = set(ic[t, :cc[t]].tolist())
        assert {n for n in needles if n < t // 4} <= sel


@pytest.mark.slow
def test_ragged_sampled():
    p = W.prefill("ragged")
    idx, cnt, out = _run(p)
    T = int(p.cu_seqlens[-1])
    rows = rows_sample(T, 4096, seed=2, cu=p.cu_seqlens.tolist())
    prefill_oracle_check(p, idx, cnt, out, rows)


@pytest.mark.slow
def test_64k_sampled():
    p = W.prefill("64k", device=DEV)
    idx, cnt, out = _run(p)
    rows = rows_sample(65536, 4096, seed=3)
    prefill_oracle_check(p, idx, cnt, out, rows)


def _select_check(p, rows, exact=False, chunk=0):
    d = p.to(DEV)
    ctx = qsa.Prefill(p.cu_seqlens, DEV, p.topk, 0, chunk)
    idx, cnt = ctx.select(d.q_idx, d.k_idx, d.w)
    torch.cuda.synchronize()
    assert ctx.device_error() == ("QSA_OK", 0)
    return prefill_oracle_check(p, idx, cnt, None, rows, exact_sel=exact)


@pytest.mark.parametrize("topk", [513, 640])
def test_selection_large_budgets_drift(topk):
    # budgets above 512 blocks on keys that drift along the sequence, so scores trend with
    # the block index
    p = W.custom_prefill([9000, 2222], topk=topk, kind="drift", seed=topk)
    T = int(p.cu_seqlens[-1])
    _select_check(p, rows_sample(T, 1536, seed=4, cu=p.cu_seqlens.tolist()))


def test_selection_budget_700_small_chunks():
    # a budget of 700 blocks with score chunks of 2048 rows
    p = W.custom_prefill([5000, 3001], topk=700, kind="normal", seed=7)
    T = int(p.cu_seqlens[-1])
    _select_check(p, rows_sample(T, 1536, seed=3, cu=p.cu_seqlens.tolist()), chunk=2048)


def test_selection_all_scores_equal():
    # w = 0 makes every score 0: each row selects its lowest topk block indices
    p = W.custom_prefill([7000, 50, 3], topk=512, kind="normal", seed=9)
    p.w.zero_()
    T = int(p.cu_seqlens[-1])
    _select_check(p, rows_sample(T, 1024, seed=5, cu=p.cu_seqlens.tolist()), exact=True)


def test_selection_integer_scores_many_ties_small_budget():
    # small-integer indexer inputs with a budget of 5 blocks: long runs of equal scores at
    # the threshold, resolved toward lower block indices
    p = W.custom_prefill([4100, 999], topk=5, kind="int", seed=10)
    T = int(p.cu_seqlens[-1])
    _select_check(p, rows_sample(T, 1024, seed=6, cu=p.cu_seqlens.tolist()), exact=True)


@pytest.mark.slow
def test_selection_rows_beyond_65536_blocks():
    # rows of more than 65,536 candidate blocks (positions past 262,144 tokens)
    L = 266_300
    p = W.custom_prefill([L], topk=512, kind="normal", seed=11, device=DEV)
    rows = np.concatenate([rows_sample(L, 256, seed=7), np.arange(L - 64, L - 8),
                           np.arange(262_140, 262_160)])
    rows = np.unique(rows)
    _select_check(p, rows)


@pytest.mark.parametrize("name", ["tiny", "8k", "8k_int", "drift"])
def test_select_mode_1_equals_mode_0(name):
    # select_mode 1 (the indexer finds each row's threshold bin, the top-k reads each row
    # once) computes the same scores and the same selection: identical indices, counts and
    # outputs, bit for bit
    p = (W.custom_prefill([9000, 2222], topk=512, kind="drift", seed=21) if name == "drift"
         else W.prefill(name))
    d = p.to(DEV)
    res = []
    for mode in (0, 1):
        ctx = qsa.Prefill(p.cu_seqlens, DEV, p.topk, select_mode=mode)
        idx, cnt = ctx.select(d.q_idx, d.k_idx, d.w)
        out = ctx.run(d.q, d.k, d.v, d.q_idx, d.k_idx, d.w)
        torch.cuda.synchronize()
        assert ctx.device_error() == ("QSA_OK", 0)
        res.append((idx, cnt, out))
    assert torch.equal(res[0][0], res[1][0]) and torch.equal(res[0][1], res[1][1])
    assert torch.equal(res[0][2], res[1][2])
    if name == "tiny":
        prefill_oracle_check(p, res[1][0], res[1][1], res[1][2], np.arange(256))
