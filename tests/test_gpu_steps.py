"""GPU parity of the individual steps: compression (a1), indexer scores (a2), top-k (a3),
cache append (a5).  Integer and byte work is compared bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_40_b200 as qsa
from block_sparse_attention_40_b200 import workloads as W
from tests.gpu_helpers import needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda:0"


def _kbar_bits(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("lengths", [[256], [1, 2, 3, 4, 5, 7, 8, 9], [1023, 4097, 33, 4],
                                     [131071]])
def test_compress_bitwise(lengths):
    p = W.custom_prefill(lengths, topk=16, kind="normal", seed=len(lengths))
    kb = qsa.compress(p.k_idx.to(DEV), p.cu_seqlens)
    torch.cuda.synchronize()
    want = oracle.compress(W.bits(p.k_idx), p.cu_seqlens.numpy().astype(np.int64))
    assert np.array_equal(_kbar_bits(kb), want)


def test_compress_order_sensitive_bitwise():
    # (a, x, -a, y) with |a| = 2^20: any other summation order changes most outputs
    g = torch.Generator().manual_seed(3)
    nb = 4096
    a = torch.where(torch.rand((nb, 64), generator=g) < 0.5, -1.0, 1.0) * 2.0 ** 20
    tok = torch.stack([a, torch.randn((nb, 64), generator=g), -a,
                       torch.randn((nb, 64), generator=g)], 1).to(torch.bfloat16).reshape(-1, 64)
    kb = qsa.compress(tok.to(DEV), [0, 4 * nb])
    want = oracle.compress(W.bits(tok), np.array([0, 4 * nb]))
    assert np.array_equal(_kbar_bits(kb), want)


def _oracle_scores_rows(p, rows):
    b = {n: W.bits(getattr(p, n)) for n in ("q_idx", "k_idx", "w")}
    cu = p.cu_seqlens.numpy().astype(np.int64)
    kbar = oracle.compress(b["k_idx"], cu)
    row_seq = np.searchsorted(cu, rows, side="right") - 1
    pr, pb = [], []
    for i, r in enumerate(rows):
        n_c = (r - cu[row_seq[i]]) // 4
        pr += [i] * n_c
        pb += list(range(n_c))
    s = oracle.score_pairs(b["q_idx"][rows], b["w"][rows], kbar, cu, row_seq, np.array(pr),
                           np.array(pb))
    return np.array(pr), np.array(pb), s


@pytest.mark.parametrize("name,exact", [("8k_int", True), ("tiny", False)])
def test_index_scores(name, exact):
    p = W.prefill(name)
    cu = p.cu_seqlens
    kb = qsa.compress(p.k_idx.to(DEV), cu)
    scores = qsa.index_scores(p.q_idx.to(DEV), p.w.to(DEV), kb, cu, topk=0)
    torch.cuda.synchronize()
    T = int(cu[-1])
    rows = np.unique(np.concatenate([np.arange(0, T, max(1, T // 61)), [T - 1, T - 2, 4, 5, 16]]))
    pr, pb, s = _oracle_scores_rows(p, rows)
    g = scores.cpu().numpy()[rows[pr], pb].astype(np.float64)
    if exact:
        assert np.array_equal(g, s)
    else:
        np.testing.assert_allclose(g, s, rtol=2e-5, atol=1e-5)


def test_index_scores_ragged_rows_and_skip():
    p = W.custom_prefill([37, 100, 16, 64, 300], topk=8, kind="int", seed=4)
    cu = p.cu_seqlens
    kb = qsa.compress(p.k_idx.to(DEV), cu)
    # a sub-range on 16-token tile boundaries: the second sequence from its 32nd token to the
    # end of the fourth sequence
    r0, r1 = 37 + 32, 37 + 100 + 16 + 64
    scores = qsa.index_scores(p.q_idx.to(DEV), p.w.to(DEV), kb, cu, row_begin=r0, row_end=r1,
                              topk=0)
    torch.cuda.synchronize()
    rows = np.arange(r0, r1)
    pr, pb, s = _oracle_scores_rows(p, rows)
    g = scores.cpu().numpy()[pr, pb].astype(np.float64)
    assert np.array_equal(g, s)
    with pytest.raises(qsa.QSAError):   # not on a tile boundary
        qsa.index_scores(p.q_idx.to(DEV), p.w.to(DEV), kb, cu, row_begin=r0 + 1, row_end=r1)


def _topk_reference(s, n, k):
    """Selection by definition: order by (-score, index), keep min(k, n), ascending."""
    if n <= k:
        return np.arange(n)
    order = np.lexsort((np.arange(n), -s[:n].astype(np.float64)))
    return np.sort(order[:k])


@pytest.mark.parametrize("k", [1, 16, 512])
def test_topk_kernel(k):
    g = torch.Generator().manual_seed(k)
    ns = [0, 1, k - 1 if k > 1 else 0, k, k + 1, 700, 5000, 40000, 70000]
    ld = max(ns) + 4
    rows = len(ns) * 3
    sc = torch.zeros((rows, ld), dtype=torch.float32)
    n_c = []
    for r in range(rows):
        n = ns[r % len(ns)]
        kind = r // len(ns)
        if kind == 0:
            v = torch.rand(n, generator=g)                      # distinct-ish values
        elif kind == 1:
            v = torch.randint(0, 7, (n,), generator=g).float()  # heavy ties
        else:
            v = torch.zeros(n)                                  # all equal
        sc[r, :n] = v
        n_c.append(n)
    n_c_t = torch.tensor(n_c, dtype=torch.int32)
    idx, cnt = qsa.topk(sc.to(DEV), n_c_t.to(DEV), k)
    torch.cuda.synchronize()
    idx, cnt = idx.cpu().numpy(), cnt.cpu().numpy()
    for r in range(rows):
        want = _topk_reference(sc[r].numpy(), n_c[r], k)
        assert cnt[r] == len(want)
        assert np.array_equal(idx[r, :cnt[r]], want), r
        assert np.all(idx[r, cnt[r]:] == -1)


def test_append_incremental_equals_bulk():
    B, cap = 3, 256
    gen = torch.Generator().manual_seed(11)
    total = [250, 97, 256]
    ks = torch.randn((B, 256, 2, 128), generator=gen).to(torch.bfloat16)
    vs = torch.randn((B, 256, 2, 128), generator=gen).to(torch.bfloat16)
    kis = torch.randn((B, 256, 64), generator=gen).to(torch.bfloat16)
    cache = qsa.KVCache(B, cap, DEV, zero=False)
    pos = [0, 0, 0]
    steps = [1, 3, 5, 2, 7, 1, 1, 64, 13, 4, 100, 60]
    for n in steps:
        counts = [max(0, min(n, total[b] - pos[b])) for b in range(B)]
        kk = torch.zeros((B, n, 2, 128), dtype=torch.bfloat16)
        vv = torch.zeros((B, n, 2, 128), dtype=torch.bfloat16)
        ki = torch.zeros((B, n, 64), dtype=torch.bfloat16)
        for b in range(B):
            c = counts[b]
            kk[b, :c], vv[b, :c], ki[b, :c] = ks[b, pos[b]:pos[b] + c], vs[b, pos[b]:pos[b] + c], \
                kis[b, pos[b]:pos[b] + c]
        cache.append(kk.to(DEV), vv.to(DEV), ki.to(DEV), counts=counts)
        pos = [pos[b] + counts[b] for b in range(B)]
    torch.cuda.synchronize()
    assert cache.len.cpu().tolist() == total == cache.h_len
    for b in range(B):
        L = total[b]
        want = oracle.compress(W.bits(kis[b, :L]), np.array([0, L]))
        got = _kbar_bits(cache.kbar[b, :L // 4])
        assert np.array_equal(got, want), b
        kb = cache.k_blocks[b].cpu()                       # [2, cap/4, 4, 128]
        kt = kb.permute(1, 2, 0, 3).reshape(cap, 2, 128)[:L]
        assert torch.equal(kt, ks[b, :L])
        vt = cache.v_blocks[b].cpu().permute(1, 2, 0, 3).reshape(cap, 2, 128)[:L]
        assert torch.equal(vt, vs[b, :L])
        # rows after the last token of an incomplete block are zeroed
        if L % 4:
            assert torch.all(kb[:, L // 4, L % 4:] == 0)
        if L % 4:
            part = cache.kbar_partial[b].cpu()
            x = kis[b, 4 * (L // 4):L].to(torch.float32)
            acc = x[0].clone()
            for j in range(1, x.shape[0]):
                acc = acc + x[j]
            assert torch.equal(part, acc)


def test_append_capacity_error():
    cache = qsa.KVCache(1, 8, DEV)
    t = torch.zeros((1, 9, 2, 128), dtype=torch.bfloat16, device=DEV)
    ti = torch.zeros((1, 9, 64), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(qsa.QSAError, match="CAPACITY"):
        cache.append(t, t, ti)
