"""GPU parity of the paged decode cache (qsa_append_kv_paged, qsa_decode_paged).

A paged cache keeps each sequence's tokens in fixed-size pages of one shared pool, listed in a
page table (aiany.app "Qwen3.8-Flash-Next", "Implementation notes": the serving recipes and KV
cache sizing for very long contexts).  Paging changes where the blocks live, not what is
computed, so a paged decode must agree bit for bit with a contiguous one fed the same tokens,
and with the oracle within the decode tolerances."""
import pytest
import torch

import block_sparse_attention_40_b200 as qsa
from block_sparse_attention_40_b200 import workloads as W
from tests.gpu_helpers import needs_gpu
from tests.test_gpu_decode import _decode_session

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda:0"


def _paged(spec, page_tokens, spare=3, seed=0):
    """A paged cache whose pages are a seeded permutation of a pool with `spare` unused pages."""
    max_pages = spec.capacity // page_tokens
    pool = spec.batch * max_pages + spare
    gen = torch.Generator().manual_seed(seed)
    perm = torch.randperm(pool, generator=gen)[:spec.batch * max_pages]
    table = perm.view(spec.batch, max_pages).to(torch.int32).to(DEV)
    return qsa.PagedKVCache(spec.batch, spec.capacity, page_tokens, pool, table, DEV, zero=False)


def _fill(cache, spec, k, v, ki, chunk):
    lmax = max(spec.context)
    for c0 in range(0, lmax, chunk):
        c1 = min(lmax, c0 + chunk)
        counts = [max(0, min(c1, L) - c0) for L in spec.context]
        cache.append(k[:, c0:c1].contiguous(), v[:, c0:c1].contiguous(),
                     ki[:, c0:c1].contiguous(), counts=counts)


def _bits(t):
    return t.contiguous().view(torch.int16).cpu()


def _paged_vs_contiguous(spec, page_tokens, steps, chunk, seed=0):
    k, v, ki = W.decode_context(spec, device=DEV)
    flat = qsa.KVCache(spec.batch, spec.capacity, DEV, zero=False)
    paged = _paged(spec, page_tokens, seed=seed)
    _fill(flat, spec, k, v, ki, chunk)
    _fill(paged, spec, k, v, ki, chunk)
    del k, v, ki
    d_flat = qsa.Decoder(flat, spec.topk)
    d_paged = qsa.Decoder(paged, spec.topk)
    for step in range(steps):
        st = W.decode_step(spec, step, device=DEV)
        for c in (flat, paged):
            c.append(st["k"], st["v"], st["k_idx"])
        o1, i1, c1 = d_flat.run(st["q"], st["q_idx"], st["w"], with_selection=True)
        o2, i2, c2 = d_paged.run(st["q"], st["q_idx"], st["w"], with_selection=True)
        torch.cuda.synchronize()
        assert d_flat.device_error() == ("QSA_OK", 0)
        assert d_paged.device_error() == ("QSA_OK", 0)
        assert torch.equal(c1, c2)
        assert torch.equal(i1, i2)
        assert torch.equal(_bits(o1), _bits(o2))
    # the two caches hold the same blocks and running sums, bit for bit
    for b in range(spec.batch):
        L = flat.h_len[b]
        assert paged.h_len[b] == L
        assert torch.equal(_bits(flat.kbar_rows(b, L // 4)), _bits(paged.kbar_rows(b, L // 4)))
        assert torch.equal(flat.kbar_partial[b].cpu(), paged.kbar_partial[b].cpu())
        for g in range(2):
            for a, p in zip(flat.kv_rows(b, g, L), paged.kv_rows(b, g, L)):
                assert torch.equal(_bits(a), _bits(p))


def test_paged_matches_contiguous_small_pages():
    # 512-token pages; contexts and bulk-append chunks (700 tokens) cross page boundaries at
    # arbitrary offsets; the decode steps append across a page boundary for sequence 2
    spec = W.small_decode_spec(batch=4, context=(1000, 1001, 2046, 3001), capacity=4096, topk=64,
                               steps=4, seed=31)
    _paged_vs_contiguous(spec, page_tokens=512, steps=spec.steps, chunk=700)


def test_paged_matches_contiguous_one_page_per_sequence():
    spec = W.small_decode_spec(batch=3, context=(3000, 3500, 4001), capacity=4096, topk=128,
                               steps=2, seed=32)
    _paged_vs_contiguous(spec, page_tokens=4096, steps=spec.steps, chunk=1024, seed=5)


def test_paged_decode_matches_oracle():
    spec = W.small_decode_spec(batch=4, context=(1000, 1023, 1535, 2047), capacity=2560, topk=64,
                               steps=3, seed=33)
    res = _decode_session(spec, check_seqs=[0, 1, 2, 3], steps=spec.steps,
                          cache_fn=lambda s: _paged(s, 512, seed=7))
    assert len(res) == 4 * spec.steps


def test_paged_matches_contiguous_256k_contexts():
    # the headline decode shape (262,140..262,143 tokens of context) with 4,096-token pages,
    # on 8 sequences: 64 pages per sequence in a shuffled pool
    spec = W.decode_spec("decode256k")
    spec.batch = 8
    spec.context = [262140 + (i % 4) for i in range(spec.batch)]
    _paged_vs_contiguous(spec, page_tokens=4096, steps=1, chunk=16384, seed=11)


def test_paged_out_of_range_page_is_reported():
    # a page table entry past the pool, for a page the sequence has reached: the decode reads
    # zeros there (TMA fill) and records QSA_ERR_DEVICE instead of touching memory outside it
    spec = W.small_decode_spec(batch=2, context=(1500, 1700), capacity=2048, topk=64, steps=1,
                               seed=34)
    k, v, ki = W.decode_context(spec, device=DEV)
    cache = _paged(spec, 512, seed=3)
    _fill(cache, spec, k, v, ki, 1024)
    st = W.decode_step(spec, 0, device=DEV)
    cache.append(st["k"], st["v"], st["k_idx"])
    cache.page_table[1, 1] = cache.pool_pages + 7
    dec = qsa.Decoder(cache, spec.topk)
    dec.run(st["q"], st["q_idx"], st["w"])
    torch.cuda.synchronize()
    assert dec.device_error()[0] == "QSA_ERR_DEVICE"
