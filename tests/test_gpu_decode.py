"""GPU parity of QSA decode (append, then steps a2, a3, a6) against the oracle.

The oracle evaluates the new token as row p = len-1 of the sequence made of the context
plus every appended token (token-major), so decode is checked against the same definition
as prefill."""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_40_b200 as qsa
from block_sparse_attention_40_b200 import workloads as W
from tests.gpu_helpers import compare_outputs, compare_selection, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda:0"


def _oracle_row(k_tok, v_tok, kidx_tok, q, q_idx, w, topk, forced=None):
    """k_tok/v_tok [L,2,128], kidx_tok [L,64] (bf16 CPU), query of row L-1."""
    L = k_tok.shape[0]
    cu = np.array([0, L], dtype=np.int64)
    kbar = oracle.compress(W.bits(kidx_tok), cu)
    fi = fc = None
    if forced is not None:
        fi, fc = forced
    idx, cnt, kth, out = oracle.rows(q_rows=W.bits(q[None]), q_idx_rows=W.bits(q_idx[None]),
                                     w_rows=W.bits(w[None]), row_seq=np.zeros(1, np.int64),
                                     row_pos=np.array([L - 1]), k=W.bits(k_tok), v=W.bits(v_tok),
                                     kbar=kbar, cu_seqlens=cu, topk=topk, forced_idx=fi,
                                     forced_cnt=fc)
    return idx, cnt, kth, out, kbar


def _decode_session(spec, check_seqs, steps, splits=0, device_gen=False, ctx_fn=None,
                    step_fn=None, exact_sel=False, cache_fn=None, check_steps=None):
    """ctx_fn(k, v, k_idx) and step_fn(step dict) may reshape the seeded inputs (ties);
    exact_sel demands the oracle's selection itself (inputs whose scores are exact);
    cache_fn(spec) builds the cache (default: a contiguous KVCache); check_steps lists the
    steps compared with the oracle (default: every step)."""
    gen_dev = DEV if device_gen else "cpu"
    k_ctx, v_ctx, ki_ctx = W.decode_context(spec, device=gen_dev)
    if ctx_fn is not None:
        k_ctx, v_ctx, ki_ctx = ctx_fn(k_ctx, v_ctx, ki_ctx)
    cache = (cache_fn(spec) if cache_fn is not None
             else qsa.KVCache(spec.batch, spec.capacity, DEV, zero=False))
    # bulk fill in chunks with per-sequence counts
    lmax = max(spec.context)
    chunk = 16384
    for c0 in range(0, lmax, chunk):
        c1 = min(lmax, c0 + chunk)
        counts = [max(0, min(c1, L) - c0) for L in spec.context]
        cache.append(k_ctx[:, c0:c1].to(DEV).contiguous(), v_ctx[:, c0:c1].to(DEV).contiguous(),
                     ki_ctx[:, c0:c1].to(DEV).contiguous(), counts=counts)
    dec = qsa.Decoder(cache, spec.topk, splits)
    # host copies for the oracle (only the checked sequences)
    seqs = {b: (k_ctx[b, :spec.context[b]].cpu(), v_ctx[b, :spec.context[b]].cpu(),
                ki_ctx[b, :spec.context[b]].cpu()) for b in check_seqs}
    del k_ctx, v_ctx, ki_ctx
    added = {b: ([], [], []) for b in check_seqs}   # tokens appended since the last check
    results = []
    for step in range(steps):
        st = W.decode_step(spec, step, device=gen_dev)
        if step_fn is not None:
            st = step_fn(st)
        cache.append(st["k"].to(DEV), st["v"].to(DEV), st["k_idx"].to(DEV))
        out, idx, cnt = dec.run(st["q"].to(DEV), st["q_idx"].to(DEV), st["w"].to(DEV),
                                with_selection=True)
        torch.cuda.synchronize()
        assert dec.device_error() == ("QSA_OK", 0)
        for b in check_seqs:
            for lst, key in zip(added[b], ("k", "v", "k_idx")):
                lst.append(st[key][b].cpu())
        if check_steps is not None and step not in check_steps:
            continue
        for b in check_seqs:
            kt, vt, kit = seqs[b]
            kt = torch.cat([kt] + added[b][0])
            vt = torch.cat([vt] + added[b][1])
            kit = torch.cat([kit] + added[b][2])
            seqs[b] = (kt, vt, kit)
            added[b] = ([], [], [])
            q, qi, w = st["q"][b].cpu(), st["q_idx"][b].cpu(), st["w"][b].cpu()
            o_idx, o_cnt, o_kth, _, kbar = _oracle_row(kt, vt, kit, q, qi, w, spec.topk)
            g_idx = idx[b:b + 1].cpu().numpy()
            g_cnt = cnt[b:b + 1].cpu().numpy()

            def score_fn(i, blocks, qi=qi, w=w, kbar=kbar, L=kt.shape[0]):
                return oracle.score_pairs(W.bits(qi[None]), W.bits(w[None]), kbar,
                                          np.array([0, L]), np.zeros(1, np.int64),
                                          np.zeros(len(blocks), np.int64), blocks)

            swaps = compare_selection(g_idx, g_cnt, o_idx, o_cnt, o_kth, score_fn,
                                      exact=exact_sel)
            _, _, _, o_out, _ = _oracle_row(kt, vt, kit, q, qi, w, spec.topk,
                                            forced=(g_idx, g_cnt))
            results.append((b, step, swaps) + compare_outputs(out[b:b + 1], o_out))
            # the compressed cache agrees bit for bit with the oracle's compression
            L = kt.shape[0]
            got = cache.kbar_rows(b, L // 4).contiguous().cpu().view(torch.int16).numpy().view(
                np.uint16)
            assert np.array_equal(got, kbar[:L // 4])
    return results


def test_small_decode_steps():
    spec = W.small_decode_spec()
    res = _decode_session(spec, check_seqs=[0, 1, 2, 3], steps=spec.steps)
    assert len(res) == 4 * spec.steps


@pytest.mark.parametrize("splits", [1, 3, 8])
def test_small_decode_splits(splits):
    spec = W.small_decode_spec(batch=2, context=(2045, 2046), capacity=2100, topk=128, steps=3,
                               seed=5)
    _decode_session(spec, check_seqs=[0, 1], steps=3, splits=splits)


def test_decode_short_contexts():
    # contexts shorter than the budget: decode equals dense attention over the prefix
    spec = W.small_decode_spec(batch=4, context=(0, 1, 3, 6), capacity=64, topk=512, steps=5,
                               seed=9)
    _decode_session(spec, check_seqs=[0, 1, 2, 3], steps=5)


def _int_ctx(k, v, ki):
    return k, v, torch.round(ki.float()).clamp(-3, 3).to(torch.bfloat16)


def _int_step(st):
    st = dict(st)
    st["k_idx"] = torch.round(st["k_idx"].float()).clamp(-3, 3).to(torch.bfloat16)
    st["q_idx"] = torch.round(st["q_idx"].float()).clamp(-3, 3).to(torch.bfloat16)
    st["w"] = torch.round(st["w"].float()).to(torch.bfloat16)
    return st


def _zero_w(st):
    st = dict(st)
    st["w"] = torch.zeros_like(st["w"])
    return st


def test_decode_integer_scores_ties():
    # small-integer indexer inputs: scores are exact multiples of 1/4 with many equal values
    # at the threshold, which the selection breaks toward lower block indices
    spec = W.small_decode_spec(batch=3, context=(5001, 5002, 6003), capacity=6100, topk=96,
                               steps=3, seed=21)
    _decode_session(spec, check_seqs=[0, 1, 2], steps=3, ctx_fn=_int_ctx, step_fn=_int_step,
                    exact_sel=True)


def test_decode_all_scores_equal():
    # w = 0: every score is 0, so the selection is the lowest topk block indices
    spec = W.small_decode_spec(batch=2, context=(4000, 4097), capacity=4200, topk=64, steps=2,
                               seed=22)
    res = _decode_session(spec, check_seqs=[0, 1], steps=2, step_fn=_zero_w, exact_sel=True)
    assert len(res) == 4


def test_decode_candidate_overflow_all_equal():
    # w = 0 on rows of more than 16384 complete blocks: the threshold bin holds every block,
    # more than the candidate buffer, so the rows take the full-row select
    spec = W.small_decode_spec(batch=2, context=(70001, 73000), capacity=73100, topk=512,
                               steps=1, seed=23)
    _decode_session(spec, check_seqs=[0, 1], steps=1, step_fn=_zero_w, exact_sel=True)


@pytest.mark.slow
def test_decode_256k_four_sequences():
    spec = W.decode_spec("decode256k")
    _decode_session(spec, check_seqs=[0, 1, 2, 3], steps=1, device_gen=True)


@pytest.mark.slow
def test_decode_1m_incremental():
    # the extended-context case as specified: 4 sequences at 1,048,509..1,048,512 tokens,
    # 64 consecutive append + decode steps, so that 16 blocks per sequence complete by
    # incremental compression; the oracle checks the first and the last step of every
    # sequence, including the compressed cache bit for bit after the last append
    spec = W.decode_spec("decode1m")
    assert spec.steps == 64
    res = _decode_session(spec, check_seqs=[0, 1, 2, 3], steps=spec.steps, device_gen=True,
                          check_steps={0, spec.steps - 1})
    assert len(res) == 8


def test_decode_batch_of_40_mixed_contexts():
    # 40 sequences of 3,000..4,799 tokens: each sequence keeps its own selection and output
    ctx = tuple(3000 + (373 * i) % 1800 for i in range(40))
    spec = W.small_decode_spec(batch=40, context=ctx, capacity=4900, topk=128, steps=2, seed=24)
    _decode_session(spec, check_seqs=[0, 17, 39], steps=2)


def test_decode_batch_of_40_all_scores_equal():
    ctx = tuple(2000 + (211 * i) % 900 for i in range(40))
    spec = W.small_decode_spec(batch=40, context=ctx, capacity=3000, topk=64, steps=1, seed=25)
    _decode_session(spec, check_seqs=[3, 38], steps=1, step_fn=_zero_w, exact_sel=True)


@pytest.mark.slow
def test_decode_batch_of_32_candidate_overflow():
    # rows of more than 16,384 blocks with all scores equal, in a batch of 32: the threshold
    # bin overflows the candidate buffer and the finish kernel takes the full-row select
    ctx = tuple(66000 + 7 * i for i in range(32))
    spec = W.small_decode_spec(batch=32, context=ctx, capacity=66400, topk=512, steps=1, seed=26)
    _decode_session(spec, check_seqs=[0, 31], steps=1, step_fn=_zero_w, exact_sel=True,
                    device_gen=True)
