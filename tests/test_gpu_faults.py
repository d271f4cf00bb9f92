"""Device-side failure reporting, exercised without faulting the GPU.

* A bounded wait that runs out: the prefill call's testing hook (qsa_params.debug_fault = 1)
  makes one attention tile post nothing for its first key chunk and gives that tile's MMA
  warp a 1 ms wait limit.  The wait gives up, the call reports QSA_ERR_TIMEOUT at that wait's
  site, every other tile's output is still right, and a normal call right after succeeds
  (the unwinding tile drained its copies and freed its tensor memory).
* Stale host lengths: a decode call whose host copy of the lengths is one indexer tile
  short of the device lengths covers fewer compressed blocks than the device holds; the
  indexer reports QSA_ERR_DEVICE (site 207) instead of letting the top-k read unwritten
  scores, and the next call with correct lengths succeeds.
"""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_40_b200 as qsa
from block_sparse_attention_40_b200 import workloads as W
from tests.gpu_helpers import compare_outputs, needs_gpu, prefill_oracle_check

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda:0"


def test_attention_wait_timeout_is_reported_and_unwound():
    p = W.prefill("tiny")
    d = p.to(DEV)
    T = p.total_tokens
    ctx = qsa.Prefill(p.cu_seqlens, DEV, p.topk, debug_fault=1)
    idx, cnt = ctx.select(d.q_idx, d.k_idx, d.w)
    out = ctx.run(d.q, d.k, d.v, d.q_idx, d.k_idx, d.w)
    torch.cuda.synchronize()
    assert ctx.device_error() == ("QSA_ERR_TIMEOUT", 23)
    # the faulted tile is the last one (tokens 250..255 at 10 tokens per tile), KV head 0:
    # every other (token, head) is still exact to the oracle
    last0 = (T - 1) // 10 * 10
    b = {n: W.bits(getattr(p, n)) for n in ("q", "k", "v", "q_idx", "k_idx", "w")}
    cu = p.cu_seqlens.numpy().astype(np.int64)
    gi, gc = idx.cpu().numpy(), cnt.cpu().numpy()
    _, _, _, o_out, _ = oracle.prefill(q=b["q"], k=b["k"], v=b["v"], q_idx=b["q_idx"],
                                       k_idx=b["k_idx"], w=b["w"], cu_seqlens=cu, topk=p.topk,
                                       forced_idx=gi, forced_cnt=gc)
    g = out.double().cpu().numpy()
    compare_outputs(g[:last0], o_out[:last0])
    compare_outputs(g[last0:, 12:], o_out[last0:, 12:])
    # a normal call right after runs clean and matches the oracle everywhere
    ctx2 = qsa.Prefill(p.cu_seqlens, DEV, p.topk)
    out2 = ctx2.run(d.q, d.k, d.v, d.q_idx, d.k_idx, d.w)
    torch.cuda.synchronize()
    assert ctx2.device_error() == ("QSA_OK", 0)
    prefill_oracle_check(p, idx, cnt, out2, np.arange(T))


def test_stale_host_lengths_are_reported():
    # one sequence: 70,001 tokens after the append -> 17,500 candidate blocks = 137 indexer
    # tiles of 128; host lengths 512 tokens short size the grid for 136 tiles
    spec = W.small_decode_spec(batch=1, context=(70000,), capacity=70100, topk=64, steps=1,
                               seed=41)
    kc, vc, kic = W.decode_context(spec)
    cache = qsa.KVCache(1, spec.capacity, DEV)
    cache.append(kc.to(DEV), vc.to(DEV), kic.to(DEV))
    st = W.decode_step(spec, 0)
    cache.append(st["k"].to(DEV), st["v"].to(DEV), st["k_idx"].to(DEV))
    dec = qsa.Decoder(cache, spec.topk)
    q, qi, w = st["q"].to(DEV), st["q_idx"].to(DEV), st["w"].to(DEV)
    true_len = list(cache.h_len)
    assert true_len == [70001]
    cache.h_len = [true_len[0] - 512]
    dec.run(q, qi, w)
    torch.cuda.synchronize()
    assert dec.device_error() == ("QSA_ERR_DEVICE", 207)
    cache.h_len = true_len
    out = dec.run(q, qi, w)
    torch.cuda.synchronize()
    assert dec.device_error() == ("QSA_OK", 0)
    assert torch.isfinite(out.float()).all()
