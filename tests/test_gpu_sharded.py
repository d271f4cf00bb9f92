"""GPU parity of the context-sharded decode (one GPU standing in for the ranks).

A batch's contexts are cut into shards (caches of consecutive tokens on 512-token
boundaries); every shard proposes its top-k candidates, the merge keeps the top-k of their
union, every shard attends its part of the selection, and the partials are merged by
log-sum-exp.  The selection must equal the one qsa_decode makes over the whole context bit
for bit (the shards' scores are the same fp32 values), and the output must match the oracle
(and the whole-context decode) within the decode tolerance."""
import numpy as np
import pytest
import torch

import oracle
import block_sparse_attention_40_b200 as qsa
from block_sparse_attention_40_b200 import binding as B
from block_sparse_attention_40_b200 import sharded as S
from block_sparse_attention_40_b200 import workloads as W
from tests.gpu_helpers import MAX_ABS, REL_L2, compare_outputs, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda:0"


def _run(spec, shard_tokens, steps=1, device_gen=False, check_seqs=()):
    gen = DEV if device_gen else "cpu"
    kc, vc, kic = W.decode_context(spec, device=gen)
    full = qsa.KVCache(spec.batch, spec.capacity, DEV, zero=False)
    nsh = spec.capacity // shard_tokens
    shards = [qsa.KVCache(spec.batch, shard_tokens, DEV, zero=False) for _ in range(nsh)]
    lmax = max(spec.context)
    for c0 in range(0, lmax, 16384):
        c1 = min(lmax, c0 + 16384)
        kk, vv, ki = (x[:, c0:c1].to(DEV).contiguous() for x in (kc, vc, kic))
        full.append(kk, vv, ki, counts=[max(0, min(c1, L) - c0) for L in spec.context])
        for r, sh in enumerate(shards):
            t0 = r * shard_tokens
            a, e = max(c0, t0), min(c1, t0 + shard_tokens)
            if a >= e:
                continue
            cnt = S.shard_counts(spec.context, t0, shard_tokens, c0, c1)
            if any(cnt):
                sh.append(kk[:, a - c0:e - c0].contiguous(), vv[:, a - c0:e - c0].contiguous(),
                          ki[:, a - c0:e - c0].contiguous(), counts=cnt)
    dec = qsa.Decoder(full, spec.topk)
    sdec = [B.ShardDecoder(sh, r * shard_tokens // 4, spec.topk) for r, sh in enumerate(shards)]
    glen = torch.tensor(spec.context, dtype=torch.int32, device=DEV)
    ctx = {b: (kc[b, :spec.context[b]].cpu(), vc[b, :spec.context[b]].cpu(),
               kic[b, :spec.context[b]].cpu()) for b in check_seqs}
    lens = list(spec.context)
    for step in range(steps):
        st = W.decode_step(spec, step, device=gen)
        k1, v1, ki1 = (st[n].to(DEV) for n in ("k", "v", "k_idx"))
        full.append(k1, v1, ki1)
        for r, sh in enumerate(shards):
            # every sequence's new token is at position lens[b]: append it where it falls
            cnt = [1 if r * shard_tokens <= lens[b] < (r + 1) * shard_tokens else 0
                   for b in range(spec.batch)]
            if any(cnt):
                sh.append(k1, v1, ki1, counts=cnt)
        lens = [L + 1 for L in lens]
        glen.copy_(torch.tensor(lens, dtype=torch.int32))
        q, qi, w = (st[n].to(DEV) for n in ("q", "q_idx", "w"))
        ref, r_idx, r_cnt = dec.run(q, qi, w, with_selection=True)
        out, s_idx, s_cnt = S.decode_step_local(sdec, q, qi, w, glen, spec.capacity // 4)
        torch.cuda.synchronize()
        assert dec.device_error() == ("QSA_OK", 0)
        for sd in sdec:
            assert sd.device_error() == ("QSA_OK", 0)
        # the selection is the whole-context selection, bit for bit
        assert torch.equal(s_cnt, r_cnt)
        assert torch.equal(s_idx, r_idx)
        # the output agrees with the whole-context decode and with the oracle
        a, b = out.double().cpu(), ref.double().cpu()
        assert (a - b).abs().max().item() <= MAX_ABS
        assert ((a - b).norm() / b.norm()).item() <= REL_L2
        for bb in check_seqs:
            kt, vt, kit = ctx[bb]
            kt = torch.cat([kt, st["k"][bb].cpu()])
            vt = torch.cat([vt, st["v"][bb].cpu()])
            kit = torch.cat([kit, st["k_idx"][bb].cpu()])
            ctx[bb] = (kt, vt, kit)
            L = kt.shape[0]
            cu = np.array([0, L], dtype=np.int64)
            kbar = oracle.compress(W.bits(kit), cu)
            _, _, _, o_out = oracle.rows(
                q_rows=W.bits(st["q"][bb:bb + 1]), q_idx_rows=W.bits(st["q_idx"][bb:bb + 1]),
                w_rows=W.bits(st["w"][bb:bb + 1]), row_seq=np.zeros(1, np.int64),
                row_pos=np.array([L - 1]), k=W.bits(kt), v=W.bits(vt), kbar=kbar,
                cu_seqlens=cu, topk=spec.topk, forced_idx=s_idx[bb:bb + 1].cpu().numpy(),
                forced_cnt=s_cnt[bb:bb + 1].cpu().numpy())
            compare_outputs(out[bb:bb + 1], o_out)
    return lens


def test_sharded_small_four_shards():
    # contexts ending in every shard, one ending right at a shard boundary, one short context
    spec = W.small_decode_spec(batch=5, context=(1500, 2047, 2048, 5000, 7000), capacity=8192,
                               topk=128, steps=3, seed=51)
    _run(spec, shard_tokens=2048, steps=3, check_seqs=(1, 4))


def test_sharded_short_contexts_dense():
    # fewer candidates than the budget: the selection is every complete block
    spec = W.small_decode_spec(batch=3, context=(100, 511, 900), capacity=1024, topk=512,
                               steps=2, seed=52)
    _run(spec, shard_tokens=512, steps=2, check_seqs=(2,))


@pytest.mark.slow
@pytest.mark.parametrize("nshards", [2, 4])
def test_sharded_1m_context(nshards):
    # the extended-context case: 4 sequences at 1,048,509..1,048,512 tokens, cut into 2 or 4
    # shards of the 1M capacity
    spec = W.decode_spec("decode1m")
    _run(spec, shard_tokens=spec.capacity // nshards, steps=2, device_gen=True, check_seqs=(0,))
