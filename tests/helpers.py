"""Shared test helpers: input conversion only (no arithmetic of the method)."""
from __future__ import annotations

import numpy as np
import torch

from block_sparse_attention_40_b200 import workloads as W


def prefill_bits(p: W.Prefill) -> dict:
    """The workload's tensors as raw bf16 bit patterns (numpy uint16) for the oracle."""
    return dict(q=W.bits(p.q), k=W.bits(p.k), v=W.bits(p.v), q_idx=W.bits(p.q_idx),
                k_idx=W.bits(p.k_idx), w=W.bits(p.w),
                cu_seqlens=p.cu_seqlens.numpy().astype(np.int64), topk=p.topk)


def to_lists(t: torch.Tensor):
    return t.to(torch.float64).cpu().tolist()


def bf16_from_float(x) -> torch.Tensor:
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def dense_gqa_reference(q, k, v, mask):
    """fp64 softmax attention via torch's scaled_dot_product_attention (library routine).

    q [T,24,128], k/v [T,2,128] (any float dtype), mask [T,T] bool (True = attend).
    Query head h reads key/value head h // 12.
    """
    qd = q.to(torch.float64).permute(1, 0, 2)                     # [24, T, 128]
    kd = k.to(torch.float64).permute(1, 0, 2).repeat_interleave(12, dim=0)
    vd = v.to(torch.float64).permute(1, 0, 2).repeat_interleave(12, dim=0)
    out = torch.nn.functional.scaled_dot_product_attention(qd, kd, vd, attn_mask=mask)
    return out.permute(1, 0, 2)                                    # [T, 24, 128]
