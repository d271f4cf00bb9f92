"""Host-side logic of bench.py that needs no GPU: the algorithmic work it divides by, checked
against the oracle's own selection, and the rule that drops a DRAM-traffic figure once the
kernel sources it was captured on have changed."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from block_sparse_attention_40_b200 import workloads as W  # noqa: E402


def test_attention_flops_count_the_keys_the_oracle_attends():
    # selected-token FLOPs = 24 heads x 128 dims x 4 flops (QK and PV) per attended key, where
    # a row attends 4 keys per selected block plus the visible part of its own block
    T, k = 300, 8
    p = W.custom_prefill([T], topk=k, seed=3)
    b = {n: W.bits(getattr(p, n)) for n in ("q_idx", "k_idx", "w")}
    idx, cnt, _, _, _ = oracle.prefill(q=None, k=None, v=None, q_idx=b["q_idx"], k_idx=b["k_idx"],
                                       w=b["w"], cu_seqlens=np.array([0, T]), topk=k)
    t = np.arange(T)
    # the number of selected blocks is the budget or every complete block before the own one
    assert np.array_equal(cnt, np.minimum(k, t // 4))
    assert all((idx[r, :cnt[r]] >= 0).all() and (idx[r, cnt[r]:] == -1).all() for r in range(T))
    keys = int((4 * cnt + t % 4 + 1).sum())
    assert bench.prefill_attention_flops(T, k) == 24 * 128 * 4 * keys


def test_traffic_stamp_is_dropped_when_its_sources_change(monkeypatch):
    per_token, _, what = bench.NCU_TRAFFIC["prefill_attention"]
    monkeypatch.setitem(bench.NCU_TRAFFIC, "prefill_attention", (per_token, "0" * 64, what))
    value, why = bench.measured_traffic("prefill_attention", 65536)
    assert value is None and "changed" in why
    sha = bench.csrc_sha(bench.TRAFFIC_SOURCES["prefill_attention"])
    monkeypatch.setitem(bench.NCU_TRAFFIC, "prefill_attention", (per_token, sha, what))
    value, _ = bench.measured_traffic("prefill_attention", 65536)
    assert value == per_token * 65536
