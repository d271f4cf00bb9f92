"""The page-printed constants agree with the oracle's geometry and the workloads."""
import json
import os

import oracle
from block_sparse_attention_40_b200 import workloads as W

GOLD = os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")


def test_page_constants():
    g = json.load(open(GOLD))
    c = oracle.constants()
    assert c["block"] == g["block_tokens"]["value"]
    assert c["num_heads"] == g["query_heads"]["value"]
    assert c["num_kv_heads"] == g["kv_heads"]["value"]
    assert g["budget_blocks"]["value"] * g["block_tokens"]["value"] == g["budget_tokens"]["value"]
    spec = W.decode_spec("decode256k")
    assert spec.capacity == g["native_context"]["value"] and spec.topk == g["budget_blocks"]["value"]
    assert max(spec.context) + 1 <= g["native_context"]["value"]
    spec = W.decode_spec("decode1m")
    assert spec.capacity >= g["extended_context_approx"]["value"]
