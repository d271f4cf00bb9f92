"""Pins of the oracle's block compression (fp32 mean in a fixed order, bf16 RNE store).

* hand-derived round-to-nearest-even cases (values worked out below, not computed by
  the oracle);
* exact means on integer inputs;
* torch's own IEEE fp32 CPU additions and fp32 -> bf16 cast as an independent
  implementation of the same definition on random inputs;
* the sign of zero survives (-0 + -0 + -0 + -0 = -0).
"""
import numpy as np
import torch

import oracle
from block_sparse_attention_40_b200 import workloads as W


def _bits(x):
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(
        np.uint16)


def _kbar_of_block(vals4):
    """vals4: 4 token values (same in every dim) -> the oracle's compressed value."""
    kid = np.repeat(_bits(vals4)[:, None], 64, axis=1)
    kb = oracle.compress(kid, np.array([0, 4]))
    return kb[0]


def test_rne_hand_cases():
    # 1 + 2^-8: mean 0.25 + 2^-10 is half an ulp (2^-9) above 0.25 -> ties to even: 0.25
    assert np.all(_kbar_of_block([1.0, 2.0 ** -8, 0.0, 0.0]) == _bits([0.25])[0])
    # 1 + 3*2^-8: mean 0.25 + 3*2^-10 lies halfway between 0.25+2^-9 (odd) and
    # 0.25+2^-8 (even) -> 0.25 + 2^-8
    assert np.all(_kbar_of_block([1.0, 2.0 ** -7, 2.0 ** -8, 0.0]) ==
                  _bits([0.25 + 2.0 ** -8])[0])
    # just above a tie rounds up: 1 + 2^-8 + 2^-16 -> 0.25 + 2^-9
    assert np.all(_kbar_of_block([1.0, 2.0 ** -8, 2.0 ** -16, 0.0]) ==
                  _bits([0.25 + 2.0 ** -9])[0])
    # the fixed order matters: ((1e8 + 1) - 1e8) + 1 in fp32 is 1 (1e8 + 1 rounds to 1e8)
    big = float(torch.tensor(1e8).to(torch.bfloat16))
    assert np.all(_kbar_of_block([big, 1.0, -big, 1.0]) == _bits([0.25])[0])


def test_negative_zero_kept():
    kb = _kbar_of_block([-0.0, -0.0, -0.0, -0.0])
    assert np.all(kb == 0x8000)
    kb = _kbar_of_block([0.0, -0.0, -0.0, -0.0])
    assert np.all(kb == 0x0000)


def test_integer_means_exact():
    p = W.custom_prefill([1001, 14], topk=4, kind="int", seed=3)
    cu = p.cu_seqlens.numpy().astype(np.int64)
    kb = oracle.compress(W.bits(p.k_idx), cu)
    got = torch.from_numpy(kb.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    parts = []
    for lo, hi in [(0, 1001), (1001, 1015)]:
        L = hi - lo
        parts.append(p.k_idx[lo:lo + 4 * (L // 4)].to(torch.float64).reshape(-1, 4, 64).mean(1))
    assert torch.equal(got, torch.cat(parts))


def test_matches_torch_fp32_and_bf16_cast():
    p = W.custom_prefill([4096 + 3, 777], topk=4, kind="normal", seed=21)
    cu = p.cu_seqlens.numpy().astype(np.int64)
    kb = oracle.compress(W.bits(p.k_idx), cu)
    parts = []
    for lo, hi in [(0, 4099), (4099, 4876)]:
        L = hi - lo
        x = p.k_idx[lo:lo + 4 * (L // 4)].to(torch.float32).reshape(-1, 4, 64)
        s = x[:, 0] + x[:, 1]
        s = s + x[:, 2]
        s = s + x[:, 3]
        parts.append((s * 0.25).to(torch.bfloat16))
    want = torch.cat(parts).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(kb, want)


def test_order_sensitive_inputs_match_torch_fp32():
    # tokens (a, x, -a, y) with |a| = 2^20: the fp32 rounding of a + x depends on the
    # summation order, so a wrong order changes the stored bf16 value for most blocks
    g = torch.Generator().manual_seed(5)
    nb = 512
    a = torch.where(torch.rand((nb, 64), generator=g) < 0.5, -1.0, 1.0) * 2.0 ** 20
    x = torch.randn((nb, 64), generator=g)
    y = torch.randn((nb, 64), generator=g)
    tok = torch.stack([a, x, -a, y], dim=1).to(torch.bfloat16)          # [nb, 4, 64]
    kb = oracle.compress(tok.reshape(-1, 64).view(torch.int16).numpy().view(np.uint16),
                         np.array([0, 4 * nb]))
    f = tok.to(torch.float32)
    s = ((f[:, 0] + f[:, 1]) + f[:, 2]) + f[:, 3]
    want = (s * 0.25).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(kb, want)
    # and the order really matters for these inputs
    s_other = ((f[:, 0] + f[:, 1]) + f[:, 3]) + f[:, 2]
    other = (s_other * 0.25).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (other != want).mean() > 0.5
