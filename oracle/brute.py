"""Pure-Python brute force of Qwen Sparse Attention for tiny inputs -- test infrastructure.

An independent second statement of the method, used only to pin the C oracle.  It
shares nothing with ``qsa_oracle.c`` beyond the definition it restates, and it takes a
different route at each step:

* fp32 sums are rounded with ``struct`` (IEEE single) and the bf16 rounding is done with
  exact ``fractions.Fraction`` arithmetic (nearest, ties to even), not bit tricks;
* block selection ranks every candidate by counting how many candidates beat it
  (higher score, or equal score and lower index), instead of sorting;
* attention loops over explicit token lists with Python floats (IEEE double).

Sources: "Long context became an architecture problem", section "Linear attention
carries the stream; sparse attention retrieves detail" (indexer over compressed
blocks, budget, uncompressed final block); axbrief "Shifting from Tokens to
Micro-Blocks" (24 query heads, 2 key-value heads); "Qwen3.8-Flash-Next Previews
Qwen4.x Architecture", FAQ (4-token micro-blocks).
"""
from __future__ import annotations

import math
import struct
from fractions import Fraction

H, HKV, G, D, HI, DI, B = 24, 2, 12, 128, 16, 64, 4


def bits_to_float(b: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (int(b) & 0xFFFF) << 16))[0]


def fl32(x: float) -> float:
    return struct.unpack("<f", struct.pack("<f", x))[0]


def bf16_round(x: float) -> float:
    """Nearest bf16 value to the float x, ties to even, computed with exact rationals."""
    if x == 0.0 or math.isinf(x) or math.isnan(x):
        return x
    fx = Fraction(x)
    a = abs(fx)
    e = math.floor(math.log2(a))
    # correct e so that 2**e <= a < 2**(e+1)
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 7)          # bf16 keeps 8 significant bits
    q, r = divmod(a, ulp)
    if r * 2 > ulp or (r * 2 == ulp and q % 2 == 1):
        q += 1
    val = q * ulp
    return float(val if fx > 0 else -val)


def compress_seq(kidx_tok):
    """kidx_tok: list over tokens of 64 floats -> list over complete blocks of 64 floats."""
    out = []
    for b in range(len(kidx_tok) // B):
        row = []
        for d in range(DI):
            s = kidx_tok[4 * b][d]
            for j in (1, 2, 3):
                s = fl32(s + kidx_tok[4 * b + j][d])
            row.append(bf16_round(fl32(s * 0.25)))
        out.append(row)
    return out


def score(qi, w, kb) -> float:
    tot = 0.0
    for h in range(HI):
        dot = math.fsum(qi[h][d] * kb[d] for d in range(DI))
        tot += w[h] * max(0.0, dot)
    return tot


def select(scores, k):
    n = len(scores)
    if n <= k:
        return list(range(n))
    chosen = []
    for b in range(n):
        beaten_by = sum(1 for c in range(n)
                        if scores[c] > scores[b] or (scores[c] == scores[b] and c < b))
        if beaten_by < k:
            chosen.append(b)
    assert len(chosen) == k
    return chosen


def attend(q, ks, vs, tokens):
    out = []
    for h in range(H):
        g = h // G
        logits = [math.fsum(q[h][d] * ks[j][g][d] for d in range(D)) / math.sqrt(D)
                  for j in tokens]
        m = max(logits)
        e = [math.exp(x - m) for x in logits]
        z = math.fsum(e)
        out.append([math.fsum(e[i] * vs[j][g][d] for i, j in enumerate(tokens)) / z
                    for d in range(D)])
    return out


def run_sequence(q, k, v, q_idx, k_idx, w, topk, rows=None):
    """All inputs are nested lists of floats for ONE sequence (token-major).

    Returns {t: (selected_blocks, out[24][128])} for each requested row t.
    """
    L = len(k_idx)
    kbar = compress_seq(k_idx)
    res = {}
    for t in (range(L) if rows is None else rows):
        c = t // B
        scores = [score(q_idx[t], w[t], kbar[b]) for b in range(c)]
        sel = select(scores, topk)
        tokens = [4 * b + j for b in sel for j in range(B)] + list(range(4 * c, t + 1))
        res[t] = (sel, attend(q[t], k, v, tokens) if q is not None else None)
    return res, kbar


def kth_ranked_score(scores, k):
    """Score of the candidate ranked k-th (exactly k-1 candidates beat it: a higher score,
    or an equal score at a lower index), or None when there are at most k candidates and
    nothing is left out.  This is the selection boundary: the lowest kept score."""
    n = len(scores)
    if n <= k:
        return None
    for b in range(n):
        beaten_by = sum(1 for c in range(n)
                        if scores[c] > scores[b] or (scores[c] == scores[b] and c < b))
        if beaten_by == k - 1:
            return scores[b]
    raise AssertionError("no candidate has rank k")


def row_scores(q_idx, k_idx, w, rows):
    """{t: [s(t, b) for every candidate block b < floor(t/4)]} for ONE sequence (nested
    lists of floats, token-major)."""
    kbar = compress_seq(k_idx)
    return {t: [score(q_idx[t], w[t], kbar[b]) for b in range(t // B)] for t in rows}
