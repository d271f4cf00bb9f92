"""CPU oracle of the Gated DeltaNet linear-attention layer -- test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may import this
module; the product library never does, and this module imports nothing from it.

The recurrence is stated token by token in fp64, exactly as written below, with no
chunking, blocking or reordering.  Per sequence and head, the state S (d_v x d_k) starts
at zero, and for each token t with gate alpha_t = exp(log_alpha_t) and writing strength
beta_t:

    S_t = alpha_t S_{t-1} + beta_t (v_t - alpha_t S_{t-1} k_t) k_t^T
    o_t = S_t q_t

("Long context became an architecture problem", section "Linear attention carries the
stream; sparse attention retrieves detail": Gated DeltaNet, a gated linear recurrence that
updates a compact state, alternates with the sparse attention layers; "Qwen3.8-Flash-Next
Previews Qwen4.x Architecture", section "Gated DeltaNet -- The Linear Attention Engine":
three of every four token-mixing layers.  The pages' table of the layer's parameters did not
survive extraction; the update above is the published gated delta rule, and q and k are
taken as given: any normalisation happens before the layer.)

parity pins: tests/test_oracle_gdn.py (closed forms: orthonormal keys, no writes, reset
gates, a single write, gated linear attention; and planted mistakes).
"""
from __future__ import annotations

import numpy as np


def gated_deltanet(q, k, v, log_alpha, beta, cu_seqlens, with_state=False):
    """Outputs [T][H][d_v] (fp64) of the recurrence above for packed sequences.

    q, k: [T][H][d_k]; v: [T][H][d_v]; log_alpha, beta: [T][H]; cu_seqlens: [S+1].
    With with_state, also returns the final state of every (sequence, head),
    [S][H][d_v][d_k].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    log_alpha = np.asarray(log_alpha, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    cu = [int(x) for x in cu_seqlens]
    T, H, dk = k.shape
    dv = v.shape[2]
    out = np.zeros((T, H, dv))
    states = np.zeros((len(cu) - 1, H, dv, dk))
    for s in range(len(cu) - 1):
        for h in range(H):
            S = np.zeros((dv, dk))
            for t in range(cu[s], cu[s + 1]):
                a = np.exp(log_alpha[t, h])
                S = a * S                                   # alpha_t S_{t-1}
                u = beta[t, h] * (v[t, h] - S @ k[t, h])    # beta_t (v_t - alpha_t S_{t-1} k_t)
                S = S + np.outer(u, k[t, h])
                out[t, h] = S @ q[t, h]
            states[s, h] = S
    return (out, states) if with_state else out
