"""The chunked form the Gated DeltaNet kernel evaluates, restated here in fp64 numpy, against the
token-by-token oracle (no GPU).  For a chunk entered with state S0, g the running sum of the
chunk's log gates (clamped at -87, as the kernel does) and A, M the gated key-key and
query-key products:
    U   = (I + diag(beta) A)^-1 diag(beta) (V - diag(e^g) K S0^T)   (forward substitution)
    O   = diag(e^g) Q S0^T + M U
    S_C = e^(g_C) S0 + (diag(e^(g_C - g)) U)^T K
This pins the algebra (and the clamp's reading of alpha = 0) independently of any kernel: a
wrong decay factor, sign or triangle shows here on the CPU."""
import numpy as np
import pytest

from block_sparse_attention_40_b200 import workloads as W
from oracle.gated_deltanet import gated_deltanet as oracle_gdn


def _chunked(q, k, v, la, beta, C, drop_state_decay=False):
    """One (sequence, head): q, k, v [T, d], la, beta [T]; returns outputs [T, d], final S."""
    T, d = q.shape
    S = np.zeros((v.shape[1], d))
    out = np.zeros((T, v.shape[1]))
    for t0 in range(0, T, C):
        sl = slice(t0, min(T, t0 + C))
        K, Q, V = k[sl], q[sl], v[sl]
        g = np.cumsum(np.maximum(la[sl], -87.0))
        b = beta[sl]
        n = len(g)
        tri = np.tril(np.ones((n, n)))
        dec = np.where(tri > 0, np.exp(np.where(tri > 0, g[:, None] - g[None, :], 0.0)), 0.0)
        A = dec * (K @ K.T) * (1 - np.eye(n))
        M = dec * (Q @ K.T)
        R = V - np.exp(g)[:, None] * (K @ S.T)
        U = np.zeros_like(R)
        for t in range(n):
            U[t] = b[t] * (R[t] - A[t, :t] @ U[:t])
        out[sl] = np.exp(g)[:, None] * (Q @ S.T) + M @ U
        carry = 1.0 if drop_state_decay else np.exp(g[-1])
        S = carry * S + (np.exp(g[-1] - g)[:, None] * U).T @ K
    return out, S


@pytest.mark.parametrize("chunk", [64, 16])
@pytest.mark.parametrize("case", ["plain", "resets", "strong_decay"])
def test_chunked_form_equals_the_recurrence(chunk, case):
    kw = {"plain": {}, "resets": {"reset_every": 37}, "strong_decay": {"gate": (0.3, 0.8)}}[case]
    w = W.gated_deltanet([200], heads=1, seed=11, **kw)
    f = lambda x: x.float().numpy().astype(np.float64)   # noqa: E731
    q, k, v, la, beta = (f(x) for x in (w.q, w.k, w.v, w.log_alpha, w.beta))
    ref, ref_state = oracle_gdn(q, k, v, la, beta, [0, 200], with_state=True)
    out, S = _chunked(q[:, 0], k[:, 0], v[:, 0], la[:, 0], beta[:, 0], chunk)
    # alpha = 0 is exp(-87) ~ 1.6e-38 in the chunked form: exact to well below 1e-12
    assert np.abs(out - ref[:, 0]).max() < 1e-9
    assert np.abs(S - ref_state[0, 0]).max() < 1e-9


def test_a_wrong_decay_is_caught():
    # the same check fails when the state's decay over the chunk is dropped
    w = W.gated_deltanet([130], heads=1, seed=12)
    f = lambda x: x.float().numpy().astype(np.float64)   # noqa: E731
    q, k, v, la, beta = (f(x) for x in (w.q, w.k, w.v, w.log_alpha, w.beta))
    ref = oracle_gdn(q, k, v, la, beta, [0, 130])
    out, _ = _chunked(q[:, 0], k[:, 0], v[:, 0], la[:, 0], beta[:, 0], 64, drop_state_decay=True)
    assert np.abs(out - ref[:, 0]).max() > 1e-3
