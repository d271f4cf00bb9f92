"""Pins of the Gated DeltaNet oracle (oracle/gated_deltanet.py) against closed forms.

Each pin is a case whose result follows from the recurrence by hand; planted mistakes in
copies of the recurrence must each fail at least one pin.
"""
import numpy as np
import pytest

from oracle.gated_deltanet import gated_deltanet

D = 8


def _orth(n, seed):
    q, _ = np.linalg.qr(np.random.default_rng(seed).standard_normal((D, D)))
    return q[:n]          # n orthonormal rows


def _one(impl, q, k, v, la, b):
    """One sequence, one head: arrays [T][d] and [T]."""
    T = len(k)
    return impl(q[:, None], k[:, None], v[:, None], la[:, None], b[:, None], [0, T])[:, 0]


# ---- pins: each returns True when the implementation satisfies it -------------------
def pin_orthonormal_retrieval(impl):
    # alpha = 1, beta = 1, orthonormal keys: querying key j after it was written returns v_j
    rng = np.random.default_rng(1)
    k = _orth(6, 2)
    v = rng.standard_normal((6, D))
    q = np.stack([k[t // 2] for t in range(6)])     # each query is an earlier (or own) key
    o = _one(impl, q, k, v, np.zeros(6), np.ones(6))
    want = np.stack([v[t // 2] for t in range(6)])
    return np.allclose(o, want, atol=1e-12)


def pin_rewrite_same_key(impl):
    # the key e written twice (gate a before the second write, strength b): querying e
    # returns (1 - b) a v1 + b v2, and with b = 1 exactly v2 (the delta rule overwrites)
    e = _orth(1, 3)[0]
    rng = np.random.default_rng(4)
    v = rng.standard_normal((2, D))
    ok = True
    for a, b in ((0.7, 1.0), (0.5, 0.3), (1.0, 0.6)):
        o = _one(impl, np.stack([e, e]), np.stack([e, e]), v, np.log([1.0, a]),
                 np.array([1.0, b]))
        ok &= np.allclose(o[1], (1 - b) * a * v[0] + b * v[1], atol=1e-12)
    return ok


def pin_no_writes(impl):
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((9, D)) for _ in range(3))
    o = _one(impl, q, k, v, np.log(rng.uniform(0.2, 1.0, 9)), np.zeros(9))
    return np.allclose(o, 0.0)


def pin_reset_gates(impl):
    # alpha = 0 forgets everything: o_t = beta_t (k_t . q_t) v_t
    rng = np.random.default_rng(6)
    q, k, v = (rng.standard_normal((7, D)) for _ in range(3))
    b = rng.uniform(0.1, 0.9, 7)
    o = _one(impl, q, k, v, np.full(7, -np.inf), b)
    want = (b * np.einsum("td,td->t", k, q))[:, None] * v
    return np.allclose(o, want, atol=1e-12)


def pin_single_write(impl):
    # only token j writes: o_t = (prod of alpha after j up to t) beta_j (k_j . q_t) v_j
    rng = np.random.default_rng(7)
    T, j = 10, 3
    q, k, v = (rng.standard_normal((T, D)) for _ in range(3))
    a = rng.uniform(0.3, 1.0, T)
    b = np.zeros(T)
    b[j] = 0.8
    o = _one(impl, q, k, v, np.log(a), b)
    want = np.zeros((T, D))
    for t in range(j, T):
        want[t] = np.prod(a[j + 1:t + 1]) * b[j] * (k[j] @ q[t]) * v[j]
    return np.allclose(o, want, atol=1e-12)


def pin_gated_linear_attention(impl):
    # orthogonal keys and beta = 1: nothing to correct, so the layer is gated linear attention
    rng = np.random.default_rng(8)
    T = D
    k = _orth(T, 9)
    q, v = rng.standard_normal((T, D)), rng.standard_normal((T, D))
    a = rng.uniform(0.5, 1.0, T)
    o, st = impl(q[:, None], k[:, None], v[:, None], np.log(a)[:, None], np.ones((T, 1)),
                 [0, T], with_state=True)
    want = np.zeros((T, D))
    S = np.zeros((D, D))
    for t in range(T):
        for j in range(t + 1):
            want[t] += np.prod(a[j + 1:t + 1]) * (k[j] @ q[t]) * v[j]
    for j in range(T):
        S += np.prod(a[j + 1:]) * np.outer(v[j], k[j])
    return np.allclose(o[:, 0], want, atol=1e-12) and np.allclose(st[0, 0], S, atol=1e-12)


def pin_sequences_independent(impl):
    # packed sequences start from a zero state: two sequences packed equal each run alone
    rng = np.random.default_rng(10)
    T0, T1, H = 5, 4, 2
    q, k, v = (rng.standard_normal((T0 + T1, H, D)) for _ in range(3))
    la, b = np.log(rng.uniform(0.5, 1.0, (T0 + T1, H))), rng.uniform(0.2, 0.9, (T0 + T1, H))
    both = impl(q, k, v, la, b, [0, T0, T0 + T1])
    first = impl(q[:T0], k[:T0], v[:T0], la[:T0], b[:T0], [0, T0])
    second = impl(q[T0:], k[T0:], v[T0:], la[T0:], b[T0:], [0, T1])
    return np.allclose(both, np.concatenate([first, second]), atol=1e-12)


PINS = [pin_orthonormal_retrieval, pin_rewrite_same_key, pin_no_writes, pin_reset_gates,
        pin_single_write, pin_gated_linear_attention, pin_sequences_independent]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin):
    assert pin(gated_deltanet)


# ---- planted mistakes: each must fail at least one pin ---------------------------------
def _mutant(kind):
    def impl(q, k, v, log_alpha, beta, cu_seqlens, with_state=False):
        q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
        la, b = np.asarray(log_alpha, dtype=np.float64), np.asarray(beta, dtype=np.float64)
        cu = [int(x) for x in cu_seqlens]
        T, H, dk = k.shape
        out = np.zeros((T, H, v.shape[2]))
        states = np.zeros((len(cu) - 1, H, v.shape[2], dk))
        for h in range(H):
            S = np.zeros((v.shape[2], dk))
            for s in range(len(cu) - 1):
                if kind != "state_carried_over":
                    S = np.zeros((v.shape[2], dk))
                for t in range(cu[s], cu[s + 1]):
                    a = 1.0 if kind == "no_decay" else np.exp(la[t, h])
                    prev = S
                    S = a * S
                    sk = (prev if kind == "decay_missing_in_correction" else S) @ k[t, h]
                    sign = 1.0 if kind == "correction_sign" else -1.0
                    u = b[t, h] * (v[t, h] + sign * sk)
                    upd = np.outer(k[t, h], u) if kind == "outer_transposed" else np.outer(u, k[t, h])
                    if kind == "output_before_write":
                        out[t, h] = S @ q[t, h]
                    S = S + upd
                    if kind != "output_before_write":
                        out[t, h] = S @ q[t, h]
                states[s, h] = S
        return (out, states) if with_state else out
    return impl


MUTANTS = ["no_decay", "decay_missing_in_correction", "correction_sign", "outer_transposed",
           "output_before_write", "state_carried_over"]


@pytest.mark.parametrize("kind", MUTANTS)
def test_planted_mistake_is_caught(kind):
    impl = _mutant(kind)
    assert not all(pin(impl) for pin in PINS), kind


def test_unmutated_copy_passes_every_pin():
    # the mutant harness itself, with no mistake planted, satisfies every pin
    assert all(pin(_mutant("none")) for pin in PINS)
