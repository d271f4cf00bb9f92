"""GPU parity of the Gated DeltaNet layer (qsa_gated_deltanet) against the oracle."""
import numpy as np
import pytest
import torch

import block_sparse_attention_40_b200 as qsa
from block_sparse_attention_40_b200 import workloads as W
from oracle.gated_deltanet import gated_deltanet as oracle_gdn
from tests.gpu_helpers import needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda:0"
MAX_ABS, REL_L2 = 2e-2, 5e-3      # bf16 outputs
STATE_ABS = 1e-3                  # fp32 final states


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _check(w, heads_seqs=None):
    d = w.to(DEV)
    out, state = qsa.gated_deltanet(d.q, d.k, d.v, d.log_alpha, d.beta, w.cu_seqlens,
                                    with_state=True)
    torch.cuda.synchronize()
    cu = [int(x) for x in w.cu_seqlens]
    pairs = heads_seqs or [(s, h) for s in range(len(cu) - 1) for h in range(w.q.shape[1])]
    errs = []
    for s, h in pairs:
        a, b = cu[s], cu[s + 1]
        ref, ref_state = oracle_gdn(_f64(w.q[a:b, h:h + 1]), _f64(w.k[a:b, h:h + 1]),
                                    _f64(w.v[a:b, h:h + 1]), _f64(w.log_alpha[a:b, h:h + 1]),
                                    _f64(w.beta[a:b, h:h + 1]), [0, b - a], with_state=True)
        got = _f64(out[a:b, h:h + 1])
        if b > a:
            err = np.abs(got - ref).max()
            rel = np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30)
            assert err <= MAX_ABS and rel <= REL_L2, (s, h, err, rel)
            errs.append(rel)
        gs = state[s, h].cpu().numpy().astype(np.float64)
        assert np.abs(gs - ref_state[0, 0]).max() <= STATE_ABS, (s, h)
    assert torch.isfinite(out.float()).all()
    return errs


def test_ragged_lengths_around_the_chunk():
    # lengths below, at and around the 64-token chunk, several chunks, and empty sequences
    w = W.gated_deltanet([1, 63, 64, 65, 0, 200, 1000, 0], heads=3, seed=1)
    _check(w)


def test_strong_decay_and_small_writes():
    w = W.gated_deltanet([777, 130], heads=2, seed=2, gate=(0.3, 0.8))
    w.beta.mul_(0.1)
    _check(w)


def test_reset_gates():
    # alpha = 0 every 37 tokens: the state restarts inside chunks and at their edges
    w = W.gated_deltanet([500, 129], heads=2, seed=3, reset_every=37)
    _check(w)


def test_no_writes_gives_zero():
    w = W.gated_deltanet([300], heads=2, seed=4)
    w.beta.zero_()
    d = w.to(DEV)
    out = qsa.gated_deltanet(d.q, d.k, d.v, d.log_alpha, d.beta, w.cu_seqlens)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0


@pytest.mark.slow
def test_bench_workload_sampled_heads():
    # the bench's size (8 sequences x 8,192 tokens, 16 heads), oracle on sampled pairs
    w = W.gated_deltanet([8192] * 8, heads=16, seed=7)
    _check(w, heads_seqs=[(0, 0), (3, 7), (7, 15)])


def test_invalid_arguments_are_refused():
    w = W.gated_deltanet([10], heads=2, seed=5).to(DEV)
    with pytest.raises(qsa.QSAError):
        # cu_seqlens not starting at 0
        qsa.gated_deltanet(w.q, w.k, w.v, w.log_alpha, w.beta, torch.tensor([1, 10]))
