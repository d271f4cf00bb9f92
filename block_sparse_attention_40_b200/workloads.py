"""Seeded synthetic inputs for QSA prefill and decode.

This module holds no step of the method's arithmetic: it only draws tensors.  Both the
CUDA path and the CPU oracle consume exactly the tensors drawn here (the oracle gets
their raw bf16 bit patterns).

Workloads (sizes from the workload list that this library is measured on; the pages
describe a 262,144-token native context extendable to 1M -- "Long context became an
architecture problem", "Open weights still require a compatible runtime"):

* ``tiny``    T=256, budget 16 blocks, N(0,1) inputs, w ~ U(0,1), 4 needle blocks.
* ``8k``      T=8,192, budget 512, N(0,1) inputs, 32 needle blocks.
* ``8k_int``  T=8,192, budget 512, integer indexer inputs: q_idx, k_idx in {-2..2},
              w in {1,2} (every score exact in fp32), no needles.
* ``64k``     T=65,536, budget 512; indexer keys and K drift per block: a per-dimension
              random walk with N(0, 0.05^2) steps per block (separate walks for k_idx
              and for K) plus N(0,1) noise; Q, V, q_idx ~ N(0,1); w ~ U(0,1).
* ``ragged``  8 sequences, lengths ~ U{1000..131071} redrawn while divisible by 4,
              N(0,1) inputs with 4 needle blocks per sequence.

Needles: "indexer keys equal to +3x the mean indexer query".  With zero-mean queries
that mean is ~0 and a needle would never win, so in needle workloads the indexer
queries are drawn as mu + N(0,1), mu a seeded +-0.5 sign vector (|mu|^2 = 16), and every
token of a needle block gets k_idx = 3 * (empirical mean of all q_idx vectors).

Decode workloads (``decode256k``: batch 64, prior context 262,140 + (i mod 4);
``decode1m``: batch 4, prior context 1,048,512 - i) draw the context and the per-step
tokens the same way as ``8k`` without needles.

Seeds: 1000 + workload id unless given.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

WORKLOAD_IDS = {"tiny": 0, "8k": 1, "8k_int": 1, "64k": 2, "decode256k": 3, "ragged": 4,
                "decode1m": 4}

NUM_HEADS, NUM_KV_HEADS, HEAD_DIM = 24, 2, 128
IDX_HEADS, IDX_DIM, BLOCK = 16, 64, 4


@dataclasses.dataclass
class Prefill:
    name: str
    q: torch.Tensor          # [T, 24, 128] bf16
    k: torch.Tensor          # [T, 2, 128]  bf16
    v: torch.Tensor          # [T, 2, 128]  bf16
    q_idx: torch.Tensor      # [T, 16, 64]  bf16
    k_idx: torch.Tensor      # [T, 64]      bf16
    w: torch.Tensor          # [T, 16]      bf16
    cu_seqlens: torch.Tensor  # [num_seqs+1] int32 (CPU)
    topk: int
    needles: dict            # seq -> sorted list of needle block indices

    @property
    def total_tokens(self) -> int:
        return int(self.cu_seqlens[-1])

    def to(self, device) -> "Prefill":
        kw = {f.name: getattr(self, f.name) for f in dataclasses.fields(self)}
        for n in ("q", "k", "v", "q_idx", "k_idx", "w"):
            kw[n] = kw[n].to(device)
        return Prefill(**kw)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _bf16(x):
    return x.to(torch.bfloat16)


def _sign_vector(g, device, n=IDX_DIM, mag=0.5):
    s = torch.randint(0, 2, (n,), generator=g, device=device).to(torch.float32)
    return (2.0 * s - 1.0) * mag


def _plant_needles(k_idx, q_idx, cu, needles):
    """Overwrite every token of each needle block with 3x the mean indexer query."""
    m = q_idx.to(torch.float32).reshape(-1, IDX_DIM).mean(dim=0)
    val = _bf16(3.0 * m)
    for s, blocks in needles.items():
        base = int(cu[s])
        for b in blocks:
            k_idx[base + 4 * b: base + 4 * b + 4] = val
    return k_idx


def _draw_needle_blocks(g, nblocks_lo, nblocks_hi, count):
    span = nblocks_hi - nblocks_lo
    perm = torch.randperm(span, generator=torch.Generator().manual_seed(int(
        torch.randint(0, 2**31 - 1, (1,), generator=g, device=g.device).item())))
    return sorted(int(x) + nblocks_lo for x in perm[:count])


def prefill(name: str, device="cpu", seed: Optional[int] = None) -> Prefill:
    """Draw one of the named prefill workloads on ``device``."""
    seed = 1000 + WORKLOAD_IDS[name] if seed is None else seed
    if name == "tiny":
        return custom_prefill([256], topk=16, kind="needle", device=device, seed=seed,
                              needles_per_seq=4, needle_range=(8, 56), name=name)
    if name == "8k":
        return custom_prefill([8192], topk=512, kind="needle", device=device, seed=seed,
                              needles_per_seq=32, needle_range=(8, 2040), name=name)
    if name == "8k_int":
        return custom_prefill([8192], topk=512, kind="int", device=device, seed=seed + 500,
                              name=name)
    if name == "64k":
        return custom_prefill([65536], topk=512, kind="drift", device=device, seed=seed,
                              name=name)
    if name == "ragged":
        gl = torch.Generator().manual_seed(seed + 7)
        lens = []
        while len(lens) < 8:
            L = int(torch.randint(1000, 131072, (1,), generator=gl).item())
            if L % 4 != 0:
                lens.append(L)
        return custom_prefill(lens, topk=512, kind="needle", device=device, seed=seed,
                              needles_per_seq=4, needle_range=(8, None), name=name)
    raise KeyError(name)


def custom_prefill(lengths, topk, kind="normal", device="cpu", seed=0, needles_per_seq=0,
                   needle_range=(8, None), name="custom", drift_sigma=0.05) -> Prefill:
    """Draw a packed varlen prefill batch.

    kind: "normal" (all N(0,1), w ~ U(0,1)), "needle" (normal + planted needle blocks),
    "int" (integer indexer inputs), "drift" (block-drifting k_idx and K).
    """
    g = _gen(device, seed)
    lengths = [int(x) for x in lengths]
    cu = torch.tensor([0] + list(torch.tensor(lengths).cumsum(0).tolist()), dtype=torch.int32)
    T = int(cu[-1])
    q = _bf16(_randn((T, NUM_HEADS, HEAD_DIM), g, device))
    v = _bf16(_randn((T, NUM_KV_HEADS, HEAD_DIM), g, device))
    needles = {}
    if kind == "int":
        k = _bf16(_randn((T, NUM_KV_HEADS, HEAD_DIM), g, device))
        q_idx = _bf16(torch.randint(-2, 3, (T, IDX_HEADS, IDX_DIM), generator=g, device=device)
                      .to(torch.float32))
        k_idx = _bf16(torch.randint(-2, 3, (T, IDX_DIM), generator=g, device=device)
                      .to(torch.float32))
        w = _bf16(torch.randint(1, 3, (T, IDX_HEADS), generator=g, device=device)
                  .to(torch.float32))
    elif kind == "drift":
        q_idx = _bf16(_randn((T, IDX_HEADS, IDX_DIM), g, device))
        w = _bf16(torch.rand((T, IDX_HEADS), generator=g, device=device))
        k_list, kidx_list = [], []
        for L in lengths:
            nb = (L + BLOCK - 1) // BLOCK
            steps_i = _randn((nb, IDX_DIM), g, device) * drift_sigma
            steps_i[0] = 0.0
            mu_i = steps_i.cumsum(0)
            steps_k = _randn((nb, NUM_KV_HEADS, HEAD_DIM), g, device) * drift_sigma
            steps_k[0] = 0.0
            mu_k = steps_k.cumsum(0)
            blk = torch.arange(L, device=device) // BLOCK
            kidx_list.append(_bf16(mu_i[blk] + _randn((L, IDX_DIM), g, device)))
            k_list.append(_bf16(mu_k[blk] + _randn((L, NUM_KV_HEADS, HEAD_DIM), g, device)))
        k = torch.cat(k_list)
        k_idx = torch.cat(kidx_list)
    elif kind in ("normal", "needle"):
        k = _bf16(_randn((T, NUM_KV_HEADS, HEAD_DIM), g, device))
        w = _bf16(torch.rand((T, IDX_HEADS), generator=g, device=device))
        if kind == "needle":
            mu = _sign_vector(g, device)
            q_idx = _bf16(mu + _randn((T, IDX_HEADS, IDX_DIM), g, device))
        else:
            q_idx = _bf16(_randn((T, IDX_HEADS, IDX_DIM), g, device))
        k_idx = _bf16(_randn((T, IDX_DIM), g, device))
        if kind == "needle" and needles_per_seq > 0:
            for s, L in enumerate(lengths):
                lo, hi = needle_range
                nb = L // BLOCK
                hi = nb if hi is None else min(hi, nb)
                if hi - lo >= needles_per_seq:
                    needles[s] = _draw_needle_blocks(g, lo, hi, needles_per_seq)
            k_idx = _plant_needles(k_idx, q_idx, cu, needles)
    else:
        raise KeyError(kind)
    return Prefill(name=name, q=q, k=k, v=v, q_idx=q_idx, k_idx=k_idx, w=w, cu_seqlens=cu,
                   topk=int(topk), needles=needles)


@dataclasses.dataclass
class DecodeSpec:
    name: str
    batch: int
    context: list            # prior context length per sequence (before the first step)
    capacity: int            # cache capacity in tokens (multiple of 4)
    topk: int
    steps: int               # decode steps (each appends one token then decodes)
    seed: int


def decode_spec(name: str) -> DecodeSpec:
    seed = 1000 + WORKLOAD_IDS[name]
    if name == "decode256k":
        return DecodeSpec(name, 64, [262140 + (i % 4) for i in range(64)], 262144, 512, 1,
                          seed)
    if name == "decode1m":
        return DecodeSpec(name, 4, [1048512 - i for i in range(4)], 1048576, 512, 64, seed)
    raise KeyError(name)


def small_decode_spec(batch=4, context=(1000, 1001, 1002, 1003), capacity=1280, topk=64,
                      steps=6, seed=77) -> DecodeSpec:
    return DecodeSpec("small", batch, list(context), capacity, topk, steps, seed)


def decode_context(spec: DecodeSpec, device="cpu", lmax=None):
    """Context tokens for every sequence, padded to the longest: k, v [B, Lmax, 2, 128],
    k_idx [B, Lmax, 64] (bf16).  Rows past a sequence's length are drawn but unused."""
    g = _gen(device, spec.seed)
    B = spec.batch
    lmax = max(spec.context) if lmax is None else lmax
    k = _bf16(_randn((B, lmax, NUM_KV_HEADS, HEAD_DIM), g, device))
    v = _bf16(_randn((B, lmax, NUM_KV_HEADS, HEAD_DIM), g, device))
    k_idx = _bf16(_randn((B, lmax, IDX_DIM), g, device))
    return k, v, k_idx


def decode_step(spec: DecodeSpec, step: int, device="cpu"):
    """Per-step new token (k, v, k_idx) and query (q, q_idx, w) for every sequence."""
    g = _gen(device, spec.seed * 1000003 + 17 * (step + 1))
    B = spec.batch
    k = _bf16(_randn((B, 1, NUM_KV_HEADS, HEAD_DIM), g, device))
    v = _bf16(_randn((B, 1, NUM_KV_HEADS, HEAD_DIM), g, device))
    k_idx = _bf16(_randn((B, 1, IDX_DIM), g, device))
    q = _bf16(_randn((B, NUM_HEADS, HEAD_DIM), g, device))
    q_idx = _bf16(_randn((B, IDX_HEADS, IDX_DIM), g, device))
    w = _bf16(torch.rand((B, IDX_HEADS), generator=g, device=device))
    return dict(k=k, v=v, k_idx=k_idx, q=q, q_idx=q_idx, w=w)


def bits(t: torch.Tensor):
    """Raw bf16 bit patterns of a tensor as a numpy uint16 array (CPU copy)."""
    assert t.dtype == torch.bfloat16
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")


# ---- the Gated DeltaNet layer ------------------------------------------------------------
@dataclasses.dataclass
class GatedDeltaNet:
    q: torch.Tensor          # [T, H, 128] bf16, each row of unit L2 norm (before bf16 rounding)
    k: torch.Tensor          # [T, H, 128] bf16, likewise
    v: torch.Tensor          # [T, H, 128] bf16, N(0,1)
    log_alpha: torch.Tensor  # [T, H] fp32: log of a gate drawn uniformly in `gate`
    beta: torch.Tensor       # [T, H] fp32, U(0,1)
    cu_seqlens: torch.Tensor  # [num_seqs+1] int32 (CPU)

    def to(self, device) -> "GatedDeltaNet":
        kw = {f.name: getattr(self, f.name) for f in dataclasses.fields(self)}
        for n in ("q", "k", "v", "log_alpha", "beta"):
            kw[n] = kw[n].to(device)
        return GatedDeltaNet(**kw)


def gated_deltanet(lengths, heads, seed=0, gate=(0.9, 1.0), reset_every=0, device="cpu"):
    """Seeded inputs of the Gated DeltaNet layer for packed sequences of the given lengths.
    q and k are unit-norm rows (the layer takes them as given; normalised keys keep the
    delta rule's state bounded), gates alpha ~ U(gate), and with reset_every > 0 every
    reset_every-th token has alpha = 0 (log_alpha = -inf)."""
    g = torch.Generator().manual_seed(5000 + seed)
    T = int(sum(lengths))
    shape = (T, heads, HEAD_DIM)

    def unit_rows():
        x = torch.randn(shape, generator=g)
        return (x / x.norm(dim=-1, keepdim=True).clamp_min(1e-6)).to(torch.bfloat16)

    q, k = unit_rows(), unit_rows()
    v = torch.randn(shape, generator=g).to(torch.bfloat16)
    lo, hi = gate
    log_alpha = torch.log(lo + (hi - lo) * torch.rand((T, heads), generator=g))
    if reset_every > 0:
        log_alpha[::reset_every] = float("-inf")
    beta = torch.rand((T, heads), generator=g)
    cu = torch.tensor([0] + torch.tensor([int(x) for x in lengths]).cumsum(0).tolist(),
                      dtype=torch.int32)
    return GatedDeltaNet(q, k, v, log_alpha, beta, cu).to(device)
