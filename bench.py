#!/usr/bin/env python
"""QSA benchmark: 64K prefill tokens/s and 256K decode tokens/s on B200, with roofline.

One step = one QSA prefill of a 65,536-token sequence (budget 512 blocks; indexer keys and
K drift per block) plus one decode step (append one token, then decode) for a batch of 64
sequences at 262,140..262,143 tokens of context.  Inputs are seeded synthetic tensors of
those shapes (no dataset is involved).  Each step is timed with CUDA events on the stream
the kernels run on; L2 is flushed before each timed part: a 256 MB write, then a 256 MB
read of another buffer, so that the written lines leave L2 before the timer starts.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl qsa|reference]
       [--workload both|prefill|decode]
Under torchrun (N > 1) every rank runs its own replica of the step on its own GPU (the
sequences are independent, no collective on the data path); rank 0 prints one JSON line
with the whole-job throughput computed from the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "QSA prefill tokens/s at 64K & decode tokens/s at 256K ctx; % of roofline"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

PREFILL_T, TOPK = 65536, 512
REF_ROWS = 256        # query rows per step of the reference arm (the CPU oracle)
DEC_BATCH, DEC_CAP = 64, 262144

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of the roofline kernels from one
# ncu capture: bytes per unit of work (prefill attention: per query token; decode step: per
# sequence), the SHA-256 of the sources in TRAFFIC_SOURCES at the capture, and what was captured.  A
# figure is reported only while the sources are unchanged; otherwise the roofline's
# "traffic" is null until a new capture is taken.
NCU_TRAFFIC = {
    # 312,955,904 B read + 175,307,008 B written by one 32K-token prefill attention launch
    # (profiles/k_sparse_attn_prefill_32k.md), per token; the attention's bytes (Q, O, the
    # gathered K/V tiles, the plan) grow with the tokens of the launch.
    "prefill_attention": (488262912 / 32768,
                          "d1ea05a60e832f72204bcec12ba314564f4d847fe9118e6a990904e7bda79a7d",
                          "ncu dram__bytes_read.sum + dram__bytes_write.sum of one 32K-token "
                          "launch (profiles/k_sparse_attn_prefill_32k.md), scaled by tokens"),
    # The seven kernels of one 256K x 64 decode step, one ncu capture each (1 pass): reads
    # 690,883,840 B, writes 6,260,224 B (profiles/decode_step_dram_decode256k_b64.md); per
    # sequence of the batch.
    "decode_step": (697144064 / 64,
                    "d6c1add7fa73aec5ec5dec7604922821ea7d8e2788d833d5ac7373ea6323d38b",
                    "ncu dram__bytes_read.sum + dram__bytes_write.sum of the seven kernels of "
                    "one 256K x 64 decode step (profiles/decode_step_dram_decode256k_b64.md)"),
}


# The sources each roofline kernel's code and launch depend on; a capture is stale once any
# of them changes.
TRAFFIC_SOURCES = {
    "prefill_attention": ("qsa_attn.cuh", "qsa_common.cuh", "qsa_api.cu"),
    "decode_step": ("qsa_api.cu", "qsa_attn.cuh", "qsa_common.cuh", "qsa_misc.cuh",
                    "qsa_score.cuh"),   # the whole step
}


def csrc_sha(files=None):
    import hashlib
    d = os.path.join(ROOT, "block_sparse_attention_40_b200", "csrc")
    h = hashlib.sha256()
    for n in sorted(os.listdir(d)):
        if n.endswith((".cu", ".cuh")) and (files is None or n in files):
            h.update(n.encode())
            h.update(open(os.path.join(d, n), "rb").read())
    return h.hexdigest()


def measured_traffic(kernel, units):
    """Per-launch DRAM bytes of `kernel` scaled to `units`, or (None, reason)."""
    rec = NCU_TRAFFIC.get(kernel)
    if rec is None:
        return None, "no ncu capture of the current kernel"
    per_unit, sha, what = rec
    if sha != csrc_sha(TRAFFIC_SOURCES[kernel]):
        return None, "kernel sources changed since the ncu capture"
    return per_unit * units, what


# ------------------------------------------------------------------------------------
# algorithmic work (definitions; the kernels never read these)
def prefill_attention_flops(T=PREFILL_T, k=TOPK):
    """Selected-token FLOPs: per token, 24 heads x 128 dims x 4 flops (QK and PV) per key."""
    tot = 0
    for t in range(T):
        keys = 4 * min(k, t // 4) + (t % 4) + 1
        tot += keys
    return 24 * 128 * 4 * tot


def prefill_indexer_flops(T=PREFILL_T):
    return sum(2 * 16 * 64 * (t // 4) for t in range(T))


def decode_bytes_per_seq(L_after, k=TOPK):
    """HBM bytes one decode step must read/write for one sequence of L_after tokens."""
    p = L_after - 1
    n_c = p // 4
    sel = min(k, n_c)
    kbar = n_c * 64 * 2
    kv = sel * 2 * 2 * 4 * 128 * 2               # K and V, 2 heads, 4 tokens, 128 dims
    tail = 2 * 2 * 4 * 128 * 2                   # own block, K and V, both heads
    q = 24 * 128 * 2 + 16 * 64 * 2 + 16 * 2      # q, q_idx, w
    out = 24 * 128 * 2
    append = 2 * 2 * 128 * 2 + 64 * 2            # new K, V rows and k_idx
    return kbar + kv + tail + q + out + append


# ------------------------------------------------------------------------------------
def load_peaks():
    try:
        d = json.load(open(PEAKS_FILE))
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"qsa_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.fh,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------
def dist_setup(n_gpus):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device):
    """Largest value of x across ranks (device time is taken as the slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------------
def run_qsa(args, rank, world, local):
    import torch
    import block_sparse_attention_40_b200 as qsa
    from block_sparse_attention_40_b200 import binding as B
    from block_sparse_attention_40_b200 import workloads as W

    dev = torch.device(f"cuda:{local}")
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = load_peaks()
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)   # 256 MB

    def flush():
        # the write evicts the step's data; the read then evicts the written (dirty) lines,
        # so the timed part does not pay for writing them back
        flush_buf.random_(0, 255)
        flush_rd.sum()

    do_prefill = args.workload in ("both", "prefill")
    do_decode = args.workload in ("both", "decode")
    res = {}

    # ---------------- prefill setup ----------------
    if do_prefill:
        if args.prefill_len == PREFILL_T:
            p = W.prefill("64k", device=dev, seed=1002 + rank)
        else:   # smaller case of the same drifting workload (profiling captures)
            p = W.custom_prefill([args.prefill_len], TOPK, kind="drift", device=dev,
                                 seed=1002 + rank)
        ctx = qsa.Prefill(p.cu_seqlens, dev, TOPK, args.rows_per_tile, args.chunk_rows,
                          select_mode=args.select_mode)
        idx = torch.empty((args.prefill_len, TOPK), dtype=torch.int32, device=dev)
        cnt = torch.empty((args.prefill_len,), dtype=torch.int32, device=dev)
        out = torch.empty_like(p.q)

    # ---------------- decode setup ----------------
    if do_decode:
        spec = W.decode_spec("decode256k")
        spec.seed += 17 * rank
        if args.decode_batch != spec.batch:   # smaller case of the same workload (captures)
            spec.batch = args.decode_batch
            spec.context = [262140 + (i % 4) for i in range(spec.batch)]
        if args.paged_tokens:
            # paged cache: every sequence's pages are drawn from a seeded shuffle of the pool
            max_pages = spec.capacity // args.paged_tokens
            pool = spec.batch * max_pages
            perm = torch.randperm(pool, generator=torch.Generator().manual_seed(4242 + rank))
            table = perm.view(spec.batch, max_pages).to(torch.int32).to(dev)
            cache = qsa.PagedKVCache(spec.batch, spec.capacity, args.paged_tokens, pool, table,
                                     dev, zero=False)
        else:
            cache = qsa.KVCache(spec.batch, spec.capacity, dev, zero=False)
        kc, vc, kic = W.decode_context(spec, device=dev)
        lmax = max(spec.context)
        for c0 in range(0, lmax, 16384):
            c1 = min(lmax, c0 + 16384)
            counts = [max(0, min(c1, L) - c0) for L in spec.context]
            cache.append(kc[:, c0:c1].contiguous(), vc[:, c0:c1].contiguous(),
                         kic[:, c0:c1].contiguous(), counts=counts)
        del kc, vc, kic
        torch.cuda.synchronize(dev)
        torch.cuda.empty_cache()
        saved_len = cache.len.clone()
        saved_part = cache.kbar_partial.clone()
        saved_hlen = list(cache.h_len)
        dec = qsa.Decoder(cache, TOPK, args.decode_splits)
        st = W.decode_step(spec, 0, device=dev)
        dec_out = torch.empty_like(st["q"])

        def reset_cache():
            cache.len.copy_(saved_len)
            cache.kbar_partial.copy_(saved_part)
            cache.h_len = list(saved_hlen)

    def step(timed, ev):
        if do_prefill:
            flush()
            ev["p0"].record(stream)
            ctx.select(p.q_idx, p.k_idx, p.w, idx, cnt)
            ev["p1"].record(stream)
            ctx.attend(p.q, p.k, p.v, idx, cnt, out)
            ev["p2"].record(stream)
        if do_decode:
            reset_cache()
            flush()
            ev["d0"].record(stream)
            if dec_graph is not None:
                dec_graph.replay()
            else:
                cache.append(st["k"], st["v"], st["k_idx"])
                dec.run(st["q"], st["q_idx"], st["w"], out=dec_out)
            ev["d1"].record(stream)

    names = ["p0", "p1", "p2", "d0", "d1"]
    dec_graph = None
    graph_launches = 0
    for _ in range(args.warmup):
        step(False, {n: torch.cuda.Event(enable_timing=True) for n in names})
    torch.cuda.synchronize(dev)
    if do_decode and args.graph:
        # one decode step (append + decode) captured as a CUDA graph and replayed per step;
        # the cache is reset outside the graph, so every replay sees the same state
        reset_cache()
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        n0 = B.launch_count()
        with torch.cuda.graph(g):
            cache.append(st["k"], st["v"], st["k_idx"])
            dec.run(st["q"], st["q_idx"], st["w"], out=dec_out)
        torch.cuda.synchronize(dev)
        graph_launches = B.launch_count() - n0   # kernels each replay runs
        dec_graph = g
        for _ in range(args.warmup):
            step(False, {n: torch.cuda.Event(enable_timing=True) for n in names})
        torch.cuda.synchronize(dev)
    barrier(world)
    launches0 = B.launch_count()
    evs = [{n: torch.cuda.Event(enable_timing=True) for n in names} for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.5)            # let nvidia-smi start sampling before the timed region
    torch.cuda.synchronize(dev)
    barrier(world)
    for i in range(args.steps):
        step(True, evs[i])
    torch.cuda.synchronize(dev)
    barrier(world)
    clk = clocks.stop()
    launches = B.launch_count() - launches0 + args.steps * graph_launches
    sel_ms = sum(e["p0"].elapsed_time(e["p1"]) for e in evs) if do_prefill else 0.0
    att_ms = sum(e["p1"].elapsed_time(e["p2"]) for e in evs) if do_prefill else 0.0
    dec_ms = sum(e["d0"].elapsed_time(e["d1"]) for e in evs) if do_decode else 0.0
    sel_ms = max_over_ranks(sel_ms, world, dev)
    att_ms = max_over_ranks(att_ms, world, dev)
    dec_ms = max_over_ranks(dec_ms, world, dev)
    K = args.steps
    errs = []
    if do_prefill:
        errs.append(ctx.device_error())
    if do_decode:
        errs.append(dec.device_error())
    assert all(e == ("QSA_OK", 0) for e in errs), errs
    union = union_stats(idx, args.prefill_len, args.rows_per_tile or 10) if do_prefill else None

    # ---------------- e2e through host buffers ----------------
    e2e = {}
    if args.e2e and do_prefill:
        hp = {n: getattr(p, n).cpu().pin_memory() for n in ("q", "k", "v", "q_idx", "k_idx", "w")}
        hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        dp = {n: torch.empty_like(getattr(p, n)) for n in hp}
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tot = 0.0
        for i in range(max(1, min(K, 3)) + 1):
            flush()
            e0.record(stream)
            for n in hp:
                dp[n].copy_(hp[n], non_blocking=True)
            ctx.run(dp["q"], dp["k"], dp["v"], dp["q_idx"], dp["k_idx"], dp["w"], out)
            hout.copy_(out, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if i > 0:
                tot += e0.elapsed_time(e1)
        n_e2e = max(1, min(K, 3))
        tot = max_over_ranks(tot, world, dev)
        h2d = sum(t.numel() * t.element_size() for t in hp.values())
        e2e["prefill"] = {"value": world * args.prefill_len * n_e2e / (tot / 1e3), "unit": "tokens/s",
                          "h2d_bytes_per_step": h2d,
                          "d2h_bytes_per_step": hout.numel() * hout.element_size()}
        del hp, hout, dp
    if args.e2e and do_decode:
        hs = {n: st[n].cpu().pin_memory() for n in st}
        ds = {n: torch.empty_like(st[n]) for n in st}
        hout = torch.empty(dec_out.shape, dtype=dec_out.dtype, pin_memory=True)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tot = 0.0
        for i in range(K + 1):
            reset_cache()
            flush()
            e0.record(stream)
            for n in hs:
                ds[n].copy_(hs[n], non_blocking=True)
            cache.append(ds["k"], ds["v"], ds["k_idx"])
            dec.run(ds["q"], ds["q_idx"], ds["w"], out=dec_out)
            hout.copy_(dec_out, non_blocking=True)
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if i > 0:
                tot += e0.elapsed_time(e1)
        tot = max_over_ranks(tot, world, dev)
        e2e["decode"] = {"value": world * args.decode_batch * K / (tot / 1e3), "unit": "tokens/s",
                         "h2d_bytes_per_step": sum(t.numel() * t.element_size() for t in hs.values()),
                         "d2h_bytes_per_step": hout.numel() * hout.element_size()}

    res = dict(sel_ms=sel_ms, att_ms=att_ms, dec_ms=dec_ms, clocks=clk, launches=launches,
               peaks=peaks, peak_src=peak_src, e2e=e2e, do_prefill=do_prefill,
               do_decode=do_decode, union=union)
    if do_decode:
        res["dec_bytes"] = sum(decode_bytes_per_seq(L + 1) for L in spec.context)
        res["dec_timing"] = "cuda graph replay of append + decode" if dec_graph is not None else "eager launches"
    return res


def union_stats(idx, T, R):
    """The prefill attention's union work, counted after the timed region from the selections
    the step returned (one sequence of T tokens): each R-token tile attends the union of its
    tokens' selected blocks and own blocks, in 32-block chunks of 128 keys for each KV head;
    a chunk is 128 rows x 128 keys x 128 dims x 2 flops for QK^T and again for PV."""
    import torch
    k = idx.shape[1]
    own = (torch.arange(T, device=idx.device, dtype=torch.int32) // 4)[:, None]
    x = torch.cat([idx[:T], own], dim=1)
    tiles = (T + R - 1) // R
    if tiles * R > T:
        x = torch.cat([x, torch.full((tiles * R - T, k + 1), -1, dtype=x.dtype,
                                     device=x.device)])
    x, _ = torch.sort(x.view(tiles, R * (k + 1)), dim=1)
    first = torch.ones_like(x, dtype=torch.bool)
    first[:, 1:] = x[:, 1:] != x[:, :-1]
    u = ((x >= 0) & first).sum(dim=1)
    chunks = int(((u + 31) // 32).sum().item()) * 2   # both KV heads
    union_flops = chunks * 128 * 128 * 128 * 2 * 2
    return {"rows_per_tile": R, "tiles": tiles, "union_blocks_per_tile": float(u.float().mean()),
            "chunks": chunks, "union_tflop": union_flops / 1e12,
            "useful_fraction": prefill_attention_flops(T) / union_flops}


GDN_LENGTHS, GDN_HEADS = [8192] * 8, 16


def run_gdn(args, rank, world, local):
    """The Gated DeltaNet layer (three of every four token-mixing layers around QSA) over 8
    sequences of 8,192 tokens with 16 heads of 128, timed on its own after the rest.  Its
    inputs (805 MB of q, k, v) exceed L2, so no flush is needed between launches."""
    import torch
    import block_sparse_attention_40_b200 as qsa
    from block_sparse_attention_40_b200 import binding as B
    from block_sparse_attention_40_b200 import workloads as W

    dev = torch.device(f"cuda:{local}")
    stream = torch.cuda.current_stream(dev)
    w = W.gated_deltanet(GDN_LENGTHS, GDN_HEADS, seed=11 + rank, device=dev)
    d_cu = w.cu_seqlens.to(dev)
    out = torch.empty_like(w.q)
    K = args.steps
    clocks = ClockSampler(local)
    clocks.start()
    launches0 = B.launch_count()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for i in range(args.warmup + K):
        e = ev[i - args.warmup] if i >= args.warmup else None
        if e:
            e[0].record(stream)
        qsa.gated_deltanet(w.q, w.k, w.v, w.log_alpha, w.beta, w.cu_seqlens, out=out,
                           d_cu_seqlens=d_cu)
        if e:
            e[1].record(stream)
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / K, world, dev)
    T = sum(GDN_LENGTHS)
    # the recurrence per token and head: S k, the rank-1 write and S q, 128 x 128 each
    flops = 6 * 128 * 128 * T * GDN_HEADS
    # the products run as TF32 tensor-core MMAs: the measured bf16 burst peak scaled by the
    # nominal dense TF32 / bf16 ratio (1.1 / 2.25 PFLOP/s)
    peaks, src = load_peaks()
    peak = peaks["bf16_tflops"] * 1.1 / 2.25
    ach = flops / (ms / 1e3) / 1e12
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    mhz = clk.get("sm_max_mhz") or 1965.0
    fma_peak = sms * 128 * 2 * mhz * 1e6 / 1e12   # fp32 FMA lanes per SM x 2 flops x clock
    return {"workload": f"{len(GDN_LENGTHS)} x {GDN_LENGTHS[0]} tokens, {GDN_HEADS} heads of 128",
            "ms": ms, "tokens_per_s": world * T / (ms / 1e3),
            "roofline": {"kernel": "k_gated_deltanet (TF32 MMAs, fp32 state, chunks of 64 tokens)",
                         "bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                         "frac": ach / peak,
                         "peak_source": f"{src} bf16 burst x 1.1/2.25 (nominal dense TF32/bf16)",
                         "fp32_fma_peak": fma_peak,
                         "algorithmic": f"{flops / 1e12:.4f} TFLOP of the recurrence per launch"},
            "clocks": clk, "gpu_launches": B.launch_count() - launches0}


# ------------------------------------------------------------------------------------
def ragged_attention_flops(lengths, k=TOPK):
    return sum(prefill_attention_flops(L, k) for L in lengths)


def ragged_indexer_flops(lengths):
    return sum(prefill_indexer_flops(L) for L in lengths)


def run_mixed(args, rank, world, local):
    """The mixed ragged workload, timed after the headline parts, each on its own:
    * a varlen prefill of 8 sequences of 1,000..131,071 tokens (not multiples of 4);
    * decode of 4 sequences at 1,048,509..1,048,512 tokens of context, 64 consecutive
      append + decode steps captured as one CUDA graph (so 16 blocks per sequence are
      completed by incremental compression inside every replay)."""
    import torch
    import block_sparse_attention_40_b200 as qsa
    from block_sparse_attention_40_b200 import binding as B
    from block_sparse_attention_40_b200 import workloads as W

    dev = torch.device(f"cuda:{local}")
    stream = torch.cuda.current_stream(dev)
    peaks, peak_src = load_peaks()
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush():
        flush_buf.random_(0, 255)
        flush_rd.sum()

    out = {}
    K = args.steps
    clocks = ClockSampler(local)
    clocks.start()
    launches0 = B.launch_count()
    graph_launches = 0
    # ---- varlen prefill ----
    p = W.prefill("ragged", device=dev, seed=1004 + rank)
    lens = (p.cu_seqlens[1:] - p.cu_seqlens[:-1]).tolist()
    T = p.total_tokens
    ctx = qsa.Prefill(p.cu_seqlens, dev, TOPK)
    idx = torch.empty((T, TOPK), dtype=torch.int32, device=dev)
    cnt = torch.empty((T,), dtype=torch.int32, device=dev)
    o = torch.empty_like(p.q)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    for i in range(args.warmup + K):
        flush()
        e = ev[i - args.warmup] if i >= args.warmup else None
        if e:
            e[0].record(stream)
        ctx.select(p.q_idx, p.k_idx, p.w, idx, cnt)
        if e:
            e[1].record(stream)
        ctx.attend(p.q, p.k, p.v, idx, cnt, o)
        if e:
            e[2].record(stream)
    torch.cuda.synchronize(dev)
    assert ctx.device_error() == ("QSA_OK", 0)
    sel = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / K, world, dev)
    att = max_over_ranks(sum(e[1].elapsed_time(e[2]) for e in ev) / K, world, dev)
    af, xf = ragged_attention_flops(lens), ragged_indexer_flops(lens)
    out["prefill_ragged"] = {
        "lengths": lens, "tokens": T, "ms": sel + att, "select_ms": sel, "attention_ms": att,
        "tokens_per_s": world * T / ((sel + att) / 1e3),
        "roofline": {"kernel": "qsa_sparse_attention", "bound": "tensor",
                     "achieved": af / (att / 1e3) / 1e12, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": af / (att / 1e3) / 1e12 / peaks["bf16_tflops"],
                     "peak_source": f"{peak_src} bf16 burst",
                     "algorithmic": f"{af / 1e12:.4f} TFLOP selected-token per launch"},
        "indexer_tflop": xf / 1e12}
    del p, ctx, idx, cnt, o
    torch.cuda.empty_cache()
    # ---- 1M decode, 64 append + decode steps per replay ----
    spec = W.decode_spec("decode1m")
    spec.seed += 17 * rank
    cache = qsa.KVCache(spec.batch, spec.capacity, dev, zero=False)
    kc, vc, kic = W.decode_context(spec, device=dev)
    lmax = max(spec.context)
    for c0 in range(0, lmax, 16384):
        c1 = min(lmax, c0 + 16384)
        counts = [max(0, min(c1, L) - c0) for L in spec.context]
        cache.append(kc[:, c0:c1].contiguous(), vc[:, c0:c1].contiguous(),
                     kic[:, c0:c1].contiguous(), counts=counts)
    del kc, vc, kic
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    saved = (cache.len.clone(), cache.kbar_partial.clone(), list(cache.h_len))
    dec = qsa.Decoder(cache, TOPK)
    steps = [W.decode_step(spec, s, device=dev) for s in range(spec.steps)]
    outs = torch.empty((spec.steps, spec.batch, 24, 128), dtype=torch.bfloat16, device=dev)

    def reset():
        cache.len.copy_(saved[0])
        cache.kbar_partial.copy_(saved[1])
        cache.h_len = list(saved[2])

    def run_steps():
        for s, st in enumerate(steps):
            cache.append(st["k"], st["v"], st["k_idx"])
            dec.run(st["q"], st["q_idx"], st["w"], out=outs[s])

    for _ in range(args.warmup):
        reset()
        run_steps()
    reset()
    torch.cuda.synchronize(dev)
    g = torch.cuda.CUDAGraph()
    n0 = B.launch_count()
    with torch.cuda.graph(g):
        run_steps()
    torch.cuda.synchronize(dev)
    per_replay = B.launch_count() - n0
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    for i in range(args.warmup + K):
        reset()
        flush()
        e = ev[i - args.warmup] if i >= args.warmup else None
        if e:
            e[0].record(stream)
        g.replay()
        if e:
            e[1].record(stream)
    torch.cuda.synchronize(dev)
    assert dec.device_error() == ("QSA_OK", 0)
    graph_launches = per_replay * (args.warmup + K)
    ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in ev) / K, world, dev)
    nbytes = sum(decode_bytes_per_seq(L + s + 1) for L in spec.context for s in range(spec.steps))
    gbs = nbytes / (ms / 1e3) / 1e9
    out["decode_1m"] = {
        "batch": spec.batch, "context": spec.context, "steps_per_replay": spec.steps,
        "ms_per_replay": ms, "ms_per_step": ms / spec.steps,
        "tokens_per_s": world * spec.batch * spec.steps / (ms / 1e3),
        "timing": "cuda graph of 64 x (append 1 token + decode), replayed; cache lengths reset "
                  "between replays; L2 flushed before each replay",
        "roofline": {"kernel": "64 whole decode steps", "bound": "hbm", "achieved": gbs,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                     "peak_source": f"{peak_src} HBM copy",
                     "algorithmic": f"{nbytes / spec.steps / spec.batch / 1e6:.2f} MB per "
                                    f"sequence per step"}}
    g.reset()
    out["clocks"] = clocks.stop()
    # kernels this part launched, warm-ups included (graph replays count their kernels; the
    # capture itself launches nothing)
    out["gpu_launches_incl_warmup"] = B.launch_count() - launches0 + graph_launches - per_replay
    return out


def cpu_baseline(seconds_target=12.0, threads=None):
    """The oracle, as it stands, on a bounded sample of the 64K prefill rows."""
    import numpy as np
    import torch
    import oracle
    from block_sparse_attention_40_b200 import workloads as W
    p = W.prefill("64k", device="cpu")
    b = {n: W.bits(getattr(p, n)) for n in ("q", "k", "v", "q_idx", "k_idx", "w")}
    threads = threads or os.cpu_count() or 1
    rng = np.random.default_rng(0)
    n = 8
    elapsed, rows_done = 0.0, 0
    while elapsed < seconds_target and rows_done < 4096:
        rows = np.sort(rng.integers(0, PREFILL_T, n))
        t0 = time.perf_counter()
        oracle.prefill(q=b["q"], k=b["k"], v=b["v"], q_idx=b["q_idx"], k_idx=b["k_idx"],
                       w=b["w"], cu_seqlens=p.cu_seqlens.numpy().astype(np.int64), topk=TOPK,
                       row_ids=rows, threads=threads)
        elapsed += time.perf_counter() - t0
        rows_done += n
        n *= 2
    del torch
    return {"value": rows_done / elapsed, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{rows_done} uniformly drawn query rows of the 65,536-token prefill "
                      f"(selection + attention per row), {elapsed:.1f} s"}


def workload_config(args, world, do_prefill, do_decode):
    """The `config` object of the JSON line; both arms print the same one."""
    return {"workload": " + ".join(
                ([f"qsa_prefill_{args.prefill_len // 1024}k"] if do_prefill else [])
                + ([f"qsa_decode_256k_b{args.decode_batch}"
                    + (f"_paged{args.paged_tokens}" if args.paged_tokens else "")]
                   if do_decode else [])),
            "prefill_seq_len": args.prefill_len, "decode_batch": args.decode_batch,
            "decode_context": "262140 + (i mod 4)", "topk_blocks": TOPK,
            "heads": "24q/2kv", "head_dim": 128, "indexer": "16x64",
            "l2": "flushed before each timed part (256 MB write, then 256 MB read)",
            "parallelism": f"replicas x{world}", "select_mode": args.select_mode}


def run_reference(args, rank, world):
    """Reference arm: the CPU oracle, as it stands, timed on the host cores.  A step is one
    bounded sample of the 64K prefill: REF_ROWS query rows drawn uniformly (selection and
    attention per row); W untimed warm-up steps, then K timed steps, each on fresh rows."""
    if rank != 0:
        return
    import numpy as np
    import oracle
    from block_sparse_attention_40_b200 import workloads as W
    threads = os.cpu_count() or 1
    p = W.prefill("64k", device="cpu")
    b = {n: W.bits(getattr(p, n)) for n in ("q", "k", "v", "q_idx", "k_idx", "w")}
    cu = p.cu_seqlens.numpy().astype(np.int64)
    rng = np.random.default_rng(0)
    times = []
    for i in range(args.warmup + args.steps):
        rows = np.sort(rng.choice(PREFILL_T, REF_ROWS, replace=False))
        t0 = time.perf_counter()
        oracle.prefill(q=b["q"], k=b["k"], v=b["v"], q_idx=b["q_idx"], k_idx=b["k_idx"],
                       w=b["w"], cu_seqlens=cu, topk=TOPK, row_ids=rows, threads=threads)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    tot = sum(times)
    value = REF_ROWS * len(times) / tot
    sample = (f"{REF_ROWS} uniformly drawn query rows of the 65,536-token prefill per step "
              f"(selection + attention per row), {len(times)} timed steps, {tot:.1f} s")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(args, 1, args.workload in ("both", "prefill"),
                                      args.workload in ("both", "decode")),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["qsa", "reference"], default="qsa")
    ap.add_argument("--workload", choices=["both", "prefill", "decode", "gdn"], default="both",
                    help="gdn: only the Gated DeltaNet layer (a line of its own)")
    ap.add_argument("--rows-per-tile", type=int, default=0)
    ap.add_argument("--chunk-rows", type=int, default=0)
    ap.add_argument("--decode-splits", type=int, default=0)
    ap.add_argument("--paged-tokens", type=int, default=0,
                    help="decode from a paged cache with pages of this many tokens (a multiple "
                         "of 512); 0 = contiguous cache")
    ap.add_argument("--decode-batch", type=int, default=DEC_BATCH,
                    help="sequences of the 256K-context decode batch (64 = the workload)")
    ap.add_argument("--prefill-len", type=int, default=PREFILL_T,
                    help="prefill sequence length (default 65536; smaller only for profiling)")
    ap.add_argument("--no-e2e", dest="e2e", action="store_false")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="time the decode step as eager launches instead of a CUDA graph replay")
    ap.add_argument("--no-cpu-baseline", dest="cpu", action="store_false")
    ap.add_argument("--select-mode", type=int, default=0,
                    help="prefill selection: 0 = default; 1 = the indexer finds each row's "
                         "threshold bin (the fused index-score + select)")
    ap.add_argument("--no-gdn", dest="gdn", action="store_false",
                    help="skip the Gated DeltaNet layer timed after the rest")
    ap.add_argument("--no-mixed", dest="mixed", action="store_false",
                    help="skip the mixed ragged workload (8-sequence varlen prefill and the "
                         "1M-context decode) that follows the headline parts")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_setup(args.gpus)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.workload == "gdn":
        gdn = run_gdn(args, rank, world, local)
        if rank == 0:
            print(json.dumps({
                "metric": "Gated DeltaNet layer tokens/s", "value": gdn["tokens_per_s"],
                "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": gdn["ms"], "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "tf32", "data": "synthetic",
                "config": {"workload": gdn["workload"], "l2": "inputs larger than L2",
                           "parallelism": f"replicas x{world}"},
                "roofline": gdn["roofline"], "clocks": gdn["clocks"],
                "gpu_launches": gdn["gpu_launches"]}), flush=True)
        return
    r = run_qsa(args, rank, world, local)
    mixed = None
    if args.mixed and args.workload == "both":
        import torch
        torch.cuda.empty_cache()
        mixed = run_mixed(args, rank, world, local)
    gdn = None
    if args.gdn and args.workload == "both":
        import torch
        torch.cuda.empty_cache()
        gdn = run_gdn(args, rank, world, local)
    if rank != 0:
        return
    K = args.steps
    peaks = r["peaks"]
    line = {"metric": METRIC}
    if r["do_prefill"]:
        pre_ms = (r["sel_ms"] + r["att_ms"]) / K
        attn_flops = prefill_attention_flops(args.prefill_len)
        att_s = r["att_ms"] / K / 1e3
        ach = attn_flops / att_s / 1e12
        line.update({"value": world * args.prefill_len / (pre_ms / 1e3), "unit": "tokens/s"})
        line["roofline"] = {"kernel": "qsa_sparse_attention (union plan + tcgen05 attention)",
                            "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                            "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
                            "peak_source": f"{r['peak_src']} bf16 burst",
                            "traffic": None, "traffic_source": None,
                            "algorithmic": f"{attn_flops / 1e12:.4f} TFLOP selected-token per launch"}
        line["roofline"]["traffic"], line["roofline"]["traffic_source"] = measured_traffic(
            "prefill_attention", args.prefill_len)
        idx_flops = prefill_indexer_flops(args.prefill_len)
        line["prefill"] = {"tokens_per_s": world * args.prefill_len / (pre_ms / 1e3),
                           "ms": pre_ms, "select_ms": r["sel_ms"] / K, "attention_ms": r["att_ms"] / K,
                           "frac_of_bf16_peak_end_to_end":
                               attn_flops / (pre_ms / 1e3) / 1e12 / peaks["bf16_tflops"],
                           "indexer_tflop": idx_flops / 1e12,
                           "select_tflops_indexer_only": idx_flops / (r["sel_ms"] / K / 1e3) / 1e12,
                           "union": dict(r["union"], tensor_floor_ms=r["union"]["union_tflop"]
                                         / peaks["bf16_tflops"] * 1e3)}
    if r["do_decode"]:
        dms = r["dec_ms"] / K
        gbs = r["dec_bytes"] / (dms / 1e3) / 1e9
        dec = {"value": world * args.decode_batch / (dms / 1e3), "unit": "tokens/s", "ms_per_step": dms,
               "timing": r["dec_timing"],
               "roofline": {"kernel": "whole decode step (append, indexer, top-k, plan, "
                                      "attention, combine)", "bound": "hbm", "achieved": gbs,
                            "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": gbs / peaks["hbm_gbs"],
                            "peak_source": f"{r['peak_src']} HBM copy",
                            "traffic": None, "traffic_source": None,
                            "algorithmic": f"{r['dec_bytes'] / 1e6:.1f} MB per step"}}
        dec["roofline"]["traffic"], dec["roofline"]["traffic_source"] = measured_traffic(
            "decode_step", args.decode_batch)
        if "decode" in r["e2e"]:
            dec["e2e"] = r["e2e"]["decode"]
        line["decode"] = dec
        if not r["do_prefill"]:
            line.update({"value": dec["value"], "unit": "tokens/s", "roofline": dec["roofline"]})
    ms = ((r["sel_ms"] + r["att_ms"] + r["dec_ms"]) / K)
    line.update({"n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms,
                 "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                 "dtype": "bf16", "data": "synthetic",
                 "config": workload_config(args, world, r["do_prefill"], r["do_decode"]),
                 "clocks": r["clocks"], "gpu_launches": r["launches"]})
    if "prefill" in r["e2e"]:
        line["e2e"] = r["e2e"]["prefill"]
    elif "decode" in r["e2e"]:
        line["e2e"] = r["e2e"]["decode"]
    if mixed is not None:
        # the mixed ragged workload, timed separately after the headline step
        line["mixed_ragged"] = mixed
    if gdn is not None:
        # the Gated DeltaNet layer, timed separately after the rest
        line["gated_deltanet"] = gdn
    if args.cpu and world == 1:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
