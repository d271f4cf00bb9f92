"""Qwen Sparse Attention (QSA) on NVIDIA B200 (sm_100a).

The kernels and the C ABI live in ``csrc/`` and build into ``lib/libqsa.so`` (declared in
``include/qsa.h``).  ``binding`` is the thin ctypes layer that tests and benchmarks call;
``workloads`` draws the seeded synthetic inputs.
"""
from .binding import (KVCache, PagedKVCache, Decoder, Prefill, QSAError, compress, index_scores,  # noqa: F401
                      gated_deltanet, last_device_error, load, prefill, prefill_select, topk,
                      version)
