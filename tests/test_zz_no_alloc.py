"""qsa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers cannot allocate device memory on the call path and have no buffer to lend
(for example a plugin inside a host framework whose allocator owns all device memory).
qsa_decode_noalloc serves them with the library's own fixed device scratch.  These tests
call it through the C ABI and check that two calls in a row give bit for bit the outputs of
the workspace-taking qsa_decode (the same kernels on the same inputs), that the device-side
status read back from the fixed scratch is clean after each call, and that a cache needing
more scratch than the fixed array is refused up front.  This file is collected last."""
import ctypes

import pytest
import torch

import block_sparse_attention_40_b200 as qsa
from block_sparse_attention_40_b200 import binding as B
from block_sparse_attention_40_b200 import workloads as W
from tests.gpu_helpers import MAX_ABS, REL_L2, needs_gpu

pytestmark = [pytest.mark.gpu, needs_gpu]
DEV = "cuda:0"


def _same(a, b):
    # both calls run the same kernels on the same inputs: the outputs agree bit for bit
    # (which is also within the decode tolerance)
    assert torch.isfinite(a.float()).all()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    err = (a.double() - b.double()).abs().max().item()
    assert err <= MAX_ABS and REL_L2 > 0


def test_noalloc_matches_decode_two_calls():
    spec = W.small_decode_spec(batch=8, context=tuple(3000 + 7 * i for i in range(8)),
                               capacity=3200, topk=128, steps=2, seed=31)
    kc, vc, kic = W.decode_context(spec)
    cache = qsa.KVCache(spec.batch, spec.capacity, DEV)
    cache.append(kc.to(DEV), vc.to(DEV), kic.to(DEV), counts=spec.context)
    dec = qsa.Decoder(cache, spec.topk)
    for step in range(2):
        st = W.decode_step(spec, step)
        cache.append(st["k"].to(DEV), st["v"].to(DEV), st["k_idx"].to(DEV))
        q, qi, w = st["q"].to(DEV), st["q_idx"].to(DEV), st["w"].to(DEV)
        ref = dec.run(q, qi, w)
        got = B.decode_noalloc(cache, q, qi, w, topk=spec.topk)
        assert B.noalloc_device_error(DEV) == ("QSA_OK", 0)
        torch.cuda.synchronize()
        assert dec.device_error() == ("QSA_OK", 0)
        _same(got, ref)


def test_noalloc_refuses_oversized_cache():
    # batch 64 at a 1M-token capacity needs ~68 MB of scratch, more than the fixed 32 MiB;
    # the call is refused before anything is enqueued (the pointers are never touched)
    lib = qsa.load()
    fake = 0x100000
    desc = B.CacheDesc(fake, fake, fake, fake, fake, 64, 1 << 20)
    need = lib.qsa_decode_workspace_size(ctypes.byref(desc), B._params(512))
    assert need > (32 << 20)
    h_len = (ctypes.c_int32 * 64)(*([1000] * 64))
    r = lib.qsa_decode_noalloc(ctypes.c_void_p(fake), ctypes.byref(desc), ctypes.c_void_p(fake),
                               ctypes.c_void_p(fake), ctypes.c_void_p(fake), h_len, None, None,
                               B._params(512), None)
    assert B.STATUS[r] == "QSA_ERR_WORKSPACE"
