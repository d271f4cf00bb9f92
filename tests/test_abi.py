"""The C ABI library builds, loads and exports every entry point that include/qsa.h declares,
and rejects bad arguments on the host before touching a GPU (no compute call is made)."""
import ctypes
import os
import re

import pytest
import torch

import block_sparse_attention_40_b200 as qsa
from block_sparse_attention_40_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "qsa.h")).read()
    return sorted(set(re.findall(r"^QSA_API[^(]*?\b(qsa_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_bound_names():
    assert _declared() == sorted(B.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = qsa.load()
    for name in _declared():
        assert hasattr(lib, name), name
    # exported with default visibility in the dynamic symbol table
    out = os.popen(f"nm -D --defined-only {B.library_path()}").read()
    for name in _declared():
        assert re.search(rf"\bT {name}\b", out), name


def test_status_strings_and_version():
    assert B.status_string(0) == "QSA_OK"
    assert B.status_string(6) == "QSA_ERR_TIMEOUT"
    assert B.status_string(99) == "QSA_ERR_UNKNOWN"
    assert qsa.version() >= 100


def test_workspace_sizes_grow_with_work():
    small = B.prefill_workspace_size([0, 256], 16)
    big = B.prefill_workspace_size([0, 65536], 512)
    assert 0 < small < big
    # bad lengths and budgets are rejected (size 0 -> error)
    with pytest.raises(B.QSAError):
        B.prefill_workspace_size([0, 0], 512)
    with pytest.raises(B.QSAError):
        B.prefill_workspace_size([0, 100], 0)
    with pytest.raises(B.QSAError):
        B.prefill_workspace_size([0, 100], 4096)
    # select_mode 1 adds each score row's threshold record; other modes are refused
    assert B.prefill_workspace_size([0, 65536], 512, select_mode=1) > big
    with pytest.raises(B.QSAError):
        B.prefill_workspace_size([0, 100], 512, select_mode=2)
    # rows of 65,536 or more candidates (16-bit counters) take mode 0: no extra workspace
    long_seq = [0, 4 * 65536 + 8]
    assert (B.prefill_workspace_size(long_seq, 512, select_mode=1) ==
            B.prefill_workspace_size(long_seq, 512))
    lib = qsa.load()
    desc = B.CacheDesc(0, 0, 0, 0, 0, 64, 262144)
    n = lib.qsa_decode_workspace_size(ctypes.byref(desc), B._params(512))
    assert n > 64 * 65535 * 4
    desc = B.CacheDesc(0, 0, 0, 0, 0, 4, 1001)   # capacity not a multiple of 4
    assert lib.qsa_decode_workspace_size(ctypes.byref(desc), B._params(512)) == 0


def _p(v):
    return ctypes.c_void_p(v)


def test_host_side_argument_errors():
    lib = qsa.load()
    cu = (ctypes.c_int32 * 2)(0, 64)
    good = 0x10000
    prm = B._params(16)
    # null pointer
    r = lib.qsa_prefill(None, _p(good), _p(good), _p(good), _p(good), _p(good), _p(good), cu, 1,
                        _p(good), _p(good), 1 << 20, prm, None)
    assert B.STATUS[r] == "QSA_ERR_INVALID_ARG"
    # misaligned pointer
    r = lib.qsa_prefill(_p(good + 2), _p(good), _p(good), _p(good), _p(good), _p(good), _p(good),
                        cu, 1, _p(good), _p(good), 1 << 20, prm, None)
    assert B.STATUS[r] == "QSA_ERR_ALIGNMENT"
    # bad cumulative lengths
    bad = (ctypes.c_int32 * 3)(0, 64, 60)
    r = lib.qsa_prefill(_p(good), _p(good), _p(good), _p(good), _p(good), _p(good), _p(good), bad,
                        2, _p(good), _p(good), 1 << 30, prm, None)
    assert B.STATUS[r] == "QSA_ERR_INVALID_ARG"
    # workspace too small
    r = lib.qsa_prefill(_p(good), _p(good), _p(good), _p(good), _p(good), _p(good), _p(good), cu, 1,
                        _p(good), _p(good), 16, prm, None)
    assert B.STATUS[r] == "QSA_ERR_WORKSPACE"
    # budget zero
    r = lib.qsa_prefill(_p(good), _p(good), _p(good), _p(good), _p(good), _p(good), _p(good), cu, 1,
                        _p(good), _p(good), 1 << 30, B._params(0), None)
    assert B.STATUS[r] == "QSA_ERR_INVALID_ARG"
    # the testing fault hook takes 0 or 1 only, and is prefill-only
    r = lib.qsa_prefill(_p(good), _p(good), _p(good), _p(good), _p(good), _p(good), _p(good), cu, 1,
                        _p(good), _p(good), 1 << 30, B._params(16, debug_fault=2), None)
    assert B.STATUS[r] == "QSA_ERR_INVALID_ARG"
    desc = B.CacheDesc(good, good, good, good, good, 2, 64)
    assert lib.qsa_decode_workspace_size(ctypes.byref(desc), B._params(16, debug_fault=1)) == 0
    # append beyond capacity
    desc = B.CacheDesc(good, good, good, good, good, 2, 64)
    h_len = (ctypes.c_int32 * 2)(60, 10)
    r = lib.qsa_append_kv(ctypes.byref(desc), _p(good), _p(good), _p(good), 8, None, h_len, None)
    assert B.STATUS[r] == "QSA_ERR_CAPACITY"
    # decode with a length of 0 (no token appended)
    h_len = (ctypes.c_int32 * 2)(0, 10)
    desc = B.CacheDesc(good, good, good, good, good, 2, 64)
    r = lib.qsa_decode(_p(good), ctypes.byref(desc), _p(good), _p(good), _p(good), h_len, None,
                       None, _p(good), 1 << 30, B._params(16), None)
    assert B.STATUS[r] == "QSA_ERR_INVALID_ARG"


def test_cpu_tensors_are_refused():
    # the product has no CPU path: CPU tensors raise before any call
    q = torch.zeros((8, 24, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        B._need(q, "q", torch.bfloat16, (24, 128), 3)


def test_paged_cache_host_side_checks():
    lib = qsa.load()
    good = 0x10000
    prm = B._params(512)

    def paged(page_tokens=4096, pool=200, cap=262144, batch=64, table=good):
        return B.PagedCacheDesc(B.CacheDesc(good, good, good, good, good, batch, cap), table,
                                page_tokens, pool)

    base = B.CacheDesc(good, good, good, good, good, 64, 262144)
    n = lib.qsa_decode_paged_workspace_size(ctypes.byref(paged()), prm)
    assert n == lib.qsa_decode_workspace_size(ctypes.byref(base), prm) > 0
    for bad in (paged(page_tokens=1000), paged(page_tokens=0), paged(cap=262144 + 512),
                paged(pool=0), paged(table=0), paged(pool=1 << 20)):
        assert lib.qsa_decode_paged_workspace_size(ctypes.byref(bad), prm) == 0
    h_len = (ctypes.c_int32 * 2)(60, 10)
    r = lib.qsa_append_kv_paged(ctypes.byref(paged(batch=2, cap=1024, page_tokens=512)), _p(good),
                                _p(good), _p(good), 1000, None, h_len, None)
    assert B.STATUS[r] == "QSA_ERR_CAPACITY"
    r = lib.qsa_append_kv_paged(ctypes.byref(paged(batch=2, cap=1024, page_tokens=1000)),
                                _p(good), _p(good), _p(good), 8, None, h_len, None)
    assert B.STATUS[r] == "QSA_ERR_INVALID_ARG"
    r = lib.qsa_append_kv_paged(ctypes.byref(paged(batch=2, cap=1024, page_tokens=512,
                                                   table=good + 2)),
                                _p(good), _p(good), _p(good), 8, None, h_len, None)
    assert B.STATUS[r] == "QSA_ERR_ALIGNMENT"
    h_len = (ctypes.c_int32 * 2)(0, 10)
    r = lib.qsa_decode_paged(_p(good), ctypes.byref(paged(batch=2, cap=1024, page_tokens=512)),
                             _p(good), _p(good), _p(good), h_len, None, None, _p(good), 1 << 30,
                             B._params(16), None)
    assert B.STATUS[r] == "QSA_ERR_INVALID_ARG"


def test_sharded_decode_host_side_checks():
    # shard entry points refuse bad geometry before anything is enqueued (no GPU needed)
    lib = qsa.load()
    good = 0x10000
    prm = B._params(512)
    desc = B.CacheDesc(good, good, good, good, good, 4, 262144)
    h_len = (ctypes.c_int32 * 4)(*([1000] * 4))
    assert lib.qsa_decode_shard_workspace_size(ctypes.byref(desc), prm) == \
        lib.qsa_decode_workspace_size(ctypes.byref(desc), prm) > 0
    for block0 in (100, -128):   # shards start on 512-token (128-block) boundaries
        r = lib.qsa_decode_shard_select(_p(good), _p(good), ctypes.byref(desc), block0, _p(good),
                                        h_len, _p(good), _p(good), _p(good), _p(good), 1 << 30,
                                        prm, None)
        assert B.STATUS[r] == "QSA_ERR_INVALID_ARG"
        r = lib.qsa_decode_shard_attend(_p(good), ctypes.byref(desc), block0, _p(good), _p(good),
                                        _p(good), _p(good), _p(good), _p(good), _p(good), 1 << 30,
                                        prm, None)
        assert B.STATUS[r] == "QSA_ERR_INVALID_ARG"
    r = lib.qsa_decode_shard_select(_p(good + 4), _p(good), ctypes.byref(desc), 0, _p(good),
                                    h_len, _p(good), _p(good), _p(good), _p(good), 1 << 30, prm,
                                    None)
    assert B.STATUS[r] == "QSA_ERR_ALIGNMENT"
    # merge: shard count, budget and block range; too many candidates for shared memory
    for shards, k, nblk, want in ((0, 512, 1024, "QSA_ERR_INVALID_ARG"),
                                  (65, 512, 1024, "QSA_ERR_INVALID_ARG"),
                                  (4, 0, 1024, "QSA_ERR_INVALID_ARG"),
                                  (4, 512, 0, "QSA_ERR_INVALID_ARG"),
                                  (64, 1024, 262144, "QSA_ERR_UNSUPPORTED")):
        r = lib.qsa_merge_candidates(_p(good), _p(good), _p(good), shards, 4, k, nblk, _p(good),
                                     _p(good), _p(good), 1 << 20, None)
        assert B.STATUS[r] == want, (shards, k, nblk)
    r = lib.qsa_merge_candidates(_p(good), _p(good), _p(good), 4, 4, 512, 1024, _p(good),
                                 _p(good), _p(good), 16, None)
    assert B.STATUS[r] == "QSA_ERR_WORKSPACE"
    r = lib.qsa_combine_partials(_p(good), _p(good), _p(good), 0, 4, _p(good), None)
    assert B.STATUS[r] == "QSA_ERR_INVALID_ARG"
