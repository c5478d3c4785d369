"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects invalid arguments before touching CUDA."""

import ctypes
import os
import re

import numpy as np
import pytest

from sparse_attention_token_02_b200 import _lib

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "dsa_indexer.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from sparse_attention_token_02_b200 import build
        build.build()
    return _lib.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"DSA_API\s+[\w\s\*]*?\b(dsa_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for must in ("dsa_indexer_prefill", "dsa_indexer_decode", "dsa_indexer_kcache_append"):
        assert must in names
    assert set(names) == set(_lib.EXPORTED)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert lib.dsa_version().decode().startswith("dsa_indexer")


def test_only_c_api_symbols_are_exported(lib):
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True, text=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    assert {s for s in exported if s.startswith("dsa_")} == set(declared_symbols())


def _fake_cache(capacity=1024, d=128, dtype=_lib.DSA_BF16, k=0x10000, k_scale=None):
    return _lib.KCache(k, k_scale, capacity, d, dtype)


def _batch(seq, ql=None, kb=None):
    seq = np.asarray(seq, np.int32)
    ql = None if ql is None else np.asarray(ql, np.int32)
    kb = None if kb is None else np.asarray(kb, np.int64)
    b = _lib.Batch(len(seq), seq.ctypes.data, None if ql is None else ql.ctypes.data,
                   None if kb is None else kb.ctypes.data)
    return b, (seq, ql, kb)


@pytest.mark.parametrize("case,expect", [
    ("null_cache", "INVALID_ARG"),
    ("bad_d", "UNSUPPORTED"),
    ("fp8_no_scale", "INVALID_ARG"),
    ("q_gt_seq", "INVALID_ARG"),
    ("capacity", "INVALID_ARG"),
    ("top_k0", "INVALID_ARG"),
    ("decode_qlen", "INVALID_ARG"),
    ("dtype_mismatch", "INVALID_ARG"),
    ("misaligned", "INVALID_ARG"),
    ("null_score_long_row", "INVALID_ARG"),
])
def test_invalid_arguments_are_rejected_before_cuda(lib, case, expect):
    kc = _fake_cache()
    q = _lib.Query(0x20000, None, _lib.DSA_BF16, 64, 128)
    b, keep = _batch([100], [100])
    fn = lib.dsa_indexer_prefill
    top_k = 16
    if case == "null_cache":
        kc_p = None
    else:
        kc_p = ctypes.byref(kc)
    if case == "bad_d":
        kc.d_I = 96
    if case == "fp8_no_scale":
        kc.dtype = _lib.DSA_FP8_E4M3
    if case == "q_gt_seq":
        b, keep = _batch([10], [11])
    if case == "capacity":
        b, keep = _batch([100], [1], [1000])
    if case == "top_k0":
        top_k = 0
    if case == "decode_qlen":
        fn = lib.dsa_indexer_decode
        b, keep = _batch([100], [5])
    if case == "dtype_mismatch":
        q.dtype = _lib.DSA_FP8_E4M3
    if case == "misaligned":
        q.data = 0x20004
    out_score = None if case == "null_score_long_row" else ctypes.c_void_p(0x50000)   # bypass needs seq <= top_k
    st = fn(ctypes.byref(q), kc_p, ctypes.c_void_p(0x30000), ctypes.byref(b), top_k, ctypes.c_void_p(0x40000),
            out_score, None)
    assert _lib.STATUS_NAMES[st] == "DSA_ERR_" + expect, lib.dsa_get_last_error()
    assert lib.dsa_get_last_error()


def test_append_and_quantise_argument_checks(lib):
    kc = _fake_cache()
    st = lib.dsa_indexer_kcache_append(ctypes.byref(kc), ctypes.c_void_p(0x10000), 7, ctypes.c_void_p(0x20000), 4, None)
    assert _lib.STATUS_NAMES[st] == "DSA_ERR_INVALID_ARG"
    st = lib.dsa_quantize_rows_fp8(ctypes.c_void_p(0x10000), _lib.DSA_BF16, 4, 100, ctypes.c_void_p(0x20000),
                                   ctypes.c_void_p(0x30000), None)
    assert _lib.STATUS_NAMES[st] == "DSA_ERR_INVALID_ARG"        # row_len not a multiple of 16
    assert lib.dsa_indexer_kcache_append(ctypes.byref(kc), None, 0, None, 0, None) == 0   # n == 0: nothing to do


def test_workspace_bytes_grows_with_the_triangle(lib):
    q = _lib.Query(0, None, _lib.DSA_BF16, 64, 128)
    small, k1 = _batch([1000])
    big, k2 = _batch([4000])
    a = lib.dsa_indexer_workspace_bytes(ctypes.byref(q), ctypes.byref(small), 2048)
    c = lib.dsa_indexer_workspace_bytes(ctypes.byref(q), ctypes.byref(big), 2048)
    assert a > 1000 * 1001 // 2 * 4 and c > 4000 * 4001 // 2 * 4 and c > a


def test_wait_expiry_self_test_checks_its_limit(lib):
    for bad in (0, -5, 3_000_000_000):
        st = lib.dsa_selftest_wait_expiry(bad, None)
        assert _lib.STATUS_NAMES[st] == "DSA_ERR_INVALID_ARG", lib.dsa_get_last_error()


def test_prebuilt_host_batch_is_used_as_given():
    from sparse_attention_token_02_b200 import api
    hb = api.host_batch([300, 7], [2, 1], [0, 400])
    assert api._batch(hb, None, None) is hb
    assert hb.total_q == 3 and hb.c.num_seqs == 2
    with pytest.raises(ValueError, match="host_batch"):
        api._batch(hb, [2, 1], None)
    fresh = api._batch([300, 7], None, None)
    assert fresh.total_q == 307 and fresh.ql is None
