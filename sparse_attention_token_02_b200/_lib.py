"""ctypes view of ``libdsa_indexer.so`` (the C ABI declared in include/dsa_indexer.h).

Loading fails loudly when the library has not been built: there is no other
implementation of these calls in this package.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# DSA_INDEXER_LIB may name another build of the same library (e.g. a tuning variant)
LIB_PATH = os.environ.get("DSA_INDEXER_LIB") or os.path.join(_HERE, "libdsa_indexer.so")

DSA_BF16, DSA_FP8_E4M3, DSA_F32 = 0, 1, 2
STATUS_NAMES = {0: "DSA_OK", 1: "DSA_ERR_INVALID_ARG", 2: "DSA_ERR_UNSUPPORTED", 3: "DSA_ERR_ALLOC",
                4: "DSA_ERR_CUDA", 5: "DSA_ERR_DEVICE_CHECK"}

# every symbol include/dsa_indexer.h declares
EXPORTED = (
    "dsa_indexer_kcache_append",
    "dsa_quantize_rows_fp8",
    "dsa_indexer_prefill",
    "dsa_indexer_decode",
    "dsa_indexer_decode_noalloc",
    "dsa_indexer_decode_host",
    "dsa_indexer_decode_host_async",
    "dsa_indexer_prefill_host",
    "dsa_indexer_prefill_host_async",
    "dsa_indexer_decode_compressed",
    "dsa_indexer_prefill_compressed",
    "dsa_indexer_kcache_append_rope",
    "dsa_rope_queries",
    "dsa_gather_rows",
    "dsa_selection_rows",
    "dsa_sort_selection",
    "dsa_indexer_scores",
    "dsa_indexer_workspace_bytes",
    "dsa_set_workspace",
    "dsa_check_device_errors",
    "dsa_selftest_wait_expiry",
    "dsa_set_profile_events",
    "dsa_kernel_launch_count",
    "dsa_get_last_error",
    "dsa_version",
)


class KCache(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("k_scale", ctypes.c_void_p), ("capacity_rows", ctypes.c_int64),
                ("d_I", ctypes.c_int32), ("dtype", ctypes.c_int)]


class Rope(ctypes.Structure):
    _fields_ = [("rope_dim", ctypes.c_int32), ("interleaved", ctypes.c_int32), ("base", ctypes.c_double)]


class Query(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("scale", ctypes.c_void_p), ("dtype", ctypes.c_int),
                ("H_I", ctypes.c_int32), ("d_I", ctypes.c_int32)]


class Batch(ctypes.Structure):
    _fields_ = [("num_seqs", ctypes.c_int32), ("seq_lens", ctypes.c_void_p), ("q_lens", ctypes.c_void_p),
                ("k_base", ctypes.c_void_p)]


class DsaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None


def load() -> ctypes.CDLL:
    """Load the library once; raise if it is missing (build it with sparse_attention_token_02_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: run `python -m sparse_attention_token_02_b200.build` "
                           "(the indexer has no implementation other than this CUDA library)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, I64, V = ctypes.POINTER, ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p
    st = ctypes.c_int
    lib.dsa_indexer_kcache_append.argtypes = [P(KCache), V, ctypes.c_int, V, I32, V]
    lib.dsa_indexer_kcache_append.restype = st
    lib.dsa_quantize_rows_fp8.argtypes = [V, ctypes.c_int, I64, I32, V, V, V]
    lib.dsa_quantize_rows_fp8.restype = st
    for name in ("dsa_indexer_prefill", "dsa_indexer_decode"):
        fn = getattr(lib, name)
        fn.argtypes = [P(Query), P(KCache), V, P(Batch), I32, V, V, V]
        fn.restype = st
    lib.dsa_indexer_decode_noalloc.argtypes = [P(Query), P(KCache), V, P(Batch), I32, V, V, V, V]
    lib.dsa_indexer_decode_noalloc.restype = st
    for name in ("dsa_indexer_decode_host", "dsa_indexer_prefill_host"):
        fn = getattr(lib, name)
        fn.argtypes = [P(Query), P(KCache), V, V, ctypes.c_int, V, I32, P(Batch), I32, V, V, V]
        fn.restype = st
        fn = getattr(lib, name + "_async")
        fn.argtypes = [P(Query), P(KCache), V, V, ctypes.c_int, V, I32, P(Batch), I32, V, V, V, V]
        fn.restype = st
    lib.dsa_indexer_decode_compressed.argtypes = [P(Query), P(KCache), V, P(Batch), I32, I32, V, V, V]
    lib.dsa_indexer_decode_compressed.restype = st
    lib.dsa_indexer_prefill_compressed.argtypes = [P(Query), P(KCache), V, P(Batch), I32, I32, V, V, V]
    lib.dsa_indexer_prefill_compressed.restype = st
    lib.dsa_indexer_kcache_append_rope.argtypes = [P(KCache), V, ctypes.c_int, V, V, I32, P(Rope), V]
    lib.dsa_indexer_kcache_append_rope.restype = st
    lib.dsa_rope_queries.argtypes = [V, ctypes.c_int, I64, I32, I32, V, P(Rope), V, ctypes.c_int, V, V]
    lib.dsa_rope_queries.restype = st
    lib.dsa_gather_rows.argtypes = [V, I64, I32, V, V, I64, I32, V, V]
    lib.dsa_gather_rows.restype = st
    lib.dsa_selection_rows.argtypes = [V, V, I64, I32, V, V]
    lib.dsa_selection_rows.restype = st
    lib.dsa_sort_selection.argtypes = [V, V, I64, I32, V]
    lib.dsa_sort_selection.restype = st
    lib.dsa_indexer_scores.argtypes = [P(Query), P(KCache), V, P(Batch), V, I64, V]
    lib.dsa_indexer_scores.restype = st
    lib.dsa_indexer_workspace_bytes.argtypes = [P(Query), P(Batch), I32]
    lib.dsa_indexer_workspace_bytes.restype = ctypes.c_size_t
    lib.dsa_set_workspace.argtypes = [V, ctypes.c_size_t, V]
    lib.dsa_set_workspace.restype = st
    lib.dsa_check_device_errors.argtypes = [V]
    lib.dsa_check_device_errors.restype = st
    lib.dsa_selftest_wait_expiry.argtypes = [I64, V]
    lib.dsa_selftest_wait_expiry.restype = st
    lib.dsa_set_profile_events.argtypes = [V, V, V]
    lib.dsa_set_profile_events.restype = st
    lib.dsa_kernel_launch_count.argtypes = []
    lib.dsa_kernel_launch_count.restype = ctypes.c_uint64
    lib.dsa_get_last_error.argtypes = []
    lib.dsa_get_last_error.restype = ctypes.c_char_p
    lib.dsa_version.argtypes = []
    lib.dsa_version.restype = ctypes.c_char_p
    _lib = lib
    return lib


def check(status: int) -> None:
    if status != 0:
        msg = load().dsa_get_last_error().decode(errors="replace")
        raise DsaError(status, msg)
