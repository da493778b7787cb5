"""ctypes binding of libdsa.so (the C ABI in include/dsa.h).

Only argument marshalling lives here: torch tensors are turned into device
pointers and the current CUDA stream handle; every step of the method runs
in the library's CUDA kernels.  There is no CPU fallback: if the library
cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

_lock = threading.Lock()
_lib = None

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_RANGE, DSA_ERR_WORKSPACE, DSA_ERR_CUDA = range(6)
DEV_ERR_PAGE, DEV_ERR_POS, DEV_ERR_SEL, DEV_ERR_K, DEV_ERR_WAIT, DEV_ERR_VALUE = 1, 2, 4, 8, 16, 32

c_i32 = ctypes.c_int32
c_vp = ctypes.c_void_p


class KvCacheC(ctypes.Structure):
    _fields_ = [("k_pool", c_vp), ("v_pool", c_vp), ("kc_pool", c_vp), ("num_pages", c_i32),
                ("block_size", c_i32), ("num_kv_heads", c_i32), ("head_dim", c_i32), ("idx_dim", c_i32)]


class SeqsC(ctypes.Structure):
    _fields_ = [("block_table", c_vp), ("max_blocks", c_i32), ("seq_lens", c_vp), ("num_seqs", c_i32)]


class QueriesC(ctypes.Structure):
    _fields_ = [("cu_q", c_vp), ("q_pos", c_vp), ("total_q", c_i32)]


# exported symbol -> (argtypes, restype); mirrors include/dsa.h
P = ctypes.POINTER
SIGNATURES = {
    "dsa_kv_append": ([P(KvCacheC), P(SeqsC), c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp], c_i32),
    "dsa_index_score": ([P(KvCacheC), P(SeqsC), P(QueriesC), c_vp, c_vp, c_i32, c_i32, c_vp, c_vp, c_vp],
                        c_i32),
    "dsa_topk_blocks": ([P(SeqsC), P(QueriesC), c_vp, c_vp, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp], c_i32),
    "dsa_index_score_i64": ([P(KvCacheC), P(SeqsC), P(QueriesC), c_vp, c_vp, c_i32, c_vp, c_vp, c_vp], c_i32),
    "dsa_index_score_fp8": ([P(KvCacheC), P(SeqsC), P(QueriesC), c_vp, c_vp, c_i32, c_i32, c_vp, c_vp, c_vp],
                            c_i32),
    "dsa_topk_blocks_i64": ([P(SeqsC), P(QueriesC), c_vp, c_vp, c_i32, c_i32, c_vp, c_vp, c_vp, c_vp], c_i32),
    "dsa_select_blocks_workspace_size": ([c_i32], ctypes.c_size_t),
    "dsa_select_blocks": ([P(KvCacheC), P(SeqsC), P(QueriesC), c_vp, c_vp, c_i32, c_i32, c_vp, c_i32, c_vp, c_vp,
                           c_vp, ctypes.c_size_t, c_vp, c_vp], c_i32),
    "dsa_select_blocks_append": ([P(KvCacheC), P(SeqsC), P(QueriesC), c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp,
                                  c_i32, c_i32, c_vp, c_i32, c_vp, c_vp, c_vp, ctypes.c_size_t, c_vp, c_vp], c_i32),
    "dsa_sparse_attn_decode_workspace_size": ([c_i32, c_i32, c_i32, c_i32], ctypes.c_size_t),
    "dsa_sparse_attn_decode": ([P(KvCacheC), P(SeqsC), P(QueriesC), c_vp, c_i32, c_vp, c_vp, c_i32,
                                ctypes.c_float, c_vp, c_vp, c_vp, ctypes.c_size_t, c_vp, c_vp], c_i32),
    "dsa_sparse_attn_prefill": ([P(KvCacheC), P(SeqsC), P(QueriesC), c_vp, c_i32, c_vp, c_vp, c_i32,
                                 ctypes.c_float, c_vp, c_vp, c_vp, c_vp], c_i32),
    "dsa_sparse_attn_decode_noalloc": ([P(KvCacheC), P(SeqsC), P(QueriesC), c_vp, c_i32, c_vp, c_vp, c_i32,
                                        ctypes.c_float, c_vp, c_vp, c_vp, c_vp], c_i32),
    "dsa_decode_fused_workspace_size": ([c_i32, c_i32, c_i32, c_i32], ctypes.c_size_t),
    "dsa_decode_fused": ([P(KvCacheC), P(SeqsC), P(QueriesC), c_vp, c_i32, c_vp, c_vp, c_vp, c_vp, c_vp, c_i32,
                          c_i32, c_vp, c_i32, c_vp, c_i32, ctypes.c_float, c_vp, c_vp, c_vp, c_vp, c_vp,
                          ctypes.c_size_t, c_vp, c_vp], c_i32),
    "dsa_stager_create": ([c_i32, c_vp, P(c_vp)], c_i32),
    "dsa_stager_destroy": ([c_vp], c_i32),
    "dsa_stager_begin": ([c_vp, c_i32, c_i32, c_vp, c_vp, c_vp], c_i32),
    "dsa_stager_end": ([c_vp, c_i32, c_i32, c_vp, c_vp, c_vp], c_i32),
    "dsa_stager_wait": ([c_vp, c_i32], c_i32),
    "dsa_stager_join": ([c_vp], c_i32),
    "dsa_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "dsa_version": ([], ctypes.c_int),
}


class DsaError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


def lib_path() -> str:
    return _build.LIB


def load():
    """Load libdsa.so (building it first if it is missing or older than its
    sources and nvcc is available).  Raises if the library cannot be loaded."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if _build.is_stale():
            try:
                _build.build()
            except Exception as e:   # no toolchain here: a present library still loads
                if not os.path.exists(_build.LIB):
                    raise RuntimeError(f"libdsa.so is missing and could not be built: {e}") from e
        lib = ctypes.CDLL(_build.LIB)
        for name, (argt, rest) in SIGNATURES.items():
            f = getattr(lib, name)
            f.argtypes = argt
            f.restype = rest
        _lib = lib
        return lib


def check(fn: str, status: int) -> None:
    if status != DSA_OK:
        msg = load().dsa_status_string(status).decode()
        raise DsaError(fn, status, msg)
