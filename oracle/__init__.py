"""The oracle: a plain, slow CPU statement of dynamic block-sparse attention.

TEST INFRASTRUCTURE ONLY.  The product (the CUDA library and its Python
binding) never imports this package; only ``tests/``, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` do.

The arithmetic lives in ``dsa_oracle.c`` (plain C, int64 / double), which this
module compiles with gcc on first use and calls through ctypes.  The wrappers
below only marshal numpy arrays; they do no arithmetic of the method.

Pages the oracle follows (cited by title and section):
  * "Day-0 Adaptation for Massive LLMs: Overcoming Sparse Attention and MXFP4
    Expert Weights", section 4 (1) index selection, (2) KV cache layout,
    (3) prefill and decode.
  * "Day-0 Adaptation for Trillion-Parameter Models: Engineering Practices and
    Technical Breakdown", section 4 (sparse attention adaptation).
  * "Day-0 Readiness for Trillion-Parameter Models: Engineering Sparse
    Attention and Expert Weight Compression", sections "Index Selection Path"
    and "KV Cache Layout".
Parity pins for every function are in ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dsa_oracle.c")
_OUT_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_OUT_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

OK, BAD_ARG, BAD_PAGE, BAD_POS = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile dsa_oracle.c into oracle/_build/liboracle.so (plain gcc -O2)."""
    os.makedirs(_OUT_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # a mutated copy of the oracle may be substituted by the mutation tests
            override = os.environ.get("DSA_ORACLE_LIB")
            lib = ctypes.CDLL(override if override else build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            lib.oracle_kv_append.argtypes = [I, P, I, P, P, I, I, I, I, P, P, P, P]
            lib.oracle_kc_append.argtypes = [I, P, I, P, P, I, I, I, P, P]
            lib.oracle_index_score.argtypes = [I, P, P, P, I, I, I, P, I, P, P, I, P]
            lib.oracle_topk.argtypes = [I, P, P, I, P, I, P, I, P, P]
            lib.oracle_index_score_fp8.argtypes = [I, P, P, P, I, I, I, P, I, P, P, I, P]
            lib.oracle_index_score_fp8.restype = I
            lib.oracle_e4m3_times_512.argtypes = [ctypes.c_uint8, ctypes.POINTER(ctypes.c_int)]
            lib.oracle_e4m3_times_512.restype = ctypes.c_int64
            lib.oracle_sparse_attention.argtypes = [I, P, P, P, I, I, I, I, I, I, P, P, P,
                                                    P, P, I, ctypes.c_double, P, P]
            for f in (lib.oracle_kv_append, lib.oracle_kc_append, lib.oracle_index_score,
                      lib.oracle_topk, lib.oracle_sparse_attention):
                f.restype = I
            _lib = lib
    return _lib


def _c(a, dtype):
    """C-contiguous array of the given dtype (a copy only when needed)."""
    return np.ascontiguousarray(np.asarray(a), dtype=dtype)


def _ptr(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _check(rc, what):
    if rc != OK:
        raise ValueError(f"oracle {what} failed with status {rc}")


def queries_to_seq(cu_q) -> np.ndarray:
    """Sequence id of every query, from the ragged offsets cu_q[num_seqs+1]."""
    cu_q = np.asarray(cu_q, dtype=np.int64)
    return np.repeat(np.arange(len(cu_q) - 1, dtype=np.int32), np.diff(cu_q)).astype(np.int32)


def _inplace(a, dtype):
    if not (isinstance(a, np.ndarray) and a.flags.c_contiguous and a.dtype == dtype):
        raise ValueError(f"pool must be a C-contiguous numpy {np.dtype(dtype)} array (updated in place)")
    return a


def kv_append(block_table, seq_lens, cu_new, k_new, v_new, k_pool, v_pool, block_size):
    """Write the new tokens' K/V rows into the paged pools, in place (uint16 bf16 bits)."""
    bt = _c(block_table, np.int32)
    num_seqs, max_blocks = bt.shape
    _inplace(k_pool, np.uint16)
    _inplace(v_pool, np.uint16)
    num_pages, bs, hkv, d = k_pool.shape
    assert bs == block_size and v_pool.shape == k_pool.shape
    rc = _load().oracle_kv_append(
        num_seqs, _ptr(bt), max_blocks, _ptr(_c(seq_lens, np.int32)), _ptr(_c(cu_new, np.int32)),
        block_size, hkv, d, num_pages, _ptr(_c(k_new, np.uint16)), _ptr(_c(v_new, np.uint16)),
        _ptr(k_pool), _ptr(v_pool))
    _check(rc, "kv_append")


def kc_append(block_table, seq_lens, cu_new, kc_new, kc_pool, block_size):
    """Write the touched blocks' coarse keys into the coarse-key pool, in place."""
    bt = _c(block_table, np.int32)
    num_seqs, max_blocks = bt.shape
    _inplace(kc_pool, np.int8)
    rc = _load().oracle_kc_append(
        num_seqs, _ptr(bt), max_blocks, _ptr(_c(seq_lens, np.int32)), _ptr(_c(cu_new, np.int32)),
        block_size, kc_pool.shape[1], kc_pool.shape[0], _ptr(_c(kc_new, np.int8)), _ptr(kc_pool))
    _check(rc, "kc_append")


def index_score(q_seq, q_pos, block_table, block_size, kc_pool, q_idx, w):
    """int64 scores [T][max_blocks]; INT64_MIN where the block is not visible."""
    bt = _c(block_table, np.int32)
    kc = _c(kc_pool, np.int8)
    qi = _c(q_idx, np.int8)
    ww = _c(w, np.int32)
    T, H, dd = qi.shape
    out = np.empty((T, bt.shape[1]), dtype=np.int64)
    rc = _load().oracle_index_score(
        T, _ptr(_c(q_seq, np.int32)), _ptr(_c(q_pos, np.int32)), _ptr(bt), bt.shape[1],
        block_size, kc.shape[0], _ptr(kc), dd, _ptr(qi), _ptr(ww), H, _ptr(out))
    _check(rc, "index_score")
    return out


def e4m3_times_512(code: int):
    """(value of the FP8 E4M3 code times 2^9 as an int, is_nan)."""
    nan = ctypes.c_int(0)
    v = _load().oracle_e4m3_times_512(int(code) & 0xFF, ctypes.byref(nan))
    return int(v), bool(nan.value)


def index_score_fp8(q_seq, q_pos, block_table, block_size, kc_pool, q_idx, w):
    """Exact FP8 E4M3 block scores times 2^18, int64 [T][max_blocks]; INT64_MIN where
    not visible.  kc_pool and q_idx hold E4M3 codes (uint8)."""
    bt = _c(block_table, np.int32)
    kc = _c(kc_pool, np.uint8)
    qi = _c(q_idx, np.uint8)
    ww = _c(w, np.int32)
    T, H, dd = qi.shape
    out = np.empty((T, bt.shape[1]), dtype=np.int64)
    rc = _load().oracle_index_score_fp8(
        T, _ptr(_c(q_seq, np.int32)), _ptr(_c(q_pos, np.int32)), _ptr(bt), bt.shape[1],
        block_size, kc.shape[0], _ptr(kc), dd, _ptr(qi), _ptr(ww), H, _ptr(out))
    _check(rc, "index_score_fp8")
    return out


def topk(q_seq, q_pos, block_size, scores, k_per_seq, k_max):
    """(sel [T][k_max] int32 ascending, -1 padded; cnt [T] int32)."""
    sc = _c(scores, np.int64)
    T, max_blocks = sc.shape
    sel = np.empty((T, k_max), dtype=np.int32)
    cnt = np.empty((T,), dtype=np.int32)
    rc = _load().oracle_topk(T, _ptr(_c(q_seq, np.int32)), _ptr(_c(q_pos, np.int32)),
                             block_size, _ptr(sc), max_blocks, _ptr(_c(k_per_seq, np.int32)),
                             k_max, _ptr(sel), _ptr(cnt))
    _check(rc, "topk")
    return sel, cnt


def sparse_attention(q_seq, q_pos, block_table, block_size, q, k_pool, v_pool,
                     sel, cnt, sm_scale):
    """(out [T][Hq][D] float64, lse [T][Hq] float64); q/k/v are bf16 bit patterns."""
    bt = _c(block_table, np.int32)
    qq = _c(q, np.uint16)
    kp = _c(k_pool, np.uint16)
    vp = _c(v_pool, np.uint16)
    sl = _c(sel, np.int32)
    T, hq, d = qq.shape
    num_pages, bs, hkv, d2 = kp.shape
    assert d2 == d and bs == block_size
    out = np.empty((T, hq, d), dtype=np.float64)
    lse = np.empty((T, hq), dtype=np.float64)
    rc = _load().oracle_sparse_attention(
        T, _ptr(_c(q_seq, np.int32)), _ptr(_c(q_pos, np.int32)), _ptr(bt), bt.shape[1],
        block_size, num_pages, hq, hkv, d, _ptr(qq), _ptr(kp), _ptr(vp), _ptr(sl),
        _ptr(_c(cnt, np.int32)), sl.shape[1], float(sm_scale), _ptr(out), _ptr(lse))
    _check(rc, "sparse_attention")
    return out, lse
