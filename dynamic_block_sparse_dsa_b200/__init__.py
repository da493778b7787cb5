"""dynamic_block_sparse_dsa_b200 -- query-driven dynamic block-sparse attention on B200.

Thin Python face of the CUDA library ``libdsa.so`` (C ABI: include/dsa.h).
The calls keep the C names and only marshal torch tensors (device pointers,
the current CUDA stream); all of the method runs in the library's kernels:

    kv_append            new tokens -> paged K/V pool + coarse keys
    index_score          int8 indexer: block scores of each query
    topk_blocks          own block + Top-(K-1) blocks, ascending logical ids
    sparse_attn_decode   exact attention over the selected blocks (split-KV)
    sparse_attn_prefill  same, each (query, KV head) pair inside one CTA

and the fused forms: select_blocks (score + Top-K, no score matrix),
select_blocks_append (the same with the append in one launch, decode),
decode_fused (a whole decode step in one launch), sparse_attn_decode_noalloc
(decode attention without a caller workspace), and step() chaining one pass.

Pages followed (cited by title and section): "Day-0 Adaptation for Massive
LLMs: Overcoming Sparse Attention and MXFP4 Expert Weights", section 4;
"Day-0 Readiness for Trillion-Parameter Models: Engineering Sparse Attention
and Expert Weight Compression", sections "Index Selection Path", "KV Cache
Layout", "Differentiated Adaptation of Prefill and Decode".
"""
from __future__ import annotations

import ctypes
import math
from dataclasses import dataclass
from typing import Optional

import torch

from . import _lib
from ._lib import DsaError, load

__all__ = [
    "PagedKVCache", "SeqBatch", "QueryBatch", "DsaError", "load",
    "kv_append", "index_score", "topk_blocks", "select_blocks", "select_blocks_append", "sparse_attn_decode",
    "sparse_attn_prefill", "decode_fused", "decode_workspace_size", "select_workspace_size",
    "decode_fused_workspace_size", "sparse_attn_decode_noalloc", "step", "PreparedStep", "Stager", "index_score_i64",
    "index_score_fp8", "topk_blocks_i64",
]

BLOCK_SIZE = 64
HEAD_DIM = 128
IDX_DIM = 64


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("dynamic_block_sparse_dsa_b200 works on CUDA tensors only (no CPU path)")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _addr(t: torch.Tensor) -> int:
    """Device address of a tensor, as a plain int (for ctypes struct fields)."""
    return _ptr(t).value


def _stream(stream) -> ctypes.c_void_p:
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _expect(t: torch.Tensor, dtype, name):
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


@dataclass
class PagedKVCache:
    """Block-paged pools: k/v bf16 [num_pages][block_size][num_kv_heads][128], kc int8
    [num_pages][64]; block_size (64, 128, 256 or 512 tokens) is the pools' second dimension."""
    k_pool: torch.Tensor
    v_pool: torch.Tensor
    kc_pool: torch.Tensor

    def ctype(self) -> _lib.KvCacheC:
        _expect(self.k_pool, torch.bfloat16, "k_pool")
        _expect(self.v_pool, torch.bfloat16, "v_pool")
        if self.kc_pool.element_size() != 1:   # int8 codes, or E4M3 codes for index_score_fp8
            raise ValueError(f"kc_pool must hold one byte per element, got {self.kc_pool.dtype}")
        n, bs, hkv, d = self.k_pool.shape
        return _lib.KvCacheC(_addr(self.k_pool), _addr(self.v_pool), _addr(self.kc_pool), n, bs, hkv, d,
                             self.kc_pool.shape[1])

    @property
    def num_kv_heads(self) -> int:
        return self.k_pool.shape[2]

    @property
    def block_size(self) -> int:
        return self.k_pool.shape[1]


@dataclass
class SeqBatch:
    """block_table int32 [num_seqs][max_blocks]; seq_lens int32 [num_seqs] (after append)."""
    block_table: torch.Tensor
    seq_lens: torch.Tensor

    def ctype(self) -> _lib.SeqsC:
        _expect(self.block_table, torch.int32, "block_table")
        _expect(self.seq_lens, torch.int32, "seq_lens")
        ns, mb = self.block_table.shape
        return _lib.SeqsC(_addr(self.block_table), mb, _addr(self.seq_lens), ns)


@dataclass
class QueryBatch:
    """cu_q int32 [num_seqs+1] ragged offsets; q_pos int32 [total_q] positions."""
    cu_q: torch.Tensor
    q_pos: torch.Tensor

    def ctype(self) -> _lib.QueriesC:
        _expect(self.cu_q, torch.int32, "cu_q")
        _expect(self.q_pos, torch.int32, "q_pos")
        return _lib.QueriesC(_addr(self.cu_q), _addr(self.q_pos), self.q_pos.numel())

    @property
    def total_q(self) -> int:
        return self.q_pos.numel()


def kv_append(cache: PagedKVCache, seqs: SeqBatch, cu_new: torch.Tensor, k_new: torch.Tensor,
              v_new: torch.Tensor, kc_new: Optional[torch.Tensor] = None,
              dev_err: Optional[torch.Tensor] = None, stream=None) -> None:
    lib = load()
    c, s = cache.ctype(), seqs.ctype()
    _lib.check("dsa_kv_append", lib.dsa_kv_append(
        ctypes.byref(c), ctypes.byref(s), _ptr(cu_new), k_new.shape[0], _ptr(k_new), _ptr(v_new),
        _ptr(kc_new), _ptr(dev_err), _stream(stream)))


def index_score(cache: PagedKVCache, seqs: SeqBatch, queries: QueryBatch, q_idx: torch.Tensor,
                w: torch.Tensor, w_abs_max: int = 16, scores: Optional[torch.Tensor] = None,
                dev_err: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """int32 scores [total_q][max_blocks]; entries past a query's own block are left as given."""
    lib = load()
    _expect(q_idx, torch.int8, "q_idx")
    _expect(w, torch.int32, "w")
    if scores is None:
        scores = torch.empty((queries.total_q, seqs.block_table.shape[1]), dtype=torch.int32,
                             device=q_idx.device)
    c, s, q = cache.ctype(), seqs.ctype(), queries.ctype()
    _lib.check("dsa_index_score", lib.dsa_index_score(
        ctypes.byref(c), ctypes.byref(s), ctypes.byref(q), _ptr(q_idx), _ptr(w), q_idx.shape[1],
        int(w_abs_max), _ptr(scores), _ptr(dev_err), _stream(stream)))
    return scores


def topk_blocks(seqs: SeqBatch, queries: QueryBatch, scores: torch.Tensor, k_per_seq: torch.Tensor,
                k_max: int, sel: Optional[torch.Tensor] = None, cnt: Optional[torch.Tensor] = None,
                dev_err: Optional[torch.Tensor] = None, stream=None, block_size: int = BLOCK_SIZE):
    """(sel int32 [total_q][k_max] ascending logical ids, -1 padded; cnt int32 [total_q]).
    ``block_size`` is the tokens per block of the cache the scores came from."""
    lib = load()
    dev = scores.device
    if sel is None:
        sel = torch.empty((queries.total_q, k_max), dtype=torch.int32, device=dev)
    if cnt is None:
        cnt = torch.empty((queries.total_q,), dtype=torch.int32, device=dev)
    s, q = seqs.ctype(), queries.ctype()
    _lib.check("dsa_topk_blocks", lib.dsa_topk_blocks(
        ctypes.byref(s), ctypes.byref(q), _ptr(scores), _ptr(k_per_seq), int(k_max), int(block_size), _ptr(sel),
        _ptr(cnt), _ptr(dev_err), _stream(stream)))
    return sel, cnt


def index_score_i64(cache: PagedKVCache, seqs: SeqBatch, queries: QueryBatch, q_idx: torch.Tensor, w: torch.Tensor,
                    scores: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None, stream=None):
    """int64 scores of the int8 indexer for any int32 weights: [total_q][max_blocks]."""
    lib = load()
    _expect(q_idx, torch.int8, "q_idx")
    _expect(w, torch.int32, "w")
    if scores is None:
        scores = torch.empty((queries.total_q, seqs.block_table.shape[1]), dtype=torch.int64, device=q_idx.device)
    c, s, q = cache.ctype(), seqs.ctype(), queries.ctype()
    _lib.check("dsa_index_score_i64", lib.dsa_index_score_i64(
        ctypes.byref(c), ctypes.byref(s), ctypes.byref(q), _ptr(q_idx), _ptr(w), q_idx.shape[1], _ptr(scores),
        _ptr(dev_err), _stream(stream)))
    return scores


def index_score_fp8(cache: PagedKVCache, seqs: SeqBatch, queries: QueryBatch, q_idx_e4m3: torch.Tensor,
                    w: torch.Tensor, w_abs_max: int = 16, scores: Optional[torch.Tensor] = None,
                    dev_err: Optional[torch.Tensor] = None, stream=None):
    """Exact FP8 (E4M3) block scores times 2^18, int64 [total_q][max_blocks].  ``q_idx_e4m3``
    and ``cache.kc_pool`` hold E4M3 codes (uint8, or torch.float8_e4m3fn viewed as uint8)."""
    lib = load()
    if q_idx_e4m3.dtype == torch.float8_e4m3fn:
        q_idx_e4m3 = q_idx_e4m3.view(torch.uint8)
    _expect(q_idx_e4m3, torch.uint8, "q_idx_e4m3")
    _expect(w, torch.int32, "w")
    if scores is None:
        scores = torch.empty((queries.total_q, seqs.block_table.shape[1]), dtype=torch.int64,
                             device=q_idx_e4m3.device)
    c, s, q = cache.ctype(), seqs.ctype(), queries.ctype()
    _lib.check("dsa_index_score_fp8", lib.dsa_index_score_fp8(
        ctypes.byref(c), ctypes.byref(s), ctypes.byref(q), _ptr(q_idx_e4m3), _ptr(w), q_idx_e4m3.shape[1],
        int(w_abs_max), _ptr(scores), _ptr(dev_err), _stream(stream)))
    return scores


def topk_blocks_i64(seqs: SeqBatch, queries: QueryBatch, scores: torch.Tensor, k_per_seq: torch.Tensor, k_max: int,
                    block_size: int = BLOCK_SIZE, sel: Optional[torch.Tensor] = None,
                    cnt: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None, stream=None):
    """topk_blocks over int64 scores (index_score_i64 / index_score_fp8)."""
    lib = load()
    _expect(scores, torch.int64, "scores")
    dev = scores.device
    if sel is None:
        sel = torch.empty((queries.total_q, k_max), dtype=torch.int32, device=dev)
    if cnt is None:
        cnt = torch.empty((queries.total_q,), dtype=torch.int32, device=dev)
    s, q = seqs.ctype(), queries.ctype()
    _lib.check("dsa_topk_blocks_i64", lib.dsa_topk_blocks_i64(
        ctypes.byref(s), ctypes.byref(q), _ptr(scores), _ptr(k_per_seq), int(k_max), int(block_size), _ptr(sel),
        _ptr(cnt), _ptr(dev_err), _stream(stream)))
    return sel, cnt


def select_workspace_size(total_q: int) -> int:
    return int(load().dsa_select_blocks_workspace_size(total_q))


def select_blocks(cache: PagedKVCache, seqs: SeqBatch, queries: QueryBatch, q_idx: torch.Tensor,
                  w: torch.Tensor, k_per_seq: torch.Tensor, k_max: int, w_abs_max: int = 16,
                  sel: Optional[torch.Tensor] = None, cnt: Optional[torch.Tensor] = None,
                  workspace: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None, stream=None):
    """index_score + topk_blocks fused (no score matrix): (sel, cnt).  ``workspace``
    is a zero-initialised uint8 tensor of select_workspace_size() bytes (allocated here if None)."""
    lib = load()
    _expect(q_idx, torch.int8, "q_idx")
    _expect(w, torch.int32, "w")
    dev = q_idx.device
    T = queries.total_q
    if sel is None:
        sel = torch.empty((T, k_max), dtype=torch.int32, device=dev)
    if cnt is None:
        cnt = torch.empty((T,), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.zeros(select_workspace_size(T), dtype=torch.uint8, device=dev)
    c, s, q = cache.ctype(), seqs.ctype(), queries.ctype()
    _lib.check("dsa_select_blocks", lib.dsa_select_blocks(
        ctypes.byref(c), ctypes.byref(s), ctypes.byref(q), _ptr(q_idx), _ptr(w), q_idx.shape[1], int(w_abs_max),
        _ptr(k_per_seq), int(k_max), _ptr(sel), _ptr(cnt), _ptr(workspace), workspace.numel(), _ptr(dev_err),
        _stream(stream)))
    return sel, cnt


def select_blocks_append(cache: PagedKVCache, seqs: SeqBatch, queries: QueryBatch, cu_new: torch.Tensor,
                         k_new: torch.Tensor, v_new: torch.Tensor, kc_new: Optional[torch.Tensor],
                         q_idx: torch.Tensor, w: torch.Tensor, k_per_seq: torch.Tensor, k_max: int,
                         w_abs_max: int = 16, sel: Optional[torch.Tensor] = None, cnt: Optional[torch.Tensor] = None,
                         workspace: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None,
                         stream=None):
    """select_blocks and kv_append in one launch for a decode batch, the
    copies overlapping the selection: (sel, cnt).  Queries whose sequence
    appends a block before their own block are refused (DEV_ERR_POS, cnt 0)."""
    lib = load()
    _expect(q_idx, torch.int8, "q_idx")
    _expect(w, torch.int32, "w")
    _expect(k_new, torch.bfloat16, "k_new")
    _expect(v_new, torch.bfloat16, "v_new")
    dev = q_idx.device
    T = queries.total_q
    if sel is None:
        sel = torch.empty((T, k_max), dtype=torch.int32, device=dev)
    if cnt is None:
        cnt = torch.empty((T,), dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = torch.zeros(select_workspace_size(T), dtype=torch.uint8, device=dev)
    c, s, q = cache.ctype(), seqs.ctype(), queries.ctype()
    _lib.check("dsa_select_blocks_append", lib.dsa_select_blocks_append(
        ctypes.byref(c), ctypes.byref(s), ctypes.byref(q), _ptr(cu_new), k_new.shape[0], _ptr(k_new), _ptr(v_new),
        _ptr(kc_new), _ptr(q_idx), _ptr(w), q_idx.shape[1], int(w_abs_max), _ptr(k_per_seq), int(k_max), _ptr(sel),
        _ptr(cnt), _ptr(workspace), workspace.numel(), _ptr(dev_err), _stream(stream)))
    return sel, cnt


def decode_workspace_size(total_q: int, num_q_heads: int, num_kv_heads: int, k_max: int) -> int:
    return int(load().dsa_sparse_attn_decode_workspace_size(total_q, num_q_heads, num_kv_heads, k_max))


def _attn_out(q, out, lse):
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:2], dtype=torch.float32, device=q.device)
    return out, lse


def sparse_attn_decode(cache: PagedKVCache, seqs: SeqBatch, queries: QueryBatch, q: torch.Tensor,
                       sel: torch.Tensor, cnt: torch.Tensor, sm_scale: Optional[float] = None,
                       out=None, lse=None, workspace: Optional[torch.Tensor] = None,
                       dev_err: Optional[torch.Tensor] = None, stream=None):
    """(out bf16 [total_q][Hq][128], lse fp32 [total_q][Hq]).  ``workspace`` is a
    zero-initialised uint8 tensor of decode_workspace_size() bytes (allocated here if None)."""
    lib = load()
    _expect(q, torch.bfloat16, "q")
    k_max = sel.shape[1]
    out, lse = _attn_out(q, out, lse)
    if workspace is None:
        workspace = torch.zeros(decode_workspace_size(queries.total_q, q.shape[1], cache.num_kv_heads, k_max),
                                dtype=torch.uint8, device=q.device)
    scale = 1.0 / math.sqrt(q.shape[2]) if sm_scale is None else float(sm_scale)
    c, s, qq = cache.ctype(), seqs.ctype(), queries.ctype()
    _lib.check("dsa_sparse_attn_decode", lib.dsa_sparse_attn_decode(
        ctypes.byref(c), ctypes.byref(s), ctypes.byref(qq), _ptr(q), q.shape[1], _ptr(sel), _ptr(cnt),
        k_max, scale, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _ptr(dev_err),
        _stream(stream)))
    return out, lse


def sparse_attn_decode_noalloc(cache: PagedKVCache, seqs: SeqBatch, queries: QueryBatch, q: torch.Tensor,
                               sel: torch.Tensor, cnt: torch.Tensor, sm_scale: Optional[float] = None,
                               out=None, lse=None, dev_err: Optional[torch.Tensor] = None, stream=None):
    """Decode attention that allocates nothing on the device: for callers that
    cannot call cudaMalloc (an engine plugin's enqueue path, a runtime that owns
    all device memory).  The split-KV scratch is a fixed 16 MiB array inside
    the library; problems needing more are rejected, and calls that overlap on
    the GPU share that array and race.  ``out``/``lse`` are allocated by torch
    here only when not given."""
    lib = load()
    _expect(q, torch.bfloat16, "q")
    out, lse = _attn_out(q, out, lse)
    scale = 1.0 / math.sqrt(q.shape[2]) if sm_scale is None else float(sm_scale)
    c, s, qq = cache.ctype(), seqs.ctype(), queries.ctype()
    _lib.check("dsa_sparse_attn_decode_noalloc", lib.dsa_sparse_attn_decode_noalloc(
        ctypes.byref(c), ctypes.byref(s), ctypes.byref(qq), _ptr(q), q.shape[1], _ptr(sel), _ptr(cnt),
        sel.shape[1], scale, _ptr(out), _ptr(lse), _ptr(dev_err), _stream(stream)))
    return out, lse


def sparse_attn_prefill(cache: PagedKVCache, seqs: SeqBatch, queries: QueryBatch, q: torch.Tensor,
                        sel: torch.Tensor, cnt: torch.Tensor, sm_scale: Optional[float] = None,
                        out=None, lse=None, dev_err: Optional[torch.Tensor] = None, stream=None):
    lib = load()
    _expect(q, torch.bfloat16, "q")
    out, lse = _attn_out(q, out, lse)
    scale = 1.0 / math.sqrt(q.shape[2]) if sm_scale is None else float(sm_scale)
    c, s, qq = cache.ctype(), seqs.ctype(), queries.ctype()
    _lib.check("dsa_sparse_attn_prefill", lib.dsa_sparse_attn_prefill(
        ctypes.byref(c), ctypes.byref(s), ctypes.byref(qq), _ptr(q), q.shape[1], _ptr(sel), _ptr(cnt),
        sel.shape[1], scale, _ptr(out), _ptr(lse), _ptr(dev_err), _stream(stream)))
    return out, lse


def decode_fused_workspace_size(total_q: int, num_q_heads: int, num_kv_heads: int, k_max: int) -> int:
    return int(load().dsa_decode_fused_workspace_size(total_q, num_q_heads, num_kv_heads, k_max))


def decode_fused(cache: PagedKVCache, seqs: SeqBatch, queries: QueryBatch, cu_new: Optional[torch.Tensor],
                 k_new: Optional[torch.Tensor], v_new: Optional[torch.Tensor], kc_new: Optional[torch.Tensor],
                 q_idx: torch.Tensor, w: torch.Tensor, k_per_seq: torch.Tensor, k_max: int, q: torch.Tensor,
                 w_abs_max: int = 16, sm_scale: Optional[float] = None, sel=None, cnt=None, out=None, lse=None,
                 workspace: Optional[torch.Tensor] = None, dev_err: Optional[torch.Tensor] = None, stream=None):
    """One decode step in a single launch (append, select, attention):
    (sel, cnt, out, lse).  ``cu_new``/``k_new``/``v_new``/``kc_new`` describe
    the tokens to append (``k_new`` None: nothing appended).  ``workspace`` is
    a zero-initialised uint8 tensor of decode_fused_workspace_size() bytes
    (allocated here if None); one workspace serves every later call."""
    lib = load()
    _expect(q, torch.bfloat16, "q")
    _expect(q_idx, torch.int8, "q_idx")
    _expect(w, torch.int32, "w")
    T, dev = queries.total_q, q.device
    if sel is None:
        sel = torch.empty((T, k_max), dtype=torch.int32, device=dev)
    if cnt is None:
        cnt = torch.empty((T,), dtype=torch.int32, device=dev)
    out, lse = _attn_out(q, out, lse)
    if workspace is None:
        workspace = torch.zeros(decode_fused_workspace_size(T, q.shape[1], cache.num_kv_heads, k_max),
                                dtype=torch.uint8, device=dev)
    total_new = 0 if k_new is None else k_new.shape[0]
    if k_new is not None:
        _expect(k_new, torch.bfloat16, "k_new")
        _expect(v_new, torch.bfloat16, "v_new")
    scale = 1.0 / math.sqrt(q.shape[2]) if sm_scale is None else float(sm_scale)
    c, s, qq = cache.ctype(), seqs.ctype(), queries.ctype()
    _lib.check("dsa_decode_fused", lib.dsa_decode_fused(
        ctypes.byref(c), ctypes.byref(s), ctypes.byref(qq), _ptr(cu_new), int(total_new), _ptr(k_new), _ptr(v_new),
        _ptr(kc_new), _ptr(q_idx), _ptr(w), q_idx.shape[1], int(w_abs_max), _ptr(k_per_seq), int(k_max), _ptr(q),
        q.shape[1], scale, _ptr(sel), _ptr(cnt), _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
        _ptr(dev_err), _stream(stream)))
    return sel, cnt, out, lse


class _Recorder:
    """Stands in for the library while PreparedStep records a step: launches
    are recorded with their marshalled arguments (and report success), size
    and status queries go to the library."""

    def __init__(self, lib):
        self._real = lib
        self.calls = []

    def __getattr__(self, name):
        real = getattr(self._real, name)
        if name.endswith("_workspace_size") or name in ("dsa_status_string", "dsa_version"):
            return real

        def record(*args):
            self.calls.append((name, real, args))
            return _lib.DSA_OK
        return record


def _host_ptr(t: torch.Tensor) -> int:
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("host staging buffers must be contiguous CPU tensors (pinned for asynchronous copies)")
    return t.data_ptr()


def _regions(pairs, host_first: bool):
    """(dst array, src array, bytes array, n) of (device, host) tensor pairs."""
    n = len(pairs)
    dst, src, nb = (ctypes.c_void_p * max(n, 1))(), (ctypes.c_void_p * max(n, 1))(), (ctypes.c_size_t * max(n, 1))()
    for i, (dev_t, host_t) in enumerate(pairs):
        if dev_t.numel() * dev_t.element_size() != host_t.numel() * host_t.element_size():
            raise ValueError("a staged device tensor and its host buffer differ in size")
        d, h = _ptr(dev_t).value, _host_ptr(host_t)
        dst[i], src[i] = (h, d) if host_first else (d, h)
        nb[i] = dev_t.numel() * dev_t.element_size()
    return dst, src, nb, n


class Stager:
    """Host staging of repeated steps (the library's dsa_stager): inputs copied
    from pinned host memory and results copied back on two copy streams of the
    library's own, so one batch's copies overlap the other batches' kernels.
    ``num_slots`` batches, each with its own device buffers; ``stream`` is the
    compute stream the steps run on (default: the current stream)."""

    def __init__(self, num_slots: int, stream=None):
        self._lib = load()
        self.stream = torch.cuda.current_stream() if stream is None else stream
        self._s = ctypes.c_void_p(self.stream.cuda_stream)
        h = ctypes.c_void_p()
        _lib.check("dsa_stager_create", self._lib.dsa_stager_create(num_slots, self._s, ctypes.byref(h)))
        self._h = h
        self.num_slots = num_slots

    def wait(self, slot: int) -> None:
        """Block until the slot's last read-back has landed."""
        _lib.check("dsa_stager_wait", self._lib.dsa_stager_wait(self._h, slot))

    def join(self) -> None:
        """Make the compute stream wait for every copy issued so far."""
        _lib.check("dsa_stager_join", self._lib.dsa_stager_join(self._h))

    def close(self) -> None:
        if getattr(self, "_h", None):
            rc = self._lib.dsa_stager_destroy(self._h)
            self._h = None
            _lib.check("dsa_stager_destroy", rc)

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class PreparedStep:
    """One pass of the hot path (the calls step() makes, same arguments) with
    every argument marshalled once, for loops that run the same step on the
    same buffers again and again (a serving loop, a benchmark).  Calling it
    issues the library calls on ``stream`` (the stream given here, else the
    current one) and returns the output buffers; the host cost per call is
    the calls themselves.  The tensors passed here must stay allocated at the
    same addresses while the object is used (it keeps references to them);
    refill them in place between calls.  Not to be built while another thread
    calls this module.

    With a ``stager`` (a Stager) the step also stages its own host data on it
    as slot ``slot``: every call first copies ``host_in`` -- (device tensor,
    pinned host tensor) pairs -- to the device and ends by copying
    ``host_out`` -- (device tensor, pinned host tensor) pairs -- back, and the
    step runs on the stager's stream.  ``stager.wait(slot)`` tells when the
    host buffers may be read (results) and rewritten (inputs)."""

    def __init__(self, cache: PagedKVCache, seqs: SeqBatch, queries: QueryBatch, *, bufs: Optional[dict] = None,
                 stream=None, stager: Optional[Stager] = None, slot: int = 0, host_in=(), host_out=(),
                 **step_kwargs):
        global load
        rec = _Recorder(_lib.load())
        saved = load
        load = lambda: rec   # noqa: E731 -- the binding's calls below go to the recorder
        try:
            self.bufs = step(cache, seqs, queries, bufs=bufs, **step_kwargs)
        finally:
            load = saved
        self.calls = rec.calls
        if stager is not None:
            if not 0 <= slot < stager.num_slots:
                raise ValueError(f"slot {slot} outside the stager's {stager.num_slots} slots")
            stream = stager.stream
            lib = _lib.load()
            self._stager = stager
            self._begin = (lib.dsa_stager_begin, (stager._h, slot, *_rotate(_regions(host_in, False))))
            self._end = (lib.dsa_stager_end, (stager._h, slot, *_rotate(_regions(host_out, True))))
        elif host_in or host_out:
            raise ValueError("host_in / host_out need a stager")
        else:
            self._stager = None
            self._begin = self._end = None
        self._stream = None if stream is None else ctypes.c_void_p(stream.cuda_stream)
        self._keep = (cache, seqs, queries, step_kwargs, stager, tuple(host_in), tuple(host_out))

    def __call__(self, stream=None):
        if self._begin is not None:
            if stream is not None:
                raise ValueError("a staged step runs on its stager's stream")
            if not self._stager._h:
                raise ValueError("the step's stager has been closed")
            fn, args = self._begin
            _lib.check("dsa_stager_begin", fn(*args))
        s = _stream(stream) if (stream is not None or self._stream is None) else self._stream
        for name, fn, args in self.calls:
            rc = fn(*args[:-1], s)
            if rc != _lib.DSA_OK:
                _lib.check(name, rc)
        if self._end is not None:
            fn, args = self._end
            _lib.check("dsa_stager_end", fn(*args))
        return self.bufs


def _rotate(r):
    """(dst, src, bytes, n) -> (n, dst, src, bytes): the C argument order."""
    dst, src, nb, n = r
    return n, dst, src, nb


def step(cache: PagedKVCache, seqs: SeqBatch, queries: QueryBatch, *, k_new, v_new, kc_new, q, q_idx, w,
         k_per_seq, k_max: int, w_abs_max: int = 16, decode: bool = True, fused_select: bool = False,
         overlap_append: bool = False, fused_decode: bool = False, bufs: Optional[dict] = None,
         dev_err: Optional[torch.Tensor] = None, stream=None):
    """One pass of the hot path: append -> index_score -> topk_blocks -> attention
    (with ``fused_select`` the middle two are the single select_blocks call;
    with ``overlap_append`` as well -- decode batches only -- the append runs
    as select_blocks_append, overlapping the selection; with ``fused_decode``
    the whole decode step is one decode_fused launch).

    ``bufs`` (optional, reused across calls) holds the scores / sel / cnt /
    out / lse / workspace tensors; missing ones are allocated.  Returns bufs.
    """
    b = {} if bufs is None else bufs
    T, dev = queries.total_q, q.device
    if "scores" not in b:
        b["scores"] = torch.empty((T, seqs.block_table.shape[1]), dtype=torch.int32, device=dev)
        b["sel"] = torch.empty((T, k_max), dtype=torch.int32, device=dev)
        b["cnt"] = torch.empty((T,), dtype=torch.int32, device=dev)
        b["out"] = torch.empty_like(q)
        b["lse"] = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
        b["workspace"] = torch.zeros(decode_workspace_size(T, q.shape[1], cache.num_kv_heads, k_max),
                                     dtype=torch.uint8, device=dev)
        b["select_ws"] = torch.zeros(select_workspace_size(T), dtype=torch.uint8, device=dev)
    if fused_decode:
        if not decode:
            raise ValueError("fused_decode needs a decode batch")
        if "fused_ws" not in b:
            b["fused_ws"] = torch.zeros(decode_fused_workspace_size(T, q.shape[1], cache.num_kv_heads, k_max),
                                        dtype=torch.uint8, device=dev)
        decode_fused(cache, seqs, queries, queries.cu_q, k_new, v_new, kc_new, q_idx, w, k_per_seq, k_max, q,
                     w_abs_max, sel=b["sel"], cnt=b["cnt"], out=b["out"], lse=b["lse"], workspace=b["fused_ws"],
                     dev_err=dev_err, stream=stream)
        return b
    if fused_select and overlap_append:
        # decode batches: the token copies overlap the selection, which never reads them
        select_blocks_append(cache, seqs, queries, queries.cu_q, k_new, v_new, kc_new, q_idx, w, k_per_seq, k_max,
                             w_abs_max, sel=b["sel"], cnt=b["cnt"], workspace=b["select_ws"], dev_err=dev_err,
                             stream=stream)
        sparse_attn_decode(cache, seqs, queries, q, b["sel"], b["cnt"], out=b["out"], lse=b["lse"],
                           workspace=b["workspace"], dev_err=dev_err, stream=stream)
        return b
    kv_append(cache, seqs, queries.cu_q, k_new, v_new, kc_new, dev_err=dev_err, stream=stream)
    if fused_select:
        select_blocks(cache, seqs, queries, q_idx, w, k_per_seq, k_max, w_abs_max, sel=b["sel"], cnt=b["cnt"],
                      workspace=b["select_ws"], dev_err=dev_err, stream=stream)
    else:
        index_score(cache, seqs, queries, q_idx, w, w_abs_max, scores=b["scores"], dev_err=dev_err,
                    stream=stream)
        topk_blocks(seqs, queries, b["scores"], k_per_seq, k_max, sel=b["sel"], cnt=b["cnt"], dev_err=dev_err,
                    stream=stream, block_size=cache.block_size)
    if decode:
        sparse_attn_decode(cache, seqs, queries, q, b["sel"], b["cnt"], out=b["out"], lse=b["lse"],
                           workspace=b["workspace"], dev_err=dev_err, stream=stream)
    else:
        sparse_attn_prefill(cache, seqs, queries, q, b["sel"], b["cnt"], out=b["out"], lse=b["lse"],
                            dev_err=dev_err, stream=stream)
    return b
