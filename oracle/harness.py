"""Run the oracle's version of one step on a synthetic workload.

TEST INFRASTRUCTURE ONLY (used by the tests, the smoke check and the CPU
baseline of the benchmark).  This module moves data between a workload's
torch tensors (on any device) and the oracle's numpy arguments; the method's
arithmetic is all in ``dsa_oracle.c``.

A step is: append the new tokens (K/V rows and the touched blocks' coarse
keys), score every visible block for each query, select Top-K blocks, attend
over the selection.  For large workloads only the KV pages the oracle's own
selection needs (plus the pages the append touches) are copied to the host;
they are copied from the workload's *input* tensors, so the harness must be
called before the device step mutates the pool.
"""
from __future__ import annotations

import time

import numpy as np
import torch

import oracle as orc


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _np(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().numpy()


def bits_to_float64(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float64 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def oracle_step(wl, queries=None, with_append: bool = True, want_scores: bool = False):
    """Oracle result of one step for the query indices ``queries`` (all if None).

    Returns a dict with ``queries``, ``sel`` [n][k_max], ``cnt`` [n], ``out``
    [n][Hq][D] float64, ``lse`` [n][Hq] float64, optionally ``scores`` (int64
    [n][max_blocks]) and ``seconds`` (time spent inside oracle calls only).
    """
    spec = wl.spec
    bs = spec.block_size
    table = _np(wl.block_table).astype(np.int32)
    seq_lens = _np(wl.seq_lens).astype(np.int32)
    cu = _np(wl.cu_q).astype(np.int32)
    q_pos_all = _np(wl.q_pos).astype(np.int32)
    q_seq_all = orc.queries_to_seq(cu)
    T = len(q_pos_all)
    qs = np.arange(T, dtype=np.int64) if queries is None else np.asarray(queries, dtype=np.int64)
    q_seq = q_seq_all[qs]
    q_pos = q_pos_all[qs]
    k_per_seq = _np(wl.k_per_seq).astype(np.int32)
    q_sel = torch.as_tensor(qs, device=wl.q_idx.device)
    q_idx = _np(wl.q_idx.index_select(0, q_sel))
    w = _np(wl.w.index_select(0, q_sel))
    q = bf16_bits(wl.q.index_select(0, q_sel))
    kc_pool = _np(wl.kc_pool).copy()
    seconds = 0.0

    if with_append:
        t0 = time.perf_counter()
        orc.kc_append(table, seq_lens, cu, _np(wl.kc_new), kc_pool, bs)
        seconds += time.perf_counter() - t0

    t0 = time.perf_counter()
    scores = orc.index_score(q_seq, q_pos, table, bs, kc_pool, q_idx, w)
    sel, cnt = orc.topk(q_seq, q_pos, bs, scores, k_per_seq, spec.k_max)
    seconds += time.perf_counter() - t0

    # KV pages needed: the selection's pages plus every page the append touches
    need = set()
    for i in range(len(qs)):
        s = q_seq[i]
        for b in sel[i, :cnt[i]]:
            need.add(int(table[s, b]))
    if with_append:
        for s in range(spec.num_seqs):
            n = cu[s + 1] - cu[s]
            if n == 0:
                continue
            L = seq_lens[s]
            for b in range((L - n) // bs, (L - 1) // bs + 1):
                need.add(int(table[s, b]))
    pages = np.array(sorted(need), dtype=np.int64)
    remap = np.full(spec.num_pages, -1, dtype=np.int64)
    remap[pages] = np.arange(len(pages))
    table_c = np.where(table >= 0, remap[np.maximum(table, 0)], -1).astype(np.int32)
    idx = torch.as_tensor(pages, device=wl.k_pool.device)
    k_c = bf16_bits(wl.k_pool.index_select(0, idx))
    v_c = bf16_bits(wl.v_pool.index_select(0, idx))

    t0 = time.perf_counter()
    if with_append:
        orc.kv_append(table_c, seq_lens, cu, bf16_bits(wl.k_new), bf16_bits(wl.v_new), k_c, v_c, bs)
    out, lse = orc.sparse_attention(q_seq, q_pos, table_c, bs, q, k_c, v_c, sel, cnt, wl.sm_scale)
    seconds += time.perf_counter() - t0

    res = {"queries": qs, "sel": sel, "cnt": cnt, "out": out, "lse": lse, "seconds": seconds}
    if want_scores:
        res["scores"] = scores
    return res
