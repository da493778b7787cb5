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

import oracle as orc


def bf16_bits(t) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    import torch
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _np(t) -> np.ndarray:
    return t.detach().cpu().numpy()


def bits_to_float64(bits: np.ndarray) -> np.ndarray:
    """uint16 bf16 bit patterns -> float64 (exact)."""
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def host_inputs(wl, queries=None, with_append: bool = True) -> dict:
    """Everything one oracle step reads, copied to host numpy arrays.

    The K/V pages copied are the ones the step needs: those of the oracle's
    own selection for the chosen queries (found here by running the oracle's
    append-of-coarse-keys, scoring and Top-K once on the host) plus every page
    the append touches.  The block table is remapped onto that compact page
    set.  The returned dict is all ``run_host`` needs; it holds no torch
    tensor, so it can be saved and reloaded by other processes.
    """
    import torch
    spec = wl.spec
    bs = spec.block_size
    table = _np(wl.block_table).astype(np.int32)
    seq_lens = _np(wl.seq_lens).astype(np.int32)
    cu = _np(wl.cu_q).astype(np.int32)
    q_pos_all = _np(wl.q_pos).astype(np.int32)
    q_seq_all = orc.queries_to_seq(cu)
    T = len(q_pos_all)
    qs = np.arange(T, dtype=np.int64) if queries is None else np.asarray(queries, dtype=np.int64)
    q_sel = torch.as_tensor(qs, device=wl.q_idx.device)
    inp = {
        "queries": qs, "block_size": np.int32(bs), "k_max": np.int32(spec.k_max), "sm_scale": np.float64(wl.sm_scale),
        "with_append": np.int32(1 if with_append else 0), "num_seqs": np.int32(spec.num_seqs),
        "table": table, "seq_lens": seq_lens, "cu": cu, "q_seq": q_seq_all[qs], "q_pos": q_pos_all[qs],
        "k_per_seq": _np(wl.k_per_seq).astype(np.int32),
        "q_idx": _np(wl.q_idx.index_select(0, q_sel)), "w": _np(wl.w.index_select(0, q_sel)),
        "q": bf16_bits(wl.q.index_select(0, q_sel)), "kc_pool": _np(wl.kc_pool).copy(),
        "kc_new": _np(wl.kc_new), "k_new": bf16_bits(wl.k_new), "v_new": bf16_bits(wl.v_new),
    }
    # the pages this step needs (the oracle's own selection; run once here, untimed)
    kc_pool = inp["kc_pool"].copy()
    if with_append:
        orc.kc_append(table, seq_lens, cu, inp["kc_new"], kc_pool, bs)
    scores = orc.index_score(inp["q_seq"], inp["q_pos"], table, bs, kc_pool, inp["q_idx"], inp["w"])
    sel, cnt = orc.topk(inp["q_seq"], inp["q_pos"], bs, scores, inp["k_per_seq"], spec.k_max)
    need = set()
    for i in range(len(qs)):
        srow = inp["q_seq"][i]
        for b in sel[i, :cnt[i]]:
            need.add(int(table[srow, b]))
    if with_append:
        for sq in range(spec.num_seqs):
            n = cu[sq + 1] - cu[sq]
            if n == 0:
                continue
            L = seq_lens[sq]
            for b in range((L - n) // bs, (L - 1) // bs + 1):
                need.add(int(table[sq, b]))
    pages = np.array(sorted(need), dtype=np.int64)
    remap = np.full(spec.num_pages, -1, dtype=np.int64)
    remap[pages] = np.arange(len(pages))
    inp["table_c"] = np.where(table >= 0, remap[np.maximum(table, 0)], -1).astype(np.int32)
    idx = torch.as_tensor(pages, device=wl.k_pool.device)
    inp["k_c"] = bf16_bits(wl.k_pool.index_select(0, idx))
    inp["v_c"] = bf16_bits(wl.v_pool.index_select(0, idx))
    return inp


def run_host(inp: dict, want_scores: bool = False) -> dict:
    """One oracle step on host arrays from ``host_inputs`` (which it does not
    modify): append, scores, Top-K, attention.  ``seconds`` is the time spent
    inside the oracle's calls only (the copies of the pools that the append
    writes into are excluded)."""
    bs = int(inp["block_size"])
    with_append = bool(int(inp["with_append"]))
    table, seq_lens, cu = inp["table"], inp["seq_lens"], inp["cu"]
    kc_pool = np.array(inp["kc_pool"], copy=True)
    k_c = np.array(inp["k_c"], copy=True)
    v_c = np.array(inp["v_c"], copy=True)
    seconds = 0.0

    t0 = time.perf_counter()
    if with_append:
        orc.kc_append(table, seq_lens, cu, inp["kc_new"], kc_pool, bs)
    scores = orc.index_score(inp["q_seq"], inp["q_pos"], table, bs, kc_pool, inp["q_idx"], inp["w"])
    sel, cnt = orc.topk(inp["q_seq"], inp["q_pos"], bs, scores, inp["k_per_seq"], int(inp["k_max"]))
    if with_append:
        orc.kv_append(inp["table_c"], seq_lens, cu, inp["k_new"], inp["v_new"], k_c, v_c, bs)
    out, lse = orc.sparse_attention(inp["q_seq"], inp["q_pos"], inp["table_c"], bs, inp["q"], k_c, v_c, sel, cnt,
                                    float(inp["sm_scale"]))
    seconds += time.perf_counter() - t0

    res = {"queries": inp["queries"], "sel": sel, "cnt": cnt, "out": out, "lse": lse, "seconds": seconds}
    if want_scores:
        res["scores"] = scores
    return res


def oracle_step(wl, queries=None, with_append: bool = True, want_scores: bool = False):
    """Oracle result of one step for the query indices ``queries`` (all if None).

    Returns a dict with ``queries``, ``sel`` [n][k_max], ``cnt`` [n], ``out``
    [n][Hq][D] float64, ``lse`` [n][Hq] float64, optionally ``scores`` (int64
    [n][max_blocks]) and ``seconds`` (time spent inside oracle calls only).
    """
    return run_host(host_inputs(wl, queries, with_append), want_scores=want_scores)


def oracle_select(wl, q_idx=None, w=None, kc_pool=None, fp8: bool = False, queries=None):
    """The oracle's scores and selection for the workload's queries (no append),
    with optional replacement indexer inputs: int8 q_idx / kc_pool (any int32
    weights), or, with ``fp8``, E4M3 codes for both (scores times 2^18).
    Returns a dict with ``queries``, ``scores`` int64 [n][max_blocks], ``sel``, ``cnt``."""
    spec = wl.spec
    table = _np(wl.block_table).astype(np.int32)
    cu = _np(wl.cu_q).astype(np.int32)
    q_pos_all = _np(wl.q_pos).astype(np.int32)
    q_seq_all = orc.queries_to_seq(cu)
    T = len(q_pos_all)
    qs = np.arange(T, dtype=np.int64) if queries is None else np.asarray(queries, dtype=np.int64)
    qi = _np(wl.q_idx if q_idx is None else q_idx)[qs]
    ww = _np(wl.w if w is None else w)[qs]
    kc = _np(wl.kc_pool if kc_pool is None else kc_pool)
    if fp8:
        scores = orc.index_score_fp8(q_seq_all[qs], q_pos_all[qs], table, spec.block_size, kc, qi, ww)
    else:
        scores = orc.index_score(q_seq_all[qs], q_pos_all[qs], table, spec.block_size, kc, qi, ww)
    sel, cnt = orc.topk(q_seq_all[qs], q_pos_all[qs], spec.block_size, scores, _np(wl.k_per_seq).astype(np.int32),
                        spec.k_max)
    return {"queries": qs, "scores": scores, "sel": sel, "cnt": cnt}


def save_inputs(inp: dict, directory: str) -> None:
    """Write ``host_inputs``' arrays as .npy files (for worker processes)."""
    import os
    os.makedirs(directory, exist_ok=True)
    for k, v in inp.items():
        np.save(os.path.join(directory, k + ".npy"), np.asarray(v))


def load_inputs(directory: str) -> dict:
    import os
    return {f[:-4]: np.load(os.path.join(directory, f), mmap_mode="r")
            for f in os.listdir(directory) if f.endswith(".npy")}


def worker_main(argv) -> int:
    """``python -m oracle.harness INPUTS_DIR BUDGET_S READY_FILE GO_FILE OUT_FILE``:
    run whole oracle steps on the inputs saved in INPUTS_DIR for about
    BUDGET_S seconds of wall time, starting once GO_FILE exists (after writing
    READY_FILE), and write "steps seconds" to OUT_FILE.  One such process per
    core gives the oracle's throughput on all of a machine's cores; the oracle
    itself stays single-threaded."""
    import os
    directory, budget_s, ready, go, out = argv[0], float(argv[1]), argv[2], argv[3], argv[4]
    inp = load_inputs(directory)
    run_host(inp)                      # loads the oracle library, touches the pages
    open(ready, "w").close()
    t_wait = time.perf_counter()
    while not os.path.exists(go):
        if time.perf_counter() - t_wait > 600:
            return 1
        time.sleep(0.005)
    t0 = time.perf_counter()
    steps = 0
    while True:
        run_host(inp)
        steps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    with open(out + ".tmp", "w") as f:
        f.write(f"{steps} {time.perf_counter() - t0}\n")
    os.replace(out + ".tmp", out)
    return 0


if __name__ == "__main__":
    import sys
    sys.exit(worker_main(sys.argv[1:]))
