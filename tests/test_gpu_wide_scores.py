"""GPU parity of the signed-weight, int64 and FP8 (E4M3) indexer paths against
the oracle, through the C ABI.

Bar: scores and selections bit-exact (integer work; the FP8 scores are exact
integers times 2^-18 on both sides), attention outputs within max-abs 2e-2 /
mean-abs 2e-3 of the oracle's float64 result.
"""
import numpy as np
import pytest
import torch

import dynamic_block_sparse_dsa_b200 as dsa
from dynamic_block_sparse_dsa_b200 import workloads as wk
from oracle.harness import oracle_select, oracle_step

pytestmark = pytest.mark.gpu

OUT_MAX, OUT_MEAN = 2e-2, 2e-3
I64_MIN = np.iinfo(np.int64).min

CASES = {
    # decode queries of varied lengths (the CUDA-core scan)
    "decode": dict(seq_lens=(5000, 700, 20000, 129, 3000), n_new=(1,) * 5, k_per_seq=(6, 2, 9, 3, 5), k_max=9),
    # prefill chunks with ragged tails (>= 16 queries per sequence: the int32
    # path runs on the tensor cores)
    "prefill": dict(seq_lens=(9000, 3000, 1100), n_new=(70, 33, 17), k_per_seq=(7, 3, 4), k_max=7),
}


def _spec(name, block_size=64, **kw):
    base = dict(num_q_heads=16, num_kv_heads=2, num_idx_heads=16, block_size=block_size)
    base.update(CASES[name])
    base.update(kw)
    return wk.sharp(wk.WorkloadSpec(f"{name}_b{block_size}", **base))


def _handles(wl):
    return (dsa.PagedKVCache(wl.k_pool, wl.v_pool, wl.kc_pool), dsa.SeqBatch(wl.block_table, wl.seq_lens),
            dsa.QueryBatch(wl.cu_q, wl.q_pos))


def _check_scores(gpu_scores, ref):
    sc = gpu_scores.index_select(0, torch.as_tensor(ref["queries"], device=gpu_scores.device)).cpu().numpy()
    vis = ref["scores"] != I64_MIN
    assert np.array_equal(sc.astype(np.int64)[vis], ref["scores"][vis]), "block scores differ"


def _check_sel(sel, cnt, ref):
    assert np.array_equal(cnt.cpu().numpy(), ref["cnt"]), "selection counts differ"
    assert np.array_equal(sel.cpu().numpy(), ref["sel"]), "selected block ids differ"


@pytest.mark.parametrize("fused", [False, True], ids=["score_topk", "fused_select"])
@pytest.mark.parametrize("name", sorted(CASES))
def test_signed_weights_int32_paths(name, fused, cuda_device):
    """Weights in [-16, 16]: every int32 scoring path and the attention after it."""
    spec = _spec(name, w_min=-16)
    wl = wk.make_workload(spec, seed=51, device=cuda_device)
    assert int(wl.w.min()) < 0
    ref = oracle_step(wl, want_scores=True)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    cache, seqs, queries = _handles(wl)
    bufs = dsa.step(cache, seqs, queries, k_new=wl.k_new, v_new=wl.v_new, kc_new=wl.kc_new, q=wl.q, q_idx=wl.q_idx,
                    w=wl.w, k_per_seq=wl.k_per_seq, k_max=spec.k_max, decode=name == "decode", fused_select=fused,
                    dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    if not fused:
        _check_scores(bufs["scores"], ref)
    _check_sel(bufs["sel"], bufs["cnt"], ref)
    d = np.abs(bufs["out"].double().cpu().numpy() - ref["out"])
    assert d.max() <= OUT_MAX and d.mean() <= OUT_MEAN


@pytest.mark.parametrize("block_size", [64, 256])
@pytest.mark.parametrize("name", sorted(CASES))
def test_int64_scores_beyond_the_int32_bound(name, block_size, cuda_device):
    """Weights up to 2^30 in magnitude: the int32 path refuses them, the int64
    path scores them exactly and its Top-K selects exactly; the attention over
    that selection equals the oracle's."""
    spec = _spec(name, block_size)
    wl = wk.make_workload(spec, seed=52, device=cuda_device)
    g = torch.Generator(device=cuda_device)
    g.manual_seed(7)
    w = torch.randint(-(1 << 30), 1 << 30, wl.w.shape, generator=g, device=cuda_device, dtype=torch.int32)
    cache, seqs, queries = _handles(wl)
    with pytest.raises(dsa.DsaError):
        dsa.index_score(cache, seqs, queries, wl.q_idx, w, w_abs_max=1 << 30)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    scores = dsa.index_score_i64(cache, seqs, queries, wl.q_idx, w, dev_err=err)
    sel, cnt = dsa.topk_blocks_i64(seqs, queries, scores, wl.k_per_seq, spec.k_max, block_size=block_size,
                                   dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = oracle_select(wl, w=w)
    assert np.abs(ref["scores"][ref["scores"] != I64_MIN]).max() >= 1 << 31   # beyond int32
    _check_scores(scores, ref)
    _check_sel(sel, cnt, ref)
    # the selection drives the gather exactly as an int32 one would
    wl.w = w
    full = oracle_step(wl, with_append=False)
    assert np.array_equal(full["sel"], ref["sel"])
    out, lse = (dsa.sparse_attn_decode if name == "decode" else dsa.sparse_attn_prefill)(
        cache, seqs, queries, wl.q, sel, cnt, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    d = np.abs(out.double().cpu().numpy() - full["out"])
    assert d.max() <= OUT_MAX and d.mean() <= OUT_MEAN


@pytest.mark.parametrize("block_size", [64, 512])
@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8_scores_and_selection_exact(name, block_size, cuda_device):
    spec = _spec(name, block_size, w_min=-16)
    wl = wk.make_workload(spec, seed=53, device=cuda_device)
    q8, kc8 = wk.e4m3_indexer(wl, seed=9)
    cache = dsa.PagedKVCache(wl.k_pool, wl.v_pool, kc8)
    _, seqs, queries = _handles(wl)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    scores = dsa.index_score_fp8(cache, seqs, queries, q8, wl.w, w_abs_max=16, dev_err=err)
    sel, cnt = dsa.topk_blocks_i64(seqs, queries, scores, wl.k_per_seq, spec.k_max, block_size=block_size,
                                   dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = oracle_select(wl, q_idx=q8, kc_pool=kc8, fp8=True)
    _check_scores(scores, ref)
    _check_sel(sel, cnt, ref)


def test_fp8_nan_code_is_flagged_and_read_as_zero(cuda_device):
    spec = _spec("decode")
    wl = wk.make_workload(spec, seed=54, device=cuda_device)
    q8, kc8 = wk.e4m3_indexer(wl, seed=10)
    q_nan = q8.clone()
    q_nan[0, 0, 3] = 0x7F
    q_zero = q8.clone()
    q_zero[0, 0, 3] = 0
    cache = dsa.PagedKVCache(wl.k_pool, wl.v_pool, kc8)
    _, seqs, queries = _handles(wl)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    s_nan = dsa.index_score_fp8(cache, seqs, queries, q_nan, wl.w, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & dsa._lib.DEV_ERR_VALUE
    s_zero = dsa.index_score_fp8(cache, seqs, queries, q_zero, wl.w)
    torch.cuda.synchronize()
    own = int(wl.q_pos[0]) // 64
    assert torch.equal(s_nan[0, :own + 1], s_zero[0, :own + 1])


def test_fp8_range_check(cuda_device):
    spec = _spec("decode")
    wl = wk.make_workload(spec, seed=55, device=cuda_device)
    q8, kc8 = wk.e4m3_indexer(wl)
    cache = dsa.PagedKVCache(wl.k_pool, wl.v_pool, kc8)
    _, seqs, queries = _handles(wl)
    with pytest.raises(dsa.DsaError):
        dsa.index_score_fp8(cache, seqs, queries, q8, wl.w, w_abs_max=1 << 20)
