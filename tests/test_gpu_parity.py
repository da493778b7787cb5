"""GPU parity: the CUDA library against the oracle, on the same seeded inputs.

Bar (stated here, used by every case):
  * scores, selected block ids and counts: bit-exact (integer work);
  * attention output (bf16, fp32 accumulation): max |gpu - oracle| <= 2e-2 and
    mean |gpu - oracle| <= 2e-3 against the oracle's float64 result;
  * lse (fp32): max |gpu - oracle| <= 2e-3.
Every call goes through the C ABI (libdsa.so) via the Python binding.

Two value profiles: "plain" draws q, k, v ~ N(0,1)/sqrt(128) as the workload
statements do; the softmax is then almost flat and outputs are ~2e-3, below
the mean tolerance, so those cases pin the logits through lse only.  "sharp"
(workloads.sharp: q x 256, v x sqrt(128)) gives logits with standard
deviation 2 and unit-variance values; every sharp case first checks on the
CPU that the oracle's mean |out| is at least ten times the mean tolerance,
so that an all-zero output, a wrong head or a wrong page cannot pass.
"""
import math

import numpy as np
import pytest
import torch

import dynamic_block_sparse_dsa_b200 as dsa
from dynamic_block_sparse_dsa_b200 import workloads as wk
from oracle.harness import oracle_select, oracle_step

pytestmark = pytest.mark.gpu

OUT_MAX, OUT_MEAN, LSE_MAX = 2e-2, 2e-3, 2e-3
DISCRIMINATIVE = 10 * OUT_MEAN   # least oracle mean |out| of a sharp case
PROFILES = ["plain", "sharp"]


def profiled(spec, profile):
    return wk.sharp(spec) if profile == "sharp" else spec


def _handles(wl):
    return (dsa.PagedKVCache(wl.k_pool, wl.v_pool, wl.kc_pool), dsa.SeqBatch(wl.block_table, wl.seq_lens),
            dsa.QueryBatch(wl.cu_q, wl.q_pos))


def gpu_step(wl, decode=True, bufs=None, fused=False, fused_decode=False, overlap=False):
    cache, seqs, queries = _handles(wl)
    err = torch.zeros(1, dtype=torch.int32, device=wl.device)
    bufs = dsa.step(cache, seqs, queries, k_new=wl.k_new, v_new=wl.v_new, kc_new=wl.kc_new, q=wl.q,
                    q_idx=wl.q_idx, w=wl.w, k_per_seq=wl.k_per_seq, k_max=wl.spec.k_max,
                    decode=decode, fused_select=fused or overlap, overlap_append=overlap,
                    fused_decode=fused_decode, bufs=bufs, dev_err=err)
    torch.cuda.synchronize()
    return bufs, int(err.item())


def compare(wl, ref, bufs, check_scores=True, fused=False):
    if wl.spec.v_scale > 1.0:
        # a discriminative case: the expected output is far above the tolerance
        assert np.abs(ref["out"]).mean() >= DISCRIMINATIVE, np.abs(ref["out"]).mean()
    qs = torch.as_tensor(ref["queries"], device=wl.device)
    sel = bufs["sel"].index_select(0, qs).cpu().numpy()
    cnt = bufs["cnt"].index_select(0, qs).cpu().numpy()
    assert np.array_equal(cnt, ref["cnt"]), "selection counts differ"
    assert np.array_equal(sel, ref["sel"]), "selected block ids differ"
    if check_scores and not fused and "scores" in ref:
        sc = bufs["scores"].index_select(0, qs).cpu().numpy().astype(np.int64)
        vis = ref["scores"] != np.iinfo(np.int64).min
        assert np.array_equal(sc[vis], ref["scores"][vis]), "block scores differ"
    out = bufs["out"].index_select(0, qs).double().cpu().numpy()
    lse = bufs["lse"].index_select(0, qs).double().cpu().numpy()
    d = np.abs(out - ref["out"])
    assert d.max() <= OUT_MAX and d.mean() <= OUT_MEAN, (d.max(), d.mean())
    assert np.abs(lse - ref["lse"]).max() <= LSE_MAX
    return d.max(), d.mean()


def _run(spec, seed, device, queries=None, decode=True, scores=True, fused=False):
    wl = wk.make_workload(spec, seed=seed, device=device)
    ref = oracle_step(wl, queries=queries, want_scores=scores)
    bufs, err = gpu_step(wl, decode=decode, fused=fused)
    assert err == 0, f"device error bits {err}"
    return wl, ref, bufs


# ----------------------------------------------------------------------------- small, all outputs
SMALL = {
    # name: spec overrides (block_size 64, head_dim 128 fixed by the library)
    "single_partial_block": dict(seq_lens=(37,), n_new=(1,), k_per_seq=(4,), k_max=4),
    "one_token": dict(seq_lens=(1,), n_new=(1,), k_per_seq=(2,), k_max=2),
    "k1_only_own": dict(seq_lens=(700, 130), n_new=(1, 1), k_per_seq=(1, 1), k_max=1),
    "k_covers_all": dict(seq_lens=(300, 511), n_new=(1, 1), k_per_seq=(16, 16), k_max=16),
    "ragged_prefill_tail": dict(seq_lens=(1000, 250, 64), n_new=(77, 0, 64), k_per_seq=(5, 3, 2), k_max=8),
    "group16": dict(seq_lens=(900,), n_new=(3,), k_per_seq=(6,), k_max=6, num_q_heads=32, num_kv_heads=2),
    "group1_mha": dict(seq_lens=(650, 200), n_new=(1, 2), k_per_seq=(4, 4), k_max=4, num_q_heads=4,
                       num_kv_heads=4),
    "many_seqs_decode": dict(seq_lens=tuple(range(129, 129 + 40 * 97, 97)), n_new=(1,) * 40,
                             k_per_seq=(8,) * 40, k_max=8),
    "prefill_two_chunks": dict(seq_lens=(3000, 2111), n_new=(200, 130), k_per_seq=(12, 7), k_max=12,
                               occupancy=0.6),
    # query tiles of 16 that straddle sequence boundaries (tensor-core scoring path)
    "prefill_tiles_straddle": dict(seq_lens=(9000, 300, 5000, 70), n_new=(30, 20, 17, 5), k_per_seq=(9, 3, 6, 2),
                                   k_max=9),
    # 48 (query, KV head) pairs: the decode entry runs one 2-CTA cluster per pair
    # (odd Top-K: unequal halves; short sequences: one half without usable blocks)
    "cluster_pairs": dict(seq_lens=tuple(range(70, 70 + 24 * 431, 431)), n_new=(1,) * 24, k_per_seq=(7,) * 24,
                          k_max=7),
    # fewer indexer heads than the 16 of a tensor-core tile (5: weights by cp.async, 8: by TMA)
    "prefill_5_idx_heads": dict(seq_lens=(20000,), n_new=(100,), k_per_seq=(10,), k_max=10, num_idx_heads=5),
    "prefill_8_idx_heads": dict(seq_lens=(5000, 3000), n_new=(40, 25), k_per_seq=(6, 5), k_max=6, num_idx_heads=8),
}


def _small_spec(name, profile="plain"):
    kw = dict(num_q_heads=16, num_kv_heads=2, num_idx_heads=16)
    kw.update(SMALL[name])
    return profiled(wk.WorkloadSpec(name, **kw), profile)


@pytest.mark.parametrize("fused", [False, True], ids=["score_topk", "fused_select"])
@pytest.mark.parametrize("decode", [True, False], ids=["decode_entry", "prefill_entry"])
@pytest.mark.parametrize("profile", PROFILES)
@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_cases_all_outputs(name, profile, decode, fused, cuda_device):
    wl, ref, bufs = _run(_small_spec(name, profile), 100 + len(name), cuda_device, decode=decode, fused=fused)
    compare(wl, ref, bufs, fused=fused)


def test_tensor_core_indexer_many_tile_switches(cuda_device):
    """Many short prefill chunks of long sequences: every 16-query tile straddles
    sequences, so each CTA of the tensor-core indexer switches block tiles many
    times and refills both of its coarse-key buffers (all scores compared)."""
    rng = np.random.default_rng(77)
    n = 120
    lens = tuple(int(x) for x in rng.integers(2000, 18000, size=n))
    n_new = tuple(int(x) for x in rng.integers(5, 31, size=n))
    spec = wk.WorkloadSpec("tc_tile_switches", seq_lens=lens, n_new=n_new, k_per_seq=(4,) * n, k_max=4,
                           num_q_heads=8, num_kv_heads=1, num_idx_heads=16)
    wl, ref, bufs = _run(spec, 2024, cuda_device, decode=False)
    compare(wl, ref, bufs)


@pytest.mark.parametrize("fused", [False, True], ids=["score_topk", "fused_select"])
@pytest.mark.parametrize("profile", PROFILES)
def test_tiny_decode_workload(profile, fused, cuda_device):
    wl, ref, bufs = _run(profiled(wk.tiny_decode(), profile), 1001, cuda_device, fused=fused)
    compare(wl, ref, bufs, fused=fused)


@pytest.mark.parametrize("fused", [False, True], ids=["score_topk", "fused_select"])
@pytest.mark.parametrize("profile", PROFILES)
def test_batched_gqa_decode_workload(profile, fused, cuda_device):
    spec = profiled(wk.batched_gqa_decode(), profile)
    wl, ref, bufs = _run(spec, 1002, cuda_device, fused=fused)
    compare(wl, ref, bufs, fused=fused)


@pytest.mark.slow
@pytest.mark.parametrize("fused", [False, True], ids=["score_topk", "fused_select"])
@pytest.mark.parametrize("profile", PROFILES)
def test_decode_1m_workload_all_outputs(profile, fused, cuda_device):
    wl, ref, bufs = _run(profiled(wk.decode_1m(), profile), 1003, cuda_device, fused=fused)
    compare(wl, ref, bufs, fused=fused)
    # the planted blocks shape the selection (non-trivial selections)
    planted = wl.planted.cpu().numpy()
    hits = [len(set(ref["sel"][s]) & set(planted[s])) for s in range(8)]
    assert min(hits) >= 1, hits


def _sample_queries(wl, n, rng):
    T = wl.spec.total_q
    pos = wl.q_pos.cpu().numpy()
    edge = [0, T - 1] + [i for i in range(T) if pos[i] % 64 in (0, 63)][:8]
    rest = rng.choice(T, size=min(T, n), replace=False).tolist()
    return sorted(set(edge + rest))


@pytest.mark.slow
@pytest.mark.parametrize("fused", [False, True], ids=["score_topk", "fused_prefill"])
@pytest.mark.parametrize("profile", PROFILES)
def test_chunked_prefill_workload_sampled(profile, fused, cuda_device):
    """Separate scoring (tensor cores) + Top-K, or the fused prefill pipeline
    (scoring and selection in one kernel, no score matrix, then attention)."""
    spec = profiled(wk.chunked_prefill(), profile)
    wl = wk.make_workload(spec, seed=1004, device=cuda_device)
    qs = _sample_queries(wl, 40, np.random.default_rng(0))
    ref = oracle_step(wl, queries=qs, want_scores=True)
    bufs, err = gpu_step(wl, decode=False, fused=fused)
    assert err == 0
    compare(wl, ref, bufs, fused=fused)
    # properties of every query at full size
    cnt = bufs["cnt"].cpu().numpy()
    sel = bufs["sel"].cpu().numpy()
    own = wl.q_pos.cpu().numpy() // 64
    assert (cnt == 64).all()
    assert (sel[:, -1] == own).all()                       # own block last (largest id)
    assert (np.diff(sel, axis=1) > 0).all()                # strictly ascending


@pytest.mark.slow
@pytest.mark.parametrize("decode,fused", [(True, False), (False, False), (True, True), (False, True)])
@pytest.mark.parametrize("profile", PROFILES)
def test_mixed_ragged_workload_sampled(profile, decode, fused, cuda_device):
    spec = profiled(wk.mixed_ragged(), profile)
    wl = wk.make_workload(spec, seed=1005, device=cuda_device)
    cu = wl.cu_q.cpu().numpy()
    decode_q = [int(cu[s]) for s in range(spec.num_seqs) if cu[s + 1] - cu[s] == 1]
    rng = np.random.default_rng(1)
    prefill_q = [int(x) for s in range(spec.num_seqs) if cu[s + 1] - cu[s] > 1
                 for x in rng.choice(np.arange(cu[s], cu[s + 1]), size=12, replace=False)]
    qs = sorted(decode_q + prefill_q)
    ref = oracle_step(wl, queries=qs, want_scores=True)
    bufs, err = gpu_step(wl, decode=decode, fused=fused)
    assert err == 0
    compare(wl, ref, bufs, fused=fused)


# ----------------------------------------------------------------------------- blocks of 128 / 256 / 512 tokens
BLOCK_SIZES = [128, 256, 512]
BLOCK_CASES = {
    # decode queries, some contexts shorter than K blocks, one inside its first block
    "decode_mix": dict(seq_lens=(5000, 700, 20000, 129, 64 * 40 + 5, 3), n_new=(1,) * 6,
                       k_per_seq=(4, 2, 6, 3, 5, 2), k_max=6),
    # prefill chunks (>= 16 queries per sequence: the tensor-core indexer), ragged tails
    "prefill_chunks": dict(seq_lens=(9000, 3000, 1100), n_new=(70, 33, 17), k_per_seq=(5, 3, 4), k_max=5,
                           occupancy=0.8),
    # 48 (query, KV head) pairs: 2-CTA clusters in the decode entry
    "cluster_pairs": dict(seq_lens=tuple(range(700, 700 + 24 * 913, 913)), n_new=(1,) * 24,
                          k_per_seq=(3,) * 24, k_max=3),
}


@pytest.mark.parametrize("fused", [False, True], ids=["score_topk", "fused_select"])
@pytest.mark.parametrize("decode", [True, False], ids=["decode_entry", "prefill_entry"])
@pytest.mark.parametrize("block_size", BLOCK_SIZES)
@pytest.mark.parametrize("name", sorted(BLOCK_CASES))
def test_block_sizes_all_outputs(name, block_size, decode, fused, cuda_device):
    kw = dict(num_q_heads=16, num_kv_heads=2, num_idx_heads=16, block_size=block_size)
    kw.update(BLOCK_CASES[name])
    spec = wk.sharp(wk.WorkloadSpec(f"{name}_b{block_size}", **kw))
    wl, ref, bufs = _run(spec, 300 + block_size + len(name), cuda_device, decode=decode, fused=fused)
    compare(wl, ref, bufs, fused=fused)


@pytest.mark.parametrize("block_size", BLOCK_SIZES)
def test_block_sizes_select_append(block_size, cuda_device):
    """The decode chain of the bench (selection with the append in its grid,
    then decode attention) with larger blocks: appended rows land in the
    right slots of the big pages and the results equal the oracle's."""
    kw = dict(num_q_heads=16, num_kv_heads=2, num_idx_heads=16, block_size=block_size)
    kw.update(BLOCK_CASES["decode_mix"])
    wl = wk.make_workload(wk.sharp(wk.WorkloadSpec("sa_b%d" % block_size, **kw)), seed=17, device=cuda_device)
    ref = oracle_step(wl)
    bufs, err = gpu_step(wl, overlap=True)
    assert err == 0
    compare(wl, ref, bufs, fused=True)
    _appended_rows_match(wl, wl.spec.num_seqs)


@pytest.mark.slow
@pytest.mark.parametrize("block_size", BLOCK_SIZES)
def test_decode_1m_block_sizes(block_size, cuda_device):
    wl, ref, bufs = _run(wk.sharp(wk.decode_1m_blocks(block_size)), 1003, cuda_device, fused=True, scores=False)
    compare(wl, ref, bufs, fused=True)


def test_single_launch_decode_refuses_larger_blocks(cuda_device):
    kw = dict(num_q_heads=16, num_kv_heads=2, num_idx_heads=16, block_size=128)
    kw.update(BLOCK_CASES["decode_mix"])
    wl = wk.make_workload(wk.WorkloadSpec("fd_b128", **kw), seed=18, device=cuda_device)
    with pytest.raises(dsa.DsaError):
        gpu_step(wl, fused_decode=True)


# ----------------------------------------------------------------------------- invariants on the GPU
def test_page_permutation_is_bit_identical(cuda_device):
    spec = _small_spec("prefill_two_chunks", "sharp")
    wl = wk.make_workload(spec, seed=7, device=cuda_device)
    wl2 = wk.make_workload(spec, seed=7, device=cuda_device)
    perm = torch.randperm(spec.num_pages, generator=torch.Generator().manual_seed(5)).to(cuda_device)
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(len(perm), device=cuda_device)
    wl2.k_pool = wl.k_pool[inv].contiguous()
    wl2.v_pool = wl.v_pool[inv].contiguous()
    wl2.kc_pool = wl.kc_pool[inv].contiguous()
    bt = wl.block_table.long()
    wl2.block_table = torch.where(bt >= 0, perm[bt.clamp(min=0)], -1).to(torch.int32).contiguous()
    b1, e1 = gpu_step(wl)
    b2, e2 = gpu_step(wl2)
    assert e1 == e2 == 0
    for k in ("sel", "cnt", "out", "lse"):
        assert torch.equal(b1[k], b2[k]), k


@pytest.mark.parametrize("block_size", [64, 256])
@pytest.mark.parametrize("fused", [False, True], ids=["score_topk", "fused_select"])
@pytest.mark.parametrize("decode", [True, False], ids=["decode_entry", "prefill_entry"])
def test_unwritten_cache_slots_holding_nan(decode, fused, block_size, cuda_device):
    """Slots of a sequence's last block past its length hold whatever the
    cache had there (here NaN in K and V).  They are masked out, and a zero
    softmax weight times NaN must not reach the output: results equal the
    oracle's, which never reads those slots."""
    kw = dict(num_q_heads=16, num_kv_heads=2, num_idx_heads=16, block_size=block_size)
    kw.update(SMALL["ragged_prefill_tail"])
    spec = wk.sharp(wk.WorkloadSpec(f"nan_tail_b{block_size}", **kw))
    wl = wk.make_workload(spec, seed=46, device=cuda_device)
    table = wl.block_table.cpu()
    for s_, L in enumerate(spec.seq_lens):
        if L % block_size:
            page = int(table[s_, (L - 1) // block_size])
            wl.k_pool[page, L % block_size:] = float("nan")
            wl.v_pool[page, L % block_size:] = float("nan")
    ref = oracle_step(wl)
    bufs, err = gpu_step(wl, decode=decode, fused=fused)
    assert err == 0
    assert not torch.isnan(bufs["out"]).any() and not torch.isnan(bufs["lse"]).any()
    compare(wl, ref, bufs, fused=fused)


def test_v_all_ones_gives_ones(cuda_device):
    spec = _small_spec("ragged_prefill_tail", "sharp")
    wl = wk.make_workload(spec, seed=8, device=cuda_device)
    wl.v_pool.fill_(1.0)
    wl.v_new.fill_(1.0)
    for decode in (True, False):
        b, e = gpu_step(wl, decode=decode)
        assert e == 0
        assert torch.all(b["out"] == 1.0)


def test_repeat_calls_reuse_workspace(cuda_device):
    # the split-KV workspace counters must be left at zero for the next call
    spec = _small_spec("many_seqs_decode", "sharp")
    wl = wk.make_workload(spec, seed=9, device=cuda_device)
    b, e = gpu_step(wl)
    first = b["out"].clone()
    for _ in range(3):
        b, e = gpu_step(wl, bufs=b)
        assert e == 0
        assert torch.equal(b["out"], first)
    assert int(b["workspace"][:4 * spec.total_q * spec.num_kv_heads].view(torch.int32).abs().sum()) == 0


@pytest.mark.parametrize("decode,fused,overlap", [(True, False, False), (True, True, True), (False, False, False),
                                                   (False, True, False)])
def test_prepared_step_matches_step(decode, fused, overlap, cuda_device):
    # a step prepared once and issued again gives what step() gives, bit for bit
    # (the appending selection takes decode batches only: one query per sequence)
    spec = _small_spec("many_seqs_decode" if overlap else "ragged_prefill_tail", "sharp")
    wl = wk.make_workload(spec, seed=12, device=cuda_device)
    want, e = gpu_step(wl, decode=decode, fused=fused, overlap=overlap)
    assert e == 0
    want = {k: want[k].clone() for k in ("sel", "cnt", "out", "lse")}
    cache, seqs, queries = _handles(wl)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ps = dsa.PreparedStep(cache, seqs, queries, k_new=wl.k_new, v_new=wl.v_new, kc_new=wl.kc_new, q=wl.q,
                          q_idx=wl.q_idx, w=wl.w, k_per_seq=wl.k_per_seq, k_max=spec.k_max, decode=decode,
                          fused_select=fused or overlap, overlap_append=overlap, dev_err=err)
    for _ in range(3):
        for k in ("out", "lse"):
            ps.bufs[k].fill_(float("nan"))
        got = ps()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        for k, v in want.items():
            assert torch.equal(got[k], v), k


# ----------------------------------------------------------------------------- device error flags
@pytest.mark.parametrize("fused", [False, True])
def test_bad_page_sets_flag_without_fault(fused, cuda_device):
    spec = _small_spec("k_covers_all")
    wl = wk.make_workload(spec, seed=10, device=cuda_device)
    wl.block_table[0, 1] = spec.num_pages + 5
    _, err = gpu_step(wl, fused=fused)
    assert err & dsa._lib.DEV_ERR_PAGE


@pytest.mark.parametrize("fused", [False, True])
def test_bad_position_and_k_set_flags(fused, cuda_device):
    spec = _small_spec("k_covers_all")
    wl = wk.make_workload(spec, seed=11, device=cuda_device)
    wl.q_pos[1] = int(wl.seq_lens[1]) + 3          # past the end of its sequence
    wl.k_per_seq[0] = 0
    b, err = gpu_step(wl, fused=fused)
    assert err & dsa._lib.DEV_ERR_POS
    assert err & dsa._lib.DEV_ERR_K
    assert int(b["cnt"][0]) == 0 and int(b["cnt"][1]) == 0


def test_host_validation_raises(cuda_device):
    spec = _small_spec("one_token")
    wl = wk.make_workload(spec, seed=12, device=cuda_device)
    cache, seqs, queries = _handles(wl)
    with pytest.raises(dsa.DsaError):
        dsa.index_score(cache, seqs, queries, wl.q_idx, wl.w, w_abs_max=1 << 12)
    with pytest.raises(ValueError):
        dsa.index_score(cache, seqs, queries, wl.q_idx.cpu(), wl.w)


def test_fused_select_equals_score_then_topk_on_ties(cuda_device):
    # all-equal coarse keys: every candidate ties, so the selection is decided
    # by the lowest-id rule alone, across chunk boundaries of the fused path
    spec = wk.WorkloadSpec("ties", seq_lens=(40000, 1500), n_new=(1, 3), k_per_seq=(33, 64), k_max=64,
                           num_q_heads=16, num_kv_heads=2)
    wl = wk.make_workload(spec, seed=31, device=cuda_device)
    wl.kc_pool.fill_(3)
    wl.kc_new.fill_(3)
    b1, e1 = gpu_step(wl, fused=False)
    b2, e2 = gpu_step(wl, fused=True)
    assert e1 == e2 == 0
    assert torch.equal(b1["sel"], b2["sel"]) and torch.equal(b1["cnt"], b2["cnt"])
    own = (wl.q_pos // 64).cpu()
    sel = b1["sel"].cpu()
    assert sel[0, :32].tolist() == list(range(32)) and int(sel[0, 32]) == int(own[0])


# ----------------------------------------------------------------------------- single-launch decode
def _decode_eligible(wl):
    """Queries whose sequence appends nothing before their own block (the
    single-launch decode step's precondition)."""
    spec = wl.spec
    cu = wl.cu_q.cpu().numpy()
    pos = wl.q_pos.cpu().numpy()
    ok = []
    for s in range(spec.num_seqs):
        first_new_block = (spec.seq_lens[s] - spec.n_new[s]) // 64
        for t in range(cu[s], cu[s + 1]):
            ok.append(spec.n_new[s] == 0 or pos[t] // 64 <= first_new_block)
    return np.array(ok, dtype=bool)


FUSED_DECODE_SMALL = sorted(n for n in SMALL if not n.startswith(("ragged_prefill", "prefill")))


@pytest.mark.parametrize("profile", PROFILES)
@pytest.mark.parametrize("name", FUSED_DECODE_SMALL)
def test_fused_decode_small_cases(name, profile, cuda_device):
    wl = wk.make_workload(_small_spec(name, profile), seed=100 + len(name), device=cuda_device)
    assert _decode_eligible(wl).all()
    ref = oracle_step(wl)
    bufs, err = gpu_step(wl, fused_decode=True)
    assert err == 0, f"device error bits {err}"
    compare(wl, ref, bufs, fused=True)


def test_fused_decode_flags_non_decode_queries(cuda_device):
    # prefill-shaped sequences: queries before the last appended block are
    # refused (cnt 0, DEV_ERR_POS); every other query is still exact
    wl = wk.make_workload(_small_spec("ragged_prefill_tail", "sharp"), seed=41, device=cuda_device)
    ok = _decode_eligible(wl)
    assert ok.any() and not ok.all()
    good = [int(t) for t in np.flatnonzero(ok)]
    ref = oracle_step(wl, queries=good)
    bufs, err = gpu_step(wl, fused_decode=True)
    assert err & dsa._lib.DEV_ERR_POS
    compare(wl, ref, bufs, fused=True)
    cnt = bufs["cnt"].cpu().numpy()
    assert (cnt[~ok] == 0).all()


@pytest.mark.parametrize("profile", PROFILES)
def test_fused_decode_tiny_workload(profile, cuda_device):
    wl, ref, bufs = _run(profiled(wk.tiny_decode(), profile), 1001, cuda_device, scores=False)
    b2, err = gpu_step(wl, fused_decode=True)
    assert err == 0
    compare(wl, ref, b2, fused=True)


@pytest.mark.parametrize("profile", PROFILES)
def test_fused_decode_batched_gqa_workload(profile, cuda_device):
    spec = profiled(wk.batched_gqa_decode(), profile)
    wl = wk.make_workload(spec, seed=1002, device=cuda_device)
    ref = oracle_step(wl)
    bufs, err = gpu_step(wl, fused_decode=True)
    assert err == 0
    compare(wl, ref, bufs, fused=True)


@pytest.mark.slow
@pytest.mark.parametrize("profile", PROFILES)
def test_fused_decode_1m_workload(profile, cuda_device):
    wl = wk.make_workload(profiled(wk.decode_1m(), profile), seed=1003, device=cuda_device)
    ref = oracle_step(wl)
    bufs, err = gpu_step(wl, fused_decode=True)
    assert err == 0
    compare(wl, ref, bufs, fused=True)


def test_fused_decode_repeat_calls_and_equals_three_kernel_path(cuda_device):
    # the workspace keeps an epoch: many calls on one workspace stay exact and
    # give the same bits as append -> select -> decode attention
    spec = wk.WorkloadSpec("fused_repeat", seq_lens=(5000, 64, 20000, 130), n_new=(1, 1, 1, 1),
                           k_per_seq=(9, 4, 33, 2), k_max=33, num_q_heads=16, num_kv_heads=2,
                           q_scale=wk.SHARP_Q_SCALE, v_scale=wk.SHARP_V_SCALE)
    wl = wk.make_workload(spec, seed=42, device=cuda_device)
    b_ref, e_ref = gpu_step(wl, fused=True)
    assert e_ref == 0
    b = None
    for _ in range(5):
        b, err = gpu_step(wl, bufs=b, fused_decode=True)
        assert err == 0
        for k in ("sel", "cnt", "out", "lse"):
            assert torch.equal(b[k], b_ref[k]), k
    ref = oracle_step(wl)
    compare(wl, ref, b, fused=True)


def test_fused_decode_wait_runs_out_and_recovers(cuda_device):
    """The single-launch step's wait for the appended tokens is bounded.  With a
    token count that can never be reached -- the workspace's appended-token
    counter (int32 word 2 of its 256-byte header) set far below zero before the
    call -- every producer gives up after the in-kernel limit (2^32 SM cycles,
    about 2 s), the call returns with DSA_DEV_ERR_WAIT, and the kernel leaves
    the workspace ready again: the next call is exact."""
    import time
    wl = wk.make_workload(_small_spec("many_seqs_decode", "sharp"), seed=45, device=cuda_device)
    ref = oracle_step(wl)
    bufs, err = gpu_step(wl, fused_decode=True)
    assert err == 0
    compare(wl, ref, bufs, fused=True)
    bufs["fused_ws"][:256].view(torch.int32)[2] = -(1 << 30)
    t0 = time.time()
    bufs, err = gpu_step(wl, bufs=bufs, fused_decode=True)   # appends the same tokens again: idempotent
    assert err & dsa._lib.DEV_ERR_WAIT
    assert time.time() - t0 < 120
    assert int(bufs["fused_ws"][:256].view(torch.int32)[2]) == 0
    bufs, err = gpu_step(wl, bufs=bufs, fused_decode=True)
    assert err == 0
    compare(wl, ref, bufs, fused=True)


@pytest.mark.parametrize("what", ["page", "pos", "k"])
def test_fused_decode_bad_metadata_sets_flags(what, cuda_device):
    spec = _small_spec("k_covers_all")
    wl = wk.make_workload(spec, seed=43, device=cuda_device)
    if what == "page":
        wl.block_table[0, 1] = spec.num_pages + 5
        bit = dsa._lib.DEV_ERR_PAGE
    elif what == "pos":
        wl.q_pos[1] = int(wl.seq_lens[1]) + 3
        bit = dsa._lib.DEV_ERR_POS
    else:
        wl.k_per_seq[0] = 0
        bit = dsa._lib.DEV_ERR_K
    b, err = gpu_step(wl, fused_decode=True)
    assert err & bit
    assert not err & dsa._lib.DEV_ERR_WAIT
    if what != "page":
        assert int(b["cnt"][0 if what == "k" else 1]) == 0


# ----------------------------------------------------------------------------- append overlapping the selection
@pytest.mark.parametrize("profile", PROFILES)
@pytest.mark.parametrize("name", FUSED_DECODE_SMALL)
def test_select_append_small_cases(name, profile, cuda_device):
    wl = wk.make_workload(_small_spec(name, profile), seed=200 + len(name), device=cuda_device)
    ref = oracle_step(wl)
    bufs, err = gpu_step(wl, overlap=True)
    assert err == 0, f"device error bits {err}"
    compare(wl, ref, bufs, fused=True)


def test_select_append_flags_non_decode_queries(cuda_device):
    wl = wk.make_workload(_small_spec("ragged_prefill_tail", "sharp"), seed=44, device=cuda_device)
    ok = _decode_eligible(wl)
    good = [int(t) for t in np.flatnonzero(ok)]
    ref = oracle_step(wl, queries=good)
    bufs, err = gpu_step(wl, overlap=True)
    assert err & dsa._lib.DEV_ERR_POS
    compare(wl, ref, bufs, fused=True)
    assert (bufs["cnt"].cpu().numpy()[~ok] == 0).all()


def _appended_rows_match(wl, n_tokens):
    """Every new token's K and V rows sit in their page slots, and the coarse
    key of the last new token of each touched block is that block's key."""
    spec = wl.spec
    table = wl.block_table.cpu().numpy()
    cu = wl.cu_q.cpu().numpy()
    lens = wl.seq_lens.cpu().numpy()
    kp, vp, kcp = wl.k_pool.cpu(), wl.v_pool.cpu(), wl.kc_pool.cpu()
    kn, vn, kcn = wl.k_new.cpu(), wl.v_new.cpu(), wl.kc_new.cpu()
    for s_ in range(spec.num_seqs):
        n = int(cu[s_ + 1] - cu[s_])
        for j in range(n):
            i = int(cu[s_]) + j
            pos = int(lens[s_]) - n + j
            bs = spec.block_size
            page, slot = int(table[s_, pos // bs]), pos % bs
            assert torch.equal(kp[page, slot], kn[i]) and torch.equal(vp[page, slot], vn[i]), (s_, j)
            if j == n - 1 or slot == bs - 1:
                assert torch.equal(kcp[page], kcn[i]), (s_, j)
    assert n_tokens == int(cu[-1])


def test_select_append_more_tokens_than_queries(cuda_device):
    """Three new tokens per sequence, all in its last block, but only the last
    one queries: the selection's grid carries three rows of append CTAs.  The
    selection equals the oracle's for those queries and the pool holds every
    new token."""
    spec = wk.WorkloadSpec("append3", seq_lens=(700, 1300, 70, 4000), n_new=(3, 3, 3, 3), k_per_seq=(4, 6, 2, 8),
                           k_max=8, num_q_heads=16, num_kv_heads=2, num_idx_heads=16)
    wl = wk.make_workload(spec, seed=321, device=cuda_device)
    cu = wl.cu_q.cpu().numpy()
    last = [int(cu[s_ + 1] - 1) for s_ in range(spec.num_seqs)]
    ref = oracle_step(wl, queries=last)
    idx = torch.as_tensor(last, device=cuda_device)
    cache, seqs, _ = _handles(wl)
    queries = dsa.QueryBatch(torch.arange(spec.num_seqs + 1, dtype=torch.int32, device=cuda_device),
                             wl.q_pos.index_select(0, idx).contiguous())
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    sel, cnt = dsa.select_blocks_append(cache, seqs, queries, wl.cu_q, wl.k_new, wl.v_new, wl.kc_new,
                                        wl.q_idx.index_select(0, idx).contiguous(),
                                        wl.w.index_select(0, idx).contiguous(), wl.k_per_seq, spec.k_max,
                                        dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(cnt.cpu().numpy(), ref["cnt"])
    assert np.array_equal(sel.cpu().numpy(), ref["sel"])
    _appended_rows_match(wl, 12)


def test_select_append_without_queries_still_appends(cuda_device):
    """No queries: no selection launch, only the append."""
    wl = wk.make_workload(_small_spec("many_seqs_decode"), seed=322, device=cuda_device)
    spec = wl.spec
    cache, seqs, _ = _handles(wl)
    queries = dsa.QueryBatch(torch.zeros(spec.num_seqs + 1, dtype=torch.int32, device=cuda_device),
                             torch.empty(0, dtype=torch.int32, device=cuda_device))
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    sel, cnt = dsa.select_blocks_append(cache, seqs, queries, wl.cu_q, wl.k_new, wl.v_new, wl.kc_new,
                                        wl.q_idx[:0], wl.w[:0], wl.k_per_seq, spec.k_max, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0 and sel.shape[0] == 0 and cnt.shape[0] == 0
    _appended_rows_match(wl, spec.num_seqs)


@pytest.mark.parametrize("profile", PROFILES)
def test_select_append_batched_gqa_workload(profile, cuda_device):
    spec = profiled(wk.batched_gqa_decode(), profile)
    wl = wk.make_workload(spec, seed=1002, device=cuda_device)
    ref = oracle_step(wl)
    bufs, err = gpu_step(wl, overlap=True)
    assert err == 0
    compare(wl, ref, bufs, fused=True)


@pytest.mark.slow
@pytest.mark.parametrize("profile", PROFILES)
def test_select_append_1m_workload(profile, cuda_device):
    wl = wk.make_workload(profiled(wk.decode_1m(), profile), seed=1003, device=cuda_device)
    ref = oracle_step(wl)
    bufs, err = gpu_step(wl, overlap=True)
    assert err == 0
    compare(wl, ref, bufs, fused=True)


# ----------------------------------------------------------------------------- many-query selection, every query
@pytest.mark.parametrize("variant", ["plain", "ties", "signed"])
@pytest.mark.parametrize("prefix", [58_000, 128_000], ids=["two_groups_per_warp", "four_groups_per_warp"])
def test_fused_selection_many_queries_every_query(prefix, variant, cuda_device):
    # 1200 queries of two sequences with about 900 (or 2000) visible blocks:
    # the fused selection runs one CTA per query with two (four) 64-block
    # groups per warp, the radix-select path; the separate score + Top-K calls
    # run the radix Top-K.  Every query's selection against the oracle, bit for
    # bit, on the pool as generated (no append).  "ties": the pool holds only
    # four distinct coarse keys (page p gets key p % 4), so every query's
    # threshold falls inside a group of hundreds of equal scores and the
    # lowest ids must win, and every third query has all-zero weights (every
    # score 0).  "signed": weights drawn from [-16, 16].
    spec = wk.WorkloadSpec("many_query_select", seq_lens=(prefix + 600, prefix - 1000), n_new=(600, 600),
                           k_per_seq=(16, 9), k_max=16, num_q_heads=8, num_kv_heads=1, num_idx_heads=16,
                           w_min=-16 if variant == "signed" else 0)
    wl = wk.make_workload(spec, seed=91, device=cuda_device)
    if variant == "ties":
        keys4 = wl.kc_pool[:4].clone()
        wl.kc_pool.copy_(keys4[torch.arange(wl.kc_pool.shape[0], device=cuda_device) % 4])
        wl.w[::3] = 0
    cache, seqs, queries = _handles(wl)
    ref = oracle_select(wl)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    sel, cnt = dsa.select_blocks(cache, seqs, queries, wl.q_idx, wl.w, wl.k_per_seq, spec.k_max, dev_err=err)
    scores = dsa.index_score(cache, seqs, queries, wl.q_idx, wl.w, dev_err=err)
    sel2, cnt2 = dsa.topk_blocks(seqs, queries, scores, wl.k_per_seq, spec.k_max, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for s_, c_ in ((sel, cnt), (sel2, cnt2)):
        assert np.array_equal(c_.cpu().numpy(), ref["cnt"])
        assert np.array_equal(s_.cpu().numpy(), ref["sel"])
