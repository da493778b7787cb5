"""The allocation-free decode entry point against the regular one.

dsa_sparse_attn_decode_noalloc serves callers that cannot call cudaMalloc
(an engine plugin's enqueue path, a runtime that owns all device memory): its
split-KV scratch is a fixed array inside the library.  Two calls in a row --
the second one finds the first one's leftovers in that shared array -- must
match dsa_sparse_attn_decode on the same selection, and the oracle, within the
parity tolerance of the other GPU tests.  The inputs use the discriminative
value scales (q x 256, v x sqrt(128)), so the outputs are O(0.1), far above
the tolerance.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import dynamic_block_sparse_dsa_b200 as dsa
from dynamic_block_sparse_dsa_b200 import workloads as wk
from oracle.harness import oracle_step

pytestmark = pytest.mark.gpu

OUT_MAX, OUT_MEAN, LSE_MAX = 2e-2, 2e-3, 2e-3


def _setup(spec, seed, device):
    wl = wk.make_workload(spec, seed=seed, device=device)
    cache = dsa.PagedKVCache(wl.k_pool, wl.v_pool, wl.kc_pool)
    seqs = dsa.SeqBatch(wl.block_table, wl.seq_lens)
    queries = dsa.QueryBatch(wl.cu_q, wl.q_pos)
    scores = dsa.index_score(cache, seqs, queries, wl.q_idx, wl.w)
    sel, cnt = dsa.topk_blocks(seqs, queries, scores, wl.k_per_seq, spec.k_max, block_size=spec.block_size)
    return wl, cache, seqs, queries, sel, cnt


@pytest.mark.parametrize("name,spec", [
    # 64 (query, KV head) pairs: the 2-CTA cluster split
    ("decode_8x32_blocks", wk.sharp(wk.WorkloadSpec("na1", seq_lens=(1 << 16,) * 8, n_new=(1,) * 8,
                                                    k_per_seq=(32,) * 8, k_max=32))),
    # 6 pairs: the split through the scratch's partial states and counters
    ("ragged_small", wk.sharp(wk.WorkloadSpec("na2", seq_lens=(900, 70, 4000), n_new=(1, 1, 1),
                                              k_per_seq=(8, 2, 16), k_max=16, num_q_heads=16, num_kv_heads=2))),
])
def test_noalloc_matches_regular_decode_twice(name, spec, cuda_device):
    wl, cache, seqs, queries, sel, cnt = _setup(spec, 77, cuda_device)
    # the oracle on the same (un-appended) pool and its own selection
    orc = oracle_step(wl, with_append=False)
    assert np.array_equal(sel.cpu().numpy(), orc["sel"]) and np.array_equal(cnt.cpu().numpy(), orc["cnt"])
    assert np.abs(orc["out"]).mean() >= 10 * OUT_MEAN     # the case can tell a wrong output from a right one
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    ref_out, ref_lse = dsa.sparse_attn_decode(cache, seqs, queries, wl.q, sel, cnt, dev_err=err)
    for _ in range(2):
        out = torch.full_like(wl.q, float("nan"))
        lse = torch.full(wl.q.shape[:2], float("nan"), dtype=torch.float32, device=cuda_device)
        dsa.sparse_attn_decode_noalloc(cache, seqs, queries, wl.q, sel, cnt, out=out, lse=lse, dev_err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        d = (out.double() - ref_out.double()).abs()
        assert float(d.max()) <= OUT_MAX and float(d.mean()) <= OUT_MEAN
        assert float((lse - ref_lse).abs().max()) <= LSE_MAX
        do = np.abs(out.double().cpu().numpy() - orc["out"])
        assert do.max() <= OUT_MAX and do.mean() <= OUT_MEAN, (do.max(), do.mean())
        assert np.abs(lse.double().cpu().numpy() - orc["lse"]).max() <= LSE_MAX


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_device):
    # 600,000 queries x 8 KV heads need more than the fixed 16 MiB scratch; the
    # call must refuse before touching any memory (the pointers are dummies)
    import ctypes
    lib = dsa._lib.load()
    L = dsa._lib
    fake = 0x10000
    cache = L.KvCacheC(fake, fake, fake, 4, 64, 8, 128, 64)
    seqs = L.SeqsC(fake, 4, fake, 1)
    queries = L.QueriesC(fake, fake, 600000)
    need = lib.dsa_sparse_attn_decode_workspace_size(600000, 64, 8, 32)
    assert need > 16 << 20
    rc = lib.dsa_sparse_attn_decode_noalloc(ctypes.byref(cache), ctypes.byref(seqs), ctypes.byref(queries),
                                            fake, 64, fake, fake, 32, 0.088, fake, None, None, None)
    assert rc == L.DSA_ERR_WORKSPACE
