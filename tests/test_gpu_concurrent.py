"""Independent batches stepped at the same time, each on a stream of its own
(the serving schedule in which one batch's latency-bound selection runs while
another batch's attention streams its pages).  The library keeps no state
shared between calls beyond the buffers each call is given, so every batch's
results equal, bit for bit, those of the same steps run one after another
(the kernels are deterministic), and no device error is raised."""
import pytest
import torch

import dynamic_block_sparse_dsa_b200 as dsa
from dynamic_block_sparse_dsa_b200 import workloads as wk

pytestmark = pytest.mark.gpu

HEADS = dict(num_q_heads=16, num_kv_heads=2, num_idx_heads=16)
SPECS = {
    # 40 decode sequences: split-KV decode attention
    "decode_40": dict(seq_lens=tuple(range(129, 129 + 40 * 97, 97)), n_new=(1,) * 40, k_per_seq=(8,) * 40,
                      k_max=8),
    # 24 decode sequences x 2 KV heads: one 2-CTA cluster per (query, KV head) pair
    "decode_cluster_pairs": dict(seq_lens=tuple(range(70, 70 + 24 * 431, 431)), n_new=(1,) * 24,
                                 k_per_seq=(7,) * 24, k_max=7),
    # prefill chunks whose query tiles straddle sequences (tensor-core scoring)
    "prefill_tiles": dict(seq_lens=(9000, 300, 5000, 70), n_new=(30, 20, 17, 5), k_per_seq=(9, 3, 6, 2), k_max=9),
}
PATHS = {"decode_40": [("fused_select", True), ("score_topk", False)],
         "decode_cluster_pairs": [("fused_select", True)],
         "prefill_tiles": [("fused_select", False), ("score_topk", False)]}
CASES = [(n, p, ov) for n in SPECS for p, ov in PATHS[n]]
N_BATCHES = 3
N_PASSES = 3
KEYS = ("sel", "cnt", "out", "lse")


class Batch:
    def __init__(self, name, seed, path, overlap, device, err):
        spec = wk.sharp(wk.WorkloadSpec(name, **HEADS, **SPECS[name]))
        self.wl = wl = wk.make_workload(spec, seed=seed, device=device)
        self.decode = all(n == 1 for n in spec.n_new)
        self.cache = dsa.PagedKVCache(wl.k_pool, wl.v_pool, wl.kc_pool)
        self.seqs, self.queries = dsa.SeqBatch(wl.block_table, wl.seq_lens), dsa.QueryBatch(wl.cu_q, wl.q_pos)
        self.kw = dict(k_new=wl.k_new, v_new=wl.v_new, kc_new=wl.kc_new, q=wl.q, q_idx=wl.q_idx, w=wl.w,
                       k_per_seq=wl.k_per_seq, k_max=spec.k_max, decode=self.decode,
                       fused_select=path == "fused_select", overlap_append=overlap, dev_err=err)
        self.bufs = None

    def step(self, stream=None):
        self.bufs = dsa.step(self.cache, self.seqs, self.queries, bufs=self.bufs, stream=stream, **self.kw)

    def snapshot(self):
        return {k: self.bufs[k].clone() for k in KEYS}

    def clear(self):
        for k in KEYS:
            self.bufs[k].fill_(-7 if k in ("sel", "cnt") else 0)


def _batches(name, path, overlap, device, err):
    bs = [Batch(name, 500 + 31 * i, path, overlap, device, err) for i in range(N_BATCHES)]
    want = []
    for b in bs:   # the steps one after another; repeated steps give the same results
        b.step()
        torch.cuda.synchronize()
        want.append(b.snapshot())
    assert int(err.item()) == 0
    # the batches differ, so results that crossed between them would show
    assert not torch.equal(want[0]["out"], want[1]["out"])
    return bs, want


def _check(bs, want, err):
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for i, (b, w) in enumerate(zip(bs, want)):
        for k in KEYS:
            assert torch.equal(b.bufs[k], w[k]), (i, k)


@pytest.mark.parametrize("name,path,overlap", CASES)
def test_batches_on_their_own_streams_match_steps_in_turn(name, path, overlap, cuda_device):
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    bs, want = _batches(name, path, overlap, cuda_device, err)
    for b in bs:
        b.clear()
    streams = [torch.cuda.Stream(cuda_device) for _ in bs]
    torch.cuda.synchronize()
    for _ in range(N_PASSES):   # issued pass by pass: the batches' launches interleave on the GPU
        for b, s in zip(bs, streams):
            b.step(stream=s)
    _check(bs, want, err)


@pytest.mark.parametrize("name", ["decode_40", "decode_cluster_pairs"])
def test_forked_graph_of_batches_matches_steps_in_turn(name, cuda_device):
    """The schedule captured once: every batch's steps on a stream forked from
    the capturing stream and joined back, replayed several times."""
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    bs, want = _batches(name, "fused_select", True, cuda_device, err)
    main = torch.cuda.Stream(cuda_device)
    sides = [torch.cuda.Stream(cuda_device) for _ in bs]
    g = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.graph(g, stream=main):
        for s in sides:
            s.wait_stream(main)
        for _ in range(N_PASSES):
            for b, s in zip(bs, sides):
                with torch.cuda.stream(s):
                    b.step()
        for s in sides:
            main.wait_stream(s)
    torch.cuda.synchronize()
    for b in bs:
        b.clear()
    torch.cuda.synchronize()
    for _ in range(4):
        g.replay()
    _check(bs, want, err)
    del g
