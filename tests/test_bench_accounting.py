"""The bench's roofline numerators, checked on CPU against the sizes the
workloads fix (no GPU, no kernel).

* 1M-context decode: 8 queries, each scanning the coarse keys of its 16,384
  visible blocks (64 B each) and reading the K and V slices of 32 selected
  blocks for 8 KV heads (64 tokens x 128 dims x 2 B each): 8 MiB + 64 MiB.
* Chunked prefill: the indexer's int8 ops are 2 x 16 heads x 64 dims per
  causally visible (query, block) pair; queries at 131072..135167 see
  p // 64 + 1 blocks each.
* Tiny decode: 64 visible blocks, 8 selected, one KV head.
"""
import bench
from dynamic_block_sparse_dsa_b200 import workloads as wk


class _W:
    def __init__(self, spec):
        self.spec = spec


def test_decode_1m_bytes():
    ab = bench.algorithmic_bytes(_W(wk.decode_1m()))
    assert ab["coarse_keys"] == 8 * 16384 * 64 == 8 * 2**20
    assert ab["kv"] == 8 * 8 * 32 * (64 * 128 * 2) * 2 == 64 * 2**20
    assert ab["total"] == 75_497_472
    # QK^T and PV over 64 query heads per selected block
    assert ab["flops"] == 8 * 32 * 4 * 64 * 64 * 128


def test_tiny_decode_bytes():
    ab = bench.algorithmic_bytes(_W(wk.tiny_decode()))
    assert ab["coarse_keys"] == 64 * 64
    assert ab["kv"] == 8 * 1 * (64 * 128 * 2) * 2
    assert ab["total"] == 266_240


def test_chunked_prefill_indexer_ops():
    spec = wk.chunked_prefill()
    first = spec.seq_lens[0] - spec.n_new[0]
    pairs = sum(p // 64 + 1 for p in range(first, first + spec.n_new[0]))
    assert pairs == 8_521_728
    assert pairs * spec.num_idx_heads * spec.idx_dim * 2 == 17_452_498_944
    ab = bench.algorithmic_bytes(_W(spec))
    # every query selects 64 blocks of its ~2080 visible ones
    assert ab["kv"] == spec.n_new[0] * 64 * 8 * (64 * 128 * 2) * 2


def test_overlapped_record_arithmetic(monkeypatch):
    """The overlapped-batches record turns its measured seconds per step into
    tokens/s and a fraction of the peak over the step's algorithmic bytes."""
    spec = wk.decode_1m()
    ab = bench.algorithmic_bytes(_W(spec))
    monkeypatch.setattr(bench, "time_overlapped", lambda cases, stream, device, steps: (20e-6, 240))
    rec = bench.overlapped_record([None] * 3, spec, ab, None, None, 200, 6450.3)
    assert rec["batches_in_flight"] == 3 and rec["steps_timed"] == 240
    assert rec["ms_per_step"] == 0.02
    assert rec["tokens_per_s"] == 400_000.0   # 8 queries per step
    assert rec["step_gbs"] == round(75_497_472 / 20e-6 / 1e9, 1) == 3774.9
    assert rec["step_frac_of_measured"] == round(3774.8736 / 6450.3, 4)
