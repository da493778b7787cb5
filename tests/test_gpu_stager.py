"""Host staging (dsa_stager through dsa.Stager / dsa.PreparedStep): steps of
several batches issued back to back, each batch's inputs copied in from
pinned host buffers and its results copied back, the copies overlapping the
other batches' kernels.  Every step must see its own inputs and leave its own
results: the host outputs of each step equal, bit for bit, those of a plain
dsa.step on the same device inputs (the kernels are deterministic)."""
import pytest
import torch

import dynamic_block_sparse_dsa_b200 as dsa
from dynamic_block_sparse_dsa_b200 import workloads as wk

pytestmark = pytest.mark.gpu

SPEC = dict(seq_lens=tuple(range(129, 129 + 40 * 97, 97)), n_new=(1,) * 40, k_per_seq=(8,) * 40, k_max=8,
            num_q_heads=16, num_kv_heads=2, num_idx_heads=16)


def _kw(wl, q, q_idx):
    return dict(k_new=wl.k_new, v_new=wl.v_new, kc_new=wl.kc_new, q=q, q_idx=q_idx, w=wl.w,
                k_per_seq=wl.k_per_seq, k_max=wl.spec.k_max, fused_select=True, overlap_append=True)


@pytest.mark.parametrize("n_slots", [1, 3])
def test_staged_steps_return_their_own_results(n_slots, cuda_device):
    wl = wk.make_workload(wk.sharp(wk.WorkloadSpec("stager", **SPEC)), seed=71, device=cuda_device)
    cache = dsa.PagedKVCache(wl.k_pool, wl.v_pool, wl.kc_pool)
    seqs, queries = dsa.SeqBatch(wl.block_table, wl.seq_lens), dsa.QueryBatch(wl.cu_q, wl.q_pos)
    n_steps = 4 * n_slots + 1
    g = torch.Generator().manual_seed(5)
    # every step its own queries: q scaled as the sharp profile does, q_idx any int8
    qs = [(torch.randn(wl.q.shape, generator=g) * 256 / 128 ** 0.5).to(torch.bfloat16) for _ in range(n_steps)]
    qis = [torch.randint(-128, 128, wl.q_idx.shape, generator=g, dtype=torch.int8) for _ in range(n_steps)]
    want = []
    for q, qi in zip(qs, qis):
        b = dsa.step(cache, seqs, queries, **_kw(wl, q.to(cuda_device), qi.to(cuda_device)))
        torch.cuda.synchronize()
        want.append((b["out"].cpu(), b["lse"].cpu(), b["sel"].cpu()))

    stream = torch.cuda.Stream(cuda_device)
    st = dsa.Stager(n_slots, stream)
    slots = []
    for k in range(n_slots):
        d_q, d_qi = torch.empty_like(wl.q), torch.empty_like(wl.q_idx)
        h_q, h_qi = torch.empty(wl.q.shape, dtype=wl.q.dtype).pin_memory(), \
            torch.empty(wl.q_idx.shape, dtype=torch.int8).pin_memory()
        with torch.cuda.stream(stream):
            bufs = dsa.step(cache, seqs, queries, **_kw(wl, d_q.zero_(), d_qi.zero_()))
        h_out = torch.empty(bufs["out"].shape, dtype=bufs["out"].dtype).pin_memory()
        h_lse = torch.empty(bufs["lse"].shape, dtype=torch.float32).pin_memory()
        h_sel = torch.empty(bufs["sel"].shape, dtype=torch.int32).pin_memory()
        ps = dsa.PreparedStep(cache, seqs, queries, bufs=bufs, stager=st, slot=k,
                              host_in=[(d_q, h_q), (d_qi, h_qi)],
                              host_out=[(bufs["out"], h_out), (bufs["lse"], h_lse), (bufs["sel"], h_sel)],
                              **_kw(wl, d_q, d_qi))
        slots.append((ps, h_q, h_qi, h_out, h_lse, h_sel))
    torch.cuda.synchronize()

    def check(i):
        _, _, _, h_out, h_lse, h_sel = slots[i % n_slots]
        out, lse, sel = want[i]
        assert torch.equal(h_sel, sel), i
        assert torch.equal(h_out, out), i
        assert torch.equal(h_lse, lse), i

    for i in range(n_steps):
        k = i % n_slots
        ps, h_q, h_qi = slots[k][:3]
        if i >= n_slots:
            st.wait(k)           # the slot's previous read-back landed; its inputs were copied long before
            check(i - n_slots)
        h_q.copy_(qs[i])
        h_qi.copy_(qis[i])
        ps()
    for i in range(n_steps - n_slots, n_steps):
        st.wait(i % n_slots)
        check(i)
    st.join()
    torch.cuda.synchronize()
    st.close()


def test_stager_rejects_bad_slots(cuda_device):
    st = dsa.Stager(2)
    with pytest.raises(dsa.DsaError):
        st.wait(2)
    with pytest.raises(dsa.DsaError):
        st.wait(-1)
    st.join()
    torch.cuda.synchronize()
    st.close()
    st.close()   # a second close is a no-op
