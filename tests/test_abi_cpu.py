"""The C ABI loads on a machine without a GPU, exports every function that
include/dsa.h declares, and rejects bad arguments on the host before any
CUDA call (so these run without a device)."""
import ctypes
import os
import re

import pytest

from dynamic_block_sparse_dsa_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"^[A-Za-z_][\w \*]*?\b(dsa_\w+)\s*\(", text, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_pipeline():
    names = _declared_functions()
    for n in ("dsa_kv_append", "dsa_index_score", "dsa_topk_blocks", "dsa_sparse_attn_decode",
              "dsa_sparse_attn_prefill"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = _lib.load()
    for n in _declared_functions():
        assert hasattr(lib, n), n
        assert n in _lib.SIGNATURES, f"binding lacks a signature for {n}"


def test_status_strings_and_version():
    lib = _lib.load()
    assert lib.dsa_version() >= 100
    assert lib.dsa_status_string(0) == b"ok"
    assert lib.dsa_status_string(3) == b"int32 score range exceeded"


FAKE = 0x10000   # a 16-byte aligned address that is never dereferenced on these paths


def _cache(**kw):
    base = dict(k_pool=FAKE, v_pool=FAKE, kc_pool=FAKE, num_pages=4, block_size=64, num_kv_heads=8,
                head_dim=128, idx_dim=64)
    base.update(kw)
    return _lib.KvCacheC(**base)


def _seqs(**kw):
    base = dict(block_table=FAKE, max_blocks=4, seq_lens=FAKE, num_seqs=1)
    base.update(kw)
    return _lib.SeqsC(**base)


def _queries(**kw):
    base = dict(cu_q=FAKE, q_pos=FAKE, total_q=1)
    base.update(kw)
    return _lib.QueriesC(**base)


def _score(cache, seqs, queries, heads=16, wmax=16, qidx=FAKE):
    lib = _lib.load()
    return lib.dsa_index_score(ctypes.byref(cache), ctypes.byref(seqs), ctypes.byref(queries), qidx, FAKE,
                               heads, wmax, FAKE, None, None)


def test_host_validation_codes():
    c, s, q = _cache(), _seqs(), _queries()
    assert _score(_cache(block_size=32), s, q) == _lib.DSA_ERR_UNSUPPORTED
    assert _score(_cache(block_size=96), s, q) == _lib.DSA_ERR_UNSUPPORTED
    assert _score(_cache(block_size=1024), s, q) == _lib.DSA_ERR_UNSUPPORTED
    assert _score(_cache(head_dim=64), s, q) == _lib.DSA_ERR_UNSUPPORTED
    assert _score(_cache(k_pool=FAKE + 8), s, q) == _lib.DSA_ERR_INVALID_ARG      # misaligned
    assert _score(_cache(num_pages=0), s, q) == _lib.DSA_ERR_INVALID_ARG
    assert _score(c, _seqs(block_table=None), q) == _lib.DSA_ERR_INVALID_ARG
    assert _score(c, s, _queries(total_q=-1)) == _lib.DSA_ERR_INVALID_ARG
    assert _score(c, s, q, heads=17) == _lib.DSA_ERR_UNSUPPORTED
    assert _score(c, s, q, heads=0) == _lib.DSA_ERR_INVALID_ARG
    # 16 heads * |w| 16 * 64 * 128^2 = 2^28 is fine; |w| 128 would overflow int32
    assert _score(c, s, q, wmax=128) == _lib.DSA_ERR_RANGE
    assert _score(c, s, q, qidx=FAKE + 4) == _lib.DSA_ERR_INVALID_ARG
    # nothing to do is fine and launches nothing
    assert _score(c, s, _queries(total_q=0)) == _lib.DSA_OK


def test_attention_validation_codes():
    lib = _lib.load()
    c, s, q = _cache(), _seqs(), _queries()

    def dec(cache=c, hq=64, k_max=32, ws=None, ws_bytes=0, scale=0.088):
        return lib.dsa_sparse_attn_decode(ctypes.byref(cache), ctypes.byref(s), ctypes.byref(q), FAKE, hq,
                                          FAKE, FAKE, k_max, scale, FAKE, None, ws, ws_bytes, None, None)

    assert dec(hq=60) == _lib.DSA_ERR_INVALID_ARG           # not a multiple of the KV heads
    assert dec(hq=8 * 17) == _lib.DSA_ERR_UNSUPPORTED       # group of 17
    assert dec(k_max=0) == _lib.DSA_ERR_INVALID_ARG
    assert dec(scale=0.0) == _lib.DSA_ERR_INVALID_ARG
    need = lib.dsa_sparse_attn_decode_workspace_size(8, 64, 8, 32)
    assert need > 0 and need % 256 == 0
    assert lib.dsa_sparse_attn_decode_workspace_size(0, 64, 8, 32) == 0
    assert lib.dsa_sparse_attn_decode_workspace_size(8, 0, 8, 32) == 0


def test_topk_and_append_validation_codes():
    lib = _lib.load()
    s, q = _seqs(), _queries()
    assert lib.dsa_topk_blocks(ctypes.byref(s), ctypes.byref(q), FAKE, FAKE, 0, 64, FAKE, FAKE, None,
                               None) == _lib.DSA_ERR_INVALID_ARG
    for bad in (32, 96, 1024):
        assert lib.dsa_topk_blocks(ctypes.byref(s), ctypes.byref(q), FAKE, FAKE, 8, bad, FAKE, FAKE, None,
                                   None) == _lib.DSA_ERR_UNSUPPORTED
    assert lib.dsa_topk_blocks(ctypes.byref(s), ctypes.byref(_queries(total_q=0)), FAKE, FAKE, 8, 64, FAKE, FAKE,
                               None, None) == _lib.DSA_OK
    c = _cache()
    assert lib.dsa_kv_append(ctypes.byref(c), ctypes.byref(s), FAKE, -1, FAKE, FAKE, None, None,
                             None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_kv_append(ctypes.byref(c), ctypes.byref(s), FAKE, 1, FAKE + 2, FAKE, None, None,
                             None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_kv_append(ctypes.byref(c), ctypes.byref(s), FAKE, 0, FAKE, FAKE, None, None,
                             None) == _lib.DSA_OK


def test_select_validation_codes():
    lib = _lib.load()
    c, s, q = _cache(), _seqs(), _queries()

    def sel(queries=q, heads=16, wmax=16, k_max=32, ws=FAKE, ws_bytes=1 << 20):
        return lib.dsa_select_blocks(ctypes.byref(c), ctypes.byref(s), ctypes.byref(queries), FAKE, FAKE, heads,
                                     wmax, FAKE, k_max, FAKE, FAKE, ws, ws_bytes, None, None)

    assert sel(k_max=65) == _lib.DSA_ERR_UNSUPPORTED        # the fused path keeps at most 64
    assert sel(heads=17) == _lib.DSA_ERR_UNSUPPORTED
    assert sel(wmax=128) == _lib.DSA_ERR_RANGE
    assert sel(ws=None) == _lib.DSA_ERR_WORKSPACE
    assert sel(ws_bytes=16) == _lib.DSA_ERR_WORKSPACE
    assert sel(ws=FAKE + 8) == _lib.DSA_ERR_WORKSPACE        # misaligned workspace
    assert sel(queries=_queries(total_q=0), ws=None, ws_bytes=0) == _lib.DSA_OK
    assert lib.dsa_select_blocks_workspace_size(0) == 0
    assert lib.dsa_select_blocks_workspace_size(8) > 0


def test_select_append_validation_codes():
    lib = _lib.load()
    c, s = _cache(), _seqs()

    def sa(queries=None, cu_new=FAKE, total_new=1, k_new=FAKE, v_new=FAKE):
        queries = queries or _queries()
        return lib.dsa_select_blocks_append(ctypes.byref(c), ctypes.byref(s), ctypes.byref(queries), cu_new,
                                            total_new, k_new, v_new, None, FAKE, FAKE, 16, 16, FAKE, 32, FAKE,
                                            FAKE, FAKE, 1 << 20, None, None)

    assert sa(total_new=-1) == _lib.DSA_ERR_INVALID_ARG
    assert sa(cu_new=None) == _lib.DSA_ERR_INVALID_ARG
    assert sa(k_new=FAKE + 2) == _lib.DSA_ERR_INVALID_ARG     # misaligned token rows
    assert sa(v_new=None) == _lib.DSA_ERR_INVALID_ARG
    # no queries and no tokens: nothing to launch
    assert sa(queries=_queries(total_q=0), total_new=0) == _lib.DSA_OK


def test_binding_refuses_host_tensors():
    """The binding has no CPU path: host tensors are refused with an error
    before anything is called, whatever the entry point."""
    import torch

    import dynamic_block_sparse_dsa_b200 as dsa
    k = torch.zeros(4, 64, 1, 128, dtype=torch.bfloat16)
    cache = dsa.PagedKVCache(k, k.clone(), torch.zeros(4, 64, dtype=torch.int8))
    seqs = dsa.SeqBatch(torch.zeros(1, 4, dtype=torch.int32), torch.tensor([100], dtype=torch.int32))
    queries = dsa.QueryBatch(torch.tensor([0, 1], dtype=torch.int32), torch.tensor([99], dtype=torch.int32))
    q_idx = torch.zeros(1, 4, 64, dtype=torch.int8)
    w = torch.zeros(1, 4, dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA"):
        dsa.index_score(cache, seqs, queries, q_idx, w)
    with pytest.raises(ValueError, match="CUDA"):
        dsa.kv_append(cache, seqs, queries.cu_q, torch.zeros(1, 1, 128, dtype=torch.bfloat16),
                      torch.zeros(1, 1, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA"):
        dsa.step(cache, seqs, queries, k_new=torch.zeros(1, 1, 128, dtype=torch.bfloat16),
                 v_new=torch.zeros(1, 1, 128, dtype=torch.bfloat16), kc_new=None,
                 q=torch.zeros(1, 8, 128, dtype=torch.bfloat16), q_idx=q_idx, w=w,
                 k_per_seq=torch.tensor([2], dtype=torch.int32), k_max=2)


def test_noalloc_refuses_bad_calls_before_any_device_work():
    """The allocation-free decode entry runs every host check of the regular
    decode entry before it enqueues anything on its shared scratch.  Without a
    GPU any CUDA call would fail with DSA_ERR_CUDA, so getting the argument
    error back here shows that the check came first.  The pointers are
    dummies that are never dereferenced."""
    lib = _lib.load()
    s = _seqs()

    def na(cache=None, total_q=4_500_000, hq=64, k_max=32, scale=0.088, out=FAKE):
        cache = cache or _cache()
        q = _queries(total_q=total_q)
        return lib.dsa_sparse_attn_decode_noalloc(ctypes.byref(cache), ctypes.byref(s), ctypes.byref(q), FAKE, hq,
                                                  FAKE, FAKE, k_max, scale, out, None, None, None)

    # 63 query heads over 8 KV heads: the workspace size query says 0 for this,
    # and 4.5M queries x 8 KV heads of split counters would overrun the scratch
    assert na(hq=63) == _lib.DSA_ERR_INVALID_ARG
    assert na(hq=8 * 17, total_q=4) == _lib.DSA_ERR_UNSUPPORTED
    assert na(k_max=0) == _lib.DSA_ERR_INVALID_ARG
    assert na(scale=0.0) == _lib.DSA_ERR_INVALID_ARG
    assert na(out=FAKE + 2) == _lib.DSA_ERR_INVALID_ARG
    assert na(cache=_cache(block_size=32)) == _lib.DSA_ERR_UNSUPPORTED
    # valid arguments, but more scratch than the fixed array holds
    assert na() == _lib.DSA_ERR_WORKSPACE
    # nothing to do: accepted without touching the device
    assert na(total_q=0) == _lib.DSA_OK


def test_wide_score_validation_codes():
    """int64 and FP8 scoring and the int64 Top-K refuse bad arguments on the
    host (dummy pointers, never dereferenced)."""
    lib = _lib.load()
    c, s, q = _cache(), _seqs(), _queries()

    def fp8(wmax=16, heads=16, qidx=FAKE):
        return lib.dsa_index_score_fp8(ctypes.byref(c), ctypes.byref(s), ctypes.byref(q), qidx, FAKE, heads, wmax,
                                       FAKE, None, None)

    # 16 heads * 64 * (448 * 2^9)^2 * w must stay below 2^63: w = 1 << 20 is too large
    assert fp8(wmax=1 << 20) == _lib.DSA_ERR_RANGE
    assert fp8(wmax=-1) == _lib.DSA_ERR_INVALID_ARG
    assert fp8(heads=17) == _lib.DSA_ERR_UNSUPPORTED
    assert fp8(qidx=FAKE + 4) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_index_score_i64(ctypes.byref(c), ctypes.byref(s), ctypes.byref(q), FAKE, FAKE, 0, FAKE, None,
                                   None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_index_score_i64(ctypes.byref(_cache(block_size=100)), ctypes.byref(s), ctypes.byref(q), FAKE,
                                   FAKE, 4, FAKE, None, None) == _lib.DSA_ERR_UNSUPPORTED
    assert lib.dsa_index_score_i64(ctypes.byref(c), ctypes.byref(s), ctypes.byref(_queries(total_q=0)), FAKE, FAKE,
                                   4, FAKE, None, None) == _lib.DSA_OK

    def tk(k_max=8, bs=64, queries=q):
        return lib.dsa_topk_blocks_i64(ctypes.byref(s), ctypes.byref(queries), FAKE, FAKE, k_max, bs, FAKE, FAKE,
                                       None, None)

    assert tk(k_max=0) == _lib.DSA_ERR_INVALID_ARG
    assert tk(k_max=65) == _lib.DSA_ERR_UNSUPPORTED
    assert tk(bs=48) == _lib.DSA_ERR_UNSUPPORTED
    assert tk(queries=_queries(total_q=0)) == _lib.DSA_OK


def test_prepared_step_replays_the_calls_step_makes(monkeypatch):
    """PreparedStep records the library calls of one step() with their
    marshalled arguments and replays them; checked on the CPU with a fake
    library that records calls (nothing is launched)."""
    import torch

    import dynamic_block_sparse_dsa_b200 as dsa
    from dynamic_block_sparse_dsa_b200 import workloads as wk

    class FakeLib:
        def __init__(self):
            self.log = []

        def __getattr__(self, name):
            if name.endswith("_workspace_size"):
                return lambda *a: 256

            def call(*args):
                self.log.append((name, tuple(getattr(x, "value", x) if not hasattr(x, "_obj") else id(x._obj)
                                             for x in args[:-1])))
                return 0
            return call

    fake = FakeLib()
    monkeypatch.setattr(dsa._lib, "load", lambda: fake)
    monkeypatch.setattr(dsa, "load", lambda: fake)
    monkeypatch.setattr(dsa, "_ptr", lambda t: None if t is None else ctypes.c_void_p(t.data_ptr()))
    monkeypatch.setattr(dsa, "_stream", lambda s: ctypes.c_void_p(7))
    spec = wk.WorkloadSpec("ps", seq_lens=(900, 300), n_new=(1, 1), k_per_seq=(4, 4), k_max=4, num_q_heads=8,
                           num_kv_heads=1, num_idx_heads=4)
    wl = wk.make_workload(spec, seed=3)
    cache = dsa.PagedKVCache(wl.k_pool, wl.v_pool, wl.kc_pool)
    seqs = dsa.SeqBatch(wl.block_table, wl.seq_lens)
    queries = dsa.QueryBatch(wl.cu_q, wl.q_pos)
    kw = dict(k_new=wl.k_new, v_new=wl.v_new, kc_new=wl.kc_new, q=wl.q, q_idx=wl.q_idx, w=wl.w,
              k_per_seq=wl.k_per_seq, k_max=spec.k_max, fused_select=True, overlap_append=True)
    bufs = dsa.step(cache, seqs, queries, **kw)
    direct = [n for n, _ in fake.log]
    fake.log.clear()
    ps = dsa.PreparedStep(cache, seqs, queries, bufs=bufs, **kw)
    assert fake.log == []                       # recording launches nothing
    assert [c[0] for c in ps.calls] == direct == ["dsa_select_blocks_append", "dsa_sparse_attn_decode"]
    for _ in range(2):
        assert ps() is bufs
    assert [n for n, _ in fake.log] == direct * 2
    assert fake.log[0][1] == fake.log[2][1]     # same marshalled arguments every time


def test_stager_validates_on_the_host():
    lib = _lib.load()
    h = ctypes.c_void_p()
    assert lib.dsa_stager_create(0, None, ctypes.byref(h)) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_stager_create(4097, None, ctypes.byref(h)) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_stager_create(2, None, None) == _lib.DSA_ERR_INVALID_ARG
    arr = (ctypes.c_void_p * 1)(FAKE)
    nb = (ctypes.c_size_t * 1)(16)
    for fn in (lib.dsa_stager_begin, lib.dsa_stager_end):
        assert fn(None, 0, 1, arr, arr, nb) == _lib.DSA_ERR_INVALID_ARG
        assert fn(None, 0, 0, None, None, None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_stager_wait(None, 0) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_stager_join(None) == _lib.DSA_ERR_INVALID_ARG
    assert lib.dsa_stager_destroy(None) == _lib.DSA_OK
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:
        has_gpu = False
    if not has_gpu:   # without a device the streams cannot be made: a CUDA error, no handle
        assert lib.dsa_stager_create(2, None, ctypes.byref(h)) == _lib.DSA_ERR_CUDA
        assert not h.value


def test_prepared_step_refuses_a_closed_stager(monkeypatch):
    """A staged PreparedStep whose Stager was closed raises instead of handing
    the library a freed handle (checked with a fake library; nothing runs)."""
    import torch

    import dynamic_block_sparse_dsa_b200 as dsa

    class FakeLib:
        def __getattr__(self, name):
            if name.endswith("_workspace_size"):
                return lambda *a: 256
            if name == "dsa_stager_create":
                def create(n, s, out):
                    out._obj.value = 0x1234
                    return 0
                return create
            return lambda *a: 0

    fake = FakeLib()
    monkeypatch.setattr(dsa._lib, "load", lambda: fake)
    monkeypatch.setattr(dsa, "load", lambda: fake)
    monkeypatch.setattr(dsa, "_ptr", lambda t: None if t is None else ctypes.c_void_p(t.data_ptr() or 16))
    monkeypatch.setattr(dsa, "_host_ptr", lambda t: t.data_ptr())

    class FakeStream:
        cuda_stream = 7

    monkeypatch.setattr(torch.cuda, "current_stream", lambda: FakeStream())
    st = dsa.Stager(1, FakeStream())
    ps = dsa.PreparedStep.__new__(dsa.PreparedStep)
    ps.calls, ps.bufs, ps._stream = [], {}, ctypes.c_void_p(7)
    ps._stager = st
    ps._begin = ps._end = (lambda *a: 0, ())
    assert ps() == {}
    st.close()
    with pytest.raises(ValueError):
        ps()


def test_prepared_step_argument_checks(monkeypatch):
    """Host buffers need a stager, slots must exist, staged pairs must match in
    size (fake library; nothing runs)."""
    import torch

    import dynamic_block_sparse_dsa_b200 as dsa

    class FakeLib:
        def __getattr__(self, name):
            if name.endswith("_workspace_size"):
                return lambda *a: 256
            if name == "dsa_stager_create":
                def create(n, s, out):
                    out._obj.value = 0x1234
                    return 0
                return create
            return lambda *a: 0

    fake = FakeLib()
    monkeypatch.setattr(dsa._lib, "load", lambda: fake)
    monkeypatch.setattr(dsa, "load", lambda: fake)

    class FakeStream:
        cuda_stream = 7

    dev = torch.zeros(64, dtype=torch.uint8)
    host = torch.zeros(64, dtype=torch.uint8)
    host_short = torch.zeros(32, dtype=torch.uint8)
    # the staged pairs are checked for size before any pointer is taken
    monkeypatch.setattr(dsa, "_ptr", lambda t: ctypes.c_void_p(16))
    with pytest.raises(ValueError):
        dsa._regions([(dev, host_short)], False)
    dst, src, nb, n = dsa._regions([(dev, host)], False)
    assert n == 1 and nb[0] == 64
    monkeypatch.setattr(torch.cuda, "current_stream", lambda: FakeStream())
    st = dsa.Stager(2, FakeStream())
    monkeypatch.setattr(dsa, "step", lambda *a, **k: {})
    with pytest.raises(ValueError):
        dsa.PreparedStep(None, None, None, host_in=[(dev, host)])          # no stager
    with pytest.raises(ValueError):
        dsa.PreparedStep(None, None, None, stager=st, slot=2)               # no such slot
    ps = dsa.PreparedStep(None, None, None, stager=st, slot=1, host_in=[(dev, host)], host_out=[(dev, host)])
    with pytest.raises(ValueError):
        ps(stream=FakeStream())                                             # staged steps run on the stager's stream
    assert ps() == {}
    st.close()
