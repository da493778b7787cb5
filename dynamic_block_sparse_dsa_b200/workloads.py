"""Seeded synthetic workloads for dynamic block-sparse attention.

This module only draws inputs: it holds none of the method's arithmetic (no
scoring, no selection, no attention).  Both the CUDA library's tests and the
oracle read the tensors it produces.

Every workload is a batch of sequences sharing one block-paged KV pool:

* ``k_pool`` / ``v_pool``: bf16 ``[num_pages][block_size][num_kv_heads][head_dim]``
  (the per-layer ``[block_id][token_in_block][head][dim]`` layout of
  "Day-0 Readiness for Trillion-Parameter Models ...", section "KV Cache Layout").
* ``kc_pool``: int8 ``[num_pages][idx_dim]``, one coarse key per KV block (the
  "compressed index blocks" of "Day-0 Adaptation for Massive LLMs ...",
  section 4(2)), indexed by the same physical page id.
* ``block_table``: int32 ``[num_seqs][max_blocks]`` logical block -> page,
  -1 past the end of a sequence.  Pages are a seeded random permutation.
* Queries are the sequence's newest tokens: sequence s has ``n_new[s]`` new
  tokens at positions ``seq_len - n_new .. seq_len - 1``; ``cu_q`` holds the
  ragged offsets and ``q_pos`` the positions.  The new tokens' K/V rows
  (``k_new``/``v_new``) and coarse-key rows (``kc_new``) are inputs of the
  append step.

Value distributions: bf16 q/k/v ~ N(0,1)/sqrt(head_dim), q times ``q_scale``
and v times ``v_scale`` for the discriminative cases (``sharp()``: logits with
standard deviation 2 and unit-variance values, so that attention outputs are
O(0.1) rather than O(0.002)); int8 indexer queries and coarse keys uniform in
[-127, 127]; int32 head weights uniform in [w_min, w_max] (w_min = 0 unless a
case asks for signed weights).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import Optional

import torch

# standard deviation of one int8 entry drawn uniformly from [-127, 127]
_SIGMA_U8 = math.sqrt((255 ** 2 - 1) / 12.0)


@dataclass(frozen=True)
class WorkloadSpec:
    """Shape of one synthetic batch (see module docstring for the recipe)."""
    name: str
    seq_lens: tuple            # context length of every sequence after the append
    n_new: tuple               # new tokens (= queries) of every sequence
    k_per_seq: tuple           # Top-K blocks of every sequence
    k_max: int
    num_q_heads: int = 64
    num_kv_heads: int = 8
    head_dim: int = 128
    num_idx_heads: int = 16
    idx_dim: int = 64
    block_size: int = 64
    w_max: int = 16
    w_min: int = 0             # signed-weight cases draw w uniformly from [w_min, w_max]
    occupancy: float = 1.0     # fraction of pool pages that hold a sequence's block
    plant: int = 0             # planted blocks per sequence (decode sequences)
    plant_sigma: float = 3.0
    q_scale: float = 1.0       # multiplies q before bf16 rounding (sharper softmax)
    v_scale: float = 1.0       # multiplies v (pool and new tokens) before bf16 rounding

    @property
    def num_seqs(self) -> int:
        return len(self.seq_lens)

    @property
    def total_q(self) -> int:
        return int(sum(self.n_new))

    @property
    def blocks_per_seq(self) -> list:
        return [-(-L // self.block_size) for L in self.seq_lens]

    @property
    def max_blocks(self) -> int:
        return max(self.blocks_per_seq)

    @property
    def num_pages(self) -> int:
        used = sum(self.blocks_per_seq)
        return used if self.occupancy >= 1.0 else int(math.ceil(used / self.occupancy))


def _cpu_gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def tiny_decode() -> WorkloadSpec:
    """1 query at position 4095 of a 4096-token context; 8 q heads, 1 KV head,
    4 indexer heads; Top-K = 8."""
    return WorkloadSpec("tiny_decode", seq_lens=(4096,), n_new=(1,), k_per_seq=(8,), k_max=8,
                        num_q_heads=8, num_kv_heads=1, num_idx_heads=4)


def batched_gqa_decode(seed: int = 1002, batch: int = 32) -> WorkloadSpec:
    """32 decode sequences, context lengths uniform in [8K, 64K]; 64/8 heads; K = 32."""
    g = _cpu_gen(seed)
    lens = torch.randint(8192, 65536 + 1, (batch,), generator=g).tolist()
    return WorkloadSpec("batched_gqa_decode", seq_lens=tuple(lens), n_new=(1,) * batch,
                        k_per_seq=(32,) * batch, k_max=32)


def decode_1m(batch: int = 8) -> WorkloadSpec:
    """8 decode sequences at 1,048,576 tokens (16,384 blocks); K = 32; 32 planted
    blocks per sequence."""
    return WorkloadSpec("decode_1m", seq_lens=(1 << 20,) * batch, n_new=(1,) * batch,
                        k_per_seq=(32,) * batch, k_max=32, plant=32)


def decode_1m_blocks(block_size: int, batch: int = 8) -> WorkloadSpec:
    """decode_1m with blocks of ``block_size`` tokens and the same selected-token
    budget (Top-K = 2048 / block_size blocks, that many planted blocks)."""
    k = 2048 // block_size
    return WorkloadSpec(f"decode_1m_b{block_size}", seq_lens=(1 << 20,) * batch, n_new=(1,) * batch,
                        k_per_seq=(k,) * batch, k_max=k, plant=k, block_size=block_size)


def decode_128k(batch: int = 8) -> WorkloadSpec:
    """decode_1m's shape at a 131,072-token context (2,048 blocks): the same
    Top-K 32 attention work with a 4 GiB pool, small enough for profiling."""
    return WorkloadSpec("decode_128k", seq_lens=(1 << 17,) * batch, n_new=(1,) * batch,
                        k_per_seq=(32,) * batch, k_max=32, plant=32)


def chunked_prefill(prefix: int = 131072, chunk: int = 4096) -> WorkloadSpec:
    """4096 new query tokens at positions 131072..135167 after a 128K prefix; K = 64."""
    return WorkloadSpec("chunked_prefill", seq_lens=(prefix + chunk,), n_new=(chunk,),
                        k_per_seq=(64,), k_max=64)


def mixed_ragged(seed: int = 1005, n_decode: int = 64, n_prefill: int = 2,
                 chunk: int = 2048) -> WorkloadSpec:
    """64 decode sequences + 2 prefill chunks of 2048 tokens; context lengths
    log-uniform in [4K, 256K]; pool at 70% occupancy; K per sequence drawn from
    {16, 32, 64}.  Each prefill chunk is the last 2048 tokens of its sequence;
    sequence order is shuffled so the chunks sit inside the batch."""
    g = _cpu_gen(seed)
    n = n_decode + n_prefill
    u = torch.rand((n,), generator=g, dtype=torch.float64)
    lens = torch.exp(math.log(4096) + u * (math.log(262144) - math.log(4096))).floor().long()
    lens = lens.clamp(4096, 262144).tolist()
    new = [1] * n_decode + [chunk] * n_prefill
    ks = [(16, 32, 64)[i] for i in torch.randint(0, 3, (n,), generator=g).tolist()]
    order = torch.randperm(n, generator=g).tolist()
    return WorkloadSpec("mixed_ragged", seq_lens=tuple(lens[i] for i in order),
                        n_new=tuple(new[i] for i in order), k_per_seq=tuple(ks[i] for i in order),
                        k_max=64, occupancy=0.7)


NAMED = {
    "tiny_decode": tiny_decode,
    "batched_gqa_decode": batched_gqa_decode,
    "decode_1m": decode_1m,
    "decode_128k": decode_128k,
    "decode_1m_b128": lambda: decode_1m_blocks(128),
    "decode_1m_b256": lambda: decode_1m_blocks(256),
    "decode_1m_b512": lambda: decode_1m_blocks(512),
    "chunked_prefill": chunked_prefill,
    "mixed_ragged": mixed_ragged,
}


@dataclass
class Workload:
    spec: WorkloadSpec
    seed: int
    k_pool: torch.Tensor
    v_pool: torch.Tensor
    kc_pool: torch.Tensor
    block_table: torch.Tensor
    seq_lens: torch.Tensor
    cu_q: torch.Tensor
    q_pos: torch.Tensor
    q: torch.Tensor
    q_idx: torch.Tensor
    w: torch.Tensor
    k_per_seq: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    kc_new: torch.Tensor
    planted: Optional[torch.Tensor] = None   # [num_seqs][plant] logical blocks, or None
    extra: dict = field(default_factory=dict)

    @property
    def device(self):
        return self.k_pool.device

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.spec.head_dim)


def _normal_bf16(shape, scale, gen, device):
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    flat = out.view(-1)
    step = 1 << 28
    for i in range(0, flat.numel(), step):
        part = flat[i:i + step]
        part.normal_(0.0, 1.0, generator=gen)
        part.mul_(scale)
    return out


def make_workload(spec: WorkloadSpec, seed: int = 0, device="cpu") -> Workload:
    """Draw every tensor of ``spec`` on ``device`` from generators seeded by ``seed``.

    Sizes and the page permutation come from a CPU generator (identical on any
    device); values come from a generator on ``device``.
    """
    device = torch.device(device)
    gcpu = _cpu_gen(seed)
    gdev = torch.Generator(device=device)
    gdev.manual_seed(seed + 7919)

    bs = spec.block_size
    nb = spec.blocks_per_seq
    num_pages = spec.num_pages
    used = sum(nb)
    pages = torch.randperm(num_pages, generator=gcpu)[:used].to(torch.int32)
    table = torch.full((spec.num_seqs, spec.max_blocks), -1, dtype=torch.int32)
    off = 0
    for s, n in enumerate(nb):
        table[s, :n] = pages[off:off + n]
        off += n

    n_new = torch.tensor(spec.n_new, dtype=torch.int64)
    lens = torch.tensor(spec.seq_lens, dtype=torch.int64)
    if bool((n_new > lens).any()) or bool((n_new < 0).any()):
        raise ValueError("every sequence needs 0 <= n_new <= seq_len")
    cu = torch.zeros(spec.num_seqs + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(n_new, 0)
    pos = torch.cat([torch.arange(L - n, L, dtype=torch.int64) for L, n in zip(spec.seq_lens, spec.n_new)])
    T = spec.total_q

    hd = spec.head_dim
    scale = 1.0 / math.sqrt(hd)
    k_pool = _normal_bf16((num_pages, bs, spec.num_kv_heads, hd), scale, gdev, device)
    v_pool = _normal_bf16((num_pages, bs, spec.num_kv_heads, hd), scale * spec.v_scale, gdev, device)
    kc_pool = torch.randint(-127, 128, (num_pages, spec.idx_dim), generator=gdev, device=device,
                            dtype=torch.int8)
    q = _normal_bf16((T, spec.num_q_heads, hd), scale * spec.q_scale, gdev, device)
    q_idx = torch.randint(-127, 128, (T, spec.num_idx_heads, spec.idx_dim), generator=gdev,
                          device=device, dtype=torch.int8)
    w = torch.randint(spec.w_min, spec.w_max + 1, (T, spec.num_idx_heads), generator=gdev, device=device,
                      dtype=torch.int32)
    k_new = _normal_bf16((T, spec.num_kv_heads, hd), scale, gdev, device)
    v_new = _normal_bf16((T, spec.num_kv_heads, hd), scale * spec.v_scale, gdev, device)
    kc_new = torch.randint(-127, 128, (T, spec.idx_dim), generator=gdev, device=device,
                           dtype=torch.int8)

    wl = Workload(spec=spec, seed=seed, k_pool=k_pool, v_pool=v_pool, kc_pool=kc_pool,
                  block_table=table.to(device), seq_lens=lens.to(torch.int32).to(device),
                  cu_q=cu.to(torch.int32).to(device), q_pos=pos.to(torch.int32).to(device),
                  q=q, q_idx=q_idx, w=w,
                  k_per_seq=torch.tensor(spec.k_per_seq, dtype=torch.int32, device=device),
                  k_new=k_new, v_new=v_new, kc_new=kc_new)
    if spec.plant:
        _plant(wl, gcpu)
    return wl


def _plant(wl: Workload, gcpu: torch.Generator) -> None:
    """Raise the coarse keys of ``plant`` seeded blocks per sequence.

    For each sequence with one query t: u = sign(sum_h w[t,h] q_idx[t,h,:])
    (0 -> +1); planted key = clamp(kc + delta*u, -127, 127) with the smallest
    integer delta in [0, 254] whose mean lift of the weighted-query dot
    product, (sum_h w q_idx) . (kc' - kc), reaches plant_sigma standard
    deviations of that dot product over uniform int8 keys.  The appended
    token's own block is never planted.  The new-token coarse-key row of a
    planted block is left as drawn (the own block is the only one touched).
    """
    spec = wl.spec
    cu = wl.cu_q.cpu().tolist()
    planted = torch.full((spec.num_seqs, spec.plant), -1, dtype=torch.int32)
    for s in range(spec.num_seqs):
        if cu[s + 1] - cu[s] != 1:
            continue
        t = cu[s]
        own = (spec.seq_lens[s] - 1) // spec.block_size
        # never plant in a block the append touches (that row gets overwritten)
        if own < spec.plant:
            continue
        blocks = torch.randperm(own, generator=gcpu)[:spec.plant].sort().values
        planted[s] = blocks.to(torch.int32)
        qbar = (wl.w[t].to(torch.int64)[:, None] * wl.q_idx[t].to(torch.int64)).sum(0)
        u = torch.where(qbar >= 0, 1, -1).to(torch.int64)
        pages = wl.block_table[s, blocks.to(wl.block_table.device).long()].long()
        kc = wl.kc_pool[pages].to(torch.int64)
        target = spec.plant_sigma * float(torch.linalg.vector_norm(qbar.double())) * _SIGMA_U8

        def lift(delta):
            kp = (kc + delta * u).clamp(-127, 127)
            return float(((kp - kc) * qbar).sum(1).double().mean())

        lo, hi = 0, 254
        if lift(hi) >= target:
            while lo < hi:
                mid = (lo + hi) // 2
                if lift(mid) >= target:
                    hi = mid
                else:
                    lo = mid + 1
        delta = hi
        wl.kc_pool[pages] = (kc + delta * u).clamp(-127, 127).to(torch.int8)
        wl.extra.setdefault("plant_delta", []).append(delta)
    wl.planted = planted.to(wl.device)


def e4m3_indexer(wl: Workload, seed: int = 0):
    """FP8 (E4M3) inputs for the FP8 indexer, drawn on the workload's device:
    (q_idx codes uint8 [T][H][idx_dim], coarse-key codes uint8 [num_pages][idx_dim]).
    Magnitudes are 2^u with u uniform in [-10, 9] and a random sign, clamped to
    the E4M3 range (448) and rounded by torch's float8 conversion, so the codes
    cover subnormals and the whole exponent range; no NaN code is drawn."""
    spec = wl.spec
    g = torch.Generator(device=wl.device)
    g.manual_seed(seed + 104729)

    def draw(shape):
        u = torch.rand(shape, generator=g, device=wl.device) * 19.0 - 10.0
        sign = torch.where(torch.rand(shape, generator=g, device=wl.device) < 0.5, -1.0, 1.0)
        x = (torch.exp2(u) * sign).clamp(-448.0, 448.0)
        return x.to(torch.float8_e4m3fn).view(torch.uint8)

    return draw((spec.total_q, spec.num_idx_heads, spec.idx_dim)), draw((spec.num_pages, spec.idx_dim))


def scaled(spec: WorkloadSpec, **kw) -> WorkloadSpec:
    """A copy of ``spec`` with fields replaced (e.g. q_scale, name)."""
    return replace(spec, **kw)


# q x 256 makes the logit q.k/sqrt(128) a N(0, 2^2) variable (q, k ~ N(0,1)/sqrt(128)
# per element), so the softmax over a few thousand tokens is dominated by a few
# dozen of them; v x sqrt(128) makes the values N(0,1).  The attention output
# is then O(0.1-1), far above the 2e-3 mean tolerance, and a wrong head, page
# or weight moves it by O(0.1).
SHARP_Q_SCALE = 256.0
SHARP_V_SCALE = math.sqrt(128.0)


def sharp(spec: WorkloadSpec) -> WorkloadSpec:
    """``spec`` with the discriminative value scales (see SHARP_Q_SCALE)."""
    return replace(spec, q_scale=SHARP_Q_SCALE, v_scale=SHARP_V_SCALE)
