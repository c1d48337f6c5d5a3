"""Seeded synthetic inputs for the paged-attention hot path.

This module builds the *inputs* only: sequence lengths, physical-block
assignment through a FIFO free list, block tables, slot mappings and random
q / K / V values.  It contains none of the attention arithmetic; both the
oracle (``oracle/``) and the CUDA library are fed from here and neither is
imported by it.

Workload shapes follow the pages' examples:

* LLaMA-2-70B-like GQA shapes (80 layers, 8 KV heads, head_dim 128, FP16) from
  the KV_Cache_Size worked example in "大模型推理内存优化从 KV Cache 分页到连续批
  处理的工程实践", section "KV Cache 的内存开销与分页机制";
* request lengths between 50 and 8000 tokens (same page, opening section);
* 16-token physical blocks handed out by a FIFO pool (same page, section
  "生产级推理引擎的内存管理与调度", ``BlockPool``: allocate pops the front of
  the free list, free pushes to the back);
* prefix blocks shared by several sequences through reference counts (page
  "KV Cache管理优化：大模型推理显存瓶颈突破", section 4.1).

No public dataset is involved: the pages name none, and every value is drawn
from seeded generators (numpy PCG64 for structure, torch's generator for the
bulk tensors) so that a workload is reproducible from its seed.
"""
from __future__ import annotations

import collections
import dataclasses
import math
from typing import Dict, List, Optional

import numpy as np
import torch

HEAD_DIM = 128


class BlockPool:
    """FIFO pool of physical block ids (harness only).

    Mirrors the pool of the pages' scheduler: the free list starts as the
    ids in order; ``allocate`` takes the front, ``free`` appends to the back.
    The harness shuffles the initial free list with the workload seed so that
    block tables are random permutations of the pool.
    """

    def __init__(self, num_blocks: int, rng: Optional[np.random.Generator] = None):
        ids = np.arange(num_blocks, dtype=np.int64)
        if rng is not None:
            ids = rng.permutation(ids)
        self.free_blocks = collections.deque(int(i) for i in ids)
        self.total_blocks = num_blocks
        self.refcount: Dict[int, int] = {}

    def available(self) -> int:
        return len(self.free_blocks)

    def allocate(self) -> int:
        if not self.free_blocks:
            raise RuntimeError("block pool exhausted")
        b = self.free_blocks.popleft()
        self.refcount[b] = 1
        return b

    def add_ref(self, block_id: int) -> None:
        self.refcount[block_id] += 1

    def release(self, block_id: int) -> None:
        self.refcount[block_id] -= 1
        if self.refcount[block_id] == 0:
            del self.refcount[block_id]
            self.free_blocks.append(block_id)


def _num_blocks_for(tokens: int, block_size: int) -> int:
    # harness-side block count for allocation (same rule the scheduler uses)
    return -(-tokens // block_size)


@dataclasses.dataclass
class PagedBatch:
    """One batch of paged-attention inputs, all torch tensors on ``device``.

    Shapes: ``k_cache``/``v_cache`` [num_blocks, block_size, num_kv_heads, D];
    ``block_tables`` int32 [B, max_blocks]; ``seq_lens`` int32 [B] (context
    length *including* the tokens appended this step); ``q`` [sum(q_lens), Hq, D]
    (one row per sequence for decode); ``k_new``/``v_new`` [T, Hkv, D] and
    ``slot_mapping`` int32 [T] for the tokens appended this step;
    ``query_start_loc`` int32 [B+1] (prefill only).
    """

    name: str
    dtype: torch.dtype
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    seq_lens: torch.Tensor
    block_tables: torch.Tensor
    q: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    slot_mapping: torch.Tensor
    query_start_loc: Optional[torch.Tensor] = None
    shared_prefix_blocks: int = 0
    group_size: int = 1
    # FP8 (e4m3) caches: k_cache / v_cache hold uint8 codes, these the fp32 per-kv-head
    # scales; None for fp16/bf16 caches
    k_scale: Optional[torch.Tensor] = None
    v_scale: Optional[torch.Tensor] = None
    # groups of consecutive sequences sharing their first blocks: int32 [groups + 1]
    # (group g = sequences group_starts[g] .. group_starts[g+1]-1) and the shared token
    # count of each group, int32 [groups]; None without sharing
    group_starts: Optional[torch.Tensor] = None
    prefix_lens: Optional[torch.Tensor] = None

    @property
    def num_seqs(self) -> int:
        return int(self.seq_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_seq_len(self) -> int:
        return int(self.seq_lens.max().item()) if self.num_seqs else 0

    @property
    def max_query_len(self) -> int:
        if self.query_start_loc is None:
            return 1
        d = self.query_start_loc[1:] - self.query_start_loc[:-1]
        return int(d.max().item()) if d.numel() else 0

    def to(self, device) -> "PagedBatch":
        kw = {}
        for f in dataclasses.fields(self):
            v = getattr(self, f.name)
            kw[f.name] = v.to(device) if isinstance(v, torch.Tensor) else v
        return PagedBatch(**kw)


def _randn(shape, dtype, gen, device):
    return torch.randn(shape, generator=gen, dtype=torch.float32, device=device).to(dtype)


def _assign_tables(seq_lens: List[int], block_size: int, num_blocks: int,
                   rng: np.random.Generator, shared_groups: Optional[List[List[int]]] = None,
                   shared_prefix_tokens: int = 0):
    """Hand out physical blocks from a shuffled FIFO pool.

    Blocks are allocated in the order a continuous-batching engine would
    request them: position by position, every sequence that reaches a new
    block takes one from the front of the free list.  Sequences listed
    together in ``shared_groups`` share their first
    ``shared_prefix_tokens / block_size`` blocks (allocated once, then
    reference-counted), the way parallel sampling shares a prompt.
    """
    pool = BlockPool(num_blocks, rng)
    B = len(seq_lens)
    nblk = [_num_blocks_for(L, block_size) for L in seq_lens]
    max_blocks = max([1] + nblk)
    tables = np.zeros((B, max_blocks), dtype=np.int32)
    owned = [0] * B
    if shared_groups:
        assert shared_prefix_tokens % block_size == 0
        npref = shared_prefix_tokens // block_size
        for grp in shared_groups:
            lead = grp[0]
            for j in range(npref):
                b = pool.allocate()
                for s in grp:
                    tables[s, j] = b
                    if s != lead:
                        pool.add_ref(b)
            for s in grp:
                owned[s] = npref
    for j in range(max_blocks):
        for s in range(B):
            if owned[s] <= j < nblk[s]:
                tables[s, j] = pool.allocate()
                owned[s] = j + 1
    return tables, pool


def make_batch(name: str, *, seq_lens: List[int], q_lens: Optional[List[int]] = None,
               num_q_heads: int, num_kv_heads: int, block_size: int, num_blocks: int,
               dtype: torch.dtype, seed: int, device="cpu",
               shared_groups: Optional[List[List[int]]] = None,
               shared_prefix_tokens: int = 0, head_dim: int = HEAD_DIM,
               prefill: Optional[bool] = None) -> PagedBatch:
    """Build a batch.  ``seq_lens`` are final context lengths (after this
    step's append); ``q_lens`` are the tokens appended this step per
    sequence (1 for decode, the chunk length for chunked prefill).

    Draw order is fixed: tables (numpy PCG64(seed)) -> K cache -> V cache ->
    q -> new K -> new V (torch generator seeded with ``seed``).  Every cache
    slot, used or not, holds an N(0,1) value; this step's tokens are then
    written by ``reshape_and_cache`` from ``k_new``/``v_new``.

    A decode batch (every q_len <= 1, unless ``prefill`` says otherwise) has one
    query row per sequence, also for empty sequences; a prefill batch has one
    row per chunk token and a ``query_start_loc``.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    B = len(seq_lens)
    if q_lens is None:
        q_lens = [1 if L > 0 else 0 for L in seq_lens]
    assert all(0 <= ql <= L for ql, L in zip(q_lens, seq_lens))
    tables, _ = _assign_tables(list(seq_lens), block_size, num_blocks, rng,
                               shared_groups, shared_prefix_tokens)
    # slot of every appended token: positions L-q_len .. L-1 of each sequence
    slots = []
    for s, (L, ql) in enumerate(zip(seq_lens, q_lens)):
        for pos in range(L - ql, L):
            slots.append(int(tables[s, pos // block_size]) * block_size + pos % block_size)
    T = len(slots)
    qsl = np.zeros(B + 1, dtype=np.int32)
    qsl[1:] = np.cumsum(q_lens)
    is_prefill = any(ql > 1 for ql in q_lens) if prefill is None else prefill

    gs_t = pl_t = None
    if shared_groups and all(g == list(range(g[0], g[0] + len(g))) for g in shared_groups):
        starts = sorted(g[0] for g in shared_groups)
        ends = {g[0]: g[0] + len(g) for g in shared_groups}
        if all(ends[a] <= b for a, b in zip(starts, starts[1:])):
            bounds = [x for a in starts for x in (a, ends[a])]
            # gaps between groups become groups with nothing shared
            gstarts, plens = [], []
            prev_end = None
            for i in range(0, len(bounds), 2):
                if gstarts and bounds[i] != prev_end:
                    gstarts.append(prev_end)
                    plens.append(0)
                gstarts.append(bounds[i])
                plens.append(shared_prefix_tokens)
                prev_end = bounds[i + 1]
            gstarts.append(prev_end)
            gs_t = torch.tensor(np.asarray(gstarts, dtype=np.int32), device=device)
            pl_t = torch.tensor(np.asarray(plens, dtype=np.int32), device=device)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    cshape = (num_blocks, block_size, num_kv_heads, head_dim)
    k_cache = _randn(cshape, dtype, gen, device)
    v_cache = _randn(cshape, dtype, gen, device)
    nq = int(qsl[-1]) if is_prefill else B
    q = _randn((nq, num_q_heads, head_dim), dtype, gen, device)
    k_new = _randn((T, num_kv_heads, head_dim), dtype, gen, device)
    v_new = _randn((T, num_kv_heads, head_dim), dtype, gen, device)
    return PagedBatch(
        name=name, dtype=dtype, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=block_size, num_blocks=num_blocks,
        scale=1.0 / math.sqrt(head_dim),
        seq_lens=torch.tensor(np.asarray(seq_lens, dtype=np.int32), device=device),
        block_tables=torch.from_numpy(tables).to(device),
        q=q, k_cache=k_cache, v_cache=v_cache, k_new=k_new, v_new=v_new,
        slot_mapping=torch.tensor(np.asarray(slots, dtype=np.int32), device=device),
        query_start_loc=torch.from_numpy(qsl).to(device) if is_prefill else None,
        shared_prefix_blocks=(shared_prefix_tokens // block_size) if shared_groups else 0,
        group_size=len(shared_groups[0]) if shared_groups else 1,
        group_starts=gs_t, prefix_lens=pl_t,
    )


# ---------------------------------------------------------------------------
# The named workloads.  Each returns a list of batches making up one step
# (decode-only workloads: one batch; the mixed workload: prefill + decode).
# ``scale`` < 1 shrinks lengths for oracle-sized parity runs while keeping the
# structure (ragged tails, several tiles per sequence, GQA shape).
# ---------------------------------------------------------------------------

def _pool_size(seq_lens, block_size, factor=1.25, minimum=0):
    demand = sum(_num_blocks_for(L, block_size) for L in seq_lens)
    return max(minimum, int(math.ceil(demand * factor)))


def tiny_mha(seed=1001, device="cpu"):
    """4 sequences, cached lengths U{1..200} plus one appended token, 8 q heads
    = 8 kv heads, fp16, block 16, a 64-block pool."""
    rng = np.random.Generator(np.random.PCG64(seed))
    lens = [int(x) + 1 for x in rng.integers(1, 201, size=4)]
    return [make_batch("tiny_mha_b4_fp16", seq_lens=lens, num_q_heads=8, num_kv_heads=8,
                       block_size=16, num_blocks=64, dtype=torch.float16,
                       seed=seed, device=device)]


def llama70b_uniform(seed=1002, device="cpu", scale=1.0):
    """16 sequences of 4096 tokens, 64 q / 8 kv heads, fp16, block 16; the
    4096-block pool is used exactly (tables are a permutation of it)."""
    L = max(16, int(4096 * scale))
    lens = [L] * 16
    nb = _pool_size(lens, 16, factor=1.0)
    return [make_batch("llama70b_gqa8_b16_l%d_fp16" % L, seq_lens=lens, num_q_heads=64,
                       num_kv_heads=8, block_size=16, num_blocks=nb, dtype=torch.float16,
                       seed=seed, device=device)]


def mixed_lengths(seed=1003, device="cpu", scale=1.0, batch=64):
    """64 sequences, lengths log-uniform on [50, 8000], 32 q / 8 kv heads,
    bf16, block 16, one token appended per sequence before decode."""
    rng = np.random.Generator(np.random.PCG64(seed))
    u = rng.uniform(math.log(50), math.log(8000), size=batch)
    lens = [max(1, int(round(math.exp(x) * scale))) for x in u]
    nb = _pool_size(lens, 16)
    return [make_batch("mixed_len_b%d_gqa4_bf16" % batch, seq_lens=lens, num_q_heads=32,
                       num_kv_heads=8, block_size=16, num_blocks=nb, dtype=torch.bfloat16,
                       seed=seed, device=device)]


def shared_prefix(block_size=16, seed=1004, device="cpu", scale=1.0, groups=8, n=8):
    """8 groups x 8 sequences; each group shares a 2048-token prefix through
    reference-counted blocks, plus a private suffix of U{1..512} tokens;
    32 q / 8 kv heads, fp16, block 16 or 32."""
    rng = np.random.Generator(np.random.PCG64(seed))
    prefix = max(block_size, int(2048 * scale) // block_size * block_size)
    suf_max = max(1, int(512 * scale))
    suffix = [int(x) for x in rng.integers(1, suf_max + 1, size=groups * n)]
    lens = [prefix + s for s in suffix]
    grp = [list(range(g * n, (g + 1) * n)) for g in range(groups)]
    demand = groups * (prefix // block_size) + sum(_num_blocks_for(s, block_size) for s in suffix)
    nb = int(math.ceil(demand * 1.25)) + 1
    return [make_batch("shared_prefix_%dx%d_bs%d_fp16" % (groups, n, block_size), seq_lens=lens,
                       num_q_heads=32, num_kv_heads=8, block_size=block_size, num_blocks=nb,
                       dtype=torch.float16, seed=seed, device=device, shared_groups=grp,
                       shared_prefix_tokens=prefix)]


def prefill_plus_decode(seed=1005, device="cpu", scale=1.0, n_prefill=4, n_decode=32):
    """4 sequences with a 512-token query chunk over a 7488-token paged
    prefix (8000 total) plus 32 decode sequences of 32768 tokens; 64 q / 8 kv
    heads, bf16, block 16.  Returns [prefill batch, decode batch]."""
    chunk = max(1, int(512 * scale))
    total = max(chunk, int(8000 * scale))
    dec_len = max(1, int(32768 * scale))
    p = make_batch("chunked_prefill_4x512_ctx8000_bf16", seq_lens=[total] * n_prefill,
                   q_lens=[chunk] * n_prefill, num_q_heads=64, num_kv_heads=8,
                   block_size=16, num_blocks=_pool_size([total] * n_prefill, 16),
                   dtype=torch.bfloat16, seed=seed, device=device)
    d = make_batch("long_decode_b32_l32768_bf16", seq_lens=[dec_len] * n_decode,
                   num_q_heads=64, num_kv_heads=8, block_size=16,
                   num_blocks=_pool_size([dec_len] * n_decode, 16),
                   dtype=torch.bfloat16, seed=seed + 100, device=device)
    return [p, d]


def varlen_step(seed=1006, device="cpu", scale=1.0, n_prefill=4, n_decode=32):
    """The chunked-prefill + long-decode step of ``prefill_plus_decode`` as ONE varlen
    batch over one cache: 4 sequences with a 512-token chunk over 8000-token contexts
    and 32 decode rows of 32768 tokens; 64 q / 8 kv heads, bf16, block 16."""
    chunk = max(2, int(512 * scale))
    total = max(chunk, int(8000 * scale))
    dec_len = max(1, int(32768 * scale))
    lens = [total] * n_prefill + [dec_len] * n_decode
    return [make_batch("varlen_4x512_ctx8000_plus_32x32768_bf16", seq_lens=lens,
                       q_lens=[chunk] * n_prefill + [1] * n_decode, num_q_heads=64,
                       num_kv_heads=8, block_size=16, num_blocks=_pool_size(lens, 16),
                       dtype=torch.bfloat16, seed=seed, device=device, prefill=True)]


def with_fp8_cache(batch: PagedBatch, seed: int = 77) -> PagedBatch:
    """The same batch (tables, lengths, q, new K/V) over an FP8 (e4m3) cache: every
    cache slot holds a seeded random e4m3 code of magnitude code 0x00..0x48 (values 0..4,
    subnormals included) with a random sign, and each kv-head has its own fp32 scales
    (K: 0.25 * (1 + h/Hkv), V: 0.5 * (1 + h/(2 Hkv))).  The step's new K/V stay in the
    batch's fp16/bf16 type: appending them quantises them."""
    rng = np.random.Generator(np.random.PCG64(seed))
    shape = tuple(batch.k_cache.shape)

    def codes():
        mag = rng.integers(0, 0x49, size=shape, dtype=np.int64)
        sign = rng.integers(0, 2, size=shape, dtype=np.int64) << 7
        return torch.from_numpy((mag | sign).astype(np.uint8)).to(batch.k_cache.device)

    kc, vc = codes(), codes()
    H = batch.num_kv_heads
    hs = np.arange(H, dtype=np.float64)
    ks = torch.tensor(0.25 * (1 + hs / H), dtype=torch.float32, device=batch.k_cache.device)
    vs = torch.tensor(0.5 * (1 + hs / (2 * H)), dtype=torch.float32, device=batch.k_cache.device)
    return dataclasses.replace(batch, name=batch.name + "_fp8kv", k_cache=kc, v_cache=vc,
                               k_scale=ks, v_scale=vs)


def mixed_lengths_fp8(seed=1003, device="cpu", scale=1.0, batch=64):
    """The mixed-length batch of ``mixed_lengths`` with an FP8 (e4m3) KV cache."""
    return [with_fp8_cache(mixed_lengths(seed=seed, device=device, scale=scale, batch=batch)[0])]


def llama70b_fp8(seed=1002, device="cpu", scale=1.0):
    """The LLaMA-70B-shaped batch of ``llama70b_uniform`` with an FP8 (e4m3) KV cache."""
    return [with_fp8_cache(llama70b_uniform(seed=seed, device=device, scale=scale)[0])]


WORKLOADS = {
    "tiny": tiny_mha,
    "llama70b": llama70b_uniform,
    "mixed": mixed_lengths,
    "shared16": lambda **kw: shared_prefix(block_size=16, **kw),
    "shared32": lambda **kw: shared_prefix(block_size=32, **kw),
    "prefill_decode": prefill_plus_decode,
    "varlen": varlen_step,
    "mixed_fp8": mixed_lengths_fp8,
    "llama70b_fp8": llama70b_fp8,
}


def private_copy(batch: PagedBatch) -> PagedBatch:
    """Same batch with every shared prefix block copied into a private
    physical block per sequence (for the sharing == private-copies check)."""
    tables = batch.block_tables.clone()
    B, M = tables.shape
    seen = {}
    extra = []
    nb = batch.num_blocks
    for s in range(B):
        for j in range(M):
            b = int(tables[s, j])
            if j < batch.shared_prefix_blocks:
                if b in seen:
                    extra.append(b)
                    tables[s, j] = nb + len(extra) - 1
                else:
                    seen[b] = s
    idx = torch.tensor(extra, dtype=torch.long, device=batch.k_cache.device)
    kc = torch.cat([batch.k_cache, batch.k_cache.index_select(0, idx)], 0) if extra else batch.k_cache.clone()
    vc = torch.cat([batch.v_cache, batch.v_cache.index_select(0, idx)], 0) if extra else batch.v_cache.clone()
    # slots of appended tokens are unchanged: they lie in private suffix blocks
    return dataclasses.replace(batch, block_tables=tables, k_cache=kc, v_cache=vc,
                               num_blocks=nb + len(extra), shared_prefix_blocks=0)


def permute_blocks(batch: PagedBatch, seed: int = 7) -> PagedBatch:
    """Same logical content with the physical blocks relabelled by a random
    permutation (cache rows moved, tables and slots rewritten to match)."""
    g = np.random.Generator(np.random.PCG64(seed))
    perm = g.permutation(batch.num_blocks)          # old id -> new id
    inv = np.argsort(perm)                          # new id -> old id
    dev = batch.k_cache.device
    kc = batch.k_cache.index_select(0, torch.from_numpy(inv).to(dev))
    vc = batch.v_cache.index_select(0, torch.from_numpy(inv).to(dev))
    pt = torch.from_numpy(perm.astype(np.int32)).to(dev)
    tables = pt[batch.block_tables.long()]
    bs = batch.block_size
    sm = batch.slot_mapping.long()
    slots = torch.where(sm >= 0, pt[(sm // bs).clamp(min=0)].long() * bs + sm % bs, sm).to(torch.int32)
    return dataclasses.replace(batch, k_cache=kc, v_cache=vc, block_tables=tables,
                               slot_mapping=slots)
