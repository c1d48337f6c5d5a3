"""Plain oracle of block-table maintenance (test infrastructure only: only tests/,
the package entry's smoke check and bench.py's baseline may use it; the library never
imports it).

Source — page "大模型推理内存优化从 KV Cache 分页到连续批处理的工程实践", section
"生产级推理引擎的内存管理与调度": a pool of physical blocks keeps its free block ids in a
FIFO queue (a new pool holds 0..N-1 in order; allocating pops the front, freeing pushes
the id on the back); the scheduler gives a sequence a new block when the blocks it needs
for its tokens (integer ceiling of tokens / block size) exceed the blocks it owns, and
when no block is free that sequence is preempted for this step while later sequences
are still considered; a finished sequence returns all its blocks to the pool.
Page "KV Cache管理优化：大模型推理显存瓶颈突破", section 4.1: a block may be shared by
several sequences (a common prompt) and carries a reference count; releasing a
reference frees the block only when the count reaches zero.

Readings where the page is silent:
- a step may append several tokens to a sequence (a prefill chunk); the sequence gets
  all the blocks it needs or none (preempted: nothing allocated, no slots);
- sequences are served in index order; a sequence's blocks are freed in table order,
  sequences in index order;
- the free queue is a ring of N entries with a head (next id to allocate) and a count;
- a token at position p of sequence s lands in slot table[s][p // bs] * bs + p % bs;
- sharing gives a sequence that owns no block the first k blocks of another sequence's
  table (one more reference each); when finished sequences release their blocks, in
  the order above, a block returns to the pool at the release that drops its count to
  zero.
"""
from __future__ import annotations

import numpy as np


def blocks_needed(num_tokens, block_size):
    """Integer ceiling of tokens / block size (the scheduler's block count)."""
    return (num_tokens + block_size - 1) // block_size


class BlockPool:
    """The FIFO free-block queue as a ring: ``ring[(head + i) % N]`` for i < count are
    the free ids, the front first."""

    def __init__(self, num_blocks):
        self.n = int(num_blocks)
        self.ring = np.arange(self.n, dtype=np.int64)
        self.head = 0
        self.count = self.n
        self.refs = np.zeros(self.n, dtype=np.int64)  # references held on each block

    def available(self):
        return self.count

    def allocate(self):
        """Pop the front id (None when empty)."""
        if self.count == 0:
            return None
        b = int(self.ring[self.head])
        self.head = (self.head + 1) % self.n
        self.count -= 1
        self.refs[b] = 1
        return b

    def free(self, block_id):
        """Push ``block_id`` on the back."""
        assert self.count < self.n
        self.ring[(self.head + self.count) % self.n] = block_id
        self.count += 1


def allocate_step(pool, block_tables, owned, seq_lens, q_lens, block_size):
    """One step of appends: sequence s (index order) holds ``seq_lens[s]`` tokens in
    ``owned[s]`` blocks and appends ``q_lens[s]`` tokens.  If it needs more blocks than
    it owns it pops them from the pool, all or none.  Updates ``block_tables`` and
    ``owned`` in place; returns (slot_mapping int64 [sum q_lens], granted bool [B]).
    A preempted sequence's slots are -1 and its table is unchanged."""
    B = len(seq_lens)
    slots, granted = [], np.zeros(B, dtype=bool)
    for s in range(B):
        L, q = int(seq_lens[s]), int(q_lens[s])
        extra = max(0, blocks_needed(L + q, block_size) - int(owned[s]))
        ok = extra <= pool.available() and int(owned[s]) + extra <= block_tables.shape[1]
        if ok:
            for _ in range(extra):
                block_tables[s, owned[s]] = pool.allocate()
                owned[s] += 1
        granted[s] = ok
        for p in range(L, L + q):
            slots.append(int(block_tables[s, p // block_size]) * block_size + p % block_size
                         if ok else -1)
    return np.asarray(slots, dtype=np.int64), granted


def share_blocks(pool, block_tables, owned, src, dst, num_shared):
    """For each pair i (in order): sequence dst[i], which owns no block, takes the first
    num_shared[i] blocks of sequence src[i]'s table, each gaining one reference.  A pair
    whose dst owns blocks, whose count is negative or above what src owns, or whose src
    is dst, is skipped.  Returns a bool array: the pairs applied."""
    done = np.zeros(len(src), dtype=bool)
    for i in range(len(src)):
        a, b, k = int(src[i]), int(dst[i]), int(num_shared[i])
        if a == b or owned[b] != 0 or k < 0 or k > owned[a]:
            continue
        for j in range(k):
            blk = int(block_tables[a, j])
            block_tables[b, j] = blk
            pool.refs[blk] += 1
        owned[b] = k
        done[i] = True
    return done


def free_sequences(pool, block_tables, owned, finished):
    """Release every block of each finished sequence (sequences in index order, blocks in
    table order): a block goes back to the pool when its last reference is released.
    Sets the owned counts of the finished sequences to 0."""
    for s in range(len(owned)):
        if finished[s]:
            for j in range(int(owned[s])):
                b = int(block_tables[s, j])
                assert pool.refs[b] > 0, "block %d released more often than it was held" % b
                pool.refs[b] -= 1
                if pool.refs[b] == 0:
                    pool.free(b)
            owned[s] = 0
