"""Pins for the block-pool oracle (no GPU): the page's FIFO pool and scheduler rule
("生产级推理引擎的内存管理与调度") and the reference-counted shared blocks of "KV Cache管理
优化：大模型推理显存瓶颈突破" 4.1, checked against a plain deque model written from the
same descriptions, hand-worked cases, and invariants (a block held by k tables carries k
references, every block either free or held), with planted mistakes that must fail a
pin."""
import collections

import numpy as np
import pytest

import oracle.block_pool as obp

MUT_ORIG = {"allocate_step": obp.allocate_step, "free_sequences": obp.free_sequences,
            "blocks_needed": obp.blocks_needed, "share_blocks": obp.share_blocks}


def _deque_run(n_blocks, bs, ops):
    """The same scenario with a Python deque as the free list (the page's VecDeque)."""
    free = collections.deque(range(n_blocks))
    tables, owned, lens = {}, {}, {}
    holders = collections.Counter()  # block -> tables holding it
    out = []
    for op in ops:
        if op[0] == "share":  # (src, dst, k): dst, holding nothing, takes src's first k
            a, b, k = op[1]
            if a != b and not tables.get(b) and 0 <= k <= len(tables.get(a, [])):
                tables[b] = list(tables[a][:k])
                lens[b] = k * bs
                holders.update(tables[b])
            continue
        if op[0] == "alloc":
            q_lens = op[1]
            slots = []
            for s, q in enumerate(q_lens):
                tables.setdefault(s, [])
                lens.setdefault(s, 0)
                need = -(-(lens[s] + q) // bs) - len(tables[s])
                need = max(0, need)
                if need <= len(free):
                    for _ in range(need):
                        tables[s].append(free.popleft())
                        holders[tables[s][-1]] += 1
                    slots += [tables[s][p // bs] * bs + p % bs for p in range(lens[s], lens[s] + q)]
                    lens[s] += q
                else:
                    slots += [-1] * q
            out.append(slots)
        else:
            for s in op[1]:
                for b in tables.get(s, []):
                    holders[b] -= 1
                    if holders[b] == 0:
                        free.append(b)
                tables[s] = []
                lens[s] = 0
    return out, list(free)


def _oracle_run(n_blocks, bs, ops, B, max_blocks):
    pool = obp.BlockPool(n_blocks)
    tables = np.zeros((B, max_blocks), dtype=np.int64)
    owned = np.zeros(B, dtype=np.int64)
    lens = np.zeros(B, dtype=np.int64)
    out = []
    for op in ops:
        if op[0] == "share":
            a, b, k = op[1]
            done = obp.share_blocks(pool, tables, owned, [a], [b], [k])
            if done[0]:
                lens[b] = k * bs
            continue
        if op[0] == "alloc":
            q = np.asarray(op[1])
            slots, granted = obp.allocate_step(pool, tables, owned, lens, q, bs)
            lens += np.where(granted, q, 0)
            out.append(slots.tolist())
        else:
            fin = np.zeros(B, dtype=bool)
            fin[list(op[1])] = True
            obp.free_sequences(pool, tables, owned, fin)
            lens[fin] = 0
    free = [int(pool.ring[(pool.head + i) % pool.n]) for i in range(pool.count)]
    return out, free, tables, owned


def _scenario(seed, B=6, steps=12, n_blocks=24, bs=16, share=False):
    rng = np.random.default_rng(seed)
    ops = []
    for t in range(steps):
        if t % 4 == 3:
            ops.append(("free", sorted(set(rng.integers(0, B, 2).tolist()))))
        elif share and t % 4 == 1:
            a, b = (int(x) for x in rng.choice(B, 2, replace=False))
            ops.append(("share", (a, b, int(rng.integers(0, 3)))))
        else:
            ops.append(("alloc", rng.choice([0, 1, 1, 1, 17, 40], size=B).tolist()))
    return ops


def check_matches_deque_model():
    for seed in range(20):
        ops = _scenario(seed)
        want_slots, want_free = _deque_run(24, 16, ops)
        got_slots, got_free, _, _ = _oracle_run(24, 16, ops, 6, 64)
        assert got_slots == want_slots, seed
        assert got_free == want_free, seed


def check_sharing_matches_deque_model():
    for seed in range(40):
        ops = _scenario(seed, B=6, steps=24, n_blocks=30, share=True)
        want_slots, want_free = _deque_run(30, 16, ops)
        got_slots, got_free, _, _ = _oracle_run(30, 16, ops, 6, 64)
        assert got_slots == want_slots, seed
        assert got_free == want_free, seed


def check_shared_worked_case():
    # seq 0 holds blocks 0, 1 (20 tokens); seqs 1 and 2 take both; freeing 0 and 1 returns
    # nothing, freeing 2 returns both in table order, after the never-used 2, 3
    ops = [("alloc", [20, 0, 0]), ("share", (0, 1, 2)), ("share", (0, 2, 2))]
    _, free, tables, owned = _oracle_run(4, 16, ops, 3, 4)
    assert free == [2, 3] and list(owned) == [2, 2, 2]
    assert list(tables[1, :2]) == [0, 1] and list(tables[2, :2]) == [0, 1]
    _, free, _, _ = _oracle_run(4, 16, ops + [("free", [0, 1])], 3, 4)
    assert free == [2, 3]
    _, free, _, owned = _oracle_run(4, 16, ops + [("free", [0, 1]), ("free", [2])], 3, 4)
    assert free == [2, 3, 0, 1] and list(owned) == [0, 0, 0]
    # released together: the block returns at the last release (sequence 2's), in order
    _, free, _, _ = _oracle_run(4, 16, [("alloc", [20, 0, 0]), ("share", (0, 2, 1)),
                                        ("free", [0, 2])], 3, 4)
    assert free == [2, 3, 1, 0]
    # the new holder appends into its own blocks: 32 shared tokens + 1 takes block 2
    got, free, tables, _ = _oracle_run(4, 16, [("alloc", [32, 0]), ("share", (0, 1, 2)),
                                               ("alloc", [0, 1])], 2, 4)
    assert list(tables[1, :3]) == [0, 1, 2] and got[-1] == [2 * 16] and free == [3]
    # a holder of blocks cannot take shared ones; nor can it take more than src owns
    _, _, _, owned = _oracle_run(4, 16, [("alloc", [16, 16]), ("share", (0, 1, 1)),
                                         ("share", (1, 0, 2))], 2, 4)
    assert list(owned) == [1, 1]


def check_worked_case():
    # bs 16; seq 0 appends 16 tokens (1 block), seq 1 appends 17 (2 blocks) -> ids 0 | 1, 2
    got, free, tables, owned = _oracle_run(4, 16, [("alloc", [16, 17])], 2, 8)
    assert got[0][:16] == list(range(0, 16)) and got[0][16:] == list(range(16, 48))[:17]
    assert tables[0, 0] == 0 and list(tables[1, :2]) == [1, 2] and free == [3]
    # one more token each: seq 0 needs a 2nd block (id 3), seq 1 fits in block 2
    got2, free2, tables2, _ = _oracle_run(4, 16, [("alloc", [16, 17]), ("alloc", [1, 1])], 2, 8)
    assert got2[1] == [3 * 16 + 0, 2 * 16 + 1] and free2 == []
    # pool empty: a sequence needing a block is preempted, the other still appends
    got3, _, _, _ = _oracle_run(4, 16, [("alloc", [16, 17]), ("alloc", [1, 1]),
                                        ("alloc", [16, 1])], 2, 8)
    assert got3[2][:16] == [-1] * 16 and got3[2][16] == 2 * 16 + 2
    # freeing pushes on the back, in table order: the front is reused first
    _, free4, _, _ = _oracle_run(4, 16, [("alloc", [16, 17]), ("free", [1])], 2, 8)
    assert free4 == [3, 1, 2]


def check_invariants():
    for seed in range(20):
        ops = _scenario(seed, B=8, steps=20, n_blocks=40)
        _, free, tables, owned = _oracle_run(40, 16, ops, 8, 64)
        held = [int(tables[s, j]) for s in range(8) for j in range(int(owned[s]))]
        assert len(set(held)) == len(held)                 # no block owned twice
        assert sorted(held + free) == list(range(40))      # every block free or owned


def check_reference_invariants():
    for seed in range(20):
        ops = _scenario(seed, B=8, steps=28, n_blocks=40, share=True)
        pool_box = {}
        orig = obp.BlockPool

        class Spy(orig):
            def __init__(self, n):
                super().__init__(n)
                pool_box["pool"] = self
        obp.BlockPool = Spy
        try:
            _, free, tables, owned = _oracle_run(40, 16, ops, 8, 64)
        finally:
            obp.BlockPool = orig
        refs = pool_box["pool"].refs
        held = collections.Counter(int(tables[s, j]) for s in range(8)
                                   for j in range(int(owned[s])))
        assert len(set(free)) == len(free)                  # no block queued twice
        assert not (set(free) & set(held))                  # a held block is never free
        assert sorted(list(held) + free) == list(range(40))  # every block free or held
        for b in range(40):                                 # k holders, k references
            assert refs[b] == held.get(b, 0), (seed, b)


def check_blocks_needed():
    assert [obp.blocks_needed(n, 16) for n in (0, 1, 15, 16, 17, 32, 33)] == [0, 1, 1, 1, 2, 2, 3]


CHECKS = [check_matches_deque_model, check_sharing_matches_deque_model, check_worked_case,
          check_shared_worked_case, check_invariants, check_reference_invariants,
          check_blocks_needed]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_block_pool_pin(check):
    check()


def _alloc_lifo(pool, block_tables, owned, seq_lens, q_lens, block_size):
    orig_alloc = pool.allocate

    def pop_back():
        if pool.count == 0:
            return None
        pool.count -= 1
        return int(pool.ring[(pool.head + pool.count) % pool.n])
    pool.allocate = pop_back
    try:
        return MUT_ORIG["allocate_step"](pool, block_tables, owned, seq_lens, q_lens, block_size)
    finally:
        pool.allocate = orig_alloc


def _alloc_partial(pool, block_tables, owned, seq_lens, q_lens, block_size):
    # gives a sequence whatever blocks remain instead of all or none
    B = len(seq_lens)
    slots, granted = [], np.ones(B, dtype=bool)
    for s in range(B):
        L, q = int(seq_lens[s]), int(q_lens[s])
        extra = max(0, obp.blocks_needed(L + q, block_size) - int(owned[s]))
        for _ in range(min(extra, pool.available())):
            block_tables[s, owned[s]] = pool.allocate()
            owned[s] += 1
        for p in range(L, L + q):
            slots.append(int(block_tables[s, p // block_size]) * block_size + p % block_size)
    return np.asarray(slots, dtype=np.int64), granted


def _free_reversed(pool, block_tables, owned, finished):
    for s in range(len(owned)):
        if finished[s]:
            for j in reversed(range(int(owned[s]))):
                pool.free(int(block_tables[s, j]))
            owned[s] = 0


def _needed_floor(num_tokens, block_size):
    return num_tokens // block_size


def _free_ignoring_refs(pool, block_tables, owned, finished):
    # returns every released block, shared or not
    for s in range(len(owned)):
        if finished[s]:
            for j in range(int(owned[s])):
                b = int(block_tables[s, j])
                pool.refs[b] = max(0, pool.refs[b] - 1)
                pool.free(b)
            owned[s] = 0


def _share_without_reference(pool, block_tables, owned, src, dst, num_shared):
    done = np.zeros(len(src), dtype=bool)
    for i in range(len(src)):
        a, b, k = int(src[i]), int(dst[i]), int(num_shared[i])
        if a == b or owned[b] != 0 or k < 0 or k > owned[a]:
            continue
        block_tables[b, :k] = block_tables[a, :k]
        owned[b] = k
        done[i] = True
    return done


MUTATIONS = {
    "allocate_from_back": ("allocate_step", _alloc_lifo),
    "partial_allocation": ("allocate_step", _alloc_partial),
    "free_reversed": ("free_sequences", _free_reversed),
    "blocks_floor": ("blocks_needed", _needed_floor),
    "free_ignoring_references": ("free_sequences", _free_ignoring_refs),
    "share_without_reference": ("share_blocks", _share_without_reference),
}


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_block_pool_mutation_is_caught(mutation, monkeypatch):
    name, fn = MUTATIONS[mutation]
    monkeypatch.setattr(obp, name, fn)
    caught = []
    for check in CHECKS:
        try:
            check()
        except Exception:
            caught.append(check.__name__)
    assert caught, "planted mistake %s passed every pin" % mutation
