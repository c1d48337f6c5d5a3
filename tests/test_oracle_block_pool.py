"""Pins for the block-pool oracle (no GPU): the page's FIFO pool and scheduler rule
("生产级推理引擎的内存管理与调度"), checked against a plain deque model written from the
same description, hand-worked cases, and invariants (no block owned twice, every block
either free or owned), with planted mistakes that must fail a pin."""
import collections

import numpy as np
import pytest

import oracle.block_pool as obp

MUT_ORIG = {"allocate_step": obp.allocate_step, "free_sequences": obp.free_sequences,
            "blocks_needed": obp.blocks_needed}


def _deque_run(n_blocks, bs, ops):
    """The same scenario with a Python deque as the free list (the page's VecDeque)."""
    free = collections.deque(range(n_blocks))
    tables, owned, lens = {}, {}, {}
    out = []
    for op in ops:
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
                    slots += [tables[s][p // bs] * bs + p % bs for p in range(lens[s], lens[s] + q)]
                    lens[s] += q
                else:
                    slots += [-1] * q
            out.append(slots)
        else:
            for s in op[1]:
                for b in tables.get(s, []):
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


def _scenario(seed, B=6, steps=12, n_blocks=24, bs=16):
    rng = np.random.default_rng(seed)
    ops = []
    for t in range(steps):
        if t % 4 == 3:
            ops.append(("free", sorted(set(rng.integers(0, B, 2).tolist()))))
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


def check_blocks_needed():
    assert [obp.blocks_needed(n, 16) for n in (0, 1, 15, 16, 17, 32, 33)] == [0, 1, 1, 1, 2, 2, 3]


CHECKS = [check_matches_deque_model, check_worked_case, check_invariants, check_blocks_needed]


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


MUTATIONS = {
    "allocate_from_back": ("allocate_step", _alloc_lifo),
    "partial_allocation": ("allocate_step", _alloc_partial),
    "free_reversed": ("free_sequences", _free_reversed),
    "blocks_floor": ("blocks_needed", _needed_floor),
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
