"""GPU parity for device-side block-table maintenance through the C ABI: after every
step, pa_block_allocate / pa_block_free / pa_block_share must leave the ring, its
{head, count}, the block tables, the owned counts and the reference counts exactly as
the oracle's FIFO pool does, and write the same slot mapping and grant flags —
including steps where the pool runs dry (a sequence preempted, later ones still
served), table rows too short, prefill-sized appends, the 4096-sequence limit, prompt
blocks shared by a group and released together, and a full loop of allocate → scatter
→ decode."""
import numpy as np
import pytest
import torch

import oracle.block_pool as obp
import oracle.paged_attention as opa
import paged_kv_cache_332_b200 as pa
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


class _Pair:
    """The same pool and tables on both sides."""

    def __init__(self, n_blocks, B, max_blocks, bs, refs=False):
        self.bs = bs
        self.pool = obp.BlockPool(n_blocks)
        self.tables = np.zeros((B, max_blocks), dtype=np.int64)
        self.owned = np.zeros(B, dtype=np.int64)
        self.lens = np.zeros(B, dtype=np.int64)
        self.ring = torch.full((n_blocks,), -7, dtype=torch.int32, device=DEV)
        self.state = torch.full((2,), -7, dtype=torch.int32, device=DEV)
        self.refs = torch.full((n_blocks,), -7, dtype=torch.int32, device=DEV) if refs else None
        pa.pa_block_pool_init(self.ring, self.state, self.refs)
        self.d_tables = torch.zeros((B, max_blocks), dtype=torch.int32, device=DEV)
        self.d_owned = torch.zeros(B, dtype=torch.int32, device=DEV)

    def alloc(self, q_lens):
        q = np.asarray(q_lens, dtype=np.int64)
        d_lens = torch.tensor(self.lens, dtype=torch.int32, device=DEV)
        d_q = torch.tensor(q, dtype=torch.int32, device=DEV)
        d_slots = torch.full((max(int(q.sum()), 1),), -9, dtype=torch.int32, device=DEV)
        d_granted = torch.full((len(q),), -9, dtype=torch.int32, device=DEV)
        pa.pa_block_allocate(self.ring, self.state, self.d_tables, self.d_owned, d_lens, d_q,
                             self.bs, d_slots, d_granted, block_refs=self.refs)
        slots, granted = obp.allocate_step(self.pool, self.tables, self.owned, self.lens, q,
                                           self.bs)
        self.lens += np.where(granted, q, 0)
        got_slots = d_slots[:int(q.sum())].cpu().numpy()
        assert np.array_equal(got_slots, slots), "slot mapping"
        assert np.array_equal(d_granted.cpu().numpy(), granted.astype(np.int32)), "granted"
        self.check()
        return slots, granted

    def free(self, seqs):
        fin = np.zeros(len(self.owned), dtype=bool)
        fin[list(seqs)] = True
        pa.pa_block_free(self.ring, self.state, self.d_tables, self.d_owned,
                         torch.tensor(fin.astype(np.int32), device=DEV), block_refs=self.refs)
        obp.free_sequences(self.pool, self.tables, self.owned, fin)
        self.lens[fin] = 0
        self.check()

    def share(self, pairs, expect_error=False):
        src, dst, k = (np.asarray([p[i] for p in pairs], dtype=np.int64) for i in range(3))
        dev = [torch.tensor(x, dtype=torch.int32, device=DEV) for x in (src, dst, k)]
        pa.pa_block_share(self.refs, self.d_tables, self.d_owned, *dev)
        done = obp.share_blocks(self.pool, self.tables, self.owned, src, dst, k)
        self.lens[dst[done]] = k[done] * self.bs
        self.check(expect_error=expect_error)
        return done

    def check(self, expect_error=False):
        torch.cuda.synchronize()
        err = pa.pa_get_device_error()
        assert err == (pa.PA_DEVERR["POOL"] if expect_error else 0), err
        if self.refs is not None:
            assert np.array_equal(self.refs.cpu().numpy(), self.pool.refs), "refs"
        st = self.state.cpu().numpy()
        assert (int(st[0]), int(st[1])) == (self.pool.head, self.pool.count), "head/count"
        assert np.array_equal(self.ring.cpu().numpy(), self.pool.ring), "ring"
        assert np.array_equal(self.d_owned.cpu().numpy(), self.owned), "owned"
        assert np.array_equal(self.d_tables.cpu().numpy(), self.tables), "tables"


def _run(seed, B, steps, n_blocks, bs, max_blocks, q_choices, free_every=4, n_free=2):
    rng = np.random.default_rng(seed)
    pair = _Pair(n_blocks, B, max_blocks, bs)
    n_preempted = 0
    for t in range(steps):
        if t % free_every == free_every - 1:
            pair.free(sorted(set(rng.integers(0, B, n_free).tolist())))
        else:
            _, granted = pair.alloc(rng.choice(q_choices, size=B))
            n_preempted += int((~granted).sum())
    return pair, n_preempted


def test_shared_prompt_blocks_match_oracle():
    # parallel sampling: the first sequence of each group of four prefills a prompt, the
    # other three take its whole blocks, every member decodes, and members finish at
    # different steps (whole groups together at the end)
    rng = np.random.default_rng(21)
    B, G = 16, 4
    pair = _Pair(300, B, 40, 16, refs=True)
    prompt = [0] * B
    for g in range(B // G):
        prompt[g * G] = int(rng.integers(20, 120))
    pair.alloc(prompt)
    pairs = [(g * G, g * G + m, int(pair.owned[g * G]) - (1 if prompt[g * G] % 16 else 0))
             for g in range(B // G) for m in range(1, G)]
    assert pair.share(pairs).all()
    for t in range(12):
        pair.alloc([1] * B)
        if t == 5:
            pair.free([1, 6, 11])
        if t == 8:
            pair.free([0, 4, 9, 14])
    pair.free(range(B))  # the rest, shared blocks returning once each
    assert pair.pool.count == 300 and (pair.pool.refs == 0).all()


@pytest.mark.parametrize("seed", [31, 32, 33])
def test_random_sharing_matches_oracle(seed):
    rng = np.random.default_rng(seed)
    B = 24
    pair = _Pair(160, B, 24, 16, refs=True)
    for t in range(30):
        if t % 5 == 4:
            pair.free(sorted(set(rng.integers(0, B, 4).tolist())))
        elif t % 5 == 2:
            empty = [s for s in range(B) if pair.owned[s] == 0]
            holders = [s for s in range(B) if pair.owned[s] > 0]
            rng.shuffle(empty)
            pairs = []
            for d in empty[:4]:
                if not holders:
                    break
                src = int(rng.choice([h for h in holders if h not in empty[:4]] or [d]))
                if src == d:
                    continue
                pairs.append((src, d, int(rng.integers(0, int(pair.owned[src]) + 1))))
            if pairs:
                pair.share(pairs)
        else:
            pair.alloc(rng.choice([0, 1, 1, 17, 40], size=B))


def test_invalid_share_is_flagged_and_skipped():
    pair = _Pair(40, 4, 8, 16, refs=True)
    pair.alloc([20, 5, 0, 0])
    done = pair.share([(0, 1, 1), (0, 2, 3), (0, 3, 2)], expect_error=True)
    # dst 1 owns a block, and 3 blocks are more than seq 0 owns: only the last pair applies
    assert done.tolist() == [False, False, True]


def test_release_below_zero_is_flagged():
    # a count cleared behind the pool's back: the block is released once more than it was
    # held; the pool flags it and keeps the block out of the ring
    pair = _Pair(8, 2, 4, 16, refs=True)
    pair.alloc([20, 0])
    blk = int(pair.tables[0, 1])
    pair.refs[blk] = 0
    pa.pa_block_free(pair.ring, pair.state, pair.d_tables, pair.d_owned,
                     torch.tensor([1, 0], dtype=torch.int32, device=DEV), block_refs=pair.refs)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == pa.PA_DEVERR["POOL"]
    head, count = pair.state.cpu().tolist()
    free = [int(pair.ring[(head + i) % 8]) for i in range(count)]
    assert blk not in free and int(pair.tables[0, 0]) in free and count == 7


def test_init_fills_ring_in_order():
    pair = _Pair(1000, 1, 4, 16)
    pair.check()
    assert pair.state.cpu().tolist() == [0, 1000]


@pytest.mark.parametrize("bs", [16, 32])
def test_decode_steps_match_oracle(bs):
    # one token per sequence per step with some prefill chunks; the pool is ample
    _run(1, B=37, steps=24, n_blocks=4000, bs=bs, max_blocks=64, q_choices=[1, 1, 1, 0, 17, 40])


def test_pool_runs_dry_and_preempts_in_index_order():
    pair, n_pre = _run(2, B=40, steps=40, n_blocks=90, bs=16, max_blocks=64,
                       q_choices=[1, 1, 16, 40, 100], free_every=5, n_free=6)
    assert n_pre > 0  # the scenario did exercise preemption
    assert pair.pool.count < 90


def test_table_row_too_short():
    pair = _Pair(500, 4, 3, 16)  # rows hold 3 blocks = 48 tokens
    _, granted = pair.alloc([48, 49, 0, 10])
    assert granted.tolist() == [True, False, True, True]
    _, granted = pair.alloc([1, 40, 0, 38])
    assert granted.tolist() == [False, True, True, True]


def test_ring_wraps_around():
    # many allocate/free rounds move head past the end of the ring several times
    _run(3, B=8, steps=60, n_blocks=20, bs=16, max_blocks=16, q_choices=[1, 16, 33],
         free_every=3, n_free=3)


def test_max_sequences_prefill_then_decode():
    rng = np.random.default_rng(4)
    B = 4096
    pair = _Pair(40000, B, 32, 16)
    pair.alloc(rng.integers(0, 120, B))        # prompts: a prefill step for every sequence
    for _ in range(3):
        pair.alloc(np.ones(B, dtype=np.int64))  # three decode steps
    pair.free(range(0, B, 3))
    pair.alloc(rng.integers(0, 40, B))


def test_empty_pool_all_preempted_but_zero_length_appends():
    pair = _Pair(2, 3, 8, 16)
    pair.alloc([32, 0, 0])                   # takes both blocks
    _, granted = pair.alloc([1, 0, 5])
    assert granted.tolist() == [False, True, False]


def test_allocate_scatter_decode_loop():
    """The device pool feeds pa_reshape_and_cache and pa_decode for several steps; the
    oracle runs the same loop with its own pool, scatter and attention."""
    rng = np.random.default_rng(11)
    B, Hq, Hkv, D, bs, N = 6, 16, 4, 128, 16, 30
    dtype = torch.float16
    pair = _Pair(N, B, 32, bs)
    kc = torch.zeros((N, bs, Hkv, D), dtype=dtype, device=DEV)
    vc = torch.zeros_like(kc)
    kc64 = np.zeros((N, bs, Hkv, D), dtype=np.float64)
    vc64 = np.zeros_like(kc64)
    steps = [[0, 1, 17, 47, 100, 250]] + [[1] * B] * 6  # 29 blocks, then 1 more
    for q_lens in steps:
        T = sum(q_lens)
        k = torch.tensor(rng.normal(0, 1, (T, Hkv, D)), dtype=dtype)
        v = torch.tensor(rng.normal(0, 1, (T, Hkv, D)), dtype=dtype)
        d_lens = torch.tensor(pair.lens, dtype=torch.int32, device=DEV)
        d_q = torch.tensor(q_lens, dtype=torch.int32, device=DEV)
        d_slots = torch.empty(T, dtype=torch.int32, device=DEV)
        d_granted = torch.empty(B, dtype=torch.int32, device=DEV)
        pa.pa_block_allocate(pair.ring, pair.state, pair.d_tables, pair.d_owned, d_lens, d_q, bs,
                             d_slots, d_granted)
        pa.pa_reshape_and_cache(k.to(DEV), v.to(DEV), kc, vc, d_slots)
        new_lens = d_lens + d_q * d_granted
        q = torch.tensor(rng.normal(0, 1, (B, Hq, D)), dtype=dtype)
        out = torch.empty((B, Hq, D), dtype=dtype, device=DEV)
        maxlen = int(new_lens.max())
        ws = torch.empty(max(pa.pa_decode_workspace_size(B, Hq, D, maxlen), 1), dtype=torch.uint8,
                         device=DEV)
        pa.pa_decode(out, q.to(DEV), kc, vc, pair.d_tables, new_lens, D ** -0.5, maxlen, 0, ws)
        # oracle loop
        slots, granted = obp.allocate_step(pair.pool, pair.tables, pair.owned, pair.lens,
                                           np.asarray(q_lens), bs)
        pair.lens += np.where(granted, q_lens, 0)
        opa.reshape_and_cache(opa.to_f64(k), opa.to_f64(v), kc64, vc64, slots)
        ref = opa.paged_decode(opa.to_f64(q), kc64, vc64, pair.tables, pair.lens, D ** -0.5)
        torch.cuda.synchronize()
        assert pa.pa_get_device_error() == 0
        assert np.array_equal(d_slots.cpu().numpy(), slots)
        assert np.array_equal(new_lens.cpu().numpy(), pair.lens)
        P.compare(out, ref, dtype, "pool-driven decode step")
    pair.check()
    assert granted.tolist() == [True, True, True, False, True, True]  # seq 3 waits
