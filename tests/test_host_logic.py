"""Host-side logic with no GPU: the seeded workloads' sharing and varlen structure, the
bench's algorithmic-byte counts (checked against an independent count of the cache
slots a step actually reads), and how the bench routes each batch to a library call."""
import numpy as np
import pytest
import torch

import bench
import workloads


def _slots_read(b):
    """Distinct (physical block, offset) slots a decode step reads: every position
    below each sequence's length, through its table."""
    bt = b.block_tables.cpu().numpy()
    seen = set()
    for s, L in enumerate(b.seq_lens.cpu().numpy()):
        for p in range(int(L)):
            seen.add((int(bt[s, p // b.block_size]), p % b.block_size))
    return seen


@pytest.mark.parametrize("bs", [16, 32])
def test_shared_prompt_groups_and_tables(bs):
    b = workloads.shared_prefix(block_size=bs, scale=1 / 8)[0]
    assert b.group_starts.tolist() == list(range(0, 65, 8))
    assert b.prefix_lens.tolist() == [256] * 8
    bt = b.block_tables.numpy()
    npre = 256 // bs
    for g in range(8):
        rows = bt[8 * g:8 * g + 8, :npre]
        assert (rows == rows[0]).all()                 # the members share the prefix blocks
    owned = [set(bt[s, npre:-(-int(L) // bs)].tolist()) for s, L in enumerate(b.seq_lens.numpy())]
    for i in range(64):
        for j in range(i + 1, 64):
            assert not owned[i] & owned[j]             # the rest is private


def test_groups_with_gaps_between_them():
    b = workloads.make_batch("gaps", seq_lens=[40, 60, 70, 80, 90, 100, 50], num_q_heads=8,
                             num_kv_heads=2, block_size=16, num_blocks=64, dtype=torch.float16,
                             seed=1, shared_groups=[[1, 2], [4, 5]], shared_prefix_tokens=32)
    assert b.group_starts.tolist() == [1, 3, 4, 6]
    assert b.prefix_lens.tolist() == [32, 0, 32]


def test_unique_bytes_of_a_shared_step_match_the_slots_read():
    b = workloads.shared_prefix(block_size=16, scale=1 / 8)[0]
    row = 2 * b.num_kv_heads * b.head_dim * b.k_cache.element_size()  # K and V of one slot
    e = b.q.element_size()
    B = b.num_seqs
    rest = 2 * B * b.num_q_heads * b.head_dim * e + \
        B * int(np.ceil(int(b.seq_lens.max()) / b.block_size)) * 4 + 4 * B
    unique = len(_slots_read(b)) * row + rest
    arrays = 4 * (b.group_starts.numel() + b.prefix_lens.numel())
    assert bench.decode_algorithmic_bytes(b, shared=True) == unique + arrays
    every = int(b.seq_lens.sum()) * row + rest
    assert bench.decode_algorithmic_bytes(b) == every
    assert every > 2 * unique


def test_varlen_step_structure():
    b = workloads.varlen_step(scale=1 / 16)[0]
    ql = (b.query_start_loc[1:] - b.query_start_loc[:-1]).tolist()
    assert ql == [32] * 4 + [1] * 32
    assert b.q.shape[0] == sum(ql) and b.slot_mapping.numel() == sum(ql)


def test_bench_routes_each_batch_to_its_call():
    import paged_kv_cache_332_b200 as pa
    shared = workloads.shared_prefix(block_size=16, scale=1 / 8)[0]
    mixed = workloads.mixed_lengths(scale=1 / 8)[0]
    fp8 = workloads.mixed_lengths_fp8(scale=1 / 8)[0]
    varlen = workloads.varlen_step(scale=1 / 16)[0]
    pre, dec = workloads.prefill_plus_decode(scale=1 / 16)
    st = bench.Step([shared, mixed, fp8, varlen, pre, dec], pa, None)
    assert st.shared[id(shared)] and not st.fused[id(shared)]
    assert st.fused[id(mixed)] and not st.shared[id(mixed)]
    assert not st.fused[id(fp8)] and not st.shared[id(fp8)]
    assert st.varlen[id(varlen)] and st.chunk_seqs[id(varlen)] == 4
    assert not st.varlen[id(pre)]
    assert st.group_bounds[id(shared)] == (8, 256)
    # every batch got a workspace of the size its call asks for
    assert st.ws[id(shared)].numel() == pa.pa_decode_shared_prefix_workspace_size(
        64, 32, 8, 128, shared.max_seq_len)
    assert st.ws[id(varlen)].numel() == pa.pa_attention_varlen_workspace_size(
        36, 32, 64, 128, varlen.max_seq_len)


def test_cpu_baseline_covers_decode_rows_and_chunks():
    import types
    args = types.SimpleNamespace(cpu_budget=0.2)
    r = bench.cpu_baseline(workloads.tiny_mha(), args)
    assert r["kind"] == "oracle" and r["cores"] == 1 and r["value"] > 0
    assert "4 of 4 sequences" in r["sample"]
    pre, dec = workloads.prefill_plus_decode(scale=1 / 64)
    r = bench.cpu_baseline([pre, dec], args, budget_s=60)
    # everything fits the budget: all 36 sequences and every (query row, key) pair
    lens = pre.seq_lens.numpy()
    n = int(pre.query_start_loc[1] - pre.query_start_loc[0])
    pairs = int(sum(n * L - n * (n - 1) // 2 for L in lens)) + int(dec.seq_lens.sum())
    assert "36 of 36 sequences" in r["sample"] and "(%d of %d" % (pairs, pairs) in r["sample"]


def test_bindings_check_array_lengths_before_any_call():
    import paged_kv_cache_332_b200 as pa
    b = workloads.shared_prefix(block_size=16, scale=1 / 8)[0]
    with pytest.raises(ValueError):
        pa.pa_decode_shared_prefix(b.q, b.q, b.k_cache, b.v_cache, b.block_tables, b.seq_lens,
                                   b.group_starts[:-1], b.prefix_lens, b.scale, 300, 8, 256)
    with pytest.raises(ValueError):
        pa.pa_decode_shared_prefix(b.q, b.q, b.k_cache, b.v_cache, b.block_tables, b.seq_lens[:5],
                                   b.group_starts, b.prefix_lens, b.scale, 300, 8, 256)
    v = workloads.varlen_step(scale=1 / 16)[0]
    with pytest.raises(ValueError):
        pa.pa_attention_varlen(v.q, v.q, v.k_cache, v.v_cache, v.block_tables, v.seq_lens,
                               v.query_start_loc[:-1], v.scale, 32, 2048)
    with pytest.raises(ValueError):
        pa.pa_attention_varlen(v.q[:5], v.q, v.k_cache, v.v_cache, v.block_tables, v.seq_lens,
                               v.query_start_loc, v.scale, 32, 2048)


def test_input_recipes_match_their_descriptions():
    m = workloads.mixed_lengths()[0]
    lens = m.seq_lens.numpy()
    assert len(lens) == 64 and lens.min() >= 50 and lens.max() <= 8000
    assert (m.num_q_heads, m.num_kv_heads, m.block_size, m.dtype) == (32, 8, 16, torch.bfloat16)
    # log-uniform: about half of the lengths below the geometric mean sqrt(50 * 8000) = 632
    assert 20 <= int((lens < 632).sum()) <= 44
    # every slot of the step's appended token is that sequence's position L-1
    bt = m.block_tables.numpy()
    sm = m.slot_mapping.numpy()
    assert all(sm[s] == bt[s, (L - 1) // 16] * 16 + (L - 1) % 16 for s, L in enumerate(lens))
    ll = workloads.llama70b_uniform()[0]
    assert ll.seq_lens.tolist() == [4096] * 16 and ll.num_blocks == 4096
    assert sorted(ll.block_tables.numpy().ravel().tolist()) == list(range(4096))  # the pool exactly
    assert (ll.num_q_heads, ll.num_kv_heads, ll.dtype) == (64, 8, torch.float16)
    sp = workloads.shared_prefix()[0]
    suffix = sp.seq_lens.numpy() - 2048
    assert suffix.min() >= 1 and suffix.max() <= 512
    pre, dec = workloads.prefill_plus_decode()
    assert pre.seq_lens.tolist() == [8000] * 4 and pre.max_query_len == 512
    assert dec.seq_lens.tolist() == [32768] * 32 and dec.num_q_heads == 64
