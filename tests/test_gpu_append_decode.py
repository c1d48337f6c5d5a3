"""GPU parity for pa_decode_append: the step's new token written into its cache slot
inside the decode launch.  Through the C ABI it must leave both caches bit-for-bit as
pa_reshape_and_cache does, return exactly what pa_decode returns after that append, and
match the fp64 oracle (append, then attention over the whole cache); edge cases: empty
sequences, a bad last table entry, a sequence longer than its table."""
import pytest
import torch

import paged_kv_cache_332_b200 as pa
import workloads
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _per_seq_new(b):
    """k_new / v_new indexed by sequence ([B, Hkv, D]); a sequence with no new token
    (seq_len 0) gets a row of zeros that must never be written."""
    kn = torch.zeros((b.num_seqs,) + tuple(b.k_new.shape[1:]), dtype=b.dtype, device=b.q.device)
    vn = torch.zeros_like(kn)
    has = (b.seq_lens > 0).nonzero().flatten().long()
    kn[has] = b.k_new
    vn[has] = b.v_new
    return kn, vn


def _fused(b, partition_size=0):
    kn, vn = _per_seq_new(b)
    B, Hq, D = b.q.shape
    ws = torch.empty(pa.pa_decode_workspace_size(B, Hq, D, b.max_seq_len, partition_size),
                     dtype=torch.uint8, device=DEV)
    out = torch.empty_like(b.q)
    pa.pa_decode_append(out, b.q, kn, vn, b.k_cache, b.v_cache, b.block_tables, b.seq_lens,
                        b.scale, b.max_seq_len, partition_size, ws)
    return out


def _check_against_unfused(bc, partition_size=0):
    fused, unfused = bc.to(DEV), bc.to(DEV)
    out_f = _fused(fused, partition_size)
    P.gpu_append(unfused)
    out_u = P.gpu_decode(unfused, partition_size)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    assert torch.equal(fused.k_cache, unfused.k_cache)
    assert torch.equal(fused.v_cache, unfused.v_cache)
    assert torch.equal(out_f, out_u)
    P.compare(out_f, P.oracle_decode(bc), bc.dtype, bc.name + " (append + decode)")


WORKLOADS = {
    "tiny": lambda: workloads.tiny_mha()[0],
    "mixed": lambda: workloads.mixed_lengths(scale=1 / 4)[0],
    "llama70b": lambda: workloads.llama70b_uniform(scale=1 / 8)[0],
    "shared16": lambda: workloads.shared_prefix(block_size=16, scale=1 / 8)[0],
    "shared32": lambda: workloads.shared_prefix(block_size=32, scale=1 / 8)[0],
    "long_g8": lambda: workloads.prefill_plus_decode(scale=1 / 32, n_decode=8)[1],
}


@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_append_decode_equals_reshape_then_decode(name):
    _check_against_unfused(WORKLOADS[name]())


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_append_decode_every_group_and_dtype(G, dtype):
    lens = [1, 15, 16, 17, 33, 250, 513]
    bc = workloads.make_batch("append_g%d" % G, seq_lens=lens, num_q_heads=4 * G,
                              num_kv_heads=4, block_size=16, num_blocks=200, dtype=dtype,
                              seed=70 + G)
    _check_against_unfused(bc)


@pytest.mark.parametrize("P_", [16, 512])
def test_append_decode_with_explicit_partitions(P_):
    # the new token's tile may sit in a short last segment of a split sequence
    _check_against_unfused(workloads.mixed_lengths(scale=1 / 8)[0], P_)


def test_append_decode_empty_sequences_write_nothing():
    lens = [0, 5, 0, 40, 1]
    bc = workloads.make_batch("append_edge", seq_lens=lens, num_q_heads=8, num_kv_heads=2,
                              block_size=16, num_blocks=16, dtype=torch.float16, seed=5)
    _check_against_unfused(bc)
    b = bc.to(DEV)
    out = _fused(b)
    torch.cuda.synchronize()
    assert float(out[0].abs().max()) == 0.0 and float(out[2].abs().max()) == 0.0


def test_append_decode_bad_last_block_flagged_nothing_written():
    bc = workloads.tiny_mha()[0]
    b = bc.to(DEV)
    s = 2
    L = int(bc.seq_lens[s])
    b.block_tables[s, (L - 1) // b.block_size] = b.num_blocks + 7  # out of range
    kc0, vc0 = b.k_cache.clone(), b.v_cache.clone()
    _fused(b)
    assert pa.pa_get_device_error() & pa.PA_DEVERR["BLOCK_RANGE"]
    # the other sequences' tokens were appended, this one's was not (and nothing else moved)
    sm = bc.slot_mapping.long()
    bs = bc.block_size
    for i in range(bc.num_seqs):
        blk, row = int(sm[i]) // bs, int(sm[i]) % bs
        if i == s:
            assert torch.equal(b.k_cache[blk, row], kc0[blk, row])
        else:
            assert torch.equal(b.k_cache[blk, row], bc.k_new[i].to(DEV))
            assert torch.equal(b.v_cache[blk, row], bc.v_new[i].to(DEV))
            kc0[blk, row] = b.k_cache[blk, row]
            vc0[blk, row] = b.v_cache[blk, row]
    assert torch.equal(b.k_cache, kc0) and torch.equal(b.v_cache, vc0)


def test_append_decode_sequence_past_its_table_flagged():
    bc = workloads.tiny_mha()[0]
    b = bc.to(DEV)
    max_blocks = b.block_tables.shape[1]
    b.seq_lens[0] = max_blocks * b.block_size + 5  # past the table: no slot to write
    kc0 = b.k_cache.clone()
    kn, vn = _per_seq_new(b)
    B, Hq, D = b.q.shape
    msl = max_blocks * b.block_size + 5
    ws = torch.empty(pa.pa_decode_workspace_size(B, Hq, D, msl, 0), dtype=torch.uint8, device=DEV)
    out = torch.empty_like(b.q)
    kn[0].fill_(7.0)  # a value that must not reach the cache
    pa.pa_decode_append(out, b.q, kn, vn, b.k_cache, b.v_cache, b.block_tables, b.seq_lens,
                        b.scale, msl, 0, ws)
    assert pa.pa_get_device_error() & pa.PA_DEVERR["SEQ_TOO_LONG"]
    assert not bool((b.k_cache == 7.0).all(dim=-1).any())
    # the other sequences appended as usual
    sm = bc.slot_mapping.long()
    for i in range(1, bc.num_seqs):
        blk, row = int(sm[i]) // bc.block_size, int(sm[i]) % bc.block_size
        assert torch.equal(b.k_cache[blk, row], kn[i])
    del kc0
