"""GPU parity: pa_reshape_and_cache and pa_decode through the C ABI against
the fp64 oracle, on the seeded workloads (oracle-sized copies that keep the
structure, and the full sizes on sampled sequences), plus edge cases and
invariances."""
import numpy as np
import pytest
import torch

import oracle.paged_attention as opa
import paged_kv_cache_332_b200 as pa
import workloads
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _decode_vs_oracle(batch_cpu, partition_size=0, what=""):
    b = batch_cpu.to(DEV)
    P.gpu_append(b)
    out = P.gpu_decode(b, partition_size=partition_size)
    assert pa.pa_get_device_error() == 0
    ref = P.oracle_decode(batch_cpu)
    return P.compare(out, ref, batch_cpu.dtype, what or batch_cpu.name)


# ------------------------------------------------------------------ reshape_and_cache

@pytest.mark.parametrize("name", ["tiny", "mixed", "shared32", "prefill_decode"])
def test_reshape_and_cache_bit_exact_whole_cache(name):
    kw = {} if name == "tiny" else {"scale": 1 / 16}
    for bc in workloads.WORKLOADS[name](**kw):
        # sentinel everywhere, so any stray write shows up
        bc.k_cache.view(torch.int16).fill_(0x2ABC)
        bc.v_cache.view(torch.int16).fill_(0x3123)
        sm = bc.slot_mapping.clone()
        if sm.numel() > 2:
            sm[1] = -1  # a padding token must be skipped
        bc.slot_mapping = sm
        b = bc.to(DEV)
        P.gpu_append(b)
        assert pa.pa_get_device_error() == 0
        kc = bc.k_cache.view(torch.int16).numpy().copy()
        vc = bc.v_cache.view(torch.int16).numpy().copy()
        opa.reshape_and_cache(bc.k_new.view(torch.int16).numpy(), bc.v_new.view(torch.int16).numpy(),
                              kc, vc, sm.numpy())
        assert np.array_equal(b.k_cache.view(torch.int16).cpu().numpy(), kc)
        assert np.array_equal(b.v_cache.view(torch.int16).cpu().numpy(), vc)


def test_reshape_and_cache_bad_slot_flagged_and_skipped():
    bc = workloads.tiny_mha()[0]
    bc.k_cache.view(torch.int16).fill_(0x1111)
    bc.v_cache.view(torch.int16).fill_(0x2222)
    nslots = bc.num_blocks * bc.block_size
    bc.slot_mapping = torch.tensor([3, nslots, nslots + 77, 5], dtype=torch.int32)
    b = bc.to(DEV)
    P.gpu_append(b)
    assert pa.pa_get_device_error() & pa.PA_DEVERR["SLOT_RANGE"]
    assert pa.pa_get_device_error() == 0  # reading clears the flag
    kc = bc.k_cache.view(torch.int16).numpy().copy()
    vc = bc.v_cache.view(torch.int16).numpy().copy()
    opa.reshape_and_cache(bc.k_new.view(torch.int16).numpy(), bc.v_new.view(torch.int16).numpy(),
                          kc, vc, np.array([3, -1, -1, 5]))
    assert np.array_equal(b.k_cache.view(torch.int16).cpu().numpy(), kc)
    assert np.array_equal(b.v_cache.view(torch.int16).cpu().numpy(), vc)


def test_reshape_and_cache_large_chunk():
    # 2048-token prefill chunk (4 x 512), as in the chunked-prefill workload
    bc = workloads.prefill_plus_decode(scale=0.25)[0]
    bc.k_cache.view(torch.int16).fill_(0x0F0F)
    bc.v_cache.view(torch.int16).fill_(0x0E0E)
    b = bc.to(DEV)
    P.gpu_append(b)
    kc = bc.k_cache.view(torch.int16).numpy().copy()
    vc = bc.v_cache.view(torch.int16).numpy().copy()
    opa.reshape_and_cache(bc.k_new.view(torch.int16).numpy(), bc.v_new.view(torch.int16).numpy(),
                          kc, vc, bc.slot_mapping.numpy())
    assert np.array_equal(b.k_cache.view(torch.int16).cpu().numpy(), kc)
    assert np.array_equal(b.v_cache.view(torch.int16).cpu().numpy(), vc)


# ------------------------------------------------------------------ decode parity

def test_decode_tiny_mha():
    _decode_vs_oracle(workloads.tiny_mha()[0])


@pytest.mark.parametrize("scale", [1 / 16, 1 / 4])
def test_decode_llama70b_shape(scale):
    _decode_vs_oracle(workloads.llama70b_uniform(scale=scale)[0])


@pytest.mark.parametrize("scale", [1 / 8, 1 / 3])
def test_decode_mixed_lengths(scale):
    _decode_vs_oracle(workloads.mixed_lengths(scale=scale)[0])


@pytest.mark.parametrize("bs", [16, 32])
def test_decode_shared_prefix(bs):
    _decode_vs_oracle(workloads.shared_prefix(block_size=bs, scale=1 / 8)[0])


def test_decode_long_sequences_bf16_g8():
    _decode_vs_oracle(workloads.prefill_plus_decode(scale=1 / 32, n_decode=8)[1])


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_decode_every_group_and_dtype(G, dtype):
    lens = [1, 2, 15, 16, 17, 31, 33, 100, 511, 512, 513, 700]
    b = workloads.make_batch("g%d" % G, seq_lens=lens, num_q_heads=4 * G, num_kv_heads=4,
                             block_size=16, num_blocks=200, dtype=dtype, seed=77 + G)
    _decode_vs_oracle(b, partition_size=256)


@pytest.mark.parametrize("P_", [16, 64, 512, 0, 2048])
def test_split_k_partition_invariance(P_):
    """The result must not depend on the split-K partition beyond rounding."""
    bc = workloads.mixed_lengths(scale=1 / 4)[0]
    st = _decode_vs_oracle(bc, partition_size=P_, what="mixed P=%d" % P_)
    assert st["n_bad"] == 0


def test_decode_seq_len_zero_and_one():
    lens = [0, 1, 5, 0, 1]
    bc = workloads.make_batch("edge", seq_lens=lens, num_q_heads=8, num_kv_heads=2, block_size=16,
                              num_blocks=16, dtype=torch.float16, seed=5)
    b = bc.to(DEV)
    P.gpu_append(b)
    out = P.gpu_decode(b).cpu()
    assert torch.all(out[0] == 0) and torch.all(out[3] == 0)
    # seq_len 1: the only value row, exactly (softmax weight 1)
    for s in (1, 4):
        slot = int(bc.slot_mapping[[i for i in range(len(lens)) if lens[i] > 0].index(s)])
        vrow = bc.v_new[[i for i in range(len(lens)) if lens[i] > 0].index(s)]
        for h in range(8):
            assert torch.equal(out[s, h], vrow[h // 4])
    _decode_vs_oracle(bc)


def test_decode_full_table_and_bs32_tail():
    # sequences that exactly fill their table, and ragged bs=32 tails
    lens = [64, 63, 33, 32, 31, 1]
    bc = workloads.make_batch("full", seq_lens=lens, num_q_heads=32, num_kv_heads=8,
                              block_size=32, num_blocks=20, dtype=torch.bfloat16, seed=9)
    assert bc.block_tables.shape[1] == 2
    _decode_vs_oracle(bc, partition_size=32)


def test_placement_and_sharing_invariance_bitwise():
    """Relabelling physical blocks, or giving each sequence private copies of
    its shared prefix, leaves the GPU result bit-for-bit unchanged."""
    bc = workloads.shared_prefix(block_size=16, scale=1 / 8)[0]
    outs = []
    for v in (bc, workloads.permute_blocks(bc), workloads.private_copy(bc)):
        b = v.to(DEV)
        P.gpu_append(b)
        outs.append(P.gpu_decode(b).cpu())
    assert torch.equal(outs[0], outs[1])
    assert torch.equal(outs[0], outs[2])


def test_decode_bad_table_entry_flagged():
    bc = workloads.tiny_mha()[0]
    # the other sequences are unaffected: oracle on the intact tables
    ref = P.oracle_decode(bc, opa.to_f64(bc.k_cache), opa.to_f64(bc.v_cache))
    bt = bc.block_tables.clone()
    bt[2, 0] = bc.num_blocks + 5
    bc.block_tables = bt
    b = bc.to(DEV)
    out = P.gpu_decode(b)
    err = pa.pa_get_device_error()
    assert err & pa.PA_DEVERR["BLOCK_RANGE"]
    keep = [0, 1, 3]
    P.compare(out.cpu()[keep], ref[keep], bc.dtype, "unaffected sequences")


def test_decode_seq_longer_than_bound_flagged():
    bc = workloads.tiny_mha()[0]
    b = bc.to(DEV)
    P.gpu_decode(b, max_seq_len=int(bc.seq_lens.max()) - 1)
    assert pa.pa_get_device_error() & pa.PA_DEVERR["SEQ_TOO_LONG"]


# ------------------------------------------------------------------ full sizes, sampled

def _sampled_full_size(batch_dev, seqs, what):
    """Full-size workload on the GPU; the oracle recomputes ``seqs`` from the
    generator's cache (copied before the GPU append) and its own scatter."""
    sub = P.sub_batch(batch_dev, seqs)      # before the append: generator output only
    bs = batch_dev.block_size
    P.gpu_append(batch_dev)
    out = P.gpu_decode(batch_dev)
    assert pa.pa_get_device_error() == 0
    kc, vc = opa.to_f64(sub["k_cache"]), opa.to_f64(sub["v_cache"])
    sm = batch_dev.slot_mapping.cpu().numpy()
    rows = list(seqs)  # decode: token t belongs to sequence t
    new_slots = np.array([sub["remap"][int(sm[r]) // bs] * bs + int(sm[r]) % bs for r in rows])
    opa.reshape_and_cache(opa.to_f64(batch_dev.k_new[rows]), opa.to_f64(batch_dev.v_new[rows]),
                          kc, vc, new_slots)
    ref = opa.paged_decode(opa.to_f64(batch_dev.q[rows]), kc, vc, sub["block_tables"].numpy(),
                           sub["seq_lens"].numpy(), batch_dev.scale)
    return P.compare(out[rows], ref, batch_dev.dtype, what)


def test_full_size_mixed_lengths_sampled():
    b = workloads.mixed_lengths(device=DEV)[0]
    lens = b.seq_lens.cpu().numpy()
    order = np.argsort(lens)
    seqs = sorted({int(order[0]), int(order[-1]), int(order[len(order) // 2]), 7, 33})
    _sampled_full_size(b, seqs, "mixed full size")


def test_full_size_llama70b_sampled():
    b = workloads.llama70b_uniform(device=DEV)[0]
    _sampled_full_size(b, [0, 9], "llama70b full size")


def test_full_size_shared_prefix_sampled():
    for bs in (16, 32):
        b = workloads.shared_prefix(block_size=bs, device=DEV)[0]
        _sampled_full_size(b, [0, 1, 12, 63], "shared prefix bs%d full size" % bs)


def test_full_size_long_decode_sampled():
    b = workloads.prefill_plus_decode(device=DEV)[1]
    _sampled_full_size(b, [3], "long decode 32768 full size")
