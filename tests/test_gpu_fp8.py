"""GPU parity for the FP8 (e4m3) KV cache through the C ABI: pa_reshape_and_cache_fp8
must write the oracle's codes bit for bit (quantisation with per-kv-head scales), and
pa_decode_fp8 must match the oracle's attention over the dequantised cache within the
output type's tolerance — every GQA group and output type, explicit partitions, empty
and one-token sequences, and sampled rows of the full-size mixed batch."""
import numpy as np
import pytest
import torch

import oracle.paged_attention as opa
import paged_kv_cache_332_b200 as pa
import workloads
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gpu_append_fp8(b):
    pa.pa_reshape_and_cache_fp8(b.k_new, b.v_new, b.k_cache, b.v_cache, b.slot_mapping,
                                b.k_scale, b.v_scale)


def _gpu_decode_fp8(b, partition_size=0):
    B, Hq, D = b.q.shape
    ws = torch.empty(pa.pa_decode_workspace_size(B, Hq, D, b.max_seq_len, partition_size),
                     dtype=torch.uint8, device=DEV)
    out = torch.empty_like(b.q)
    pa.pa_decode_fp8(out, b.q, b.k_cache, b.v_cache, b.k_scale, b.v_scale, b.block_tables,
                     b.seq_lens, b.scale, b.max_seq_len, partition_size, ws)
    return out


def _oracle_append_fp8(bc):
    kc, vc = bc.k_cache.numpy().copy(), bc.v_cache.numpy().copy()
    opa.reshape_and_cache_fp8(opa.to_f64(bc.k_new).astype(np.float32),
                              opa.to_f64(bc.v_new).astype(np.float32), kc, vc,
                              bc.slot_mapping.numpy(), bc.k_scale.numpy(), bc.v_scale.numpy())
    return kc, vc


def _oracle_decode_fp8(bc, kc=None, vc=None):
    if kc is None:
        kc, vc = _oracle_append_fp8(bc)
    return opa.paged_decode(opa.to_f64(bc.q), opa.dequantize_cache(kc, bc.k_scale.numpy()),
                            opa.dequantize_cache(vc, bc.v_scale.numpy()),
                            bc.block_tables.numpy(), bc.seq_lens.numpy(), bc.scale)


def _fp8_vs_oracle(bc, partition_size=0, what=""):
    b = bc.to(DEV)
    _gpu_append_fp8(b)
    out = _gpu_decode_fp8(b, partition_size)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    kc, vc = _oracle_append_fp8(bc)
    assert np.array_equal(b.k_cache.cpu().numpy(), kc)
    assert np.array_equal(b.v_cache.cpu().numpy(), vc)
    return P.compare(out, _oracle_decode_fp8(bc, kc, vc), bc.dtype, what or bc.name)


@pytest.mark.parametrize("name,maker", [
    ("tiny", lambda: workloads.with_fp8_cache(workloads.tiny_mha()[0])),
    ("mixed", lambda: workloads.mixed_lengths_fp8(scale=1 / 4)[0]),
    ("llama70b", lambda: workloads.llama70b_fp8(scale=1 / 8)[0]),
    ("shared32", lambda: workloads.with_fp8_cache(workloads.shared_prefix(block_size=32,
                                                                           scale=1 / 8)[0])),
])
def test_fp8_append_bit_exact_and_decode(name, maker):
    _fp8_vs_oracle(maker())


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_fp8_every_group_and_dtype(G, dtype):
    lens = [1, 15, 16, 17, 33, 250, 513]
    bc = workloads.make_batch("fp8_g%d" % G, seq_lens=lens, num_q_heads=4 * G, num_kv_heads=4,
                              block_size=16, num_blocks=200, dtype=dtype, seed=90 + G)
    _fp8_vs_oracle(workloads.with_fp8_cache(bc, seed=G))


@pytest.mark.parametrize("P_", [16, 512, 0])
def test_fp8_split_k_partition_invariance(P_):
    bc = workloads.mixed_lengths_fp8(scale=1 / 8)[0]
    _fp8_vs_oracle(bc, P_, "mixed fp8, partition %d" % P_)


def test_fp8_seq_len_zero_and_one():
    lens = [0, 1, 0, 2, 17]
    bc = workloads.make_batch("fp8_edge", seq_lens=lens, num_q_heads=16, num_kv_heads=2,
                              block_size=16, num_blocks=16, dtype=torch.float16, seed=4)
    bc = workloads.with_fp8_cache(bc)
    st = _fp8_vs_oracle(bc)
    b = bc.to(DEV)
    _gpu_append_fp8(b)
    out = _gpu_decode_fp8(b)
    torch.cuda.synchronize()
    assert float(out[0].abs().max()) == 0.0 and float(out[2].abs().max()) == 0.0
    del st


def test_fp8_saturation_in_append():
    # new K/V far past the e4m3 range saturate to +-448 * scale, bit-exactly
    bc = workloads.with_fp8_cache(workloads.tiny_mha()[0])
    bc.k_new = (bc.k_new.float() * 1e4).to(bc.dtype)
    _fp8_vs_oracle(bc, 0, "tiny fp8, saturating append")


def test_fp8_full_size_mixed_sampled():
    """Full mixed-length batch on an FP8 cache; the oracle recomputes sampled sequences."""
    b = workloads.mixed_lengths_fp8(device=DEV)[0]
    seqs = [0, 7, 31, 63]
    sub = P.sub_batch(b, seqs)  # generator's cache codes, before the GPU append
    _gpu_append_fp8(b)
    out = _gpu_decode_fp8(b)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    kc, vc = sub["k_cache"].numpy().copy(), sub["v_cache"].numpy().copy()
    bs = b.block_size
    sm = b.slot_mapping.cpu().numpy()
    new_slots = np.array([sub["remap"][int(sm[s]) // bs] * bs + int(sm[s]) % bs for s in seqs])
    opa.reshape_and_cache_fp8(opa.to_f64(b.k_new[seqs]).astype(np.float32),
                              opa.to_f64(b.v_new[seqs]).astype(np.float32), kc, vc, new_slots,
                              b.k_scale.cpu().numpy(), b.v_scale.cpu().numpy())
    ref = opa.paged_decode(opa.to_f64(b.q[seqs]),
                           opa.dequantize_cache(kc, b.k_scale.cpu().numpy()),
                           opa.dequantize_cache(vc, b.v_scale.cpu().numpy()),
                           sub["block_tables"].numpy(), sub["seq_lens"].numpy(), b.scale)
    P.compare(out[seqs], ref, b.dtype, "mixed fp8 full size, sampled")
