"""GPU parity for pa_chunked_prefill (tcgen05 kernel) through the C ABI against the
fp64 oracle: small and scaled workloads element by element, every GQA group, both
dtypes and block sizes, edge cases of the chunk layout, and sampled rows of the
full-size chunked-prefill workload."""
import numpy as np
import pytest
import torch

import oracle.paged_attention as opa
import paged_kv_cache_332_b200 as pa
import workloads
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _prefill_vs_oracle(batch_cpu, what=""):
    b = batch_cpu.to(DEV)
    P.gpu_append(b)
    out = P.gpu_prefill(b)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    ref = P.oracle_prefill(batch_cpu)
    return P.compare(out, ref, batch_cpu.dtype, what or batch_cpu.name)


def _batch(lens, qlens, G, dtype, bs=16, Hkv=2, seed=11, extra_blocks=8):
    nb = sum(-(-L // bs) for L in lens) + extra_blocks
    return workloads.make_batch("prefill_g%d" % G, seq_lens=lens, q_lens=qlens,
                                num_q_heads=Hkv * G, num_kv_heads=Hkv, block_size=bs,
                                num_blocks=nb, dtype=dtype, seed=seed, prefill=True)


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_prefill_every_group_and_dtype(G, dtype):
    # ragged chunks over ragged prefixes: tails inside a key tile, several key tiles,
    # a chunk that is the whole sequence, a one-token chunk
    lens = [300, 129, 77, 1]
    qlens = [45, 129, 1, 1]
    _prefill_vs_oracle(_batch(lens, qlens, G, dtype, seed=20 + G))


@pytest.mark.parametrize("bs", [16, 32])
def test_prefill_block_sizes_and_long_context(bs):
    lens = [700, 515]
    qlens = [256, 200]
    _prefill_vs_oracle(_batch(lens, qlens, 8, torch.bfloat16, bs=bs, Hkv=2, seed=5))


def test_prefill_chunk_workload_scaled():
    p, _ = workloads.prefill_plus_decode(scale=1 / 16, n_decode=1)
    _prefill_vs_oracle(p, "chunked prefill 1/16")


def test_prefill_chunk_workload_quarter():
    p, _ = workloads.prefill_plus_decode(scale=1 / 4, n_prefill=2, n_decode=1)
    _prefill_vs_oracle(p, "chunked prefill 1/4")


def test_prefill_empty_chunks_and_zero_rows():
    # sequences with no new queries in the middle of the batch
    lens = [50, 40, 90, 33]
    qlens = [10, 0, 90, 0]
    b = _batch(lens, qlens, 4, torch.float16, seed=3)
    st = _prefill_vs_oracle(b)
    assert st["n"] == 100 * b.num_q_heads * 128


def test_prefill_last_query_equals_decode():
    """The last query of a chunk sees every key, exactly like decode at that length."""
    lens = [333, 160]
    qlens = [64, 17]
    bc = _batch(lens, qlens, 4, torch.bfloat16, seed=8)
    b = bc.to(DEV)
    P.gpu_append(b)
    outp = P.gpu_prefill(b)
    last = (b.query_start_loc[1:] - 1).long()
    dec = workloads.PagedBatch(**{**b.__dict__, "q": b.q[last].contiguous(),
                                  "query_start_loc": None})
    outd = P.gpu_decode(dec)
    torch.cuda.synchronize()
    d = (outp[last].float() - outd.float()).abs().max().item()
    assert d <= P.TOL[bc.dtype], d


def test_prefill_bad_query_layout_flagged():
    bc = _batch([40, 40], [10, 10], 2, torch.float16, seed=1)
    bc.query_start_loc = torch.tensor([0, 10, 60], dtype=torch.int32)  # second chunk > L
    b = bc.to(DEV)
    out = torch.zeros((20, b.num_q_heads, 128), dtype=b.dtype, device=DEV)
    pa.pa_chunked_prefill(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.seq_lens,
                          b.query_start_loc, b.scale, 50, 40)
    assert pa.pa_get_device_error() & pa.PA_DEVERR["QUERY_LAYOUT"]


def test_prefill_full_size_sampled_rows():
    """Full chunked-prefill workload (4 x 512 queries over 8000 keys, 64 q / 8 kv
    heads, bf16); the oracle recomputes sampled (query, head) rows one by one."""
    p = workloads.prefill_plus_decode(device=DEV, n_decode=1)[0]
    bs = p.block_size
    seqs = [0, 3]
    sub = P.sub_batch(p, seqs)  # generator's cache, before the GPU append
    P.gpu_append(p)
    out = P.gpu_prefill(p)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    kc, vc = opa.to_f64(sub["k_cache"]), opa.to_f64(sub["v_cache"])
    qsl = p.query_start_loc.cpu().numpy()
    sm = p.slot_mapping.cpu().numpy()
    rows = [t for s in seqs for t in range(int(qsl[s]), int(qsl[s + 1]))]
    new_slots = np.array([sub["remap"][int(sm[t]) // bs] * bs + int(sm[t]) % bs for t in rows])
    opa.reshape_and_cache(opa.to_f64(p.k_new[rows]), opa.to_f64(p.v_new[rows]), kc, vc, new_slots)
    Hq, Hkv = p.num_q_heads, p.num_kv_heads
    rng = np.random.default_rng(0)
    got, want = [], []
    for si, s in enumerate(seqs):
        L = int(sub["seq_lens"][si])
        n = int(qsl[s + 1] - qsl[s])
        for g in range(Hkv):
            K = opa.gather_kv(kc, sub["block_tables"][si].numpy(), L, g)
            V = opa.gather_kv(vc, sub["block_tables"][si].numpy(), L, g)
            for i in sorted(set(rng.integers(0, n, size=6).tolist()) | {0, n - 1}):
                for hq in (g * (Hq // Hkv), g * (Hq // Hkv) + Hq // Hkv - 1):
                    vis = L - n + i + 1
                    want.append(opa.attend(opa.to_f64(p.q[int(qsl[s]) + i, hq]), K[:vis], V[:vis],
                                           p.scale))
                    got.append(out[int(qsl[s]) + i, hq])
    P.compare(torch.stack(got), np.stack(want), p.dtype, "chunked prefill full size, sampled")


def _prefill_with_workspace(b):
    ws = torch.empty(pa.pa_chunked_prefill_workspace_size(b.num_seqs, b.max_query_len,
                                                          b.num_q_heads, 128, b.max_seq_len),
                     dtype=torch.uint8, device=DEV)
    out = torch.empty_like(b.q)
    pa.pa_chunked_prefill(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.seq_lens,
                          b.query_start_loc, b.scale, b.max_query_len, b.max_seq_len, ws)
    return out, pa.pa_last_launch_count()


@pytest.mark.parametrize("lens,qlens", [
    ([300, 400, 250, 500], [160, 160, 160, 160]),   # 160 items: a 12-item tail wave on 148 SMs
    ([300, 40, 250, 500], [160, 10, 160, 33]),      # ragged chunks: split items with no rows
    ([700], [64]),                                  # 16 items: every item split
])
def test_prefill_wave_tail_split(lens, qlens):
    """With the optional workspace the last wave's items run as two halves of their keys
    and are merged; the result matches the oracle and the unsplit call."""
    bc = _batch(lens, qlens, 8, torch.bfloat16, Hkv=8, seed=31)
    b = bc.to(DEV)
    P.gpu_append(b)
    plain = P.gpu_prefill(b)
    split, launches = _prefill_with_workspace(b)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    qblocks = -(-max(qlens) // 32)
    items = len(lens) * 8 * qblocks
    tail = items % sms
    assert launches == (2 if 0 < 2 * tail <= sms else 1)
    ref = P.oracle_prefill(bc)
    P.compare(split, ref, bc.dtype, "prefill with the wave tail split")
    assert (split.float() - plain.float()).abs().max().item() <= P.TOL[bc.dtype]
