"""GPU parity for the mixed continuous-batching call (pa_attention_varlen) through the C
ABI: a varlen batch of decode rows and prefill chunks ([P1] "工程边界与架构取舍", chunked
prefill mixed with decode steps) must match the oracle's chunked prefill row by row;
a batch of decode rows only must equal pa_decode bit for bit, a batch of chunks only
the oracle and pa_chunked_prefill (to the rounding of its wave-tail merge); sequences without rows are left alone and a decode row outside q is
flagged, not read."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle.paged_attention as opa
import paged_kv_cache_332_b200 as pa
import workloads
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _varlen(b, rows=None, qsl=None, max_chunk_seqs=-1):
    B, Hq, D = b.num_seqs, b.num_q_heads, b.head_dim
    mq = b.max_query_len
    ws = torch.empty(pa.pa_attention_varlen_workspace_size(B, mq, Hq, D, b.max_seq_len),
                     dtype=torch.uint8, device=DEV)
    q = b.q if rows is None else b.q[:rows]
    out = torch.full_like(q, float("nan"))
    pa.pa_attention_varlen(out, q, b.k_cache, b.v_cache, b.block_tables, b.seq_lens,
                           b.query_start_loc if qsl is None else qsl, b.scale, mq, b.max_seq_len,
                           ws, max_chunk_seqs=max_chunk_seqs)
    return out


def _batch(name, lens, q_lens, G, dtype, bs=16, Hkv=4, seed=0):
    return workloads.make_batch(name, seq_lens=lens, q_lens=q_lens, num_q_heads=G * Hkv,
                                num_kv_heads=Hkv, block_size=bs,
                                num_blocks=sum(-(-L // bs) for L in lens) + 8, dtype=dtype,
                                seed=seed, prefill=True)


@pytest.mark.parametrize("G,dtype,bs", [(4, torch.bfloat16, 16), (8, torch.float16, 16),
                                        (1, torch.float16, 32), (2, torch.bfloat16, 32)])
def test_mixed_step_matches_oracle(G, dtype, bs):
    # decode rows (q_len 1), chunks of several sizes, a sequence with no rows (q_len 0),
    # a chunk that is the whole prompt
    lens = [300, 1, 40, 700, 17, 129, 2000, 64, 90, 513]
    q_lens = [1, 1, 40, 1, 5, 64, 1, 0, 33, 1]
    bc = _batch("varlen_g%d" % G, lens, q_lens, G, dtype, bs=bs, seed=20 + G)
    b = bc.to(DEV)
    P.gpu_append(b)
    out = _varlen(b)
    launches = pa.pa_last_launch_count()
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    assert launches >= 3  # decode + its merge + prefill
    P.compare(out, P.oracle_prefill(bc), bc.dtype, "mixed varlen step G=%d" % G)


def test_chunk_bound_exact_and_too_small():
    lens = [300, 40, 700, 129, 2000, 90]
    q_lens = [1, 40, 1, 64, 1, 33]  # three chunks
    bc = _batch("varlen_bound", lens, q_lens, 4, torch.float16, seed=31)
    b = bc.to(DEV)
    P.gpu_append(b)
    ref = P.oracle_prefill(bc)
    out = _varlen(b, max_chunk_seqs=3)  # the exact count: a grid over the three chunks
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    P.compare(out, ref, bc.dtype, "varlen, chunk bound exact")
    out = _varlen(b, max_chunk_seqs=2)  # too small: flagged, the third chunk not computed
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() & pa.PA_DEVERR["QUERY_LAYOUT"]
    qsl = bc.query_start_loc.tolist()
    first_two = list(range(qsl[1], qsl[2])) + list(range(qsl[3], qsl[4]))
    decode_rows = [qsl[0], qsl[2], qsl[4]]
    keep = sorted(first_two + decode_rows)
    P.compare(out[keep], ref[keep], bc.dtype, "varlen, rows inside the bound")


def test_decode_rows_only_equal_pa_decode_bitwise():
    bc = workloads.mixed_lengths(scale=1 / 8)[0]
    b = bc.to(DEV)
    P.gpu_append(b)
    want = P.gpu_decode(b)
    qsl = torch.arange(b.num_seqs + 1, dtype=torch.int32, device=DEV)
    vb = dataclasses.replace(b, query_start_loc=qsl)
    got = _varlen(vb)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_chunks_only_match_oracle_and_pa_chunked_prefill():
    # pa_chunked_prefill may run the items of its last wave as two halves merged after;
    # the mixed-step grid runs every item whole, so the two agree to the merge's rounding
    bc = workloads.prefill_plus_decode(scale=1 / 16)[0]
    b = bc.to(DEV)
    P.gpu_append(b)
    B, Hq, D = b.num_seqs, b.num_q_heads, b.head_dim
    ws = torch.empty(pa.pa_chunked_prefill_workspace_size(B, b.max_query_len, Hq, D,
                                                          b.max_seq_len),
                     dtype=torch.uint8, device=DEV)
    want = torch.empty_like(b.q)
    pa.pa_chunked_prefill(want, b.q, b.k_cache, b.v_cache, b.block_tables, b.seq_lens,
                          b.query_start_loc, b.scale, b.max_query_len, b.max_seq_len, ws)
    got = _varlen(b)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    ref = P.oracle_prefill(bc)
    P.compare(got, ref, bc.dtype, "varlen, chunks only")
    P.compare(want, ref, bc.dtype, "pa_chunked_prefill")
    diff = (got.float() - want.float()).abs().max().item()
    assert diff <= 2 * torch.finfo(bc.dtype).eps * max(1.0, want.float().abs().max().item())


def test_decode_row_outside_q_flagged():
    lens = [50, 60, 70]
    bc = _batch("varlen_bad", lens, [4, 1, 1], 4, torch.float16, seed=9)
    b = bc.to(DEV)
    P.gpu_append(b)
    pa.pa_get_device_error()
    # q holds 5 rows, but the last sequence's row is declared at 5
    qsl = torch.tensor([0, 4, 5, 6], dtype=torch.int32, device=DEV)
    out = _varlen(b, rows=5, qsl=qsl)
    assert pa.pa_get_device_error() & pa.PA_DEVERR["QUERY_LAYOUT"]
    ref = P.oracle_prefill(bc)
    P.compare(out[:5], ref[:5], bc.dtype, "rows inside q")


def test_full_size_prefill_plus_decode_in_one_call_sampled():
    """The chunked-prefill + long-decode step as one varlen batch over one cache: 4 chunks
    of 512 queries (8000-token contexts) and 32 decode rows of 32768 tokens; sampled decode
    rows against the oracle (the chunks' rows are covered at oracle size above)."""
    chunk, total, dec = 512, 8000, 32768
    lens = [total] * 4 + [dec] * 32
    q_lens = [chunk] * 4 + [1] * 32
    b = workloads.make_batch("varlen_full", seq_lens=lens, q_lens=q_lens, num_q_heads=64,
                             num_kv_heads=8, block_size=16,
                             num_blocks=sum(-(-L // 16) for L in lens) + 16,
                             dtype=torch.bfloat16, seed=77, device=DEV, prefill=True)
    seqs = [4, 35]  # the first and the last decode row
    sub = P.sub_batch(b, seqs)
    P.gpu_append(b)
    out = _varlen(b)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    kc, vc = opa.to_f64(sub["k_cache"]), opa.to_f64(sub["v_cache"])
    qsl = b.query_start_loc.cpu().numpy()
    sm = b.slot_mapping.cpu().numpy()
    rows, new_slots, sub_qsl = [], [], [0]
    for s in seqs:
        r = list(range(int(qsl[s]), int(qsl[s + 1])))
        rows += r
        sub_qsl.append(sub_qsl[-1] + len(r))
        for t in r:
            new_slots.append(sub["remap"][int(sm[t]) // 16] * 16 + int(sm[t]) % 16)
    opa.reshape_and_cache(opa.to_f64(b.k_new[rows]), opa.to_f64(b.v_new[rows]), kc, vc,
                          np.array(new_slots))
    ref = opa.chunked_prefill(opa.to_f64(b.q[rows]), kc, vc, sub["block_tables"].numpy(),
                              sub["seq_lens"].numpy(), np.array(sub_qsl), b.scale)
    P.compare(out[rows], ref, b.dtype, "prefill + decode in one call, sampled")
