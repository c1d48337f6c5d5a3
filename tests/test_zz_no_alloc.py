"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers of this library never call cudaMalloc themselves: their device memory
belongs to an engine's pre-allocated KV pool or to a host framework that forbids raw
allocations, or they run in a latency-critical loop where an allocation could
synchronise the device.  pa_decode_noalloc serves them by keeping its workspace (the
merge records and the split-K partials) in a fixed array inside the library.
These checks run through the C ABI on a GPU: two calls in a row must reproduce
pa_decode with a caller-provided workspace (within the parity tolerance), and sizes
whose partials do not fit the array must be refused before anything is launched.  The file sorts last so a fail-fast run has already run
every other test when it gets here.
"""
import dataclasses

import pytest
import torch

import paged_kv_cache_332_b200 as pa
import workloads
from tests import _parity as P
from tests._devmem import devmem

pytestmark = pytest.mark.gpu


def test_noalloc_matches_workspace_decode_twice():
    b = workloads.mixed_lengths(scale=1 / 4, device="cuda")[0]
    P.gpu_append(b)
    B, Hq, D = b.q.shape
    need = pa.pa_decode_workspace_size(B, Hq, D, b.max_seq_len, 0)
    assert 0 < need <= pa.pa_decode_noalloc_scratch_bytes()
    ref = P.gpu_decode(b)  # pa_decode with a torch-allocated workspace
    tol = P.TOL[b.dtype]
    for _ in range(2):  # the second call reuses the array the first one left behind
        out = torch.full_like(b.q, float("nan"))
        pa.pa_decode_noalloc(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.seq_lens,
                             b.scale, b.max_seq_len)
        torch.cuda.synchronize()
        assert pa.pa_get_device_error() == 0
        assert torch.isfinite(out).all()
        diff = (out.float() - ref.float()).abs().max().item()
        assert diff <= tol, diff


def test_noalloc_single_partition():
    b = workloads.tiny_mha(device="cuda")[0]
    P.gpu_append(b)
    ref = P.gpu_decode(b, partition_size=256)  # one partition: no merge pass
    out = torch.empty_like(b.q)
    pa.pa_decode_noalloc(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.seq_lens, b.scale,
                         b.max_seq_len, partition_size=256)
    torch.cuda.synchronize()
    assert (out.float() - ref.float()).abs().max().item() <= P.TOL[b.dtype]


def _fresh_workspace_decode(b, partition_size):
    """pa_decode with a NaN-filled workspace of its own (nothing left over)."""
    B, Hq, D = b.q.shape
    ws = torch.full((pa.pa_decode_workspace_size(B, Hq, D, b.max_seq_len, partition_size),),
                    255, dtype=torch.uint8, device=b.q.device)
    out = torch.empty_like(b.q)
    pa.pa_decode(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.seq_lens, b.scale,
                 b.max_seq_len, partition_size, ws)
    return out


def test_noalloc_smaller_batch_after_larger():
    # a large batch leaves merge records and partial rows in the shared array; the next,
    # smaller call (explicit 512-token partitions, some sequences empty or short) must not
    # pick up any of them
    big = workloads.mixed_lengths(scale=1 / 4, device="cuda")[0]
    P.gpu_append(big)
    out_big = torch.empty_like(big.q)
    pa.pa_decode_noalloc(out_big, big.q, big.k_cache, big.v_cache, big.block_tables,
                         big.seq_lens, big.scale, big.max_seq_len, partition_size=512)
    ref_big = _fresh_workspace_decode(big, 512)
    torch.cuda.synchronize()
    assert (out_big.float() - ref_big.float()).abs().max().item() <= P.TOL[big.dtype]
    small = workloads.mixed_lengths(scale=1 / 4, device="cuda")[0]
    keep = torch.arange(0, small.num_seqs, 3, device="cuda")[:12]
    lens = small.seq_lens[keep].clone()
    lens[0] = 0
    lens[3] = 0
    lens[5] = torch.clamp(lens[5], max=7)
    sb = dataclasses.replace(small, q=small.q[keep].contiguous(),
                             block_tables=small.block_tables[keep].contiguous(),
                             seq_lens=lens.contiguous())
    ref = _fresh_workspace_decode(sb, 512)
    for _ in range(2):
        out = torch.full_like(sb.q, float("nan"))
        pa.pa_decode_noalloc(out, sb.q, sb.k_cache, sb.v_cache, sb.block_tables, sb.seq_lens,
                             sb.scale, sb.max_seq_len, partition_size=512)
        torch.cuda.synchronize()
        assert pa.pa_get_device_error() == 0
        assert torch.isfinite(out).all()
        assert (out.float() - ref.float()).abs().max().item() <= P.TOL[sb.dtype]
        assert (out[0] == 0).all() and (out[3] == 0).all()  # empty sequences give zeros


def test_noalloc_refuses_sizes_beyond_its_array():
    cap = pa.pa_decode_noalloc_scratch_bytes()
    # 16 sequences x 8 q-heads, 32768-token bound, 16-token partitions: partials far
    # above the fixed array; every address is real (zero-filled) device memory
    B, Hq, D, L = 16, 8, 128, 32768
    assert pa.pa_decode_workspace_size(B, Hq, D, L, 16) > cap
    m = devmem()
    o, q, kc, vc, bt, sl = (m.region() for _ in range(6))
    st = pa.lib().pa_decode_noalloc(o, q, kc, vc, bt, 2048, sl, B, Hq, 8, D, 0.1, 16, 16, L, 16,
                                    0, None)
    assert st == 3  # PA_ERR_WORKSPACE_TOO_SMALL
    assert pa.pa_last_launch_count() == 0
