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
import ctypes

import pytest
import torch

import paged_kv_cache_332_b200 as pa
import workloads
from tests import _parity as P

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


def test_noalloc_refuses_sizes_beyond_its_array():
    cap = pa.pa_decode_noalloc_scratch_bytes()
    B, Hq, D, L = 4096, 64, 128, 32768  # partials far above the fixed array
    assert pa.pa_decode_workspace_size(B, Hq, D, L, 512) > cap
    p = ctypes.c_void_p(4096)
    st = pa.lib().pa_decode_noalloc(p, p, p, p, p, 2048, p, B, Hq, 8, D, 0.1, 16, 1 << 20, L, 512,
                                    0, None)
    assert st == 3  # PA_ERR_WORKSPACE_TOO_SMALL
    assert pa.pa_last_launch_count() == 0
