"""The bounded pipeline waits, exercised on the GPU without any fault: the testing hook
pa_testing_wait_fault makes one launch withhold one arrival (CTA 0's first K/V tile of
the decode kernel, or its first K tile of the chunked-prefill kernel) with a short wait
limit.  The waiting warp must give up, flag PA_DEVERR_TIMEOUT, stop issuing copies and
arrivals, wait for what it has in flight (bulk copies; in the prefill kernel also the
tensor-core products, before its tensor memory is freed) and return within
milliseconds; the context stays usable and the next ordinary call matches the oracle."""
import time

import pytest
import torch

import paged_kv_cache_332_b200 as pa
import workloads
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"
LIMIT = 100_000  # SM cycles, ~50 us at B200 clocks


def _timed(fn):
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    fn()
    torch.cuda.synchronize()
    return time.perf_counter() - t0


def test_decode_wait_gives_up_then_next_call_is_exact():
    bc = workloads.mixed_lengths(scale=1 / 4)[0]
    b = bc.to(DEV)
    P.gpu_append(b)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    ref = P.oracle_decode(bc)
    pa.pa_testing_wait_fault("decode", LIMIT)
    secs = _timed(lambda: P.gpu_decode(b))
    err = pa.pa_get_device_error()
    assert err & pa.PA_DEVERR["TIMEOUT"], err
    assert secs < 0.5, secs  # gave up after its short limit, not the default ~2 s
    for _ in range(2):  # the hook was one-shot: ordinary calls, exact again
        out = P.gpu_decode(b)
        torch.cuda.synchronize()
        assert pa.pa_get_device_error() == 0
        P.compare(out, ref, bc.dtype, "decode after a timed-out launch")


def test_prefill_wait_gives_up_frees_tmem_then_next_call_is_exact():
    lens, qlens = [700, 515, 300], [256, 200, 45]
    nb = sum(-(-L // 16) for L in lens) + 8
    bc = workloads.make_batch("prefill_wait", seq_lens=lens, q_lens=qlens, num_q_heads=16,
                              num_kv_heads=2, block_size=16, num_blocks=nb,
                              dtype=torch.bfloat16, seed=3, prefill=True)
    b = bc.to(DEV)
    P.gpu_append(b)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    ref = P.oracle_prefill(bc)
    pa.pa_testing_wait_fault("prefill", LIMIT)
    secs = _timed(lambda: P.gpu_prefill(b))
    err = pa.pa_get_device_error()
    assert err & pa.PA_DEVERR["TIMEOUT"], err
    assert secs < 0.5, secs
    # every CTA freed its tensor memory: a full grid of CTAs that each allocate all 512
    # TMEM columns runs again, twice, and matches the oracle
    for _ in range(2):
        out = P.gpu_prefill(b)
        torch.cuda.synchronize()
        assert pa.pa_get_device_error() == 0
        P.compare(out, ref, bc.dtype, "prefill after a timed-out launch")


def test_hook_is_one_shot_and_checked():
    with pytest.raises(pa.PagedAttnError):
        pa.lib()  # the library is loaded
        st = pa.lib().pa_testing_wait_fault(1, 0)  # a zero limit is refused
        pa._check(st, "pa_testing_wait_fault")
    pa.pa_testing_wait_fault("decode", LIMIT)
    pa.pa_testing_wait_fault(None)  # cleared before any launch
    bc = workloads.tiny_mha()[0]
    b = bc.to(DEV)
    P.gpu_append(b)
    P.gpu_decode(b)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
