"""Stream order of the decode launches on the GPU.  The decode grid is launched as a
programmatic dependent of the stream's previous kernel (its CTAs start while that kernel
ends and wait for it before reading any input), and the split-K merge as a dependent of
the decode grid.  Here every input of a call is produced by ordinary kernels queued on
the same stream just before it, with no host synchronisation in between, starting from
poisoned values: the output must match the oracle on the final values, call after
call.  A call that read an input early would see the poison (NaN q, garbage cache rows,
wrong lengths or table rows) and fail the comparison."""
import pytest
import torch

import paged_kv_cache_332_b200 as pa
import workloads
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _decode_into(out, b, ws, stream):
    pa.pa_decode(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.seq_lens, b.scale,
                 b.max_seq_len, 0, ws, stream=stream)


def test_inputs_written_just_before_each_call():
    bc = workloads.mixed_lengths(scale=1 / 8)[0]
    ref = P.oracle_decode(bc)
    b = bc.to(DEV)
    P.gpu_append(b)
    torch.cuda.synchronize()
    # the final inputs, kept aside; the call's own tensors start poisoned
    q_ok, kc_ok, vc_ok = b.q.clone(), b.k_cache.clone(), b.v_cache.clone()
    lens_ok, bt_ok = b.seq_lens.clone(), b.block_tables.clone()
    B, Hq, D = b.q.shape
    ws = torch.empty(pa.pa_decode_workspace_size(B, Hq, D, b.max_seq_len, 0), dtype=torch.uint8,
                     device=DEV)
    s = torch.cuda.Stream()
    outs = []
    with torch.cuda.stream(s):
        for it in range(4):
            # poison, then write the real values with ordinary kernels on the same stream
            b.q.fill_(float("nan"))
            b.k_cache.fill_(float("nan"))
            b.v_cache.fill_(float("nan"))
            b.seq_lens.fill_(0)
            b.block_tables.fill_(-1)
            b.q.copy_(q_ok)
            b.k_cache.copy_(kc_ok)
            b.v_cache.copy_(vc_ok)
            b.seq_lens.copy_(lens_ok)
            b.block_tables.copy_(bt_ok)
            out = torch.full_like(b.q, float("nan"))
            _decode_into(out, b, ws, s.cuda_stream)
            outs.append(out)
    s.synchronize()
    assert pa.pa_get_device_error() == 0
    for it, out in enumerate(outs):
        P.compare(out, ref, bc.dtype, "decode %d after its inputs were rewritten" % it)


def _shared_into(out, b, ws, stream):
    gs, pl = b.group_starts, b.prefix_lens
    max_group = int((gs[1:] - gs[:-1]).max())
    pa.pa_decode_shared_prefix(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.seq_lens, gs,
                               pl, b.scale, b.max_seq_len, max_group, int(pl.max()), ws,
                               stream=stream)


def test_back_to_back_calls_share_one_workspace():
    # consecutive calls of three kinds on one stream and one workspace: each call's decode
    # grid may start while the previous call's merge ends, and must not overwrite the
    # partials or merge records that merge still reads
    batches = [workloads.mixed_lengths(scale=1 / 8)[0],
               workloads.llama70b_uniform(scale=1 / 16)[0],
               workloads.shared_prefix(block_size=16, scale=1 / 8)[0]]
    refs = [P.oracle_decode(bc) for bc in batches]
    devs = [bc.to(DEV) for bc in batches]
    for b in devs:
        P.gpu_append(b)
    torch.cuda.synchronize()
    n = 0
    for b in devs:
        B, Hq, D = b.q.shape
        n = max(n, pa.pa_decode_workspace_size(B, Hq, D, b.max_seq_len, 0),
                pa.pa_decode_shared_prefix_workspace_size(B, Hq, b.num_kv_heads, D, b.max_seq_len))
    ws = torch.empty(n, dtype=torch.uint8, device=DEV)
    s = torch.cuda.Stream()
    outs = []
    with torch.cuda.stream(s):
        for it in range(9):
            k = it % 3
            b = devs[k]
            out = torch.full_like(b.q, float("nan"))
            if k == 2:
                _shared_into(out, b, ws, s.cuda_stream)
            else:
                _decode_into(out, b, ws, s.cuda_stream)
            outs.append((k, out))
    s.synchronize()
    assert pa.pa_get_device_error() == 0
    for it, (k, out) in enumerate(outs):
        P.compare(out, refs[k], batches[k].dtype, "back-to-back call %d" % it)
