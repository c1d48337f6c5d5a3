"""Shared helpers for the GPU parity tests: run the hot path through the C ABI,
run the oracle on the same seeded inputs, compare element by element.

Tolerance (max-abs error against the fp64 oracle rounded to the output type):
2e-3 for fp16 and 1e-2 for bf16.  One unit in the last place of the output
type can exceed those bounds at |o| >= 4 (fp16) or |o| >= 2 (bf16), where a
correctly rounded fp32 result may land one ulp away from the correctly
rounded fp64 one; such elements are accepted only when they are exactly one
ulp off, and are counted and reported separately.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle.paged_attention as opa
import paged_kv_cache_332_b200 as pa
import workloads

TOL = {torch.float16: 2e-3, torch.bfloat16: 1e-2}
FMT = {torch.float16: "float16", torch.bfloat16: "bfloat16"}
MANT = {torch.float16: 10, torch.bfloat16: 7}


def ulp(x, dtype):
    """Spacing of the output type at |x| (normal range)."""
    a = np.maximum(np.abs(x), 2.0 ** -14)
    return 2.0 ** (np.floor(np.log2(a)) - MANT[dtype])


def compare(got, ref64, dtype, what=""):
    """got: torch tensor (any device) of ``dtype``; ref64: fp64 numpy oracle.
    Returns a dict of statistics; raises AssertionError on a mismatch."""
    g = opa.to_f64(got)
    r = opa.round_rne(ref64, FMT[dtype])
    assert g.shape == r.shape, (g.shape, r.shape)
    assert np.all(np.isfinite(g)), "%s: non-finite output" % what
    err = np.abs(g - r)
    tol = TOL[dtype]
    over = err > tol
    one_ulp = over & np.isclose(err, ulp(r, dtype), rtol=0, atol=0)
    bad = over & ~one_ulp
    stats = dict(max_err=float(err.max()) if err.size else 0.0, max_ref=float(np.abs(r).max()) if r.size else 0.0,
                 n=int(err.size), n_one_ulp=int(one_ulp.sum()), n_bad=int(bad.sum()))
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError("%s: %d elements over tolerance %g (max err %g); first at %s: got %r want %r"
                             % (what, int(bad.sum()), tol, float(err.max()), idx.tolist(),
                                [float(g[tuple(i)]) for i in idx], [float(r[tuple(i)]) for i in idx]))
    if one_ulp.any():
        print("%s: %d element(s) exactly one ulp off beyond tolerance (|ref| up to %g)"
              % (what, int(one_ulp.sum()), stats["max_ref"]))
    return stats


# ---------------------------------------------------------------- GPU side

def gpu_append(batch: workloads.PagedBatch, stream=None):
    """pa_reshape_and_cache of the batch's new tokens (in place on the device caches)."""
    pa.pa_reshape_and_cache(batch.k_new, batch.v_new, batch.k_cache, batch.v_cache,
                            batch.slot_mapping, stream=stream)


def gpu_decode(batch: workloads.PagedBatch, partition_size=0, max_seq_len=None, stream=None):
    B, Hq, D = batch.q.shape
    msl = batch.max_seq_len if max_seq_len is None else max_seq_len
    ws_bytes = pa.pa_decode_workspace_size(B, Hq, D, msl, partition_size)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=batch.q.device)
    out = torch.empty_like(batch.q)
    pa.pa_decode(out, batch.q, batch.k_cache, batch.v_cache, batch.block_tables, batch.seq_lens,
                 batch.scale, msl, partition_size, ws, stream=stream)
    return out


def gpu_prefill(batch: workloads.PagedBatch, max_seq_len=None, stream=None):
    out = torch.empty_like(batch.q)
    msl = batch.max_seq_len if max_seq_len is None else max_seq_len
    pa.pa_chunked_prefill(out, batch.q, batch.k_cache, batch.v_cache, batch.block_tables,
                          batch.seq_lens, batch.query_start_loc, batch.scale, batch.max_query_len,
                          msl, None, stream=stream)
    return out


# ---------------------------------------------------------------- oracle side

def sub_batch(batch: workloads.PagedBatch, seqs):
    """CPU copy of the sequences ``seqs`` with only the blocks they use, block ids
    compacted (a relabelling, which the oracle's result does not depend on)."""
    seqs = list(seqs)
    bt = batch.block_tables[seqs].cpu()
    lens = batch.seq_lens[seqs].cpu()
    bs = batch.block_size
    used = sorted({int(bt[i, j]) for i in range(len(seqs))
                   for j in range(opa.blocks_needed(int(lens[i]), bs))})
    remap = {b: i for i, b in enumerate(used)}
    new_bt = torch.zeros_like(bt)
    for i in range(len(seqs)):
        for j in range(opa.blocks_needed(int(lens[i]), bs)):
            new_bt[i, j] = remap[int(bt[i, j])]
    idx = torch.tensor(used, dtype=torch.long, device=batch.k_cache.device)
    kc = batch.k_cache.index_select(0, idx).cpu()
    vc = batch.v_cache.index_select(0, idx).cpu()
    return dict(k_cache=kc, v_cache=vc, block_tables=new_bt, seq_lens=lens, remap=remap)


def oracle_append(batch_cpu: workloads.PagedBatch):
    """Oracle reshape_and_cache on fp64 copies of the CPU caches; returns (kc, vc)."""
    kc = opa.to_f64(batch_cpu.k_cache)
    vc = opa.to_f64(batch_cpu.v_cache)
    opa.reshape_and_cache(opa.to_f64(batch_cpu.k_new), opa.to_f64(batch_cpu.v_new), kc, vc,
                          batch_cpu.slot_mapping.numpy())
    return kc, vc


def oracle_decode(batch_cpu: workloads.PagedBatch, kc=None, vc=None):
    if kc is None:
        kc, vc = oracle_append(batch_cpu)
    return opa.paged_decode(opa.to_f64(batch_cpu.q), kc, vc, batch_cpu.block_tables.numpy(),
                            batch_cpu.seq_lens.numpy(), batch_cpu.scale)


def oracle_prefill(batch_cpu: workloads.PagedBatch, kc=None, vc=None):
    if kc is None:
        kc, vc = oracle_append(batch_cpu)
    return opa.chunked_prefill(opa.to_f64(batch_cpu.q), kc, vc, batch_cpu.block_tables.numpy(),
                               batch_cpu.seq_lens.numpy(), batch_cpu.query_start_loc.numpy(),
                               batch_cpu.scale)
