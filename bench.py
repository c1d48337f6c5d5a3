#!/usr/bin/env python
"""Benchmark of the paged-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one pass of the whole hot path over one batch of the workload: the
append of this step's new tokens and the decode attention, as one
pa_decode_append call (decode kernel with the append + log-sum-exp merge) — and,
for the mixed prefill workload, pa_reshape_and_cache of the chunk tokens and
pa_chunked_prefill as well.  Inputs are seeded synthetic tensors already
resident in HBM when the timed region starts; L2 is flushed (by reading a
buffer twice its size) before every timed step and every timed call.  The step
runs as one CUDA graph replay.  Times are CUDA-event times on the launching
stream, bracketed by barrier + synchronize, max over ranks.  Rank 0 prints one
JSON line.

With --gpus N > 1 (launched by torch.distributed.run) every rank runs an
independent replica of the workload (the sequences of a decode batch are
independent; the path has no exchange step), so the value is the whole-job
throughput of N replicas (weak scaling).

--impl reference times the fp64 CPU oracle (the plain restatement of what the
path computes) on the host cores, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

L2_BYTES = 126 * 1024 * 1024
DEFAULT_WORKLOAD = "mixed"
# measured beside the default workload: LLaMA-2-70B-shaped decode, shared prompts (block
# size 16 and 32), chunked prefill + long decode (two calls, and one varlen call), tiny
OTHERS = ("llama70b", "shared16", "shared32", "prefill_decode", "varlen", "tiny")
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------- helpers

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=FALLBACK_HBM_GBS, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                source="fallback")


def kernel_source_sha(path: str, start: str, end: str) -> str:
    """sha256 of a kernel's source text: from the line holding `start` up to `end`."""
    import hashlib
    with open(os.path.join(ROOT, path), encoding="utf-8") as f:
        text = f.read()
    i = text.index(start)
    j = text.index(end, i)
    return hashlib.sha256(text[i:j].encode()).hexdigest()


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu record, or None when the kernel's
    source text changed since the capture (or no capture matches the workload)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f).get(kernel)
        if not rec or rec.get("workload") != workload:
            return None
        h = kernel_source_sha(rec["source"], rec["region_start"], rec["region_end"])
        return int(rec["dram_bytes_per_launch"]) if h.startswith(rec["source_sha256_prefix"]) else None
    except Exception:
        return None


def decode_algorithmic_bytes(b: workloads.PagedBatch, shared: bool = False) -> int:
    """KV of every token at its exact length, q and out, table rows, seq_lens (plus the
    per-kv-head scales of an FP8 cache).  With ``shared``, the tokens of a group's shared
    prefix count once per group (and the group arrays are added)."""
    e = b.q.element_size()
    ekv = b.k_cache.element_size()
    lens = b.seq_lens.cpu().numpy().astype(np.int64)
    B = len(lens)
    tokens = int(lens.sum())
    if shared:
        gs = b.group_starts.cpu().numpy().astype(np.int64)
        pl = b.prefix_lens.cpu().numpy().astype(np.int64)
        tokens -= int(((gs[1:] - gs[:-1] - 1).clip(min=0) * pl).sum())
        extra = 4 * (len(gs) + len(pl))
    else:
        extra = 0
    kv = tokens * 2 * b.num_kv_heads * b.head_dim * ekv + extra
    if b.k_scale is not None:
        kv += 2 * 4 * b.num_kv_heads
    qo = 2 * B * b.num_q_heads * b.head_dim * e
    tables = B * int(math.ceil(int(lens.max()) / b.block_size)) * 4
    return kv + qo + tables + 4 * B


def prefill_flops(b: workloads.PagedBatch) -> int:
    """4*D*Hq per (query, visible key) pair (QK^T and PV, 2 flops per MAC)."""
    lens = b.seq_lens.cpu().numpy().astype(np.int64)
    qsl = b.query_start_loc.cpu().numpy().astype(np.int64)
    pairs = 0
    for s in range(len(lens)):
        n = int(qsl[s + 1] - qsl[s])
        L = int(lens[s])
        pairs += sum(L - n + i + 1 for i in range(n))
    return 4 * b.head_dim * b.num_q_heads * pairs


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def aggregate_max(value: float, device) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


# ---------------------------------------------------------------- the step

class Step:
    """All device buffers of one workload and the hot-path calls of one step."""

    def __init__(self, batches, pa, stream):
        self.pa = pa
        self.stream = stream
        self.batches = batches
        self.decode = [b for b in batches if b.query_start_loc is None]
        self.prefill = [b for b in batches if b.query_start_loc is not None]
        # a decode batch whose every sequence appends one token runs pa_decode_append
        # (the append inside the decode launch); others append with pa_reshape_and_cache
        # a batch whose sequences share prompt blocks runs pa_decode_shared_prefix (the
        # shared blocks read once per group), after pa_reshape_and_cache
        self.shared = {id(b): b.group_starts is not None and b.k_scale is None
                       for b in self.decode}
        self.fused = {id(b): int(b.k_new.shape[0]) == b.num_seqs and b.k_scale is None
                      and not self.shared[id(b)] for b in self.decode}
        # a varlen batch mixing rows of one query and longer chunks runs
        # pa_attention_varlen (decode kernel + prefill kernel in one call)
        self.varlen = {}
        self.chunk_seqs = {}
        for b in self.prefill:
            ql = (b.query_start_loc[1:] - b.query_start_loc[:-1]).cpu()
            self.varlen[id(b)] = bool((ql == 1).any()) and bool((ql > 1).any())
            self.chunk_seqs[id(b)] = int((ql > 1).sum())
        self.group_bounds = {}
        for b in self.decode:
            if self.shared[id(b)]:
                sizes = (b.group_starts[1:] - b.group_starts[:-1]).cpu()
                self.group_bounds[id(b)] = (int(sizes.max()), int(b.prefix_lens.max()))
        self.ws = {}
        self.out = {}
        for b in batches:
            self.out[id(b)] = torch.empty_like(b.q)
            if b.query_start_loc is None and self.shared[id(b)]:
                n = pa.pa_decode_shared_prefix_workspace_size(b.num_seqs, b.num_q_heads,
                                                              b.num_kv_heads, b.head_dim,
                                                              b.max_seq_len)
            elif b.query_start_loc is None:
                n = pa.pa_decode_workspace_size(b.num_seqs, b.num_q_heads, b.head_dim, b.max_seq_len, 0)
            elif self.varlen[id(b)]:
                n = pa.pa_attention_varlen_workspace_size(b.num_seqs, b.max_query_len,
                                                          b.num_q_heads, b.head_dim, b.max_seq_len)
            else:
                n = pa.pa_chunked_prefill_workspace_size(b.num_seqs, b.max_query_len, b.num_q_heads,
                                                         b.head_dim, b.max_seq_len)
            self.ws[id(b)] = torch.empty(n, dtype=torch.uint8, device=b.q.device)
        self.max_len = {id(b): b.max_seq_len for b in batches}
        self.max_q = {id(b): b.max_query_len for b in batches}
        self.launches = 0

    def run_prefill(self, record=None):
        n = 0
        for b in self.prefill:
            if record is not None:
                record[0].record(self.stream)
            if self.varlen[id(b)]:
                self.pa.pa_attention_varlen(self.out[id(b)], b.q, b.k_cache, b.v_cache,
                                            b.block_tables, b.seq_lens, b.query_start_loc,
                                            b.scale, self.max_q[id(b)], self.max_len[id(b)],
                                            self.ws[id(b)], stream=self.stream,
                                            max_chunk_seqs=self.chunk_seqs[id(b)])
            else:
                self.pa.pa_chunked_prefill(self.out[id(b)], b.q, b.k_cache, b.v_cache,
                                           b.block_tables, b.seq_lens, b.query_start_loc, b.scale,
                                           self.max_q[id(b)], self.max_len[id(b)], self.ws[id(b)],
                                           stream=self.stream)
            n += self.pa.pa_last_launch_count()
            if record is not None:
                record[1].record(self.stream)
        return n

    def run_decode(self, record=None):
        n = 0
        for b in self.decode:
            if record is not None:
                record[0].record(self.stream)
            if b.k_scale is not None:
                self.pa.pa_decode_fp8(self.out[id(b)], b.q, b.k_cache, b.v_cache, b.k_scale,
                                      b.v_scale, b.block_tables, b.seq_lens, b.scale,
                                      self.max_len[id(b)], 0, self.ws[id(b)], stream=self.stream)
            elif self.shared[id(b)]:
                mg, mp = self.group_bounds[id(b)]
                self.pa.pa_decode_shared_prefix(self.out[id(b)], b.q, b.k_cache, b.v_cache,
                                                b.block_tables, b.seq_lens, b.group_starts,
                                                b.prefix_lens, b.scale, self.max_len[id(b)], mg,
                                                mp, self.ws[id(b)], stream=self.stream)
            elif self.fused[id(b)]:
                self.pa.pa_decode_append(self.out[id(b)], b.q, b.k_new, b.v_new, b.k_cache,
                                         b.v_cache, b.block_tables, b.seq_lens, b.scale,
                                         self.max_len[id(b)], 0, self.ws[id(b)],
                                         stream=self.stream)
            else:
                self.pa.pa_decode(self.out[id(b)], b.q, b.k_cache, b.v_cache, b.block_tables,
                                  b.seq_lens, b.scale, self.max_len[id(b)], 0, self.ws[id(b)],
                                  stream=self.stream)
            n += self.pa.pa_last_launch_count()
            if record is not None:
                record[1].record(self.stream)
        return n

    def run(self):
        """One step: append the new tokens, then chunked prefill, then decode.
        Returns the number of kernels launched."""
        n = 0
        for b in self.batches:
            if self.fused.get(id(b)):
                continue  # appended inside its decode launch
            if b.k_scale is not None:
                self.pa.pa_reshape_and_cache_fp8(b.k_new, b.v_new, b.k_cache, b.v_cache,
                                                 b.slot_mapping, b.k_scale, b.v_scale,
                                                 stream=self.stream)
            else:
                self.pa.pa_reshape_and_cache(b.k_new, b.v_new, b.k_cache, b.v_cache,
                                             b.slot_mapping, stream=self.stream)
            n += self.pa.pa_last_launch_count()
        n += self.run_prefill()
        n += self.run_decode()
        self.launches += n
        return n


SPLIT_K = ("balanced split-K (partition_size 0): the 16-token tiles of every (sequence, "
           "kv-head group) laid end to end, each CTA of a persistent grid (one per SM) takes "
           "an equal share; a group split over several CTAs is merged by log-sum-exp")


def rooflines(step, dec_ms, pre_ms, peaks):
    """The roofline objects of one workload: `roofline` for its decode call (HBM) or, for
    a varlen step, the call's serial speed of light; `roofline_prefill` (tensor cores) for
    a separate chunked-prefill call."""
    out = {}
    dec = step.decode[0] if step.decode else None
    pre = step.prefill[0] if step.prefill else None
    if dec is not None:
        ab = decode_algorithmic_bytes(dec)
        if step.fused[id(dec)]:  # the append inside the launch: read k/v_new, write the slots
            ab += 2 * 2 * dec.num_seqs * dec.num_kv_heads * dec.head_dim * dec.q.element_size()
        shared = step.shared[id(dec)]
        if shared:  # the shared blocks are read once per group
            ab_unshared = ab
            ab = decode_algorithmic_bytes(dec, shared=True)
        dmean = statistics.mean(dec_ms)
        ach = ab / (dmean / 1e3) / 1e9
        kname = ("pa_decode_fp8" if dec.k_scale is not None else
                 "pa_decode_shared_prefix" if shared else
                 "pa_decode_append" if step.fused[id(dec)] else "pa_decode")
        kparts = (" (paged_decode_kernel over own keys and prefix chunks + merge_kernel)"
                  if shared else " (paged_decode_kernel + merge_kernel)")
        out["roofline"] = {"kernel": kname + kparts,
                           "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                           "peak_source": peaks["source"], "unit": "GB/s",
                           "frac": round(ach / peaks["hbm_gbs"], 4),
                           "frac_of_8TBs_spec": round(ach / 8000.0, 4),
                           "algorithmic_bytes": ab, "ms_per_launch": round(dmean, 5),
                           "traffic": recorded_traffic("paged_decode_kernel", dec.name)}
        if shared:
            out["roofline"]["algorithmic_bytes_unshared"] = ab_unshared
            out["roofline"]["note"] = ("bytes count each shared prefix block once per group; "
                                       "algorithmic_bytes_unshared counts it once per member")
    if pre is not None and step.varlen[id(pre)]:
        # one call: its speed of light is the decode rows' bytes at the HBM peak plus the
        # chunks' flops at the tensor peak
        ql = (pre.query_start_loc[1:] - pre.query_start_loc[:-1]).cpu().numpy()
        lens = pre.seq_lens.cpu().numpy().astype(np.int64)
        dec_rows = ql == 1
        e = pre.q.element_size()
        dec_bytes = int(lens[dec_rows].sum()) * 2 * pre.num_kv_heads * pre.head_dim * e + \
            2 * int(dec_rows.sum()) * pre.num_q_heads * pre.head_dim * e + \
            int(dec_rows.sum()) * int(math.ceil(int(lens.max()) / pre.block_size)) * 4
        fl = 4 * pre.head_dim * pre.num_q_heads * sum(
            sum(int(L) - int(n) + i + 1 for i in range(int(n))) for L, n in zip(lens, ql) if n > 1)
        pmean = statistics.mean(pre_ms)
        ideal_ms = (dec_bytes / (peaks["hbm_gbs"] * 1e9) + fl / (peaks["bf16_tflops"] * 1e12)) * 1e3
        out["roofline"] = {"kernel": "pa_attention_varlen (varlen_list_kernel + varlen_kernel:"
                                     " decode CTAs beside chunked-prefill CTAs + merge_kernel)",
                           "bound": "hbm (decode rows) beside tensor (chunks)",
                           "achieved": round(ideal_ms / pmean, 4), "peak": 1.0,
                           "unit": "fraction of the serial speed of light",
                           "frac": round(ideal_ms / pmean, 4), "ms_per_launch": round(pmean, 5),
                           "ideal_ms": round(ideal_ms, 5), "decode_bytes": dec_bytes,
                           "chunk_flop": fl, "peak_source": peaks["source"], "traffic": None}
    elif pre is not None:
        fl = prefill_flops(pre)
        pmean = statistics.mean(pre_ms)
        tf = fl / (pmean / 1e3) / 1e12
        peak_tf = peaks["bf16_tflops"]
        out["roofline_prefill"] = {"kernel": "pa_chunked_prefill (chunked_prefill_kernel, tcgen05)",
                                   "bound": "tensor", "achieved": round(tf, 1), "peak": peak_tf,
                                   "peak_source": peaks["source"] + " bf16 dense burst",
                                   "unit": "TFLOP/s", "frac": round(tf / peak_tf, 4),
                                   "flop_per_launch": fl, "ms_per_launch": round(pmean, 5),
                                   "traffic": None}
    return out


def step_tokens(step):
    return sum(b.num_seqs for b in step.decode) + sum(int(b.q.shape[0]) for b in step.prefill)


def measure_other(name, args, device, pa, stream, l2_flush, peaks):
    """One more workload in the same process: its step replayed as a CUDA graph (tokens/s,
    L2 flushed before every step) and its decode / prefill calls timed one by one for the
    roofline, inside one clock record."""
    batches = workloads.WORKLOADS[name](device=device)
    step = Step(batches, pa, stream)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            l2_flush()
            step.run()
    torch.cuda.synchronize(device)
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream):
        step.run()
    timed = {k: timing_graph(step, k, stream, l2_flush) for k, bb in
             (("decode", step.decode), ("prefill", step.prefill)) if bb}
    steps = max(3, min(args.steps, 20))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            l2_flush()
            g_step.replay()
        for g, _ in timed.values():
            g.replay()
    torch.cuda.synchronize(device)
    with ClockSampler(device) as clocks:
        with torch.cuda.stream(stream):
            for i in range(steps):
                l2_flush()
                ev[i][0].record(stream)
                g_step.replay()
                ev[i][1].record(stream)
        torch.cuda.synchronize(device)
        ms = {}
        for k, (g, evs) in timed.items():
            with torch.cuda.stream(stream):
                g.replay()
            torch.cuda.synchronize(device)
            ms[k] = [a.elapsed_time(b) for a, b in evs]
    step_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    r = rooflines(step, ms.get("decode", []), ms.get("prefill", []), peaks)
    res = {"value": round(step_tokens(step) / (step_ms / 1e3), 1), "unit": "tokens/s",
           "ms_per_step": round(step_ms, 5), "steps": steps,
           "workload": "+".join(b.name for b in batches), "clocks": clocks.summary()}
    for k in ("roofline", "roofline_prefill"):
        if k in r:
            res[k] = {kk: r[k][kk] for kk in ("kernel", "achieved", "unit", "frac",
                                              "ms_per_launch") if kk in r[k]}
    del g_step, timed, step, batches
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()
    return res


N_KERNEL_TIMED = 8


def timing_graph(step, kind, stream, l2_flush):
    """A graph of N calls of the step's decode (or prefill) calls, each bracketed by
    event-record nodes and preceded by an L2 flush."""
    evs = [(torch.cuda.Event(enable_timing=True, external=True),
            torch.cuda.Event(enable_timing=True, external=True)) for _ in range(N_KERNEL_TIMED)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(N_KERNEL_TIMED):
            l2_flush()
            if kind == "decode":
                step.run_decode(evs[i])
            else:
                step.run_prefill(evs[i])
    return g, evs


# ---------------------------------------------------------------- arms

def block_pool_timing(pa, dec, stream, device, n=8):
    """Device time of the block-table calls for one decode step of ``dec``'s sequences:
    pa_block_allocate with one new token per sequence (sequences at a block boundary take
    a block) and pa_block_free of every 16th sequence.  Pool, tables and owned counts are
    restored from a snapshot before each timed call, so every call does the same work."""
    B, bs = dec.num_seqs, dec.block_size
    lens = dec.seq_lens
    max_blocks = -(-(int(lens.max()) + 1) // bs)
    n_blocks = int(((lens + 1 + bs - 1) // bs).sum()) + B
    ring = torch.empty(n_blocks, dtype=torch.int32, device=device)
    state = torch.empty(2, dtype=torch.int32, device=device)
    tables = torch.zeros((B, max_blocks), dtype=torch.int32, device=device)
    owned = torch.zeros(B, dtype=torch.int32, device=device)
    zeros = torch.zeros(B, dtype=torch.int32, device=device)
    ones = torch.ones(B, dtype=torch.int32, device=device)
    slots = torch.empty(max(int(lens.sum()), B, 1), dtype=torch.int32, device=device)
    granted = torch.empty(B, dtype=torch.int32, device=device)
    finished = (torch.arange(B, device=device) % 16 == 0).to(torch.int32)
    with torch.cuda.stream(stream):
        pa.pa_block_pool_init(ring, state, stream=stream)
        # prompts: every sequence's first seq_lens tokens
        pa.pa_block_allocate(ring, state, tables, owned, zeros, lens, bs, slots, granted,
                             stream=stream)
    torch.cuda.synchronize(device)
    snap = [t.clone() for t in (ring, state, tables, owned)]
    new_blocks = int(((lens % bs) == 0).sum())

    def timed(call):
        # captured as one graph (restore, event, call, event) x n, so the host's launch
        # latency stays out of the device time between the events
        evs = [(torch.cuda.Event(enable_timing=True, external=True),
                torch.cuda.Event(enable_timing=True, external=True)) for _ in range(n)]
        with torch.cuda.stream(stream):
            call()  # first-call set-up outside the capture
        torch.cuda.synchronize(device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for a, b in evs:
                for dst, src in zip((ring, state, tables, owned), snap):
                    dst.copy_(src)
                a.record(stream)
                call()
                b.record(stream)
        with torch.cuda.stream(stream):
            g.replay()  # warm
            g.replay()
        torch.cuda.synchronize(device)
        return statistics.mean(a.elapsed_time(b) for a, b in evs) * 1e3

    alloc_us = timed(lambda: pa.pa_block_allocate(ring, state, tables, owned, lens, ones, bs,
                                                  slots, granted, stream=stream))
    free_us = timed(lambda: pa.pa_block_free(ring, state, tables, owned, finished,
                                             stream=stream))
    return {"allocate_us": round(alloc_us, 2), "free_us": round(free_us, 2), "num_seqs": B,
            "new_blocks_per_allocate": new_blocks, "freed_seqs": int(finished.sum()),
            "bound": "latency (one CTA per call; a few KB of table traffic)",
            "note": "pa_block_allocate: one token per sequence; pa_block_free: every 16th "
                    "sequence; state restored before each of %d timed calls" % n}


def run_ours(args, rank, world, device):
    import paged_kv_cache_332_b200 as pa
    pa.lib()  # fails loudly if the library is missing
    torch.cuda.set_device(device)
    stream = torch.cuda.Stream(device=device)
    batches = workloads.WORKLOADS[args.workload](device=device)
    step = Step(batches, pa, stream)
    dec = step.decode[0] if step.decode else None
    pre = step.prefill[0] if step.prefill else None
    kv_bytes = sum(b.k_cache.numel() * b.k_cache.element_size() * 2 for b in batches)
    # L2 is flushed between timed iterations for every workload (outside the timed
    # span), so no call finds the previous call's KV in the 126 MB L2.  The flush READS
    # a buffer twice the size of L2: it leaves clean lines behind, so the timed kernel
    # pays no write-back of the flush's own data.
    flush_buf = torch.zeros(2 * L2_BYTES // 4, dtype=torch.float32, device=device)

    def l2_flush():
        torch.sum(flush_buf)

    def one():
        l2_flush()
        return step.run()

    # eager warm-up: first calls set up per-device state (error flag, kernel attributes)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            one()
    torch.cuda.synchronize(device)
    step.launches = 0
    with torch.cuda.stream(stream):
        per_step_launches = step.run()
    torch.cuda.synchronize(device)

    # The step is replayed as a CUDA graph (reshape_and_cache, chunked prefill, decode),
    # so the host's per-call work stays off the GPU timeline.
    g_step = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step, stream=stream):
        step.run()
    # Per-call device time of pa_decode / pa_chunked_prefill: a graph of N calls, each
    # bracketed by event-record nodes and preceded by an L2 flush.
    n_kt = N_KERNEL_TIMED
    g_dec = timing_graph(step, "decode", stream, l2_flush) if dec is not None else None
    g_pre = timing_graph(step, "prefill", stream, l2_flush) if pre is not None else None
    # The pages' indirection comparison: the same decode with identity tables (each
    # sequence's blocks contiguous and in order), when the pool holds every sequence's
    # blocks without sharing.
    g_ident = g_paged = None
    if dec is not None:
        nb = [-(-int(L) // dec.block_size) for L in dec.seq_lens.tolist()]
        if sum(nb) <= dec.num_blocks:
            ident = torch.zeros_like(dec.block_tables)
            off = 0
            for i, n in enumerate(nb):
                ident[i, :n] = torch.arange(off, off + n, dtype=torch.int32, device=device)
                off += n
            out_ident = torch.empty_like(dec.q)

            def decode_graph(tables):
                evs = [(torch.cuda.Event(enable_timing=True, external=True),
                        torch.cuda.Event(enable_timing=True, external=True)) for _ in range(n_kt)]
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for i in range(n_kt):
                        l2_flush()
                        evs[i][0].record(stream)
                        if dec.k_scale is not None:
                            pa.pa_decode_fp8(out_ident, dec.q, dec.k_cache, dec.v_cache,
                                             dec.k_scale, dec.v_scale, tables, dec.seq_lens,
                                             dec.scale, step.max_len[id(dec)], 0,
                                             step.ws[id(dec)], stream=stream)
                        else:
                            pa.pa_decode(out_ident, dec.q, dec.k_cache, dec.v_cache, tables,
                                         dec.seq_lens, dec.scale, step.max_len[id(dec)], 0,
                                         step.ws[id(dec)], stream=stream)
                        evs[i][1].record(stream)
                return g, evs
            g_paged = decode_graph(dec.block_tables)
            g, evs = decode_graph(ident)
            g_ident = (g, evs)
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            l2_flush()
            g_step.replay()
        for timed in (g_dec, g_pre, g_ident, g_paged):
            if timed is not None:
                timed[0].replay()
    torch.cuda.synchronize(device)

    # ---- timed region (device-resident inputs)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    with ClockSampler(device) as clocks:
        barrier()
        torch.cuda.synchronize(device)
        with torch.cuda.stream(stream):
            for i in range(args.steps):
                l2_flush()
                ev[i][0].record(stream)
                g_step.replay()
                ev[i][1].record(stream)
        torch.cuda.synchronize(device)
        barrier()
        # kernel timing for the roofline, inside the same clock record
        def kernel_ms(timed):
            if timed is None:
                return []
            graph, events = timed
            with torch.cuda.stream(stream):
                graph.replay()
            torch.cuda.synchronize(device)
            return [a.elapsed_time(b) for a, b in events]
        dec_ms = kernel_ms(g_dec)
        pre_ms = kernel_ms(g_pre)
        ident_ms = kernel_ms(g_ident)
        paged_ms = kernel_ms(g_paged)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    local_ms = sum(step_ms)
    launches = per_step_launches * args.steps
    total_ms = aggregate_max(local_ms, device)

    # ---- end to end through the C ABI: every step uploads that step's inputs (q, new
    # K/V, slot mapping, lengths, block tables) from pinned host memory and reads the
    # outputs back.  The inputs of a step are packed into one pinned buffer and one device
    # staging buffer (one copy each way per step); two staging buffers alternate, so the
    # upload of step i+1 runs on a copy stream while step i computes.
    e2e_steps = max(3, min(args.steps, 20))
    fields = ["q", "k_new", "v_new", "slot_mapping", "seq_lens", "block_tables",
              "query_start_loc", "group_starts", "prefix_lens"]

    def packed_layout():
        offs, off = [], 0
        for bb in batches:
            o = {}
            for n in fields:
                t = getattr(bb, n)
                if t is None:
                    continue
                o[n] = off
                off += -(-t.numel() * t.element_size() // 256) * 256
            offs.append(o)
        return offs, off
    offs, in_bytes = packed_layout()
    host_in = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
    for bb, o in zip(batches, offs):
        for n, off in o.items():
            t = getattr(bb, n).contiguous().view(-1).view(torch.uint8).cpu()
            host_in[off:off + t.numel()].copy_(t)

    def staged_step():
        dev_in = host_in.to(device)  # the Step reads lengths from it when it sizes itself
        views = []
        for bb, o in zip(batches, offs):
            kw = {}
            for n, off in o.items():
                t = getattr(bb, n)
                nbytes = t.numel() * t.element_size()
                kw[n] = dev_in[off:off + nbytes].view(t.dtype).view(t.shape)
            views.append(dataclasses.replace(bb, **kw))
        st = Step(views, pa, stream)
        outs = [st.out[id(v)] for v in views]
        out_bytes = sum(t.numel() * t.element_size() for t in outs)
        dev_out = torch.empty(out_bytes, dtype=torch.uint8, device=device)
        off = 0
        for v, t in zip(views, outs):
            nbytes = t.numel() * t.element_size()
            st.out[id(v)] = dev_out[off:off + nbytes].view(t.dtype).view(t.shape)
            off += nbytes
        host_out = torch.empty(out_bytes, dtype=torch.uint8).pin_memory()
        return dev_in, st, dev_out, host_out
    stages = [staged_step() for _ in range(2)]
    h2d = in_bytes
    d2h = stages[0][2].numel()
    # uploads and read-backs on two copy streams of their own, so an upload never waits
    # behind the previous step's read-back
    copy_stream = torch.cuda.Stream(device=device)
    back_stream = torch.cuda.Stream(device=device)
    ready = [torch.cuda.Event() for _ in range(2)]
    computed = [torch.cuda.Event() for _ in range(2)]
    done = [torch.cuda.Event() for _ in range(2)]
    with torch.cuda.stream(stream):  # warm the staged calls once (first-call set-up)
        for dev_in, st, dev_out, host_out in stages:
            dev_in.copy_(host_in, non_blocking=True)
            st.run()
    torch.cuda.synchronize(device)
    # each staging buffer's step as a CUDA graph of the same library calls, as an engine
    # that captures its decode step would run them
    graphs = []
    for dev_in, st, dev_out, host_out in stages:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            st.run()
        graphs.append(g)
    barrier()
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        copy_stream.wait_event(e0)
        for i in range(e2e_steps):
            j = i % 2
            dev_in, st, dev_out, host_out = stages[j]
            with torch.cuda.stream(copy_stream):
                if i >= 2:
                    copy_stream.wait_event(computed[j])  # step i-2 has read its inputs
                dev_in.copy_(host_in, non_blocking=True)
                ready[j].record(copy_stream)
            stream.wait_event(ready[j])
            if i >= 2:
                stream.wait_event(done[j])  # step i-2's outputs are back on the host
            graphs[j].replay()
            computed[j].record(stream)
            with torch.cuda.stream(back_stream):
                # the read-back runs beside the next step's compute
                back_stream.wait_event(computed[j])
                host_out.copy_(dev_out, non_blocking=True)
                done[j].record(back_stream)
        for j in range(min(2, e2e_steps)):
            stream.wait_event(done[j])
        e1.record(stream)
    torch.cuda.synchronize(device)
    barrier()
    e2e_ms = aggregate_max(e0.elapsed_time(e1), device)
    del graphs

    pool_line = block_pool_timing(pa, dec, stream, device) if dec is not None else None

    # ---- metric
    tokens = sum(b.num_seqs for b in step.decode) + sum(int(b.q.shape[0]) for b in step.prefill)
    value = world * tokens * args.steps / (total_ms / 1e3)
    peaks = measured_peaks()
    line = {
        "metric": "paged decode tokens/s (one layer) and achieved HBM GB/s of pa_decode",
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("bf16" if batches[0].dtype == torch.bfloat16 else "fp16")
                 + ("; KV cache e4m3" if any(b.k_scale is not None for b in batches) else ""),
        "data": "synthetic (seeded N(0,1) q/K/V, FIFO free-list block tables)",
        "impl": "ours",
        "gpu_launches": launches,
    }
    cfg = {"workload": "+".join(b.name for b in batches), "parallelism": "replicas%d" % world,
           "launch": "each step replays one CUDA graph of the library calls",
           "l2": "flushed between timed steps and between timed calls (%.0f MB of KV cache "
                 "per replica)" % (kv_bytes / 1e6),
           "split_k": SPLIT_K}
    if dec is not None:
        cfg.update(num_seqs=dec.num_seqs, q_heads=dec.num_q_heads, kv_heads=dec.num_kv_heads,
                   head_dim=dec.head_dim, block_size=dec.block_size,
                   context_tokens=int(dec.seq_lens.sum().item()))
    line["config"] = cfg
    line.update(rooflines(step, dec_ms, pre_ms, peaks))
    if dec is not None:
        if ident_ms:
            im, pm = statistics.mean(ident_ms), statistics.mean(paged_ms)
            line["indirection"] = {"paged_ms": round(pm, 5), "identity_tables_ms": round(im, 5),
                                   "overhead": round(pm / im - 1, 4),
                                   "note": "pa_decode with the workload's tables vs each "
                                           "sequence's blocks contiguous and in order"}
        line["context_tokens_per_s"] = round(world * int(dec.seq_lens.sum().item()) * args.steps
                                             / (total_ms / 1e3), 1)
    line["e2e"] = {"value": round(world * tokens * e2e_steps / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                   "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                   "note": "the C-ABI calls of each step replayed as a CUDA graph; each step's "
                           "inputs packed in one pinned buffer and uploaded on a copy stream "
                           "while the previous step computes (two staging buffers); outputs "
                           "copied back to pinned host memory every step on a second copy "
                           "stream"}
    if pool_line is not None:
        line["block_pool"] = pool_line
    line["clocks"] = clocks.summary()
    if args.others and args.workload == DEFAULT_WORKLOAD:
        # the other workloads of the method's configurations, measured in this process
        del stages
        torch.cuda.empty_cache()
        line["other_workloads"] = {
            n: measure_other(n, args, device, pa, stream, l2_flush, peaks) for n in OTHERS}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:  # the oracle at N = 1 only
        line["cpu_baseline"] = cpu_baseline(batches, args)
    return line


def cpu_baseline(batches, args, budget_s=None):
    """Time the oracle, as it stands, on a bounded sample of the workload and scale to
    the metric (query rows of a full step per second: decoded tokens plus chunk rows).
    The work of a sequence is its (query row, visible key) pairs; sequences of every
    batch are drawn in a seeded order until the budget is spent, and the time is scaled
    by the pairs of the whole step over the pairs done."""
    import oracle.paged_attention as opa
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
        blas_threads = max([p.get("num_threads", 0) for p in threadpool_info()
                            if p.get("user_api") == "blas"] or [0])
        limiter = threadpool_limits(1)
    except Exception:  # pragma: no cover
        limiter, blas_threads = None, None
    budget_s = budget_s if budget_s is not None else args.cpu_budget
    units, total_pairs, total_rows = [], 0, 0
    for bi, b in enumerate(batches):
        lens = b.seq_lens.cpu().numpy().astype(np.int64)
        if b.query_start_loc is None:
            ql = np.ones(len(lens), dtype=np.int64)
        else:
            qsl = b.query_start_loc.cpu().numpy().astype(np.int64)
            ql = qsl[1:] - qsl[:-1]
        for s in range(len(lens)):
            n, L = int(ql[s]), int(lens[s])
            pairs = n * L - n * (n - 1) // 2  # row i of n sees L - n + i + 1 keys
            units.append((bi, s, n, L, pairs))
            total_pairs += pairs
            total_rows += n
    order = np.random.Generator(np.random.PCG64(0)).permutation(len(units))
    t_used, pairs_done, seqs_done = 0.0, 0, 0
    for k in order:
        bi, s, n, L, pairs = units[int(k)]
        if n == 0:
            continue
        b = batches[bi]
        bt = b.block_tables[s:s + 1].cpu()
        nblk = -(-L // b.block_size)
        ids = bt[0, :nblk].long().to(b.k_cache.device)
        kc = b.k_cache.index_select(0, ids).cpu()
        vc = b.v_cache.index_select(0, ids).cpu()
        tbl = np.arange(nblk, dtype=np.int32)[None, :]
        if b.query_start_loc is None:
            q = opa.to_f64(b.q[s:s + 1])
        else:
            q0 = int(b.query_start_loc[s])
            q = opa.to_f64(b.q[q0:q0 + n])
        t0 = time.perf_counter()
        if b.k_scale is not None:  # FP8 cache: the oracle dequantises, then attends
            kc = opa.dequantize_cache(kc.numpy(), b.k_scale.cpu().numpy())
            vc = opa.dequantize_cache(vc.numpy(), b.v_scale.cpu().numpy())
        else:
            kc, vc = opa.to_f64(kc), opa.to_f64(vc)
        if b.query_start_loc is None:
            opa.paged_decode(q, kc, vc, tbl, np.array([L]), b.scale)
        else:
            opa.chunked_prefill(q, kc, vc, tbl, np.array([L]), np.array([0, n]), b.scale)
        t_used += time.perf_counter() - t0
        pairs_done += pairs
        seqs_done += 1
        if t_used >= budget_s:
            break
    if limiter is not None:
        limiter.unregister() if hasattr(limiter, "unregister") else None
    est_step_s = t_used * total_pairs / max(pairs_done, 1)
    value = total_rows / est_step_s
    return {"value": round(value, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "host_cores": os.cpu_count(), "blas_threads": blas_threads,
            "threads_used": "1 (the oracle runs single-threaded: BLAS pool limited to 1)",
            "sample": "%d of %d sequences of %s (%d of %d query-key pairs), oracle time %.1f s "
                      "scaled by query-key pairs to one full step"
                      % (seqs_done, len(units), "+".join(b.name for b in batches), pairs_done,
                         total_pairs, t_used)}


def run_reference(args, rank, world):
    """The oracle as the reference arm (rank 0 only)."""
    if rank != 0:
        return None
    batches = workloads.WORKLOADS[args.workload](device="cpu")
    for _ in range(args.warmup):
        cpu_baseline(batches, args, budget_s=1.0)
    vals = []
    t0 = time.perf_counter()
    last = None
    for _ in range(args.steps):
        last = cpu_baseline(batches, args, budget_s=args.ref_step_budget)
        vals.append(last["value"])
    wall = time.perf_counter() - t0
    value = statistics.mean(vals)
    rows = sum(b.num_seqs if b.query_start_loc is None else int(b.q.shape[0]) for b in batches)
    line = {
        "metric": "paged decode tokens/s (one layer) and achieved HBM GB/s of pa_decode",
        "value": round(value, 3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(rows / value * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded N(0,1) q/K/V, FIFO free-list block tables)",
        "impl": "reference",
        "config": {"workload": "+".join(x.name for x in batches), "parallelism": "replicas%d" % world},
        "cpu_baseline": {"value": round(value, 3), "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "host_cores": last["host_cores"], "blas_threads": last["blas_threads"],
                         "sample": last["sample"] + "; each step a bounded sample, %.1f s wall" % wall},
        "e2e": {"value": round(value, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    return line


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle time for cpu_baseline")
    ap.add_argument("--ref-step-budget", type=float, default=5.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-others", dest="others", action="store_false",
                    help="skip the other workloads measured beside the default one")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl == "ours":
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
    else:
        line = run_ours(args, rank, world, local)
    if rank == 0 and line is not None:
        print(json.dumps(line), flush=True)
    if world > 1 and args.impl == "ours":
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
