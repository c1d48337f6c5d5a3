"""Plain fp64 NumPy oracle (test infrastructure only; see the package header).

Sources (web pages on KV-cache paging; cited by title and section):

[P1] "大模型推理内存优化从 KV Cache 分页到连续批处理的工程实践" (seekfood.cn),
     sections "KV Cache 的内存开销与分页机制" (KV-cache memory cost and the
     paging mechanism), "PagedAttention 的 CUDA Kernel 实现" (the kernel),
     "生产级推理引擎的内存管理与调度" (block pool and scheduler),
     "工程边界与架构取舍" (trade-offs: decode reads the whole cache, chunked
     prefill).
[P2] "KV Cache管理优化：大模型推理显存瓶颈突破" (intelliparadigm), section 4.1
     (blocks shared across sequences through reference counts).

The method reaches exactly the dense attention result, only faster, so this
oracle computes the dense definition, reaching each key/value row through
the block table.  Readings taken where the pages are silent are stated at
each function.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# Sizes
# ---------------------------------------------------------------------------


def kv_cache_size_bytes(num_layers, seq_len, num_kv_heads, head_dim, dtype_size, batch_size):
    """[P1] "KV Cache 的内存开销与分页机制", KV_Cache_Size formula: one K and one
    V vector of ``num_kv_heads * head_dim`` elements per layer, token and
    sequence."""
    return 2 * num_layers * seq_len * num_kv_heads * head_dim * dtype_size * batch_size


def blocks_needed(num_tokens, block_size):
    """[P1] "生产级推理引擎的内存管理与调度", the scheduler's block count: the
    smallest number of fixed-size blocks that holds ``num_tokens`` tokens
    (integer ceiling; the operators of the printed code were lost in
    extraction and are read as ``(n + BS - 1) / BS``)."""
    return (num_tokens + block_size - 1) // block_size


# ---------------------------------------------------------------------------
# Addressing
# ---------------------------------------------------------------------------


def slot_of(table_row, pos, block_size):
    """[P1] "KV Cache 的内存开销与分页机制": a sequence's logical block ``j``
    lives in physical block ``table_row[j]``; blocks fill in token order and a
    new block is taken only when the current one is full, so token ``pos`` sits
    in logical block ``pos // block_size`` at offset ``pos % block_size``.
    A slot is ``physical_block * block_size + offset``."""
    return int(table_row[pos // block_size]) * block_size + pos % block_size


def reshape_and_cache(k, v, k_cache, v_cache, slot_mapping):
    """Scatter each new token's K and V rows into its cache slot (in place).

    ``k``, ``v``: [T, Hkv, D]; caches [num_blocks, block_size, Hkv, D]; any
    element type (the copy is bitwise, so pass raw 16-bit patterns to compare
    bit-for-bit).  A negative slot marks a padding token and is skipped
    (reading; the pages do not treat padding).  [P1] "KV Cache 的内存开销与分页
    机制": the generated token's K/V go to the next free place of the
    sequence's current block."""
    bs = k_cache.shape[1]
    for t in range(len(slot_mapping)):
        s = int(slot_mapping[t])
        if s < 0:
            continue
        b, o = s // bs, s % bs
        k_cache[b, o] = k[t]
        v_cache[b, o] = v[t]
    return k_cache, v_cache


def kv_head_of(q_head, num_q_heads, num_kv_heads):
    """GQA head mapping (reading: the pages only give the KV-head count):
    q-heads ``[g*G, (g+1)*G)`` share kv-head ``g``, ``G = Hq / Hkv``."""
    group = num_q_heads // num_kv_heads
    return q_head // group


def gather_kv(cache, table_row, seq_len, kv_head):
    """Dense [seq_len, D] fp64 rows of one sequence and kv-head, each reached
    through the block table ([P1] "PagedAttention 的 CUDA Kernel 实现": look
    up the physical block of a logical block, then read the vector inside
    it)."""
    bs = cache.shape[1]
    D = cache.shape[3]
    out = np.empty((seq_len, D), dtype=np.float64)
    for j in range(seq_len):
        out[j] = cache[int(table_row[j // bs]), j % bs, kv_head, :]
    return out


def attend(q_vec, K, V, scale):
    """softmax(scale * K q) V for one query, in fp64.  An empty key set gives
    a zero vector (reading for seq_len 0; the pages are silent)."""
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    x = scale * (K @ q_vec)
    w = np.exp(x - x.max())
    return (w / w.sum()) @ V


# ---------------------------------------------------------------------------
# The two attention passes
# ---------------------------------------------------------------------------


def paged_decode(q, k_cache, v_cache, block_tables, seq_lens, scale):
    """Single-query attention of each sequence over all of its cached tokens
    ([P1] "工程边界与架构取舍": decode emits one token per step and reads the
    whole KV cache of the sequence).  ``q`` [B, Hq, D]; returns fp64
    [B, Hq, D].  ``seq_lens`` count the token appended this step (it was
    cached by reshape_and_cache first, so it attends to itself)."""
    B, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for s in range(B):
        L = int(seq_lens[s])
        for g in range(Hkv):
            K = gather_kv(k_cache, block_tables[s], L, g)
            V = gather_kv(v_cache, block_tables[s], L, g)
            for h in range(Hq):
                if kv_head_of(h, Hq, Hkv) == g:
                    out[s, h] = attend(np.asarray(q[s, h], dtype=np.float64), K, V, scale)
    return out


def chunked_prefill(q, k_cache, v_cache, block_tables, seq_lens, query_start_loc, scale):
    """Causal attention of a chunk of queries over the paged context ([P1]
    "工程边界与架构取舍": long prompts are processed in chunks).  Sequence
    ``s`` has ``n = qsl[s+1] - qsl[s]`` queries; its chunk is the last ``n``
    positions of its ``seq_lens[s]`` tokens (all already cached), so query
    ``i`` sits at position ``L - n + i`` and sees keys ``0 .. L - n + i``
    inclusive (reading: a query attends to its own key).  ``q`` [sum n, Hq, D];
    returns fp64 of the same shape."""
    T, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    out = np.zeros((T, Hq, D), dtype=np.float64)
    for s in range(len(seq_lens)):
        L = int(seq_lens[s])
        a, b = int(query_start_loc[s]), int(query_start_loc[s + 1])
        n = b - a
        for g in range(Hkv):
            K = gather_kv(k_cache, block_tables[s], L, g)
            V = gather_kv(v_cache, block_tables[s], L, g)
            for i in range(n):
                visible = L - n + i + 1
                for h in range(Hq):
                    if kv_head_of(h, Hq, Hkv) == g:
                        out[a + i, h] = attend(np.asarray(q[a + i, h], dtype=np.float64),
                                               K[:visible], V[:visible], scale)
    return out


# ---------------------------------------------------------------------------
# Rounding to the storage type
# ---------------------------------------------------------------------------

_FORMATS = {
    # significand bits incl. the hidden one, smallest normal exponent, largest finite
    "float16": (11, -14, 65504.0),
    "bfloat16": (8, -126, float.fromhex("0x1.fep127")),
}


def round_rne(x, fmt):
    """Round fp64 values to the nearest value of ``fmt`` ("float16" or
    "bfloat16"), ties to even, directly from fp64 (no intermediate fp32).
    Values past the largest finite round to +-inf (only when the rounded
    magnitude would exceed it).  Returns fp64."""
    p, emin, fmax = _FORMATS[fmt]
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                   # x = m * 2**e, 0.5 <= |m| < 1
    # exponent of the value's leading bit is e-1; quantum 2**(e-1-(p-1)),
    # never finer than the subnormal quantum 2**(emin-(p-1))
    q_exp = np.maximum(e - p, emin - (p - 1))
    scaled = np.ldexp(x, -q_exp)         # exact (power-of-two scaling)
    r = np.ldexp(np.round(scaled), q_exp)  # np.round rounds half to even
    r = np.where(np.abs(r) > fmax, np.copysign(np.inf, x), r)
    return np.where(np.isfinite(x), r, x)


def round_to(x, torch_dtype_name):
    """``round_rne`` keyed by the torch dtype name ("float16"/"bfloat16")."""
    return round_rne(x, torch_dtype_name)


def to_f64(t):
    """fp16/bf16/fp32 torch tensor -> fp64 numpy array (exact)."""
    import torch
    return t.detach().to("cpu").to(torch.float64).numpy()
