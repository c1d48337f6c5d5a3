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


# ---------------------------------------------------------------------------
# FP8 (e4m3) KV cache
# ---------------------------------------------------------------------------
# [P1] "工程边界与架构取舍", on quantization and KV-cache precision: storing the cache in
# FP8 instead of FP16 halves its memory (at some accuracy cost on long sequences).
# The pages fix no format, scale granularity or rounding.  Readings:
#  - the e4m3 format with no infinities: 1 sign bit, 4 exponent bits (bias 7), 3
#    mantissa bits; exponent field 0 holds the subnormals 2^-6 * m/8; the largest finite
#    value is 1.75 * 2^8 = 448; codes 0x7F and 0xFF are NaN;
#  - one fp32 scale per kv-head for K and one for V: a stored code c stands for
#    value(c) * scale;
#  - quantisation computes x * (1 / scale) in fp32 (the reciprocal rounded to fp32,
#    then the product rounded to fp32), rounds to the nearest e4m3 value, ties to the
#    even code, and saturates to +-448.

E4M3_MAX = 448.0


def e4m3_value(code):
    """fp64 value of e4m3 codes (array of 0..255): (-1)^s 2^(e-7) (1 + m/8) for
    exponent field e > 0, (-1)^s 2^-6 (m/8) for e = 0; 0x7F and 0xFF are NaN."""
    c = np.asarray(code).astype(np.int64) & 0xFF
    s, e, m = (c >> 7) & 1, (c >> 3) & 0xF, c & 7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    val = np.where(s == 1, -mag, mag)
    return np.where((c & 0x7F) == 0x7F, np.nan, val)


# the 127 non-negative finite values (codes 0x00..0x7E), increasing
_E4M3_POS = e4m3_value(np.arange(0x7F))


def e4m3_round(x):
    """Nearest e4m3 code (uint8) to each fp64 value: the nearest of the finite values,
    ties to the even code (last mantissa bit 0), magnitudes past 448 saturate to 448,
    the sign kept (a negative value that rounds to zero gives 0x80); NaN gives 0x7F."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(_E4M3_POS, a, side="left"), 1, 0x7E)  # _POS[hi-1] < a <= _POS[hi]
    lo = hi - 1
    d_lo, d_hi = a - _E4M3_POS[lo], _E4M3_POS[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    mag = np.where(pick_hi, hi, lo)
    mag = np.where(a == 0, 0, mag)
    code = np.where(np.signbit(x), mag | 0x80, mag)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


def quantize_e4m3(x, scale):
    """Codes of ``x`` (fp16/bf16/fp32 values as an array) with per-kv-head ``scale``
    broadcast against it: e4m3_round(float32(x) * float32(1/float32(scale)))."""
    inv = (np.float32(1.0) / np.asarray(scale, dtype=np.float32)).astype(np.float32)
    y = (np.asarray(x, dtype=np.float32) * inv).astype(np.float32)
    return e4m3_round(y.astype(np.float64))


def reshape_and_cache_fp8(k, v, k_cache, v_cache, slot_mapping, k_scale, v_scale):
    """reshape_and_cache into uint8 e4m3 caches [N, bs, Hkv, D]: token t's rows
    k[t], v[t] ([Hkv, D], the values of the step's fp16/bf16 K/V) are quantised with
    the per-head scales (``k_scale``/``v_scale`` [Hkv]) and stored at slot
    ``slot_mapping[t]`` (negative = padding, skipped), in place."""
    bs = k_cache.shape[1]
    ks = np.asarray(k_scale, dtype=np.float32)[:, None]
    vs = np.asarray(v_scale, dtype=np.float32)[:, None]
    for t, slot in enumerate(np.asarray(slot_mapping)):
        if slot < 0:
            continue
        b, r = divmod(int(slot), bs)
        k_cache[b, r] = quantize_e4m3(k[t], ks)
        v_cache[b, r] = quantize_e4m3(v[t], vs)


def dequantize_cache(cache_codes, scale):
    """fp64 values of an e4m3 cache [N, bs, Hkv, D] with per-kv-head ``scale`` [Hkv]:
    value(code) * scale.  Attention over an FP8 cache is the attention of the oracle
    above over these values."""
    return e4m3_value(cache_codes) * np.asarray(scale, dtype=np.float64)[None, None, :, None]
