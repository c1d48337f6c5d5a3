"""Pins for the fp64 oracle, against things other than the oracle itself.

Each ``check_*`` function raises AssertionError when the oracle is wrong.
The checks use closed forms, the page's worked example (``tests/golden/``),
invariants the paging design guarantees, and two independent brute-force
implementations (a plain-C dense attention and pure-Python loops).  The
mutation tests at the end plant plausible mistakes in the oracle (on the
CPU) and require at least one check to catch each.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import oracle.paged_attention as opa
from tests import _dense_c
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# checks
# ---------------------------------------------------------------------------

def check_kv_size():
    g = _golden("kv_size_worked_example.json")
    per = opa.kv_cache_size_bytes(g["num_layers"], g["seq_len"], g["num_kv_heads"],
                                  g["head_dim"], g["dtype_bytes"], 1)
    assert "%.2f" % (per / 1e9) == g["printed_per_request_GB"]
    batch = opa.kv_cache_size_bytes(g["num_layers"], g["seq_len"], g["num_kv_heads"],
                                    g["head_dim"], g["dtype_bytes"], g["printed_batch"])
    assert "%.1f" % (math.floor(batch / 1e8) / 10) == g["printed_batch_GB"]
    # exact integer value: 2 * 80 * 4096 * 8 * 128 * 2
    assert per == 1_342_177_280
    assert batch == 16 * per


def check_block_counts():
    g = _golden("block_counts.json")
    for n, b in zip(g["tokens"], g["blocks"]):
        assert opa.blocks_needed(n, g["block_size"]) == b, (n, b)
    # defining property of the count: enough blocks, and no spare whole block
    for bs in (16, 32):
        for n in range(1, 1200):
            k = opa.blocks_needed(n, bs)
            assert k * bs >= n and (k - 1) * bs < n
        assert opa.blocks_needed(0, bs) == 0


def check_slots():
    rng = np.random.default_rng(0)
    for bs in (16, 32):
        table = rng.permutation(40)[:10]
        seen = set()
        for pos in range(10 * bs):
            s = opa.slot_of(table, pos, bs)
            lo = int(table[pos // bs]) * bs
            assert lo <= s < lo + bs
            if pos % bs:
                assert s == opa.slot_of(table, pos - 1, bs) + 1
            seen.add(s)
        assert len(seen) == 10 * bs


def check_reshape_and_cache():
    rng = np.random.default_rng(1)
    N, bs, H, D = 6, 16, 2, 8
    kc = np.full((N, bs, H, D), 0xABCD, dtype=np.uint16)
    vc = np.full((N, bs, H, D), 0x1234, dtype=np.uint16)
    T = 9
    slots = rng.choice(N * bs, size=T, replace=False).astype(np.int32)
    slots[3] = -1
    k = rng.integers(0, 0x7C00, size=(T, H, D), dtype=np.uint16)
    v = rng.integers(0, 0x7C00, size=(T, H, D), dtype=np.uint16)
    opa.reshape_and_cache(k, v, kc, vc, slots)
    written = set()
    for t, s in enumerate(slots):
        if s < 0:
            continue
        written.add(int(s))
        assert np.array_equal(kc.reshape(N * bs, H, D)[s], k[t])
        assert np.array_equal(vc.reshape(N * bs, H, D)[s], v[t])
    for s in range(N * bs):
        if s not in written:
            assert np.all(kc.reshape(N * bs, H, D)[s] == 0xABCD)
            assert np.all(vc.reshape(N * bs, H, D)[s] == 0x1234)


def check_softmax_special_cases():
    rng = np.random.default_rng(2)
    D = 16
    s = 1 / math.sqrt(D)
    # L = 1: the only value row, exactly
    q, K, V = rng.normal(size=D), rng.normal(size=(1, D)), rng.normal(size=(1, D))
    assert np.array_equal(opa.attend(q, K, V, s), V[0])
    # q = 0 (all logits equal): mean of V
    K, V = rng.normal(size=(7, D)), rng.normal(size=(7, D))
    assert np.allclose(opa.attend(np.zeros(D), K, V, s), V.mean(0), atol=1e-14)
    # all keys equal: mean of V
    Kc = np.repeat(rng.normal(size=(1, D)), 7, 0)
    assert np.allclose(opa.attend(q, Kc, V, s), V.mean(0), atol=1e-14)
    # one logit 60 above the rest: that row (to ~e^-60)
    qu = np.zeros(D); qu[0] = 1.0
    Kd = np.zeros((7, D)); Kd[4, 0] = 60.0 / s
    assert np.allclose(opa.attend(qu, Kd, V, s), V[4], atol=1e-20)
    # L = 2: o = v0 + (v1 - v0) * logistic(s * q.(k1 - k0)), worked by hand
    K2, V2 = rng.normal(size=(2, D)), rng.normal(size=(2, D))
    t = s * float(q @ (K2[1] - K2[0]))
    want = V2[0] + (V2[1] - V2[0]) / (1.0 + math.exp(-t))
    assert np.allclose(opa.attend(q, K2, V2, s), want, rtol=0, atol=1e-13)
    # shifting every logit by the same amount changes nothing
    c = 3.7
    Ks = K + c * q / (s * float(q @ q))
    assert np.allclose(opa.attend(q, Ks, V, s), opa.attend(q, K, V, s), atol=1e-12)
    # empty key set: zeros (reading for seq_len 0)
    assert np.array_equal(opa.attend(q, np.zeros((0, D)), np.zeros((0, D)), s), np.zeros(D))


def _tiny_paged(rng, B=3, Hq=4, Hkv=2, D=16, bs=4, lens=(1, 7, 13), N=12, ident=False):
    nblk = [opa.blocks_needed(L, bs) for L in lens]
    M = max(nblk)
    if ident:
        tables = np.zeros((B, M), dtype=np.int32)
        off = 0
        for b in range(B):
            tables[b, :nblk[b]] = np.arange(off, off + nblk[b])
            off += nblk[b]
        N = off
    else:
        perm = rng.permutation(N)
        tables = np.zeros((B, M), dtype=np.int32)
        off = 0
        for b in range(B):
            tables[b, :nblk[b]] = perm[off:off + nblk[b]]
            off += nblk[b]
    kc = rng.normal(size=(N, bs, Hkv, D))
    vc = rng.normal(size=(N, bs, Hkv, D))
    q = rng.normal(size=(B, Hq, D))
    return q, kc, vc, tables, np.array(lens, dtype=np.int32)


def _contig(cache, b_first, L, g):
    """Rows of a contiguous (identity-table) layout, read without any table."""
    bs = cache.shape[1]
    flat = cache.reshape(-1, cache.shape[2], cache.shape[3])
    return flat[b_first * bs: b_first * bs + L, g, :]


def check_identity_table_vs_bruteforce():
    rng = np.random.default_rng(3)
    q, kc, vc, tables, lens = _tiny_paged(rng, ident=True)
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    G = Hq // Hkv
    s = 0.25
    got = opa.paged_decode(q, kc, vc, tables, lens, s)
    for b in range(B):
        for h in range(Hq):
            K = _contig(kc, int(tables[b, 0]), int(lens[b]), h // G)
            V = _contig(vc, int(tables[b, 0]), int(lens[b]), h // G)
            c_ref = _dense_c.dense_attention(q[b, h], K, V, s)
            # pure-Python loops, a third formulation
            logits = [s * sum(q[b, h, d] * K[j, d] for d in range(D)) for j in range(len(K))]
            mx = max(logits)
            w = [math.exp(x - mx) for x in logits]
            py = [sum(w[j] * V[j, d] for j in range(len(K))) / sum(w) for d in range(D)]
            assert np.allclose(got[b, h], c_ref, rtol=0, atol=1e-12)
            assert np.allclose(got[b, h], py, rtol=0, atol=1e-12)


def check_placement_invariance():
    rng = np.random.default_rng(4)
    q, kc, vc, tables, lens = _tiny_paged(rng)
    ref = opa.paged_decode(q, kc, vc, tables, lens, 0.3)
    N = kc.shape[0]
    perm = rng.permutation(N)          # old -> new
    inv = np.argsort(perm)
    got = opa.paged_decode(q, kc[inv], vc[inv], perm[tables], lens, 0.3)
    assert np.allclose(got, ref, rtol=0, atol=1e-13)


def check_gqa_mapping():
    rng = np.random.default_rng(5)
    q, kc, vc, tables, lens = _tiny_paged(rng, Hq=8, Hkv=4)
    for g in range(4):
        vc[:, :, g, :] = g + 1.0
    out = opa.paged_decode(q, kc, vc, tables, lens, 0.2)
    for h in range(8):
        assert np.allclose(out[:, h, :], h // 2 + 1.0, atol=1e-13)


def check_sharing_equals_private():
    b = workloads.shared_prefix(block_size=16, scale=1 / 64, groups=2, n=3)[0]
    p = workloads.private_copy(b)
    assert not torch.equal(b.block_tables, p.block_tables)
    args = lambda x: (opa.to_f64(x.q), opa.to_f64(x.k_cache), opa.to_f64(x.v_cache),
                      x.block_tables.numpy(), x.seq_lens.numpy(), x.scale)
    assert np.array_equal(opa.paged_decode(*args(b)), opa.paged_decode(*args(p)))


def check_prefill_bruteforce():
    rng = np.random.default_rng(6)
    bs, Hq, Hkv, D = 4, 4, 2, 16
    lens, qlens = [9, 5, 12], [4, 5, 1]
    q0, kc, vc, tables, L = _tiny_paged(rng, Hq=Hq, Hkv=Hkv, D=D, bs=bs, lens=lens, ident=True)
    qsl = np.concatenate([[0], np.cumsum(qlens)]).astype(np.int32)
    q = rng.normal(size=(qsl[-1], Hq, D))
    s = 0.3
    got = opa.chunked_prefill(q, kc, vc, tables, L, qsl, s)
    for b in range(3):
        for h in range(Hq):
            K = _contig(kc, int(tables[b, 0]), lens[b], h // (Hq // Hkv))
            V = _contig(vc, int(tables[b, 0]), lens[b], h // (Hq // Hkv))
            ref = _dense_c.dense_causal_chunk(q[qsl[b]:qsl[b + 1], h], K, V, s)
            assert np.allclose(got[qsl[b]:qsl[b + 1], h], ref, rtol=0, atol=1e-12)


def check_prefill_causal_boundary():
    """A dominant key at the query's own position is seen; one just after
    it is not."""
    bs, D = 4, 8
    L, n = 10, 4
    kc = np.zeros((3, bs, 1, D)); vc = np.zeros((3, bs, 1, D))
    tables = np.array([[2, 0, 1]], dtype=np.int32)
    for j in range(L):
        vc[tables[0, j // bs], j % bs, 0, :] = j        # V row j == j
    q = np.zeros((n, 1, D)); q[:, 0, 0] = 1.0
    qsl = np.array([0, n], dtype=np.int32)
    for i in range(n):
        own = L - n + i
        k2 = kc.copy()
        k2[tables[0, own // bs], own % bs, 0, 0] = 200.0
        out = opa.chunked_prefill(q, k2, vc, tables, np.array([L]), qsl, 1.0)
        assert np.allclose(out[i, 0], own, atol=1e-9)
        if i + 1 < n:
            nxt = own + 1
            k3 = kc.copy()
            k3[tables[0, nxt // bs], nxt % bs, 0, 0] = 200.0
            out = opa.chunked_prefill(q, k3, vc, tables, np.array([L]), qsl, 1.0)
            # key nxt is invisible to query i: uniform over keys 0..own
            assert np.allclose(out[i, 0], own / 2.0, atol=1e-9)


def check_rounding():
    rng = np.random.default_rng(7)
    # fp16: numpy's own double -> half conversion (round to nearest even)
    x = np.concatenate([rng.normal(size=20000) * 10.0 ** rng.integers(-8, 5, size=20000),
                        rng.uniform(-7e-8, 7e-8, size=2000)])
    assert np.array_equal(opa.round_rne(x, "float16"), x.astype(np.float16).astype(np.float64))
    # bf16: torch's fp32 -> bf16 conversion, on fp32-representable inputs
    x32 = (rng.normal(size=20000) * 10.0 ** rng.integers(-30, 30, size=20000)).astype(np.float32)
    want = torch.from_numpy(x32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(opa.round_rne(x32.astype(np.float64), "bfloat16"), want)
    # ties to even, worked by hand
    assert opa.round_rne(1 + 2 ** -8, "bfloat16") == 1.0
    assert opa.round_rne(1 + 3 * 2 ** -8, "bfloat16") == 1 + 2 ** -6
    assert opa.round_rne(2049.0, "float16") == 2048.0
    assert opa.round_rne(2051.0, "float16") == 2052.0
    assert opa.round_rne(65519.0, "float16") == 65504.0
    assert np.isinf(opa.round_rne(65520.0, "float16"))
    # a value just above a tie must round up (no double rounding through fp32)
    assert opa.round_rne(1 + 2 ** -8 + 2 ** -40, "bfloat16") == 1 + 2 ** -7


CHECKS = [check_kv_size, check_block_counts, check_slots, check_reshape_and_cache,
          check_softmax_special_cases, check_identity_table_vs_bruteforce,
          check_placement_invariance, check_gqa_mapping, check_sharing_equals_private,
          check_prefill_bruteforce, check_prefill_causal_boundary, check_rounding]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_pin(check):
    check()


# ---------------------------------------------------------------------------
# mutation tests: plant a mistake in the oracle, require a check to fail
# ---------------------------------------------------------------------------

def _attend_no_scale(q, K, V, scale):
    return MUT_ORIG["attend"](q, K, V, 1.0)


def _attend_wrong_sign(q, K, V, scale):
    return MUT_ORIG["attend"](q, K, V, -scale)


def _attend_unnormalized(q, K, V, scale):
    if K.shape[0] == 0:
        return np.zeros(V.shape[1])
    x = scale * (K @ q)
    return np.exp(x - x.max()) @ V


def _head_mod(q_head, num_q_heads, num_kv_heads):
    return q_head % num_kv_heads


def _gather_swapped(cache, table_row, seq_len, kv_head):
    bs = cache.shape[1]
    out = np.empty((seq_len, cache.shape[3]))
    for j in range(seq_len):
        out[j] = cache[int(table_row[j % bs]) if j % bs < len(table_row) else 0, j // bs % bs, kv_head]
    return out


def _gather_untabled(cache, table_row, seq_len, kv_head):
    bs = cache.shape[1]
    flat = cache.reshape(-1, cache.shape[2], cache.shape[3])
    return np.array(flat[:seq_len, kv_head, :], dtype=np.float64)


def _gather_drop_last(cache, table_row, seq_len, kv_head):
    return MUT_ORIG["gather_kv"](cache, table_row, max(seq_len - 1, 0), kv_head)


def _blocks_floor(n, bs):
    return n // bs


def _prefill_exclusive(q, k_cache, v_cache, block_tables, seq_lens, query_start_loc, scale):
    # query i sees keys 0 .. L-n+i-1 (its own key dropped)
    T, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    out = np.zeros((T, Hq, D))
    for s in range(len(seq_lens)):
        L = int(seq_lens[s]); a, b = int(query_start_loc[s]), int(query_start_loc[s + 1]); n = b - a
        for g in range(Hkv):
            K = opa.gather_kv(k_cache, block_tables[s], L, g)
            V = opa.gather_kv(v_cache, block_tables[s], L, g)
            for i in range(n):
                for h in range(Hq):
                    if opa.kv_head_of(h, Hq, Hkv) == g:
                        out[a + i, h] = opa.attend(q[a + i, h], K[:L - n + i], V[:L - n + i], scale)
    return out


def _round_floor(x, fmt):
    p, emin, fmax = opa._FORMATS[fmt]
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)
    q_exp = np.maximum(e - p, emin - (p - 1))
    return np.ldexp(np.floor(np.ldexp(x, -q_exp)), q_exp)


def _kv_size_one_kv(num_layers, seq_len, num_kv_heads, head_dim, dtype_size, batch_size):
    return num_layers * seq_len * num_kv_heads * head_dim * dtype_size * batch_size


MUT_ORIG = {n: getattr(opa, n) for n in ("attend", "gather_kv", "kv_head_of", "blocks_needed",
                                          "chunked_prefill", "round_rne", "kv_cache_size_bytes")}

MUTATIONS = {
    "attend_no_scale": ("attend", _attend_no_scale),
    "attend_wrong_sign": ("attend", _attend_wrong_sign),
    "attend_unnormalized": ("attend", _attend_unnormalized),
    "gqa_modulo": ("kv_head_of", _head_mod),
    "gather_swapped_index": ("gather_kv", _gather_swapped),
    "gather_ignores_table": ("gather_kv", _gather_untabled),
    "gather_drops_last": ("gather_kv", _gather_drop_last),
    "blocks_floor": ("blocks_needed", _blocks_floor),
    "prefill_exclusive": ("chunked_prefill", _prefill_exclusive),
    "round_floor": ("round_rne", _round_floor),
    "kv_size_single": ("kv_cache_size_bytes", _kv_size_one_kv),
}


@pytest.mark.parametrize("mutation", sorted(MUTATIONS))
def test_mutation_is_caught(mutation, monkeypatch):
    name, fn = MUTATIONS[mutation]
    monkeypatch.setattr(opa, name, fn)
    caught = []
    for check in CHECKS:
        try:
            check()
        except Exception:
            caught.append(check.__name__)
    assert caught, "planted mistake %s passed every pin" % mutation
