"""C-ABI checks that need no GPU: the library builds and loads, it exports every
entry point ``include/pagedattn.h`` declares, and host-side validation returns
the documented status codes before touching the device."""
import ctypes
import os
import re

import pytest

from tests._devmem import devmem

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pagedattn.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def palib():
    from paged_kv_cache_332_b200 import build
    build.build()
    import paged_kv_cache_332_b200 as pa
    return pa


def test_header_declares_the_hot_path():
    syms = declared_symbols()
    for s in ("pa_reshape_and_cache", "pa_decode", "pa_chunked_prefill", "pa_decode_workspace_size",
              "pa_get_device_error", "pa_status_string"):
        assert s in syms


def test_library_exports_every_declared_symbol(palib):
    L = ctypes.CDLL(palib.library_path)
    missing = [s for s in declared_symbols() if not hasattr(L, s)]
    assert not missing, missing
    assert sorted(palib.EXPORTED_SYMBOLS) == declared_symbols()


def test_only_pa_symbols_exported(palib):
    # hidden visibility: nothing but the C ABI leaks out of the library
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", palib.library_path], capture_output=True,
                         text=True).stdout
    names = [l.split()[-1] for l in out.splitlines() if " T " in l]
    assert names and all(n.startswith("pa_") for n in names), names


def test_status_strings(palib):
    assert palib.pa_status_string(0) == "PA_OK"
    assert palib.pa_status_string(3) == "PA_ERR_WORKSPACE_TOO_SMALL"
    assert palib.pa_status_string(99) == "PA_ERR_UNKNOWN"


def _ws_bound(B, Hq, L, P, D=128):
    """The documented upper bound: merge records (8 B per sequence and q-head, padded
    to 256 B) and partial rows of D+2 fp32: (256 + B) * Hq, plus, with an explicit
    partition, B * Hq * ceil(ceil(L/16) / (P/16)) + Hq."""
    rows = (256 + B) * Hq
    if P:
        rows += B * Hq * -(-(-(-L // 16)) // (P // 16)) + Hq
    return -(-(B * Hq * 8) // 256) * 256 + rows * (D + 2) * 4


def test_workspace_size_arithmetic(palib):
    for B, Hq, L, P in [(64, 32, 64, 0), (64, 32, 8000, 0), (64, 32, 8000, 512),
                        (32, 64, 32768, 512), (2, 8, 100, 16), (1, 1, 0, 0)]:
        assert palib.pa_decode_workspace_size(B, Hq, 128, L, P) == _ws_bound(B, Hq, L, P)
    # the balanced split needs no more scratch for longer sequences
    assert palib.pa_decode_workspace_size(64, 32, 128, 8000, 0) == \
        palib.pa_decode_workspace_size(64, 32, 128, 64, 0)
    # 16 sequences x 64 q-heads, 32768 tokens, 512-token partitions: 64 partitions each
    assert palib.pa_decode_workspace_size(16, 64, 128, 32768, 512) == \
        16 * 64 * 8 + ((256 + 16) * 64 + 16 * 64 * 64 + 64) * 130 * 4
    assert palib.pa_decode_workspace_size(0, 8, 128, 100, 16) == 0  # invalid shape
    # prefill's optional wave-tail split: <= 128 items of 2 halves x 256 rows
    per_item = 256 * (2 * 130 * 4 + 4)  # 2 halves x 256 rows of 130 fp32, 256 row ids
    assert palib.pa_chunked_prefill_workspace_size(4, 512, 64, 128, 8000) == 128 * per_item
    assert palib.pa_chunked_prefill_workspace_size(1, 32, 2, 128, 100) == 2 * per_item
    assert palib.pa_chunked_prefill_workspace_size(0, 32, 2, 128, 100) == 0


def _raw(palib):
    return palib.lib()


def test_invalid_arguments_rejected_on_host(palib):
    L = _raw(palib)
    nul = None
    # reshape_and_cache: unsupported head_dim / block_size / dtype, negative count
    assert L.pa_reshape_and_cache(nul, nul, nul, nul, nul, 4, 8, 64, 16, 16, 0, nul) == 2
    assert L.pa_reshape_and_cache(nul, nul, nul, nul, nul, 4, 8, 128, 16, 24, 0, nul) == 2
    assert L.pa_reshape_and_cache(nul, nul, nul, nul, nul, 4, 8, 128, 16, 16, 7, nul) == 2
    assert L.pa_reshape_and_cache(nul, nul, nul, nul, nul, -1, 8, 128, 16, 16, 0, nul) == 1
    assert L.pa_reshape_and_cache(nul, nul, nul, nul, nul, 4, 8, 128, 16, 16, 0, nul) == 1
    assert L.pa_reshape_and_cache(nul, nul, nul, nul, nul, 0, 8, 128, 16, 16, 0, nul) == 0
    m = devmem()
    args = dict(out=m.region(), q=m.region(), kc=m.region(), vc=m.region(), bt=m.region(), mb=8,
                sl=m.region(), B=2, Hq=8, Hkv=8, D=128, scale=0.1,
                bs=16, N=16, maxlen=100, P=0, ws=None, wsb=0, dt=0, st=None)

    def dec(**kw):
        a = dict(args); a.update(kw)
        return L.pa_decode(a["out"], a["q"], a["kc"], a["vc"], a["bt"], a["mb"], a["sl"], a["B"],
                           a["Hq"], a["Hkv"], a["D"], a["scale"], a["bs"], a["N"], a["maxlen"],
                           a["P"], a["ws"], a["wsb"], a["dt"], a["st"])
    assert dec(D=64) == 2                    # head_dim must be 128
    assert dec(bs=8) == 2                    # block size 16 or 32
    assert dec(Hq=12, Hkv=8) == 1            # Hq not a multiple of Hkv
    assert dec(Hq=24, Hkv=8) == 2            # GQA group 3 not built
    assert dec(Hq=128, Hkv=8) == 2           # GQA group 16 not built
    assert dec(P=24) == 1                    # partition not a multiple of 16
    assert dec(P=4096) == 2                  # partition above 2048 tokens
    assert dec(q=None) == 1                  # null pointer
    assert dec(q=m.region(4)) == 1           # misaligned
    assert dec(dt=3) == 2
    assert dec(B=0) == 0                     # nothing to do
    assert dec(B=5000) == 2                  # more sequences than the schedule holds
    assert dec(P=512) == 3                   # every call needs a workspace (merge records)
    assert dec(maxlen=8000, P=512, ws=m.region(), wsb=100) == 3
    assert dec(maxlen=8000, P=512, ws=m.region(16), wsb=1 << 24) == 1  # alignment
    assert palib.pa_last_launch_count() == 0


def test_append_decode_arguments_rejected_on_host(palib):
    L = _raw(palib)
    m = devmem()
    o, q, kc, vc, bt, sl = (m.region() for _ in range(6))
    kn0, vn0 = m.region(), m.region()

    def app(kn=kn0, vn=vn0, B=2, D=128, ws=None, wsb=0):
        return L.pa_decode_append(o, q, kn, vn, kc, vc, bt, 8, sl, B, 8, 8, D, 0.1, 16, 16, 100,
                                  512, ws, wsb, 0, None)
    assert app(kn=None) == 1                     # new K missing
    assert app(vn=None) == 1                     # new V missing
    assert app(kn=m.region(4)) == 1              # misaligned
    assert app(D=64) == 2                        # head_dim must be 128
    assert app(B=0) == 0                         # nothing to do
    assert app() == 3                            # needs a workspace
    assert palib.pa_last_launch_count() == 0


def test_fp8_arguments_rejected_on_host(palib):
    L = _raw(palib)
    m = devmem()
    k, v, kc, vc, sm, ks0, vs0 = (m.region() for _ in range(7))
    nul = None
    # scatter: missing scales, odd block size, bad source type
    assert L.pa_reshape_and_cache_fp8(k, v, kc, vc, sm, nul, vs0, 4, 8, 128, 16, 16, 0, nul) == 1
    assert L.pa_reshape_and_cache_fp8(k, v, kc, vc, sm, ks0, vs0, 4, 8, 128, 16, 24, 0, nul) == 2
    assert L.pa_reshape_and_cache_fp8(k, v, kc, vc, sm, ks0, vs0, 4, 8, 128, 16, 16, 7, nul) == 2
    assert L.pa_reshape_and_cache_fp8(k, v, kc, vc, sm, ks0, vs0, 0, 8, 128, 16, 16, 0, nul) == 0
    o, q, bt, sl = (m.region() for _ in range(4))

    def dec(ks=ks0, vs=vs0, B=2, ws=None, wsb=0):
        return L.pa_decode_fp8(o, q, kc, vc, ks, vs, bt, 8, sl, B, 8, 8, 128, 0.1, 16, 16, 100,
                               512, ws, wsb, 0, None)
    assert dec(ks=None) == 1 and dec(vs=None) == 1
    assert dec(B=0) == 0
    assert dec() == 3  # needs a workspace
    assert palib.pa_last_launch_count() == 0


def test_shared_prefix_arguments_rejected_on_host(palib):
    L = _raw(palib)
    m = devmem()
    o, q, kc, vc, bt, sl, gs0, pl0 = (m.region() for _ in range(8))
    nul = None

    def dec(B=8, gs=gs0, pl=pl0, ng=2, mg=4, mp=256, ws=None, wsb=0):
        return L.pa_decode_shared_prefix(o, q, kc, vc, bt, 32, sl, B, gs, pl, ng, mg, mp, 32, 8,
                                         128, 0.1, 16, 1000, 512, ws, wsb, 0, nul)
    assert dec(ng=-1) == 1 and dec(mg=-1) == 1 and dec(mp=-1) == 1
    assert dec(ng=9) == 1 and dec(mg=9) == 1       # more groups / members than sequences
    assert dec(gs=nul) == 1 and dec(pl=nul) == 1
    assert dec(B=0, ng=0, mg=0) == 0               # nothing to do
    assert dec() == 3 and dec(mp=0) == 3            # needs a workspace (shared or plain)
    base = palib.pa_decode_workspace_size(8, 32, 128, 512, 0)
    # chunk partials: (256 + num_seqs) x num_kv_heads x 16 rows of 130 fp32 after the base,
    # then the members' chunk records (num_seqs x num_kv_heads int4)
    up = lambda n: -(-n // 256) * 256  # noqa: E731
    assert palib.pa_decode_shared_prefix_workspace_size(8, 32, 8, 128, 512) == \
        up(up(base) + (256 + 8) * 8 * 16 * 130 * 4) + 8 * 8 * 16
    assert palib.pa_decode_shared_prefix_workspace_size(0, 32, 8, 128, 512) == 0
    assert palib.pa_decode_shared_prefix_workspace_size(8, 32, 0, 128, 512) == 0
    assert palib.pa_last_launch_count() == 0


def test_varlen_arguments_rejected_on_host(palib):
    L = _raw(palib)
    m = devmem()
    o, q, kc, vc, bt, sl, qsl0 = (m.region() for _ in range(7))
    nul = None

    def call(B=4, rows=10, mq=5, qsl=qsl0, ws=None, wsb=0):
        return L.pa_attention_varlen(o, q, kc, vc, bt, 32, sl, qsl, B, rows, mq, -1, 32, 8, 128,
                                     0.1, 16, 1000, 512, ws, wsb, 0, nul)
    assert call(B=-1) == 1 and call(rows=-1) == 1 and call(mq=-1) == 1
    assert call(B=0) == 0 and call(rows=0) == 0 and call(mq=0) == 0   # nothing to do
    assert call(qsl=nul) == 1
    assert call() == 3                                                  # needs a workspace
    d = palib.pa_decode_workspace_size(4, 32, 128, 512, 0)
    pf = palib.pa_chunked_prefill_workspace_size(4, 5, 32, 128, 512)
    assert palib.pa_attention_varlen_workspace_size(4, 5, 32, 128, 512) >= d + pf + 5 * 4
    assert palib.pa_last_launch_count() == 0


def test_block_pool_arguments_rejected_on_host(palib):
    L = _raw(palib)
    m = devmem()
    ring0, state, tables, owned, lens, qlens, slots0, granted, fin0 = (
        m.region() for _ in range(9))
    nul = None
    refs = m.region()
    assert L.pa_block_pool_init(ring0, state, refs, 0, nul) == 1  # empty pool
    assert L.pa_block_pool_init(nul, state, refs, 8, nul) == 1    # ring missing

    def alloc(ring=ring0, n=64, mb=8, B=4, bs=16, slots=slots0):
        return L.pa_block_allocate(ring, state, refs, n, tables, mb, owned, lens, qlens, B, bs,
                                   slots, granted, nul)
    assert alloc(n=0) == 1 and alloc(mb=0) == 1 and alloc(B=-1) == 1
    assert alloc(bs=8) == 2                                  # block size 16 or 32
    assert alloc(B=4097) == 2                                # one CTA's limit
    assert alloc(B=0) == 0                                   # nothing to do
    assert alloc(ring=nul) == 1 and alloc(slots=nul) == 1

    def free(n=64, B=4, fin=fin0):
        return L.pa_block_free(ring0, state, refs, n, tables, 8, owned, fin, B, nul)
    assert free(n=0) == 1 and free(B=4097) == 2 and free(B=0) == 0 and free(fin=nul) == 1
    src, dst, k = m.region(), m.region(), m.region()

    def share(rf=refs, n=64, B=4, pairs=2, s_=src):
        return L.pa_block_share(rf, n, tables, 8, owned, B, s_, dst, k, pairs, nul)
    assert share(rf=nul) == 1                                # shares need reference counts
    assert share(n=0) == 1 and share(B=-1) == 1 and share(pairs=-1) == 1
    assert share(pairs=0) == 0 and share(s_=nul) == 1
    assert palib.pa_last_launch_count() == 0


def test_product_package_does_not_touch_oracle():
    # the product path never imports the oracle
    pkg = os.path.join(ROOT, "paged_kv_cache_332_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".c", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "dense_attention" not in text, f
