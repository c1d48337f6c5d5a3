"""Python binding for libpagedattn (PagedAttention hot path on B200).

A thin ctypes layer over the C ABI declared in ``include/pagedattn.h``: each
function here has the name of the C entry point it calls, takes torch tensors
(device memory, contiguous, the layouts of the header), passes their pointers
and sizes, and raises :class:`PagedAttnError` on a non-OK status.  All
computation happens in the CUDA kernels of ``libpagedattn.so``; there is no
fallback, and importing this package fails loudly when the library is missing.

Build the library with ``python -m paged_kv_cache_332_b200.build``.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "PagedAttnError", "lib", "library_path", "pa_status_string", "pa_reshape_and_cache",
    "pa_decode_workspace_size", "pa_decode", "pa_decode_append", "pa_decode_noalloc",
    "pa_reshape_and_cache_fp8", "pa_decode_fp8", "pa_block_pool_init", "pa_block_allocate",
    "pa_block_free", "pa_block_share", "pa_decode_shared_prefix_workspace_size", "pa_decode_shared_prefix",
    "pa_attention_varlen_workspace_size", "pa_attention_varlen",
    "pa_decode_noalloc_scratch_bytes",
    "pa_chunked_prefill_workspace_size",
    "pa_chunked_prefill", "pa_get_device_error", "pa_last_launch_count",
    "pa_testing_wait_fault", "EXPORTED_SYMBOLS",
    "PA_DEVERR",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libpagedattn.so")

PA_OK = 0
PA_F16, PA_BF16 = 0, 1
PA_DEVERR = {"SLOT_RANGE": 0x1, "BLOCK_RANGE": 0x2, "SEQ_TOO_LONG": 0x4, "QUERY_LAYOUT": 0x8,
             "TIMEOUT": 0x10, "POOL": 0x20, "PREFIX": 0x40}

# (name, restype, argtypes) of every entry point declared in include/pagedattn.h
_vp, _i32, _sz, _f = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
_SIGS = [
    ("pa_status_string", ctypes.c_char_p, [_i32]),
    ("pa_reshape_and_cache", _i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp]),
    ("pa_decode_workspace_size", _sz, [_i32, _i32, _i32, _i32, _i32]),
    ("pa_decode", _i32, [_vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _f, _i32, _i32,
                         _i32, _i32, _vp, _sz, _i32, _vp]),
    ("pa_decode_append", _i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32,
                                _f, _i32, _i32, _i32, _i32, _vp, _sz, _i32, _vp]),
    ("pa_reshape_and_cache_fp8", _i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32,
                                        _i32, _i32, _vp]),
    ("pa_decode_fp8", _i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32,
                             _f, _i32, _i32, _i32, _i32, _vp, _sz, _i32, _vp]),
    ("pa_block_pool_init", _i32, [_vp, _vp, _vp, _i32, _vp]),
    ("pa_block_allocate", _i32, [_vp, _vp, _vp, _i32, _vp, _i32, _vp, _vp, _vp, _i32, _i32, _vp,
                                 _vp, _vp]),
    ("pa_block_free", _i32, [_vp, _vp, _vp, _i32, _vp, _i32, _vp, _vp, _i32, _vp]),
    ("pa_block_share", _i32, [_vp, _i32, _vp, _i32, _vp, _i32, _vp, _vp, _vp, _i32, _vp]),
    ("pa_decode_shared_prefix_workspace_size", _sz, [_i32, _i32, _i32, _i32, _i32]),
    ("pa_attention_varlen_workspace_size", _sz, [_i32, _i32, _i32, _i32, _i32]),
    ("pa_attention_varlen", _i32, [_vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32,
                                   _i32, _i32, _i32, _i32, _f, _i32, _i32, _i32, _vp, _sz, _i32,
                                   _vp]),
    ("pa_decode_shared_prefix", _i32, [_vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _vp, _vp, _i32,
                                       _i32, _i32, _i32, _i32, _i32, _f, _i32, _i32, _i32, _vp,
                                       _sz, _i32, _vp]),
    ("pa_decode_noalloc", _i32, [_vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _f,
                                 _i32, _i32, _i32, _i32, _i32, _vp]),
    ("pa_decode_noalloc_scratch_bytes", _sz, []),
    ("pa_chunked_prefill_workspace_size", _sz, [_i32, _i32, _i32, _i32, _i32]),
    ("pa_chunked_prefill", _i32, [_vp, _vp, _vp, _vp, _vp, _i32, _vp, _vp, _i32, _i32, _i32, _i32,
                                  _i32, _f, _i32, _i32, _i32, _vp, _sz, _i32, _vp]),
    ("pa_get_device_error", _i32, [_vp, ctypes.POINTER(ctypes.c_int32)]),
    ("pa_last_launch_count", _i32, []),
    ("pa_testing_wait_fault", _i32, [_i32, ctypes.c_longlong]),
]
EXPORTED_SYMBOLS = [n for n, _, _ in _SIGS]

_lib = None


class PagedAttnError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__("%s: %s" % (what, pa_status_string(status)))


def lib():
    """The loaded ``libpagedattn.so`` (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise ImportError("libpagedattn.so not built: run `python -m paged_kv_cache_332_b200.build`"
                              " (no CPU fallback exists)")
        L = ctypes.CDLL(library_path)
        for name, res, args in _SIGS:
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def pa_status_string(status: int) -> str:
    return lib().pa_status_string(int(status)).decode()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return PA_F16
    if t.dtype == torch.bfloat16:
        return PA_BF16
    raise TypeError("libpagedattn takes float16 or bfloat16 tensors, got %s" % t.dtype)


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libpagedattn takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libpagedattn takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _i32tensor(t, what):
    if t.dtype != torch.int32:
        raise TypeError("%s must be int32" % what)
    return _ptr(t)


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(status, what):
    if status != PA_OK:
        raise PagedAttnError(status, what)


def pa_reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, stream=None):
    """Scatter ``k``/``v`` [T, Hkv, D] into ``k_cache``/``v_cache``
    [N, bs, Hkv, D] at ``slot_mapping`` (int32 [T], negative = skip)."""
    N, bs, Hkv, D = k_cache.shape
    T = k.shape[0]
    _check(lib().pa_reshape_and_cache(_ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache),
                                      _i32tensor(slot_mapping, "slot_mapping"), T, Hkv, D, N, bs,
                                      _dtype_code(k_cache), _stream(stream)),
           "pa_reshape_and_cache")


def pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_seq_len, partition_size=0):
    return int(lib().pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_seq_len,
                                              partition_size))


def pa_decode(out, q, k_cache, v_cache, block_tables, seq_lens, scale, max_seq_len,
              partition_size=0, workspace=None, stream=None):
    """Paged single-query attention.  ``q``/``out`` [B, Hq, D]; ``block_tables``
    int32 [B, max_blocks]; ``seq_lens`` int32 [B]; ``workspace`` a device
    tensor of at least :func:`pa_decode_workspace_size` bytes (256-byte
    aligned, as torch's allocator returns)."""
    N, bs, Hkv, D = k_cache.shape
    B, Hq, _ = q.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().pa_decode(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                           _i32tensor(block_tables, "block_tables"), block_tables.shape[1],
                           _i32tensor(seq_lens, "seq_lens"), B, Hq, Hkv, D, float(scale), bs, N,
                           int(max_seq_len), int(partition_size), _ptr(workspace), ws_bytes,
                           _dtype_code(k_cache), _stream(stream)),
           "pa_decode")


def pa_decode_append(out, q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens, scale,
                     max_seq_len, partition_size=0, workspace=None, stream=None):
    """pa_decode with each sequence's new token (``k_new``/``v_new`` [B, Hkv, D])
    written into its cache slot (position seq_len-1 through the table) in the same
    launch; equals pa_reshape_and_cache followed by pa_decode."""
    N, bs, Hkv, D = k_cache.shape
    B, Hq, _ = q.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().pa_decode_append(_ptr(out), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                  _ptr(v_cache), _i32tensor(block_tables, "block_tables"),
                                  block_tables.shape[1], _i32tensor(seq_lens, "seq_lens"), B, Hq,
                                  Hkv, D, float(scale), bs, N, int(max_seq_len),
                                  int(partition_size), _ptr(workspace), ws_bytes,
                                  _dtype_code(k_cache), _stream(stream)),
           "pa_decode_append")


def _f32tensor(t, what):
    if t.dtype != torch.float32:
        raise TypeError("%s must be float32" % what)
    return _ptr(t)


def _u8cache(t, what):
    if t.dtype != torch.uint8:
        raise TypeError("%s must be a uint8 (e4m3 code) tensor" % what)
    return _ptr(t)


def pa_reshape_and_cache_fp8(k, v, k_cache, v_cache, slot_mapping, k_scale, v_scale,
                             stream=None):
    """Quantise ``k``/``v`` [T, Hkv, D] (fp16/bf16) to e4m3 codes with the per-kv-head
    fp32 scales and scatter them into the uint8 caches [N, bs, Hkv, D]."""
    N, bs, Hkv, D = k_cache.shape
    _check(lib().pa_reshape_and_cache_fp8(_ptr(k), _ptr(v), _u8cache(k_cache, "k_cache"),
                                          _u8cache(v_cache, "v_cache"),
                                          _i32tensor(slot_mapping, "slot_mapping"),
                                          _f32tensor(k_scale, "k_scale"),
                                          _f32tensor(v_scale, "v_scale"), k.shape[0], Hkv, D, N,
                                          bs, _dtype_code(k), _stream(stream)),
           "pa_reshape_and_cache_fp8")


def pa_decode_fp8(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, seq_lens, scale,
                  max_seq_len, partition_size=0, workspace=None, stream=None):
    """pa_decode over uint8 e4m3 caches with per-kv-head fp32 scales; ``q``/``out``
    fp16/bf16 [B, Hq, D]."""
    N, bs, Hkv, D = k_cache.shape
    B, Hq, _ = q.shape
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().pa_decode_fp8(_ptr(out), _ptr(q), _u8cache(k_cache, "k_cache"),
                               _u8cache(v_cache, "v_cache"), _f32tensor(k_scale, "k_scale"),
                               _f32tensor(v_scale, "v_scale"),
                               _i32tensor(block_tables, "block_tables"), block_tables.shape[1],
                               _i32tensor(seq_lens, "seq_lens"), B, Hq, Hkv, D, float(scale), bs,
                               N, int(max_seq_len), int(partition_size), _ptr(workspace),
                               ws_bytes, _dtype_code(q), _stream(stream)),
           "pa_decode_fp8")


def pa_block_pool_init(ring, state, block_refs=None, stream=None):
    """Fill the device ring (int32 [N]) with 0..N-1, state (int32 [2]) with {0, N} and
    ``block_refs`` (int32 [N], optional) with zeros."""
    _check(lib().pa_block_pool_init(_i32tensor(ring, "ring"), _i32tensor(state, "state"),
                                    _opt_i32(block_refs, "block_refs", ring.numel()),
                                    ring.numel(), _stream(stream)), "pa_block_pool_init")


def _opt_i32(t, what, n):
    if t is None:
        return None
    if t.numel() != n:
        raise ValueError("%s needs %d entries" % (what, n))
    return _i32tensor(t, what)


def pa_block_allocate(ring, state, block_tables, blocks_owned, seq_lens, q_lens, block_size,
                      slot_mapping, granted, block_refs=None, stream=None):
    """One step of appends on the device pool: grows ``block_tables``/``blocks_owned`` in
    place and writes ``slot_mapping`` (int32 [sum q_lens]) and ``granted`` (int32 [B]);
    every block handed out gets one reference in ``block_refs`` (optional)."""
    _check(lib().pa_block_allocate(_i32tensor(ring, "ring"), _i32tensor(state, "state"),
                                   _opt_i32(block_refs, "block_refs", ring.numel()),
                                   ring.numel(), _i32tensor(block_tables, "block_tables"),
                                   block_tables.shape[1], _i32tensor(blocks_owned, "blocks_owned"),
                                   _i32tensor(seq_lens, "seq_lens"), _i32tensor(q_lens, "q_lens"),
                                   seq_lens.numel(), int(block_size),
                                   _i32tensor(slot_mapping, "slot_mapping"),
                                   _i32tensor(granted, "granted"), _stream(stream)),
           "pa_block_allocate")


def pa_block_free(ring, state, block_tables, blocks_owned, finished, block_refs=None,
                  stream=None):
    """Release the blocks of every sequence with ``finished[s] != 0`` (int32 [B]): each
    goes to the back of the device ring, or, with ``block_refs``, when its last reference
    is released."""
    _check(lib().pa_block_free(_i32tensor(ring, "ring"), _i32tensor(state, "state"),
                               _opt_i32(block_refs, "block_refs", ring.numel()),
                               ring.numel(), _i32tensor(block_tables, "block_tables"),
                               block_tables.shape[1], _i32tensor(blocks_owned, "blocks_owned"),
                               _i32tensor(finished, "finished"), finished.numel(),
                               _stream(stream)),
           "pa_block_free")


def pa_block_share(block_refs, block_tables, blocks_owned, src_seqs, dst_seqs, num_shared,
                   stream=None):
    """Sequence ``dst_seqs[i]`` (owning no block) takes the first ``num_shared[i]`` blocks
    of sequence ``src_seqs[i]``'s table, one more reference each (int32 [pairs] arrays)."""
    n = src_seqs.numel()
    if dst_seqs.numel() != n or num_shared.numel() != n:
        raise ValueError("src_seqs, dst_seqs and num_shared need one entry per pair")
    _check(lib().pa_block_share(_i32tensor(block_refs, "block_refs"), block_refs.numel(),
                                _i32tensor(block_tables, "block_tables"), block_tables.shape[1],
                                _i32tensor(blocks_owned, "blocks_owned"), blocks_owned.numel(),
                                _i32tensor(src_seqs, "src_seqs"), _i32tensor(dst_seqs, "dst_seqs"),
                                _i32tensor(num_shared, "num_shared"), n, _stream(stream)),
           "pa_block_share")


def pa_decode_shared_prefix_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                           max_seq_len):
    return int(lib().pa_decode_shared_prefix_workspace_size(num_seqs, num_q_heads, num_kv_heads,
                                                            head_dim, max_seq_len))


def pa_decode_shared_prefix(out, q, k_cache, v_cache, block_tables, seq_lens, group_starts,
                            prefix_lens, scale, max_seq_len, max_group_size, max_prefix_len,
                            workspace=None, stream=None):
    """pa_decode for groups of sequences sharing a prefix: ``group_starts`` int32
    [G+1] (group g = sequences group_starts[g] .. group_starts[g+1]-1), ``prefix_lens``
    int32 [G] (shared tokens, multiples of the block size); ``workspace`` at least
    :func:`pa_decode_shared_prefix_workspace_size` bytes."""
    N, bs, Hkv, D = k_cache.shape
    B, Hq, _ = q.shape
    if group_starts.numel() != prefix_lens.numel() + 1:
        raise ValueError("group_starts needs one more entry than prefix_lens")
    if seq_lens.numel() != B or block_tables.shape[0] != B:
        raise ValueError("q, seq_lens and block_tables disagree on the number of sequences")
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().pa_decode_shared_prefix(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _i32tensor(block_tables, "block_tables"),
        block_tables.shape[1], _i32tensor(seq_lens, "seq_lens"), B,
        _i32tensor(group_starts, "group_starts"), _i32tensor(prefix_lens, "prefix_lens"),
        prefix_lens.numel(), int(max_group_size), int(max_prefix_len), Hq, Hkv, D, float(scale),
        bs, N, int(max_seq_len), _ptr(workspace), ws_bytes, _dtype_code(k_cache), _stream(stream)),
        "pa_decode_shared_prefix")


def pa_attention_varlen_workspace_size(num_seqs, max_query_len, num_q_heads, head_dim,
                                       max_seq_len):
    return int(lib().pa_attention_varlen_workspace_size(num_seqs, max_query_len, num_q_heads,
                                                        head_dim, max_seq_len))


def pa_attention_varlen(out, q, k_cache, v_cache, block_tables, seq_lens, query_start_loc, scale,
                        max_query_len, max_seq_len, workspace=None, stream=None,
                        max_chunk_seqs=-1):
    """A mixed step: rows of one query (decode) on the decode kernel, chunks on the
    prefill kernel.  ``q``/``out`` [rows, Hq, D]; ``query_start_loc`` int32 [B+1];
    ``max_chunk_seqs`` a bound on the sequences with more than one row (-1: B);
    ``workspace`` at least :func:`pa_attention_varlen_workspace_size` bytes."""
    N, bs, Hkv, D = k_cache.shape
    rows, Hq, _ = q.shape
    B = seq_lens.numel()
    if query_start_loc.numel() != B + 1 or block_tables.shape[0] != B:
        raise ValueError("query_start_loc needs B + 1 entries and block_tables B rows")
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().pa_attention_varlen(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _i32tensor(block_tables, "block_tables"),
        block_tables.shape[1], _i32tensor(seq_lens, "seq_lens"),
        _i32tensor(query_start_loc, "query_start_loc"), B, rows, int(max_query_len),
        int(max_chunk_seqs), Hq, Hkv, D,
        float(scale), bs, N, int(max_seq_len), _ptr(workspace), ws_bytes, _dtype_code(k_cache),
        _stream(stream)), "pa_attention_varlen")


def pa_decode_noalloc(out, q, k_cache, v_cache, block_tables, seq_lens, scale, max_seq_len,
                      partition_size=0, stream=None):
    """pa_decode for callers that cannot allocate device memory: the split-K
    partials live in a fixed array inside the library
    (:func:`pa_decode_noalloc_scratch_bytes` per device, held until exit), as do
    the merge records of the split-K pass.
    Calls on one device share that array, so calls that overlap on the GPU
    race; make the first call on a device before any stream capture."""
    N, bs, Hkv, D = k_cache.shape
    B, Hq, _ = q.shape
    _check(lib().pa_decode_noalloc(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                   _i32tensor(block_tables, "block_tables"), block_tables.shape[1],
                                   _i32tensor(seq_lens, "seq_lens"), B, Hq, Hkv, D, float(scale),
                                   bs, N, int(max_seq_len), int(partition_size),
                                   _dtype_code(k_cache), _stream(stream)),
           "pa_decode_noalloc")


def pa_decode_noalloc_scratch_bytes() -> int:
    return int(lib().pa_decode_noalloc_scratch_bytes())


def pa_chunked_prefill_workspace_size(num_seqs, max_query_len, num_q_heads, head_dim, max_seq_len):
    return int(lib().pa_chunked_prefill_workspace_size(num_seqs, max_query_len, num_q_heads,
                                                       head_dim, max_seq_len))


def pa_chunked_prefill(out, q, k_cache, v_cache, block_tables, seq_lens, query_start_loc, scale,
                       max_query_len, max_seq_len, workspace=None, stream=None):
    """Causal chunk attention over the paged context.  ``q``/``out``
    [total_q, Hq, D]; ``query_start_loc`` int32 [B+1]."""
    N, bs, Hkv, D = k_cache.shape
    _, Hq, _ = q.shape
    B = seq_lens.shape[0]
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().pa_chunked_prefill(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                    _i32tensor(block_tables, "block_tables"), block_tables.shape[1],
                                    _i32tensor(seq_lens, "seq_lens"),
                                    _i32tensor(query_start_loc, "query_start_loc"), B,
                                    int(max_query_len), Hq, Hkv, D, float(scale), bs, N,
                                    int(max_seq_len), _ptr(workspace), ws_bytes,
                                    _dtype_code(k_cache), _stream(stream)),
           "pa_chunked_prefill")


def pa_get_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error bits."""
    code = ctypes.c_int32(0)
    st = lib().pa_get_device_error(_stream(stream), ctypes.byref(code))
    if st not in (PA_OK, 5):
        raise PagedAttnError(st, "pa_get_device_error")
    return int(code.value)


def pa_last_launch_count() -> int:
    return int(lib().pa_last_launch_count())


def pa_testing_wait_fault(kernel, wait_limit_cycles=0):
    """Testing hook: the calling thread's next launch of ``kernel`` ("decode" or
    "prefill"; None clears) withholds one pipeline arrival and gives every wait
    ``wait_limit_cycles`` SM cycles, so the bounded-wait path runs (PA_DEVERR_TIMEOUT)."""
    code = {None: 0, "decode": 1, "prefill": 2}[kernel]
    _check(lib().pa_testing_wait_fault(code, int(wait_limit_cycles)), "pa_testing_wait_fault")
