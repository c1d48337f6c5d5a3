"""GPU parity for the shared-prefix decode (pa_decode_shared_prefix) through the C ABI:
groups of sequences whose block tables share their first blocks ([P1] "KV Cache 的内存
开销与分页机制", block-level sharing; [P2] 4.1) must get the oracle's paged attention —
the same result as pa_decode — while the shared blocks are read once per group.  Covers
both cached workloads with shared prompts, every GQA group and output type, sequences
outside any group, groups of one, groups with nothing shared, members with no keys of
their own, more members than one CTA's M-tiles hold, prefixes cut into several pieces
with ragged tiles, flagged invalid prefixes, and sampled rows at full size."""
import numpy as np
import pytest
import torch

import oracle.paged_attention as opa
import paged_kv_cache_332_b200 as pa
import workloads
from tests import _parity as P

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _gpu_shared(b, group_starts=None, prefix_lens=None, max_prefix=None):
    gs = b.group_starts if group_starts is None else group_starts
    pl = b.prefix_lens if prefix_lens is None else prefix_lens
    B, Hq, D = b.q.shape
    ws = torch.empty(pa.pa_decode_shared_prefix_workspace_size(B, Hq, b.num_kv_heads, D,
                                                               b.max_seq_len),
                     dtype=torch.uint8, device=DEV)
    out = torch.full_like(b.q, float("nan"))
    sizes = (gs[1:] - gs[:-1]).cpu()
    max_group = int(sizes.max()) if sizes.numel() else 0
    mp = int(pl.max()) if max_prefix is None else max_prefix
    pa.pa_decode_shared_prefix(out, b.q, b.k_cache, b.v_cache, b.block_tables, b.seq_lens, gs, pl,
                               b.scale, b.max_seq_len, max_group, mp, ws)
    return out


def _vs_oracle(bc, what, append=True):
    b = bc.to(DEV)
    if append:
        P.gpu_append(b)
    out = _gpu_shared(b)
    launches = pa.pa_last_launch_count()
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    if append:
        ref = P.oracle_decode(bc)
    else:
        ref = opa.paged_decode(opa.to_f64(bc.q), opa.to_f64(bc.k_cache), opa.to_f64(bc.v_cache),
                               bc.block_tables.numpy(), bc.seq_lens.numpy(), bc.scale)
    P.compare(out, ref, bc.dtype, what)
    return out, launches


def _grouped_batch(name, lens, groups, prefix, G, dtype, bs=16, Hkv=4, seed=0):
    return workloads.make_batch(name, seq_lens=lens, num_q_heads=G * Hkv, num_kv_heads=Hkv,
                                block_size=bs, num_blocks=sum(-(-L // bs) for L in lens) + 8,
                                dtype=dtype, seed=seed, shared_groups=groups,
                                shared_prefix_tokens=prefix)


@pytest.mark.parametrize("bs", [16, 32])
def test_shared_prompt_workloads(bs):
    bc = workloads.shared_prefix(block_size=bs, scale=1 / 8)[0]
    _, launches = _vs_oracle(bc, "shared prefix bs%d" % bs)
    assert launches == 2  # one decode grid over own keys and chunks, then the merge


@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_every_group_and_dtype(G, dtype):
    # seq 0 and 9 outside any group; a group of one (seq 3); ragged prefix (176 tokens:
    # one full and one partial 128-key tile)
    lens = [50, 177, 200, 190, 181, 300, 177, 250, 400, 33]
    groups = [[1, 2], [3], [4, 5, 6, 7, 8]]
    bc = _grouped_batch("grp_g%d" % G, lens, groups, 176, G, dtype, seed=10 + G)
    assert bc.group_starts.tolist() == [1, 3, 4, 9]
    _vs_oracle(bc, "groups, G=%d %s" % (G, dtype))


def test_groups_with_nothing_shared_and_gaps():
    lens = [40, 60, 70, 80, 90, 100]
    bc = _grouped_batch("gaps", lens, [[1, 2], [4, 5]], 32, 4, torch.float16, seed=3)
    assert bc.prefix_lens.tolist() == [32, 0, 32]  # seq 3 forms a group with no prefix
    _vs_oracle(bc, "groups with a gap")


def test_many_members_long_prefix_several_pieces():
    # 40 members of one group at G = 8: twenty chunks of two members over a 1040-token
    # prefix (65 tiles), spread over many CTAs
    lens = [1040 + 1 + (7 * i) % 90 for i in range(40)]
    bc = _grouped_batch("many", lens, [list(range(40))], 1040, 8, torch.bfloat16, Hkv=2, seed=5)
    _vs_oracle(bc, "40 members, prefix 1040")


def test_members_without_keys_of_their_own():
    # seq_len == prefix: the whole context is shared (no append this step)
    lens = [64, 64, 64, 100]
    bc = _grouped_batch("nokeys", lens, [[0, 1, 2, 3]], 64, 4, torch.float16, seed=6)
    _vs_oracle(bc, "members with only the shared prefix", append=False)


def test_nothing_shared_is_pa_decode_bitwise():
    bc = workloads.shared_prefix(block_size=16, scale=1 / 8)[0]
    b = bc.to(DEV)
    P.gpu_append(b)
    want = P.gpu_decode(b)
    got = _gpu_shared(b, prefix_lens=torch.zeros_like(b.prefix_lens), max_prefix=0)
    torch.cuda.synchronize()
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


def test_invalid_prefix_flagged():
    lens = [40, 60, 70]
    bc = _grouped_batch("bad", lens, [[0, 1, 2]], 32, 4, torch.float16, seed=7)
    b = bc.to(DEV)
    pa.pa_get_device_error()
    for bad in (24, 48):  # not a multiple of the block size; longer than seq 0
        _gpu_shared(b, prefix_lens=torch.tensor([bad], dtype=torch.int32, device=DEV))
        assert pa.pa_get_device_error() & pa.PA_DEVERR["PREFIX"], bad
    # a prefix above max_prefix_len is flagged too
    _gpu_shared(b, max_prefix=16)
    assert pa.pa_get_device_error() & pa.PA_DEVERR["PREFIX"]


def test_full_size_shared_prompts_sampled():
    for bs in (16, 32):
        b = workloads.shared_prefix(block_size=bs, device=DEV)[0]
        seqs = [0, 1, 12, 63]
        sub = P.sub_batch(b, seqs)  # generator's cache, before the GPU append
        P.gpu_append(b)
        out = _gpu_shared(b)
        torch.cuda.synchronize()
        assert pa.pa_get_device_error() == 0
        kc, vc = opa.to_f64(sub["k_cache"]), opa.to_f64(sub["v_cache"])
        sm = b.slot_mapping.cpu().numpy()
        new_slots = np.array([sub["remap"][int(sm[r]) // bs] * bs + int(sm[r]) % bs for r in seqs])
        opa.reshape_and_cache(opa.to_f64(b.k_new[seqs]), opa.to_f64(b.v_new[seqs]), kc, vc,
                              new_slots)
        ref = opa.paged_decode(opa.to_f64(b.q[seqs]), kc, vc, sub["block_tables"].numpy(),
                               sub["seq_lens"].numpy(), b.scale)
        P.compare(out[seqs], ref, b.dtype, "shared prompts bs%d full size, sampled" % bs)
