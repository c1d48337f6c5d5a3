// Chunked prefill over the paged KV cache, on the sm_100a tensor cores (tcgen05).
//
// What it computes — page "大模型推理内存优化从 KV Cache 分页到连续批处理的工程实践",
// section "工程边界与架构取舍": a long prompt is processed in chunks, and prefill is a
// dense matrix product.  Sequence s has n = qsl[s+1]-qsl[s] new queries, the last n of
// its L = seq_len[s] tokens (their K/V already cached).  Query i sits at position
// L-n+i and attends causally to keys 0..L-n+i (inclusive), reached through the block
// table:  out[qsl[s]+i, qh] = softmax_j(scale * q . K[j]) V[j].
//
// Design:
//  * CTA = (sequence, kv-head, block of 2*MQ queries).  Rows of a 128-row M-tile are
//    (query, q-head of the kv-head's GQA group): MQ = 128/G queries x G heads, so one
//    K/V tile serves every head of the group.  Two M-tiles per CTA share each K/V tile
//    and ping-pong: while the softmax of one runs, the tensor core works on the other.
//  * TMEM (512 columns): S0, S1 (128 fp32 columns each, keys of the tile), O0, O1
//    (128 columns, head_dim).  P (16-bit) is written back over the first 64 columns of
//    S and fed to the P.V MMA straight from TMEM.
//  * Q: each softmax thread copies its own row (bounds-checked 16-byte loads; rows past
//    the chunk are zero) into shared memory in the 128-byte-swizzled K-major layout the
//    MMA reads.  Warp 0 is the TMA producer: per 128-key tile, one box per 16-token run
//    of a physical block for K and for V (block id from the block table), into a
//    two-stage K ring and a two-stage V ring.
//  * Warp 1: allocates TMEM and issues every tcgen05.mma from one thread:
//    S_a = Q_a K^T (M=128, N=128, K=128 as 8 x K16), O_a += P_a V (A in TMEM,
//    V as an MN-major B operand), tcgen05.commit to mbarriers.
//  * Warps 4-7 / 8-11: softmax of M-tile 0 / 1, one thread per row: causal mask on
//    the diagonal tiles, row max, ex2 in the log2 domain, row sum, P packed to 16 bits.
//    The output row is rescaled only when the running max grows by more than 8 (a
//    factor 256); every p stays <= 2^8, and the final normalisation uses the same
//    reference, so the result is unchanged.
//  * Keys at or past L in the last tile: K is masked in the softmax; V rows are
//    zero-filled (TMA out-of-range fill for whole runs, a shared-memory clear for the
//    tail of a partial block) so that 0 * (stale value) never reaches the sum.
// Every wait is bounded; on a timeout the CTA flags PA_DEVERR_TIMEOUT, runs to its end
// without further waits and frees its TMEM.
#include <algorithm>
#include <type_traits>

#include "pa_device.cuh"
#include "pa_host.h"
#include "prefill_body.cuh"

namespace pa {
namespace prefill {

template <typename T, int G>
__global__ void __launch_bounds__(kThreads, 1)
    chunked_prefill_kernel(const __grid_constant__ CUtensorMap tmK,
                           const __grid_constant__ CUtensorMap tmV, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  prefill_body<T, G>(tmK, tmV, a, smem_raw, blockIdx.x);
}

// Merge of the two halves of each split item: one warp per output row, lanes over
// head_dim; o = (w0 o0 + w1 o1) / (w0 + w1), w_i = l_i 2^(m_i - max m).
template <typename T>
__global__ void __launch_bounds__(256) merge_split_kernel(const Args a) {
  // a programmatic dependent of the prefill grid: wait for its partials
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= a.split_items * 2 * kM) return;
  const int dst = a.rowmap[row];
  if (dst < 0) return;
  const int sidx = row / (2 * kM), rr = row - sidx * 2 * kM;
  const long long p0 = (long long)(sidx * 2) * 2 * kM + rr, p1 = p0 + 2 * kM;
  const float2 ml0 = *reinterpret_cast<const float2*>(a.part_ml + p0 * 2);
  const float2 ml1 = *reinterpret_cast<const float2*>(a.part_ml + p1 * 2);
  const float4 o0 = *reinterpret_cast<const float4*>(a.part_o + p0 * kD + lane * 4);
  const float4 o1 = *reinterpret_cast<const float4*>(a.part_o + p1 * kD + lane * 4);
  const float M = fmaxf(ml0.x, ml1.x);
  const float w0 = ml0.x == -INFINITY ? 0.f : ml0.y * fast_exp2(ml0.x - M);
  const float w1 = ml1.x == -INFINITY ? 0.f : ml1.y * fast_exp2(ml1.x - M);
  const float inv = w0 + w1 > 0.f ? 1.f / (w0 + w1) : 0.f;
  T* ob = static_cast<T*>(a.out) + (long long)dst * kD + lane * 4;
  *reinterpret_cast<uint2*>(ob) =
      make_uint2(pack16<T>((w0 * o0.x + w1 * o1.x) * inv, (w0 * o0.y + w1 * o1.y) * inv),
                 pack16<T>((w0 * o0.z + w1 * o1.z) * inv, (w0 * o0.w + w1 * o1.w) * inv));
}

// Workspace of the wave-tail split for `split` items.
inline size_t split_bytes(long long split) {
  return (size_t)split * 2 * kM * (2 * (kD + 2) * sizeof(float) + sizeof(int));
}

template <typename T, int G>
pa_status launch(const CUtensorMap& tk, const CUtensorMap& tv, Args a, void* workspace,
                 size_t workspace_bytes, cudaStream_t stream) {
  auto kern = chunked_prefill_kernel<T, G>;
  if (!ensure_dynamic_smem(reinterpret_cast<const void*>(kern), SMEM_BYTES)) return PA_ERR_CUDA;
  const long long items = (long long)a.num_seqs * a.num_kv_heads * a.qblocks;
  if (items <= 0) return PA_OK;
  if (items > 0x3fffffffLL) return PA_ERR_UNSUPPORTED;
  // One CTA per SM: the items run in waves of `sms`.  When the last wave is at most half
  // full, its items run as two CTAs each (one per half of the keys), so that wave takes
  // about half as long; this needs the caller's workspace.
  const int sms = std::max(1, num_sms());
  long long split = 0;
  const long long rem = items % sms;
  if (workspace && rem > 0 && 2 * rem <= sms && workspace_bytes >= split_bytes(rem) &&
      !((uintptr_t)workspace & 255))
    split = rem;
  a.whole_items = (int)(items - split);
  a.split_items = (int)split;
  if (split) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    a.part_o = reinterpret_cast<float*>(ws);
    a.part_ml = a.part_o + (size_t)split * 2 * 2 * kM * kD;
    a.rowmap = reinterpret_cast<int*>(a.part_ml + (size_t)split * 2 * 2 * kM * 2);
  } else {
    a.part_o = a.part_ml = nullptr;
    a.rowmap = nullptr;
  }
  const long long grid = items + split;
  kern<<<(unsigned)grid, kThreads, SMEM_BYTES, stream>>>(tk, tv, a);
  if (check_launch() != PA_OK) return PA_ERR_CUDA;
  int launches = 1;
  if (split) {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    const long long warps = split * 2 * kM;
    cfg.gridDim = dim3((unsigned)((warps + 7) / 8));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, merge_split_kernel<T>, a) != cudaSuccess) return PA_ERR_CUDA;
    if (check_launch() != PA_OK) return PA_ERR_CUDA;
    ++launches;
  }
  set_launch_count(launches);
  return PA_OK;
}

template <typename T>
pa_status dispatch(int G, const CUtensorMap& tk, const CUtensorMap& tv, const Args& a,
                   void* ws, size_t wsb, cudaStream_t stream) {
  switch (G) {
    case 1: return launch<T, 1>(tk, tv, a, ws, wsb, stream);
    case 2: return launch<T, 2>(tk, tv, a, ws, wsb, stream);
    case 4: return launch<T, 4>(tk, tv, a, ws, wsb, stream);
    case 8: return launch<T, 8>(tk, tv, a, ws, wsb, stream);
    default: return PA_ERR_UNSUPPORTED;
  }
}

}  // namespace prefill

}  // namespace pa

extern "C" size_t pa_chunked_prefill_workspace_size(int num_seqs, int max_query_len,
                                                    int num_q_heads, int head_dim,
                                                    int max_seq_len) {
  (void)head_dim;
  (void)max_seq_len;
  if (num_seqs <= 0 || max_query_len <= 0 || num_q_heads <= 0) return 0;
  // at most half a wave of items is split (SMs <= 256), and never more items than exist
  // (query blocks hold at least 32 queries; kv-heads <= q-heads)
  const long long items = (long long)num_seqs * num_q_heads * ((max_query_len + 31) / 32);
  return pa::prefill::split_bytes(std::min<long long>(128, items));
}

namespace pa {
pa_status chunked_prefill_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* seq_lens, const int32_t* query_start_loc,
                               int num_seqs, int max_query_len, int num_q_heads, int num_kv_heads,
                               int head_dim, float scale, int block_size, int num_blocks,
                               int max_seq_len, void* workspace, size_t workspace_bytes,
                               pa_dtype dtype, void* stream, bool skip_single,
                               const int32_t* chunk_ids, int chunk_cap, void* prep_args,
                               CUtensorMap* prep_tk, CUtensorMap* prep_tv) {
  pa::set_launch_count(0);
  if (num_seqs < 0 || max_query_len < 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
      head_dim <= 0 || block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 ||
      max_seq_len < 0)
    return PA_ERR_INVALID_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (head_dim != 128 || (block_size != 16 && block_size != 32)) return PA_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads) return PA_ERR_INVALID_ARG;
  const int G = num_q_heads / num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0 || max_query_len == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || !query_start_loc)
    return PA_ERR_INVALID_ARG;
  if (((uintptr_t)out | (uintptr_t)q | (uintptr_t)k_cache | (uintptr_t)v_cache) & 15)
    return PA_ERR_INVALID_ARG;
  int* err = pa::launch_prologue();
  if (!err) return PA_ERR_CUDA;
  const int MQ = 128 / G;
  CUtensorMap tk, tv;
  const uint64_t row = (uint64_t)head_dim * 2;
  const uint64_t cdims[4] = {(uint64_t)head_dim, (uint64_t)num_kv_heads, (uint64_t)block_size,
                             (uint64_t)num_blocks};
  const uint64_t cstr[3] = {row, row * num_kv_heads, row * num_kv_heads * block_size};
  const uint32_t cbox[4] = {64, 1, 16, 1};
  if (!pa::encode_tmap_16bit(&tk, k_cache, 4, cdims, cstr, cbox, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !pa::encode_tmap_16bit(&tv, v_cache, 4, cdims, cstr, cbox, CU_TENSOR_MAP_SWIZZLE_128B))
    return PA_ERR_CUDA;
  pa::prefill::Args a;
  a.out = out;
  a.q = q;
  a.block_tables = block_tables;
  a.seq_lens = seq_lens;
  a.qsl = query_start_loc;
  a.err = err;
  a.num_seqs = chunk_ids ? chunk_cap : num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.max_blocks = max_blocks_per_seq;
  a.log2_bs = block_size == 16 ? 4 : 5;
  a.num_blocks = num_blocks;
  a.max_query_len = max_query_len;
  a.seq_cap = (int)std::min<long long>((long long)max_blocks_per_seq * block_size, max_seq_len);
  a.qblocks = (max_query_len + 2 * MQ - 1) / (2 * MQ);
  a.qscale = scale * 1.4426950408889634f;
  a.wait_limit = pa::take_wait_limit(pa::kTestPrefill, &a.test_withhold);
  a.skip_single = skip_single ? 1 : 0;
  a.wait_list = 0;
  a.chunk_ids = chunk_ids;
  a.chunk_cap = chunk_cap;
  // the split's row map stores output row numbers as int
  const long long rows = (long long)num_seqs * max_query_len * num_q_heads;
  if (rows > 0x7fffffffLL) workspace = nullptr;
  if (prep_args) {  // the caller launches: every item whole, no split
    const long long items = (long long)a.num_seqs * a.num_kv_heads * a.qblocks;
    if (items > 0x3fffffffLL) return PA_ERR_UNSUPPORTED;
    a.whole_items = (int)items;
    a.split_items = 0;
    a.part_o = a.part_ml = nullptr;
    a.rowmap = nullptr;
    *static_cast<pa::prefill::Args*>(prep_args) = a;
    *prep_tk = tk;
    *prep_tv = tv;
    return PA_OK;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dtype == PA_F16
             ? pa::prefill::dispatch<__half>(G, tk, tv, a, workspace, workspace_bytes, st)
             : pa::prefill::dispatch<__nv_bfloat16>(G, tk, tv, a, workspace, workspace_bytes, st);
}
}  // namespace pa

extern "C" pa_status pa_chunked_prefill(void* out, const void* q, const void* k_cache,
                                        const void* v_cache, const int32_t* block_tables,
                                        int max_blocks_per_seq, const int32_t* seq_lens,
                                        const int32_t* query_start_loc, int num_seqs,
                                        int max_query_len, int num_q_heads, int num_kv_heads,
                                        int head_dim, float scale, int block_size, int num_blocks,
                                        int max_seq_len, void* workspace, size_t workspace_bytes,
                                        pa_dtype dtype, void* stream) {
  return pa::chunked_prefill_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                  seq_lens, query_start_loc, num_seqs, max_query_len, num_q_heads,
                                  num_kv_heads, head_dim, scale, block_size, num_blocks,
                                  max_seq_len, workspace, workspace_bytes, dtype, stream, false,
                                  nullptr, 0);
}
