/*
 * libpagedattn — PagedAttention hot path for NVIDIA B200 (sm_100a).
 *
 * Sources (web pages on KV-cache paging, cited by title and section):
 *   [P1] "大模型推理内存优化从 KV Cache 分页到连续批处理的工程实践" (seekfood.cn):
 *        "KV Cache 的内存开销与分页机制" (fixed-size physical blocks, per-sequence
 *        block table, on-demand allocation, shared prefix blocks),
 *        "PagedAttention 的 CUDA Kernel 实现" (attention reads K/V indirectly through
 *        the block table), "工程边界与架构取舍" (decode is memory-bound and reads
 *        the whole cache; long prompts are prefilled in chunks).
 *   [P2] "KV Cache管理优化：大模型推理显存瓶颈突破" (intelliparadigm), 2.1 (one
 *        pre-allocated pool, no per-request allocation), 2.2 (blocks of 16-32 tokens),
 *        4.1 (blocks shared across sequences by reference counting).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every tensor pointer is a DEVICE pointer owned by the caller, contiguous in the
 *    stated row-major layout; the library keeps no reference after the call returns.
 *  - KV caches: k_cache, v_cache [num_blocks, block_size, num_kv_heads, head_dim] of
 *    fp16 or bf16 (PA_F16 / PA_BF16), or of e4m3 codes for the *_fp8 calls; the two
 *    caches share one layout.
 *  - Block tables: int32 [num_seqs, max_blocks_per_seq]; entry j of row s is the
 *    physical block that holds tokens j*block_size .. j*block_size+block_size-1 of
 *    sequence s.  Entries past a sequence's last block are never read.
 *  - A slot is physical_block * block_size + offset_in_block.
 *  - GQA: q-heads [g*G, (g+1)*G) use kv-head g, with G = num_q_heads / num_kv_heads.
 *  - Supported: head_dim 128, block_size 16 or 32, G in {1, 2, 4, 8}, fp16 / bf16,
 *    up to 4096 sequences per decode call.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy default
 *    stream) and never synchronise the host.  The library allocates no device memory
 *    on any call; scratch space comes from the caller (`workspace`), or from the fixed
 *    array of pa_decode_noalloc.  pa_last_launch_count() tells how many kernels the
 *    calling thread's last call launched.
 *  - Return value: PA_OK once the kernels are launched, or an error found on the host
 *    before any launch (nothing is launched then).  PA_ERR_CUDA reports a failed launch
 *    or tensor-map encoding; a call of several kernels may have queued the earlier ones
 *    when a later one fails to launch.  A launching call first clears a non-sticky CUDA error left
 *    pending on the calling thread by earlier work (cudaGetLastError), so its status
 *    reports its own launches only.
 *  - Errors that depend on device data (a slot or block id outside the cache, a
 *    sequence longer than its table or than max_seq_len, an inconsistent
 *    query_start_loc) never fault or trap: the kernel skips the offending rows (their
 *    outputs are unspecified), ORs a PA_DEVERR_* bit into a per-device flag and goes
 *    on.  Read and clear the flag with pa_get_device_error().
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,          /* null pointer, negative size, inconsistent shape */
  PA_ERR_UNSUPPORTED = 2,          /* head_dim, block_size, GQA group or dtype not built */
  PA_ERR_WORKSPACE_TOO_SMALL = 3,  /* workspace_bytes below the matching *_workspace_size */
  PA_ERR_CUDA = 4,                 /* a CUDA runtime/driver call failed (launch, tensor map) */
  PA_ERR_DEVICE_DATA = 5           /* pa_get_device_error found a device-side data error */
} pa_status;

/* Device-side error bits (pa_get_device_error). */
#define PA_DEVERR_SLOT_RANGE   0x1  /* reshape_and_cache: slot >= num_blocks*block_size   */
#define PA_DEVERR_BLOCK_RANGE  0x2  /* a needed block-table entry outside [0, num_blocks) */
#define PA_DEVERR_SEQ_TOO_LONG 0x4  /* seq_len > max_blocks_per_seq*block_size or > max_seq_len */
#define PA_DEVERR_QUERY_LAYOUT 0x8  /* prefill: query_start_loc not monotone, q_len > seq_len
                                       or q_len > max_query_len */
#define PA_DEVERR_TIMEOUT      0x10 /* an in-kernel pipeline wait gave up (never expected) */
#define PA_DEVERR_POOL         0x20 /* block pool: state out of range, or more blocks freed
                                       than the ring holds (nothing changed) */
#define PA_DEVERR_PREFIX       0x40 /* shared-prefix decode: a prefix length negative, not a
                                       multiple of block_size, above max_prefix_len or
                                       above a member's seq_len */

/* Human-readable name of a status code (static string, never NULL). */
PA_API const char* pa_status_string(int status);

/*
 * reshape_and_cache — write this step's K/V rows into their cache slots.
 * [P1] "KV Cache 的内存开销与分页机制": a generated token's K and V go to the next
 * free place of the sequence's current block (a new block is taken when it is full).
 *
 *   k, v          [T, num_kv_heads, head_dim]  rows to store (same dtype as the caches)
 *   k_cache,
 *   v_cache       [num_blocks, block_size, num_kv_heads, head_dim]  updated in place
 *   slot_mapping  int32 [T]: destination slot of token t; a negative slot skips the
 *                 token (padding).  Two tokens with one slot in a call: undefined.
 * The copy is bitwise.  A slot >= num_blocks*block_size is skipped and sets
 * PA_DEVERR_SLOT_RANGE.  T == 0 launches nothing.
 */
PA_API pa_status pa_reshape_and_cache(const void* k, const void* v, void* k_cache, void* v_cache,
                               const int32_t* slot_mapping, int num_tokens, int num_kv_heads,
                               int head_dim, int num_blocks, int block_size, pa_dtype dtype,
                               void* stream);

/*
 * Bytes of scratch `pa_decode` needs, as an upper bound valid for every kv-head count
 * and GPU: merge records (8 bytes per sequence and q-head, padded to 256 bytes), then
 * split-K partial rows of head_dim+2 fp32 (normalised partial output, running max and
 * sum): (256 + num_seqs) * num_q_heads rows, plus, when partition_size > 0,
 * num_seqs * num_q_heads * ceil(ceil(max_seq_len/16) / (partition_size/16)) +
 * num_q_heads rows.  0 means invalid arguments.
 */
PA_API size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int head_dim, int max_seq_len,
                                int partition_size);

/*
 * pa_decode — single-query attention of each sequence over its paged KV cache.
 * [P1] "PagedAttention 的 CUDA Kernel 实现" and "工程边界与架构取舍": each sequence's
 * query attends to every cached token of the sequence (the token appended this step
 * included: call pa_reshape_and_cache first), K/V reached through the block table.
 *
 *   out           [num_seqs, num_q_heads, head_dim]   softmax(scale * q K^T) V, rounded
 *                                                     to nearest even in `dtype`
 *   q             [num_seqs, num_q_heads, head_dim]
 *   block_tables  int32 [num_seqs, max_blocks_per_seq]
 *   seq_lens      int32 [num_seqs] (device): tokens of each sequence, 0 gives zeros
 *   max_seq_len   host-side upper bound of seq_lens; sizes the grid and the
 *                 partition count.  A longer sequence sets PA_DEVERR_SEQ_TOO_LONG.
 *   partition_size  0 = balanced split-K: the 16-token tiles of every (sequence, group of
 *                 up to 8 kv-heads) are laid end to end and a persistent grid of one CTA
 *                 per SM takes equal shares; a sequence held by one CTA is written
 *                 directly; the pieces of the others leave normalised partials that a
 *                 second, dependent launch merges by log-sum-exp.  > 0 (a
 *                 multiple of 16, at most 2048) also caps every share at that many
 *                 tokens, using more CTAs.
 *   workspace     device scratch, 256-byte aligned, of at least
 *                 pa_decode_workspace_size(...) bytes; contents need no initialisation.
 *                 Calls that overlap on the GPU must not share a workspace.
 * Limits: head_dim 128, block_size 16 or 32, G = num_q_heads/num_kv_heads in
 * {1, 2, 4, 8}, num_seqs <= 4096 (else PA_ERR_UNSUPPORTED).
 */
PA_API pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int max_blocks_per_seq,
                    const int32_t* seq_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                    int head_dim, float scale, int block_size, int num_blocks,
                    int max_seq_len, int partition_size, void* workspace,
                    size_t workspace_bytes, pa_dtype dtype, void* stream);

/*
 * pa_decode_append — pa_reshape_and_cache of each sequence's new token followed by
 * pa_decode, in one launch.  [P1] "PagedAttention 的 CUDA Kernel 实现" and "工程边界与架构
 * 取舍": a decode step appends the token it produced (its K/V go into the slot of position
 * seq_len-1 through the block table) and then attends over the whole cache.
 *
 *   k_new, v_new  [num_seqs, num_kv_heads, head_dim] in `dtype`, 16-byte aligned: the new
 *                 token of sequence s, written bitwise to
 *                 k_cache/v_cache[table[s][(L-1)/bs], (L-1)%bs, :, :] with L = seq_lens[s]
 *                 (L counts the new token), and attended to by the same call.
 *   everything else as pa_decode (same workspace size).
 * A sequence with L = 0 appends nothing; one whose L exceeds its table (flagged
 * PA_DEVERR_SEQ_TOO_LONG) or whose last table entry is out of range (flagged
 * PA_DEVERR_BLOCK_RANGE) appends nothing.  The appended slot must not be read by another
 * sequence of the same call (true whenever shared blocks are full, as with copy-on-write
 * prefix sharing).  Result and cache contents equal pa_reshape_and_cache (slot of
 * position L-1) followed by pa_decode.
 */
PA_API pa_status pa_decode_append(void* out, const void* q, const void* k_new, const void* v_new,
                                  void* k_cache, void* v_cache, const int32_t* block_tables,
                                  int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                                  int num_q_heads, int num_kv_heads, int head_dim, float scale,
                                  int block_size, int num_blocks, int max_seq_len,
                                  int partition_size, void* workspace, size_t workspace_bytes,
                                  pa_dtype dtype, void* stream);

/*
 * FP8 (e4m3) KV cache.  [P1] "工程边界与架构取舍", on quantization and KV-cache precision:
 * an FP8 cache takes half the memory of FP16 (and decode, which reads the whole cache,
 * half the bytes).  The pages fix no format; this library stores e4m3 codes (1 sign, 4
 * exponent bits with bias 7, 3 mantissa bits, subnormals, no infinities, largest
 * finite 448) with one fp32 scale per kv-head for K and one for V: code c stands for
 * value(c) * scale[h].  Caches are uint8 [num_blocks, block_size, num_kv_heads,
 * head_dim]; k_scale / v_scale are device fp32 [num_kv_heads].
 */

/*
 * pa_reshape_and_cache_fp8 — pa_reshape_and_cache into e4m3 caches: element x of
 * kv-head h of token t (k / v in `dtype`, [T, num_kv_heads, head_dim]) is stored as the
 * e4m3 code nearest to x * (1 / scale[h]) computed in fp32 (reciprocal, then product),
 * ties to even, saturated to +-448.  Slot handling and errors as pa_reshape_and_cache.
 */
PA_API pa_status pa_reshape_and_cache_fp8(const void* k, const void* v, void* k_cache,
                                          void* v_cache, const int32_t* slot_mapping,
                                          const float* k_scale, const float* v_scale,
                                          int num_tokens, int num_kv_heads, int head_dim,
                                          int num_blocks, int block_size, pa_dtype dtype,
                                          void* stream);

/*
 * pa_decode_fp8 — pa_decode over e4m3 caches: the result is the attention over the
 * dequantised values value(code) * scale[h], with q and out in `dtype`.  q.k and p.V
 * run as mma.sync fragments in f16 (e4m3 values are exact in f16; q is rounded to f16
 * once; P is rounded to f16); the K scale multiplies the logits and the V scale the
 * output, both in fp32.  Arguments, limits, workspace and errors as pa_decode.
 */
PA_API pa_status pa_decode_fp8(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const float* k_scale, const float* v_scale,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* seq_lens, int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, float scale, int block_size,
                               int num_blocks, int max_seq_len, int partition_size,
                               void* workspace, size_t workspace_bytes, pa_dtype dtype,
                               void* stream);

/*
 * pa_decode_shared_prefix — pa_decode for a batch in which groups of sequences share the
 * first tokens of their context (parallel sampling or beam search over one prompt: [P1]
 * "KV Cache 的内存开销与分页机制", block-level sharing of prefix blocks, and [P2] 4.1,
 * reference-counted blocks that several block tables point at).  The result is
 * pa_decode's, within the same tolerance; the shared blocks are read once per group
 * instead of once per member.
 *   group_starts  int32 [num_groups + 1], device: group g is the sequences
 *                 group_starts[g] .. group_starts[g+1]-1 (ascending, within [0, num_seqs]);
 *                 sequences outside every group share nothing
 *   prefix_lens   int32 [num_groups], device: tokens shared by the members of group g, a
 *                 multiple of block_size, at most max_prefix_len and each member's seq_len;
 *                 the first prefix_lens[g] / block_size table entries of the members hold
 *                 the same K/V (normally the same physical blocks); they are read through
 *                 the table row of the group's first member
 *   max_group_size, max_prefix_len  host bounds (grid sizing)
 * Two launches: one decode grid over a schedule that holds
 * every sequence's keys after its prefix and, appended to the batch, the "chunks": each
 * group's members cut into runs of 16 / G, whose q-heads make 16 rows per kv-head, over the
 * group's prefix (read through the table row of its first member).  A chunk's tiles are
 * whole blocks, as for any sequence; its consumer warps run the 16 rows as two tensor-core
 * tiles, so the prefix is read once per chunk (two chunks of one group are scheduled side
 * by side, and the second read is served by L2); then the merge pass folds each member's
 * own pieces with its chunk's by log-sum-exp.  Workspace: at least
 * pa_decode_shared_prefix_workspace_size(num_seqs, num_q_heads, num_kv_heads, head_dim,
 * max_seq_len) bytes, 256-byte aligned.  An invalid prefix sets PA_DEVERR_PREFIX (outputs
 * of its group unspecified).  fp16/bf16 caches, num_seqs <= 2048 (else
 * PA_ERR_UNSUPPORTED); other limits as pa_decode (partition_size 0).  With num_groups,
 * max_group_size or max_prefix_len 0 it is pa_decode.
 */
PA_API size_t pa_decode_shared_prefix_workspace_size(int num_seqs, int num_q_heads,
                                                     int num_kv_heads, int head_dim,
                                                     int max_seq_len);
PA_API pa_status pa_decode_shared_prefix(void* out, const void* q, const void* k_cache,
                                         const void* v_cache, const int32_t* block_tables,
                                         int max_blocks_per_seq, const int32_t* seq_lens,
                                         int num_seqs, const int32_t* group_starts,
                                         const int32_t* prefix_lens, int num_groups,
                                         int max_group_size, int max_prefix_len, int num_q_heads,
                                         int num_kv_heads, int head_dim, float scale,
                                         int block_size, int num_blocks, int max_seq_len,
                                         void* workspace, size_t workspace_bytes, pa_dtype dtype,
                                         void* stream);

/*
 * pa_attention_varlen — one call for a continuous-batching step that mixes decode
 * sequences and prefill chunks ([P1] "工程边界与架构取舍": long prompts are prefilled in
 * chunks with decode steps in between).  Layout as pa_chunked_prefill: sequence s has
 * n = query_start_loc[s+1] - query_start_loc[s] query rows (its last n tokens, already
 * cached), q / out [num_q_rows, num_q_heads, 128].  Sequences with n == 1 are served as
 * by pa_decode (reading q and writing out at row query_start_loc[s]), those with n > 1
 * as by pa_chunked_prefill on the tcgen05 tensor cores; the result of each row is that
 * of pa_chunked_prefill (a chunk item always runs whole, without the wave-tail split).
 * Launches on `stream`: a small kernel lists the sequences with more than one query row;
 * one persistent grid, whose first CTAs run the split-K decode over the one-row
 * sequences and whose other CTAs run the chunks' prefill items (max_chunk_seqs of them:
 * a host bound on their number, like max_query_len; negative = num_seqs; more chunks
 * than the bound set PA_DEVERR_QUERY_LAYOUT and the extra ones are not computed); then
 * the merge of the decode rows' split segments.  With max_query_len <= 1 (or a bound of
 * 0) it is the decode launch and its merge only.  Workspace: at least
 * pa_attention_varlen_workspace_size(...) bytes, 256-byte aligned.  Limits as pa_decode
 * and pa_chunked_prefill; a decode row outside [0, num_q_rows) sets
 * PA_DEVERR_QUERY_LAYOUT and is skipped.
 */
PA_API size_t pa_attention_varlen_workspace_size(int num_seqs, int max_query_len, int num_q_heads,
                                                 int head_dim, int max_seq_len);
PA_API pa_status pa_attention_varlen(void* out, const void* q, const void* k_cache,
                                     const void* v_cache, const int32_t* block_tables,
                                     int max_blocks_per_seq, const int32_t* seq_lens,
                                     const int32_t* query_start_loc, int num_seqs, int num_q_rows,
                                     int max_query_len, int max_chunk_seqs, int num_q_heads,
                                     int num_kv_heads, int head_dim, float scale, int block_size,
                                     int num_blocks, int max_seq_len, void* workspace,
                                     size_t workspace_bytes, pa_dtype dtype, void* stream);

/*
 * Device-side block-table maintenance.  [P1] "生产级推理引擎的内存管理与调度": a pool
 * keeps the free block ids in a FIFO queue (a new pool holds 0..N-1 in order; allocation
 * pops the front, freeing pushes the back); a sequence gets new blocks when the blocks
 * its tokens need, ceil(tokens / block_size), exceed the blocks it owns; with too few
 * free blocks it is preempted for the step while later sequences are still served; a
 * finished sequence returns its blocks.  The queue lives on the device as a ring
 * `ring` int32 [num_blocks] with `state` int32 [2] = {head, count}; the free ids are
 * ring[(head + i) % num_blocks], i < count, the front first.  All arguments are device
 * pointers; each call is one kernel on `stream`.
 *
 * Shared blocks ([P2] 4.1, reference-counted blocks; [P1] "KV Cache 的内存开销与分页机制",
 * blocks shared by sequences of one prompt): `block_refs` int32 [num_blocks] holds the
 * number of table entries that refer to each block (0 for a free block).  Pass the same
 * array to every call of a pool, or NULL to every call; without it every block belongs
 * to exactly one sequence and pa_block_share is unavailable.
 */

/* pa_block_pool_init — ring = 0..num_blocks-1, head = 0, count = num_blocks, and
 * block_refs (if not NULL) all 0. */
PA_API pa_status pa_block_pool_init(int32_t* ring, int32_t* state, int32_t* block_refs,
                                    int num_blocks, void* stream);

/*
 * pa_block_allocate — one step of appends.  Sequence s holds seq_lens[s] tokens in
 * blocks_owned[s] blocks (the first entries of its block_tables row) and appends
 * q_lens[s] tokens.  In index order, a sequence that needs more blocks takes all of them
 * from the front of the ring (appended to its table, blocks_owned updated) or, if the
 * ring holds fewer than it needs or its table row is too short, none (granted[s] = 0).
 *   slot_mapping  int32 [sum q_lens] out: the slot of every appended token, sequences in
 *                 index order (positions seq_lens[s] .. seq_lens[s]+q_lens[s]-1), -1 for a
 *                 sequence not granted — ready for pa_reshape_and_cache
 *   granted       int32 [num_seqs] out
 * Each block handed out gets block_refs[b] = 1 (when block_refs is not NULL).
 * seq_lens is not updated (the caller adds q_lens of granted sequences).  Limits:
 * num_seqs <= 4096, block_size 16 or 32.  Device-side errors (PA_DEVERR_POOL, read with
 * pa_get_device_error): a state that is not {0 <= head < num_blocks, 0 <= count <=
 * num_blocks} changes nothing; a sequence with a negative length or a blocks_owned[s]
 * outside [0, max_blocks_per_seq] is not granted.
 */
PA_API pa_status pa_block_allocate(int32_t* ring, int32_t* state, int32_t* block_refs,
                                   int num_blocks, int32_t* block_tables,
                                   int max_blocks_per_seq, int32_t* blocks_owned,
                                   const int32_t* seq_lens, const int32_t* q_lens, int num_seqs,
                                   int block_size, int32_t* slot_mapping, int32_t* granted,
                                   void* stream);

/*
 * pa_block_free — every sequence with finished[s] != 0 releases its blocks_owned[s]
 * table entries and gets blocks_owned[s] = 0.  Without block_refs each released block
 * goes to the back of the ring (sequences in index order, blocks in table order).  With
 * block_refs each entry drops one reference, and a block goes to the back of the ring at
 * the release that brings its count to zero, in that same order (a block shared by two
 * finished sequences returns once, at the later one's entry).  Returning more blocks than
 * the ring can hold, or a state that is not a pool state, leaves ring, state and counts
 * unchanged and sets PA_DEVERR_POOL; so does a table entry outside [0, num_blocks)
 * (skipped) or a count that would fall below zero (the block stays out of the ring).
 * Limits: num_seqs <= 4096.
 */
PA_API pa_status pa_block_free(int32_t* ring, int32_t* state, int32_t* block_refs,
                               int num_blocks, const int32_t* block_tables,
                               int max_blocks_per_seq, int32_t* blocks_owned,
                               const int32_t* finished, int num_seqs, void* stream);

/*
 * pa_block_share — prompt sharing ([P2] 4.1; [P1] "KV Cache 的内存开销与分页机制": the
 * sequences sampled from one prompt share its blocks).  For each pair i, sequence
 * dst_seqs[i], which must own no block, takes the first num_shared[i] blocks of sequence
 * src_seqs[i]'s table row (blocks_owned[dst] = num_shared[i]); each of those blocks gains
 * one reference in block_refs (required).  Appends to dst then go to new blocks once the
 * shared ones are full (share whole blocks: dst's length is num_shared * block_size).
 *   src_seqs, dst_seqs, num_shared  int32 [num_pairs], sequence indices in [0, num_seqs)
 * A pair whose dst owns blocks, whose count is negative or above what src owns, whose
 * src equals dst or lies outside the batch, or whose src row holds an id outside
 * [0, num_blocks), is skipped and sets PA_DEVERR_POOL.  Pairs are applied in parallel: a
 * sequence may be dst of one pair only, and no dst may be another pair's src.
 */
PA_API pa_status pa_block_share(int32_t* block_refs, int num_blocks, int32_t* block_tables,
                                int max_blocks_per_seq, int32_t* blocks_owned, int num_seqs,
                                const int32_t* src_seqs, const int32_t* dst_seqs,
                                const int32_t* num_shared, int num_pairs, void* stream);

/*
 * pa_decode_noalloc — pa_decode for callers that cannot allocate device memory.
 * The pages have no counterpart to this call; it exists for callers whose device memory
 * is owned by someone else (an engine's pre-allocated KV pool, a host framework that
 * forbids raw cudaMalloc) or who must not risk the device-wide synchronisation an
 * allocation can cause.  Arguments and results are those of pa_decode without the
 * workspace: the merge records and split-K partials go to a fixed array inside the library,
 * pa_decode_noalloc_scratch_bytes() long (32 MiB), which every GPU that loads the
 * library holds until the process exits.
 *  - Sizes whose partials need more than that (pa_decode_workspace_size(...) >
 *    pa_decode_noalloc_scratch_bytes()) return PA_ERR_WORKSPACE_TOO_SMALL and launch
 *    nothing.
 *  - The first call on a device looks up that device's array address (with the device
 *    current); make that first call before any stream capture.  The address is kept for
 *    the life of the process: after cudaDeviceReset, or anything else that destroys the
 *    device's primary context, do not call this function again in that process.
 *  - Every call on a device shares the one array and leaves its last contents there;
 *    nothing in it needs to start at zero.  Calls that overlap on the GPU (different
 *    streams, no ordering between them) race on the array: order them.
 *  - The call itself allocates no memory.
 */
PA_API pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* block_tables,
                                   int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                                   int num_q_heads, int num_kv_heads, int head_dim, float scale,
                                   int block_size, int num_blocks, int max_seq_len,
                                   int partition_size, pa_dtype dtype, void* stream);

/* Size in bytes of the fixed scratch array pa_decode_noalloc uses (per device). */
PA_API size_t pa_decode_noalloc_scratch_bytes(void);

/*
 * Bytes of the optional pa_chunked_prefill workspace that lets it split its last wave
 * (see pa_chunked_prefill): per split item 2 halves x 256 rows of head_dim+2 fp32 plus a
 * 256-entry int32 row map, for up to min(128, num_seqs * num_q_heads *
 * ceil(max_query_len / 32)) items.  0 means invalid arguments.
 */
PA_API size_t pa_chunked_prefill_workspace_size(int num_seqs, int max_query_len, int num_q_heads,
                                         int head_dim, int max_seq_len);

/*
 * pa_chunked_prefill — causal attention of a chunk of new queries over the paged
 * context.  [P1] "工程边界与架构取舍": a long prompt is processed in chunks; prefill is
 * a dense matrix product (tensor cores).  The chunk's own K/V must already be in the
 * cache (pa_reshape_and_cache first).
 *
 *   out, q            [total_q, num_q_heads, head_dim], total_q = query_start_loc[num_seqs]
 *   query_start_loc   int32 [num_seqs+1] (device): exclusive prefix sum of chunk lengths
 *   seq_lens          int32 [num_seqs] (device): context length including the chunk.
 *                     Query i of sequence s sits at position seq_lens[s]-q_len_s+i and
 *                     attends to keys 0 .. that position, inclusive.
 *   max_query_len     host-side upper bound of the chunk lengths
 *   max_seq_len       host-side upper bound of seq_lens
 *   workspace         optional (NULL allowed), 256-byte aligned device scratch of
 *                     pa_chunked_prefill_workspace_size(...) bytes.  With it, when the
 *                     last wave of (sequence, kv-head, query block) CTAs would fill at
 *                     most half of the SMs, each of those items runs as two CTAs over
 *                     the two halves of its keys and a second launch merges their
 *                     normalised partials (log-sum-exp); the result differs from the
 *                     unsplit one only by rounding.  Calls that overlap on the GPU must
 *                     not share a workspace.
 */
PA_API pa_status pa_chunked_prefill(void* out, const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, int max_blocks_per_seq,
                             const int32_t* seq_lens, const int32_t* query_start_loc,
                             int num_seqs, int max_query_len, int num_q_heads,
                             int num_kv_heads, int head_dim, float scale, int block_size,
                             int num_blocks, int max_seq_len, void* workspace,
                             size_t workspace_bytes, pa_dtype dtype, void* stream);

/*
 * Synchronise `stream`, then read and clear the calling device's PA_DEVERR_* flag into
 * *code.  Returns PA_OK when the flag was 0, PA_ERR_DEVICE_DATA when it was not, or
 * PA_ERR_CUDA if the synchronisation or the copy failed.
 */
PA_API pa_status pa_get_device_error(void* stream, int32_t* code);

/* Number of kernel launches the most recent call on this host thread issued (0 when it
 * returned an error before launching).  For launch accounting in benchmarks. */
PA_API int pa_last_launch_count(void);

/*
 * pa_testing_wait_fault — testing hook for the bounded pipeline waits (no counterpart
 * on the pages).  Every wait inside the kernels gives up after a limit (about 2 s of SM
 * cycles), flags PA_DEVERR_TIMEOUT, stops issuing copies and arrivals, waits (bounded)
 * for its copies and tensor-core products in flight, frees its tensor memory and exits,
 * so that a lost arrival can never hang the GPU.  This hook makes the calling thread's
 * next launch of one kernel withhold one arrival, so the path can be exercised:
 *   kernel  1: the next paged decode kernel (CTA 0's first K/V tile is never copied nor
 *              announced); 2: the next chunked-prefill kernel (CTA 0's first K tile);
 *              0: clear the hook
 *   wait_limit_cycles  the wait limit of that one launch (> 0), in SM clock cycles
 * The launch then ends with PA_DEVERR_TIMEOUT set and unspecified outputs; later calls
 * are unaffected.  One-shot: the hook clears itself when that launch takes it.
 */
PA_API pa_status pa_testing_wait_fault(int kernel, long long wait_limit_cycles);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H */
