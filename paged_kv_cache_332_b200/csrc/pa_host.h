// Host-side helpers shared by the libpagedattn entry points (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pagedattn.h"

namespace pa {

// Device address of the calling device's PA_DEVERR_* flag (nullptr on failure).
int* device_error_flag();

// Streaming multiprocessors of the current device (cached per device).
int num_sms();

// Allow `func` at least `bytes` of dynamic shared memory on the current device.  The
// attribute is set once per (kernel, device) and only raised afterwards, so steady-state
// calls cost a map lookup instead of a driver call.
bool ensure_dynamic_smem(const void* func, int bytes);

// Encode a 4-D tiled TMA descriptor over a KV cache
// [num_blocks, block_size, num_kv_heads, head_dim] of 16-bit elements whose box is
// `box_rows` consecutive tokens x head_dim of one kv-head of one block.
bool encode_cache_tmap(CUtensorMap* out, const void* cache, int num_blocks, int block_size,
                       int num_kv_heads, int head_dim, int box_rows);

// Encode a tiled TMA descriptor over a row-major tensor of 16-bit elements.
// dims/box innermost first; strides_bytes[i] is the stride of dimension i+1.
// Encode a tiled TMA descriptor of `type` elements (rank <= 5, dims innermost first,
// strides in bytes for dims 1.., element strides 1, no interleave, L2 promotion 256 B).
bool encode_tmap(CUtensorMap* out, CUtensorMapDataType type, const void* base, int rank,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle);
bool encode_tmap_16bit(CUtensorMap* out, const void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapSwizzle swizzle);

// Launch accounting for pa_last_launch_count().
void set_launch_count(int n);
int launch_count();

// Shared-prefix decode, first pass (prefill.cu): the attention of every member's q-heads
// over its group's shared prefix, on the tcgen05 prefill kernel (the members' queries of
// one kv-head form the rows of one M-tile), as `chunks` pieces of normalised partial rows
// in pre_o [slots][q_rows * num_q_heads][128] and (max, sum) in pre_ml.
constexpr int kMaxPrefixChunks = 8;  // partial slots at most
struct SharedPrefixPlan {
  int ksplit;   // groups fit one M-tile: the two M-tiles take alternate key tiles
  int qblocks;  // query blocks per (group, kv-head)
  int pieces;   // key pieces per (group, kv-head, query block)
  int slots;    // partial rows per output row: pieces (x 2 with ksplit)
};
// pa_chunked_prefill; with skip_single, sequences of one query row are left out (the
// varlen call serves them with the decode kernel); with chunk_ids (a device list of the
// sequences with more than one query row, its length at chunk_ids[chunk_cap]) the grid
// covers chunk_cap sequences of that list instead of all num_seqs.
pa_status chunked_prefill_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* seq_lens, const int32_t* query_start_loc,
                               int num_seqs, int max_query_len, int num_q_heads, int num_kv_heads,
                               int head_dim, float scale, int block_size, int num_blocks,
                               int max_seq_len, void* workspace, size_t workspace_bytes,
                               pa_dtype dtype, void* stream, bool skip_single,
                               const int32_t* chunk_ids, int chunk_cap);

SharedPrefixPlan plan_shared_prefix(int num_groups, int num_kv_heads, int G, int max_group_size,
                                    int max_prefix_len);
pa_status shared_prefix_pass(const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, int max_blocks_per_seq,
                             const int32_t* group_starts, const int32_t* prefix_lens,
                             int num_groups, int max_group_size, int max_prefix_len, int q_rows,
                             int num_q_heads, int num_kv_heads, float scale, int block_size,
                             int num_blocks, const SharedPrefixPlan& plan, float* pre_o,
                             float* pre_ml, pa_dtype dtype, int* err, cudaStream_t stream);

inline pa_status check_launch() {
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa
