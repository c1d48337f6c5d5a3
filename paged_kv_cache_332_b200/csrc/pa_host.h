// Host-side helpers shared by the libpagedattn entry points (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/pagedattn.h"

namespace pa {

// Device address of the calling device's PA_DEVERR_* flag (nullptr on failure).
int* device_error_flag();

// Start of every launching entry point, after its host-side checks: clears a non-sticky
// CUDA error left pending on this thread by earlier, unrelated work (so that the launch
// checks below report this call's launches only) and returns the device error flag.
int* launch_prologue();

// Streaming multiprocessors of the current device (cached per device).
int num_sms();

// Allow `func` at least `bytes` of dynamic shared memory on the current device.  The
// attribute is set once per (kernel, device) and only raised afterwards, so steady-state
// calls cost a map lookup instead of a driver call.
bool ensure_dynamic_smem(const void* func, int bytes);

// Encode a tiled TMA descriptor of `type` elements (rank <= 5, dims innermost first,
// strides in bytes for dims 1.., element strides 1, no interleave, L2 promotion 256 B);
// the _16bit form takes 16-bit elements.
bool encode_tmap(CUtensorMap* out, CUtensorMapDataType type, const void* base, int rank,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                 CUtensorMapSwizzle swizzle);
bool encode_tmap_16bit(CUtensorMap* out, const void* base, int rank, const uint64_t* dims,
                       const uint64_t* strides_bytes, const uint32_t* box,
                       CUtensorMapSwizzle swizzle);

// Longest any single pipeline wait may take before a kernel gives up, in SM clock cycles
// (the per-SM counter is cheap to read; ~2 s at B200 clocks).  Kernels take the limit as
// an argument: always this value, except under the testing hook that shortens it.
constexpr long long kWaitLimitCycles = 4000000000ll;

// Testing hook (pa_testing_wait_fault): the wait limit for the next launch of `kind` on
// this thread, and whether that launch withholds one pipeline arrival.  One-shot: the
// hook is cleared when taken; without it the limit is kWaitLimitCycles.
constexpr int kTestDecode = 1;
constexpr int kTestPrefill = 2;
long long take_wait_limit(int kind, int* withhold);

// Launch accounting for pa_last_launch_count().
void set_launch_count(int n);
int launch_count();

// pa_chunked_prefill; with skip_single, sequences of one query row are left out (the
// varlen call serves them with the decode kernel); with chunk_ids (a device list of the
// sequences with more than one query row, its length at chunk_ids[chunk_cap]) the grid
// covers chunk_cap sequences of that list instead of all num_seqs.
// With `prep_args` (a prefill::Args) and the two tensor maps, nothing is launched: the
// prepared arguments are returned for a kernel of the caller's.
pa_status chunked_prefill_impl(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* seq_lens, const int32_t* query_start_loc,
                               int num_seqs, int max_query_len, int num_q_heads, int num_kv_heads,
                               int head_dim, float scale, int block_size, int num_blocks,
                               int max_seq_len, void* workspace, size_t workspace_bytes,
                               pa_dtype dtype, void* stream, bool skip_single,
                               const int32_t* chunk_ids, int chunk_cap, void* prep_args = nullptr,
                               CUtensorMap* prep_tk = nullptr, CUtensorMap* prep_tv = nullptr);

inline pa_status check_launch() {
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa
