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

// Encode a 4-D tiled TMA descriptor over a KV cache
// [num_blocks, block_size, num_kv_heads, head_dim] of 16-bit elements whose box is
// `box_rows` consecutive tokens x head_dim of one kv-head of one block.
bool encode_cache_tmap(CUtensorMap* out, const void* cache, int num_blocks, int block_size,
                       int num_kv_heads, int head_dim, int box_rows);

// Launch accounting for pa_last_launch_count().
void set_launch_count(int n);

inline pa_status check_launch() {
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

}  // namespace pa
