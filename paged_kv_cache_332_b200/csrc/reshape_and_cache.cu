// reshape_and_cache: scatter this step's K/V rows into their cache slots.
//
// Page "大模型推理内存优化从 KV Cache 分页到连续批处理的工程实践", section
// "KV Cache 的内存开销与分页机制": a new token's K and V are stored at the next
// free place of the sequence's current physical block.  The caller passes the
// destination slot (block * block_size + offset) of every token.
//
// In the cache layout [num_blocks, block_size, num_kv_heads, head_dim] all kv-heads
// of one slot form one contiguous row of num_kv_heads*head_dim elements, exactly
// like a token's row of k / v [T, num_kv_heads, head_dim].  So the scatter is one
// contiguous row copy per token: one warp per token moves the K row and the V row
// with 16-byte vector loads and stores.  The work is pure HBM traffic:
// 2 * T * num_kv_heads * head_dim * 2 bytes read and the same written.
#include <cuda_fp8.h>

#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {

__global__ void __launch_bounds__(256) reshape_and_cache_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, uint4* __restrict__ k_cache,
    uint4* __restrict__ v_cache, const int32_t* __restrict__ slot_mapping, int num_tokens,
    int row_vecs, long long num_slots, int* err) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= num_tokens) return;
  const long long slot = slot_mapping[warp];
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (lane == 0) flag_error(err, PA_DEVERR_SLOT_RANGE);
    return;
  }
  const uint4* ks = k + (long long)warp * row_vecs;
  const uint4* vs = v + (long long)warp * row_vecs;
  uint4* kd = k_cache + slot * row_vecs;
  uint4* vd = v_cache + slot * row_vecs;
  for (int i = lane; i < row_vecs; i += 32) {
    const uint4 a = __ldg(ks + i);
    const uint4 b = __ldg(vs + i);
    kd[i] = a;
    vd[i] = b;
  }
}

// FP8 (e4m3) cache: page section "工程边界与架构取舍" (quantization and KV-cache
// precision) — an FP8 cache halves the memory.  Each element x of kv-head h is stored
// as the e4m3 code nearest to x * (1 / scale[h]) (reciprocal and product in fp32), ties
// to even, saturated to +-448.  One warp per token; a lane converts 8 elements (16 bytes
// in, 8 bytes out) per step.
template <typename T>
__device__ __forceinline__ uint32_t quantize4(uint32_t w01, uint32_t w23, float inv) {
  const float2 a = Elem<T>::unpack2(w01), b = Elem<T>::unpack2(w23);
  const __nv_fp8x2_storage_t lo =
      __nv_cvt_float2_to_fp8x2(make_float2(a.x * inv, a.y * inv), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi =
      __nv_cvt_float2_to_fp8x2(make_float2(b.x * inv, b.y * inv), __NV_SATFINITE, __NV_E4M3);
  return (uint32_t)lo | ((uint32_t)hi << 16);
}

template <typename T>
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, uint2* __restrict__ k_cache,
    uint2* __restrict__ v_cache, const int32_t* __restrict__ slot_mapping,
    const float* __restrict__ k_scale, const float* __restrict__ v_scale, int num_tokens,
    int row_vecs, long long num_slots, int* err) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= num_tokens) return;
  const long long slot = slot_mapping[warp];
  if (slot < 0) return;  // padding token
  if (slot >= num_slots) {
    if (lane == 0) flag_error(err, PA_DEVERR_SLOT_RANGE);
    return;
  }
  const uint4* ks = k + (long long)warp * row_vecs;
  const uint4* vs = v + (long long)warp * row_vecs;
  uint2* kd = k_cache + slot * row_vecs;
  uint2* vd = v_cache + slot * row_vecs;
  for (int i = lane; i < row_vecs; i += 32) {
    const int h = i >> 4;  // 16 groups of 8 elements per 128-element head
    const float ik = 1.0f / __ldg(k_scale + h), iv = 1.0f / __ldg(v_scale + h);
    const uint4 a = __ldg(ks + i);
    const uint4 b = __ldg(vs + i);
    kd[i] = make_uint2(quantize4<T>(a.x, a.y, ik), quantize4<T>(a.z, a.w, ik));
    vd[i] = make_uint2(quantize4<T>(b.x, b.y, iv), quantize4<T>(b.z, b.w, iv));
  }
}

}  // namespace pa

extern "C" pa_status pa_reshape_and_cache_fp8(const void* k, const void* v, void* k_cache,
                                              void* v_cache, const int32_t* slot_mapping,
                                              const float* k_scale, const float* v_scale,
                                              int num_tokens, int num_kv_heads, int head_dim,
                                              int num_blocks, int block_size, pa_dtype dtype,
                                              void* stream) {
  pa::set_launch_count(0);
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 ||
      block_size <= 0)
    return PA_ERR_INVALID_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (head_dim != 128 || (block_size != 16 && block_size != 32)) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping || !k_scale || !v_scale)
    return PA_ERR_INVALID_ARG;
  const uintptr_t al = (uintptr_t)k | (uintptr_t)v | (uintptr_t)k_cache | (uintptr_t)v_cache;
  if (al & 15) return PA_ERR_INVALID_ARG;
  int* err = pa::launch_prologue();
  if (!err) return PA_ERR_CUDA;
  const int row_vecs = num_kv_heads * head_dim / 8;  // 8 elements per step
  const int threads = 256;
  const int blocks = (int)(((long long)num_tokens * 32 + threads - 1) / threads);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const long long slots = (long long)num_blocks * block_size;
  if (dtype == PA_F16)
    pa::reshape_and_cache_fp8_kernel<__half><<<blocks, threads, 0, st>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint2*>(k_cache),
        static_cast<uint2*>(v_cache), slot_mapping, k_scale, v_scale, num_tokens, row_vecs, slots,
        err);
  else
    pa::reshape_and_cache_fp8_kernel<__nv_bfloat16><<<blocks, threads, 0, st>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint2*>(k_cache),
        static_cast<uint2*>(v_cache), slot_mapping, k_scale, v_scale, num_tokens, row_vecs, slots,
        err);
  const pa_status s = pa::check_launch();
  if (s == PA_OK) pa::set_launch_count(1);
  return s;
}

extern "C" pa_status pa_reshape_and_cache(const void* k, const void* v, void* k_cache,
                                          void* v_cache, const int32_t* slot_mapping,
                                          int num_tokens, int num_kv_heads, int head_dim,
                                          int num_blocks, int block_size, pa_dtype dtype,
                                          void* stream) {
  pa::set_launch_count(0);
  if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 ||
      block_size <= 0)
    return PA_ERR_INVALID_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (head_dim != 128 || (block_size != 16 && block_size != 32)) return PA_ERR_UNSUPPORTED;
  if (num_tokens == 0) return PA_OK;
  if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
  const uintptr_t al = (uintptr_t)k | (uintptr_t)v | (uintptr_t)k_cache | (uintptr_t)v_cache;
  if (al & 15) return PA_ERR_INVALID_ARG;  // 16-byte vector access
  int* err = pa::launch_prologue();
  if (!err) return PA_ERR_CUDA;
  const int row_vecs = num_kv_heads * head_dim * 2 / 16;
  const int threads = 256;
  const int blocks = (int)(((long long)num_tokens * 32 + threads - 1) / threads);
  pa::reshape_and_cache_kernel<<<blocks, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), static_cast<uint4*>(k_cache),
      static_cast<uint4*>(v_cache), slot_mapping, num_tokens, row_vecs,
      (long long)num_blocks * block_size, err);
  const pa_status st = pa::check_launch();
  if (st == PA_OK) pa::set_launch_count(1);
  return st;
}
