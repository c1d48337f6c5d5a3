// Device-side block-table maintenance: the block pool and the scheduler's allocation
// rule on the GPU, so that a decode step can grow its block tables and append without a
// round trip to the host.
//
// Page "大模型推理内存优化从 KV Cache 分页到连续批处理的工程实践", section
// "生产级推理引擎的内存管理与调度": free block ids wait in a FIFO queue (a new pool holds
// 0..N-1 in order; allocation pops the front, freeing pushes the back); a sequence gets a
// new block when the blocks its tokens need (ceil(tokens / block_size)) exceed the blocks
// it owns; when none is free the sequence is preempted for the step and the following
// sequences are still served; a finished sequence returns its blocks.
//
// Here the queue is a ring `ring[N]` with `state = {head, count}` in device memory.  A
// step may append several tokens to a sequence (a prefill chunk): the sequence takes all
// the blocks it needs or none, sequences in index order.  Both kernels run as one CTA
// (a step touches a few thousand sequences at most): block-wide prefix sums give every
// sequence its place in the ring; the rare step where the pool cannot serve everyone is
// decided by one thread walking the sequences in order.
//
// Page "KV Cache管理优化：大模型推理显存瓶颈突破", section 4.1: a block may be held by
// several sequences (a shared prompt) and carries a reference count.  With the optional
// `refs[N]` array, allocation sets a handed-out block's count to 1, pa_block_share gives a
// sequence the first blocks of another's table (+1 each), and freeing drops one reference
// per table entry; a block goes back on the ring only at the release that brings its count
// to zero, in the order a sequential walk (sequences in index order, entries in table
// order) would push it.
#include <algorithm>
#include <climits>

#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {
namespace pool {

constexpr int kThreads = 1024;
constexpr int kMaxSeqs = 4096;

// Exclusive prefix sum over v[0..n) in shared memory (n <= kMaxSeqs), in place; returns
// the total.  All threads of the CTA call it.
__device__ int block_exclusive_scan(int* v, int n, int* warp_sums) {
  const int per = (n + kThreads - 1) / kThreads;  // consecutive elements per thread
  const int lo = min(n, (int)threadIdx.x * per), hi = min(n, lo + per);
  int sum = 0;
  for (int i = lo; i < hi; ++i) sum += v[i];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) warp_sums[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sums[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    warp_sums[lane] = wi - w;  // exclusive over warps
    if (lane == 31) warp_sums[32] = wi;
  }
  __syncthreads();
  int run = warp_sums[warp] + incl - sum;
  for (int i = lo; i < hi; ++i) {
    const int x = v[i];
    v[i] = run;
    run += x;
  }
  const int total = warp_sums[32];
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kThreads) init_kernel(int32_t* ring, int32_t* state,
                                                       int32_t* refs, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    ring[i] = i;
    if (refs) refs[i] = 0;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    state[0] = 0;  // head
    state[1] = n;  // count
  }
}

__global__ void __launch_bounds__(kThreads) allocate_kernel(
    int32_t* __restrict__ ring, int32_t* __restrict__ state, int n,
    int32_t* __restrict__ tables, int max_blocks, int32_t* __restrict__ owned,
    const int32_t* __restrict__ seq_lens, const int32_t* __restrict__ q_lens, int B,
    int log2_bs, int32_t* __restrict__ slots, int32_t* __restrict__ granted,
    int32_t* __restrict__ refs, int* err) {
  __shared__ int need[kMaxSeqs];   // blocks to take, then their offset in the ring order
  __shared__ int tok[kMaxSeqs];    // tokens to append, then their offset in `slots`
  __shared__ unsigned char ok[kMaxSeqs];  // granted (its table row can hold the blocks)
  __shared__ int warp_sums[33];
  __shared__ int all_fit, taken;
  const int head = state[0], count = state[1];
  if (count < 0 || count > n || head < 0 || head >= n) {  // not a pool state
    if (threadIdx.x == 0) flag_error(err, PA_DEVERR_POOL);
    return;
  }
  if (threadIdx.x == 0) all_fit = 1;
  __syncthreads();
  for (int s = threadIdx.x; s < B; s += blockDim.x) {
    const int L = seq_lens[s], q = q_lens[s], have = owned[s];
    const bool sane = L >= 0 && q >= 0 && have >= 0 && have <= max_blocks;
    if (!sane) flag_error(err, PA_DEVERR_POOL);
    const int want = sane ? (L + q + (1 << log2_bs) - 1) >> log2_bs : 0;
    need[s] = max(0, want - have);
    tok[s] = max(q, 0);
    ok[s] = sane && want <= max_blocks ? 1 : 0;  // the table cannot hold more
    if (!ok[s]) all_fit = 0;
  }
  __syncthreads();
  const int total_need = block_exclusive_scan(need, B, warp_sums);  // need[] now offsets
  const int total_tok = block_exclusive_scan(tok, B, warp_sums);
  (void)total_tok;
  if (threadIdx.x == 0) {
    if (all_fit && total_need <= count) {
      taken = total_need;  // every sequence served: offsets as scanned
    } else {
      // serve in index order, all or none, as blocks remain
      int t = 0;
      for (int s = 0; s < B; ++s) {
        const int extra = (s + 1 < B ? need[s + 1] : total_need) - need[s];
        const unsigned char fits = ok[s] && t + extra <= count;
        ok[s] = fits;
        need[s] = fits ? t : -1;
        if (fits) t += extra;
      }
      taken = t;
    }
  }
  __syncthreads();
  // hand out the blocks: sequence s takes ring[(head + need[s] + j) % n], j < extra
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int s = warp; s < B; s += nwarps) {
    const int L = seq_lens[s], q = max(q_lens[s], 0), have = owned[s];
    const int g = ok[s];
    const int extra = g ? max(0, ((L + q + (1 << log2_bs) - 1) >> log2_bs) - have) : 0;
    if (g)
      for (int j = lane; j < extra; j += 32) {
        const int b = ring[(head + need[s] + j) % n];
        tables[(long long)s * max_blocks + have + j] = b;
        if (refs && (unsigned)b < (unsigned)n) refs[b] = 1;
      }
    __syncwarp();
    if (g && lane == 0) owned[s] = have + extra;
    if (lane == 0) granted[s] = g;
    // slots of the appended tokens (the table entries above are visible to the warp)
    for (int i = lane; i < q; i += 32) {
      const int p = L + i;
      int v = -1;
      if (g) v = (tables[(long long)s * max_blocks + (p >> log2_bs)] << log2_bs) + (p & ((1 << log2_bs) - 1));
      slots[tok[s] + i] = v;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    state[0] = (head + taken) % n;
    state[1] = count - taken;
  }
}

__global__ void __launch_bounds__(kThreads) free_kernel(
    int32_t* __restrict__ ring, int32_t* __restrict__ state, int n,
    const int32_t* __restrict__ tables, int max_blocks, int32_t* __restrict__ owned,
    const int32_t* __restrict__ finished, int B, int* err) {
  __shared__ int cnt[kMaxSeqs];
  __shared__ int warp_sums[33];
  const int head = state[0], count = state[1];
  if (count < 0 || count > n || head < 0 || head >= n) {  // not a pool state
    if (threadIdx.x == 0) flag_error(err, PA_DEVERR_POOL);
    return;
  }
  for (int s = threadIdx.x; s < B; s += blockDim.x)
    cnt[s] = finished[s] ? min(max(owned[s], 0), max_blocks) : 0;
  __syncthreads();
  const int total = block_exclusive_scan(cnt, B, warp_sums);
  if (count + total > n) {  // more blocks returned than were handed out
    if (threadIdx.x == 0) flag_error(err, PA_DEVERR_POOL);
    return;
  }
  const int tail = (head + count) % n;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int s = warp; s < B; s += nwarps) {
    if (!finished[s]) continue;
    const int k = (s + 1 < B ? cnt[s + 1] : total) - cnt[s];
    for (int j = lane; j < k; j += 32)
      ring[(tail + cnt[s] + j) % n] = tables[(long long)s * max_blocks + j];
    __syncwarp();
    if (lane == 0) owned[s] = 0;
  }
  __syncthreads();
  if (threadIdx.x == 0) state[1] = count + total;
}

// Reference-counted release.  The table entries of the finished sequences, in sequential
// order (sequence, then entry), are numbered e = 0..E-1; each thread takes a contiguous
// range of them.  Pass 1 drops one reference per entry.  A block whose count is now zero
// returns to the ring at its last entry: pass 2 marks such blocks (count -> kMark) and
// pass 3 raises the mark to kMark + 1 + (its largest entry number), so the entry holding
// the final value pushes the block, at the position a prefix sum over the pushing entries
// gives.  Counts below zero (a block released more often than it was held) are flagged
// and the block stays out of the ring.
constexpr int kMark = INT_MIN;

__device__ __forceinline__ int ld_volatile(const int32_t* p) {
  return *reinterpret_cast<const volatile int32_t*>(p);
}

__global__ void __launch_bounds__(kThreads) free_kernel_refs(
    int32_t* __restrict__ ring, int32_t* __restrict__ state, int32_t* refs, int n,
    const int32_t* __restrict__ tables, int max_blocks, int32_t* __restrict__ owned,
    const int32_t* __restrict__ finished, int B, int* err) {
  __shared__ int cnt[kMaxSeqs];
  __shared__ int tsum[kThreads];
  __shared__ int warp_sums[33];
  const int head = state[0], count = state[1];
  if (count < 0 || count > n || head < 0 || head >= n) {  // not a pool state
    if (threadIdx.x == 0) flag_error(err, PA_DEVERR_POOL);
    return;
  }
  for (int s = threadIdx.x; s < B; s += blockDim.x)
    cnt[s] = finished[s] ? min(max(owned[s], 0), max_blocks) : 0;
  __syncthreads();
  const int E = block_exclusive_scan(cnt, B, warp_sums);  // cnt[] now entry offsets
  const int per = (E + kThreads - 1) / kThreads;
  const int e0 = min(E, (int)threadIdx.x * per), e1 = min(E, e0 + per);
  // sequence holding entry e0: the last s with cnt[s] <= e0
  int s0 = 0;
  if (e0 < e1) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (cnt[mid] <= e0) lo = mid; else hi = mid - 1;
    }
    s0 = lo;
  }
  // block of every entry in [e0, e1), or -1 when out of range (flagged once per entry)
  auto for_each = [&](auto&& fn) {
    int s = s0;
    for (int e = e0; e < e1; ++e) {
      while (s + 1 < B && cnt[s + 1] <= e) ++s;
      const int b = tables[(long long)s * max_blocks + (e - cnt[s])];
      fn(e, (unsigned)b < (unsigned)n ? b : -1);
    }
  };
  for_each([&](int, int b) {  // pass 1: drop the references
    if (b < 0) flag_error(err, PA_DEVERR_POOL);
    else atomicSub(refs + b, 1);
  });
  __syncthreads();
  for_each([&](int, int b) {  // pass 2: mark the blocks no one holds any more
    if (b < 0) return;
    const int v = ld_volatile(refs + b);
    if (v == 0) refs[b] = kMark;
    else if (v < 0 && v != kMark) flag_error(err, PA_DEVERR_POOL);
  });
  __syncthreads();
  for_each([&](int e, int b) {  // pass 3: the last entry of a marked block
    if (b >= 0 && ld_volatile(refs + b) < -(1 << 30)) atomicMax(refs + b, kMark + 1 + e);
  });
  __syncthreads();
  int mine = 0;
  for_each([&](int e, int b) { mine += b >= 0 && ld_volatile(refs + b) == kMark + 1 + e; });
  tsum[threadIdx.x] = mine;
  __syncthreads();
  const int pushed = block_exclusive_scan(tsum, kThreads, warp_sums);
  if (count + pushed > n) {
    // more blocks than the ring holds (not a pool state): put every count back
    if (threadIdx.x == 0) flag_error(err, PA_DEVERR_POOL);
    for_each([&](int, int b) {
      if (b >= 0 && ld_volatile(refs + b) < -(1 << 30)) refs[b] = 0;
    });
    __syncthreads();
    for_each([&](int, int b) {
      if (b >= 0) atomicAdd(refs + b, 1);
    });
    return;
  }
  const int tail = (head + count) % n;
  int pos = tsum[threadIdx.x];
  for_each([&](int e, int b) {
    if (b >= 0 && ld_volatile(refs + b) == kMark + 1 + e) {
      ring[(tail + pos) % n] = b;
      ++pos;
    }
  });
  __syncthreads();
  for_each([&](int e, int b) {  // the pushing entry clears its block's count
    if (b >= 0 && ld_volatile(refs + b) == kMark + 1 + e) refs[b] = 0;
  });
  for (int s = threadIdx.x; s < B; s += blockDim.x)
    if (finished[s]) owned[s] = 0;
  __syncthreads();
  if (threadIdx.x == 0) state[1] = count + pushed;
}

// pa_block_share: pair i gives sequence dst[i] (which must own no block) the first k[i]
// blocks of sequence src[i]'s table, one more reference each.  One warp per pair.
__global__ void __launch_bounds__(kThreads) share_kernel(
    int32_t* refs, int n, int32_t* __restrict__ tables, int max_blocks,
    int32_t* __restrict__ owned, int B, const int32_t* __restrict__ src,
    const int32_t* __restrict__ dst, const int32_t* __restrict__ nshared, int pairs, int* err) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  for (int i = warp; i < pairs; i += nwarps) {
    const int a = src[i], b = dst[i], k = nshared[i];
    bool ok = (unsigned)a < (unsigned)B && (unsigned)b < (unsigned)B && a != b;
    const int ha = ok ? owned[a] : 0;
    ok = ok && owned[b] == 0 && k >= 0 && k <= ha && ha <= max_blocks;
    if (!ok) {
      if (lane == 0) flag_error(err, PA_DEVERR_POOL);
      continue;
    }
    bool range_ok = true;
    for (int j = lane; j < k; j += 32)
      range_ok &= (unsigned)tables[(long long)a * max_blocks + j] < (unsigned)n;
    if (!__all_sync(0xffffffffu, range_ok)) {  // a table entry outside the pool
      if (lane == 0) flag_error(err, PA_DEVERR_POOL);
      continue;
    }
    for (int j = lane; j < k; j += 32) {
      const int blk = tables[(long long)a * max_blocks + j];
      tables[(long long)b * max_blocks + j] = blk;
      atomicAdd(refs + blk, 1);
    }
    __syncwarp();
    if (lane == 0) owned[b] = k;
  }
}

}  // namespace pool
}  // namespace pa

extern "C" pa_status pa_block_pool_init(int32_t* ring, int32_t* state, int32_t* block_refs,
                                        int num_blocks, void* stream) {
  pa::set_launch_count(0);
  if (num_blocks <= 0) return PA_ERR_INVALID_ARG;
  if (!ring || !state) return PA_ERR_INVALID_ARG;
  if (!pa::launch_prologue()) return PA_ERR_CUDA;
  const int blocks = std::min(1024, (num_blocks + pa::pool::kThreads - 1) / pa::pool::kThreads);
  pa::pool::init_kernel<<<blocks, pa::pool::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      ring, state, block_refs, num_blocks);
  const pa_status st = pa::check_launch();
  if (st == PA_OK) pa::set_launch_count(1);
  return st;
}

extern "C" pa_status pa_block_allocate(int32_t* ring, int32_t* state, int32_t* block_refs,
                                       int num_blocks, int32_t* block_tables,
                                       int max_blocks_per_seq, int32_t* blocks_owned,
                                       const int32_t* seq_lens, const int32_t* q_lens,
                                       int num_seqs, int block_size, int32_t* slot_mapping,
                                       int32_t* granted, void* stream) {
  pa::set_launch_count(0);
  if (num_blocks <= 0 || max_blocks_per_seq <= 0 || num_seqs < 0) return PA_ERR_INVALID_ARG;
  if (block_size != 16 && block_size != 32) return PA_ERR_UNSUPPORTED;
  if (num_seqs > pa::pool::kMaxSeqs) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (!ring || !state || !block_tables || !blocks_owned || !seq_lens || !q_lens || !slot_mapping ||
      !granted)
    return PA_ERR_INVALID_ARG;
  int* err = pa::launch_prologue();
  if (!err) return PA_ERR_CUDA;
  pa::pool::allocate_kernel<<<1, pa::pool::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      ring, state, num_blocks, block_tables, max_blocks_per_seq, blocks_owned, seq_lens, q_lens,
      num_seqs, block_size == 16 ? 4 : 5, slot_mapping, granted, block_refs, err);
  const pa_status st = pa::check_launch();
  if (st == PA_OK) pa::set_launch_count(1);
  return st;
}

extern "C" pa_status pa_block_free(int32_t* ring, int32_t* state, int32_t* block_refs,
                                   int num_blocks, const int32_t* block_tables,
                                   int max_blocks_per_seq, int32_t* blocks_owned,
                                   const int32_t* finished, int num_seqs, void* stream) {
  pa::set_launch_count(0);
  if (num_blocks <= 0 || max_blocks_per_seq <= 0 || num_seqs < 0) return PA_ERR_INVALID_ARG;
  if (num_seqs > pa::pool::kMaxSeqs) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (!ring || !state || !block_tables || !blocks_owned || !finished) return PA_ERR_INVALID_ARG;
  int* err = pa::launch_prologue();
  if (!err) return PA_ERR_CUDA;
  cudaStream_t st_ = static_cast<cudaStream_t>(stream);
  if (block_refs)
    pa::pool::free_kernel_refs<<<1, pa::pool::kThreads, 0, st_>>>(
        ring, state, block_refs, num_blocks, block_tables, max_blocks_per_seq, blocks_owned,
        finished, num_seqs, err);
  else
    pa::pool::free_kernel<<<1, pa::pool::kThreads, 0, st_>>>(
        ring, state, num_blocks, block_tables, max_blocks_per_seq, blocks_owned, finished,
        num_seqs, err);
  const pa_status st = pa::check_launch();
  if (st == PA_OK) pa::set_launch_count(1);
  return st;
}

extern "C" pa_status pa_block_share(int32_t* block_refs, int num_blocks, int32_t* block_tables,
                                    int max_blocks_per_seq, int32_t* blocks_owned, int num_seqs,
                                    const int32_t* src_seqs, const int32_t* dst_seqs,
                                    const int32_t* num_shared, int num_pairs, void* stream) {
  pa::set_launch_count(0);
  if (num_blocks <= 0 || max_blocks_per_seq <= 0 || num_seqs < 0 || num_pairs < 0)
    return PA_ERR_INVALID_ARG;
  if (num_pairs == 0) return PA_OK;
  if (!block_refs || !block_tables || !blocks_owned || !src_seqs || !dst_seqs || !num_shared)
    return PA_ERR_INVALID_ARG;
  int* err = pa::launch_prologue();
  if (!err) return PA_ERR_CUDA;
  pa::pool::share_kernel<<<1, pa::pool::kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      block_refs, num_blocks, block_tables, max_blocks_per_seq, blocks_owned, num_seqs, src_seqs,
      dst_seqs, num_shared, num_pairs, err);
  const pa_status st = pa::check_launch();
  if (st == PA_OK) pa::set_launch_count(1);
  return st;
}
