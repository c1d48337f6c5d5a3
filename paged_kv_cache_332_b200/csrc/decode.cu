// Paged decode attention (single query per sequence) for sm_100a.
//
// What it computes — page "大模型推理内存优化从 KV Cache 分页到连续批处理的工程实践":
//   section "PagedAttention 的 CUDA Kernel 实现": attention reads each key/value row
//   indirectly, first looking up the physical block of a logical block in the
//   sequence's block table, then reading the row inside that block;
//   section "工程边界与架构取舍": a decode step emits one token and reads the whole KV
//   cache of the sequence, so the pass is bound by memory bandwidth.
// For sequence s and q-head qh (kv-head h = qh / G):
//   out[s, qh] = sum_j softmax_j(scale * q[s, qh] . K[s, h, j]) V[s, h, j],  j < seq_len[s].
//
// Design on B200.  The page's kernel tricks (block-table entries in shared memory,
// coalesced in-block reads, prefetching the next block) are kept where they pay:
//  * Reads are whole physical blocks: one 4-D TMA box brings 16 tokens of K for HB
//    kv-heads (HB = all eight of a LLaMA-70B-style layer: one contiguous 32 KB block), a
//    second box the same of V.  Measured on B200, boxes of one or two kv-heads (256 or
//    512-byte runs scattered over randomly placed blocks) stream at 2.4-4.4 TB/s while
//    whole 2 KB rows stream at 7 TB/s.
//  * Balanced split-K.  The tiles of every (sequence, group of HB kv-heads) are laid end
//    to end, and CTA c of a persistent grid (one per SM) takes the c-th equal share of
//    that list.  Every CTA moves the same number of bytes, whatever the length mix, and
//    a sequence is split only where a share boundary falls inside it.  The piece of a
//    sequence that a CTA sees is a segment: a sequence held by one CTA is written to
//    `out` directly; the others leave normalised partials (o, m, l) in the caller's
//    workspace at slot c + group, merged by a log-sum-exp pass (lse_reduce_kernel).
//    An explicit partition size caps the share, so no segment is longer.
//  * One consumer warp per kv-head of the group handles all G q-heads of that kv-head,
//    so no two warps share an output.  q.k: 8 lanes split a token's 128 dims (16 each,
//    two 16-byte shared-memory reads), packed f32x2 FMAs, then a warp-shuffle halving
//    exchange that sums all G heads at once.  Online softmax (running max m, sum l) in
//    the log2 domain (q pre-scaled by scale*log2 e: one ex2 per logit); p.V with lanes
//    over head_dim.
//  * G = 8 (LLaMA-70B-style GQA) is the exception: its two contractions cost 4 FMAs per
//    byte of KV, more than the FP32 pipe sustains at HBM rate, so q.k and p.V of a tile
//    run as mma.sync m16n8k16 tensor-core fragments (fp32 accumulate); the online
//    softmax, masking and the split-K bookkeeping are the same.
//  * A staging warp cuts the CTA's share into units of at most 128 tiles and, up to two
//    units ahead, copies their block-table entries into shared memory (one coalesced
//    read per 32 entries) and starts the TMA copy of their q rows.  A producer thread
//    walks the tiles in order and issues the two boxes of each as soon as a slot of the
//    shared ring frees (blocking waits take no issue slots from the consumers).
// Two more modes share the kernel:
//  * shared prefixes (pa_decode_shared_prefix): a sequence whose first tokens are shared
//    with its group reads only its tiles after the prefix; the prefix pass (prefill.cu)
//    left the attention over the prefix as partials, and the merge folds them in;
//  * varlen rows (pa_attention_varlen): only sequences with one query row are served,
//    q and out rows come from query_start_loc, and CTA 0 lists the other sequences for
//    the prefill kernel that follows.
// Every wait is bounded; bad table entries or lengths never fault (skipped, flagged).
#include <cuda_fp8.h>

#include <algorithm>
#include <climits>
#include <mutex>
#include <type_traits>

#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {

struct DecodeArgs {
  void* out;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  float* part_o;   // [slots, HB*G, 128]   normalised partial outputs
  float* part_ml;  // [slots, HB*G, 2]     (max in log2 units, sum)
  int2* meta;      // [B * NHP]            (first slot, slot count) of each group
  // append in the same launch (k_new != nullptr): the step's new token of each sequence,
  // [B, Hkv, 128], written into its cache slot at position seq_len-1 before it is read
  const void* k_new;
  const void* v_new;
  void* k_cache;
  void* v_cache;
  // FP8 (e4m3) cache: fp32 scale of each kv-head's K and V codes, [Hkv]
  const float* k_scale;
  const float* v_scale;
  // shared-prefix decode (num_groups > 0): sequences [group_starts[g], group_starts[g+1])
  // share their first prefix_lens[g] tokens.  The prefix pass left the attention of every
  // member's q-heads over those tokens in pre_o / pre_ml ([pre_chunks][B * Hq rows],
  // normalised rows and (max in log2 units, sum)); this launch reads only the keys after
  // a sequence's prefix and the merge folds both parts together.
  const int32_t* group_starts;
  const int32_t* prefix_lens;
  const float* pre_o;
  const float* pre_ml;
  int num_groups, pre_chunks;
  // varlen batch (qsl != nullptr): only sequences with one query row (qsl[s+1]-qsl[s] == 1)
  // are served here, reading q and writing out at row qsl[s] of num_q_rows
  const int32_t* qsl;
  int num_q_rows;
  // varlen: CTA 0 also lists the sequences with more than one query row for the prefill
  // kernel that follows (chunk_ids[0..n), n = chunk_ids[chunk_cap] <= chunk_cap)
  int32_t* chunk_ids;
  int chunk_cap;
  int* err;
  int num_seqs, num_q_heads, num_kv_heads, max_blocks, log2_bs, num_blocks;
  int seq_cap;
  int ring_off, nslots;  // shared-memory offset of the tile ring and its slot count
  float qscale;          // scale * log2(e)
};

constexpr int kD = 128;
constexpr int kTileTok = 16;
constexpr int kRowBytes = kD * 2;      // one token of one kv-head
constexpr int kQSlots = 2;             // units staged ahead
constexpr int kMaxSlots = 8;
constexpr int kMaxTilesPerUnit = 128;
constexpr int kMaxGrid = 256;          // persistent grid: min(SMs, this)
// unit flags
constexpr int kFirst = 1;   // first unit of a segment: load q, reset the softmax state
constexpr int kLast = 2;    // last unit of a segment: write the result
constexpr int kDirect = 4;  // the segment is the whole group: write `out`

template <int G_, int HB_, bool F8_>
struct DecodeCfg {
  static constexpr int G = G_;
  static constexpr int HB = HB_;                  // kv-heads per group = consumer warps
  static constexpr bool F8 = F8_;                 // e4m3 cache (else fp16/bf16)
  static constexpr bool MMA = F8 || G == 8;       // tensor-core consumers
  static constexpr int KROW = kD * (F8 ? 1 : 2);  // one token of one kv-head in the cache
  static constexpr int GW = G;                    // q-heads per consumer warp
  static constexpr int WARP_PROD = 0;
  static constexpr int WARP_STAGE = 1;
  static constexpr int WARP_FILL = 2;             // zero-fills empty sequences
  static constexpr int WARP_C0 = 4;               // first consumer warp
  static constexpr int THREADS = 128 + HB * 32;
  static constexpr int DUPMASK = GW == 4 ? 1 : (GW == 2 ? 3 : 7);  // CUDA-core path (G <= 4)
  static constexpr int TILE_BYTES = kTileTok * HB * KROW;       // K (or V) of a tile
  static constexpr int SLOT_BYTES = 2 * TILE_BYTES;
  static constexpr int QBYTES = HB * G * kRowBytes;             // q rows of a group
  // shared-memory carve-up (bytes); the sequence arrays and then the ring follow
  static constexpr int OFF_FULL = 0;
  static constexpr int OFF_EMPTY = OFF_FULL + kMaxSlots * 8;
  static constexpr int OFF_QFULL = OFF_EMPTY + kMaxSlots * 8;
  static constexpr int OFF_QEMPTY = OFF_QFULL + kQSlots * 8;
  static constexpr int OFF_TFULL = OFF_QEMPTY + kQSlots * 8;
  static constexpr int OFF_TEMPTY = OFF_TFULL + kQSlots * 8;
  static constexpr int OFF_ADONE = OFF_TEMPTY + kQSlots * 8;    // append of a unit written
  static constexpr int OFF_UNIT = OFF_ADONE + kQSlots * 8;      // 8 ints per staged unit
  static constexpr int OFF_ABORT = OFF_UNIT + kQSlots * 32;
  static constexpr int OFF_TBL = ((OFF_ABORT + 16 + 127) / 128) * 128;
  static constexpr int OFF_Q = OFF_TBL + kQSlots * kMaxTilesPerUnit * 4;
  // p pairs and alpha per warp (CUDA-core path only; the G = 8 path keeps them in
  // registers, which leaves room for a third 64 KB ring slot)
  static constexpr int OFF_P = OFF_Q + kQSlots * QBYTES;
  static constexpr int OFF_A = OFF_P + (MMA ? 0 : HB * kTileTok * GW * 8);
  static constexpr int OFF_SEQ = ((OFF_A + (MMA ? 0 : HB * GW * 4) + 15) / 16) * 16;  // 3B+1 ints
  static_assert(OFF_Q % 128 == 0 && OFF_P % 16 == 0, "alignment");
};

__device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }
__device__ __forceinline__ int clamp_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }

// merge records: (first slot, slot count | kHasPrefix when prefix partials join the merge)
constexpr int kHasPrefix = 1 << 30;

// Shared-prefix length of sequence s: prefix_lens[g] of the group holding s (the last g
// with group_starts[g] <= s, if s < group_starts[g+1]), else 0.
__device__ __forceinline__ int shared_prefix_of(const DecodeArgs& a, int s) {
  if (a.num_groups <= 0 || s < __ldg(a.group_starts)) return 0;
  int lo = 0, hi = a.num_groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(a.group_starts + mid) <= s) lo = mid; else hi = mid - 1;
  }
  return s < __ldg(a.group_starts + lo + 1) ? __ldg(a.prefix_lens + lo) : 0;
}

// Bounded wait that turns into a no-op once any warp of the CTA gave up.
__device__ __forceinline__ void wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag, int* err) {
  if (*abort_flag) return;
  if (!mbar_wait(bar, parity, err)) *abort_flag = 1;
}

// Sum per-lane partial dot products over each 8-lane token group for GW heads at
// once (halving exchange).  Returns the sum for head hh(lane):
//   GW=4: hh = 2*bit2 + bit1;  GW=2: hh = bit2;
//   GW=1: hh = 0.
template <int GW>
__device__ __forceinline__ float reduce_heads(const float (&d)[GW], int lane);

template <>
__device__ __forceinline__ float reduce_heads<4>(const float (&d)[4], int lane) {
  const bool b2 = lane & 4;
  float k0 = b2 ? d[2] : d[0], k1 = b2 ? d[3] : d[1];
  const float s0 = b2 ? d[0] : d[2], s1 = b2 ? d[1] : d[3];
  k0 += __shfl_xor_sync(0xffffffffu, s0, 4);
  k1 += __shfl_xor_sync(0xffffffffu, s1, 4);
  const bool b1 = lane & 2;
  float k = b1 ? k1 : k0;
  const float s = b1 ? k0 : k1;
  k += __shfl_xor_sync(0xffffffffu, s, 2);
  k += __shfl_xor_sync(0xffffffffu, k, 1);
  return k;
}

template <>
__device__ __forceinline__ float reduce_heads<2>(const float (&d)[2], int lane) {
  const bool b2 = lane & 4;
  float k = b2 ? d[1] : d[0];
  const float s = b2 ? d[0] : d[1];
  k += __shfl_xor_sync(0xffffffffu, s, 4);
  k += __shfl_xor_sync(0xffffffffu, k, 2);
  k += __shfl_xor_sync(0xffffffffu, k, 1);
  return k;
}

template <>
__device__ __forceinline__ float reduce_heads<1>(const float (&d)[1], int lane) {
  float k = d[0];
  k += __shfl_xor_sync(0xffffffffu, k, 4);
  k += __shfl_xor_sync(0xffffffffu, k, 2);
  k += __shfl_xor_sync(0xffffffffu, k, 1);
  return k;
}

template <int GW>
__device__ __forceinline__ int head_of_lane(int lane) {
  return GW == 4 ? (((lane >> 2) & 1) * 2 + ((lane >> 1) & 1)) : (GW == 2 ? ((lane >> 2) & 1) : 0);
}

// A lane that holds head jj's value after reduce_heads (with tp = 0).
template <int GW>
__device__ __forceinline__ int lane_of_head(int jj) {
  return GW == 4 ? (((jj >> 1) << 2) | ((jj & 1) << 1)) : (GW == 2 ? jj * 4 : 0);
}


// mma.sync m16n8k16 with fp32 accumulate, A row-major / B column-major fragments, and
// the packing of two fp32 values into one register of the element type.
template <typename T>
struct Mma;
template <>
struct Mma<__nv_bfloat16> {
  static __device__ __forceinline__ void run(float (&d)[4], uint32_t a0, uint32_t a1,
                                             uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};
template <>
struct Mma<__half> {
  static __device__ __forceinline__ void run(float (&d)[4], uint32_t a0, uint32_t a1,
                                             uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
        "{%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
  }
  static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

// Two e4m3 codes (low 16 bits of x; the lower code first) -> their f16 values as one
// f16x2 register.  Exact: every e4m3 value is an f16 value.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t x) {
  const __half2_raw h =
      __nv_cvt_fp8x2_to_halfraw2(static_cast<__nv_fp8x2_storage_t>(x & 0xFFFFu), __NV_E4M3);
  return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// Transpose of an 8x8 matrix of 16-bit elements held as one fragment register per lane
// (lane l: row l/4, columns 2(l%4), 2(l%4)+1).
__device__ __forceinline__ uint32_t transpose8x8(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
  return d;
}

// CTA holding global tile `pos` when T tiles are shared out over `grid` CTAs
// (CTA c holds [c*T/grid, (c+1)*T/grid)).
__device__ __forceinline__ int cta_of(int pos, int T, int grid) {
  return (int)((((long long)pos + 1) * grid - 1) / T);
}

template <typename T, int G, int HB, bool F8>
__global__ void __launch_bounds__(DecodeCfg<G, HB, F8>::THREADS, 1)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmQ, const DecodeArgs a) {
  using C = DecodeCfg<G, HB, F8>;
  constexpr int GW = C::GW;
  constexpr int HBG = HB * G;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_FULL);
  uint64_t* empty = reinterpret_cast<uint64_t*>(smem + C::OFF_EMPTY);
  uint64_t* qfull = reinterpret_cast<uint64_t*>(smem + C::OFF_QFULL);
  uint64_t* qempty = reinterpret_cast<uint64_t*>(smem + C::OFF_QEMPTY);
  uint64_t* tfull = reinterpret_cast<uint64_t*>(smem + C::OFF_TFULL);
  uint64_t* tempty = reinterpret_cast<uint64_t*>(smem + C::OFF_TEMPTY);
  uint64_t* adone = reinterpret_cast<uint64_t*>(smem + C::OFF_ADONE);
  volatile int* unit = reinterpret_cast<volatile int*>(smem + C::OFF_UNIT);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);
  int* tbl = reinterpret_cast<int*>(smem + C::OFF_TBL);
  uint8_t* qbuf = smem + C::OFF_Q;
  float2* pbuf = reinterpret_cast<float2*>(smem + C::OFF_P);
  float* abuf = reinterpret_cast<float*>(smem + C::OFF_A);
  const int B = a.num_seqs;
  int* sstart = reinterpret_cast<int*>(smem + C::OFF_SEQ);  // [B+1] first tile of each sequence
  int* slen = sstart + B + 1;                                // [B]   clamped lengths
  int* sfirst = slen + B;  // [B] first tile after the shared prefix (0 without one)
  uint8_t* ring = smem + a.ring_off;
  const int nslots = a.nslots;
  const int NHP = a.num_kv_heads / HB;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // the merge pass may be scheduled now; it waits for this grid's results itself
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- clamped lengths and the prefix of tiles over (sequence, head group)
  if (warp == 0) {
    const int per = (B + 31) / 32;
    const int lo = min(B, lane * per), hi = min(B, lo + per);
    int sum = 0;
    for (int s = lo; s < hi; ++s) {
      const int raw = a.seq_lens[s];
      const int L = clamp_len(raw, a.seq_cap);
      if (raw != L && blockIdx.x == 0) flag_error(a.err, PA_DEVERR_SEQ_TOO_LONG);
      slen[s] = L;
      int first = 0;
      if (a.qsl != nullptr) {  // varlen: decode rows only; the others are prefill chunks
        const int q0 = __ldg(a.qsl + s), nq = __ldg(a.qsl + s + 1) - q0;
        if (nq != 1) first = -1;
        else if (q0 < 0 || q0 >= a.num_q_rows) {
          if (blockIdx.x == 0) flag_error(a.err, PA_DEVERR_QUERY_LAYOUT);
          first = -1;
        }
      }
      if (first == 0 && a.num_groups > 0) {
        const int p = shared_prefix_of(a, s);
        if ((p < 0 || p > L || (p & ((1 << a.log2_bs) - 1))) && blockIdx.x == 0)
          flag_error(a.err, PA_DEVERR_PREFIX);
        first = clamp_len(p, L) / kTileTok;
      }
      sfirst[s] = first;
      sum += first < 0 ? 0 : NHP * (cdiv(L, kTileTok) - first);
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int run = incl - sum;
    for (int s = lo; s < hi; ++s) {
      sstart[s] = run;
      run += sfirst[s] < 0 ? 0 : NHP * (cdiv(slen[s], kTileTok) - sfirst[s]);
    }
    if (lane == 31) sstart[B] = incl;
    if (a.chunk_ids != nullptr && blockIdx.x == 0) {
      int c = 0;
      for (int s = lo; s < hi; ++s) c += (__ldg(a.qsl + s + 1) - __ldg(a.qsl + s)) > 1;
      int ci = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, ci, o);
        if (lane >= o) ci += t;
      }
      int r = ci - c;
      for (int s = lo; s < hi; ++s)
        if (__ldg(a.qsl + s + 1) - __ldg(a.qsl + s) > 1) {
          if (r < a.chunk_cap) a.chunk_ids[r] = s;
          ++r;
        }
      if (lane == 31) {
        a.chunk_ids[a.chunk_cap] = min(ci, a.chunk_cap);
        if (ci > a.chunk_cap) flag_error(a.err, PA_DEVERR_QUERY_LAYOUT);
      }
    }
  }
  if (threadIdx.x == C::WARP_STAGE * 32) {
    for (int i = 0; i < nslots; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], HB);
    }
    for (int i = 0; i < kQSlots; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], HB);
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 1);
      mbar_init(&adone[i], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int Ttot = sstart[B];
  // The launch sizes the grid for the longest possible batch; when the batch holds
  // fewer tiles than CTAs, only the first Ttot CTAs take a share, so every share is
  // non-empty and the segments of a group sit in consecutive CTAs (and slots).
  const int grid = min((int)gridDim.x, max(Ttot, 1));
  const int cta = blockIdx.x;
  const int r0 = cta < grid ? (int)(((long long)cta * Ttot) / grid) : Ttot;
  const int r1 = cta < grid ? (int)(((long long)(cta + 1) * Ttot) / grid) : Ttot;

  if (warp < C::WARP_C0) {
    if (warp == C::WARP_FILL) {
      // ===== empty sequences: no CTA visits them; zero their output and merge record =====
      for (int s = cta; s < B; s += gridDim.x) {
        if (sfirst[s] < 0) {  // not served by this kernel: no merge, no output
          for (int h = lane; h < NHP; h += 32) a.meta[s * NHP + h] = make_int2(0, 0);
          continue;
        }
        if (cdiv(slen[s], kTileTok) != sfirst[s]) continue;
        // no keys of its own: a sequence with a shared prefix takes the prefix part alone
        const int pre = sfirst[s] > 0 ? kHasPrefix : 0;
        for (int h = lane; h < NHP; h += 32) a.meta[s * NHP + h] = make_int2(0, pre);
        if (pre) continue;
        const int orow = a.qsl ? __ldg(a.qsl + s) : s;
        T* ob = static_cast<T*>(a.out) + (long long)orow * a.num_q_heads * kD;
        for (int i = lane; i < a.num_q_heads * kD / 8; i += 32)
          reinterpret_cast<uint4*>(ob)[i] = make_uint4(0u, 0u, 0u, 0u);
      }
      return;
    }
    if (warp == C::WARP_STAGE) {
      // ===== staging warp: cuts the share into units; table entries + q, two units ahead =====
      if (lane == 0) prefetch_tmap(&tmQ);
      int pos = r0;
      int s = 0;
      if (pos < r1) {  // sequence holding pos: the last s with sstart[s] <= pos
        int lo = 0, hi = B - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (sstart[mid] <= pos) lo = mid; else hi = mid - 1;
        }
        s = lo;
      }
      for (int k = 0;; ++k) {
        const int qs = k % kQSlots;
        const uint32_t par = ((k / kQSlots) & 1) ^ 1;
        wait_or_abort(&qempty[qs], par, abort_flag, a.err);  // consumers read unit k-2's q
        wait_or_abort(&tempty[qs], par, abort_flag, a.err);  // its tiles were issued
        volatile int* u = unit + qs * 8;
        if (pos >= r1 || *abort_flag) {  // tell the other warps there is no more work
          if (lane == 0) {
            u[0] = -1;
            mbar_arrive_expect_tx(&qfull[qs], 0);
            mbar_arrive(&tfull[qs]);
          }
          break;
        }
        const int nt = cdiv(slen[s], kTileTok);
        const int ts = sfirst[s];         // tiles [ts, nt) are read here
        const int cnt = nt - ts;          // > 0: pos lies in this sequence
        const int off = pos - sstart[s];
        const int hp = off / cnt;
        const int t0 = ts + off - hp * cnt;
        const int t1 = min(nt, t0 + min(r1 - pos, kMaxTilesPerUnit));
        const int grp = s * NHP + hp;
        const int gs = sstart[s] + hp * cnt;  // the group's first and one-past-last tile
        const int ge = gs + cnt;
        int flags = 0;
        if (t0 == ts || pos == r0) flags |= kFirst;
        if (t1 == nt || pos + (t1 - t0) == r1) flags |= kLast;
        if (gs >= r0 && ge <= r1 && ts == 0) flags |= kDirect;
        const int32_t* trow = a.block_tables + (long long)s * a.max_blocks;
        int ids[kMaxTilesPerUnit / 32];
  #pragma unroll
        for (int j = 0; j < kMaxTilesPerUnit / 32; ++j) {
          const int t = t0 + j * 32 + lane;
          ids[j] = t < t1 ? __ldg(trow + ((t * kTileTok) >> a.log2_bs)) : -1;
        }
  #pragma unroll
        for (int j = 0; j < kMaxTilesPerUnit / 32; ++j) {
          const int i = j * 32 + lane;
          if (t0 + i < t1) {
            int id = ids[j];
            if ((unsigned)id >= (unsigned)a.num_blocks) {
              flag_error(a.err, PA_DEVERR_BLOCK_RANGE);
              id = -1;
            }
            tbl[qs * kMaxTilesPerUnit + i] = id;
          }
        }
        __syncwarp();
        // The unit holding a sequence's last tile also writes the step's new token (K and
        // V rows of the group's kv-heads, one 2 KB run each for 8 heads) into its slot.
        // The rows are loaded now, the unit is published, and the stores follow; the
        // producer waits for them (adone) only before copying that last tile.
        constexpr int kAppendVecs = (HB * 16 + 31) / 32;  // 16-byte vectors per lane
        uint4 kv_k[kAppendVecs], kv_v[kAppendVecs];
        uint4* kd = nullptr;
        uint4* vd = nullptr;
        bool append = false;
        if (a.k_new != nullptr && t1 == nt) {
          const int raw = __ldg(a.seq_lens + s);
          const int bid = tbl[qs * kMaxTilesPerUnit + (t1 - 1 - t0)];
          if (raw == slen[s] && bid >= 0) {
            append = true;
            const int row = (raw - 1) & ((1 << a.log2_bs) - 1);
            const size_t dst = ((((size_t)bid << a.log2_bs) + row) * a.num_kv_heads + hp * HB) * 16;
            const size_t src = ((size_t)s * a.num_kv_heads + hp * HB) * 16;  // in 16-byte units
            kd = static_cast<uint4*>(a.k_cache) + dst;
            vd = static_cast<uint4*>(a.v_cache) + dst;
#pragma unroll
            for (int j = 0; j < kAppendVecs; ++j) {
              const int i = j * 32 + lane;
              if (i < HB * 16) {
                kv_k[j] = __ldg(static_cast<const uint4*>(a.k_new) + src + i);
                kv_v[j] = __ldg(static_cast<const uint4*>(a.v_new) + src + i);
              }
            }
          }
        }
        if (lane == 0) {
          if (t0 == ts)
            a.meta[grp] = make_int2(cta + grp, (cta_of(ge - 1, Ttot, grid) - cta + 1) |
                                                   (ts > 0 ? kHasPrefix : 0));
          u[0] = s;
          u[1] = hp;
          u[2] = t0;
          u[3] = t1;
          u[4] = flags;
          u[5] = cta + grp;
          u[6] = append ? 1 : 0;
          u[7] = a.qsl ? __ldg(a.qsl + s) : s;  // q / out row
          if (flags & kFirst) {
            mbar_arrive_expect_tx(&qfull[qs], C::QBYTES);
            tma_load_3d(qbuf + qs * C::QBYTES, &tmQ, 0, hp * HBG, u[7], &qfull[qs]);
          } else {
            mbar_arrive_expect_tx(&qfull[qs], 0);
          }
          mbar_arrive(&tfull[qs]);
        }
        if (append) {
#pragma unroll
          for (int j = 0; j < kAppendVecs; ++j) {
            const int i = j * 32 + lane;
            if (i < HB * 16) {
              kd[i] = kv_k[j];
              vd[i] = kv_v[j];
            }
          }
          asm volatile("fence.proxy.async.global;" ::: "memory");  // before the TMA reads
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&adone[qs]);  // every unit, so phases stay one per unit
        pos += t1 - t0;
        while (s + 1 < B && sstart[s + 1] <= pos) ++s;
      }
      return;
    }

    if (warp == C::WARP_PROD) {
      // ===== producer: one thread walks every tile in order into the shared ring =====
      if (lane == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        const int bs_mask = (1 << a.log2_bs) - 1;
        int cnt = 0;
        for (int k = 0;; ++k) {
          const int qs = k % kQSlots;
          wait_or_abort(&tfull[qs], (k / kQSlots) & 1, abort_flag, a.err);
          const volatile int* u = unit + qs * 8;
          const int s = u[0];
          if (s < 0 || *abort_flag) break;
          const int hp = u[1], t0 = u[2], t1 = u[3], append = u[6];
          for (int t = t0; t < t1; ++t, ++cnt) {
            const int slot = cnt % nslots;
            // the new token's row is in the last tile: its stores must have landed
            if (append && t == t1 - 1)
              wait_or_abort(&adone[qs], (k / kQSlots) & 1, abort_flag, a.err);
            wait_or_abort(&empty[slot], ((cnt / nslots) & 1) ^ 1, abort_flag, a.err);
            const int bid = *abort_flag ? -1 : tbl[qs * kMaxTilesPerUnit + (t - t0)];
            mbar_arrive_expect_tx(&full[slot], bid >= 0 ? C::SLOT_BYTES : 0);
            if (bid >= 0) {
              const int row = (t * kTileTok) & bs_mask;
              uint8_t* dst = ring + slot * C::SLOT_BYTES;
              tma_load_4d(dst, &tmK, 0, hp * HB, row, bid, &full[slot]);
              tma_load_4d(dst + C::TILE_BYTES, &tmV, 0, hp * HB, row, bid, &full[slot]);
            }
          }
          mbar_arrive(&tempty[qs]);
        }
      }
      return;
    }

    return;  // warp 3 idles
  }

  // ===================== consumer warps: warp w <-> kv-head hp*HB + w =====================
  const int w = warp - C::WARP_C0;
  if constexpr (C::MMA) {
    // Tensor-core consumer (G = 8, and every G on an FP8 cache).  Per 16-token tile: S^T = K Q^T (M = 16 tokens, N = 8
    // q-heads, K = 128 dims: 8 MMAs) and O^T += V^T P^T (M = 128 dims in 8 tiles, N = 8
    // q-heads, K = 16 tokens: 8 MMAs).  Lane (g, tq) = (lane/4, lane%4) holds the logits
    // of tokens g and g+8 for q-heads 2tq and 2tq+1, and the output of those two heads
    // for dims [16g, 16g+16).  The contraction over dims may take the dims in any order
    // as long as K and Q agree: k-step 2j (2j+1) uses the first (last) two dim pairs of
    // the 16-byte chunk tq + 4j, so each fragment register is one aligned 32-bit read.
    // FP8: the same tile with e4m3 K/V converted to f16 on the way into the fragments
    // (exact: every e4m3 value is an f16 value), q rounded to f16 once per segment, the
    // K scale folded into the logit scale and the V scale into the final normalisation;
    // with G < 8 the q-heads past G are zero columns of the MMAs and are not written.
    using MT = typename std::conditional<F8, __half, T>::type;  // MMA operand type
    constexpr int RS = HB * C::KROW;  // bytes between consecutive tokens of a tile
    const int g = lane >> 2, tq = lane & 3;
    uint32_t qf[8][2];  // Q^T fragments of the 8 k-steps
    float oacc[8][4];   // O^T: [m-tile mt] dims 16g+mt / 16g+8+mt x heads 2tq, 2tq+1
    float mh0 = -INFINITY, mh1 = -INFINITY, lh0 = 0.f, lh1 = 0.f;  // heads 2tq, 2tq+1
    int cnt = 0;
    for (int k = 0;; ++k) {
      const int qs = k % kQSlots;
      wait_or_abort(&qfull[qs], (k / kQSlots) & 1, abort_flag, a.err);
      const volatile int* u = unit + qs * 8;
      const int s = u[0];
      if (s < 0 || *abort_flag) break;
      const int hp = u[1], t0 = u[2], t1 = u[3], flags = u[4], pslot = u[5], orow = u[7];
      if (flags & kFirst) {
        const uint8_t* qrow = qbuf + qs * C::QBYTES + (w * G + g) * kRowBytes;
        if constexpr (F8) {
          // k-step 4c+i takes dims 4i..4i+3 of the 16-dim chunk tq + 4c (one 32-bit
          // word of e4m3 codes); Q takes the same dims, as f16 pairs
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint8_t* src = qrow + (tq + 4 * c) * 32;
            uint32_t wq[8];
            *reinterpret_cast<uint4*>(wq) = *reinterpret_cast<const uint4*>(src);
            *reinterpret_cast<uint4*>(wq + 4) = *reinterpret_cast<const uint4*>(src + 16);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const float2 f = Elem<T>::unpack2(wq[i]);
              wq[i] = g < G ? Mma<__half>::pack(f.x, f.y) : 0u;
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              qf[4 * c + i][0] = wq[2 * i];
              qf[4 * c + i][1] = wq[2 * i + 1];
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 v = *reinterpret_cast<const uint4*>(qrow + (tq + 4 * j) * 16);
            qf[2 * j][0] = v.x;
            qf[2 * j][1] = v.y;
            qf[2 * j + 1][0] = v.z;
            qf[2 * j + 1][1] = v.w;
          }
        }
        mh0 = mh1 = -INFINITY;
        lh0 = lh1 = 0.f;
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&qempty[qs]);
      const int L = slen[s];
      const int kvh = hp * HB + w;
      const float lsc = F8 ? a.qscale * __ldg(a.k_scale + kvh) : a.qscale;

      for (int t = t0; t < t1; ++t, ++cnt) {
        const int slot = cnt % nslots;
        wait_or_abort(&full[slot], (cnt / nslots) & 1, abort_flag, a.err);
        const int nvalid = min(kTileTok, L - t * kTileTok);
        // tile layout (TMA box): [16 tokens][HB kv-heads][128 dims]
        const uint8_t* Ks = ring + slot * C::SLOT_BYTES + w * C::KROW;
        const uint8_t* Vs = Ks + C::TILE_BYTES;

        // ---- S^T = K Q^T: rows tokens g, g+8; columns heads 2tq, 2tq+1
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (F8) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint4 ka = *reinterpret_cast<const uint4*>(Ks + g * RS + (tq + 4 * c) * 16);
            const uint4 kb = *reinterpret_cast<const uint4*>(Ks + (g + 8) * RS + (tq + 4 * c) * 16);
            const uint32_t wa[4] = {ka.x, ka.y, ka.z, ka.w}, wb[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
              Mma<__half>::run(sc, e4m3x2_to_f16x2(wa[i]), e4m3x2_to_f16x2(wb[i]),
                               e4m3x2_to_f16x2(wa[i] >> 16), e4m3x2_to_f16x2(wb[i] >> 16),
                               qf[4 * c + i][0], qf[4 * c + i][1]);
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 ka = *reinterpret_cast<const uint4*>(Ks + g * RS + (tq + 4 * j) * 16);
            const uint4 kb = *reinterpret_cast<const uint4*>(Ks + (g + 8) * RS + (tq + 4 * j) * 16);
            Mma<T>::run(sc, ka.x, kb.x, ka.y, kb.y, qf[2 * j][0], qf[2 * j][1]);
            Mma<T>::run(sc, ka.z, kb.z, ka.w, kb.w, qf[2 * j + 1][0], qf[2 * j + 1][1]);
          }
        }
        // ---- online softmax over the tile (log2 domain), per head
        const bool v0 = g < nvalid, v8 = g + 8 < nvalid;
        const float x0 = v0 ? sc[0] * lsc : -INFINITY;  // token g,   head 2tq
        const float x1 = v0 ? sc[1] * lsc : -INFINITY;  // token g,   head 2tq+1
        const float x2 = v8 ? sc[2] * lsc : -INFINITY;  // token g+8, head 2tq
        const float x3 = v8 ? sc[3] * lsc : -INFINITY;  // token g+8, head 2tq+1
        float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
        }
        const float mn0 = fmaxf(mh0, mx0), mn1 = fmaxf(mh1, mx1);
        const float al0 = fast_exp2(mh0 - mn0), al1 = fast_exp2(mh1 - mn1);  // -inf -> 0
        mh0 = mn0;
        mh1 = mn1;
        const float p0 = fast_exp2(x0 - mn0), p1 = fast_exp2(x1 - mn1);
        const float p2 = fast_exp2(x2 - mn0), p3 = fast_exp2(x3 - mn1);
        lh0 = lh0 * al0 + (p0 + p2);
        lh1 = lh1 * al1 + (p1 + p3);
        if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
          const float2 al = make_float2(al0, al1);
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            const float2 lo = __fmul2_rn(make_float2(oacc[mt][0], oacc[mt][1]), al);
            const float2 hi = __fmul2_rn(make_float2(oacc[mt][2], oacc[mt][3]), al);
            oacc[mt][0] = lo.x;
            oacc[mt][1] = lo.y;
            oacc[mt][2] = hi.x;
            oacc[mt][3] = hi.y;
          }
        }
        // ---- P^T fragments: [tokens 2tq, 2tq+1 | 8+2tq, 9+2tq] x head g
        const uint32_t pb0 = transpose8x8(Mma<MT>::pack(p0, p1));
        const uint32_t pb1 = transpose8x8(Mma<MT>::pack(p2, p3));
        // ---- V^T fragments: dims [16g, 16g+16) of tokens 2tq, 2tq+1, 2tq+8, 2tq+9,
        // paired along tokens; rows past the sequence end are zeroed (p is 0 there, but
        // the block's unused rows may hold anything)
        uint32_t vw[4][8];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int tk = 2 * tq + (i & 1) + (i >> 1) * 8;
          uint4 lo, hi;
          if constexpr (F8) {  // 16 e4m3 codes -> 8 f16 pairs
            const uint4 c8 = *reinterpret_cast<const uint4*>(Vs + tk * RS + g * 16);
            lo = make_uint4(e4m3x2_to_f16x2(c8.x), e4m3x2_to_f16x2(c8.x >> 16),
                            e4m3x2_to_f16x2(c8.y), e4m3x2_to_f16x2(c8.y >> 16));
            hi = make_uint4(e4m3x2_to_f16x2(c8.z), e4m3x2_to_f16x2(c8.z >> 16),
                            e4m3x2_to_f16x2(c8.w), e4m3x2_to_f16x2(c8.w >> 16));
          } else {
            lo = *reinterpret_cast<const uint4*>(Vs + tk * RS + g * 32);
            hi = *reinterpret_cast<const uint4*>(Vs + tk * RS + g * 32 + 16);
          }
          const bool ok = tk < nvalid;
          vw[i][0] = ok ? lo.x : 0u;
          vw[i][1] = ok ? lo.y : 0u;
          vw[i][2] = ok ? lo.z : 0u;
          vw[i][3] = ok ? lo.w : 0u;
          vw[i][4] = ok ? hi.x : 0u;
          vw[i][5] = ok ? hi.y : 0u;
          vw[i][6] = ok ? hi.z : 0u;
          vw[i][7] = ok ? hi.w : 0u;
        }
        // ---- O^T += V^T P^T, m-tile mt: rows dims 16g+mt (g) and 16g+8+mt (g+8)
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          const int r = mt >> 1;
          const uint32_t sel = (mt & 1) ? 0x7632u : 0x5410u;
          const uint32_t a0 = __byte_perm(vw[0][r], vw[1][r], sel);
          const uint32_t a1 = __byte_perm(vw[0][4 + r], vw[1][4 + r], sel);
          const uint32_t a2 = __byte_perm(vw[2][r], vw[3][r], sel);
          const uint32_t a3 = __byte_perm(vw[2][4 + r], vw[3][4 + r], sel);
          Mma<MT>::run(oacc[mt], a0, a1, a2, a3, pb0, pb1);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
      }
      if (!(flags & kLast)) continue;

      // ---- end of segment: sums over the 8 token rows g, then heads 2tq and 2tq+1
      float lt0 = lh0, lt1 = lh1;
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        lt0 += __shfl_xor_sync(0xffffffffu, lt0, o);
        lt1 += __shfl_xor_sync(0xffffffffu, lt1, o);
      }
      const float vsc = F8 ? __ldg(a.v_scale + kvh) : 1.f;
      const float inv0 = lt0 > 0.f ? vsc / lt0 : 0.f;
      const float inv1 = lt1 > 0.f ? vsc / lt1 : 0.f;
      const int j0 = w * G + 2 * tq;  // q-heads j0, j0+1 within the group
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        if (2 * tq + e >= G) continue;  // a zero column (G < 8)
        const float inv = e ? inv1 : inv0;
        if (flags & kDirect) {
          uint32_t pk[8];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            pk[i] = Elem<T>::pack2(oacc[2 * i][e] * inv, oacc[2 * i + 1][e] * inv);
            pk[4 + i] = Elem<T>::pack2(oacc[2 * i][2 + e] * inv, oacc[2 * i + 1][2 + e] * inv);
          }
          T* ob = static_cast<T*>(a.out) +
                  ((long long)orow * a.num_q_heads + hp * HBG + j0 + e) * kD + 16 * g;
          reinterpret_cast<uint4*>(ob)[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          reinterpret_cast<uint4*>(ob)[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else {
          const long long row = (long long)pslot * HBG + j0 + e;
          float4* po = reinterpret_cast<float4*>(a.part_o + row * kD + 16 * g);
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            po[i] = make_float4(oacc[4 * i][e] * inv, oacc[4 * i + 1][e] * inv,
                                oacc[4 * i + 2][e] * inv, oacc[4 * i + 3][e] * inv);
            po[2 + i] = make_float4(oacc[4 * i][2 + e] * inv, oacc[4 * i + 1][2 + e] * inv,
                                    oacc[4 * i + 2][2 + e] * inv, oacc[4 * i + 3][2 + e] * inv);
          }
          if (g == 0)
            *reinterpret_cast<float2*>(a.part_ml + row * 2) =
                make_float2(e ? mh1 : mh0, e ? lt1 : lt0);
        }
      }
    }
    return;
  } else {
    const int sub = lane & 7;
    const int tp = lane >> 3;
    const int hh = head_of_lane<GW>(lane);
    const bool writer = (lane & C::DUPMASK) == 0;
    float2* pw = pbuf + w * kTileTok * GW;
    int cnt = 0;
    float2 q2[GW][8];  // q of this warp's G heads (dims of lane `sub`), log2-domain scaled
    float m = -INFINITY, l = 0.f;
    float2 acc[GW][2];

    for (int k = 0;; ++k) {
      const int qs = k % kQSlots;
      wait_or_abort(&qfull[qs], (k / kQSlots) & 1, abort_flag, a.err);
      const volatile int* u = unit + qs * 8;
      const int s = u[0];
      if (s < 0 || *abort_flag) break;
      const int hp = u[1], t0 = u[2], t1 = u[3], flags = u[4], pslot = u[5], orow = u[7];
      if (flags & kFirst) {
        // dims [8*sub, 8*sub+8) and [64+8*sub, 64+8*sub+8) as (even, odd) pairs
        const uint8_t* qb = qbuf + qs * C::QBYTES + w * G * kRowBytes;
#pragma unroll
        for (int j = 0; j < GW; ++j) {
          const uint4 w0 = *reinterpret_cast<const uint4*>(qb + j * kRowBytes + sub * 16);
          const uint4 w1 = *reinterpret_cast<const uint4*>(qb + j * kRowBytes + 128 + sub * 16);
          const uint32_t wd[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float2 f = Elem<T>::unpack2(wd[i]);
            q2[j][i] = make_float2(f.x * a.qscale, f.y * a.qscale);
          }
        }
        m = -INFINITY;
        l = 0.f;
#pragma unroll
        for (int j = 0; j < GW; ++j) acc[j][0] = acc[j][1] = make_float2(0.f, 0.f);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&qempty[qs]);
      const int L = slen[s];

      for (int t = t0; t < t1; ++t, ++cnt) {
        const int slot = cnt % nslots;
        wait_or_abort(&full[slot], (cnt / nslots) & 1, abort_flag, a.err);
        const int nvalid = min(kTileTok, L - t * kTileTok);
        // tile layout (TMA box): [16 tokens][HB kv-heads][128 dims]
        const uint8_t* Ks = ring + slot * C::SLOT_BYTES + w * kRowBytes;
        const uint8_t* Vs = Ks + C::TILE_BYTES;

        // ---- logits of the tile's 16 tokens (4 passes of 4 tokens)
        float x[4];
#pragma unroll
        for (int ps = 0; ps < 4; ++ps) {
          const int rr = ps * 4 + tp;
          const uint8_t* kr = Ks + rr * (HB * kRowBytes);
          const uint4 w0 = *reinterpret_cast<const uint4*>(kr + sub * 16);
          const uint4 w1 = *reinterpret_cast<const uint4*>(kr + 128 + sub * 16);
          const uint32_t wd[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
          float2 kf[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) kf[i] = Elem<T>::unpack2(wd[i]);
          float d[GW];
#pragma unroll
          for (int jj = 0; jj < GW; ++jj) {
            float2 e = make_float2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 8; ++i) e = __ffma2_rn(q2[jj][i], kf[i], e);
            d[jj] = e.x + e.y;
          }
          const float xv = reduce_heads<GW>(d, lane);
          x[ps] = rr < nvalid ? xv : -INFINITY;
        }
        // ---- online softmax over the tile, per head hh
        float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m, mx);
        const float alpha = fast_exp2(m - m_new);  // m = -inf -> 0
        m = m_new;
        float psum = 0.f;
#pragma unroll
        for (int ps = 0; ps < 4; ++ps) {
          const float pv = fast_exp2(x[ps] - m_new);  // masked -> 0
          psum += pv;
          if (writer) pw[(ps * 4 + tp) * GW + hh] = make_float2(pv, pv);
        }
        l = l * alpha + psum;
        if (writer && tp == 0) abuf[w * GW + hh] = alpha;
        __syncwarp();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int jj = 0; jj < GW; ++jj) {
            const float al = abuf[w * GW + jj];
            const float2 a2 = make_float2(al, al);
            acc[jj][0] = __fmul2_rn(acc[jj][0], a2);
            acc[jj][1] = __fmul2_rn(acc[jj][1], a2);
          }
        }
        // ---- p.V: lane owns dims [4*lane, 4*lane+4)
        auto pv_row = [&](int tt) {
          const uint2 vw = *reinterpret_cast<const uint2*>(Vs + tt * (HB * kRowBytes) + lane * 8);
          const float2 v01 = Elem<T>::unpack2(vw.x), v23 = Elem<T>::unpack2(vw.y);
#pragma unroll
          for (int jj = 0; jj < GW; ++jj) {
            const float2 pp = pw[tt * GW + jj];
            acc[jj][0] = __ffma2_rn(pp, v01, acc[jj][0]);
            acc[jj][1] = __ffma2_rn(pp, v23, acc[jj][1]);
          }
        };
        if (nvalid == kTileTok) {
#pragma unroll
          for (int tt = 0; tt < kTileTok; ++tt) pv_row(tt);
        } else {
          for (int tt = 0; tt < nvalid; ++tt) pv_row(tt);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
      }
      if (!(flags & kLast)) continue;

      // ---- end of segment: l summed over the 4 token groups; m and l of every head
      float lt = l + __shfl_xor_sync(0xffffffffu, l, 8);
      lt += __shfl_xor_sync(0xffffffffu, lt, 16);
#pragma unroll
      for (int jj = 0; jj < GW; ++jj) {
        const float lj = __shfl_sync(0xffffffffu, lt, lane_of_head<GW>(jj));
        const float mj = __shfl_sync(0xffffffffu, m, lane_of_head<GW>(jj));
        const float inv = lj > 0.f ? 1.f / lj : 0.f;
        const int j = w * G + jj;  // q-head within the group
        const float o0 = acc[jj][0].x * inv, o1 = acc[jj][0].y * inv;
        const float o2 = acc[jj][1].x * inv, o3 = acc[jj][1].y * inv;
        if (flags & kDirect) {
          T* ob = static_cast<T*>(a.out) + ((long long)orow * a.num_q_heads + hp * HBG + j) * kD +
                  lane * 4;
          *reinterpret_cast<uint2*>(ob) = make_uint2(Elem<T>::pack2(o0, o1), Elem<T>::pack2(o2, o3));
        } else {
          const long long row = (long long)pslot * HBG + j;
          *reinterpret_cast<float4*>(a.part_o + row * kD + lane * 4) = make_float4(o0, o1, o2, o3);
          if (lane == 0) *reinterpret_cast<float2*>(a.part_ml + row * 2) = make_float2(mj, lj);
        }
      }
    }
  }  // G < 8
}

// Log-sum-exp merge of the split-K partials: one warp per (sequence, q-head), lanes
// over head_dim.  o = sum_i w_i o_i / sum_i w_i with w_i = l_i * 2^(m_i - M), M the
// largest m_i, over the segments i of the (sequence, head group), which sit in
// consecutive slots, and the sequence's shared-prefix partials.
//
// Fold the segments of one output row into (M, den, num): the n slots of this launch
// (rows row0 + i * hbg) and, with PRE, the npre shared-prefix partials (row gw of each).
// One pass with a running maximum: up to eight segments per round, all loads of a round
// in flight together (most groups span fewer than eight CTAs: one round).
template <bool PRE>
__device__ __forceinline__ void fold_segments(const DecodeArgs& a, long long row0, int hbg,
                                              int n, int npre, int gw, int lane, float& M,
                                              float& den, float4& num) {
  const int total = n + (PRE ? npre : 0);
  const long long prow_stride = (long long)a.num_seqs * a.num_q_heads;
  for (int i0 = 0; i0 < total; i0 += 8) {
    float2 mlv[8];
    float4 ov[8];
    float Mr = -INFINITY;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int i = i0 + u;
      if (i < total) {
        if (!PRE || i < n) {
          const long long row = row0 + (long long)i * hbg;
          mlv[u] = *reinterpret_cast<const float2*>(a.part_ml + row * 2);
          ov[u] = *reinterpret_cast<const float4*>(a.part_o + row * kD + lane * 4);
        } else {
          const long long row = (long long)(i - n) * prow_stride + gw;
          mlv[u] = *reinterpret_cast<const float2*>(a.pre_ml + row * 2);
          ov[u] = *reinterpret_cast<const float4*>(a.pre_o + row * kD + lane * 4);
        }
        Mr = fmaxf(Mr, mlv[u].x);
      }
    }
    const float Mn = fmaxf(M, Mr);
    if (Mn == -INFINITY) continue;  // only empty segments so far
    const float sc = fast_exp2(M - Mn);  // M = -inf -> 0
    den *= sc;
    num.x *= sc; num.y *= sc; num.z *= sc; num.w *= sc;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (i0 + u < total) {
        const float f = mlv[u].x == -INFINITY ? 0.f : fast_exp2(mlv[u].x - Mn) * mlv[u].y;
        den += f;
        num.x += f * ov[u].x; num.y += f * ov[u].y; num.z += f * ov[u].z; num.w += f * ov[u].w;
      }
    }
    M = Mn;
  }
}

template <typename T>
__global__ void __launch_bounds__(256) lse_reduce_kernel(const DecodeArgs a, int hbg) {
  // launched as a programmatic dependent of the decode kernel: its CTAs may start while
  // the decode grid drains; this waits until that grid has finished and its writes are
  // visible (a no-op when launched without the dependency)
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= a.num_seqs * a.num_q_heads) return;
  const int s = gw / a.num_q_heads;
  const int qh = gw - s * a.num_q_heads;
  const int nhp = a.num_q_heads / hbg;
  const int j = qh % hbg;
  const int2 mt = a.meta[s * nhp + qh / hbg];
  const int n = mt.y & (kHasPrefix - 1);                 // segments of this launch
  const int npre = (mt.y & kHasPrefix) ? a.pre_chunks : 0;  // shared-prefix partials
  if (n <= 1 && npre == 0) return;  // written by the decode kernel
  const long long row0 = (long long)mt.x * hbg + j;
  float M = -INFINITY, den = 0.f;
  float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
  if (npre == 0)
    fold_segments<false>(a, row0, hbg, n, 0, gw, lane, M, den, num);
  else
    fold_segments<true>(a, row0, hbg, n, npre, gw, lane, M, den, num);
  const float inv = den > 0.f ? 1.f / den : 0.f;
  const long long orow = a.qsl ? __ldg(a.qsl + s) : s;
  T* ob = static_cast<T*>(a.out) + (orow * a.num_q_heads + qh) * kD + lane * 4;
  *reinterpret_cast<uint2*>(ob) =
      make_uint2(Elem<T>::pack2(num.x * inv, num.y * inv), Elem<T>::pack2(num.z * inv, num.w * inv));
}

constexpr int kMaxPartition = kMaxTilesPerUnit * kTileTok;
constexpr int kMaxSeqs = 4096;
constexpr int kMaxSmem = 227 * 1024;

// kv-heads per group: all of them up to eight (whole 2 KB rows for 8 heads of 128)
inline int heads_per_item(int num_kv_heads) {
  for (int hb = 8; hb > 1; hb >>= 1)
    if (num_kv_heads % hb == 0) return hb;
  return 1;
}

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace of one launch: merge records, then partial outputs, then (m, l) pairs.
struct WsLayout {
  size_t meta, part_o, part_ml, total;
};
inline WsLayout ws_layout(long long groups, long long slots, int hbg, int head_dim) {
  WsLayout w;
  w.meta = 0;
  w.part_o = align256((size_t)groups * sizeof(int2));
  w.part_ml = w.part_o + (size_t)slots * hbg * head_dim * sizeof(float);
  w.total = w.part_ml + (size_t)slots * hbg * 2 * sizeof(float);
  return w;
}

template <typename T, int G, int HB, bool F8>
pa_status launch_decode(const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQ,
                        DecodeArgs a, int grid, cudaStream_t stream) {
  using C = DecodeCfg<G, HB, F8>;
  const size_t ring_off = ((C::OFF_SEQ + (size_t)(3 * a.num_seqs + 1) * 4 + 1023) / 1024) * 1024;
  const long long room = (long long)kMaxSmem - (long long)ring_off;
  const int nslots = (int)std::min<long long>(kMaxSlots, room / C::SLOT_BYTES);
  if (nslots < 2) return PA_ERR_UNSUPPORTED;
  a.ring_off = (int)ring_off;
  a.nslots = nslots;
  const size_t smem = ring_off + (size_t)nslots * C::SLOT_BYTES;
  auto kern = paged_decode_kernel<T, G, HB, F8>;
  if (!ensure_dynamic_smem(reinterpret_cast<const void*>(kern), (int)smem)) return PA_ERR_CUDA;
  kern<<<grid, C::THREADS, smem, stream>>>(tmK, tmV, tmQ, a);
  if (check_launch() != PA_OK) return PA_ERR_CUDA;
  int launches = 1;
  if (grid > 1 || a.num_groups > 0) {
    const int warps = a.num_seqs * a.num_q_heads;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)((warps + 7) / 8));
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, lse_reduce_kernel<T>, a, HB * G) != cudaSuccess)
      return PA_ERR_CUDA;
    if (check_launch() != PA_OK) return PA_ERR_CUDA;
    ++launches;
  }
  set_launch_count(launches);
  return PA_OK;
}

template <typename T, int G, bool F8>
pa_status dispatch_hb(int HB, const CUtensorMap& tmK, const CUtensorMap& tmV,
                      const CUtensorMap& tmQ, const DecodeArgs& a, int grid, cudaStream_t stream) {
  switch (HB) {
    case 1: return launch_decode<T, G, 1, F8>(tmK, tmV, tmQ, a, grid, stream);
    case 2: return launch_decode<T, G, 2, F8>(tmK, tmV, tmQ, a, grid, stream);
    case 4: return launch_decode<T, G, 4, F8>(tmK, tmV, tmQ, a, grid, stream);
    case 8: return launch_decode<T, G, 8, F8>(tmK, tmV, tmQ, a, grid, stream);
    default: return PA_ERR_UNSUPPORTED;
  }
}

template <typename T, bool F8>
pa_status dispatch_group(int G, int HB, const CUtensorMap& tmK, const CUtensorMap& tmV,
                         const CUtensorMap& tmQ, const DecodeArgs& a, int grid,
                         cudaStream_t stream) {
  switch (G) {
    case 1: return dispatch_hb<T, 1, F8>(HB, tmK, tmV, tmQ, a, grid, stream);
    case 2: return dispatch_hb<T, 2, F8>(HB, tmK, tmV, tmQ, a, grid, stream);
    case 4: return dispatch_hb<T, 4, F8>(HB, tmK, tmV, tmQ, a, grid, stream);
    case 8: return dispatch_hb<T, 8, F8>(HB, tmK, tmV, tmQ, a, grid, stream);
    default: return PA_ERR_UNSUPPORTED;
  }
}

}  // namespace pa

extern "C" size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int head_dim,
                                           int max_seq_len, int partition_size) {
  if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_seq_len < 0 ||
      partition_size < 0)
    return 0;
  // Bounds over every kv-head count: groups <= B*Hq; partial rows = (grid + groups) *
  // (q-heads per group) <= grid*Hq + B*Hq, grid <= kMaxGrid + (tiles / tiles per
  // partition when a partition is given).
  const long long B = num_seqs, Hq = num_q_heads;
  long long rows = ((long long)pa::kMaxGrid + B) * Hq;
  if (partition_size > 0) {
    const long long nt = (max_seq_len + pa::kTileTok - 1) / pa::kTileTok;
    const long long tpp = std::max(1, partition_size / pa::kTileTok);
    rows += B * Hq * ((nt + tpp - 1) / tpp) + Hq;
  }
  return pa::align256((size_t)B * Hq * sizeof(int2)) +
         (size_t)rows * (head_dim + 2) * sizeof(float);
}

namespace {
// Groups of sequences sharing a prefix (pa_decode_shared_prefix).
struct SharedPrefixArgs {
  const int32_t* group_starts;
  const int32_t* prefix_lens;
  int num_groups, max_group_size, max_prefix_len;
};

// pa_decode, pa_decode_append when k_new / v_new are given, pa_decode_fp8 with scales,
// pa_decode_shared_prefix with `sp`
pa_status decode_impl(void* out, const void* q, const void* k_new, const void* v_new,
                      const void* k_cache, const void* v_cache, const float* k_scale,
                      const float* v_scale, const int32_t* block_tables,
                      int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                      int num_q_heads, int num_kv_heads, int head_dim, float scale,
                      int block_size, int num_blocks, int max_seq_len, int partition_size,
                      void* workspace, size_t workspace_bytes, pa_dtype dtype, void* stream,
                      const SharedPrefixArgs* sp = nullptr, const int32_t* qsl = nullptr,
                      int num_q_rows = 0, int32_t* chunk_ids = nullptr, int chunk_cap = 0) {
  pa::set_launch_count(0);
  if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
      block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0 || max_seq_len < 0 ||
      partition_size < 0)
    return PA_ERR_INVALID_ARG;
  if (dtype != PA_F16 && dtype != PA_BF16) return PA_ERR_UNSUPPORTED;
  if (head_dim != 128 || (block_size != 16 && block_size != 32)) return PA_ERR_UNSUPPORTED;
  if (num_q_heads % num_kv_heads) return PA_ERR_INVALID_ARG;
  const int G = num_q_heads / num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8) return PA_ERR_UNSUPPORTED;
  if (partition_size % 16) return PA_ERR_INVALID_ARG;
  if (partition_size > pa::kMaxPartition) return PA_ERR_UNSUPPORTED;
  if (num_seqs == 0) return PA_OK;
  if (num_seqs > pa::kMaxSeqs) return PA_ERR_UNSUPPORTED;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens) return PA_ERR_INVALID_ARG;
  if (((uintptr_t)out | (uintptr_t)q | (uintptr_t)k_cache | (uintptr_t)v_cache) & 15)
    return PA_ERR_INVALID_ARG;
  if ((k_new == nullptr) != (v_new == nullptr)) return PA_ERR_INVALID_ARG;
  if (((uintptr_t)k_new | (uintptr_t)v_new) & 15) return PA_ERR_INVALID_ARG;
  const bool f8 = k_scale != nullptr;
  if (f8 && (!v_scale || k_new)) return PA_ERR_INVALID_ARG;

  const int HB = pa::heads_per_item(num_kv_heads);
  const int NHP = num_kv_heads / HB;
  const int HBG = HB * G;
  const long long cap_tbl = (long long)max_blocks_per_seq * block_size;
  const int seq_cap = (int)std::min<long long>(cap_tbl, max_seq_len);
  const long long nt_max = (seq_cap + pa::kTileTok - 1) / pa::kTileTok;
  const long long tiles_max = (long long)num_seqs * NHP * nt_max;
  if (tiles_max > INT_MAX / 2) return PA_ERR_UNSUPPORTED;
  // persistent grid of one CTA per SM; an explicit partition caps each CTA's share
  long long grid = std::min<long long>(std::max(1, pa::num_sms()), pa::kMaxGrid);
  grid = std::max<long long>(1, std::min<long long>(grid, tiles_max));
  if (partition_size > 0)
    grid = std::max<long long>(grid, (tiles_max + partition_size / 16 - 1) / (partition_size / 16));
  const long long groups = (long long)num_seqs * NHP;
  const pa::WsLayout lay = pa::ws_layout(groups, grid + groups, HBG, head_dim);
  // shared prefix: the prefix pass's partial rows follow the decode workspace
  pa::SharedPrefixPlan plan = {};
  size_t pre_off = 0, need = lay.total;
  if (sp) {
    plan = pa::plan_shared_prefix(sp->num_groups, num_kv_heads, G, sp->max_group_size,
                                  sp->max_prefix_len);
    pre_off = pa::align256(lay.total);
    need = pre_off + (size_t)plan.slots * num_seqs * num_q_heads * (head_dim + 2) * sizeof(float);
  }
  if (!workspace || workspace_bytes < need) return PA_ERR_WORKSPACE_TOO_SMALL;
  if ((uintptr_t)workspace & 255) return PA_ERR_INVALID_ARG;
  int* err = pa::device_error_flag();
  if (!err) return PA_ERR_CUDA;

  CUtensorMap tmK, tmV, tmQ;
  const uint64_t row = (uint64_t)head_dim * 2;
  const uint64_t crow = (uint64_t)head_dim * (f8 ? 1 : 2);  // one kv-head of one token
  const uint64_t cdims[4] = {(uint64_t)head_dim, (uint64_t)num_kv_heads, (uint64_t)block_size,
                             (uint64_t)num_blocks};
  const uint64_t cstr[3] = {crow, crow * num_kv_heads, crow * num_kv_heads * block_size};
  const uint32_t cbox[4] = {(uint32_t)head_dim, (uint32_t)HB, 16, 1};
  const uint64_t qdims[3] = {(uint64_t)head_dim, (uint64_t)num_q_heads,
                             (uint64_t)(qsl ? num_q_rows : num_seqs)};
  const uint64_t qstr[2] = {row, row * num_q_heads};
  const uint32_t qbox[3] = {(uint32_t)head_dim, (uint32_t)HBG, 1};
  const CUtensorMapDataType ct =
      f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
  if (!pa::encode_tmap(&tmK, ct, k_cache, 4, cdims, cstr, cbox, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !pa::encode_tmap(&tmV, ct, v_cache, 4, cdims, cstr, cbox, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !pa::encode_tmap_16bit(&tmQ, q, 3, qdims, qstr, qbox, CU_TENSOR_MAP_SWIZZLE_NONE))
    return PA_ERR_CUDA;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  pa::DecodeArgs a;
  a.out = out;
  a.block_tables = block_tables;
  a.seq_lens = seq_lens;
  a.meta = reinterpret_cast<int2*>(ws + lay.meta);
  a.k_new = k_new;
  a.v_new = v_new;
  a.k_cache = const_cast<void*>(k_cache);
  a.v_cache = const_cast<void*>(v_cache);
  a.k_scale = k_scale;
  a.v_scale = v_scale;
  a.part_o = reinterpret_cast<float*>(ws + lay.part_o);
  a.part_ml = reinterpret_cast<float*>(ws + lay.part_ml);
  a.err = err;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.max_blocks = max_blocks_per_seq;
  a.log2_bs = block_size == 16 ? 4 : 5;
  a.num_blocks = num_blocks;
  a.seq_cap = seq_cap;
  a.ring_off = 0;
  a.nslots = 0;
  a.qscale = scale * 1.4426950408889634f;
  a.group_starts = a.prefix_lens = nullptr;
  a.pre_o = a.pre_ml = nullptr;
  a.num_groups = a.pre_chunks = 0;
  a.qsl = qsl;
  a.num_q_rows = qsl ? num_q_rows : num_seqs;
  a.chunk_ids = chunk_ids;
  a.chunk_cap = chunk_cap;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (sp) {
    // pass 1: every group's prefix, once for all its members (tensor cores); pass 2 (the
    // decode kernel below) reads each sequence's own keys; the merge combines them
    float* pre_o = reinterpret_cast<float*>(ws + pre_off);
    float* pre_ml = pre_o + (size_t)plan.slots * num_seqs * num_q_heads * head_dim;
    const pa_status ps = pa::shared_prefix_pass(
        q, k_cache, v_cache, block_tables, max_blocks_per_seq, sp->group_starts,
        sp->prefix_lens, sp->num_groups, sp->max_group_size, sp->max_prefix_len, num_seqs,
        num_q_heads, num_kv_heads, scale, block_size, num_blocks, plan, pre_o, pre_ml, dtype,
        err, st);
    if (ps != PA_OK) return ps;
    a.group_starts = sp->group_starts;
    a.prefix_lens = sp->prefix_lens;
    a.num_groups = sp->num_groups;
    a.pre_o = pre_o;
    a.pre_ml = pre_ml;
    a.pre_chunks = plan.slots;
    const pa_status ds =
        dtype == PA_F16
            ? pa::dispatch_group<__half, false>(G, HB, tmK, tmV, tmQ, a, (int)grid, st)
            : pa::dispatch_group<__nv_bfloat16, false>(G, HB, tmK, tmV, tmQ, a, (int)grid, st);
    if (ds == PA_OK) pa::set_launch_count(pa::launch_count() + 1);
    return ds;
  }
  if (f8)
    return dtype == PA_F16
               ? pa::dispatch_group<__half, true>(G, HB, tmK, tmV, tmQ, a, (int)grid, st)
               : pa::dispatch_group<__nv_bfloat16, true>(G, HB, tmK, tmV, tmQ, a, (int)grid, st);
  return dtype == PA_F16
             ? pa::dispatch_group<__half, false>(G, HB, tmK, tmV, tmQ, a, (int)grid, st)
             : pa::dispatch_group<__nv_bfloat16, false>(G, HB, tmK, tmV, tmQ, a, (int)grid, st);
}
}  // namespace

extern "C" pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* seq_lens, int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, float scale, int block_size,
                               int num_blocks, int max_seq_len, int partition_size,
                               void* workspace, size_t workspace_bytes, pa_dtype dtype,
                               void* stream) {
  return decode_impl(out, q, nullptr, nullptr, k_cache, v_cache, nullptr, nullptr, block_tables,
                     max_blocks_per_seq, seq_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, scale, block_size,
                     num_blocks, max_seq_len, partition_size, workspace, workspace_bytes, dtype,
                     stream);
}

extern "C" pa_status pa_decode_append(void* out, const void* q, const void* k_new,
                                      const void* v_new, void* k_cache, void* v_cache,
                                      const int32_t* block_tables, int max_blocks_per_seq,
                                      const int32_t* seq_lens, int num_seqs, int num_q_heads,
                                      int num_kv_heads, int head_dim, float scale, int block_size,
                                      int num_blocks, int max_seq_len, int partition_size,
                                      void* workspace, size_t workspace_bytes, pa_dtype dtype,
                                      void* stream) {
  if (num_seqs > 0 && (!k_new || !v_new)) return PA_ERR_INVALID_ARG;
  return decode_impl(out, q, k_new, v_new, k_cache, v_cache, nullptr, nullptr, block_tables,
                     max_blocks_per_seq, seq_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, scale, block_size,
                     num_blocks, max_seq_len, partition_size, workspace, workspace_bytes, dtype,
                     stream);
}

extern "C" pa_status pa_decode_fp8(void* out, const void* q, const void* k_cache,
                                   const void* v_cache, const float* k_scale,
                                   const float* v_scale, const int32_t* block_tables,
                                   int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
                                   int num_q_heads, int num_kv_heads, int head_dim, float scale,
                                   int block_size, int num_blocks, int max_seq_len,
                                   int partition_size, void* workspace, size_t workspace_bytes,
                                   pa_dtype dtype, void* stream) {
  if (num_seqs > 0 && (!k_scale || !v_scale)) return PA_ERR_INVALID_ARG;
  return decode_impl(out, q, nullptr, nullptr, k_cache, v_cache, k_scale, v_scale, block_tables,
                     max_blocks_per_seq, seq_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                     scale, block_size, num_blocks, max_seq_len, partition_size, workspace,
                     workspace_bytes, dtype, stream);
}

// Decode without any caller-provided scratch.
//
// Some callers cannot allocate device memory on their own: code that runs inside a
// serving loop whose memory is entirely owned by an engine's pre-allocated pool (the
// pool hands out KV blocks, not scratch buffers), plugins whose host framework forbids
// raw cudaMalloc, and latency-critical paths where an allocation could synchronise the
// device.  For them this entry point keeps its workspace (the merge records and the
// split-K partials) in a fixed array that
// lives in this file (kNoAllocScratchBytes on every GPU that loads the library, held
// until the process exits) and otherwise runs exactly pa_decode.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_decode_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[64] = {};

// Device address of this device's scratch array (looked up once per device, with that
// device current).  nullptr if the lookup failed.
void* scratch_for_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_ptr[dev] = p;
  }
  return g_scratch_ptr[dev];
}
}  // namespace

extern "C" pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache,
                                       const void* v_cache, const int32_t* block_tables,
                                       int max_blocks_per_seq, const int32_t* seq_lens,
                                       int num_seqs, int num_q_heads, int num_kv_heads,
                                       int head_dim, float scale, int block_size, int num_blocks,
                                       int max_seq_len, int partition_size, pa_dtype dtype,
                                       void* stream) {
  pa::set_launch_count(0);
  const size_t need =
      pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_seq_len, partition_size);
  if (need > kNoAllocScratchBytes) return PA_ERR_WORKSPACE_TOO_SMALL;
  void* scratch = scratch_for_current_device();
  if (!scratch) return PA_ERR_CUDA;
  return pa_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens,
                   num_seqs, num_q_heads, num_kv_heads, head_dim, scale, block_size, num_blocks,
                   max_seq_len, partition_size, scratch, kNoAllocScratchBytes, dtype,
                   stream);
}

extern "C" size_t pa_decode_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

extern "C" size_t pa_decode_shared_prefix_workspace_size(int num_seqs, int num_q_heads,
                                                         int head_dim, int max_seq_len) {
  const size_t base = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_seq_len, 0);
  if (base == 0) return 0;
  return pa::align256(base) + (size_t)pa::kMaxPrefixChunks * num_seqs * num_q_heads *
                                  (head_dim + 2) * sizeof(float);
}

extern "C" pa_status pa_decode_shared_prefix(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens, int num_seqs,
    const int32_t* group_starts, const int32_t* prefix_lens, int num_groups, int max_group_size,
    int max_prefix_len, int num_q_heads, int num_kv_heads, int head_dim, float scale,
    int block_size, int num_blocks, int max_seq_len, void* workspace, size_t workspace_bytes,
    pa_dtype dtype, void* stream) {
  pa::set_launch_count(0);
  if (num_groups < 0 || max_group_size < 0 || max_prefix_len < 0 || num_seqs < 0 ||
      num_groups > num_seqs || max_group_size > num_seqs)
    return PA_ERR_INVALID_ARG;
  if (num_groups == 0 || max_group_size == 0 || max_prefix_len == 0)  // nothing shared
    return decode_impl(out, q, nullptr, nullptr, k_cache, v_cache, nullptr, nullptr,
                       block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_q_heads,
                       num_kv_heads, head_dim, scale, block_size, num_blocks, max_seq_len, 0,
                       workspace, workspace_bytes, dtype, stream);
  if (!group_starts || !prefix_lens) return PA_ERR_INVALID_ARG;
  const SharedPrefixArgs sp = {group_starts, prefix_lens, num_groups, max_group_size,
                               max_prefix_len};
  return decode_impl(out, q, nullptr, nullptr, k_cache, v_cache, nullptr, nullptr, block_tables,
                     max_blocks_per_seq, seq_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                     scale, block_size, num_blocks, max_seq_len, 0, workspace, workspace_bytes,
                     dtype, stream, &sp);
}

// Mixed varlen batch: decode rows on the decode kernel, prefill chunks on the tcgen05
// prefill kernel, in one call.
extern "C" size_t pa_attention_varlen_workspace_size(int num_seqs, int max_query_len,
                                                     int num_q_heads, int head_dim,
                                                     int max_seq_len) {
  const size_t d = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_seq_len, 0);
  if (d == 0) return 0;
  return pa::align256(d) + pa::align256((size_t)(num_seqs + 1) * sizeof(int32_t)) +
         pa_chunked_prefill_workspace_size(num_seqs, max_query_len, num_q_heads, head_dim,
                                           max_seq_len);
}

extern "C" pa_status pa_attention_varlen(
    void* out, const void* q, const void* k_cache, const void* v_cache,
    const int32_t* block_tables, int max_blocks_per_seq, const int32_t* seq_lens,
    const int32_t* query_start_loc, int num_seqs, int num_q_rows, int max_query_len,
    int max_chunk_seqs, int num_q_heads, int num_kv_heads, int head_dim, float scale,
    int block_size, int num_blocks, int max_seq_len, void* workspace, size_t workspace_bytes,
    pa_dtype dtype, void* stream) {
  pa::set_launch_count(0);
  if (num_seqs < 0 || num_q_rows < 0 || max_query_len < 0) return PA_ERR_INVALID_ARG;
  if (num_seqs == 0 || num_q_rows == 0 || max_query_len == 0) return PA_OK;
  if (!query_start_loc) return PA_ERR_INVALID_ARG;
  if (num_q_heads <= 0 || head_dim <= 0) return PA_ERR_INVALID_ARG;
  // a bound on the sequences with more than one query row (negative: num_seqs)
  const int cap = max_query_len > 1 ? (max_chunk_seqs < 0 ? num_seqs
                                                          : std::min(max_chunk_seqs, num_seqs))
                                    : 0;
  const size_t dws = pa::align256(
      pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_seq_len, 0));
  const size_t lws = pa::align256((size_t)(num_seqs + 1) * sizeof(int32_t));
  if (!workspace || workspace_bytes < dws + lws) return PA_ERR_WORKSPACE_TOO_SMALL;
  // listed whenever chunks may exist, so that more of them than the bound is flagged
  int32_t* chunk_ids = max_query_len > 1
                           ? reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + dws)
                           : nullptr;
  // the rows of one query: the decode kernel (it skips the others, and lists the chunks)
  pa_status st = decode_impl(out, q, nullptr, nullptr, k_cache, v_cache, nullptr, nullptr,
                             block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_q_heads,
                             num_kv_heads, head_dim, scale, block_size, num_blocks, max_seq_len,
                             0, workspace, dws, dtype, stream, nullptr, query_start_loc,
                             num_q_rows, chunk_ids, cap);
  if (st != PA_OK) return st;
  int launches = pa::launch_count();
  if (cap > 0) {
    // the chunks: the prefill kernel over the listed sequences
    const size_t rest = workspace_bytes - dws - lws;
    st = pa::chunked_prefill_impl(
        out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, query_start_loc,
        num_seqs, max_query_len, num_q_heads, num_kv_heads, head_dim, scale, block_size,
        num_blocks, max_seq_len, rest ? static_cast<uint8_t*>(workspace) + dws + lws : nullptr,
        rest, dtype, stream, true, chunk_ids, cap);
    if (st != PA_OK) return st;
    launches += pa::launch_count();
  }
  pa::set_launch_count(launches);
  return PA_OK;
}
