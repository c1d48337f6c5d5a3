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
//    workspace at slot c + group, merged by a log-sum-exp pass (merge_kernel, a
//    programmatic dependent of this launch).
//    An explicit partition size caps the share, so no segment is longer.
//  * One consumer warp per kv-head of the group handles all G q-heads of that kv-head,
//    so no two warps share an output.  q.k and p.V of a tile run as mma.sync m16n8k16
//    tensor-core fragments (fp32 accumulate; q-heads past G are zero columns): S^T = K Q^T
//    (M = 16 tokens, N = 8 heads), online softmax (running max m, sum l) in the log2
//    domain on the accumulator fragment (q pre-scaled by scale*log2 e: one ex2 per logit),
//    O^T += V^T P^T.  At G = 8 the two contractions cost 4 FMAs per byte of KV, more than
//    the FP32 pipe sustains at HBM rate; warp-shuffle dot products on CUDA cores, kept for
//    G <= 4 at first, were also measured slower there (mixed batch 88.1 -> 84.0 us).
//  * A staging warp cuts the CTA's share into units of at most 128 tiles and, up to two
//    units ahead, copies their block-table entries into shared memory (one coalesced
//    read per 32 entries) and starts the TMA copy of their q rows.  A producer thread
//    walks the tiles in order and issues the two boxes of each as soon as a slot of the
//    shared ring frees (blocking waits take no issue slots from the consumers).
// Two more modes share the kernel:
//  * shared prefixes (pa_decode_shared_prefix; page "KV Cache管理优化：大模型推理显存瓶颈
//    突破" 4.1, blocks shared by reference): a sequence whose first tokens are shared with
//    its group reads only its tiles after the prefix; the group's members are cut into
//    chunks of 16 q-rows per kv-head (16/G members), and each chunk is one more sequence of
//    the schedule over the prefix, whose consumer warps run its rows as two tensor-core n8
//    tiles; the merge pass folds each member's own pieces with its chunk's;
//  * varlen rows (pa_attention_varlen): only sequences with one query row are served,
//    q and out rows come from query_start_loc, and CTA 0 lists the other sequences for
//    the prefill kernel that follows.
// Every wait is bounded; bad table entries or lengths never fault (skipped, flagged).

#include <algorithm>
#include <climits>
#include <mutex>
#include <type_traits>

#include "pa_device.cuh"
#include "pa_host.h"
#include "prefill_body.cuh"

namespace pa {

struct DecodeArgs {
  void* out;
  const void* q;   // [rows, Hq, 128] (read directly only by the shared-prefix chunk rows)
  const int32_t* block_tables;
  const int32_t* seq_lens;
  float* part_o;   // [slots, HB*G, 128]   normalised partial outputs
  float* part_ml;  // [slots, HB*G, 2]     (max in log2 units, sum)
  // merge records for the log-sum-exp pass, per (sequence, head group) [B * NHP]: its own
  // segments (first slot, segment count; count 0 when nothing is left to merge: written
  // directly, or no keys), and with shared prefixes its chunk's segments (first chunk slot,
  // count, the member's first row in the chunk's rows of a kv-head, 0)
  int2* meta;
  int4* cmeta;
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
  // share their first prefix_lens[g] tokens (whole blocks).  A sequence reads only its keys
  // after the prefix.  The members of a group with a prefix are cut into chunks of `mc`
  // members (16 rows per kv-head: mc * G); each chunk is a virtual sequence appended to the
  // batch (indices num_seqs ..): prefix_lens[g] tokens read through the table row of the
  // group's first member, its queries the chunk's members' q-heads, its normalised
  // partial rows in vpart_o / vpart_ml ([slots, HB*16, 128] / [slots, HB*16, 2]).
  const int32_t* group_starts;
  const int32_t* prefix_lens;
  float* vpart_o;
  float* vpart_ml;
  int num_groups, mc, vcap;  // groups, members per chunk, bound on the chunks
  int max_prefix;            // host bound on prefix_lens (a longer prefix is flagged)
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
  long long wait_limit;  // SM cycles any pipeline wait may take before the CTA gives up
  int test_withhold;     // testing hook: CTA 0's producer withholds its first tile
  int wait_prior;        // launched as a programmatic dependent: wait before reading inputs
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
constexpr int kVirtual = 8;  // a chunk of a group's members over their shared prefix
// a staged unit: [0] sequence (-1: no more work; >= num_seqs: a chunk), [1] head group,
// [2..3] tiles [t0, t1), [4] flags, [5] partial slot of this segment, [6] append, [7] q /
// out row (a chunk: its first member), [10] members of a chunk
constexpr int kUnitInts = 16;
constexpr int kChunkRows = 16;           // q rows of a chunk per kv-head (members x G)

template <int G_, int HB_, bool F8_, bool SP_ = false>
struct DecodeCfg {
  static constexpr int G = G_;
  static constexpr int HB = HB_;                  // kv-heads per group = consumer warps
  static constexpr bool F8 = F8_;                 // e4m3 cache (else fp16/bf16)
  static constexpr int KROW = kD * (F8 ? 1 : 2);  // one token of one kv-head in the cache
  static constexpr int WARP_PROD = 0;
  static constexpr int WARP_STAGE = 1;
  static constexpr int WARP_FILL = 2;             // zero-fills empty sequences
  static constexpr int WARP_C0 = 4;               // first consumer warp
  static constexpr int THREADS = 128 + HB * 32;
  static constexpr int TILE_BYTES = kTileTok * HB * KROW;       // K (or V) of a tile
  static constexpr int SLOT_BYTES = 2 * TILE_BYTES;
  // A K (V) tile is copied as 128-byte-wide column slabs of its rows (two slabs of 64 dims
  // for 16-bit elements, one of 128 e4m3 codes), each laid out [kv-head][token][128 B] with
  // the 128-byte swizzle: see swz().
  static constexpr int SLABS = KROW / 128;
  static constexpr int SLAB_BYTES = TILE_BYTES / SLABS;
  static constexpr int QBYTES = HB * G * kRowBytes;             // q rows of a group
  // shared-memory carve-up (bytes); the sequence arrays and then the ring follow
  static constexpr int OFF_FULL = 0;
  static constexpr int OFF_EMPTY = OFF_FULL + kMaxSlots * 8;
  static constexpr int OFF_QFULL = OFF_EMPTY + kMaxSlots * 8;
  static constexpr int OFF_QEMPTY = OFF_QFULL + kQSlots * 8;
  static constexpr int OFF_TFULL = OFF_QEMPTY + kQSlots * 8;
  static constexpr int OFF_TEMPTY = OFF_TFULL + kQSlots * 8;
  static constexpr int OFF_ADONE = OFF_TEMPTY + kQSlots * 8;    // append of a unit written
  static constexpr int OFF_UNIT = OFF_ADONE + kQSlots * 8;      // 16 ints per staged unit
  static constexpr int OFF_ABORT = OFF_UNIT + kQSlots * 64;
  static constexpr int OFF_TBL = ((OFF_ABORT + 16 + 127) / 128) * 128;
  static constexpr int OFF_Q = OFF_TBL + kQSlots * kMaxTilesPerUnit * 4;
  static constexpr int OFF_SEQ = OFF_Q + kQSlots * QBYTES;  // the schedule arrays
  static_assert(OFF_Q % 128 == 0 && OFF_SEQ % 16 == 0, "alignment");
};

__device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }
__device__ __forceinline__ int clamp_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }

// Byte offset, inside one column slab of a ring tile, of 16-byte chunk c (0..7) of token t of
// kv-head w.  The slab holds 128-byte rows ordered [kv-head][token]; the copy's 128-byte
// swizzle stores chunk c of row r at chunk position c ^ (r & 7) (the slab starts on a
// 1024-byte boundary, so r & 7 = t & 7).  Rows of consecutive tokens then start in different
// banks, which the consumers' fragment reads rely on to be free of bank conflicts.
__device__ __forceinline__ int swz(int w, int t, int c) {
  return ((w * kTileTok + t) << 7) | ((c ^ (t & 7)) << 4);
}


// Group holding sequence s: the last g with group_starts[g] <= s, if s < group_starts[g+1];
// else -1.
__device__ __forceinline__ int group_of(const DecodeArgs& a, int s) {
  if (a.num_groups <= 0 || s < __ldg(a.group_starts)) return -1;
  int lo = 0, hi = a.num_groups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(a.group_starts + mid) <= s) lo = mid; else hi = mid - 1;
  }
  return s < __ldg(a.group_starts + lo + 1) ? lo : -1;
}

// Bounded wait that turns into a no-op once any warp of the CTA gave up (and stops
// waiting as soon as one does).  After a wait that may have been skipped, a warp makes no
// further arrival on a barrier that counts transaction bytes: its previous phase may still
// be pending.
__device__ __forceinline__ void wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag, int* err,
                                              long long limit) {
  if (*abort_flag || mbar_try_wait(bar, parity)) return;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return;
    if (clock64() - t0 > limit) {
      flag_error(err, PA_DEVERR_TIMEOUT);
      *abort_flag = 1;
      return;
    }
  }
}

// After an abort: wait (bounded, ignoring the abort flag) for the phase of `bar` that the
// calling thread's last copy into a buffer completes, so that no bulk copy is still
// writing the CTA's shared memory when it exits.
__device__ __forceinline__ void drain_copy(uint64_t* bar, uint32_t parity, int* err,
                                           long long limit) {
  (void)mbar_wait(bar, parity, err, limit);
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

// Four e4m3 codes (byte 0 of x first) -> their f16 values as two f16x2 registers: lo holds
// codes 0 and 1, hi codes 2 and 3, each with the lower byte's value in its low half.  One
// conversion per pair, with the 16-bit halves of x as its operands (no shifts or masks).
// Exact: every e4m3 value is an f16 value.
__device__ __forceinline__ void e4m3x4_to_f16x2x2(uint32_t x, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(x));
}

// Transpose of an 8x8 matrix of 16-bit elements held as one fragment register per lane
// (lane l: row l/4, columns 2(l%4), 2(l%4)+1).
__device__ __forceinline__ uint32_t transpose8x8(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(d) : "r"(a));
  return d;
}

// Tensor-core consumers, S^T = K Q^T over a 16-bit tile: k-steps 2j and 2j+1 of lane quad tq
// take the eight dims of 16-byte chunk kchunk(tq, j) (of 16; chunks 0..7 in slab 0).  The
// contraction may visit dims in any order as long as K and Q agree; this one puts the lanes
// of tokens g and g^1 (one shared-memory phase) on chunks of opposite parity, so that under
// the slab swizzle the eight 16-byte reads of a phase hit eight different bank groups.
__device__ __forceinline__ int kchunk(int tq, int j) { return 8 * (j >> 1) + 2 * tq + (j & 1); }

// O^T += V^T P^T for one 16-token tile of kv-head w (tensor-core consumers, 16-bit cache).
// Lane (g, tq) reads one 16-byte chunk per token for tokens 2tq, 2tq+1, 2tq+8, 2tq+9 (zero
// past nvalid): chunk g of each slab, dims [8g, 8g+8) and [64+8g, 64+8g+8).  Word r of a
// lane's chunk h makes m-tile 4h+r, its row g the chunk's dim 2r and its row g+8 dim 2r+1,
// with tokens paired along k as the P^T fragments pb0 (tokens 2tq, 2tq+1) and pb1 (2tq+8,
// 2tq+9) expect.  Under the swizzle the reads of a phase (tokens 2tq+b of chunks g, g^1) fall
// in eight different bank groups.  NT column tiles of 8 share every V fragment; SLAB is the
// tile's slab size in bytes.
template <typename MT, int NT, int SLAB>
__device__ __forceinline__ void pv_tile(float (&oacc)[NT][8][4], const uint8_t* Vs, int w, int g,
                                        int tq, int nvalid, const uint32_t (&pb)[NT][2]) {
  // token 2tq+b+8c sits 8 rows (1 KB) after token 2tq+b, with the same swizzle
  const int vofs0 = swz(w, 2 * tq, g), vofs1 = swz(w, 2 * tq + 1, g);
  auto vofs = [&](int i) { return ((i & 1) ? vofs1 : vofs0) + (i >> 1) * 1024; };
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t vw[4][4];  // [token i][word r]
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int tk = 2 * tq + (i & 1) + (i >> 1) * 8;
      const uint4 c = tk < nvalid ? *reinterpret_cast<const uint4*>(Vs + h * SLAB + vofs(i))
                                  : make_uint4(0u, 0u, 0u, 0u);
      vw[i][0] = c.x;
      vw[i][1] = c.y;
      vw[i][2] = c.z;
      vw[i][3] = c.w;
    }
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const uint32_t a0 = __byte_perm(vw[0][r], vw[1][r], 0x5410);
      const uint32_t a1 = __byte_perm(vw[0][r], vw[1][r], 0x7632);
      const uint32_t a2 = __byte_perm(vw[2][r], vw[3][r], 0x5410);
      const uint32_t a3 = __byte_perm(vw[2][r], vw[3][r], 0x7632);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        Mma<MT>::run(oacc[nt][4 * h + r], a0, a1, a2, a3, pb[nt][0], pb[nt][1]);
    }
  }
}

// The same product over an e4m3 tile, as two steps, so that a consumer can issue a tile's V
// reads and conversions before the tile's softmax.  Lane (g, tq) reads the 16 codes
// [16g, 16g+16) of tokens 2tq, 2tq+1, 2tq+8, 2tq+9 (one 16-byte chunk each, zero past
// nvalid).  Fragment [h][r][0..3]
// is the A operand of m-tile 4h+r: the codes of tokens 2p and 2p+1 paired byte by byte
// before the conversion, so that each converted f16x2 is already a fragment register
// (token 2p in its low half).
__device__ __forceinline__ void pv_frags_f8(const uint8_t* Vs, int w, int g, int tq, int nvalid,
                                            uint32_t (&fr)[2][4][4]) {
  // token 2tq+b+8c sits 8 rows (1 KB) after token 2tq+b, with the same swizzle
  const int vofs0 = swz(w, 2 * tq, g), vofs1 = swz(w, 2 * tq + 1, g);
  uint4 v8[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int tk = 2 * tq + (i & 1) + (i >> 1) * 8;
    v8[i] = tk < nvalid ? *reinterpret_cast<const uint4*>(Vs + ((i & 1) ? vofs1 : vofs0) +
                                                          (i >> 1) * 1024)
                        : make_uint4(0u, 0u, 0u, 0u);
  }
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int p = 0; p < 2; ++p) {
      const uint4& t0 = v8[2 * p];
      const uint4& t1 = v8[2 * p + 1];
      const uint32_t x0 = h ? t0.z : t0.x, y0 = h ? t1.z : t1.x;  // codes 0-3 of the chunk half
      const uint32_t x1 = h ? t0.w : t0.y, y1 = h ? t1.w : t1.y;  // codes 4-7
      e4m3x4_to_f16x2x2(__byte_perm(x0, y0, 0x5140), fr[h][0][2 * p], fr[h][0][2 * p + 1]);
      e4m3x4_to_f16x2x2(__byte_perm(x0, y0, 0x7362), fr[h][1][2 * p], fr[h][1][2 * p + 1]);
      e4m3x4_to_f16x2x2(__byte_perm(x1, y1, 0x5140), fr[h][2][2 * p], fr[h][2][2 * p + 1]);
      e4m3x4_to_f16x2x2(__byte_perm(x1, y1, 0x7362), fr[h][3][2 * p], fr[h][3][2 * p + 1]);
    }
}
template <int NT>
__device__ __forceinline__ void pv_mma_f8(float (&oacc)[NT][8][4], const uint32_t (&fr)[2][4][4],
                                          const uint32_t (&pb)[NT][2]) {
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
        Mma<__half>::run(oacc[nt][4 * h + r], fr[h][r][0], fr[h][r][1], fr[h][r][2], fr[h][r][3],
                         pb[nt][0], pb[nt][1]);
}

// The output dims pv_tile leaves in a lane (g, tq): for column e of its tiles, dims d0 + 2i
// and d0 + 2i + 1 in acc[i][e] and acc[i][2+e] (i < 4) and dims d1 + 2i, +1 in acc[4+i][..],
// with (d0, d1) = (8g, 64+8g) for 16-bit tiles and (16g, 16g+8) for e4m3 ones.  These write
// them, times inv, as two runs of 8: to a 16-bit row, or to an fp32 row.
template <bool F8>
__device__ __forceinline__ int pv_dim(int g, int h) {
  return F8 ? 16 * g + 8 * h : 8 * g + 64 * h;
}
template <typename T, bool F8>
__device__ __forceinline__ void store_pv_row(T* row, const float (&acc)[8][4], int e, float inv,
                                             int g) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float(*c)[4] = acc + 4 * h;
    *reinterpret_cast<uint4*>(row + pv_dim<F8>(g, h)) =
        make_uint4(Elem<T>::pack2(c[0][e] * inv, c[0][2 + e] * inv),
                   Elem<T>::pack2(c[1][e] * inv, c[1][2 + e] * inv),
                   Elem<T>::pack2(c[2][e] * inv, c[2][2 + e] * inv),
                   Elem<T>::pack2(c[3][e] * inv, c[3][2 + e] * inv));
  }
}
template <bool F8>
__device__ __forceinline__ void store_pv_row_f32(float* row, const float (&acc)[8][4], int e,
                                                 float inv, int g) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float(*c)[4] = acc + 4 * h;
    float4* d = reinterpret_cast<float4*>(row + pv_dim<F8>(g, h));
    d[0] = make_float4(c[0][e] * inv, c[0][2 + e] * inv, c[1][e] * inv, c[1][2 + e] * inv);
    d[1] = make_float4(c[2][e] * inv, c[2][2 + e] * inv, c[3][e] * inv, c[3][2 + e] * inv);
  }
}

// CTA holding global tile `pos` when T tiles are shared out over `grid` CTAs
// (CTA c holds [c*T/grid, (c+1)*T/grid)).
__device__ __forceinline__ int cta_of(int pos, int T, int grid) {
  return (int)((((long long)pos + 1) * grid - 1) / T);
}

// Log-sum-exp merge of the split-K partials: one warp per (sequence, q-head), lanes over
// head_dim.  o = sum_i w_i o_i / sum_i w_i with w_i = l_i * 2^(m_i - M), M the largest m_i,
// over the sequence's own segments (consecutive slots of its head group's record) and, with
// a shared prefix, the segments of the chunk that holds it (rows of its chunk slots).  One
// pass with a running maximum, in rounds of 4, 8 or 16 rows by the piece count, all their
// loads in flight.  Launched as a programmatic dependent of the decode kernel.
template <typename T, int G, bool SP>
__global__ void __launch_bounds__(256) merge_kernel(const DecodeArgs a, int HB) {
  griddep_wait();  // the decode grid has finished and its writes are visible
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= a.num_seqs * a.num_q_heads) return;
  const int s = gw / a.num_q_heads;
  const int qh = gw - s * a.num_q_heads;
  const int hbg = HB * G, NHP = a.num_kv_heads / HB;
  const int hp = qh / hbg, j = qh - hp * hbg;
  const int2 mo = a.meta[s * NHP + hp];
  const int so0 = mo.x, no = mo.y;
  int sv0 = 0, nv = 0, vrow = 0;
  if constexpr (SP) {  // loaded beside the own record: one round trip for both
    const int4 cm = a.cmeta[s * NHP + hp];
    sv0 = cm.x;
    nv = cm.y;
    vrow = (j / G) * kChunkRows + cm.z + (qh % G);
  }
  const int total = no + nv;
  if (total == 0) return;  // written by the decode kernel (or nothing to write)
  float M = -INFINITY, den = 0.f;
  float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
  // Rounds of R pieces, R = 4, 8 or 16 by the piece count (uniform over the warp).  A
  // round's loads are unconditional (past the last piece: its row again, ignored after) so
  // that they are all in flight before the first is used; loads behind a branch each
  // waited for the previous piece's use (measured: LLaMA-70B 57.1 -> 55.1 us per call).
  auto rounds = [&](auto rc) {
    constexpr int R = decltype(rc)::value;
    for (int i0 = 0; i0 < total; i0 += R) {
      float2 mlv[R];
      float4 ov[R];
#pragma unroll
      for (int u = 0; u < R; ++u) {
        const int i = min(i0 + u, total - 1);
        const bool own = i < no;
        const long long row = own ? (long long)(so0 + i) * hbg + j
                                  : (long long)(sv0 + i - no) * (HB * kChunkRows) + vrow;
        mlv[u] = __ldg(reinterpret_cast<const float2*>((own ? a.part_ml : a.vpart_ml) + row * 2));
        ov[u] = __ldg(reinterpret_cast<const float4*>((own ? a.part_o : a.vpart_o) + row * kD) +
                      lane);
      }
      float Mr = -INFINITY;
#pragma unroll
      for (int u = 0; u < R; ++u)
        if (i0 + u < total) Mr = fmaxf(Mr, mlv[u].x);
      const float Mn = fmaxf(M, Mr);
      if (Mn == -INFINITY) continue;  // only empty segments so far
      const float sc = fast_exp2(M - Mn);  // M = -inf -> 0
      den *= sc;
      num.x *= sc; num.y *= sc; num.z *= sc; num.w *= sc;
#pragma unroll
      for (int u = 0; u < R; ++u) {
        if (i0 + u < total) {
          const float f = mlv[u].x == -INFINITY ? 0.f : fast_exp2(mlv[u].x - Mn) * mlv[u].y;
          den += f;
          num.x += f * ov[u].x; num.y += f * ov[u].y; num.z += f * ov[u].z; num.w += f * ov[u].w;
        }
      }
      M = Mn;
    }
  };
  if (total <= 4) rounds(std::integral_constant<int, 4>{});
  else if (total <= 8) rounds(std::integral_constant<int, 8>{});
  else rounds(std::integral_constant<int, 16>{});
  const float inv = den > 0.f ? 1.f / den : 0.f;
  const long long orow = a.qsl ? __ldg(a.qsl + s) : s;
  T* ob = static_cast<T*>(a.out) + (orow * a.num_q_heads + qh) * kD + lane * 4;
  *reinterpret_cast<uint2*>(ob) =
      make_uint2(Elem<T>::pack2(num.x * inv, num.y * inv), Elem<T>::pack2(num.z * inv, num.w * inv));
}

// The decode CTA `cta` of `ncta` (the persistent grid's share of the tiles), with its
// dynamic shared memory at `smem` (1024-byte aligned).  The CTA may hold more threads than
// the configuration's; the extra warps leave after the prologue.
template <typename T, int G, int HB, bool F8, bool SP>
__device__ __forceinline__ void decode_body(const CUtensorMap& tmK, const CUtensorMap& tmV,
                                            const CUtensorMap& tmQ, const DecodeArgs& a,
                                            uint8_t* smem, const int cta, const int ncta) {
  using C = DecodeCfg<G, HB, F8, SP>;
  constexpr int HBG = HB * G;
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
  const int B = a.num_seqs;
  const int VC = SP ? a.vcap : 0;  // room for chunk sequences after the batch
  int* sstart = reinterpret_cast<int*>(smem + C::OFF_SEQ);  // [B+VC+1] first tile of each sequence
  int* slen = sstart + B + VC + 1;                           // [B+VC] clamped lengths
  int* sfirst = slen + B + VC;  // [B+VC] first tile after a shared prefix (0 without; -1 not served)
  int* cstart = sfirst + B + VC;  // [groups+1] first chunk of each group
  volatile int* nchunks = abort_flag + 1;  // chunks in the schedule (<= VC)
  uint8_t* ring = smem + a.ring_off;
  const int nslots = a.nslots;
  const int NHP = a.num_kv_heads / HB;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // the merge pass may be scheduled now; it waits for this grid's results itself
  griddep_launch_dependents();
  // This CTA's slice of the block tables into L2 (a hint: the lines are read later, after
  // the lengths, by the staging warp), then, when this grid was launched as a dependent of
  // the previous kernel of the stream, wait for it before any input is read.
  if (threadIdx.x == 0 && ((uintptr_t)a.block_tables & 15) == 0) {
    const long long tb = ((long long)B * a.max_blocks * 4) & ~15LL;
    const long long per = (((tb + ncta - 1) / ncta) + 15) & ~15LL;
    const long long off = per * cta;
    if (off < tb)
      prefetch_l2_bulk(reinterpret_cast<const uint8_t*>(a.block_tables) + off,
                       (uint32_t)min(per, tb - off));
  }
  if (a.wait_prior) griddep_wait();

  // ---- clamped lengths and the prefix of tiles over (sequence, head group)
  if (warp == 0) {
    int V = 0;
    if constexpr (SP) {
      // the members of a group with a shared prefix, cut into chunks of a.mc: the chunk
      // count of each group and their exclusive prefix sum
      const int ng = a.num_groups;
      const int gper = (ng + 31) / 32;
      const int glo = min(ng, lane * gper), ghi = min(ng, glo + gper);
      auto chunks_of = [&](int g) {
        const int n = __ldg(a.group_starts + g + 1) - __ldg(a.group_starts + g);
        return (n > 0 && __ldg(a.prefix_lens + g) > 0) ? cdiv(n, a.mc) : 0;
      };
      int csum = 0;
      for (int g = glo; g < ghi; ++g) csum += chunks_of(g);
      int cincl = csum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, cincl, o);
        if (lane >= o) cincl += t;
      }
      int crun = cincl - csum;
      for (int g = glo; g < ghi; ++g) {
        cstart[g] = crun;
        crun += chunks_of(g);
      }
      const int total = __shfl_sync(0xffffffffu, cincl, 31);
      if (lane == 0) {
        cstart[ng] = total;
        if (total > VC && cta == 0) flag_error(a.err, PA_DEVERR_PREFIX);
      }
      V = min(total, VC);
      __syncwarp();
    }
    const int NS = B + V;  // the batch, then the chunks
    const int per = (NS + 31) / 32;
    const int lo = min(NS, lane * per), hi = min(NS, lo + per);
    int sum = 0;
    for (int s = lo; s < hi; ++s) {
      int L, first = 0;
      if (SP && s >= B) {
        // chunk s-B: its group's prefix, read through the group's first member's table row
        const int vs = s - B;
        int glo2 = 0, ghi2 = a.num_groups - 1;  // the last g with cstart[g] <= vs
        while (glo2 < ghi2) {
          const int mid = (glo2 + ghi2 + 1) >> 1;
          if (cstart[mid] <= vs) glo2 = mid; else ghi2 = mid - 1;
        }
        L = clamp_len(__ldg(a.prefix_lens + glo2), min(a.seq_cap, a.max_prefix));
      } else {
        const int raw = a.seq_lens[s];
        L = clamp_len(raw, a.seq_cap);
        if (raw != L && cta == 0) flag_error(a.err, PA_DEVERR_SEQ_TOO_LONG);
        if (a.qsl != nullptr) {  // varlen: decode rows only; the others are prefill chunks
          const int q0 = __ldg(a.qsl + s), nq = __ldg(a.qsl + s + 1) - q0;
          if (nq != 1) first = -1;
          else if (q0 < 0 || q0 >= a.num_q_rows) {
            if (cta == 0) flag_error(a.err, PA_DEVERR_QUERY_LAYOUT);
            first = -1;
          }
        }
        if (SP && first == 0) {
          const int g = group_of(a, s);
          const int p = g < 0 ? 0 : __ldg(a.prefix_lens + g);
          if ((p < 0 || p > L || p > a.max_prefix || (p & ((1 << a.log2_bs) - 1))) &&
              cta == 0)
            flag_error(a.err, PA_DEVERR_PREFIX);
          first = clamp_len(p, L) / kTileTok;
        }
      }
      slen[s] = L;
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
    if (lane == 31) {
      sstart[NS] = incl;
      *nchunks = V;
    }
    if (a.chunk_ids != nullptr && cta == 0) {
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
  const int V = *nchunks;
  const int NS = B + V;
  const int Ttot = sstart[NS];
  // The launch sizes the grid for the longest possible batch; when the batch holds
  // fewer tiles than CTAs, only the first Ttot CTAs take a share, so every share is
  // non-empty and the segments of a group sit in consecutive CTAs (and slots).
  const int grid = min(ncta, max(Ttot, 1));
  // c*Ttot/grid in 32-bit arithmetic: c*(Ttot/grid) + c*(Ttot%grid)/grid, c*(Ttot%grid) < grid^2
  const int tq = Ttot / grid, tr = Ttot % grid;
  const int r0 = cta < grid ? cta * tq + (cta * tr) / grid : Ttot;
  const int r1 = cta < grid ? (cta + 1) * tq + ((cta + 1) * tr) / grid : Ttot;

  if (warp < C::WARP_C0) {
    if (warp == C::WARP_FILL) {
      // ===== sequences without keys of their own: no CTA's share visits them; their merge
      // records say "nothing to merge" and their outputs are zeros (all keys shared: the
      // merge pass takes its chunk's pieces alone) =====
      for (int s = cta; s < B; s += ncta) {
        if (sfirst[s] >= 0 && cdiv(slen[s], kTileTok) != sfirst[s]) continue;
        for (int h = lane; h < NHP; h += 32) a.meta[s * NHP + h] = make_int2(0, 0);
        if (sfirst[s] < 0) continue;  // not served by this kernel
        if constexpr (SP) {
          const int g = group_of(a, s);
          if (g >= 0 && __ldg(a.prefix_lens + g) > 0 &&
              cstart[g] + (s - __ldg(a.group_starts + g)) / a.mc < V)
            continue;
        }
        const int orow = a.qsl ? __ldg(a.qsl + s) : s;
        T* ob = static_cast<T*>(a.out) + (long long)orow * a.num_q_heads * kD;
        for (int i = lane; i < a.num_q_heads * kD / 8; i += 32)
          reinterpret_cast<uint4*>(ob)[i] = make_uint4(0u, 0u, 0u, 0u);
      }
      if constexpr (SP) {
        // each member's chunk record for the merge pass: the chunk's segments over its
        // prefix (as the staging warps cut them: first slot, count) and the member's rows
        for (int s = cta; s < B; s += ncta) {
          int vs = -1, voff = 0;
          const int g = group_of(a, s);
          if (g >= 0 && __ldg(a.prefix_lens + g) > 0) {
            const int off = s - __ldg(a.group_starts + g);
            const int v = cstart[g] + off / a.mc;
            if (v < V) {
              vs = v;
              voff = (off % a.mc) * G;
            }
          }
          const int cntv = vs >= 0 ? cdiv(slen[B + vs], kTileTok) : 0;
          for (int h = lane; h < NHP; h += 32) {
            int4 r = make_int4(0, 0, 0, 0);
            if (cntv > 0) {
              const int gs = sstart[B + vs] + h * cntv;
              const int c0 = cta_of(gs, Ttot, grid), c1 = cta_of(gs + cntv - 1, Ttot, grid);
              r = make_int4(c0 + vs * NHP + h, c1 - c0 + 1, voff, 0);
            }
            a.cmeta[s * NHP + h] = r;
          }
        }
      }
      return;
    }
    if (warp == C::WARP_STAGE) {
      // ===== staging warp: cuts the share into units; table entries + q, two units ahead =====
      if (lane == 0) prefetch_tmap(&tmQ);
      int pos = r0;
      int s = 0;
      if (pos < r1) {  // sequence holding pos: the last s with sstart[s] <= pos
        int lo = 0, hi = NS - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (sstart[mid] <= pos) lo = mid; else hi = mid - 1;
        }
        s = lo;
      }
      uint32_t q_issued = 0;  // bit i: unit k-1-i copied q rows (as the producer's mask)
      for (int k = 0;; ++k) {
        const int qs = k % kQSlots;
        const uint32_t par = ((k / kQSlots) & 1) ^ 1;
        if (k >= kQSlots) {  // the first units' slots were never used
          wait_or_abort(&qempty[qs], par, abort_flag, a.err, a.wait_limit);  // consumers read unit k-2's q
          wait_or_abort(&tempty[qs], par, abort_flag, a.err, a.wait_limit);  // its tiles were issued
        }
        volatile int* u = unit + qs * kUnitInts;
        // after an abort a wait may have been skipped: no more arrivals
        const bool stop = warp_flag(abort_flag);
        if (!stop && pos >= r1 && lane == 0) {  // tell the other warps there is no more work
          u[0] = -1;
          mbar_arrive_expect_tx(&qfull[qs], 0);
          mbar_arrive(&tfull[qs]);
        }
        if (stop || pos >= r1) {
          // no q copy may still be landing when the CTA exits (a no-op unless the consumers
          // abort): units k-1 and k-2 after an abort; only k-1 after the arrival above,
          // which completed the phase after unit k-2's in the same slot
          if (lane == 0)
            for (int i = 0; i < (stop ? kQSlots : 1) && i < k; ++i)
              if (q_issued & (1u << i)) {
                const int c = k - 1 - i;
                drain_copy(&qfull[c % kQSlots], (c / kQSlots) & 1, a.err, a.wait_limit);
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
        const int gs = sstart[s] + hp * cnt;  // the group's first and one-past-last tile
        const int ge = gs + cnt;
        // a chunk (s >= B): members m0 .. m0+nm-1 of group g over its prefix, read through
        // the table row of the group's first member; its slots are numbered apart
        const bool virt = SP && s >= B;
        int m0 = 0, nm = 0, trow_seq = s;
        if (virt) {
          const int vs = s - B;
          int glo = 0, ghi = a.num_groups - 1;  // the last g with cstart[g] <= vs
          while (glo < ghi) {
            const int mid = (glo + ghi + 1) >> 1;
            if (cstart[mid] <= vs) glo = mid; else ghi = mid - 1;
          }
          trow_seq = __ldg(a.group_starts + glo);
          m0 = trow_seq + (vs - cstart[glo]) * a.mc;
          nm = min(a.mc, __ldg(a.group_starts + glo + 1) - m0);
        }
        const int grp = (virt ? s - B : s) * NHP + hp;
        int flags = virt ? kVirtual : 0;
        if (t0 == ts || pos == r0) flags |= kFirst;
        if (t1 == nt || pos + (t1 - t0) == r1) flags |= kLast;
        if (gs >= r0 && ge <= r1 && ts == 0 && !virt) flags |= kDirect;
        const int32_t* trow = a.block_tables + (long long)trow_seq * a.max_blocks;
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
        if (a.k_new != nullptr && t1 == nt && !virt) {
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
          u[0] = s;
          u[1] = hp;
          u[2] = t0;
          u[3] = t1;
          u[4] = flags;
          u[5] = cta + grp;
          u[6] = append ? 1 : 0;
          u[7] = virt ? m0 : (a.qsl ? __ldg(a.qsl + s) : s);  // q / out row
          u[10] = nm;
          q_issued <<= 1;
          if ((flags & kFirst) && !virt) {  // a chunk's rows are read by its consumers
            mbar_arrive_expect_tx(&qfull[qs], C::QBYTES);
            tma_load_3d(qbuf + qs * C::QBYTES, &tmQ, 0, hp * HBG, u[7], &qfull[qs]);
            q_issued |= 1u;
          } else {
            mbar_arrive_expect_tx(&qfull[qs], 0);
          }
          mbar_arrive(&tfull[qs]);
          if (t0 == ts && !virt) {
            // the group's first unit, once published: its merge record (the group's segments
            // sit in CTAs c0..c1, their partials in slots c0+grp..c1+grp)
            const int c0 = cta_of(gs, Ttot, grid), c1 = cta_of(ge - 1, Ttot, grid);
            a.meta[grp] = make_int2(c0 + grp, (flags & kDirect) ? 0 : c1 - c0 + 1);
          }
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
        while (s + 1 < NS && sstart[s + 1] <= pos) ++s;
      }
      return;
    }

    if (warp == C::WARP_PROD) {
      // ===== producer: one thread walks every tile in order into the shared ring =====
      if (lane == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        const uint64_t pol_stream = l2_policy_evict_first(), pol_keep = l2_policy_evict_normal();
        const int bs_mask = (1 << a.log2_bs) - 1;
        // bit i: tile cnt-1-i was copied.  Each ring slot is reused only after its previous
        // copy was consumed, so only the last nslots tiles can still be landing.
        uint32_t issued = 0;
        int cnt = 0;
        for (int k = 0;; ++k) {
          const int qs = k % kQSlots;
          wait_or_abort(&tfull[qs], (k / kQSlots) & 1, abort_flag, a.err, a.wait_limit);
          const volatile int* u = unit + qs * kUnitInts;
          const int s = u[0];
          if (s < 0 || *abort_flag) break;  // (one thread: a plain read)
          const int hp = u[1], t0 = u[2], t1 = u[3], append = u[6];
          // a sequence's own keys are read once: evict them first from L2, so the stream
          // displaces itself rather than other lines; a shared prefix is read again by the
          // group's other chunks
          const uint64_t pol = (u[4] & kVirtual) ? pol_keep : pol_stream;
          for (int t = t0; t < t1; ++t, ++cnt) {
            const int slot = cnt % nslots;
            // the new token's row is in the last tile: its stores must have landed
            if (append && t == t1 - 1)
              wait_or_abort(&adone[qs], (k / kQSlots) & 1, abort_flag, a.err, a.wait_limit);
            wait_or_abort(&empty[slot], ((cnt / nslots) & 1) ^ 1, abort_flag, a.err, a.wait_limit);
            if (*abort_flag) break;  // a wait may have been skipped: no more arrivals
            issued <<= 1;
            if (a.test_withhold && cta == 0 && cnt == 0) continue;  // testing hook
            const int bid = tbl[qs * kMaxTilesPerUnit + (t - t0)];
            mbar_arrive_expect_tx(&full[slot], bid >= 0 ? C::SLOT_BYTES : 0);
            if (bid >= 0) {
              const int row = (t * kTileTok) & bs_mask;
              uint8_t* dst = ring + slot * C::SLOT_BYTES;
#pragma unroll
              for (int h = 0; h < C::SLABS; ++h) {  // map coordinates: dim, token, kv-head, block
                tma_load_4d_hint(dst + h * C::SLAB_BYTES, &tmK, h * 64, row, hp * HB, bid,
                                 &full[slot], pol);
                tma_load_4d_hint(dst + C::TILE_BYTES + h * C::SLAB_BYTES, &tmV, h * 64, row,
                                 hp * HB, bid, &full[slot], pol);
              }
              issued |= 1u;
            }
          }
          if (*abort_flag) break;
          mbar_arrive(&tempty[qs]);
        }
        // no copy may still be landing in the ring when the CTA exits (the consumers have
        // waited for all of them unless the CTA aborted)
        for (int i = 0; i < nslots && i < cnt; ++i)
          if (issued & (1u << i)) {
            const int c = cnt - 1 - i;
            drain_copy(&full[c % nslots], (c / nslots) & 1, a.err, a.wait_limit);
          }
      }
      return;
    }
    return;  // warp 3 idles
  }

  // ===================== consumer warps: warp w <-> kv-head hp*HB + w =====================
  const int w = warp - C::WARP_C0;
  if (w >= HB) return;  // a CTA shared with other work may hold more threads

  // A chunk segment (shared prefix): the 16 rows r = mloc*G + jj of kv-head hp*HB + w (member
  // m0+mloc, q-head jj; rows past nm*G are zero queries, not written), as two mma.sync n8
  // tiles that share every K and V^T fragment.  Per 16-token tile: S^T = K Q^T (M = 16
  // tokens, N = 2 x 8 rows, K = 128 dims: 16 MMAs), the online softmax of each row, and
  // O^T += V^T P^T (M = 128 dims in 8 tiles, K = 16 tokens: 16 MMAs).  Lane (g, tq) holds
  // the logits of tokens g and g+8 for rows nt*8 + 2tq, +1 and their outputs for the dims
  // pv_tile gives it; K and q dims go in kchunk order.  The rows' q is read from global
  // memory once per segment.  Returns false when the CTA aborted.
  auto chunk_segment = [&](int& k, int& cnt, int qs, const volatile int* u) -> bool {
    const int s = u[0], hp = u[1], pslot = u[5], m0 = u[7];
    const int nm = u[10];
    int t0 = u[2], t1 = u[3], flags = u[4];
    const int g = lane >> 2, tq = lane & 3;
    const int kvh = hp * HB + w;
    // K chunks 2tq (k-steps j even) and 2tq+1 (j odd) of token g; kchunk adds the slab
    const int kofs0 = swz(w, g, 2 * tq), kofs1 = swz(w, g, 2 * tq + 1);
    uint32_t qf[2][8][2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int r = nt * 8 + g, ml = r / G, jj = r % G;
      const uint4* src = reinterpret_cast<const uint4*>(
          static_cast<const T*>(a.q) + ((long long)(m0 + ml) * a.num_q_heads + kvh * G + jj) * kD);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint4 v = ml < nm ? __ldg(src + kchunk(tq, j)) : make_uint4(0u, 0u, 0u, 0u);
        qf[nt][2 * j][0] = v.x;
        qf[nt][2 * j][1] = v.y;
        qf[nt][2 * j + 1][0] = v.z;
        qf[nt][2 * j + 1][1] = v.w;
      }
    }
    float oacc[2][8][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) oacc[nt][mt][0] = oacc[nt][mt][1] = oacc[nt][mt][2] = oacc[nt][mt][3] = 0.f;
    float mh[2][2] = {{-INFINITY, -INFINITY}, {-INFINITY, -INFINITY}};
    float lh[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
    const int L = slen[s];
    for (;;) {  // the segment's units
      __syncwarp();
      if (lane == 0) mbar_arrive(&qempty[qs]);
      for (int t = t0; t < t1; ++t, ++cnt) {
        const int slot = cnt % nslots;
        wait_or_abort(&full[slot], (cnt / nslots) & 1, abort_flag, a.err, a.wait_limit);
        const int nvalid = min(kTileTok, L - t * kTileTok);
        const uint8_t* Ks = ring + slot * C::SLOT_BYTES;
        const uint8_t* Vs = Ks + C::TILE_BYTES;
        float sc4[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint8_t* kj = Ks + (j >> 1) * C::SLAB_BYTES + ((j & 1) ? kofs1 : kofs0);
          const uint4 ka = *reinterpret_cast<const uint4*>(kj);
          const uint4 kb = *reinterpret_cast<const uint4*>(kj + 1024);  // token g+8
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            Mma<T>::run(sc4[nt], ka.x, kb.x, ka.y, kb.y, qf[nt][2 * j][0], qf[nt][2 * j][1]);
            Mma<T>::run(sc4[nt], ka.z, kb.z, ka.w, kb.w, qf[nt][2 * j + 1][0], qf[nt][2 * j + 1][1]);
          }
        }
        const bool v0 = g < nvalid, v8 = g + 8 < nvalid;
        uint32_t pb[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          const float x0 = v0 ? sc4[nt][0] * a.qscale : -INFINITY;  // token g,   row 2tq
          const float x1 = v0 ? sc4[nt][1] * a.qscale : -INFINITY;  // token g,   row 2tq+1
          const float x2 = v8 ? sc4[nt][2] * a.qscale : -INFINITY;  // token g+8, row 2tq
          const float x3 = v8 ? sc4[nt][3] * a.qscale : -INFINITY;  // token g+8, row 2tq+1
          float mx0 = fmaxf(x0, x2), mx1 = fmaxf(x1, x3);
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
          }
          const float mn0 = fmaxf(mh[nt][0], mx0), mn1 = fmaxf(mh[nt][1], mx1);
          const float al0 = fast_exp2(mh[nt][0] - mn0), al1 = fast_exp2(mh[nt][1] - mn1);
          mh[nt][0] = mn0;
          mh[nt][1] = mn1;
          const float p0 = fast_exp2(x0 - mn0), p1 = fast_exp2(x1 - mn1);
          const float p2 = fast_exp2(x2 - mn0), p3 = fast_exp2(x3 - mn1);
          lh[nt][0] = lh[nt][0] * al0 + (p0 + p2);
          lh[nt][1] = lh[nt][1] * al1 + (p1 + p3);
          if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
            const float2 al = make_float2(al0, al1);
#pragma unroll
            for (int mt = 0; mt < 8; ++mt) {
              const float2 lo = __fmul2_rn(make_float2(oacc[nt][mt][0], oacc[nt][mt][1]), al);
              const float2 hi = __fmul2_rn(make_float2(oacc[nt][mt][2], oacc[nt][mt][3]), al);
              oacc[nt][mt][0] = lo.x;
              oacc[nt][mt][1] = lo.y;
              oacc[nt][mt][2] = hi.x;
              oacc[nt][mt][3] = hi.y;
            }
          }
          pb[nt][0] = transpose8x8(Mma<T>::pack(p0, p1));
          pb[nt][1] = transpose8x8(Mma<T>::pack(p2, p3));
        }
        pv_tile<T, 2, C::SLAB_BYTES>(oacc, Vs, w, g, tq, nvalid, pb);
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[slot]);
      }
      ++k;
      if (flags & kLast) break;
      qs = k % kQSlots;
      wait_or_abort(&qfull[qs], (k / kQSlots) & 1, abort_flag, a.err, a.wait_limit);
      u = unit + qs * kUnitInts;
      if (u[0] < 0 || warp_flag(abort_flag)) return false;
      t0 = u[2];
      t1 = u[3];
      flags = u[4];
    }
    // ---- end of segment: normalised partial rows of the chunk's slot, and (max, sum)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      float lt0 = lh[nt][0], lt1 = lh[nt][1];
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) {
        lt0 += __shfl_xor_sync(0xffffffffu, lt0, o);
        lt1 += __shfl_xor_sync(0xffffffffu, lt1, o);
      }
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int r = nt * 8 + 2 * tq + e;
        if (r / G >= nm) continue;  // past the chunk's members
        const float lt = e ? lt1 : lt0;
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        const long long row = (long long)pslot * (HB * kChunkRows) + w * kChunkRows + r;
        store_pv_row_f32<false>(a.vpart_o + row * kD, oacc[nt], e, inv, g);
        if (g == 0)
          *reinterpret_cast<float2*>(a.vpart_ml + row * 2) = make_float2(mh[nt][e], lt);
      }
    }
    (void)s;
    return true;
  };
  {
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
    const int g = lane >> 2, tq = lane & 3;
    // K chunks 2tq and 2tq+1 of token g (16-bit: k-steps of even / odd j, slab j/2; e4m3:
    // c = 0 / 1)
    const int kofs0 = swz(w, g, 2 * tq), kofs1 = swz(w, g, 2 * tq + 1);
    int cnt = 0;
    // one segment per iteration: its first unit (kFirst) loads q, its last (kLast) writes
    // the result; the segment's state is dead once it is written
    for (int k = 0;;) {
      int qs = k % kQSlots;
      wait_or_abort(&qfull[qs], (k / kQSlots) & 1, abort_flag, a.err, a.wait_limit);
      const volatile int* u = unit + qs * kUnitInts;
      const int s = u[0];
      if (s < 0 || warp_flag(abort_flag)) break;
      if constexpr (SP) {
        if (u[4] & kVirtual) {
          if (!chunk_segment(k, cnt, qs, u)) break;
          continue;
        }
      }
      const int hp = u[1], pslot = u[5], orow = u[7];
      int t0 = u[2], t1 = u[3], flags = u[4];
      uint32_t qf[8][2];    // Q^T fragments of the 8 k-steps
      float oaccs[1][8][4];  // O^T: [m-tile] x heads 2tq, 2tq+1 (dims: pv_tile)
      float(&oacc)[8][4] = oaccs[0];
      float mh0 = -INFINITY, mh1 = -INFINITY, lh0 = 0.f, lh1 = 0.f;  // heads 2tq, 2tq+1
      {
        const uint8_t* qrow = qbuf + qs * C::QBYTES + (w * G + g) * kRowBytes;
        if constexpr (F8) {
          // k-step 4c+i takes dims 4i..4i+3 of the 16-dim chunk 2tq + c (one 32-bit
          // word of e4m3 codes); Q takes the same dims, as f16 pairs
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint8_t* src = qrow + (2 * tq + c) * 32;
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
          for (int j = 0; j < 4; ++j) {  // q-heads past G (rows of the next warp): zero
            const uint4 v = g < G ? *reinterpret_cast<const uint4*>(qrow + kchunk(tq, j) * 16)
                                  : make_uint4(0u, 0u, 0u, 0u);
            qf[2 * j][0] = v.x;
            qf[2 * j][1] = v.y;
            qf[2 * j + 1][0] = v.z;
            qf[2 * j + 1][1] = v.w;
          }
        }
      }
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;
      const int L = slen[s];
      const int kvh = hp * HB + w;
      const float lsc = F8 ? a.qscale * __ldg(a.k_scale + kvh) : a.qscale;
      bool stop = false;
      for (;;) {  // the segment's units
        __syncwarp();
        if (lane == 0) mbar_arrive(&qempty[qs]);
        for (int t = t0; t < t1; ++t, ++cnt) {
          const int slot = cnt % nslots;
          wait_or_abort(&full[slot], (cnt / nslots) & 1, abort_flag, a.err, a.wait_limit);
          const int nvalid = min(kTileTok, L - t * kTileTok);
          // tile layout: column slabs of [HB kv-heads][16 tokens][128 B] (swz)
          const uint8_t* Ks = ring + slot * C::SLOT_BYTES;
          const uint8_t* Vs = Ks + C::TILE_BYTES;

          // ---- S^T = K Q^T: rows tokens g, g+8; columns heads 2tq, 2tq+1
          float sc[4] = {0.f, 0.f, 0.f, 0.f};
          // e4m3: the tile's V^T fragments first, so that their reads and conversions
          // overlap the S products and the softmax
          uint32_t vfr[2][4][4];
          if constexpr (F8) pv_frags_f8(Vs, w, g, tq, nvalid, vfr);
          if constexpr (F8) {
            float sc2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const uint8_t* kc = Ks + (c ? kofs1 : kofs0);
              const uint4 ka = *reinterpret_cast<const uint4*>(kc);
              const uint4 kb = *reinterpret_cast<const uint4*>(kc + 1024);  // token g+8
              const uint32_t wa[4] = {ka.x, ka.y, ka.z, ka.w}, wb[4] = {kb.x, kb.y, kb.z, kb.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                uint32_t alo, ahi, blo, bhi;
                e4m3x4_to_f16x2x2(wa[i], alo, ahi);
                e4m3x4_to_f16x2x2(wb[i], blo, bhi);
                // two accumulators: two chains of four dependent products, not one of eight
                Mma<__half>::run((i & 1) ? sc2 : sc, alo, blo, ahi, bhi, qf[4 * c + i][0],
                                 qf[4 * c + i][1]);
              }
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[e] += sc2[e];
          } else {
            float sc2[4] = {0.f, 0.f, 0.f, 0.f};  // odd k-steps: two chains of four products
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint8_t* kj = Ks + (j >> 1) * C::SLAB_BYTES + ((j & 1) ? kofs1 : kofs0);
              const uint4 ka = *reinterpret_cast<const uint4*>(kj);
              const uint4 kb = *reinterpret_cast<const uint4*>(kj + 1024);  // token g+8
              Mma<T>::run(sc, ka.x, kb.x, ka.y, kb.y, qf[2 * j][0], qf[2 * j][1]);
              Mma<T>::run(sc2, ka.z, kb.z, ka.w, kb.w, qf[2 * j + 1][0], qf[2 * j + 1][1]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) sc[e] += sc2[e];
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
          // ---- O^T += V^T P^T (rows past the sequence end are zeroed: p is 0 there, but the
          // block's unused rows may hold anything)
          const uint32_t pb[1][2] = {{pb0, pb1}};
          if constexpr (F8)
            pv_mma_f8<1>(oaccs, vfr, pb);
          else
            pv_tile<MT, 1, C::SLAB_BYTES>(oaccs, Vs, w, g, tq, nvalid, pb);
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[slot]);
        }
        ++k;
        if (flags & kLast) break;
        qs = k % kQSlots;
        wait_or_abort(&qfull[qs], (k / kQSlots) & 1, abort_flag, a.err, a.wait_limit);
        u = unit + qs * kUnitInts;
        if (u[0] < 0 || warp_flag(abort_flag)) {
          stop = true;
          break;
        }
        t0 = u[2];
        t1 = u[3];
        flags = u[4];
      }
      if (stop) break;

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
          store_pv_row<T, F8>(static_cast<T*>(a.out) +
                                  ((long long)orow * a.num_q_heads + hp * HBG + j0 + e) * kD,
                              oacc, e, inv, g);
        } else {
          const long long row = (long long)pslot * HBG + j0 + e;
          store_pv_row_f32<F8>(a.part_o + row * kD, oacc, e, inv, g);
          if (g == 0)
            *reinterpret_cast<float2*>(a.part_ml + row * 2) =
                make_float2(e ? mh1 : mh0, e ? lt1 : lt0);
        }
      }
    }
  }
}

template <typename T, int G, int HB, bool F8, bool SP>
__global__ void __launch_bounds__(DecodeCfg<G, HB, F8, SP>::THREADS, 1)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV,
                        const __grid_constant__ CUtensorMap tmQ, const DecodeArgs a) {
  extern __shared__ __align__(1024) uint8_t smem[];
  decode_body<T, G, HB, F8, SP>(tmK, tmV, tmQ, a, smem, blockIdx.x, gridDim.x);
}

// A mixed step in one grid (pa_attention_varlen): CTAs [0, D) are the persistent decode grid
// over the sequences of one query row; the rest are chunked-prefill items over the listed
// chunk sequences, which take the SMs left free and then those the decode CTAs leave, so the
// chunks' tensor-core work runs beside the decode rows' HBM stream instead of after it.
template <typename T, int G, int HB>
__global__ void __launch_bounds__(prefill::kThreads, 1)
    varlen_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const __grid_constant__ CUtensorMap tmQ,
                  const __grid_constant__ CUtensorMap tpK,
                  const __grid_constant__ CUtensorMap tpV, const DecodeArgs a,
                  const prefill::Args p, int D) {
  static_assert(DecodeCfg<G, HB, false>::THREADS <= prefill::kThreads, "CTA size");
  extern __shared__ __align__(1024) uint8_t smem[];
  if ((int)blockIdx.x < D)
    decode_body<T, G, HB, false, false>(tmK, tmV, tmQ, a, smem, blockIdx.x, D);
  else
    prefill::prefill_body<T, G>(tpK, tpV, p, smem, blockIdx.x - D);
}

// The sequences of a mixed step with more than one query row (the chunks), in index order:
// chunk_ids[0..n), n = chunk_ids[cap] <= cap; more of them than cap is flagged.  The
// mixed-step kernel starts as its programmatic dependent and its prefill CTAs wait for it.
__global__ void __launch_bounds__(1024) varlen_list_kernel(const int32_t* __restrict__ qsl, int B,
                                                           int32_t* __restrict__ chunk_ids,
                                                           int cap, int* err) {
  griddep_launch_dependents();
  __shared__ int wsum[33];
  const int per = (B + 1023) / 1024;
  const int lo = min(B, (int)threadIdx.x * per), hi = min(B, lo + per);
  int c = 0;
  for (int s = lo; s < hi; ++s) c += (__ldg(qsl + s + 1) - __ldg(qsl + s)) > 1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int wv = wsum[lane];
    int wi = wv;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += t;
    }
    wsum[lane] = wi - wv;
    if (lane == 31) wsum[32] = wi;
  }
  __syncthreads();
  int run = wsum[warp] + incl - c;
  for (int s = lo; s < hi; ++s)
    if (__ldg(qsl + s + 1) - __ldg(qsl + s) > 1) {
      if (run < cap) chunk_ids[run] = s;
      ++run;
    }
  if (threadIdx.x == 0) {
    chunk_ids[cap] = min(wsum[32], cap);
    if (wsum[32] > cap) flag_error(err, PA_DEVERR_QUERY_LAYOUT);
  }
}

constexpr int kMaxPartition = kMaxTilesPerUnit * kTileTok;
constexpr int kMaxSeqs = 4096;
constexpr int kMaxSeqsShared = 2048;  // batch + chunks in the schedule arrays
constexpr int kMaxSmem = 227 * 1024;

// kv-heads per group: all of them up to eight (whole 2 KB rows for 8 heads of 128)
inline int heads_per_item(int num_kv_heads) {
  for (int hb = 8; hb > 1; hb >>= 1)
    if (num_kv_heads % hb == 0) return hb;
  return 1;
}

inline size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace of one launch: merge records (first slot, count) of each (sequence, head
// group), then partial outputs, then (m, l) pairs.
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

template <typename T, int G, int HB, bool F8, bool SP>
pa_status launch_decode(const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQ,
                        DecodeArgs a, int grid, cudaStream_t stream) {
  using C = DecodeCfg<G, HB, F8, SP>;
  // schedule arrays: 3 ints per sequence (batch and chunks) + 1, and the groups' chunk starts
  const long long seq_ints = 3LL * (a.num_seqs + (SP ? a.vcap : 0)) + 1 + (SP ? a.num_groups + 1 : 0);
  const size_t ring_off = ((C::OFF_SEQ + (size_t)seq_ints * 4 + 1023) / 1024) * 1024;
  const long long room = (long long)kMaxSmem - (long long)ring_off;
  const int nslots = (int)std::min<long long>(kMaxSlots, room / C::SLOT_BYTES);
  if (nslots < 2) return PA_ERR_UNSUPPORTED;
  a.ring_off = (int)ring_off;
  a.nslots = nslots;
  const size_t smem = ring_off + (size_t)nslots * C::SLOT_BYTES;
  auto kern = paged_decode_kernel<T, G, HB, F8, SP>;
  if (!ensure_dynamic_smem(reinterpret_cast<const void*>(kern), (int)smem)) return PA_ERR_CUDA;
  // a programmatic dependent of the stream's previous kernel: the grid's launch and setup
  // overlap that kernel's end; the CTAs wait for it before reading any input
  a.wait_prior = 1;
  {
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(C::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kern, tmK, tmV, tmQ, a) != cudaSuccess) {
      (void)cudaGetLastError();
      return PA_ERR_CUDA;
    }
  }
  if (check_launch() != PA_OK) return PA_ERR_CUDA;
  int launches = 1;
  if (grid > 1 || SP) {
    // the merge of split groups, as a programmatic dependent: its CTAs may start while the
    // decode grid drains and wait for it inside
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
    if (cudaLaunchKernelEx(&cfg, merge_kernel<T, G, SP>, a, HB) != cudaSuccess) {
      (void)cudaGetLastError();
      return PA_ERR_CUDA;
    }
    if (check_launch() != PA_OK) return PA_ERR_CUDA;
    ++launches;
  }
  set_launch_count(launches);
  return PA_OK;
}

template <typename T, int G, bool F8, bool SP>
pa_status dispatch_hb(int HB, const CUtensorMap& tmK, const CUtensorMap& tmV,
                      const CUtensorMap& tmQ, const DecodeArgs& a, int grid, cudaStream_t stream) {
  switch (HB) {
    case 1: return launch_decode<T, G, 1, F8, SP>(tmK, tmV, tmQ, a, grid, stream);
    case 2: return launch_decode<T, G, 2, F8, SP>(tmK, tmV, tmQ, a, grid, stream);
    case 4: return launch_decode<T, G, 4, F8, SP>(tmK, tmV, tmQ, a, grid, stream);
    case 8: return launch_decode<T, G, 8, F8, SP>(tmK, tmV, tmQ, a, grid, stream);
    default: return PA_ERR_UNSUPPORTED;
  }
}

// A decode launch's arguments, prepared by decode_impl for a caller that launches them in
// a kernel of its own (the mixed-step kernel of pa_attention_varlen).
struct PreparedDecode {
  DecodeArgs a;
  CUtensorMap tmK, tmV, tmQ;
  int grid, G, HB;
};

template <typename T, bool F8, bool SP = false>
pa_status dispatch_group(int G, int HB, const CUtensorMap& tmK, const CUtensorMap& tmV,
                         const CUtensorMap& tmQ, const DecodeArgs& a, int grid,
                         cudaStream_t stream) {
  switch (G) {
    case 1: return dispatch_hb<T, 1, F8, SP>(HB, tmK, tmV, tmQ, a, grid, stream);
    case 2: return dispatch_hb<T, 2, F8, SP>(HB, tmK, tmV, tmQ, a, grid, stream);
    case 4: return dispatch_hb<T, 4, F8, SP>(HB, tmK, tmV, tmQ, a, grid, stream);
    case 8: return dispatch_hb<T, 8, F8, SP>(HB, tmK, tmV, tmQ, a, grid, stream);
    default: return PA_ERR_UNSUPPORTED;
  }
}

// The mixed step: the chunk list, the mixed-step grid (D decode CTAs + P prefill items, a
// programmatic dependent of the list) and the merge of the decode rows' split groups.
template <typename T, int G, int HB>
pa_status launch_varlen(PreparedDecode& d, const prefill::Args& p, const CUtensorMap& tpK,
                        const CUtensorMap& tpV, int D, int P, const int32_t* qsl, int B,
                        int32_t* chunk_ids, int cap, cudaStream_t stream) {
  using C = DecodeCfg<G, HB, false>;
  const size_t ring_off =
      ((C::OFF_SEQ + (size_t)(3LL * d.a.num_seqs + 1) * 4 + 1023) / 1024) * 1024;
  const long long room = (long long)kMaxSmem - (long long)ring_off;
  const int nslots = (int)std::min<long long>(kMaxSlots, room / C::SLOT_BYTES);
  if (nslots < 2) return PA_ERR_UNSUPPORTED;
  d.a.ring_off = (int)ring_off;
  d.a.nslots = nslots;
  const size_t smem =
      std::max(ring_off + (size_t)nslots * C::SLOT_BYTES, (size_t)prefill::SMEM_BYTES);
  auto kern = varlen_kernel<T, G, HB>;
  if (!ensure_dynamic_smem(reinterpret_cast<const void*>(kern), (int)smem)) return PA_ERR_CUDA;
  varlen_list_kernel<<<1, 1024, 0, stream>>>(qsl, B, chunk_ids, cap, d.a.err);
  if (check_launch() != PA_OK) return PA_ERR_CUDA;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(D + P));
  cfg.blockDim = dim3(prefill::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kern, d.tmK, d.tmV, d.tmQ, tpK, tpV, d.a, p, D) != cudaSuccess) {
    (void)cudaGetLastError();
    return PA_ERR_CUDA;
  }
  if (check_launch() != PA_OK) return PA_ERR_CUDA;
  const int warps = d.a.num_seqs * d.a.num_q_heads;
  cudaLaunchConfig_t mcfg = cfg;
  mcfg.gridDim = dim3((unsigned)((warps + 7) / 8));
  mcfg.blockDim = dim3(256);
  mcfg.dynamicSmemBytes = 0;
  if (cudaLaunchKernelEx(&mcfg, merge_kernel<T, G, false>, d.a, HB) != cudaSuccess) {
    (void)cudaGetLastError();
    return PA_ERR_CUDA;
  }
  if (check_launch() != PA_OK) return PA_ERR_CUDA;
  set_launch_count(3);
  return PA_OK;
}

template <typename T>
pa_status dispatch_varlen(PreparedDecode& d, const prefill::Args& p, const CUtensorMap& tpK,
                          const CUtensorMap& tpV, int D, int P, const int32_t* qsl, int B,
                          int32_t* chunk_ids, int cap, cudaStream_t stream) {
#define PA_VARLEN_HB(GG)                                                                 \
  switch (d.HB) {                                                                        \
    case 1: return launch_varlen<T, GG, 1>(d, p, tpK, tpV, D, P, qsl, B, chunk_ids, cap, stream); \
    case 2: return launch_varlen<T, GG, 2>(d, p, tpK, tpV, D, P, qsl, B, chunk_ids, cap, stream); \
    case 4: return launch_varlen<T, GG, 4>(d, p, tpK, tpV, D, P, qsl, B, chunk_ids, cap, stream); \
    case 8: return launch_varlen<T, GG, 8>(d, p, tpK, tpV, D, P, qsl, B, chunk_ids, cap, stream); \
    default: return PA_ERR_UNSUPPORTED;                                                  \
  }
  switch (d.G) {
    case 1: PA_VARLEN_HB(1)
    case 2: PA_VARLEN_HB(2)
    case 4: PA_VARLEN_HB(4)
    case 8: PA_VARLEN_HB(8)
    default: return PA_ERR_UNSUPPORTED;
  }
#undef PA_VARLEN_HB
}

// Share of the SMs the decode rows of a mixed step take; the chunks' items run on the
// others and then on those the decode CTAs leave.
constexpr int kVarlenDecodeShareNum = 2, kVarlenDecodeShareDen = 3;

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
                      int num_q_rows = 0, int32_t* chunk_ids = nullptr, int chunk_cap = 0,
                      pa::PreparedDecode* prep = nullptr) {
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
  // shared prefixes: the chunks of each group's members over the group's prefix join the
  // schedule after the batch (at most one chunk per member)
  int mc = 0, vcap = 0;
  long long vtiles = 0;
  if (sp) {
    if (num_seqs > pa::kMaxSeqsShared) return PA_ERR_UNSUPPORTED;
    mc = pa::kChunkRows / G;
    vcap = (int)std::min<long long>(
        num_seqs, (long long)sp->num_groups * ((sp->max_group_size + mc - 1) / mc));
    vtiles = (long long)vcap * NHP *
             ((std::min<long long>(sp->max_prefix_len, seq_cap) + pa::kTileTok - 1) / pa::kTileTok);
  }
  const long long tiles_max = (long long)num_seqs * NHP * nt_max + vtiles;
  if (tiles_max > INT_MAX / 2) return PA_ERR_UNSUPPORTED;
  // persistent grid of one CTA per SM; an explicit partition caps each CTA's share
  long long grid = std::min<long long>(std::max(1, pa::num_sms()), pa::kMaxGrid);
  grid = std::max<long long>(1, std::min<long long>(grid, tiles_max));
  if (partition_size > 0)
    grid = std::max<long long>(grid, (tiles_max + partition_size / 16 - 1) / (partition_size / 16));
  const long long groups = (long long)num_seqs * NHP;
  const pa::WsLayout lay = pa::ws_layout(groups, grid + groups, HBG, head_dim);
  // shared prefixes: the chunks' partial rows follow, (grid + chunks x head groups) slots of
  // HB x 16 rows, then the members' chunk records (one per sequence and head group)
  const long long vslots = sp ? grid + (long long)vcap * NHP : 0;
  const long long vrows = vslots * HB * pa::kChunkRows;
  size_t voff = 0, cmeta_off = 0, need = lay.total;
  if (sp) {
    voff = pa::align256(lay.total);
    cmeta_off = pa::align256(voff + (size_t)vrows * (head_dim + 2) * sizeof(float));
    need = cmeta_off + (size_t)num_seqs * NHP * sizeof(int4);
  }
  if (!workspace || workspace_bytes < need) return PA_ERR_WORKSPACE_TOO_SMALL;
  if ((uintptr_t)workspace & 255) return PA_ERR_INVALID_ARG;
  int* err = pa::launch_prologue();
  if (!err) return PA_ERR_CUDA;

  CUtensorMap tmK, tmV, tmQ;
  const uint64_t row = (uint64_t)head_dim * 2;
  const uint64_t crow = (uint64_t)head_dim * (f8 ? 1 : 2);  // one kv-head of one token
  // the cache viewed as [block][token][kv-head][dim] with token and kv-head swapped in the
  // map: a box of 16 tokens x HB kv-heads x one 128-byte column slab lands as
  // [kv-head][token][128 B], swizzled (the kernel's swz)
  const uint64_t cdims[4] = {(uint64_t)head_dim, (uint64_t)block_size, (uint64_t)num_kv_heads,
                             (uint64_t)num_blocks};
  const uint64_t cstr[3] = {crow * num_kv_heads, crow, crow * num_kv_heads * block_size};
  const uint32_t cbox[4] = {f8 ? 128u : 64u, 16, (uint32_t)HB, 1};
  const uint64_t qdims[3] = {(uint64_t)head_dim, (uint64_t)num_q_heads,
                             (uint64_t)(qsl ? num_q_rows : num_seqs)};
  const uint64_t qstr[2] = {row, row * num_q_heads};
  const uint32_t qbox[3] = {(uint32_t)head_dim, (uint32_t)HBG, 1};
  const CUtensorMapDataType ct =
      f8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_UINT16;
  if (!pa::encode_tmap(&tmK, ct, k_cache, 4, cdims, cstr, cbox, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !pa::encode_tmap(&tmV, ct, v_cache, 4, cdims, cstr, cbox, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !pa::encode_tmap_16bit(&tmQ, q, 3, qdims, qstr, qbox, CU_TENSOR_MAP_SWIZZLE_NONE))
    return PA_ERR_CUDA;

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  pa::DecodeArgs a;
  a.out = out;
  a.block_tables = block_tables;
  a.seq_lens = seq_lens;
  a.q = q;
  a.meta = reinterpret_cast<int2*>(ws + lay.meta);
  a.cmeta = nullptr;
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
  a.wait_limit = pa::take_wait_limit(pa::kTestDecode, &a.test_withhold);
  a.wait_prior = 0;  // set by the launch that makes the grid a programmatic dependent
  a.group_starts = a.prefix_lens = nullptr;
  a.vpart_o = a.vpart_ml = nullptr;
  a.num_groups = a.mc = a.vcap = a.max_prefix = 0;
  a.qsl = qsl;
  a.num_q_rows = qsl ? num_q_rows : num_seqs;
  a.chunk_ids = chunk_ids;
  a.chunk_cap = chunk_cap;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (prep) {  // the caller launches (the mixed-step kernel)
    prep->a = a;
    prep->tmK = tmK;
    prep->tmV = tmV;
    prep->tmQ = tmQ;
    prep->grid = (int)grid;
    prep->G = G;
    prep->HB = HB;
    return PA_OK;
  }
  if (sp) {
    // one decode grid: every sequence's own keys, and each chunk of every group's members
    // over the group's prefix (the prefix read once per chunk); the merge pass folds both
    a.group_starts = sp->group_starts;
    a.prefix_lens = sp->prefix_lens;
    a.num_groups = sp->num_groups;
    a.mc = mc;
    a.vcap = vcap;
    a.max_prefix = sp->max_prefix_len;
    a.vpart_o = reinterpret_cast<float*>(ws + voff);
    a.vpart_ml = a.vpart_o + (size_t)vrows * head_dim;
    a.cmeta = reinterpret_cast<int4*>(ws + cmeta_off);
    return dtype == PA_F16
               ? pa::dispatch_group<__half, false, true>(G, HB, tmK, tmV, tmQ, a, (int)grid, st)
               : pa::dispatch_group<__nv_bfloat16, false, true>(G, HB, tmK, tmV, tmQ, a,
                                                                 (int)grid, st);
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
// device current, and kept for the life of the process: a cudaDeviceReset invalidates
// it).  nullptr if the lookup failed.
void* scratch_for_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) {
      (void)cudaGetLastError();  // the failed lookup is reported here, not by a later launch
      return nullptr;
    }
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
                                                         int num_kv_heads, int head_dim,
                                                         int max_seq_len) {
  const size_t base = pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_seq_len, 0);
  if (base == 0 || num_kv_heads <= 0) return 0;
  // the chunks' partial rows: (grid + chunks x head groups) slots of (kv-heads per group x 16)
  // rows, at most (256 + num_seqs) x num_kv_heads x 16 rows of head_dim + 2 fp32; then the
  // members' chunk records (at most num_seqs x num_kv_heads int4)
  return pa::align256(pa::align256(base) + ((size_t)pa::kMaxGrid + num_seqs) * num_kv_heads *
                                               pa::kChunkRows * (head_dim + 2) * sizeof(float)) +
         (size_t)num_seqs * num_kv_heads * 4 * sizeof(int);
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
  if (cap == 0)  // rows of one query only: the decode kernel (it lists stray chunks)
    return decode_impl(out, q, nullptr, nullptr, k_cache, v_cache, nullptr, nullptr,
                       block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_q_heads,
                       num_kv_heads, head_dim, scale, block_size, num_blocks, max_seq_len, 0,
                       workspace, dws, dtype, stream, nullptr, query_start_loc, num_q_rows,
                       chunk_ids, 0);
  // one grid for both: the decode rows' arguments and the chunks' items, prepared
  pa::PreparedDecode d;
  pa_status st = decode_impl(out, q, nullptr, nullptr, k_cache, v_cache, nullptr, nullptr,
                             block_tables, max_blocks_per_seq, seq_lens, num_seqs, num_q_heads,
                             num_kv_heads, head_dim, scale, block_size, num_blocks, max_seq_len,
                             0, workspace, dws, dtype, stream, nullptr, query_start_loc,
                             num_q_rows, nullptr, 0, &d);
  if (st != PA_OK) return st;
  pa::prefill::Args p;
  CUtensorMap tpK, tpV;
  st = pa::chunked_prefill_impl(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                seq_lens, query_start_loc, num_seqs, max_query_len, num_q_heads,
                                num_kv_heads, head_dim, scale, block_size, num_blocks, max_seq_len,
                                nullptr, 0, dtype, stream, true, chunk_ids, cap, &p, &tpK, &tpV);
  if (st != PA_OK) return st;
  p.wait_list = 1;
  const int D = std::max(
      1, std::min(d.grid, (pa::num_sms() * pa::kVarlenDecodeShareNum + pa::kVarlenDecodeShareDen - 1) /
                              pa::kVarlenDecodeShareDen));
  if ((long long)D + p.whole_items > INT_MAX) return PA_ERR_UNSUPPORTED;
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  return dtype == PA_F16 ? pa::dispatch_varlen<__half>(d, p, tpK, tpV, D, p.whole_items,
                                                       query_start_loc, num_seqs, chunk_ids, cap, cs)
                         : pa::dispatch_varlen<__nv_bfloat16>(d, p, tpK, tpV, D, p.whole_items,
                                                              query_start_loc, num_seqs, chunk_ids,
                                                              cap, cs);
}
