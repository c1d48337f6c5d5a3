// Chunked-prefill CTA body (tcgen05), shared by the chunked-prefill kernel (prefill.cu) and
// the mixed-step kernel of pa_attention_varlen (decode.cu).  What it computes and how:
// prefill.cu's header.
#pragma once

#include <algorithm>
#include <type_traits>

#include "pa_device.cuh"

namespace pa {
namespace prefill {

constexpr int kD = 128;
constexpr int kBN = 128;              // keys per tile
constexpr int kM = 128;               // rows per M-tile
constexpr int kHalfBytes = kM * 128;  // 128 rows x 64 elements x 2 B (one SW128 half)
constexpr int kTileBytes = 2 * kHalfBytes;  // 32 KB: a 128 x 128 16-bit tile
constexpr int kThreads = 12 * 32;

struct Args {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  const int32_t* qsl;
  int* err;
  int num_seqs, num_q_heads, num_kv_heads, max_blocks, log2_bs, num_blocks;
  int max_query_len, seq_cap, qblocks;
  float qscale;  // scale * log2(e)
  // wave tail: the last `split_items` items (after `whole_items`) run as two CTAs each,
  // one per half of the item's key tiles, writing normalised partials that
  // merge_split_kernel combines ([split item][half][256 rows] fp32 rows and (m, l);
  // rowmap [split item][256 rows]: the output row, -1 for rows past the chunk)
  int whole_items, split_items;
  float* part_o;
  float* part_ml;
  int* rowmap;
  // varlen call: sequences with a single query row are left to the decode kernel.  With
  // chunk_ids, item "sequence" r is the r-th sequence with more than one query row,
  // chunk_ids[r] (chunk_ids[chunk_cap] holds how many; num_seqs = chunk_cap)
  int skip_single;
  const int32_t* chunk_ids;
  int chunk_cap;
  int wait_list;  // chunk_ids is written by the previous launch of the stream (wait for it)
  long long wait_limit;  // SM cycles any pipeline wait may take before the CTA gives up
  int test_withhold;     // testing hook: CTA 0's producer withholds its first K tile
};

// shared memory carve-up
constexpr int OFF_Q = 0;                               // 2 M-tiles x 32 KB
constexpr int OFF_K = OFF_Q + 2 * kTileBytes;          // 2 stages x 32 KB
constexpr int OFF_V = OFF_K + 2 * kTileBytes;          // 2 stages x 32 KB
constexpr int OFF_BAR = OFF_V + 2 * kTileBytes;
// barriers: q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], p_full[2],
// o_full[2], drain (the MMA issuer's last commit after an abort)
constexpr int NBAR = 1 + 2 * 7 + 1;
constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
constexpr int OFF_ABORT = OFF_TMEM + 8;
constexpr int SMEM_BYTES = OFF_ABORT + 8 + 1024;  // + alignment slack

// max of three (one instruction on sm_100)
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo_bytes,
                                               uint32_t sbo_bytes) {
  return (uint64_t)((saddr & 0x3FFFF) >> 4) | ((uint64_t)(lbo_bytes >> 4) << 16) |
         ((uint64_t)(sbo_bytes >> 4) << 32) | (1ull << 46) | (2ull << 61);
}

// kind::f16 instruction descriptor: fp32 accumulate, M=128, N=128.
__host__ __device__ constexpr uint32_t idesc_f16(bool bf16, bool b_mn_major) {
  return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) |
         ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kM >> 4) << 24);
}

__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accum));
}

__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                       uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accum));
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 64 consecutive columns of this thread's TMEM lane, waited for inside the same asm
// statement, so no use of the registers can be scheduled before the data is there.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float* v) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]),
        "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]),
        "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]),
        "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]),
        "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 64; ++i) v[i] = __uint_as_float(r[i]);
}

// 128 consecutive columns of this thread's TMEM lane in one load, waited for inside the
// same asm statement (one wait per row of S instead of two).
__device__ __forceinline__ void tmem_ld128(uint32_t taddr, float* v) {
  uint32_t r[128];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x128.b32 {"
      "%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
      "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
      "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63,"
      "%64,%65,%66,%67,%68,%69,%70,%71,%72,%73,%74,%75,%76,%77,%78,%79,"
      "%80,%81,%82,%83,%84,%85,%86,%87,%88,%89,%90,%91,%92,%93,%94,%95,"
      "%96,%97,%98,%99,%100,%101,%102,%103,%104,%105,%106,%107,%108,%109,%110,%111,"
      "%112,%113,%114,%115,%116,%117,%118,%119,%120,%121,%122,%123,%124,%125,%126,%127}, [%128];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]),
        "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]),
        "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]),
        "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]),
        "=r"(r[63]), "=r"(r[64]), "=r"(r[65]), "=r"(r[66]), "=r"(r[67]), "=r"(r[68]), "=r"(r[69]),
        "=r"(r[70]), "=r"(r[71]), "=r"(r[72]), "=r"(r[73]), "=r"(r[74]), "=r"(r[75]), "=r"(r[76]),
        "=r"(r[77]), "=r"(r[78]), "=r"(r[79]), "=r"(r[80]), "=r"(r[81]), "=r"(r[82]), "=r"(r[83]),
        "=r"(r[84]), "=r"(r[85]), "=r"(r[86]), "=r"(r[87]), "=r"(r[88]), "=r"(r[89]), "=r"(r[90]),
        "=r"(r[91]), "=r"(r[92]), "=r"(r[93]), "=r"(r[94]), "=r"(r[95]), "=r"(r[96]), "=r"(r[97]),
        "=r"(r[98]), "=r"(r[99]), "=r"(r[100]), "=r"(r[101]), "=r"(r[102]), "=r"(r[103]), "=r"(r[104]),
        "=r"(r[105]), "=r"(r[106]), "=r"(r[107]), "=r"(r[108]), "=r"(r[109]), "=r"(r[110]), "=r"(r[111]),
        "=r"(r[112]), "=r"(r[113]), "=r"(r[114]), "=r"(r[115]), "=r"(r[116]), "=r"(r[117]), "=r"(r[118]),
        "=r"(r[119]), "=r"(r[120]), "=r"(r[121]), "=r"(r[122]), "=r"(r[123]), "=r"(r[124]), "=r"(r[125]),
        "=r"(r[126]), "=r"(r[127])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 128; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&w)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(w[0]), "r"(w[1]), "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7]),
      "r"(w[8]), "r"(w[9]), "r"(w[10]), "r"(w[11]), "r"(w[12]), "r"(w[13]), "r"(w[14]),
      "r"(w[15])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Wait that stops waiting once the CTA has given up (at once, or as soon as another warp
// does).  After a wait that may have been skipped, a thread makes no further arrival on a
// barrier that counts transaction bytes (its previous phase may still be pending).
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

template <typename T>
__device__ __forceinline__ uint32_t pack16(float lo, float hi) {
  return Elem<T>::pack2(lo, hi);
}

// The prefill CTA of grid position `cta` (its item, or its half of a split item), with its
// dynamic shared memory at `smem_raw`.  The CTA has kThreads threads.
template <typename T, int G>
__device__ __forceinline__ void prefill_body(const CUtensorMap& tmK, const CUtensorMap& tmV,
                                             const Args& a, uint8_t* smem_raw, const int cta) {
  constexpr int MQ = kM / G;  // queries per M-tile
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bar;
  uint64_t* k_full = bar + 1;
  uint64_t* k_empty = bar + 3;
  uint64_t* v_full = bar + 5;
  uint64_t* v_empty = bar + 7;
  uint64_t* s_full = bar + 9;
  uint64_t* p_full = bar + 11;
  uint64_t* o_full = bar + 13;
  uint64_t* drain = bar + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // the merge of split items may be scheduled now; it waits for this grid itself
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- which (sequence, kv-head, query block), and which part of its keys
  int item = cta, part = -1;  // part -1: all keys; 0 / 1: first / second half
  if (a.split_items > 0 && cta >= a.whole_items) {
    const int j = cta - a.whole_items;
    item = a.whole_items + (j >> 1);
    part = j & 1;
  }
  const int sidx = item - a.whole_items;  // index among the split items (part >= 0)
  auto mark_rows_unused = [&]() {         // a split item that writes no rows
    if (part == 0)
      for (int i = threadIdx.x; i < 2 * kM; i += blockDim.x) a.rowmap[sidx * 2 * kM + i] = -1;
  };
  const int qb = item % a.qblocks;
  const int h = (item / a.qblocks) % a.num_kv_heads;
  int s = item / (a.qblocks * a.num_kv_heads);
  if (a.chunk_ids != nullptr) {
    if (a.wait_list) griddep_wait();  // the list comes from the launch before this one
    if (s >= __ldg(a.chunk_ids + a.chunk_cap)) {  // fewer chunks than the bound
      mark_rows_unused();
      return;
    }
    s = __ldg(a.chunk_ids + s);
  }
  const int q_begin = a.qsl[s];
  const int n = a.qsl[s + 1] - q_begin;
  const int Lraw = a.seq_lens[s];
  const int L = Lraw < 0 ? 0 : (Lraw > a.seq_cap ? a.seq_cap : Lraw);
  const int q0 = qb * 2 * MQ;
  if (n < 0 || n > L || n > a.max_query_len || Lraw != L) {
    if (threadIdx.x == 0 && qb == 0 && h == 0)
      flag_error(a.err, (n < 0 || n > L || n > a.max_query_len) ? PA_DEVERR_QUERY_LAYOUT
                                                               : PA_DEVERR_SEQ_TOO_LONG);
    if (n < 0 || n > L || n > a.max_query_len) {
      mark_rows_unused();
      return;
    }
  }
  if (q0 >= n || (a.skip_single && n == 1)) {  // past the chunk, or a decode row
    mark_rows_unused();
    return;
  }
  // keys any row of this CTA can see: [0, kv_end); this CTA takes tiles [kt_lo, kt_hi)
  const int kv_end = min(L, L - n + min(n, q0 + 2 * MQ));
  const int n_kt_all = (kv_end + kBN - 1) / kBN;
  const int kt_lo = part == 1 ? n_kt_all / 2 : 0;
  const int kt_hi = part == 0 ? n_kt_all / 2 : n_kt_all;
  const int n_kt = kt_hi - kt_lo;  // tiles here; loops below count them from 0

  if (threadIdx.x == 0) {
    mbar_init(q_full, 8);  // one arrival per softmax warp once its Q rows are in place
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
      mbar_init(&v_full[i], 1);
      mbar_init(&v_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 4);
      mbar_init(&o_full[i], 1);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(
                     smem_u32(tmem_slot))
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= 4) {
    // softmax warpgroups: 192 registers each thread (one S row of 128 fp32 in registers)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 192;\n" ::: "memory");
    // ======================== softmax warpgroups ========================
    const int mt = (warp - 4) >> 2;
    const int wq = warp & 3;              // TMEM lane quarter
    const int r = wq * 32 + lane;         // row of the M-tile
    const int qi = q0 + mt * MQ + r / G;  // query index within the chunk
    const bool row_valid = qi < n;
    // last visible key (inclusive), causal
    const int limit = L - n + min(qi, n - 1);
    const uint32_t t_s = tmem + ((uint32_t)(wq * 32) << 16) + mt * 128;
    const uint32_t t_o = tmem + ((uint32_t)(wq * 32) << 16) + 256 + mt * 128;
    // lowest limit in the warp decides whether a tile needs the causal mask
    int wlim = limit;
#pragma unroll
    for (int o = 16; o; o >>= 1) wlim = min(wlim, __shfl_xor_sync(0xffffffffu, wlim, o));
    {
      // this thread's Q row -> shared memory, 128-byte swizzle: 16-byte chunk j of row r
      // of a 64-element half sits at chunk position j ^ (r % 8)
      const uint4* src = reinterpret_cast<const uint4*>(
          static_cast<const T*>(a.q) +
          ((long long)(q_begin + qi) * a.num_q_heads + h * G + (r % G)) * kD);
      uint8_t* dst = smem + OFF_Q + mt * kTileBytes + r * 128;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        const uint4 w = row_valid ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
        *reinterpret_cast<uint4*>(dst + (c >> 3) * kHalfBytes + (((c & 7) ^ (r & 7)) << 4)) = w;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
    }
    float m_ref = -INFINITY, l = 0.f;
    for (int kt = 0; kt < n_kt; ++kt) {
      wait_or_abort(&s_full[mt], kt & 1, abort_flag, a.err, a.wait_limit);
      tc_fence_after();
      const int key0 = (kt_lo + kt) * kBN;
      // the whole S row (128 keys) in registers: one pass over TMEM
      float v[kBN];
      tmem_ld128(t_s, v);
      if (key0 + kBN - 1 > wlim) {  // causal diagonal or sequence end in this tile
#pragma unroll
        for (int i = 0; i < kBN; ++i)
          if (key0 + i > limit) v[i] = -INFINITY;
      }
      // row max: eight independent chains of three-input maxima (the softmax warps are
      // bound by instruction issue, so every instruction here counts)
      float mx8[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        mx8[j] = v[j];
#pragma unroll
        for (int i = 8; i < kBN - 8; i += 16) mx8[j] = fmax3(mx8[j], v[i + j], v[i + 8 + j]);
        mx8[j] = fmaxf(mx8[j], v[kBN - 8 + j]);
      }
      const float mx = fmax3(fmax3(mx8[0], mx8[1], mx8[2]), fmax3(mx8[3], mx8[4], mx8[5]),
                             fmaxf(mx8[6], mx8[7])) *
                       a.qscale;
      // lazy reference max: move it only when this tile exceeds it by more than 8
      float alpha = 1.f;
      if (mx > m_ref + 8.f) {
        alpha = fast_exp2(m_ref - mx);  // m_ref = -inf -> 0
        m_ref = mx;
      }
      if (kt > 0 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float o[32];
          tmem_ld32(t_o + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 r = __fmul2_rn(make_float2(o[i], o[i + 1]), make_float2(alpha, alpha));
            o[i] = r.x;
            o[i + 1] = r.y;
          }
          tmem_st32(t_o + c * 32, o);
        }
      }
      // p = 2^(x*qscale - m_ref); masked keys hold -inf and give 0 (the offset is kept
      // finite while every key so far was masked); pairs of logits scaled and summed as
      // f32x2 (one instruction per pair)
      const float nm = m_ref == -INFINITY ? 0.f : -m_ref;
      const float2 qs2 = make_float2(a.qscale, a.qscale), nm2 = make_float2(nm, nm);
      float2 sum4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                        make_float2(0.f, 0.f)};
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t w[16];
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const float2 x = __ffma2_rn(make_float2(v[c * 32 + i], v[c * 32 + i + 1]), qs2, nm2);
          const float2 p = make_float2(fast_exp2(x.x), fast_exp2(x.y));
          sum4[(i >> 1) & 3] = __fadd2_rn(sum4[(i >> 1) & 3], p);
          w[i >> 1] = pack16<T>(p.x, p.y);
        }
        tmem_st16(t_s + c * 16, w);
      }
      const float sum = ((sum4[0].x + sum4[0].y) + (sum4[1].x + sum4[1].y)) +
                        ((sum4[2].x + sum4[2].y) + (sum4[3].x + sum4[3].y));
      l = l * alpha + sum;
      // keys past the sequence end in the last tile: clear their V rows
      if (mt == 0 && kt_lo + kt == n_kt_all - 1 && L < key0 + kBN) {
        wait_or_abort(&v_full[kt & 1], (kt >> 1) & 1, abort_flag, a.err, a.wait_limit);
        uint8_t* vt = smem + OFF_V + (kt & 1) * kTileBytes;
        const int first = L - key0;  // first row to clear
        for (int i = threadIdx.x & 127; i < (kBN - first) * 16; i += 128) {
          const int rr = first + i / 16, chunk = i % 16;  // 16 x 16 B per row (two halves)
          *reinterpret_cast<uint4*>(vt + (chunk >> 3) * kHalfBytes + rr * 128 + (chunk & 7) * 16) =
              make_uint4(0, 0, 0, 0);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[mt]);
    }
    // ---- epilogue: O / l -> out
    wait_or_abort(&o_full[mt], 0, abort_flag, a.err, a.wait_limit);
    tc_fence_after();
    const float inv = l > 0.f ? 1.f / l : 0.f;
    if (part < 0) {
      T* orow = static_cast<T*>(a.out) +
                ((long long)(q_begin + qi) * a.num_q_heads + h * G + (r % G)) * kD;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(t_o + c * 32, v);
        if (row_valid && n_kt > 0) {
          uint32_t w[16];
#pragma unroll
          for (int i = 0; i < 32; i += 2) w[i >> 1] = pack16<T>(v[i] * inv, v[i + 1] * inv);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            *reinterpret_cast<uint4*>(orow + c * 32 + j * 8) =
                make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
        }
      }
    } else {
      // half of a split item: normalised partial row and its (reference max, sum)
      const bool any = n_kt > 0 && l > 0.f;
      const long long prow = (long long)(sidx * 2 + part) * 2 * kM + mt * kM + r;
      float* po = a.part_o + prow * kD;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(t_o + c * 32, v);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<float4*>(po + c * 32 + j * 4) =
              any ? make_float4(v[4 * j] * inv, v[4 * j + 1] * inv, v[4 * j + 2] * inv,
                                v[4 * j + 3] * inv)
                  : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      *reinterpret_cast<float2*>(a.part_ml + prow * 2) =
          any ? make_float2(m_ref, l) : make_float2(-INFINITY, 0.f);
      if (part == 0)
        a.rowmap[sidx * 2 * kM + mt * kM + r] =
            row_valid && n_kt_all > 0
                ? (int)(((long long)(q_begin + qi) * a.num_q_heads + h * G + (r % G)))
                : -1;
    }
  } else {
    // producer / MMA issuer / two idle warps: 120 registers each thread (fewer spill the
    // producer's block-id runs); 128 x 120 + 256 x 192 = 384 x 168, the registers the CTA
    // is launched with
    asm volatile("setmaxnreg.dec.sync.aligned.u32 120;\n" ::: "memory");
    if (warp == 0) {
      // ======================== TMA producer ========================
      if (lane == 0) {
        prefetch_tmap(&tmK);
        prefetch_tmap(&tmV);
        const int32_t* trow = a.block_tables + (long long)s * a.max_blocks;
        const int bs_mask = (1 << a.log2_bs) - 1;
        // block-table entries of a tile's eight 16-token runs, read one tile ahead so
        // that their latency overlaps the previous tile's waits and copies
        auto table_ids = [&](int kt, int (&id)[8]) {
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const int pos = (kt_lo + kt) * kBN + r * 16;
            id[r] = pos < L ? __ldg(trow + (pos >> a.log2_bs)) : -1;
          }
        };
        int next_id[8];
        if (n_kt > 0) table_ids(0, next_id);
        // K tiles (V tiles) handled so far, and bit i: the copy of the i-th last of them was
        // issued.  A stage is reused only after its previous tile was consumed, so only the
        // last two tiles of each ring can still be landing.
        uint32_t k_issued = 0, v_issued = 0;
        int nk = 0, nv = 0;
        for (int kt = 0; kt < n_kt; ++kt) {
          const int st = kt & 1;
          const uint32_t ph = ((kt >> 1) & 1) ^ 1;
          // block ids of the tile's eight 16-token runs (out of range -> zero fill)
          int bid[8], row[8];
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const int pos = (kt_lo + kt) * kBN + r * 16;
            const int id = next_id[r];
            bid[r] = a.num_blocks;  // past the tensor: TMA fills zeros
            row[r] = pos & bs_mask;
            if (pos < L) {
              if ((unsigned)id < (unsigned)a.num_blocks) bid[r] = id;
              else flag_error(a.err, PA_DEVERR_BLOCK_RANGE);
            }
          }
          if (kt + 1 < n_kt) table_ids(kt + 1, next_id);
          wait_or_abort(&k_empty[st], ph, abort_flag, a.err, a.wait_limit);
          if (*abort_flag) break;  // a wait may have been skipped: no more arrivals
          k_issued <<= 1;
          ++nk;
          if (!(a.test_withhold && cta == 0 && kt == 0)) {  // (testing hook)
            mbar_arrive_expect_tx(&k_full[st], kTileBytes);
  #pragma unroll
            for (int r = 0; r < 8; ++r)
  #pragma unroll
              for (int kh = 0; kh < 2; ++kh)
                tma_load_4d(smem + OFF_K + st * kTileBytes + kh * kHalfBytes + r * 16 * 128, &tmK,
                            kh * 64, h, row[r], bid[r], &k_full[st]);
            k_issued |= 1u;
          }
          wait_or_abort(&v_empty[st], ph, abort_flag, a.err, a.wait_limit);
          if (*abort_flag) break;
          v_issued <<= 1;
          ++nv;
          mbar_arrive_expect_tx(&v_full[st], kTileBytes);
  #pragma unroll
          for (int r = 0; r < 8; ++r)
  #pragma unroll
            for (int kh = 0; kh < 2; ++kh)
              tma_load_4d(smem + OFF_V + st * kTileBytes + kh * kHalfBytes + r * 16 * 128, &tmV,
                          kh * 64, h, row[r], bid[r], &v_full[st]);
          v_issued |= 1u;
        }
        {  // no copy may still be landing in shared memory at the exit (a no-op unless the
           // CTA aborted: the MMA issuer has waited for every copy otherwise)
          for (int i = 0; i < 2; ++i) {
            const int ck = nk - 1 - i, cv = nv - 1 - i;
            if (ck >= 0 && (k_issued & (1u << i)))
              (void)mbar_wait(&k_full[ck & 1], (ck >> 1) & 1, a.err, a.wait_limit);
            if (cv >= 0 && (v_issued & (1u << i)))
              (void)mbar_wait(&v_full[cv & 1], (cv >> 1) & 1, a.err, a.wait_limit);
          }
        }
      }
    } else if (warp == 1) {
      // ======================== MMA issuer ========================
      if (lane == 0) {
        constexpr bool BF = sizeof(T) == 2 && !std::is_same<T, __half>::value;
        const uint32_t id_qk = idesc_f16(BF, false);
        const uint32_t id_pv = idesc_f16(BF, true);
        const uint32_t sQ = smem_u32(smem + OFF_Q);
        const uint32_t sK = smem_u32(smem + OFF_K);
        const uint32_t sV = smem_u32(smem + OFF_V);
        auto issue_s = [&](int mt, int kt) {
          const int st = kt & 1;
  #pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            const uint64_t da = sw128_desc(sQ + mt * kTileBytes + off, 16, 1024);
            const uint64_t db = sw128_desc(sK + st * kTileBytes + off, 16, 1024);
            mma_ss(tmem + mt * 128, da, db, id_qk, kk > 0);
          }
          mma_commit(&s_full[mt]);
        };
        auto issue_pv = [&](int mt, int kt, bool acc) {
          const int st = kt & 1;
  #pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            const uint64_t db = sw128_desc(sV + st * kTileBytes + kk * 2048, kHalfBytes, 1024);
            mma_ts(tmem + 256 + mt * 128, tmem + mt * 128 + kk * 8, db, id_pv, (acc || kk > 0));
          }
        };
        wait_or_abort(q_full, 0, abort_flag, a.err, a.wait_limit);
        tc_fence_after();
        if (n_kt > 0) {
          wait_or_abort(&k_full[0], 0, abort_flag, a.err, a.wait_limit);
          tc_fence_after();
          issue_s(0, 0);
          issue_s(1, 0);
          mma_commit(&k_empty[0]);
        }
        for (int kt = 0; kt < n_kt; ++kt) {
          const int st = kt & 1;
          const bool more = kt + 1 < n_kt;
          wait_or_abort(&v_full[st], (kt >> 1) & 1, abort_flag, a.err, a.wait_limit);
          if (more) wait_or_abort(&k_full[(kt + 1) & 1], ((kt + 1) >> 1) & 1, abort_flag, a.err, a.wait_limit);
          for (int mt = 0; mt < 2; ++mt) {
            wait_or_abort(&p_full[mt], kt & 1, abort_flag, a.err, a.wait_limit);
            tc_fence_after();
            issue_pv(mt, kt, kt > 0);
            if (more) issue_s(mt, kt + 1);
          }
          if (more) mma_commit(&k_empty[(kt + 1) & 1]);
          mma_commit(&v_empty[st]);
        }
        mma_commit(&o_full[0]);
        mma_commit(&o_full[1]);
        if (*abort_flag) {
          // the softmax warps may not have waited for the last products: the MMAs issued so
          // far must be complete before the TMEM they write is freed
          mma_commit(drain);
          (void)mbar_wait(drain, 0, a.err, a.wait_limit);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
  }
}

}  // namespace prefill
}  // namespace pa
