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
// Design on B200 (the page's own kernel tricks — block-table entries in shared
// memory, coalesced in-block reads, prefetch of the next block — kept where they
// still pay):
//  * Work item = (sequence, kv-head, partition of `P` tokens).  A persistent grid of
//    one CTA per SM walks the items round-robin, so the KV stream never drains
//    between items.
//  * One producer warp stages each item's block-table entries in shared memory
//    (one coalesced load per 32 tiles) and issues one 4-D TMA copy per 16-token tile
//    of K and of V (a tile = 16 rows x 256 B of one kv-head inside one physical
//    block) into an NSTAGE-deep ring of shared-memory stages guarded by mbarriers.
//  * Consumer warps share each K/V tile across the G q-heads of the kv-head (GQA).
//    For q.k, 8 lanes split one token's 128 dims (16 each, two 16-byte shared-memory
//    reads); a warp-shuffle halving exchange sums up to 4 heads at once, leaving every
//    lane with one (token, head) logit.  Each warp keeps its own online softmax
//    (running max m, sum l, fp32 accumulator) over its slice of every stage;
//    p.V uses lanes over head_dim (4 dims per lane).
//  * At the end of an item the warps' states are merged in shared memory.  A
//    sequence that fits one partition writes `out` directly; longer ones write the
//    normalised partial (o, m, l) to the caller's workspace and a log-sum-exp pass
//    (lse_reduce_kernel) merges the partitions.
//  * Logits are kept in the log2 domain (q pre-scaled by scale*log2 e) so the
//    exponentials are single ex2 instructions.
// Every wait is bounded; bad table entries or lengths never fault (they are
// skipped and flagged).
#include <algorithm>

#include "pa_device.cuh"
#include "pa_host.h"

namespace pa {

struct DecodeArgs {
  void* out;
  const void* q;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  float* part_o;   // [B, Hq, max_parts, 128]
  float* part_ml;  // [B, Hq, max_parts, 2]   (running max in log2 units, sum)
  int* err;
  int num_seqs, num_q_heads, num_kv_heads, max_blocks, log2_bs, num_blocks;
  int part_size, max_parts, seq_cap, flag_cta;
  float qscale;  // scale * log2(e)
};

constexpr int kD = 128;
constexpr int kTileTok = 16;
constexpr int kTileBytes = kTileTok * kD * 2;  // one TMA box: 16 rows x 256 B

template <int G_, int NCW_>
struct DecodeCfg {
  static constexpr int G = G_;
  static constexpr int NCW = NCW_;                     // consumer warps
  static constexpr int GW = G < 4 ? G : 4;             // heads per warp
  static constexpr int HG = G / GW;                    // head groups
  static constexpr int TGS = NCW / HG;                 // token groups
  static constexpr int TPW = 8;                        // tokens per warp per stage
  static constexpr int TOK_STAGE = TPW * TGS;
  static constexpr int TPS = TOK_STAGE / kTileTok;     // tiles per stage
  static constexpr int NPASS = TPW / 4;
  static constexpr int STAGE_BYTES = TPS * kTileBytes;  // K part; V part follows
  static constexpr int NSTAGE = (128 * 1024) / (2 * STAGE_BYTES);
  static constexpr int THREADS = (NCW + 1) * 32;
  static constexpr int DUPMASK = GW == 4 ? 1 : (GW == 2 ? 3 : 7);
  // shared-memory carve-up (bytes)
  static constexpr int OFF_BAR = NSTAGE * 2 * STAGE_BYTES;
  static constexpr int OFF_TBL = OFF_BAR + 2 * NSTAGE * 8;
  static constexpr int OFF_MISC = OFF_TBL + 32 * 4;  // abort flag (+pad)
  static constexpr int OFF_P = OFF_MISC + 16;
  static constexpr int OFF_A = OFF_P + NCW * TPW * GW * 4;
  static constexpr int OFF_RACC = OFF_A + NCW * GW * 4;
  static constexpr int OFF_RM = OFF_RACC + NCW * GW * kD * 4;
  static constexpr int OFF_RL = OFF_RM + NCW * GW * 4;
  static constexpr int OFF_SEQ = OFF_RL + NCW * GW * 4;  // int seq_start[B+1], int len[B]
  static_assert(TOK_STAGE % kTileTok == 0, "stage must hold whole tiles");
  static_assert(32 % TPS == 0, "table chunk must hold whole stages");
  static_assert(NSTAGE >= 2, "need a pipeline");
  static_assert(OFF_RACC % 16 == 0, "float4 alignment");
};

__device__ __forceinline__ int cdiv(int a, int b) { return (a + b - 1) / b; }

__device__ __forceinline__ int clamp_len(int L, int cap) { return L < 0 ? 0 : (L > cap ? cap : L); }

// Bounded wait that turns into a no-op once any warp of the CTA gave up.
__device__ __forceinline__ void wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                              int* err) {
  if (*abort_flag) return;
  if (!mbar_wait(bar, parity, err)) *abort_flag = 1;
}

// Sum a warp's per-lane partial dot products over each 8-lane token group for
// GW heads at once.  Returns the full sum of head hh(lane):
//   GW=4: hh = 2*bit2 + bit1;  GW=2: hh = bit2;  GW=1: hh = 0.
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

// Unpack 8 packed 16-bit values into fp32.
template <typename T>
__device__ __forceinline__ void unpack8(const uint4& w, float* f) {
  float2 a = Elem<T>::unpack2(w.x), b = Elem<T>::unpack2(w.y);
  float2 c = Elem<T>::unpack2(w.z), d = Elem<T>::unpack2(w.w);
  f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
  f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

// Item index -> (sequence, partition, kv-head).  Items are ordered
// (sequence, partition, kv-head); seq_start holds each sequence's first
// (sequence, partition) pair.
__device__ __forceinline__ void decode_item(int item, int Hkv, const int* seq_start, int B, int& s,
                                            int& p, int& h) {
  const int sp = item / Hkv;
  h = item - sp * Hkv;
  int lo = 0, hi = B - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (seq_start[mid] <= sp) lo = mid; else hi = mid - 1;
  }
  s = lo;
  p = sp - seq_start[lo];
}

template <typename T, int G, int NCW>
__global__ void __launch_bounds__(DecodeCfg<G, NCW>::THREADS, 1)
    paged_decode_kernel(const __grid_constant__ CUtensorMap tmK,
                        const __grid_constant__ CUtensorMap tmV, const DecodeArgs a) {
  using C = DecodeCfg<G, NCW>;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + C::NSTAGE;
  int* tbl = reinterpret_cast<int*>(smem + C::OFF_TBL);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  float* pbuf = reinterpret_cast<float*>(smem + C::OFF_P);
  float* abuf = reinterpret_cast<float*>(smem + C::OFF_A);
  float* racc = reinterpret_cast<float*>(smem + C::OFF_RACC);
  float* rm = reinterpret_cast<float*>(smem + C::OFF_RM);
  float* rl = reinterpret_cast<float*>(smem + C::OFF_RL);
  int* seq_start = reinterpret_cast<int*>(smem + C::OFF_SEQ);
  int* seq_len = seq_start + a.num_seqs + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int B = a.num_seqs;
  const int Hkv = a.num_kv_heads;
  const int P = a.part_size;

  // ---- per-sequence partition counts and their prefix sum (warp 0)
  if (warp == 0) {
    const int per = (B + 31) / 32;
    const int lo = min(B, lane * per), hi = min(B, lo + per);
    int sum = 0;
    for (int s = lo; s < hi; ++s) {
      const int raw = a.seq_lens[s];
      const int L = clamp_len(raw, a.seq_cap);
      if (raw != L && blockIdx.x == a.flag_cta) flag_error(a.err, PA_DEVERR_SEQ_TOO_LONG);
      seq_len[s] = L;
      sum += max(1, cdiv(L, P));
    }
    int incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int run = incl - sum;
    for (int s = lo; s < hi; ++s) {
      seq_start[s] = run;
      run += max(1, cdiv(seq_len[s], P));
    }
    if (lane == 31) seq_start[B] = incl;
  }
  if (threadIdx.x == 32) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::NCW);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  const int total = seq_start[B] * Hkv;

  if (warp == C::NCW) {
    // ================= producer warp: block-table staging + TMA =================
    if (lane == 0) {
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
    }
    int st = 0;
    uint32_t ph = 0;
    const int bs_mask = (1 << a.log2_bs) - 1;
    for (int item = blockIdx.x; item < total; item += gridDim.x) {
      int s, p, h;
      decode_item(item, Hkv, seq_start, B, s, p, h);
      const int tok0 = p * P;
      const int tok1 = min(seq_len[s], tok0 + P);
      const int ntile = cdiv(max(tok1 - tok0, 0), kTileTok);
      const int32_t* trow = a.block_tables + (long long)s * a.max_blocks;
      for (int c = 0; c < ntile; c += 32) {
        int id = -1;
        if (c + lane < ntile) {
          const int pos = tok0 + (c + lane) * kTileTok;
          id = __ldg(trow + (pos >> a.log2_bs));
          if ((unsigned)id >= (unsigned)a.num_blocks) {
            flag_error(a.err, PA_DEVERR_BLOCK_RANGE);
            id = -1;
          }
        }
        __syncwarp();
        tbl[lane] = id;
        __syncwarp();
        if (lane == 0) {
          const int nchunk = min(32, ntile - c);
          for (int j = 0; j < nchunk; j += C::TPS) {
            wait_or_abort(&empty[st], ph ^ 1, abort_flag, a.err);
            const int nv = min(C::TPS, nchunk - j);
            uint32_t bytes = 0;
            if (!*abort_flag)
              for (int t = 0; t < nv; ++t) bytes += tbl[j + t] >= 0 ? 2 * kTileBytes : 0;
            mbar_arrive_expect_tx(&full[st], bytes);
            if (bytes) {
              uint8_t* kd = smem + st * 2 * C::STAGE_BYTES;
              for (int t = 0; t < nv; ++t) {
                const int bid = tbl[j + t];
                if (bid < 0) continue;
                const int row = (tok0 + (c + j + t) * kTileTok) & bs_mask;
                tma_load_4d(kd + t * kTileBytes, &tmK, 0, h, row, bid, &full[st]);
                tma_load_4d(kd + C::STAGE_BYTES + t * kTileBytes, &tmV, 0, h, row, bid, &full[st]);
              }
            }
            if (++st == C::NSTAGE) { st = 0; ph ^= 1; }
          }
        }
      }
    }
    return;
  }

  // ======================= consumer warps =======================
  constexpr int GW = C::GW;
  const int hg = warp % C::HG;
  const int tg = warp / C::HG;
  const int sub = lane & 7;
  const int tp = lane >> 3;
  const int hh = head_of_lane<GW>(lane);
  const bool writer = (lane & C::DUPMASK) == 0;
  const int wt0 = tg * C::TPW;
  float* pw = pbuf + warp * C::TPW * GW;
  int st = 0;
  uint32_t ph = 0;

  for (int item = blockIdx.x; item < total; item += gridDim.x) {
    int s, p, h;
    decode_item(item, Hkv, seq_start, B, s, p, h);
    const int tok0 = p * P;
    const int tok1 = min(seq_len[s], tok0 + P);
    const int ntile = cdiv(max(tok1 - tok0, 0), kTileTok);
    const int qh0 = h * G + hg * GW;

    // q for this warp's GW heads: dims [8*sub, 8*sub+8) and [64+8*sub, 64+8*sub+8)
    float qf[GW][16];
    {
      const T* qb = static_cast<const T*>(a.q) + ((long long)s * a.num_q_heads + qh0) * kD;
#pragma unroll
      for (int j = 0; j < GW; ++j) {
        const uint4 w0 = __ldg(reinterpret_cast<const uint4*>(qb + j * kD + 8 * sub));
        const uint4 w1 = __ldg(reinterpret_cast<const uint4*>(qb + j * kD + 64 + 8 * sub));
        unpack8<T>(w0, qf[j]);
        unpack8<T>(w1, qf[j] + 8);
#pragma unroll
        for (int i = 0; i < 16; ++i) qf[j][i] *= a.qscale;
      }
    }
    float m = -INFINITY, l = 0.f;
    float acc[GW][4];
#pragma unroll
    for (int j = 0; j < GW; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[j][i] = 0.f;

    for (int j0 = 0; j0 < ntile; j0 += C::TPS) {
      wait_or_abort(&full[st], ph, abort_flag, a.err);
      const int valid = min(C::TOK_STAGE, tok1 - (tok0 + j0 * kTileTok));
      const int nv = min(max(valid - wt0, 0), C::TPW);
      if (nv > 0) {
        const uint8_t* Ks = smem + st * 2 * C::STAGE_BYTES;
        const uint8_t* Vs = Ks + C::STAGE_BYTES;
        float x[C::NPASS];
#pragma unroll
        for (int ps = 0; ps < C::NPASS; ++ps) {
          const int r = wt0 + ps * 4 + tp;
          const uint4 w0 = *reinterpret_cast<const uint4*>(Ks + r * 256 + sub * 16);
          const uint4 w1 = *reinterpret_cast<const uint4*>(Ks + r * 256 + 128 + sub * 16);
          float kf[16];
          unpack8<T>(w0, kf);
          unpack8<T>(w1, kf + 8);
          float d[GW];
#pragma unroll
          for (int jj = 0; jj < GW; ++jj) {
            float e0 = 0.f, e1 = 0.f;
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
              e0 = fmaf(qf[jj][i], kf[i], e0);
              e1 = fmaf(qf[jj][i + 1], kf[i + 1], e1);
            }
            d[jj] = e0 + e1;
          }
          const float xv = reduce_heads<GW>(d, lane);
          x[ps] = (ps * 4 + tp < nv) ? xv : -INFINITY;
        }
        // online softmax over the warp's tokens of this stage, per head hh
        float mx = x[0];
#pragma unroll
        for (int ps = 1; ps < C::NPASS; ++ps) mx = fmaxf(mx, x[ps]);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m, mx);
        const float alpha = fast_exp2(m - m_new);  // m = -inf -> 0
        m = m_new;
        float psum = 0.f;
#pragma unroll
        for (int ps = 0; ps < C::NPASS; ++ps) {
          const float pv = fast_exp2(x[ps] - m_new);  // masked -> 0
          psum += pv;
          if (writer) pw[(ps * 4 + tp) * GW + hh] = pv;
        }
        l = l * alpha + psum;
        if (writer && tp == 0) abuf[warp * GW + hh] = alpha;
        __syncwarp();
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
          for (int jj = 0; jj < GW; ++jj) {
            const float al = abuf[warp * GW + jj];
#pragma unroll
            for (int i = 0; i < 4; ++i) acc[jj][i] *= al;
          }
        }
        for (int t = 0; t < nv; ++t) {
          const uint2 vw = *reinterpret_cast<const uint2*>(Vs + (wt0 + t) * 256 + lane * 8);
          const float2 v01 = Elem<T>::unpack2(vw.x), v23 = Elem<T>::unpack2(vw.y);
          float pj[GW];
#pragma unroll
          for (int jj = 0; jj < GW; ++jj) pj[jj] = pw[t * GW + jj];
#pragma unroll
          for (int jj = 0; jj < GW; ++jj) {
            acc[jj][0] = fmaf(pj[jj], v01.x, acc[jj][0]);
            acc[jj][1] = fmaf(pj[jj], v01.y, acc[jj][1]);
            acc[jj][2] = fmaf(pj[jj], v23.x, acc[jj][2]);
            acc[jj][3] = fmaf(pj[jj], v23.y, acc[jj][3]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      if (++st == C::NSTAGE) { st = 0; ph ^= 1; }
    }

    // ---- merge the warps' (m, l, acc) and write
    l += __shfl_xor_sync(0xffffffffu, l, 8);
    l += __shfl_xor_sync(0xffffffffu, l, 16);
#pragma unroll
    for (int jj = 0; jj < GW; ++jj)
      *reinterpret_cast<float4*>(racc + (warp * GW + jj) * kD + lane * 4) =
          make_float4(acc[jj][0], acc[jj][1], acc[jj][2], acc[jj][3]);
    if (writer && tp == 0) {
      rm[warp * GW + hh] = m;
      rl[warp * GW + hh] = l;
    }
    named_bar_sync(1, C::NCW * 32);
    const int nparts = seq_start[s + 1] - seq_start[s];
    for (int o = threadIdx.x; o < G * 32; o += C::NCW * 32) {
      const int r = o >> 5;   // head within the kv group
      const int c4 = o & 31;  // 4-dim chunk
      const int g2 = r / GW, jj = r % GW;
      float M = -INFINITY;
#pragma unroll
      for (int t2 = 0; t2 < C::TGS; ++t2) M = fmaxf(M, rm[(t2 * C::HG + g2) * GW + jj]);
      float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
      float den = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int t2 = 0; t2 < C::TGS; ++t2) {
          const int w2 = t2 * C::HG + g2;
          const float mw = rm[w2 * GW + jj];
          const float f = mw == -INFINITY ? 0.f : fast_exp2(mw - M);
          den += f * rl[w2 * GW + jj];
          const float4 v = *reinterpret_cast<const float4*>(racc + (w2 * GW + jj) * kD + c4 * 4);
          num.x += f * v.x; num.y += f * v.y; num.z += f * v.z; num.w += f * v.w;
        }
      }
      const float inv = den > 0.f ? 1.f / den : 0.f;
      const int qh = h * G + r;
      if (nparts == 1) {
        const uint32_t lo = Elem<T>::pack2(num.x * inv, num.y * inv);
        const uint32_t hi = Elem<T>::pack2(num.z * inv, num.w * inv);
        T* ob = static_cast<T*>(a.out) + ((long long)s * a.num_q_heads + qh) * kD + c4 * 4;
        *reinterpret_cast<uint2*>(ob) = make_uint2(lo, hi);
      } else {
        const long long row = ((long long)s * a.num_q_heads + qh) * a.max_parts + p;
        *reinterpret_cast<float4*>(a.part_o + row * kD + c4 * 4) =
            make_float4(num.x * inv, num.y * inv, num.z * inv, num.w * inv);
        if (c4 == 0) *reinterpret_cast<float2*>(a.part_ml + row * 2) = make_float2(M, den);
      }
    }
    named_bar_sync(1, C::NCW * 32);
  }
}

// Log-sum-exp merge of the split-K partials: one warp per (sequence, q-head), lanes
// over head_dim.  o = sum_p w_p o_p / sum_p w_p with w_p = l_p * 2^(m_p - max m).
template <typename T>
__global__ void __launch_bounds__(256) lse_reduce_kernel(const DecodeArgs a) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= a.num_seqs * a.num_q_heads) return;
  const int s = gw / a.num_q_heads;
  const int L = clamp_len(a.seq_lens[s], a.seq_cap);
  const int n = max(1, cdiv(L, a.part_size));
  if (n <= 1) return;  // written by the decode kernel
  const float2* ml = reinterpret_cast<const float2*>(a.part_ml) + (long long)gw * a.max_parts;
  float M = -INFINITY;
  for (int i = lane; i < n; i += 32) M = fmaxf(M, ml[i].x);
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float den = 0.f;
  float4 num = make_float4(0.f, 0.f, 0.f, 0.f);
  const float* po = a.part_o + (long long)gw * a.max_parts * kD + lane * 4;
  for (int i = 0; i < n; ++i) {
    const float2 v = ml[i];
    const float f = v.x == -INFINITY ? 0.f : fast_exp2(v.x - M) * v.y;
    den += f;
    const float4 o = *reinterpret_cast<const float4*>(po + (long long)i * kD);
    num.x += f * o.x; num.y += f * o.y; num.z += f * o.z; num.w += f * o.w;
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  T* ob = static_cast<T*>(a.out) + (long long)gw * kD + lane * 4;
  *reinterpret_cast<uint2*>(ob) =
      make_uint2(Elem<T>::pack2(num.x * inv, num.y * inv), Elem<T>::pack2(num.z * inv, num.w * inv));
}

constexpr int kDefaultPartition = 512;
constexpr int kConsumerWarps = 8;
constexpr int kMaxSeqs = 8192;

inline int choose_partition(int partition_size) {
  return partition_size > 0 ? partition_size : kDefaultPartition;
}

inline int num_parts_host(int max_seq_len, int P) {
  return std::max(1, (max_seq_len + P - 1) / P);
}

template <typename T, int G>
pa_status launch_decode(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeArgs& a,
                        cudaStream_t stream) {
  using C = DecodeCfg<G, kConsumerWarps>;
  const size_t smem = C::OFF_SEQ + (size_t)(2 * a.num_seqs + 1) * 4;
  if (smem > 227 * 1024) return PA_ERR_UNSUPPORTED;
  auto kern = paged_decode_kernel<T, G, kConsumerWarps>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return PA_ERR_CUDA;
  const long long items_max = (long long)a.num_seqs * a.num_kv_heads * a.max_parts;
  const int sms = num_sms();
  if (sms <= 0) return PA_ERR_CUDA;
  const int grid = (int)std::min<long long>(items_max, sms);
  kern<<<grid, C::THREADS, smem, stream>>>(tmK, tmV, a);
  if (check_launch() != PA_OK) return PA_ERR_CUDA;
  int launches = 1;
  if (a.max_parts > 1) {
    const int warps = a.num_seqs * a.num_q_heads;
    lse_reduce_kernel<T><<<(warps + 7) / 8, 256, 0, stream>>>(a);
    if (check_launch() != PA_OK) return PA_ERR_CUDA;
    ++launches;
  }
  set_launch_count(launches);
  return PA_OK;
}

template <typename T>
pa_status dispatch_group(int G, const CUtensorMap& tmK, const CUtensorMap& tmV,
                         const DecodeArgs& a, cudaStream_t stream) {
  switch (G) {
    case 1: return launch_decode<T, 1>(tmK, tmV, a, stream);
    case 2: return launch_decode<T, 2>(tmK, tmV, a, stream);
    case 4: return launch_decode<T, 4>(tmK, tmV, a, stream);
    case 8: return launch_decode<T, 8>(tmK, tmV, a, stream);
    default: return PA_ERR_UNSUPPORTED;
  }
}

}  // namespace pa

extern "C" size_t pa_decode_workspace_size(int num_seqs, int num_q_heads, int head_dim,
                                           int max_seq_len, int partition_size) {
  if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_seq_len < 0) return 0;
  const int P = pa::choose_partition(partition_size);
  const int parts = pa::num_parts_host(max_seq_len, P);
  if (parts <= 1) return 0;
  return (size_t)num_seqs * num_q_heads * parts * (head_dim + 2) * sizeof(float);
}

extern "C" pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                               const int32_t* block_tables, int max_blocks_per_seq,
                               const int32_t* seq_lens, int num_seqs, int num_q_heads,
                               int num_kv_heads, int head_dim, float scale, int block_size,
                               int num_blocks, int max_seq_len, int partition_size,
                               void* workspace, size_t workspace_bytes, pa_dtype dtype,
                               void* stream) {
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
  if (num_seqs == 0) return PA_OK;
  if (num_seqs > pa::kMaxSeqs) return PA_ERR_UNSUPPORTED;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens) return PA_ERR_INVALID_ARG;
  if (((uintptr_t)out | (uintptr_t)q | (uintptr_t)k_cache | (uintptr_t)v_cache) & 15)
    return PA_ERR_INVALID_ARG;
  const int P = pa::choose_partition(partition_size);
  const int parts = pa::num_parts_host(max_seq_len, P);
  const size_t need =
      pa_decode_workspace_size(num_seqs, num_q_heads, head_dim, max_seq_len, partition_size);
  if (need && (!workspace || workspace_bytes < need)) return PA_ERR_WORKSPACE_TOO_SMALL;
  if (need && ((uintptr_t)workspace & 15)) return PA_ERR_INVALID_ARG;
  int* err = pa::device_error_flag();
  if (!err) return PA_ERR_CUDA;

  CUtensorMap tmK, tmV;
  if (!pa::encode_cache_tmap(&tmK, k_cache, num_blocks, block_size, num_kv_heads, head_dim, 16) ||
      !pa::encode_cache_tmap(&tmV, v_cache, num_blocks, block_size, num_kv_heads, head_dim, 16))
    return PA_ERR_CUDA;

  pa::DecodeArgs a;
  a.out = out;
  a.q = q;
  a.block_tables = block_tables;
  a.seq_lens = seq_lens;
  a.part_o = need ? static_cast<float*>(workspace) : nullptr;
  a.part_ml = need ? static_cast<float*>(workspace) + (size_t)num_seqs * num_q_heads * parts * head_dim
                   : nullptr;
  a.err = err;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.max_blocks = max_blocks_per_seq;
  a.log2_bs = block_size == 16 ? 4 : 5;
  a.num_blocks = num_blocks;
  a.part_size = P;
  a.max_parts = parts;
  const long long cap_tbl = (long long)max_blocks_per_seq * block_size;
  const long long cap_grid = (long long)parts * P;
  a.seq_cap = (int)std::min<long long>(std::min<long long>(cap_tbl, cap_grid), max_seq_len);
  a.flag_cta = 0;
  a.qscale = scale * 1.4426950408889634f;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dtype == PA_F16 ? pa::dispatch_group<__half>(G, tmK, tmV, a, st)
                         : pa::dispatch_group<__nv_bfloat16>(G, tmK, tmV, a, st);
}
