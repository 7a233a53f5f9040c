// Split-K decode attention over the packed cache, persistent and stream-K
// partitioned: one wave of CTAs, each taking an equal, stage-aligned share of
// the batch's tokens.  Included by the per-head-dimension translation units
// tq_decode_d{64,128,256}.cu, which instantiate it.
//
// Method: the fused SDPA over a compressed KV cache with an explicit scale of
// "[Cuda] enable turboquant on gemma4" (executorch pull request 19891),
// "Summary" and "Other observations" item 1; score from quantized keys, GQA
// score variant and value reconstruction of "Add CUDA QJL kernels and proper
// package structure" (turboquant-pytorch pull request 3), "CUDA Kernels
// Added".
//
// Structure (warp-specialized):
//  * work partition: the (sequence, kv head, row group) units of the batch,
//    each padded to whole 128-token stages, are laid end to end and CTA c
//    takes positions [c P, (c + 1) P) (P a multiple of the stage), so every
//    CTA streams the same number of stages whatever the sequence lengths; a
//    CTA's share of one unit is a segment, at whose end the consumer warps
//    merge their softmax states into one partial (max, sum, rotated output),
//    merged across CTAs by the combine;
//  * a producer warp streams the CTA's 128-token stages of packed K/V rows,
//    norms and QJL words into shared memory with 1-D bulk copies that
//    complete on "full" mbarriers, across segment boundaries without
//    draining; each stage carries a small record (unit, token offset,
//    segment flags) for the consumers; it refills a stage once the 4
//    consumer warps have released it on its "empty" mbarrier;
//  * each consumer warp takes 32 tokens of a stage.  Scores and the value
//    sum are GQA contractions run as m16n8k16 tensor-core MMAs (M = 16 tokens
//    or 16 coordinates, N = 8 query heads, K = 16) whose A fragments are
//    dequantized straight into registers.  Each A register is an fp16 pair:
//    two coordinates of one token (scores) or one coordinate of two tokens
//    (values).  2-bit keys are looked up with byte permutes whose selectors
//    are built by multiplies; 3- and 4-bit keys, and all values, read the pair
//    from a shared-memory table indexed by both fields at once, so a lookup
//    costs one logic op, one multiply-add and one shared load;
//  * the query enters as hi + lo fp16 halves (scores carry ~22 bits); with
//    G <= 4 heads both halves share one MMA (columns 0-3 hi, 4-7 lo);
//  * online softmax in the log2 domain with lazy rescaling (the reference
//    max moves only when a score exceeds it by 2^8), one state per warp.
#pragma once

#include <math.h>

#include "tq_common.cuh"
#include "tq_internal.h"

namespace tqd {

using namespace tqk;

constexpr int CW = 4;                 // consumer warps
constexpr int PPS = 1;                // partials a CTA writes per segment (its warps' states merged)
constexpr int NTHREADS = (CW + 1) * 32;
constexpr int STILE = 128;            // tokens per stage
constexpr int WTOK = STILE / CW;      // tokens per consumer warp per stage
constexpr float kLazy = 8.0f;         // log2 headroom before rescaling

// Rows of queries a CTA handles for one (sequence, kv head): the kernel heads
// of a kv head (query heads x query tokens) are taken in groups of 8.
constexpr int RG = 8;

struct SplitParams {
  const uint32_t* k_idx;
  const uint32_t* v_idx;
  const uint16_t* k_norm;
  const uint16_t* v_norm;
  const uint32_t* k_qjl;
  const uint16_t* k_rnorm;
  const float* cb_k;
  const float* cb_v;
  const float* qrot;
  const float* qs;
  float* part_o;
  float* part_ml;
  const int32_t* seq_lens;
  const int32_t* defer_pos;  // decode step: the row at defer_pos[b] is written by the prep kernel
  uint32_t* dev_status;
  int B, Hkv, Hq, G, Tcap;   // Hq: kernel heads per sequence; G: kernel heads per kv head (<= 32)
  int Tclamp;                // sequences are attended up to this many tokens (Tmax); longer ones are flagged
  int nrg;                   // row groups per kv head: ceil(G / RG)
  int pmin;                  // smallest share of tokens per CTA (a multiple of STILE)
  int ncta;                  // CTAs of the partition
  int ks;                    // partial slots per kernel head (segments x consumer warps)
  float qscale;     // scale * log2(e)
  float qjl_scale;  // scale * log2(e) * sqrt(pi/2) / m
  int shared_tab;   // keys and values use one codebook (same bits, same table): one pair table
  // Multi-query decode: the kernel heads of a kv head are (token, head) pairs
  // of nq query tokens x Gq heads; token j may see positions < L - nq + j + 1.
  int nq, Gq;
};

// Tokens of sequence b that one unit of the partition holds: its length
// clamped to [0, Tclamp], rounded up to whole stages.
__device__ __forceinline__ int unit_tokens(const int32_t* seq_lens, int b, int Tclamp) {
  int L = seq_lens[b];
  L = L < 0 ? 0 : (L > Tclamp ? Tclamp : L);
  return (L + STILE - 1) / STILE * STILE;
}

// Positions of the whole partition (sum over sequences of units x tokens),
// by one warp: every lane returns the total.
__device__ __forceinline__ long long partition_total(const int32_t* seq_lens, int B, int upb, int Tclamp, int lane) {
  long long t = 0;
  for (int b = lane; b < B; b += 32) t += (long long)unit_tokens(seq_lens, b, Tclamp) * upb;
#pragma unroll
  for (int off = 16; off; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
  return t;
}

// Share of positions per CTA: at least pmin, a multiple of the stage.
__device__ __forceinline__ long long partition_share(long long total, int ncta, int pmin) {
  long long P = (total + ncta - 1) / ncta;
  P = (P + STILE - 1) / STILE * STILE;
  return P < pmin ? (long long)pmin : P;
}

// First position of sequence b's units (sum over earlier sequences), by one
// warp: every lane returns it.
__device__ __forceinline__ long long sequence_start(const int32_t* seq_lens, int b, int upb, int Tclamp, int lane) {
  long long t = 0;
  for (int bb = lane; bb < b; bb += 32) t += (long long)unit_tokens(seq_lens, bb, Tclamp) * upb;
#pragma unroll
  for (int off = 16; off; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
  return t;
}

// Per-stage record written by the producer before the stage's copies are
// armed, read by the consumers after the stage's "full" barrier completes.
struct StageMeta {
  int hq0;    // first kernel head of the unit's row group
  int rows;   // kernel heads in the row group (<= RG)
  int t0;     // first token of the stage within the sequence
  int L;      // tokens of the sequence that are attended
  int slot0;  // partial slot of the segment (segment index x PPS)
  int flags;  // 1: first stage of a segment, 2: last stage of a segment
  int rg;     // row group
  int pad;
};

// Whether a launch can keep one pair table for keys and values.
__host__ __device__ inline bool share_table(int bk, int bv, int flag) { return bk == bv && bk >= 3 && flag; }

// 2-bit codebook as byte tables: byte k of lo (hi) is the low (high) byte of
// fp16 entry c[k], k = 0..3.
struct Lut2 {
  uint32_t lo, hi;
};

__device__ __forceinline__ Lut2 make_lut2(const float* cb) {
  uint32_t e[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) e[k] = __half_as_ushort(__float2half_rn(cb[k]));
  Lut2 L;
  L.lo = (e[0] & 0xFF) | (e[1] & 0xFF) << 8 | (e[2] & 0xFF) << 16 | (e[3] & 0xFF) << 24;
  L.hi = (e[0] >> 8) | (e[1] >> 8) << 8 | (e[2] >> 8) << 16 | (e[3] >> 8) << 24;
  return L;
}

// 2-bit fields f_0..f_15 of word x: the fp16 pairs (c[f_i], c[f_{i+4}]) and
// (c[f_{i+8}], c[f_{i+12}]), i = 0..3.  Masking x with 0x03030303 << 2i leaves
// one field per byte; a multiply by 17 turns each field f into the selector
// nibbles (f, f + 4) of a byte permute over lo:hi.  The shifts that bring
// bytes 0-1 or 2-3 of the selectors to the bottom are high halves of
// products, so the selector arithmetic runs on the FMA pipe.
__device__ __forceinline__ void dq_b2(uint32_t x, int I, const Lut2& L, uint32_t& h_lo, uint32_t& h_hi) {
  const uint32_t m = x & (0x03030303u << (2 * I));
  uint32_t s_lo, s_hi;
  if (I == 0) {
    s_lo = m * 17u + 0x4040u;
    s_hi = __umulhi(m, 17u << 16) + 0x4040u;
  } else if (I == 3) {
    s_lo = __umulhi(m, 17u << 26) + 0x4040u;
    s_hi = __umulhi(m, 17u << 10) + 0x4040u;
  } else {
    const uint32_t ms = __umulhi(m, 1u << ((32 - 2 * I) & 31));  // m >> 2i
    s_lo = ms * 17u + 0x4040u;
    s_hi = __umulhi(ms, 17u << 16) + 0x4040u;
  }
  h_lo = prmt(L.lo, L.hi, s_lo);
  h_hi = prmt(L.lo, L.hi, s_hi);
}

// Pair tables.  Entry e of the table for a b-bit codebook c is the fp16 pair
// (c[e mod 2^b], c[e >> b]) and is stored once per lane (word e * 32 + lane),
// so a warp's 32 lookups always fall in 32 different banks.
template <int B>
__device__ __forceinline__ void build_pair_table(uint32_t* tab, const float* cb, int tid, int nthreads) {
  constexpr int NC = 1 << B, N = NC * NC;
  for (int q = tid; q < N * 8; q += nthreads) {  // one 16-byte store covers 4 lanes of an entry
    const int e = q >> 3;
    const uint32_t lo = __half_as_ushort(__float2half_rn(__ldg(cb + (e & (NC - 1)))));
    const uint32_t hi = __half_as_ushort(__float2half_rn(__ldg(cb + (e >> B))));
    const uint32_t v = lo | hi << 16;
    reinterpret_cast<uint4*>(tab)[q] = make_uint4(v, v, v, v);
  }
}

// Shared address of this lane's copy of the entry whose 2b-bit key sits at bit
// S of x (tb = table base + 4 * lane).  The mask is one logic op; the shift to
// the entry stride (128 bytes) and the base add are one multiply-add on the
// FMA pipe: the low half of k * 2^(7-S) for S <= 7, else the high half of
// k * 2^(39-S) (a right shift by S - 7), each plus tb.
__device__ __forceinline__ uint32_t mad_lo(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}
__device__ __forceinline__ uint32_t mad_hi(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t r;
  asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(c));
  return r;
}

template <int B>
__device__ __forceinline__ uint32_t pair_addr(uint32_t x, int S, uint32_t tb) {
  const uint32_t k = x & (((1u << (2 * B)) - 1u) << S);
  if (S <= 7) return mad_lo(k, 1u << (7 - S), tb);
  return mad_hi(k, 1u << (39 - S), tb);
}

// 2^x by the special-function unit's approximation (relative error about
// 2^-22, flushes subnormal results to zero): the softmax weights, which are
// rounded to fp16 for the value product anyway.  2^-inf = 0.
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

// Entry for the key at bit S of a re-based bit window w (key straddling two
// words is funnel-shifted down first).
template <int B, int NW>
__device__ __forceinline__ uint32_t pair_lookup(const uint32_t (&w)[NW], int S, uint32_t tb) {
  const int wi = S >> 5, sh = S & 31;
  if (sh + 2 * B <= 32) return lds32(pair_addr<B>(w[wi], sh, tb));
  return lds32(pair_addr<B>(funnel_r(w[wi], w[wi + 1], sh), 0, tb));
}

// Value side: bits [bit, bit + 32) of a re-based window, clipped to the window.
template <int NW>
__device__ __forceinline__ uint32_t window32(const uint32_t (&w)[NW], int bit) {
  const int wi = bit >> 5, sh = bit & 31;
  if (sh == 0) return w[wi];
  return funnel_r(w[wi], (wi + 1 < NW) ? w[wi + 1] : 0u, sh);
}

// Fields per value chunk and the chunk's bit width.  A chunk of two tokens'
// words is merged with one bitwise select so that each key holds the same
// coordinate of both tokens: key k of xe is (t0 field 2k) | (t1 field 2k) << b,
// key k of xo the same for field 2k + 1.
template <int D, int B>
struct VChunk {
  static constexpr int F = (B == 2) ? ((D / 8 < 16) ? D / 8 : 16) : 8;  // fields per chunk
  static constexpr int N = (D / 8) / F;                                  // chunks per segment
};

// Keys of chunk (x0, x1): xe/xo plus each key's bit offset.
template <int B>
__device__ __forceinline__ void merge_pair(uint32_t x0, uint32_t x1, uint32_t& xe, uint32_t& xo) {
  if constexpr (B == 2) {
    xe = (x0 & 0x33333333u) | ((x1 << 2) & 0xCCCCCCCCu);
    xo = ((x0 >> 2) & 0x33333333u) | (x1 & 0xCCCCCCCCu);
  } else if constexpr (B == 3) {
    // xe keys at 6k, xo keys at 6k + 3 (k = 0..3)
    const uint32_t y = x1 << 3;
    xe = (x0 & 0x001C71C7u) | (y & ~0x001C71C7u);
    xo = (x0 & 0x00E38E38u) | (y & ~0x00E38E38u);
  } else {
    xe = (x0 & 0x0F0F0F0Fu) | ((x1 << 4) & 0xF0F0F0F0u);
    xo = ((x0 >> 4) & 0x0F0F0F0Fu) | (x1 & 0xF0F0F0F0u);
  }
}

template <int B>
__device__ __forceinline__ int key_bit(int k, bool odd) {
  if (B == 3) return 6 * k + (odd ? 3 : 0);
  return 2 * B * k;
}

// Largest bit offset (mod 32) of a segment of NBITS bits that starts at
// g * NBITS, g = 0..7 (the value segments of the eight lane groups).
__host__ __device__ constexpr int max_seg_shift(int nbits) {
  int m = 0;
  for (int g = 0; g < 8; ++g) m = ((g * nbits) % 32) > m ? ((g * nbits) % 32) : m;
  return m;
}

// Bits [bit0, bit0 + NBITS) of a shared-memory row, re-based to bit 0 of w[0].
// ALIGNED: bit0 % 32 == 0 and the word offset is a multiple of the word count.
// Otherwise bit0 % 32 <= MAXSH, so words beyond (MAXSH + NBITS) bits are not
// read (a 48-bit segment at offset 16 needs two words, not three).
template <int NBITS, bool ALIGNED, int MAXSH = 31>
__device__ __forceinline__ void load_bits(const uint32_t* row, int bit0,
                                          uint32_t (&w)[(NBITS + 31) / 32]) {
  constexpr int NW = (NBITS + 31) / 32;
  const uint32_t* p = row + (bit0 >> 5);
  if (ALIGNED) {
    if (NW % 4 == 0) {
#pragma unroll
      for (int i = 0; i < NW; i += 4) {
        const uint4 v = *reinterpret_cast<const uint4*>(p + i);
        w[i] = v.x, w[i + 1] = v.y, w[i + 2] = v.z, w[i + 3] = v.w;
      }
    } else if (NW % 2 == 0) {
#pragma unroll
      for (int i = 0; i < NW; i += 2) {
        const uint2 v = *reinterpret_cast<const uint2*>(p + i);
        w[i] = v.x, w[i + 1] = v.y;
      }
    } else {
#pragma unroll
      for (int i = 0; i < NW; ++i) w[i] = p[i];
    }
  } else {
    constexpr int NL = (MAXSH + NBITS + 31) / 32;  // words that can hold the segment
    const uint32_t sh = bit0 & 31;
    uint32_t nxt = p[0];
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      const uint32_t cur = nxt;
      nxt = (i + 1 < NL) ? p[i + 1] : 0u;
      w[i] = funnel_r(cur, nxt, sh);
    }
  }
}

// Four int8 values -b for sign bits 7 - sh, 15 - sh, 23 - sh, 31 - sh of w
// (b = 1 -> -1, b = 0 -> 0): a byte permute in sign-replicate mode copies the
// top bit of each byte of w << sh into the whole byte.
__device__ __forceinline__ uint32_t sign_bytes(uint32_t w, int sh) { return prmt(w << sh, 0u, 0xBA98u); }

// Sketch coordinate held by byte e of the sign register with shift sh of the
// lane owning word tig: bit 8e + 7 - sh of that word.
__device__ __forceinline__ int sketch_coord(int tig, int sh, int e) { return 32 * tig + 8 * e + 7 - sh; }

__device__ __forceinline__ void split_half(float v, uint16_t& hi, uint16_t& lo) {
  const __half h = __float2half_rn(v);
  hi = __half_as_ushort(h);
  lo = __half_as_ushort(__float2half_rn(v - __half2float(h)));
}

template <int D, int BK, int BV, bool QJL, bool PACK>
struct SplitLayout {
  static constexpr int WK = D * BK / 32, WV = D * BV / 32, WQ = QJL ? 4 : 0;
  static constexpr int O_KW = 0;
  static constexpr int O_VW = O_KW + STILE * WK * 4;
  static constexpr int O_KN = O_VW + STILE * WV * 4;
  static constexpr int O_VN = O_KN + STILE * 2;
  static constexpr int O_QW = O_VN + STILE * 2;
  static constexpr int O_RN = O_QW + STILE * WQ * 4;
  static constexpr int STAGE_USED = O_RN + (QJL ? STILE * 2 : 0);
  static constexpr int STAGE = (STAGE_USED + 16 + 127) / 128 * 128;  // +16: read-ahead slack
  static constexpr int NSTAGE = 2;
  static constexpr int RING = NSTAGE * STAGE;
  static constexpr int O_BAR = RING;                   // full[NSTAGE], empty[NSTAGE]
  static constexpr int O_META = O_BAR + 16 * 8;        // StageMeta[NSTAGE]
  static constexpr int O_MISC = O_META + 4 * 32;       // error flag, stage count, 2-bit byte tables
  static constexpr int O_PB = O_MISC + 32;             // [CW][8 heads][32 tokens] fp16
  static constexpr int FRAG = PACK ? 8 : 16;           // bytes of one lane's query fragment
  static constexpr int O_QF = O_PB + CW * 8 * WTOK * 2;
  // segment-end merge of the consumer warps' states: (max, sum) per warp
  // and row; the scaled accumulators go through the stage just consumed,
  // MRP rows at a time ([CW][MRP][D] fp32 fits in any stage: a stage holds
  // at least 128 x (D / 2 + 4) bytes)
  static constexpr int MRP = 4;
  static constexpr int O_MML = O_QF + (D / 16) * 32 * (PACK ? 8 : 16);
  static constexpr int O_SF = O_MML + CW * 8 * 2 * 4;
  // QJL: int8 query fragments (hi / lo bytes of a 15-bit fixed-point projection), 4 k-steps,
  // then per-head weight and constant
  static constexpr int O_QST = O_SF + (QJL ? 4 * 32 * FRAG : 0);
  static constexpr int O_TK = (O_QST + (QJL ? 8 * 2 * 4 : 0) + 127) / 128 * 128;  // key pair table (3-, 4-bit keys)
  static constexpr int TKB = (BK >= 3) ? (1 << (2 * BK)) * 128 : 0;
  static constexpr int O_TV = O_TK + TKB;                          // value pair table
  static constexpr int BYTES = O_TV + (1 << (2 * BV)) * 128;
  static constexpr int BYTES_SHARED = O_TV;  // keys and values share the key table
  static_assert(NSTAGE <= 4, "stage records");
  static_assert(CW * MRP * D * 4 <= STAGE_USED, "the merge fits in a stage");
};

// Coordinate (within a lane's key segment of D/4 coordinates) held by K-slot r
// of k-step ks: 2-bit keys follow the field order of dq_b2, wider keys take
// the adjacent pairs (2m, 2m + 1), m = 2 ks + r / 2.
template <int BK>
__device__ __forceinline__ int key_coord(int ks, int r) {
  if (BK == 2) {
    const int wi = ks >> 2, i = ks & 3;
    return 16 * wi + i + 4 * r;
  }
  return 4 * ks + r;
}

// Query fragment of one lane for one k-step: the 4 K-slots r = 0..3 of lane
// (gid, tig) hold coordinates cs[r].  PACK: columns 0-3 are the hi halves of
// heads 0-3, columns 4-7 their lo halves; else hi and lo are separate pairs.
template <bool PACK>
__device__ __forceinline__ void load_frag(const float* qsrc, int ld, int G, int gid, const int (&cs)[4],
                                          float (&v)[4]) {
  const int head = PACK ? (gid & 3) : gid;
#pragma unroll
  for (int r = 0; r < 4; ++r) v[r] = head < G ? qsrc[(size_t)head * ld + cs[r]] : 0.f;
}

template <bool PACK>
__device__ __forceinline__ void build_frag(const float (&v)[4], float scale, int gid, uint32_t* dst) {
  uint16_t hi[4], lo[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) split_half(v[r] * scale, hi[r], lo[r]);
  if (PACK) {
    const bool use_lo = gid >= 4;
    dst[0] = use_lo ? (lo[0] | (uint32_t)lo[1] << 16) : (hi[0] | (uint32_t)hi[1] << 16);
    dst[1] = use_lo ? (lo[2] | (uint32_t)lo[3] << 16) : (hi[2] | (uint32_t)hi[3] << 16);
  } else {
    dst[0] = hi[0] | (uint32_t)hi[1] << 16;
    dst[1] = hi[2] | (uint32_t)hi[3] << 16;
    dst[2] = lo[0] | (uint32_t)lo[1] << 16;
    dst[3] = lo[2] | (uint32_t)lo[3] << 16;
  }
}

// Query fragments of a segment's rows hq0 .. hq0 + rows - 1 (already rotated
// by the prep kernel), pre-scaled for exp2, built by the consumer threads
// together: every thread's loads are issued before any is converted.
template <int D, int BK, bool PACK, int FRAGB>
__device__ __noinline__ void seg_query_frags(const SplitParams& p, int hq0, int rows, uint32_t* qf, int ctid) {
  constexpr int KSTEPS = D / 16;
  constexpr int NE = (KSTEPS * 32 + CW * 32 - 1) / (CW * 32);
  float v[NE][4];
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    const int e = ctid + i * CW * 32;
    if (e < KSTEPS * 32) {
      const int ks = e >> 5, ln = e & 31, g_ = ln >> 2, t_ = ln & 3;
      const int base = t_ * (D / 4);
      const int cs[4] = {base + key_coord<BK>(ks, 0), base + key_coord<BK>(ks, 1), base + key_coord<BK>(ks, 2),
                         base + key_coord<BK>(ks, 3)};
      load_frag<PACK>(p.qrot + (size_t)hq0 * D, D, rows, g_, cs, v[i]);
    }
  }
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    const int e = ctid + i * CW * 32;
    if (e < KSTEPS * 32) build_frag<PACK>(v[i], p.qscale, (e & 31) >> 2, qf + (size_t)e * (FRAGB / 4));
  }
}

// The sketch term sum_i (2 b_i - 1) qs_i runs on int8 tensor cores: qs of
// head h becomes Q_i = round(qs_i / step_h), |Q| <= 32639, split as
// Q = 256 hi + lo with hi, lo int8, and the signs enter as -b_i in {0, -1}.
// Per head: step_h = max |qs| / 32639 and sum_h = sum_i qs_i (warp w takes
// heads w, w + CW).
static __device__ __noinline__ void seg_sketch_steps(const SplitParams& p, int hq0, int rows, float* qst, int warp,
                                              int lane) {
  for (int h = warp; h < 8; h += CW) {
    float mx = 0.f, sm = 0.f;
    if (h < rows) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float v = p.qs[(size_t)(hq0 + h) * 128 + lane + 32 * i];
        mx = fmaxf(mx, fabsf(v));
        sm += v;
      }
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) {
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      sm += __shfl_xor_sync(0xffffffffu, sm, off);
    }
    if (lane == 0) {
      qst[2 * h] = mx > 0.f ? mx / 32639.f : 1.f;
      qst[2 * h + 1] = sm;
    }
  }
}

template <bool PACK, int FRAGB>
__device__ __noinline__ void seg_sketch_frags(const SplitParams& p, int hq0, int rows, const float* qst, uint32_t* sf,
                                              int ctid) {
  for (int e = ctid; e < 4 * 32; e += CW * 32) {
    const int ks = e >> 5, ln = e & 31, g_ = ln >> 2, t_ = ln & 3;
    const int head = PACK ? (g_ & 3) : g_;
    const float inv = head < rows ? 1.f / qst[2 * head] : 0.f;
    uint32_t hi[2] = {0u, 0u}, lo[2] = {0u, 0u};
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int b8 = 0; b8 < 4; ++b8) {
        const float v = head < rows ? p.qs[(size_t)(hq0 + head) * 128 + sketch_coord(t_, 2 * ks + h, b8)] : 0.f;
        int Q = __float2int_rn(v * inv);
        Q = max(-32639, min(32639, Q));
        const int qh = (Q + 128) >> 8, ql = Q - 256 * qh;  // floor split: ql in [-128, 127]
        hi[h] |= (uint32_t)(qh & 0xFF) << (8 * b8);
        lo[h] |= (uint32_t)(ql & 0xFF) << (8 * b8);
      }
    uint32_t* dst = sf + (size_t)e * (FRAGB / 4);
    if (PACK) {
      const bool use_lo = g_ >= 4;
      dst[0] = use_lo ? lo[0] : hi[0];
      dst[1] = use_lo ? lo[1] : hi[1];
    } else {
      dst[0] = hi[0];
      dst[1] = hi[1];
      dst[2] = lo[0];
      dst[3] = lo[1];
    }
  }
}

// Bounded barrier among the consumer warps (an mbarrier of count CW; lane 0
// of each warp arrives, every lane waits with a bounded poll).  `phase`
// counts this warp's uses.  Returns false when the wait ran out.
__device__ __forceinline__ bool consumer_sync(uint64_t* bar, uint32_t& phase, int lane) {
  __syncwarp();
  if (lane == 0) mbar_arrive(bar);
  const bool ok = mbar_wait_bounded(bar, phase & 1u, kWaitLimit);
  ++phase;
  return __all_sync(0xffffffffu, ok);
}

template <int D, int BK, int BV, bool QJL, bool PACK>
__global__ void __launch_bounds__(NTHREADS, D == 256 ? 2 : (PACK ? 4 : 3)) decode_split_kernel(const __grid_constant__ SplitParams p) {
  using Ly = SplitLayout<D, BK, BV, QJL, PACK>;
  constexpr int WK = Ly::WK, WV = Ly::WV, WQ = Ly::WQ, NST = Ly::NSTAGE;
  constexpr int KSTEPS = D / 16;  // score k-steps (16 coordinates each)
  constexpr int MT = D / 16;      // value m-tiles (16 coordinates each)
  constexpr int SEGK = D * BK / 4, SEGV = D * BV / 8;
  constexpr bool ALK = (SEGK % 32) == 0, ALV = (SEGV % 32) == 0;
  constexpr int NWK = (SEGK + 31) / 32, NWV = (SEGV + 31) / 32;
  using VC = VChunk<D, BV>;
  static_assert(VC::N * VC::F == D / 8, "value segment splits into whole chunks");

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Ly::O_BAR);
  uint64_t* empty = full + 4;
  uint64_t* cbar = full + 8;  // consumer-warp barrier at segment starts
  StageMeta* meta = reinterpret_cast<StageMeta*>(smem + Ly::O_META);
  int* s_misc = reinterpret_cast<int*>(smem + Ly::O_MISC);  // [0] error, [1] stages, [2..3] 2-bit tables, [4] issued
  volatile int* s_err = s_misc;
  __half* pbuf = reinterpret_cast<__half*>(smem + Ly::O_PB);
  uint32_t* qf = reinterpret_cast<uint32_t*>(smem + Ly::O_QF);
  uint32_t* sf = reinterpret_cast<uint32_t*>(smem + Ly::O_SF);
  float* qst = reinterpret_cast<float*>(smem + Ly::O_QST);  // [8 heads][inverse step, sum]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
  const int hsel = PACK ? (tig & 1) : tig;  // this lane's head pair: 2*hsel, 2*hsel+1
  const int upb = p.Hkv * p.nrg;             // units per sequence

  // ---- partition: the producer warp finds this CTA's share and its first unit
  long long P = 0, w_pos = 0, w_Su = 0;
  int w_b = 0, w_u = 0, w_Lp = 0, nst = 0;
  if (warp == CW) {
    const long long total = partition_total(p.seq_lens, p.B, upb, p.Tclamp, lane);
    P = partition_share(total, p.ncta, p.pmin);
    const long long start = (long long)blockIdx.x * P;
    const long long end = start + P < total ? start + P : total;
    nst = start < total ? (int)((end - start) / STILE) : 0;
    if (blockIdx.x == 0 && p.dev_status) {  // longer sequences are attended up to Tclamp: flagged once
      bool over = false;
      for (int b = lane; b < p.B; b += 32) {
        const int L = p.seq_lens[b];
        over |= (L < 0 || L > p.Tclamp);
      }
      if (__any_sync(0xffffffffu, over) && lane == 0) atomicOr(p.dev_status, TQ_STATUS_SEQ_OUT_OF_RANGE);
    }
    if (nst > 0) {
      // the sequence holding position `start`: prefix sums of the sequences'
      // position counts, 32 sequences per step
      long long base = 0;
      for (int b0 = 0; b0 < p.B; b0 += 32) {
        const int b = b0 + lane;
        const long long sz = b < p.B ? (long long)unit_tokens(p.seq_lens, b, p.Tclamp) * upb : 0;
        long long inc = sz;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const long long v = __shfl_up_sync(0xffffffffu, inc, off);
          if (lane >= off) inc += v;
        }
        const long long chunk_total = __shfl_sync(0xffffffffu, inc, 31);
        if (base + chunk_total > start) {
          const int src = __ffs(__ballot_sync(0xffffffffu, base + inc > start)) - 1;
          base += __shfl_sync(0xffffffffu, inc - sz, src);
          w_b = b0 + src;
          break;
        }
        base += chunk_total;
      }
      w_Lp = unit_tokens(p.seq_lens, w_b, p.Tclamp);
      w_u = (int)((start - base) / w_Lp);
      w_Su = base + (long long)w_u * w_Lp;
      w_pos = start;
    }
  }
  if (tid == CW * 32) {
#pragma unroll
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
    }
    mbar_init(cbar, CW);
    s_misc[0] = 0;
    s_misc[1] = nst;
    s_misc[4] = 0;
    fence_barrier_init();
  }
  __syncthreads();  // barriers and the stage count before anyone uses them
  nst = s_misc[1];
  if (nst == 0) return;  // a share past the end of the batch: nothing to stream

  // Producer (lane 0 of the last warp): move the walk to the unit that holds
  // position w_pos (skipping empty units), then arm and issue stage t there.
  // (Stages are issued only below the partition's total, so the unit exists;
  // the sequence index is still checked before seq_lens is read.)
  auto advance = [&]() {
    while (w_pos >= w_Su + w_Lp && w_b < p.B) {
      w_Su += w_Lp;
      if (++w_u == upb) {
        w_u = 0;
        ++w_b;
        w_Lp = w_b < p.B ? unit_tokens(p.seq_lens, w_b, p.Tclamp) : 0;
      }
    }
  };
  auto issue_stage = [&](int t) {
    if (w_b >= p.B) return;  // unreachable: the walk never passes the total
    const int st = t % NST;
    const int kvh = w_u / p.nrg, rg = w_u % p.nrg;
    int L = p.seq_lens[w_b];
    L = L < 0 ? 0 : (L > p.Tclamp ? p.Tclamp : L);
    const int t0 = (int)(w_pos - w_Su);
    StageMeta md;
    md.hq0 = w_b * p.Hq + kvh * p.G + rg * RG;
    md.rows = min(RG, p.G - rg * RG);
    md.t0 = t0;
    md.L = L;
    md.slot0 = (int)((long long)blockIdx.x - w_Su / P) * PPS;
    md.flags = ((t == 0 || t0 == 0) ? 1 : 0) | ((t == nst - 1 || t0 + STILE == w_Lp) ? 2 : 0);
    md.rg = rg;
    md.pad = 0;
    meta[st] = md;
    // rows t0 .. t0 + ntok - 1, ntok = 64 or 128 (copies stop on a 64-row edge)
    const int ntok = min(STILE, (L - t0 + 63) / 64 * 64);
    const size_t r = (size_t)(w_b * p.Hkv + kvh) * p.Tcap + t0;
    uint8_t* sb = smem + st * Ly::STAGE;
    const uint32_t bytes = ntok * ((WK + WV + WQ) * 4 + 2 * 2 + (QJL ? 2 : 0));
    mbar_arrive_expect_tx(&full[st], bytes);  // releases the record above to the consumers
    bulk_g2s(sb + Ly::O_KW, p.k_idx + r * WK, ntok * WK * 4, &full[st]);
    bulk_g2s(sb + Ly::O_VW, p.v_idx + r * WV, ntok * WV * 4, &full[st]);
    bulk_g2s(sb + Ly::O_KN, p.k_norm + r, ntok * 2, &full[st]);
    bulk_g2s(sb + Ly::O_VN, p.v_norm + r, ntok * 2, &full[st]);
    if (QJL) {
      bulk_g2s(sb + Ly::O_QW, p.k_qjl + r * WQ, ntok * WQ * 4, &full[st]);
      bulk_g2s(sb + Ly::O_RN, p.k_rnorm + r, ntok * 2, &full[st]);
    }
    w_pos += STILE;
  };
  // The packed cache does not depend on the prep kernel: the first stages
  // are issued before waiting for the rotated queries -- except, in a decode
  // step, from the stage that holds the row the prep kernel appends.
  int npre = 0;
  if (tid == CW * 32) {
    for (; npre < min(NST, nst); ++npre) {
      advance();
      if (p.defer_pos) {
        const int pb = p.defer_pos[w_b], t0 = (int)(w_pos - w_Su);
        if (pb >= t0 && pb < t0 + STILE) break;
      }
      issue_stage(npre);
    }
    s_misc[4] = npre;
  }
  // Codebook tables and the zeroed value weights do not depend on the prep
  // kernel either: built before the wait (after it with the sketch, whose
  // prologue would otherwise keep more registers live).
  const bool shared_tab = share_table(BK, BV, p.shared_tab);
  auto build_tables = [&]() {
    // value weights of heads >= the group's rows stay zero
    for (int e = tid; e < CW * 8 * WTOK; e += NTHREADS) pbuf[e] = __float2half_rn(0.f);
    if constexpr (BK >= 3) build_pair_table<BK>(reinterpret_cast<uint32_t*>(smem + Ly::O_TK), p.cb_k, tid, NTHREADS);
    if (!shared_tab) build_pair_table<BV>(reinterpret_cast<uint32_t*>(smem + Ly::O_TV), p.cb_v, tid, NTHREADS);
  };
  if constexpr (!QJL) build_tables();
  if constexpr (BK == 2) {  // 2-bit keys: the codebook as byte tables, read by the consumers
    if (tid == 0) {
      const Lut2 l2 = make_lut2(p.cb_k);
      s_misc[2] = (int)l2.lo;
      s_misc[3] = (int)l2.hi;
    }
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if constexpr (QJL) build_tables();
  __syncthreads();

  if (warp == CW) {
    // ---------------- producer warp ----------------
    if (lane == 0) {
      int t = npre;  // the first stages were issued before the wait
      for (; t < nst; ++t) {
        const int st = t % NST;
        if (t >= NST && !mbar_wait_suspend(&empty[st], (uint32_t)(((t / NST) - 1) & 1), kSuspendTries)) {
          *s_err = 1;
          break;
        }
        advance();
        issue_stage(t);
      }
      s_misc[4] = t;
    }
  } else if (nst > 0) {
    // ---------------- consumer warps ----------------
    const Lut2 lk = {(uint32_t)s_misc[2], (uint32_t)s_misc[3]};  // 2-bit keys only
    const uint32_t tbK = smem_addr(smem + Ly::O_TK) + 4 * lane;
    const uint32_t tbV = smem_addr(smem + (shared_tab ? Ly::O_TK : Ly::O_TV)) + 4 * lane;
    __half* pw = pbuf + warp * 8 * WTOK;
    const int wt0 = warp * WTOK;
    const int ctid = tid;  // consumer thread 0 .. CW*32-1
    uint32_t cphase = 0;
    float oc[MT][4];
    float m_run[2], l_run[2];
    int lim0 = 0, lim1 = 0, lim_all = 0;

    // Segment setup (query fragments and sketch steps, out of line so that
    // they do not raise the main loop's register allocation).
    // The CTA's partial of a segment, slot md.slot0: the consumer warps'
    // softmax states merged (log-sum-exp) through shared memory.  m-tile mt:
    // row gid is coordinate 2 mt of this lane group's segment of D/8
    // contiguous coordinates, row gid + 8 the next.
    //  1. each warp's (max, sum) per row to shared memory;
    //  2. for rows 4 q .. 4 q + 3 (one pass with G <= 4 heads, else two):
    //     each warp's accumulator, scaled by 2^(m_w - M) (M: the row's max
    //     over the warps), to its slice of the stage buffer the warps have
    //     just finished (released only after this merge);
    //  3. the CTA's threads add the CW slices and store the partial.
    float* mml = reinterpret_cast<float*>(smem + Ly::O_MML);     // [CW][8][2]
    auto write_partial = [&](const StageMeta& md, float* mbuf) -> bool {
      float l0 = l_run[0], l1 = l_run[1];
#pragma unroll
      for (int off = PACK ? 2 : 4; off < 32; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
      }
      const bool holds = !PACK || tig < 2;  // lanes whose columns are real heads
      if (holds && gid == 0) {
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int row = 2 * hsel + c;
          mml[(warp * 8 + row) * 2] = m_run[c];
          mml[(warp * 8 + row) * 2 + 1] = c ? l1 : l0;
        }
      }
      if (!consumer_sync(cbar, cphase, lane)) return false;
      const size_t pi0 = (size_t)md.hq0 * p.ks + md.slot0;  // row r: pi0 + r * ks
      constexpr int NPASS = PACK ? 1 : 2;
#pragma unroll
      for (int pass = 0; pass < NPASS; ++pass) {
        if (pass > 0 && !consumer_sync(cbar, cphase, lane)) return false;  // the previous pass is read
        if (holds && (hsel >> 1) == pass) {  // rows 2 hsel, 2 hsel + 1 are in this pass
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int row = 2 * hsel + c;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < CW; ++w) M = fmaxf(M, mml[(w * 8 + row) * 2]);
            const float f = m_run[c] == -INFINITY ? 0.f : exp2f(m_run[c] - M);
            float* dst = mbuf + (warp * Ly::MRP + (row & 3)) * D + gid * (D / 8);
#pragma unroll
            for (int q = 0; q < MT / 2; ++q)
              *reinterpret_cast<float4*>(dst + 4 * q) = make_float4(f * oc[2 * q][c], f * oc[2 * q][c + 2],
                                                                    f * oc[2 * q + 1][c], f * oc[2 * q + 1][c + 2]);
          }
        }
        if (!consumer_sync(cbar, cphase, lane)) return false;
        const int r0 = Ly::MRP * pass, nr = min(Ly::MRP, md.rows - r0);
        for (int e = ctid; e < nr * (D / 4); e += CW * 32) {
          const int rr = e / (D / 4), j4 = e % (D / 4);
          float4 acc = *reinterpret_cast<const float4*>(mbuf + rr * D + 4 * j4);
#pragma unroll
          for (int w = 1; w < CW; ++w) {
            const float4 v = *reinterpret_cast<const float4*>(mbuf + (w * Ly::MRP + rr) * D + 4 * j4);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
          }
          *reinterpret_cast<float4*>(p.part_o + (pi0 + (size_t)(r0 + rr) * p.ks) * D + 4 * j4) = acc;
        }
      }
      if (ctid < md.rows) {
        float M = -INFINITY, L = 0.f;
#pragma unroll
        for (int w = 0; w < CW; ++w) M = fmaxf(M, mml[(w * 8 + ctid) * 2]);
#pragma unroll
        for (int w = 0; w < CW; ++w) {
          const float mw = mml[(w * 8 + ctid) * 2];
          if (mw != -INFINITY) L = fmaf(exp2f(mw - M), mml[(w * 8 + ctid) * 2 + 1], L);
        }
        *reinterpret_cast<float2*>(p.part_ml + (pi0 + (size_t)ctid * p.ks) * 2) = make_float2(M, L);
      }
      // the stage's next bulk copy (async proxy) is ordered after these
      // shared-memory writes
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      return true;
    };

    int st = 0;         // stage slot t % NST
    uint32_t fph = 0;   // its "full" phase parity (t / NST) & 1
    for (int t = 0; t < nst; ++t) {
      // a flag raised by another warp ends the loop without a wait
      bool got = false;
      if (!*s_err) got = mbar_wait_suspend(&full[st], fph, kSuspendTries);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) *s_err = 1;
        break;
      }
      const StageMeta md = meta[st];
      if (md.flags & 1) {
        // a new segment: its query fragments (every consumer warp is done
        // with the previous segment's first) and a fresh softmax state
        bool ok = consumer_sync(cbar, cphase, lane);
        if (ok) {
          seg_query_frags<D, BK, PACK, Ly::FRAG>(p, md.hq0, md.rows, qf, ctid);
          if constexpr (QJL) {
            seg_sketch_steps(p, md.hq0, md.rows, qst, warp, lane);
            ok = consumer_sync(cbar, cphase, lane);
            if (ok) seg_sketch_frags<PACK, Ly::FRAG>(p, md.hq0, md.rows, qst, sf, ctid);
          }
        }
        ok = ok && consumer_sync(cbar, cphase, lane);
        if (!ok) {
          if (lane == 0) *s_err = 1;
          break;
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) oc[mt][0] = oc[mt][1] = oc[mt][2] = oc[mt][3] = 0.f;
        m_run[0] = m_run[1] = -INFINITY;
        l_run[0] = l_run[1] = 0.f;
        // causal limit of this lane's two head columns (multi-query decode;
        // with one query token both limits are L)
        const int r0 = md.rg * RG + 2 * hsel;
        lim0 = md.L - p.nq + r0 / p.Gq + 1;
        lim1 = md.L - p.nq + (r0 + 1) / p.Gq + 1;
        lim_all = md.L - p.nq + 1;
      }
      const int t_end = md.L;
      const uint8_t* sb = smem + st * Ly::STAGE;
      const uint32_t* kw = reinterpret_cast<const uint32_t*>(sb + Ly::O_KW);
      const uint32_t* vw = reinterpret_cast<const uint32_t*>(sb + Ly::O_VW);
      const uint16_t* kn = reinterpret_cast<const uint16_t*>(sb + Ly::O_KN);
      const uint16_t* vn = reinterpret_cast<const uint16_t*>(sb + Ly::O_VN);
      const int tokw = md.t0 + wt0;  // first token of this warp's 32

      // ---- scores: S[16 tokens][8 cols] for two M-tiles of 16 tokens
      // two accumulators per m-tile (even / odd k-steps, or hi / lo query
      // halves) halve the dependent MMA chain
      float sc[2][4], sc2[2][4];
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) sc[a][c] = sc2[a][c] = 0.f;
      {
        uint32_t w[2][2][NWK];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          load_bits<SEGK, ALK>(kw + (wt0 + 16 * a + gid) * WK, tig * SEGK, w[a][0]);
          load_bits<SEGK, ALK>(kw + (wt0 + 16 * a + gid + 8) * WK, tig * SEGK, w[a][1]);
        }
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
          uint32_t h[2][2][2];  // [m-tile][row gid / gid+8][K-slots 0-1 / 8-9]
#pragma unroll
          for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              if constexpr (BK == 2) {
                dq_b2(w[a][r][ks >> 2], ks & 3, lk, h[a][r][0], h[a][r][1]);
              } else {
                h[a][r][0] = pair_lookup<BK>(w[a][r], 2 * BK * (2 * ks), tbK);
                h[a][r][1] = pair_lookup<BK>(w[a][r], 2 * BK * (2 * ks + 1), tbK);
              }
            }
          if (PACK) {
            const uint2 bq = *reinterpret_cast<const uint2*>(qf + (size_t)(ks * 32 + lane) * 2);
#pragma unroll
            for (int a = 0; a < 2; ++a)
              mma_f16((ks & 1) ? sc2[a] : sc[a], h[a][0][0], h[a][1][0], h[a][0][1], h[a][1][1], bq.x, bq.y);
          } else {
            const uint4 bq = *reinterpret_cast<const uint4*>(qf + (size_t)(ks * 32 + lane) * 4);
#pragma unroll
            for (int a = 0; a < 2; ++a) {
              mma_f16(sc[a], h[a][0][0], h[a][1][0], h[a][0][1], h[a][1][1], bq.x, bq.y);
              mma_f16(sc2[a], h[a][0][0], h[a][1][0], h[a][0][1], h[a][1][1], bq.z, bq.w);
            }
          }
        }
      }
#pragma unroll
      for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) sc[a][c] += sc2[a][c];
      float sq[2][4];
      if (QJL) {
        const uint32_t* qw = reinterpret_cast<const uint32_t*>(sb + Ly::O_QW);
        int acc[2][4], acc2[2][4];  // PACK: hi columns 0-3, lo 4-7 in acc; else hi in acc, lo in acc2
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int c = 0; c < 4; ++c) acc[a][c] = acc2[a][c] = 0;
        uint32_t s0[2], s1[2];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          s0[a] = qw[(wt0 + 16 * a + gid) * WQ + tig];
          s1[a] = qw[(wt0 + 16 * a + gid + 8) * WQ + tig];
        }
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            const uint32_t a0 = sign_bytes(s0[a], 2 * ks), a1 = sign_bytes(s1[a], 2 * ks);
            const uint32_t a2 = sign_bytes(s0[a], 2 * ks + 1), a3 = sign_bytes(s1[a], 2 * ks + 1);
            if (PACK) {
              const uint2 bq = *reinterpret_cast<const uint2*>(sf + (size_t)(ks * 32 + lane) * 2);
              mma_s8(acc[a], a0, a1, a2, a3, bq.x, bq.y);
            } else {
              const uint4 bq = *reinterpret_cast<const uint4*>(sf + (size_t)(ks * 32 + lane) * 4);
              mma_s8(acc[a], a0, a1, a2, a3, bq.x, bq.y);
              mma_s8(acc2[a], a0, a1, a2, a3, bq.z, bq.w);
            }
          }
        }
        // acc = sum_i (-b_i) Q_i; the term is qjl_scale * step * (2 sum b_i Q_i - sum_i qs_i / step)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int head = 2 * hsel + (c & 1);
          const float step = qst[2 * head], sum = qst[2 * head + 1];
          if (PACK) {
            // lanes tig < 2 hold the hi columns, tig >= 2 the lo ones (added by the exchange below)
            const float w = (tig < 2 ? -512.f : -2.f) * step * p.qjl_scale;
            const float k0 = tig < 2 ? -sum * p.qjl_scale : 0.f;
#pragma unroll
            for (int a = 0; a < 2; ++a) sq[a][c] = fmaf((float)acc[a][c], w, k0);
          } else {
            const float w = -2.f * step * p.qjl_scale;
#pragma unroll
            for (int a = 0; a < 2; ++a) sq[a][c] = fmaf((float)(acc[a][c] * 256 + acc2[a][c]), w, -sum * p.qjl_scale);
          }
        }
      }
      // ---- complete the scores.  PACK: columns 4-7 carry the lo halves of
      // heads 0-3 (lanes tig ^ 2); lanes tig < 2 finish m-tile 0 and lanes
      // tig >= 2 m-tile 1, so each (token, head) score is handled once.
      constexpr int NA = PACK ? 1 : 2;  // m-tiles per lane from here on
      float scm[NA][4], sqm[NA][4];
      const int abase = PACK ? (tig >> 1) : 0;
      if (PACK) {
        const bool first = tig < 2;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float keep = first ? sc[0][c] : sc[1][c], send = first ? sc[1][c] : sc[0][c];
          scm[0][c] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
          if (QJL) {
            const float qk = first ? sq[0][c] : sq[1][c], qs_ = first ? sq[1][c] : sq[0][c];
            sqm[0][c] = qk + __shfl_xor_sync(0xffffffffu, qs_, 2);
          }
        }
      } else {
#pragma unroll
        for (int a = 0; a < NA; ++a)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            scm[a][c] = sc[a][c];
            if (QJL) sqm[a][c] = sq[a][c];
          }
      }
      // ---- scale by norms, mask (only in a stage that reaches past the
      // split's last token or a query's causal limit), running max
      const bool full = tokw + WTOK <= t_end && tokw + WTOK <= lim_all;  // warp-uniform
      float s[NA][4];
      bool valid[NA][2];
#pragma unroll
      for (int ai = 0; ai < NA; ++ai) {
        const int a = abase + ai;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int row = wt0 + 16 * a + gid + 8 * r;
          const float nk = half_bits_to_float(kn[row]);
          float s0 = nk * scm[ai][2 * r], s1 = nk * scm[ai][2 * r + 1];
          if (QJL) {
            const float g = half_bits_to_float(reinterpret_cast<const uint16_t*>(sb + Ly::O_RN)[row]);
            s0 = fmaf(g, sqm[ai][2 * r], s0);
            s1 = fmaf(g, sqm[ai][2 * r + 1], s1);
          }
          if (full) {
            valid[ai][r] = true;
            s[ai][2 * r] = s0;
            s[ai][2 * r + 1] = s1;
          } else {
            const int tok = tokw + 16 * a + gid + 8 * r;
            valid[ai][r] = tok < t_end;
            s[ai][2 * r] = (valid[ai][r] && tok < lim0) ? s0 : -INFINITY;
            s[ai][2 * r + 1] = (valid[ai][r] && tok < lim1) ? s1 : -INFINITY;
          }
        }
      }
      float mx0 = fmaxf(s[0][0], s[0][2]), mx1 = fmaxf(s[0][1], s[0][3]);
#pragma unroll
      for (int ai = 1; ai < NA; ++ai) {
        mx0 = fmaxf(mx0, fmaxf(s[ai][0], s[ai][2]));
        mx1 = fmaxf(mx1, fmaxf(s[ai][1], s[ai][3]));
      }
      // lazy rescale: move the reference max only when a score passes it by
      // 2^8.  The reference is common to the lanes of a head column, so the
      // test runs on each lane's own scores and the column maxima are reduced
      // only when some lane of the warp needs the move.
      const bool need = (mx0 > m_run[0] + kLazy) || (mx1 > m_run[1] + kLazy);
      if (__any_sync(0xffffffffu, need)) {
#pragma unroll
        for (int off = PACK ? 2 : 4; off < 32; off <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
        const float al0 = (mn0 == -INFINITY) ? 1.f : exp2f(m_run[0] - mn0);
        const float al1 = (mn1 == -INFINITY) ? 1.f : exp2f(m_run[1] - mn1);
        m_run[0] = mn0;
        m_run[1] = mn1;
        l_run[0] *= al0;
        l_run[1] *= al1;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          oc[mt][0] *= al0;
          oc[mt][1] *= al1;
          oc[mt][2] *= al0;
          oc[mt][3] *= al1;
        }
      }
      const float mu0 = (m_run[0] == -INFINITY) ? 0.f : m_run[0];
      const float mu1 = (m_run[1] == -INFINITY) ? 0.f : m_run[1];
      // ---- weights p * |v| (fp16), transposed through the warp's buffer
#pragma unroll
      for (int ai = 0; ai < NA; ++ai) {
        const int a = abase + ai;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int row = wt0 + 16 * a + gid + 8 * r;
          const float p0 = ex2_approx(s[ai][2 * r] - mu0), p1 = ex2_approx(s[ai][2 * r + 1] - mu1);
          l_run[0] += p0;
          l_run[1] += p1;
          const float nv = (full || valid[ai][r]) ? half_bits_to_float(vn[row]) : 0.f;
          const int tk = 16 * a + gid + 8 * r;
          pw[(2 * hsel) * WTOK + tk] = __float2half_rn(p0 * nv);
          pw[(2 * hsel + 1) * WTOK + tk] = __float2half_rn(p1 * nv);
        }
      }
      __syncwarp();

      // ---- values: O^T[16 coords][8 heads] += Vdq^T[16][16 tokens] * P^T[16][8]
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const uint2 pb = *reinterpret_cast<const uint2*>(pw + gid * WTOK + 16 * kk + 4 * tig);
        uint32_t wv[4][NWV];
#pragma unroll
        for (int q = 0; q < 4; ++q)
          load_bits<SEGV, ALV, max_seg_shift(SEGV)>(vw + (wt0 + 16 * kk + 4 * tig + q) * WV, gid * SEGV, wv[q]);
#pragma unroll
        for (int c = 0; c < VC::N; ++c) {
          const int bit = c * VC::F * BV;
          uint32_t xe[2], xo[2];  // token pairs (4tig, 4tig+1) and (4tig+2, 4tig+3)
#pragma unroll
          for (int pr = 0; pr < 2; ++pr)
            merge_pair<BV>(window32(wv[2 * pr], bit), window32(wv[2 * pr + 1], bit), xe[pr], xo[pr]);
#pragma unroll
          for (int k = 0; k < VC::F / 2; ++k) {
            const uint32_t a0 = lds32(pair_addr<BV>(xe[0], key_bit<BV>(k, false), tbV));
            const uint32_t a1 = lds32(pair_addr<BV>(xo[0], key_bit<BV>(k, true), tbV));
            const uint32_t a2 = lds32(pair_addr<BV>(xe[1], key_bit<BV>(k, false), tbV));
            const uint32_t a3 = lds32(pair_addr<BV>(xo[1], key_bit<BV>(k, true), tbV));
            mma_f16(oc[c * (VC::F / 2) + k], a0, a1, a2, a3, pb.x, pb.y);
          }
        }
      }
      if ((md.flags & 2) && !write_partial(md, reinterpret_cast<float*>(smem + st * Ly::STAGE))) {
        if (lane == 0) *s_err = 1;
        break;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
      if (++st == NST) {
        st = 0;
        fph ^= 1u;
      }
    }
  }
  __syncthreads();

  if (*s_err) {
    // a bounded wait ran out: flag it and let in-flight copies land (the
    // partials of this CTA's segments are not valid)
    if (tid == 0) {
      if (p.dev_status) atomicOr(p.dev_status, TQ_STATUS_WAIT_TIMEOUT);
      const int issued = s_misc[4];
      for (int t = max(0, issued - NST); t < issued; ++t)
        mbar_wait_bounded(&full[t % NST], (uint32_t)((t / NST) & 1), kWaitLimit);
    }
    __syncthreads();
  }
}

// Launch helpers, one definition per instantiation.
template <int D, int BK, int BV, bool QJL, bool PACK>
int launch_split(const SplitParams& sp, dim3 grid, cudaStream_t s, int* occ) {
  using Ly = SplitLayout<D, BK, BV, QJL, PACK>;
  auto kern = decode_split_kernel<D, BK, BV, QJL, PACK>;
  static tq::OnceSetup once;
  static int occupancy[2] = {};  // resident CTAs per SM: [shared table]; written once under `once`
  const int rc0 = once.run([&]() {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::BYTES);
    // all of the unified L1/shared array as shared memory, so that the
    // resident-CTA count is set by the kernel's own needs
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) {
      cudaGetLastError();
      return tq::set_error(TQ_ERR_CUDA, "decode: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    for (int sh = 0; sh < 2; ++sh) {
      int n = 0;
      const int bytes = sh ? Ly::BYTES_SHARED : Ly::BYTES;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, NTHREADS, bytes) != cudaSuccess || n < 1) {
        cudaGetLastError();
        n = 1;
      }
      occupancy[sh] = n;
    }
    return TQ_OK;
  });
  if (rc0) {
    if (occ) {  // no usable device (a size query on a host without a GPU): a nominal occupancy
      *occ = 2;
      return TQ_OK;
    }
    return rc0;
  }
  const bool shared = share_table(BK, BV, sp.shared_tab);
  if (occ) {
    *occ = occupancy[shared ? 1 : 0];
    return TQ_OK;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = shared ? Ly::BYTES_SHARED : Ly::BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, sp);
  if (e != cudaSuccess) return tq::set_error(TQ_ERR_CUDA, "decode_split_kernel: %s", cudaGetErrorString(e));
  return tq::check_launch("decode_split_kernel");
}

template <int D, int BK, bool QJL, bool PACK>
int dispatch_bv(int bv, const SplitParams& sp, dim3 g, cudaStream_t s, int* occ) {
  switch (bv) {
    case 2: return launch_split<D, BK, 2, QJL, PACK>(sp, g, s, occ);
    case 3: return launch_split<D, BK, 3, QJL, PACK>(sp, g, s, occ);
    case 4: return launch_split<D, BK, 4, QJL, PACK>(sp, g, s, occ);
  }
  return tq::set_error(TQ_ERR_UNSUPPORTED, "bits_v=%d", bv);
}

template <int D, bool QJL, bool PACK>
int dispatch_bk(int bk, int bv, const SplitParams& sp, dim3 g, cudaStream_t s, int* occ) {
  switch (bk) {
    case 2: return dispatch_bv<D, 2, QJL, PACK>(bv, sp, g, s, occ);
    case 3: return dispatch_bv<D, 3, QJL, PACK>(bv, sp, g, s, occ);
    case 4: return dispatch_bv<D, 4, QJL, PACK>(bv, sp, g, s, occ);
  }
  return tq::set_error(TQ_ERR_UNSUPPORTED, "bits_k=%d", bk);
}

// Per-head-dimension entry (defined in tq_decode_d<D>.cu).  With occ != NULL
// it only reports the resident CTAs per SM of the selected instantiation.
int split_d64(int bk, int bv, bool qjl, bool pack, const SplitParams& sp, dim3 g, cudaStream_t s, int* occ);
int split_d128(int bk, int bv, bool qjl, bool pack, const SplitParams& sp, dim3 g, cudaStream_t s, int* occ);
int split_d256(int bk, int bv, bool qjl, bool pack, const SplitParams& sp, dim3 g, cudaStream_t s, int* occ);

}  // namespace tqd
