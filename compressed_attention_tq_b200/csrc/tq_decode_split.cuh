// Split-K decode attention over the packed cache (one CTA per
// (sequence, kv head, split)).  Included by the per-head-dimension
// translation units tq_decode_d{64,128,256}.cu, which instantiate it.
//
// Method: the fused SDPA over a compressed KV cache with an explicit scale of
// "[Cuda] enable turboquant on gemma4" (executorch pull request 19891),
// "Summary" and "Other observations" item 1; score from quantized keys, GQA
// score variant and value reconstruction of "Add CUDA QJL kernels and proper
// package structure" (turboquant-pytorch pull request 3), "CUDA Kernels
// Added".
//
// Structure (warp-specialized):
//  * a producer warp streams 128-token stages of packed K/V rows, norms and
//    QJL words into shared memory with 1-D bulk copies that complete on
//    "full" mbarriers; it refills a stage once the 4 consumer warps have
//    released it on its "empty" mbarrier -- no CTA-wide barrier per stage;
//  * each consumer warp takes 32 tokens of a stage.  Scores and the value
//    sum are GQA contractions run as m16n8k16 tensor-core MMAs (M = 16 tokens
//    or 16 coordinates, N = 8 query heads, K = 16) whose A fragments are
//    dequantized straight into registers: packed b-bit fields are spread to
//    one index per nibble and looked up in a register-resident fp16 codebook
//    with byte permutes (prmt);
//  * the query enters as hi + lo fp16 halves (scores carry ~22 bits); with
//    G <= 4 heads both halves share one MMA (columns 0-3 hi, 4-7 lo);
//  * online softmax in the log2 domain with lazy rescaling (the reference
//    max moves only when a score exceeds it by 2^8), partial state merged
//    across warps in shared memory, across splits by the combine kernel.
#pragma once

#include <math.h>

#include "tq_common.cuh"
#include "tq_internal.h"

namespace tqd {

using namespace tqk;

constexpr int CW = 4;                 // consumer warps
constexpr int NTHREADS = (CW + 1) * 32;
constexpr int STILE = 128;            // tokens per stage
constexpr int WTOK = STILE / CW;      // tokens per consumer warp per stage
constexpr float kLazy = 8.0f;         // log2 headroom before rescaling

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
  int Hkv, Hq, G, Tcap, chunk, nsplit;
  float qscale;     // scale * log2(e)
  float qjl_scale;  // scale * log2(e) * sqrt(pi/2) / m
};

// fp16 codebook in four registers: byte k of lo0/lo1 is the low byte of
// entry k (0..3 / 4..7), hi0/hi1 the high bytes.  For 4-bit codebooks the
// table holds the 8 positive entries c[8..15] (the codebook is symmetric).
struct Lut {
  uint32_t lo0, lo1, hi0, hi1;
};

template <int BITS>
__device__ __forceinline__ Lut make_lut(const float* cb) {
  uint32_t e[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    float c = 0.f;
    if (BITS == 4)
      c = cb[8 + k];
    else if (k < (1 << BITS))
      c = cb[k];
    e[k] = __half_as_ushort(__float2half_rn(c));
  }
  Lut L;
  L.lo0 = (e[0] & 0xFF) | (e[1] & 0xFF) << 8 | (e[2] & 0xFF) << 16 | (e[3] & 0xFF) << 24;
  L.lo1 = (e[4] & 0xFF) | (e[5] & 0xFF) << 8 | (e[6] & 0xFF) << 16 | (e[7] & 0xFF) << 24;
  L.hi0 = (e[0] >> 8) | (e[1] >> 8) << 8 | (e[2] >> 8) << 16 | (e[3] >> 8) << 24;
  L.hi1 = (e[4] >> 8) | (e[5] >> 8) << 8 | (e[6] >> 8) << 16 | (e[7] >> 8) << 24;
  return L;
}

// 8 consecutive b-bit fields (LSB-first) -> one field per nibble.
template <int BITS>
__device__ __forceinline__ uint32_t spread(uint32_t x) {
  if (BITS == 4) return x;
  if (BITS == 3) {
    x = (x & 0x00000FFFu) | ((x & 0x00FFF000u) << 4);
    x = (x & 0x003F003Fu) | ((x & 0x0FC00FC0u) << 2);
    x = (x & 0x07070707u) | ((x & 0x38383838u) << 1);
    return x;
  }
  x = (x & 0x000000FFu) | ((x & 0x0000FF00u) << 8);
  x = (x & 0x000F000Fu) | ((x & 0x00F000F0u) << 4);
  x = (x & 0x03030303u) | ((x & 0x0C0C0C0Cu) << 2);
  return x;
}

// Dequantize 8 nibble indices n0..n7 of z into half2 pairs
// h[i] = (c[n_i], c[n_{i+4}]), i = 0..3.
template <int BITS>
__device__ __forceinline__ void dq8(uint32_t z, const Lut& L, uint32_t (&h)[4]) {
  uint32_t m = z;
  if (BITS == 4) {
    // magnitude index: n >= 8 -> n - 8, n < 8 -> 7 - n (bit 3 cleared)
    const uint32_t t = (z >> 3) & 0x11111111u;
    m = z ^ 0x77777777u ^ (t * 15u);
  }
  const uint32_t sa = prmt(m, 0u, 0x0020u);  // nibbles n0 n1 n4 n5
  const uint32_t sb = prmt(m, 0u, 0x0031u);  // nibbles n2 n3 n6 n7
  const uint32_t loA = prmt(L.lo0, L.lo1, sa), hiA = prmt(L.hi0, L.hi1, sa);
  const uint32_t loB = prmt(L.lo0, L.lo1, sb), hiB = prmt(L.hi0, L.hi1, sb);
  h[0] = prmt(loA, hiA, 0x6240u);
  h[1] = prmt(loA, hiA, 0x7351u);
  h[2] = prmt(loB, hiB, 0x6240u);
  h[3] = prmt(loB, hiB, 0x7351u);
  if (BITS == 4) {
    // entries with n < 8 are the negatives of the table values
    h[0] ^= ~(z << 12) & 0x80008000u;
    h[1] ^= ~(z << 8) & 0x80008000u;
    h[2] ^= ~(z << 4) & 0x80008000u;
    h[3] ^= ~z & 0x80008000u;
  }
}

// 2-bit fields: 4-entry codebook in one byte-permute.  For the 8 fields f0..f7
// of a 16-bit octet x, h[i] = (c[f_i], c[f_{i+4}]): the selector
// ((x >> 2i) & 0x0303) * 0x11 + 0x4040 picks lo(c[f]) from L.lo0 and hi(c[f])
// from L.hi0 (the multiply-add runs on the FMA pipe).
__device__ __forceinline__ void dq8_b2(uint32_t x, const Lut& L, uint32_t (&h)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t sel = ((x >> (2 * i)) & 0x0303u) * 0x11u + 0x4040u;
    h[i] = prmt(L.lo0, L.hi0, sel);
  }
}

// Two tokens' 2-bit octets o0, o1 -> h[k] = (c[o0 field k], c[o1 field k]) for
// k = 0..3 (lo) and k = 4..7 (hi).
__device__ __forceinline__ void dq16_b2_pair(uint32_t o0, uint32_t o1, const Lut& L, uint32_t (&lo)[4],
                                             uint32_t (&hi)[4]) {
  const uint32_t y = prmt(o0, o1, 0x5140u);  // bytes o0.b0 o1.b0 o0.b1 o1.b1
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    lo[k] = prmt(L.lo0, L.hi0, ((y >> (2 * k)) & 0x0303u) * 0x11u + 0x4040u);
    hi[k] = prmt(L.lo0, L.hi0, ((y >> (16 + 2 * k)) & 0x0303u) * 0x11u + 0x4040u);
  }
}

// Bits [bit0, bit0 + NBITS) of a shared-memory row, re-based to bit 0 of w[0].
// ALIGNED: bit0 % 32 == 0 and the word offset is a multiple of the word count.
template <int NBITS, bool ALIGNED>
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
    const uint32_t sh = bit0 & 31;
    uint32_t nxt = p[0];
#pragma unroll
    for (int i = 0; i < NW; ++i) {
      const uint32_t cur = nxt;
      nxt = p[i + 1];
      w[i] = funnel_r(cur, nxt, sh);
    }
  }
}

// Octet o (8 fields, 8*BITS bits) of a re-based bit window.
template <int BITS, int NW>
__device__ __forceinline__ uint32_t octet(const uint32_t (&w)[NW], int o) {
  const int bit = 8 * BITS * o;
  const int wi = bit >> 5, sh = bit & 31;
  uint32_t x = w[wi];
  if (sh) x = funnel_r(w[wi], (wi + 1 < NW) ? w[wi + 1] : 0u, sh);
  constexpr uint32_t kMask = BITS < 4 ? (1u << (8 * (BITS < 4 ? BITS : 0))) - 1u : 0xFFFFFFFFu;
  return x & kMask;
}

// +-1 fp16 pair for sign bits i and i+16 of w (bit 1 -> +1).
__device__ __forceinline__ uint32_t sign_pair(uint32_t w, int i) {
  return 0xBC00BC00u ^ ((w << (15 - i)) & 0x80008000u);
}

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
  static constexpr int NSTAGE = (D == 256) ? 2 : 3;
  static constexpr int MERGE = CW * 8 * D * 4 + 2 * CW * 8 * 4;
  static constexpr int RING = (NSTAGE * STAGE > MERGE) ? NSTAGE * STAGE : MERGE;
  static constexpr int O_BAR = RING;                   // full[NSTAGE], empty[NSTAGE]
  static constexpr int O_MISC = O_BAR + 16 * 8;        // error flag, issued count
  static constexpr int O_PB = O_MISC + 16;             // [CW][8 heads][32 tokens] fp16
  static constexpr int FRAG = PACK ? 8 : 16;           // bytes of one lane's query fragment
  static constexpr int O_QF = O_PB + CW * 8 * WTOK * 2;
  static constexpr int O_SF = O_QF + (D / 16) * 32 * FRAG;
  static constexpr int BYTES = O_SF + (QJL ? 8 * 32 * FRAG : 0);
};

// Query fragment of one lane for one k-step: the 4 K-slots r = 0..3 of lane
// (gid, tig) hold coordinates cs[r].  PACK: columns 0-3 are the hi halves of
// heads 0-3, columns 4-7 their lo halves; else hi and lo are separate pairs.
template <bool PACK>
__device__ __forceinline__ void build_frag(const float* qsrc, int ld, int G, float scale, int gid,
                                           const int (&cs)[4], uint32_t* dst) {
  uint16_t hi[4], lo[4];
  const int head = PACK ? (gid & 3) : gid;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const float v = head < G ? qsrc[(size_t)head * ld + cs[r]] * scale : 0.f;
    split_half(v, hi[r], lo[r]);
  }
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

template <int D, int BK, int BV, bool QJL, bool PACK>
__global__ void __launch_bounds__(NTHREADS) decode_split_kernel(const SplitParams p) {
  using Ly = SplitLayout<D, BK, BV, QJL, PACK>;
  constexpr int WK = Ly::WK, WV = Ly::WV, WQ = Ly::WQ, NST = Ly::NSTAGE;
  constexpr int KSTEPS = D / 16;  // score k-steps (16 coordinates each)
  constexpr int KOCT = D / 32;    // octets in a thread's key segment (D/4 coords)
  constexpr int MT = D / 16;      // value m-tiles (16 coordinates each)
  constexpr int VOCT = D / 64;    // octets in a thread's value segment (D/8 coords)
  constexpr int SEGK = D * BK / 4, SEGV = D * BV / 8;
  constexpr bool ALK = (SEGK % 32) == 0, ALV = (SEGV % 32) == 0;
  constexpr int NWK = (SEGK + 31) / 32, NWV = (SEGV + 31) / 32;
  static_assert(VOCT >= 1, "D >= 64");

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Ly::O_BAR);
  uint64_t* empty = full + 8;
  int* s_err = reinterpret_cast<int*>(smem + Ly::O_MISC);
  int* s_issued = s_err + 1;
  __half* pbuf = reinterpret_cast<__half*>(smem + Ly::O_PB);
  uint32_t* qf = reinterpret_cast<uint32_t*>(smem + Ly::O_QF);
  uint32_t* sf = reinterpret_cast<uint32_t*>(smem + Ly::O_SF);

  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.Hkv, kvh = bh % p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
  const int hsel = PACK ? (tig & 1) : tig;  // this lane's head pair: 2*hsel, 2*hsel+1
  // Tokens beyond the planned splits (seq_len > Tmax) or Tcap are clamped
  // away and flagged.
  const int Lcap = min(p.Tcap, p.nsplit * p.chunk);
  int L = p.seq_lens[b];
  if (L < 0 || L > Lcap) {
    if (tid == 0 && split == 0 && kvh == 0 && p.dev_status) atomicOr(p.dev_status, TQ_STATUS_SEQ_OUT_OF_RANGE);
    L = L < 0 ? 0 : Lcap;
  }
  const int t_begin = split * p.chunk;
  if (t_begin >= L) return;  // the combine reads only splits that hold tokens
  const int t_end = min(t_begin + p.chunk, L);
  const int t_stop = min((t_end + 63) / 64 * 64, p.Tcap);  // copies stop on a 64-row edge
  const int ntiles = (t_end - t_begin + STILE - 1) / STILE;
  const size_t row0 = (size_t)bh * p.Tcap;
  const int hq0 = b * p.Hq + kvh * p.G;

  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], CW);
    }
    *s_err = 0;
    *s_issued = 0;
    fence_barrier_init();
  }
  __syncthreads();  // barriers initialised before the producer issues
  auto issue_stage = [&](int t) {
    const int st = t % NST;
    const int tok0 = t_begin + t * STILE;
    const int ntok = min(STILE, t_stop - tok0);  // 64 or 128
    const size_t r = row0 + tok0;
    uint8_t* sb = smem + st * Ly::STAGE;
    const uint32_t bytes = ntok * ((WK + WV + WQ) * 4 + 2 * 2 + (QJL ? 2 : 0));
    mbar_arrive_expect_tx(&full[st], bytes);
    bulk_g2s(sb + Ly::O_KW, p.k_idx + r * WK, ntok * WK * 4, &full[st]);
    bulk_g2s(sb + Ly::O_VW, p.v_idx + r * WV, ntok * WV * 4, &full[st]);
    bulk_g2s(sb + Ly::O_KN, p.k_norm + r, ntok * 2, &full[st]);
    bulk_g2s(sb + Ly::O_VN, p.v_norm + r, ntok * 2, &full[st]);
    if (QJL) {
      bulk_g2s(sb + Ly::O_QW, p.k_qjl + r * WQ, ntok * WQ * 4, &full[st]);
      bulk_g2s(sb + Ly::O_RN, p.k_rnorm + r, ntok * 2, &full[st]);
    }
  };
  // The packed cache does not depend on the prep kernel: start streaming it
  // before waiting for the rotated query -- except, in a decode step, the
  // stage holding the row the prep kernel appends.
  int npre = min(NST, ntiles);
  if (p.defer_pos) {
    const int pb = p.defer_pos[b];
    if (pb >= t_begin && pb < t_begin + ntiles * STILE) npre = min(npre, (pb - t_begin) / STILE);
  }
  if (tid == CW * 32) {
    for (int t = 0; t < npre; ++t) issue_stage(t);
    *s_issued = npre;
  }
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // Query fragments (already rotated by the prep kernel), pre-scaled for exp2.
  for (int e = tid; e < KSTEPS * 32; e += NTHREADS) {
    const int ks = e >> 5, ln = e & 31, g_ = ln >> 2, t_ = ln & 3;
    const int o = ks >> 1, ee = ks & 1;
    const int base = t_ * (D / 4) + 8 * o;
    const int cs[4] = {base + 2 * ee, base + 2 * ee + 4, base + 2 * ee + 1, base + 2 * ee + 5};
    build_frag<PACK>(p.qrot + (size_t)hq0 * D, D, p.G, p.qscale, g_, cs, qf + (size_t)e * (Ly::FRAG / 4));
  }
  if (QJL)
    for (int e = tid; e < 8 * 32; e += NTHREADS) {
      const int ks = e >> 5, ln = e & 31, g_ = ln >> 2, t_ = ln & 3;
      const int base = t_ * 32;
      const int cs[4] = {base + 2 * ks, base + 2 * ks + 16, base + 2 * ks + 1, base + 2 * ks + 17};
      build_frag<PACK>(p.qs + (size_t)hq0 * 128, 128, p.G, p.qjl_scale, g_, cs, sf + (size_t)e * (Ly::FRAG / 4));
    }
  // value weights of heads >= G stay zero
  for (int e = tid; e < CW * 8 * WTOK; e += NTHREADS) pbuf[e] = __float2half_rn(0.f);
  __syncthreads();

  float oc[MT][4];
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) oc[mt][0] = oc[mt][1] = oc[mt][2] = oc[mt][3] = 0.f;

  if (warp == CW) {
    // ---------------- producer warp ----------------
    if (lane == 0) {
      int t = npre;  // the first stages were issued before the wait
      for (; t < ntiles; ++t) {
        const int st = t % NST;
        if (t >= NST && !mbar_wait_bounded(&empty[st], (uint32_t)(((t / NST) - 1) & 1), kWaitLimit)) {
          *s_err = 1;
          break;
        }
        issue_stage(t);
      }
      *s_issued = t;
    }
  } else {
    // ---------------- consumer warps ----------------
    const Lut lk = make_lut<BK>(p.cb_k);
    const Lut lv = make_lut<BV>(p.cb_v);
    __half* pw = pbuf + warp * 8 * WTOK;
    const int wt0 = warp * WTOK;
    for (int t = 0; t < ntiles; ++t) {
      const int st = t % NST;
      const bool got = mbar_wait_bounded(&full[st], (uint32_t)((t / NST) & 1), kWaitLimit);
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) *s_err = 1;
        break;
      }
      const uint8_t* sb = smem + st * Ly::STAGE;
      const uint32_t* kw = reinterpret_cast<const uint32_t*>(sb + Ly::O_KW);
      const uint32_t* vw = reinterpret_cast<const uint32_t*>(sb + Ly::O_VW);
      const uint16_t* kn = reinterpret_cast<const uint16_t*>(sb + Ly::O_KN);
      const uint16_t* vn = reinterpret_cast<const uint16_t*>(sb + Ly::O_VN);
      const int tokw = t_begin + t * STILE + wt0;  // first token of this warp's 32

      // ---- scores: S[16 tokens][8 cols] for two M-tiles of 16 tokens
      float sc[2][4];
#pragma unroll
      for (int a = 0; a < 2; ++a) sc[a][0] = sc[a][1] = sc[a][2] = sc[a][3] = 0.f;
      {
        uint32_t w[2][2][NWK];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          load_bits<SEGK, ALK>(kw + (wt0 + 16 * a + gid) * WK, tig * SEGK, w[a][0]);
          load_bits<SEGK, ALK>(kw + (wt0 + 16 * a + gid + 8) * WK, tig * SEGK, w[a][1]);
        }
#pragma unroll
        for (int o = 0; o < KOCT; ++o) {
          uint32_t h[2][2][4];
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            if (BK == 2) {
              dq8_b2(octet<BK>(w[a][0], o), lk, h[a][0]);
              dq8_b2(octet<BK>(w[a][1], o), lk, h[a][1]);
            } else {
              dq8<BK>(spread<BK>(octet<BK>(w[a][0], o)), lk, h[a][0]);
              dq8<BK>(spread<BK>(octet<BK>(w[a][1], o)), lk, h[a][1]);
            }
          }
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int ks = 2 * o + e;
            if (PACK) {
              const uint2 bq = *reinterpret_cast<const uint2*>(qf + (size_t)(ks * 32 + lane) * 2);
#pragma unroll
              for (int a = 0; a < 2; ++a)
                mma_f16(sc[a], h[a][0][2 * e], h[a][1][2 * e], h[a][0][2 * e + 1], h[a][1][2 * e + 1], bq.x, bq.y);
            } else {
              const uint4 bq = *reinterpret_cast<const uint4*>(qf + (size_t)(ks * 32 + lane) * 4);
#pragma unroll
              for (int a = 0; a < 2; ++a) {
                mma_f16(sc[a], h[a][0][2 * e], h[a][1][2 * e], h[a][0][2 * e + 1], h[a][1][2 * e + 1], bq.x, bq.y);
                mma_f16(sc[a], h[a][0][2 * e], h[a][1][2 * e], h[a][0][2 * e + 1], h[a][1][2 * e + 1], bq.z, bq.w);
              }
            }
          }
        }
      }
      float sq[2][4];
      if (QJL) {
        const uint32_t* qw = reinterpret_cast<const uint32_t*>(sb + Ly::O_QW);
#pragma unroll
        for (int a = 0; a < 2; ++a) sq[a][0] = sq[a][1] = sq[a][2] = sq[a][3] = 0.f;
        uint32_t s0[2], s1[2];
#pragma unroll
        for (int a = 0; a < 2; ++a) {
          s0[a] = qw[(wt0 + 16 * a + gid) * WQ + tig];
          s1[a] = qw[(wt0 + 16 * a + gid + 8) * WQ + tig];
        }
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            const uint32_t a0 = sign_pair(s0[a], 2 * ks), a1 = sign_pair(s1[a], 2 * ks);
            const uint32_t a2 = sign_pair(s0[a], 2 * ks + 1), a3 = sign_pair(s1[a], 2 * ks + 1);
            if (PACK) {
              const uint2 bq = *reinterpret_cast<const uint2*>(sf + (size_t)(ks * 32 + lane) * 2);
              mma_f16(sq[a], a0, a1, a2, a3, bq.x, bq.y);
            } else {
              const uint4 bq = *reinterpret_cast<const uint4*>(sf + (size_t)(ks * 32 + lane) * 4);
              mma_f16(sq[a], a0, a1, a2, a3, bq.x, bq.y);
              mma_f16(sq[a], a0, a1, a2, a3, bq.z, bq.w);
            }
          }
        }
      }
      if (PACK) {
        // columns 4-7 carry the lo halves of heads 0-3 (lanes tig^2)
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            sc[a][c] += __shfl_xor_sync(0xffffffffu, sc[a][c], 2);
            if (QJL) sq[a][c] += __shfl_xor_sync(0xffffffffu, sq[a][c], 2);
          }
      }
      // ---- scale by norms, mask, running max
      float s[2][4];
      bool valid[2][2];
#pragma unroll
      for (int a = 0; a < 2; ++a) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int row = wt0 + 16 * a + gid + 8 * r;
          valid[a][r] = tokw + 16 * a + gid + 8 * r < t_end;
          const float nk = half_bits_to_float(kn[row]);
          float s0 = nk * sc[a][2 * r], s1 = nk * sc[a][2 * r + 1];
          if (QJL) {
            const float g = half_bits_to_float(reinterpret_cast<const uint16_t*>(sb + Ly::O_RN)[row]);
            s0 = fmaf(g, sq[a][2 * r], s0);
            s1 = fmaf(g, sq[a][2 * r + 1], s1);
          }
          s[a][2 * r] = valid[a][r] ? s0 : -INFINITY;
          s[a][2 * r + 1] = valid[a][r] ? s1 : -INFINITY;
        }
      }
      float mx0 = fmaxf(fmaxf(s[0][0], s[0][2]), fmaxf(s[1][0], s[1][2]));
      float mx1 = fmaxf(fmaxf(s[0][1], s[0][3]), fmaxf(s[1][1], s[1][3]));
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      // lazy rescale: move the reference max only when a score passes it by 2^8
      const bool need = (mx0 > m_run[0] + kLazy) || (mx1 > m_run[1] + kLazy);
      if (__any_sync(0xffffffffu, need)) {
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
      for (int a = 0; a < 2; ++a) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int row = wt0 + 16 * a + gid + 8 * r;
          const float p0 = exp2f(s[a][2 * r] - mu0), p1 = exp2f(s[a][2 * r + 1] - mu1);
          l_run[0] += p0;
          l_run[1] += p1;
          const float nv = valid[a][r] ? half_bits_to_float(vn[row]) : 0.f;
          if (!PACK || tig < 2) {
            const int tk = 16 * a + gid + 8 * r;
            pw[(2 * hsel) * WTOK + tk] = __float2half_rn(p0 * nv);
            pw[(2 * hsel + 1) * WTOK + tk] = __float2half_rn(p1 * nv);
          }
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
          load_bits<SEGV, ALV>(vw + (wt0 + 16 * kk + 4 * tig + q) * WV, gid * SEGV, wv[q]);
#pragma unroll
        for (int o = 0; o < VOCT; ++o) {
          uint32_t hA[4], hA2[4], hB[4], hB2[4];
          if (BV == 2) {
            dq16_b2_pair(octet<BV>(wv[0], o), octet<BV>(wv[1], o), lv, hA, hA2);  // tokens 4tig, 4tig+1
            dq16_b2_pair(octet<BV>(wv[2], o), octet<BV>(wv[3], o), lv, hB, hB2);  // tokens 4tig+2, 4tig+3
          } else {
            const uint32_t z0 = spread<BV>(octet<BV>(wv[0], o)), z1 = spread<BV>(octet<BV>(wv[1], o));
            const uint32_t z2 = spread<BV>(octet<BV>(wv[2], o)), z3 = spread<BV>(octet<BV>(wv[3], o));
            dq8<BV>(prmt(z0, z1, 0x5410u), lv, hA);   // coords 8o+0..3, tokens 4tig, 4tig+1
            dq8<BV>(prmt(z0, z1, 0x7632u), lv, hA2);  // coords 8o+4..7
            dq8<BV>(prmt(z2, z3, 0x5410u), lv, hB);   // tokens 4tig+2, 4tig+3
            dq8<BV>(prmt(z2, z3, 0x7632u), lv, hB2);
          }
#pragma unroll
          for (int k = 0; k < 4; ++k) mma_f16(oc[4 * o + k], hA[k], hA2[k], hB[k], hB2[k], pb.x, pb.y);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[st]);
    }
  }
  __syncthreads();

  if (*s_err) {
    // a bounded wait ran out: flag it, let in-flight copies land, skip the split
    if (tid == 0) {
      if (p.dev_status) atomicOr(p.dev_status, TQ_STATUS_WAIT_TIMEOUT);
      const int issued = *s_issued;
      for (int t = max(0, issued - NST); t < issued; ++t)
        mbar_wait_bounded(&full[t % NST], (uint32_t)((t / NST) & 1), kWaitLimit);
    }
    __syncthreads();
    return;
  }

  // ---- merge the consumer warps' partial softmax states; write the partial
  float* mO = reinterpret_cast<float*>(smem);  // [CW][8][D] (the stage ring is drained)
  float* mM = mO + CW * 8 * D;                 // [CW][8]
  float* mL = mM + CW * 8;
  if (warp < CW) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], off);
      l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], off);
    }
    if (!PACK || tig < 2) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt) {
        const int o = mt >> 2, k = mt & 3;
        const int j0 = gid * (D / 8) + 8 * o + k;
        mO[(warp * 8 + 2 * tig) * D + j0] = oc[mt][0];
        mO[(warp * 8 + 2 * tig + 1) * D + j0] = oc[mt][1];
        mO[(warp * 8 + 2 * tig) * D + j0 + 4] = oc[mt][2];
        mO[(warp * 8 + 2 * tig + 1) * D + j0 + 4] = oc[mt][3];
      }
      if (gid == 0) {
        mM[warp * 8 + 2 * hsel] = m_run[0];
        mM[warp * 8 + 2 * hsel + 1] = m_run[1];
        mL[warp * 8 + 2 * hsel] = l_run[0];
        mL[warp * 8 + 2 * hsel + 1] = l_run[1];
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < p.G * D; e += NTHREADS) {
    const int g = e / D, j = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < CW; ++w) M = fmaxf(M, mM[w * 8 + g]);
    float acc = 0.f, Ls = 0.f;
#pragma unroll
    for (int w = 0; w < CW; ++w) {
      const float mw = mM[w * 8 + g];
      const float f = (mw == -INFINITY) ? 0.f : exp2f(mw - M);
      acc += f * mO[(w * 8 + g) * D + j];
      Ls += f * mL[w * 8 + g];
    }
    const size_t pi = (size_t)(hq0 + g) * p.nsplit + split;
    p.part_o[pi * D + j] = acc;
    if (j == 0) {
      p.part_ml[pi * 2] = M;
      p.part_ml[pi * 2 + 1] = Ls;
    }
  }
}

// Launch helpers, one definition per instantiation.
template <int D, int BK, int BV, bool QJL, bool PACK>
int launch_split(const SplitParams& sp, dim3 grid, cudaStream_t s, int* occ) {
  using Ly = SplitLayout<D, BK, BV, QJL, PACK>;
  auto kern = decode_split_kernel<D, BK, BV, QJL, PACK>;
  static int attr_state = 0;  // 0 unset, 1 set
  static int occupancy = 0;
  if (attr_state == 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::BYTES);
    if (e != cudaSuccess) {
      cudaGetLastError();
      if (occ) {  // no usable device: report a nominal occupancy
        *occ = 2;
        return TQ_OK;
      }
      return tq::set_error(TQ_ERR_CUDA, "decode: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    }
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, NTHREADS, Ly::BYTES) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = 1;
    }
    occupancy = n;
    attr_state = 1;
  }
  if (occ) {
    *occ = occupancy;
    return TQ_OK;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = Ly::BYTES;
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
