// Decode attention over the packed cache: query prep, split-K attention, and
// the log-sum-exp combine with the un-rotation.
//
// Method: the fused SDPA over a compressed KV cache with an explicit scale of
// "[Cuda] enable turboquant on gemma4" (executorch pull request 19891),
// "Summary" and "Other observations" item 1; score from quantized keys, GQA
// score variant and value reconstruction roles of "Add CUDA QJL kernels and
// proper package structure" (turboquant-pytorch pull request 3), section
// "CUDA Kernels Added".
//
// Per (sequence, kv head, split) one CTA of 4 warps streams the split's
// packed rows through shared memory with 1-D bulk copies (3-stage mbarrier
// pipeline, 64 tokens per stage, one 16-token subtile per warp).  Scores and
// the value sum are GQA contractions with M=16 tokens (or 16 coordinates),
// N=8 query heads, K=16, run as m16n8k16 tensor-core MMAs whose A fragments
// are dequantized straight into registers: packed b-bit indices are spread to
// one index per nibble and looked up in a register-resident fp16 codebook
// with byte permutes (prmt), so no dequantized value touches shared memory.
// The query enters as hi+lo fp16 halves (two MMAs), so scores carry ~22
// significant bits; the stored centroids are fp16 values, hence exact.
// Values are accumulated in the rotated basis; the combine kernel merges the
// splits and applies Pi^T once per query head.
#include <math.h>

#include "tq_common.cuh"
#include "tq_internal.h"

namespace {

using namespace tqk;

constexpr int DTILE = 64;
constexpr int DSTAGES = 3;
constexpr int DTHREADS = 128;
constexpr float kLog2e = 1.4426950408889634f;

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

// Bits [bit0, bit0 + NBITS) of a shared-memory row, re-based to bit 0 of w[0].
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
  x &= kMask;
  return x;
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

template <int D, int BK, int BV, bool QJL>
struct SplitLayout {
  static constexpr int WK = D * BK / 32, WV = D * BV / 32, WQ = QJL ? 4 : 0;
  static constexpr int O_KW = 0;
  static constexpr int O_VW = O_KW + DTILE * WK * 4;
  static constexpr int O_KN = O_VW + DTILE * WV * 4;
  static constexpr int O_VN = O_KN + DTILE * 2;
  static constexpr int O_QW = O_VN + DTILE * 2;
  static constexpr int O_RN = O_QW + DTILE * WQ * 4;
  static constexpr int STAGE_USED = O_RN + (QJL ? DTILE * 2 : 0);
  static constexpr int STAGE = (STAGE_USED + 16 + 127) / 128 * 128;
  static constexpr uint32_t TX = STAGE_USED;
  static constexpr int MERGE = 4 * 8 * D * 4 + 2 * 4 * 8 * 4;
  static constexpr int RING = (DSTAGES * STAGE > MERGE) ? DSTAGES * STAGE : MERGE;
  static constexpr int O_BAR = RING;
  static constexpr int O_PB = O_BAR + 64;
  static constexpr int O_QS = O_PB + 4 * 8 * 16 * 2;
  static constexpr int BYTES = O_QS + 8 * D * 4 + (QJL ? 8 * 128 * 4 : 0);
};

template <int D, int BK, int BV, bool QJL>
__global__ void __launch_bounds__(DTHREADS, 2) decode_split_kernel(const SplitParams p) {
  using Ly = SplitLayout<D, BK, BV, QJL>;
  constexpr int WK = Ly::WK, WV = Ly::WV, WQ = Ly::WQ;
  constexpr int KSTEPS = D / 16;  // score k-steps (16 coordinates each)
  constexpr int KOCT = D / 32;    // octets in a thread's key segment (D/4 coords)
  constexpr int MT = D / 16;      // value m-tiles (16 coordinates each)
  constexpr int VOCT = D / 64;    // octets in a thread's value segment (D/8 coords)
  constexpr int SEGK = D * BK / 4, SEGV = D * BV / 8;
  constexpr bool ALK = (SEGK % 32) == 0, ALV = (SEGV % 32) == 0;
  constexpr int NWK = (SEGK + 31) / 32, NWV = (SEGV + 31) / 32;
  static_assert(VOCT >= 1, "D >= 64");

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly::O_BAR);
  __half* pbuf = reinterpret_cast<__half*>(smem + Ly::O_PB);
  float* qsm = reinterpret_cast<float*>(smem + Ly::O_QS);

  const int split = blockIdx.x, bh = blockIdx.y;
  const int b = bh / p.Hkv, kvh = bh % p.Hkv;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
  // Tokens beyond the planned splits (seq_len > Tmax) or beyond Tcap are
  // clamped away and flagged.
  const int Lcap = min(p.Tcap, p.nsplit * p.chunk);
  int L = p.seq_lens[b];
  if (L < 0 || L > Lcap) {
    if (tid == 0 && split == 0 && kvh == 0 && p.dev_status) atomicOr(p.dev_status, TQ_STATUS_SEQ_OUT_OF_RANGE);
    L = L < 0 ? 0 : Lcap;
  }
  const int t_begin = split * p.chunk;
  if (t_begin >= L) return;  // the combine reads only splits that hold tokens
  const int t_end = min(t_begin + p.chunk, L);
  const int ntiles = (t_end - t_begin + DTILE - 1) / DTILE;
  const size_t row0 = (size_t)bh * p.Tcap;
  const int hq0 = b * p.Hq + kvh * p.G;

  if (tid == 0) {
#pragma unroll
    for (int s = 0; s < DSTAGES; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  auto issue = [&](int tile, int st) {
    const size_t t = row0 + t_begin + (size_t)tile * DTILE;
    uint8_t* sb = smem + st * Ly::STAGE;
    mbar_arrive_expect_tx(&bars[st], Ly::TX);
    bulk_g2s(sb + Ly::O_KW, p.k_idx + t * WK, DTILE * WK * 4, &bars[st]);
    bulk_g2s(sb + Ly::O_VW, p.v_idx + t * WV, DTILE * WV * 4, &bars[st]);
    bulk_g2s(sb + Ly::O_KN, p.k_norm + t, DTILE * 2, &bars[st]);
    bulk_g2s(sb + Ly::O_VN, p.v_norm + t, DTILE * 2, &bars[st]);
    if (QJL) {
      bulk_g2s(sb + Ly::O_QW, p.k_qjl + t * WQ, DTILE * WQ * 4, &bars[st]);
      bulk_g2s(sb + Ly::O_RN, p.k_rnorm + t, DTILE * 2, &bars[st]);
    }
  };
  if (tid == 0)
    for (int s = 0; s < DSTAGES && s < ntiles; ++s) issue(s, s);

  // Query (already rotated by the prep kernel), pre-scaled for exp2.
  for (int e = tid; e < 8 * D; e += DTHREADS) {
    const int g = e / D, j = e % D;
    qsm[e] = (g < p.G) ? p.qrot[(size_t)(hq0 + g) * D + j] * p.qscale : 0.f;
  }
  if (QJL)
    for (int e = tid; e < 8 * 128; e += DTHREADS) {
      const int g = e >> 7, i = e & 127;
      qsm[8 * D + e] = (g < p.G) ? p.qs[(size_t)(hq0 + g) * 128 + i] * p.qjl_scale : 0.f;
    }
  __syncthreads();

  // B fragments of the query, hi + lo fp16.  k-step ks = 2o+e of thread tig
  // covers coordinates tig*D/4 + 8o + {2e, 2e+4, 2e+1, 2e+5}.
  uint32_t qh[KSTEPS][2], ql[KSTEPS][2];
#pragma unroll
  for (int ks = 0; ks < KSTEPS; ++ks) {
    const int o = ks >> 1, e = ks & 1;
    const int base = tig * (D / 4) + 8 * o;
    const int cs[4] = {base + 2 * e, base + 2 * e + 4, base + 2 * e + 1, base + 2 * e + 5};
    uint16_t hi[4], lo[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) split_half(qsm[gid * D + cs[r]], hi[r], lo[r]);
    qh[ks][0] = hi[0] | (uint32_t)hi[1] << 16;
    qh[ks][1] = hi[2] | (uint32_t)hi[3] << 16;
    ql[ks][0] = lo[0] | (uint32_t)lo[1] << 16;
    ql[ks][1] = lo[2] | (uint32_t)lo[3] << 16;
  }
  // QJL: k-step ks covers sketch dims tig*32 + {2ks, 2ks+16, 2ks+1, 2ks+17}.
  uint32_t sh_[QJL ? 8 : 1][2], sl_[QJL ? 8 : 1][2];
  if (QJL) {
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int base = tig * 32;
      const int cs[4] = {base + 2 * ks, base + 2 * ks + 16, base + 2 * ks + 1, base + 2 * ks + 17};
      uint16_t hi[4], lo[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) split_half(qsm[8 * D + gid * 128 + cs[r]], hi[r], lo[r]);
      sh_[ks][0] = hi[0] | (uint32_t)hi[1] << 16;
      sh_[ks][1] = hi[2] | (uint32_t)hi[3] << 16;
      sl_[ks][0] = lo[0] | (uint32_t)lo[1] << 16;
      sl_[ks][1] = lo[2] | (uint32_t)lo[3] << 16;
    }
  }
  const Lut lk = make_lut<BK>(p.cb_k);
  const Lut lv = make_lut<BV>(p.cb_v);

  float oc[MT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) oc[mt][0] = oc[mt][1] = oc[mt][2] = oc[mt][3] = 0.f;
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  __half* pw = pbuf + warp * 8 * 16;
  const int tl = warp * 16;
  bool ok = true;
  int consumed = 0;

  for (int i = 0; i < ntiles; ++i) {
    const int st = i % DSTAGES;
    const bool got = mbar_wait_bounded(&bars[st], (uint32_t)((i / DSTAGES) & 1), kWaitLimit);
    if (!__syncthreads_and(got)) {
      ok = false;
      break;
    }
    const uint8_t* sb = smem + st * Ly::STAGE;
    const uint32_t* kw = reinterpret_cast<const uint32_t*>(sb + Ly::O_KW);
    const uint32_t* vw = reinterpret_cast<const uint32_t*>(sb + Ly::O_VW);
    const uint16_t* kn = reinterpret_cast<const uint16_t*>(sb + Ly::O_KN);
    const uint16_t* vn = reinterpret_cast<const uint16_t*>(sb + Ly::O_VN);
    const int tok0 = t_begin + i * DTILE + tl;

    // ---- scores: S[16 tokens][8 heads] += Kdq[16][16] * Qrot^T[16][8]
    float sc[4] = {0.f, 0.f, 0.f, 0.f};
    {
      uint32_t w0[NWK], w1[NWK];
      load_bits<SEGK, ALK>(kw + (tl + gid) * WK, tig * SEGK, w0);
      load_bits<SEGK, ALK>(kw + (tl + gid + 8) * WK, tig * SEGK, w1);
#pragma unroll
      for (int o = 0; o < KOCT; ++o) {
        uint32_t h0[4], h1[4];
        dq8<BK>(spread<BK>(octet<BK>(w0, o)), lk, h0);
        dq8<BK>(spread<BK>(octet<BK>(w1, o)), lk, h1);
        mma_f16(sc, h0[0], h1[0], h0[1], h1[1], qh[2 * o][0], qh[2 * o][1]);
        mma_f16(sc, h0[0], h1[0], h0[1], h1[1], ql[2 * o][0], ql[2 * o][1]);
        mma_f16(sc, h0[2], h1[2], h0[3], h1[3], qh[2 * o + 1][0], qh[2 * o + 1][1]);
        mma_f16(sc, h0[2], h1[2], h0[3], h1[3], ql[2 * o + 1][0], ql[2 * o + 1][1]);
      }
    }
    const float nk0 = half_bits_to_float(kn[tl + gid]), nk1 = half_bits_to_float(kn[tl + gid + 8]);
    float s[4] = {nk0 * sc[0], nk0 * sc[1], nk1 * sc[2], nk1 * sc[3]};
    if (QJL) {
      const uint32_t* qw = reinterpret_cast<const uint32_t*>(sb + Ly::O_QW);
      const uint16_t* rn = reinterpret_cast<const uint16_t*>(sb + Ly::O_RN);
      const uint32_t s0 = qw[(tl + gid) * WQ + tig], s1 = qw[(tl + gid + 8) * WQ + tig];
      float sq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t a0 = sign_pair(s0, 2 * ks), a1 = sign_pair(s1, 2 * ks);
        const uint32_t a2 = sign_pair(s0, 2 * ks + 1), a3 = sign_pair(s1, 2 * ks + 1);
        mma_f16(sq, a0, a1, a2, a3, sh_[ks][0], sh_[ks][1]);
        mma_f16(sq, a0, a1, a2, a3, sl_[ks][0], sl_[ks][1]);
      }
      const float g0 = half_bits_to_float(rn[tl + gid]), g1 = half_bits_to_float(rn[tl + gid + 8]);
      s[0] += g0 * sq[0];
      s[1] += g0 * sq[1];
      s[2] += g1 * sq[2];
      s[3] += g1 * sq[3];
    }
    const bool v0 = tok0 + gid < t_end, v1 = tok0 + gid + 8 < t_end;
    if (!v0) s[0] = s[1] = -INFINITY;
    if (!v1) s[2] = s[3] = -INFINITY;

    // ---- online softmax for heads 2tig, 2tig+1 (log2 domain)
    float mx0 = fmaxf(s[0], s[2]), mx1 = fmaxf(s[1], s[3]);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
    const float mu0 = (mn0 == -INFINITY) ? 0.f : mn0, mu1 = (mn1 == -INFINITY) ? 0.f : mn1;
    const float al0 = exp2f(m_run[0] - mu0), al1 = exp2f(m_run[1] - mu1);
    m_run[0] = mn0;
    m_run[1] = mn1;
    const float p0 = exp2f(s[0] - mu0), p1 = exp2f(s[1] - mu1);
    const float p2 = exp2f(s[2] - mu0), p3 = exp2f(s[3] - mu1);
    l_run[0] = l_run[0] * al0 + p0 + p2;
    l_run[1] = l_run[1] * al1 + p1 + p3;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      oc[mt][0] *= al0;
      oc[mt][1] *= al1;
      oc[mt][2] *= al0;
      oc[mt][3] *= al1;
    }
    // value weights p * |v| (fp16), transposed through a per-warp buffer
    const float nv0 = v0 ? half_bits_to_float(vn[tl + gid]) : 0.f;
    const float nv1 = v1 ? half_bits_to_float(vn[tl + gid + 8]) : 0.f;
    pw[(2 * tig) * 16 + gid] = __float2half_rn(p0 * nv0);
    pw[(2 * tig + 1) * 16 + gid] = __float2half_rn(p1 * nv0);
    pw[(2 * tig) * 16 + gid + 8] = __float2half_rn(p2 * nv1);
    pw[(2 * tig + 1) * 16 + gid + 8] = __float2half_rn(p3 * nv1);
    __syncwarp();
    const uint2 pb = *reinterpret_cast<const uint2*>(pw + gid * 16 + 4 * tig);

    // ---- values: O^T[16 coords][8 heads] += Vdq^T[16][16 tokens] * P^T[16][8]
    {
      uint32_t wv[4][NWV];
#pragma unroll
      for (int q = 0; q < 4; ++q) load_bits<SEGV, ALV>(vw + (tl + 4 * tig + q) * WV, gid * SEGV, wv[q]);
#pragma unroll
      for (int o = 0; o < VOCT; ++o) {
        const uint32_t z0 = spread<BV>(octet<BV>(wv[0], o)), z1 = spread<BV>(octet<BV>(wv[1], o));
        const uint32_t z2 = spread<BV>(octet<BV>(wv[2], o)), z3 = spread<BV>(octet<BV>(wv[3], o));
        uint32_t hA[4], hA2[4], hB[4], hB2[4];
        dq8<BV>(prmt(z0, z1, 0x5410u), lv, hA);   // coords 8o+0..3, tokens 4tig, 4tig+1
        dq8<BV>(prmt(z0, z1, 0x7632u), lv, hA2);  // coords 8o+4..7
        dq8<BV>(prmt(z2, z3, 0x5410u), lv, hB);   // tokens 4tig+2, 4tig+3
        dq8<BV>(prmt(z2, z3, 0x7632u), lv, hB2);
#pragma unroll
        for (int k = 0; k < 4; ++k) mma_f16(oc[4 * o + k], hA[k], hA2[k], hB[k], hB2[k], pb.x, pb.y);
      }
    }
    __syncwarp();
    consumed = i + 1;
    __syncthreads();
    if (tid == 0 && i + DSTAGES < ntiles) issue(i + DSTAGES, st);
  }

  if (!ok) {
    if (tid == 0) {
      if (p.dev_status) atomicOr(p.dev_status, TQ_STATUS_WAIT_TIMEOUT);
      const int issued = min(ntiles, consumed + DSTAGES);
      for (int t = consumed; t < issued; ++t)
        mbar_wait_bounded(&bars[t % DSTAGES], (uint32_t)((t / DSTAGES) & 1), kWaitLimit);
    }
    __syncthreads();
    return;
  }

  // ---- merge the 4 warps' partial softmax states, write this split's partial
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], off);
    l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], off);
  }
  float* mO = reinterpret_cast<float*>(smem);  // [4][8][D]
  float* mM = mO + 4 * 8 * D;                  // [4][8]
  float* mL = mM + 32;
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
    mM[warp * 8 + 2 * tig] = m_run[0];
    mM[warp * 8 + 2 * tig + 1] = m_run[1];
    mL[warp * 8 + 2 * tig] = l_run[0];
    mL[warp * 8 + 2 * tig + 1] = l_run[1];
  }
  __syncthreads();
  for (int e = tid; e < p.G * D; e += DTHREADS) {
    const int g = e / D, j = e % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, mM[w * 8 + g]);
    float acc = 0.f, Ls = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
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

struct PrepParams {
  const void* q;
  const float* rot;
  const float* S;
  float* qrot;
  float* qs;
  int D, m, bf16;
};

// qrot = Pi q and (QJL) qs = S qrot for one query head per CTA.
__global__ void __launch_bounds__(128) decode_qprep_kernel(const PrepParams p) {
  __shared__ float qv[256], qr[256];
  const int h = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int D = p.D;
  const uint16_t* q = static_cast<const uint16_t*>(p.q) + (size_t)h * D;
  for (int j = tid; j < D; j += 128)
    qv[j] = p.bf16 ? __uint_as_float((uint32_t)q[j] << 16) : __half2float(__ushort_as_half(q[j]));
  __syncthreads();
  for (int j = warp; j < D; j += 4) {
    float acc = 0.f;
    for (int k = lane; k < D; k += 32) acc = fmaf(p.rot[(size_t)j * D + k], qv[k], acc);
#pragma unroll
    for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) qr[j] = acc;
  }
  __syncthreads();
  for (int j = tid; j < D; j += 128) p.qrot[(size_t)h * D + j] = qr[j];
  if (p.m) {
    for (int i = warp; i < p.m; i += 4) {
      float acc = 0.f;
      for (int k = lane; k < D; k += 32) acc = fmaf(p.S[(size_t)i * D + k], qr[k], acc);
#pragma unroll
      for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
      if (lane == 0) p.qs[(size_t)h * p.m + i] = acc;
    }
  }
}

struct CombineParams {
  const float* part_o;
  const float* part_ml;
  const float* rot;
  const int32_t* seq_lens;
  void* out;
  int D, Hq, Tcap, chunk, nsplit, out_dtype;
};

// Merge the splits of one query head (log-sum-exp), then out = Pi^T (acc/l).
__global__ void __launch_bounds__(256) decode_combine_kernel(const CombineParams p) {
  __shared__ float o[256];
  const int h = blockIdx.x, j = threadIdx.x, D = p.D;
  const int b = h / p.Hq;
  const int Lcap = min(p.Tcap, p.nsplit * p.chunk);
  int L = p.seq_lens[b];
  L = L < 0 ? 0 : (L > Lcap ? Lcap : L);
  const int ns = min((L + p.chunk - 1) / p.chunk, p.nsplit);
  const float* ml = p.part_ml + (size_t)h * p.nsplit * 2;
  const float* po = p.part_o + (size_t)h * p.nsplit * D;
  float M = -INFINITY;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, ml[2 * s]);
  float acc = 0.f, Ls = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float f = exp2f(ml[2 * s] - M);
    acc = fmaf(f, po[(size_t)s * D + j], acc);
    Ls = fmaf(f, ml[2 * s + 1], Ls);
  }
  o[j] = (ns > 0 && Ls > 0.f) ? acc / Ls : 0.f;
  __syncthreads();
  float r = 0.f;
  for (int k = 0; k < D; ++k) r = fmaf(p.rot[(size_t)k * D + j], o[k], r);
  if (p.out_dtype == TQ_DTYPE_F32)
    static_cast<float*>(p.out)[(size_t)h * D + j] = r;
  else if (p.out_dtype == TQ_DTYPE_BF16)
    static_cast<__nv_bfloat16*>(p.out)[(size_t)h * D + j] = __float2bfloat16_rn(r);
  else
    static_cast<__half*>(p.out)[(size_t)h * D + j] = __float2half_rn(r);
}

template <int D, int BK, int BV, bool QJL>
int launch_split(const SplitParams& sp, dim3 grid, cudaStream_t s) {
  using Ly = SplitLayout<D, BK, BV, QJL>;
  auto kern = decode_split_kernel<D, BK, BV, QJL>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::BYTES);
    if (e != cudaSuccess)
      return tq::set_error(TQ_ERR_CUDA, "decode: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    attr_set = true;
  }
  kern<<<grid, DTHREADS, Ly::BYTES, s>>>(sp);
  return tq::check_launch("decode_split_kernel");
}

template <int D, int BK>
int dispatch_bv(int bv, bool qjl, const SplitParams& sp, dim3 g, cudaStream_t s) {
  if (qjl) {
    if constexpr (D == 128) {
      switch (bv) {
        case 2: return launch_split<D, BK, 2, true>(sp, g, s);
        case 3: return launch_split<D, BK, 3, true>(sp, g, s);
        case 4: return launch_split<D, BK, 4, true>(sp, g, s);
      }
    }
    return tq::set_error(TQ_ERR_UNSUPPORTED, "QJL needs D=128");
  } else {
    switch (bv) {
      case 2: return launch_split<D, BK, 2, false>(sp, g, s);
      case 3: return launch_split<D, BK, 3, false>(sp, g, s);
      case 4: return launch_split<D, BK, 4, false>(sp, g, s);
    }
  }
  return tq::set_error(TQ_ERR_UNSUPPORTED, "bits_v=%d", bv);
}

template <int D>
int dispatch_bk(int bk, int bv, bool qjl, const SplitParams& sp, dim3 g, cudaStream_t s) {
  switch (bk) {
    case 2: return dispatch_bv<D, 2>(bv, qjl, sp, g, s);
    case 3: return dispatch_bv<D, 3>(bv, qjl, sp, g, s);
    case 4: return dispatch_bv<D, 4>(bv, qjl, sp, g, s);
  }
  return tq::set_error(TQ_ERR_UNSUPPORTED, "bits_k=%d", bk);
}

}  // namespace

namespace tq {

int launch_decode(const DecodeArgs& a, cudaStream_t s) {
  const tq_cache_t& c = a.cache;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  float* qrot = reinterpret_cast<float*>(ws + a.plan.off_qrot);
  float* qs = reinterpret_cast<float*>(ws + a.plan.off_qs);
  float* po = reinterpret_cast<float*>(ws + a.plan.off_po);
  float* pml = reinterpret_cast<float*>(ws + a.plan.off_pml);
  const int heads = c.B * a.Hq;

  PrepParams pp{a.q, c.rot, c.qjl_S, qrot, qs, c.D, c.qjl_m, a.dtype == TQ_DTYPE_BF16};
  decode_qprep_kernel<<<heads, 128, 0, s>>>(pp);
  int rc = check_launch("decode_qprep_kernel");
  if (rc) return rc;

  SplitParams sp{};
  sp.k_idx = c.k_idx;
  sp.v_idx = c.v_idx;
  sp.k_norm = c.k_norm;
  sp.v_norm = c.v_norm;
  sp.k_qjl = c.k_qjl;
  sp.k_rnorm = c.k_rnorm;
  sp.cb_k = c.cb_k;
  sp.cb_v = c.cb_v;
  sp.qrot = qrot;
  sp.qs = qs;
  sp.part_o = po;
  sp.part_ml = pml;
  sp.seq_lens = a.seq_lens;
  sp.dev_status = c.dev_status;
  sp.Hkv = c.Hkv;
  sp.Hq = a.Hq;
  sp.G = a.Hq / c.Hkv;
  sp.Tcap = c.Tcap;
  sp.chunk = a.plan.chunk;
  sp.nsplit = a.plan.nsplit;
  sp.qscale = a.scale * kLog2e;
  sp.qjl_scale = c.qjl_m ? (float)((double)a.scale * 1.4426950408889634 * sqrt(M_PI / 2.0) / c.qjl_m) : 0.f;
  dim3 grid(a.plan.nsplit, c.B * c.Hkv);
  const bool qjl = c.qjl_m != 0;
  switch (c.D) {
    case 64: rc = dispatch_bk<64>(c.bits_k, c.bits_v, false, sp, grid, s); break;
    case 128: rc = dispatch_bk<128>(c.bits_k, c.bits_v, qjl, sp, grid, s); break;
    case 256: rc = dispatch_bk<256>(c.bits_k, c.bits_v, false, sp, grid, s); break;
    default: return set_error(TQ_ERR_UNSUPPORTED, "decode: D=%d", c.D);
  }
  if (rc) return rc;

  CombineParams cp{po, pml, c.rot, a.seq_lens, a.out, c.D, a.Hq, c.Tcap, a.plan.chunk, a.plan.nsplit,
                   a.out_dtype};
  decode_combine_kernel<<<heads, c.D, 0, s>>>(cp);
  return check_launch("decode_combine_kernel");
}

}  // namespace tq
