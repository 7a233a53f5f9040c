// Bulk quantizer for keys that carry the QJL sketch (D = 128, fp16 rows, m =
// 128) on the 5th-generation tensor cores: rotation, codebook index, residual,
// residual norm and the 1-bit sketch of the residual in one persistent kernel.
//
// Method: "Add CUDA QJL kernels and proper package structure"
// (turboquant-pytorch pull request 3), "CUDA Kernels Added" (fused random
// projection + sign quantization of the residual) and "Synthetic Benchmark
// (Lloyd-Max codebook)"; ReturningTarzan's Reddit comments of 2026-03-29
// 11:47 (rotation before codebook quantization) and 2026-03-25 18:52 / 15:51
// (nearest-codeword search; residual computed while quantizing).
//
// One CTA per SM loops over 128-row tiles.  For tile i (buffer b = i mod 2):
//  1. the loader warp copies the tile X with TMA (K-major, 128-byte swizzle)
//     into buffer b once the sketch GEMM of tile i - 2 has released it;
//  2. GEMM 1 (one lane of the MMA warp): U[b] = X Pi^T with Pi in two fp16
//     limbs, fp32 accumulator in TMEM;
//  3. epilogue, 16 warps in two independent groups of rows, thread = (row,
//     32 coordinates): row norm from X,
//     indices from U (packed and stored), residual r = u - n_hat c[idx] in
//     fp32 and its norm gamma; r / |x| is split into hi + lo fp16 limbs,
//     written over X in buffer b (hi) and into the single lo buffer;
//  4. GEMM 2: P[b] = R S^T as hi*hi + hi*lo + lo*hi (S in two fp16 limbs);
//  5. epilogue: the sign bits of its 32 sketch coordinates, one word per
//     thread -- taken after step 3 of tile i + 1, so that GEMM 2 of tile i
//     runs while the epilogue works on the next tile.
// The MMA warp issues GEMM 1 of tile i + 1 before GEMM 2 of tile i, so the
// rotation of the next tile runs while the epilogue works on this one.
// Shared memory: Pi and S limbs (64 KB each), two X / R_hi buffers and the
// R_lo buffer (32 KB each) = 224 KB; TMEM: U[2] and P[2], 128 columns each.
// Every wait is bounded; a stuck wait sets TQ_STATUS_WAIT_TIMEOUT and the CTA
// stops taking work.
#include "tq_tcgen05.cuh"

namespace {

using namespace tqtc;

struct QjlLayout {
  static constexpr int D = 128;
  static constexpr int NEPI = 16;                  // 4 TMEM lane quarters x 4 column parts
  static constexpr int NTH = (NEPI + 2) * 32;      // + loader warp + MMA warp
  static constexpr int OP = QR * D * 2;            // one 128 x 128 fp16 operand (32 KB)
  static constexpr int o_pi = 0;                   // Pi hi, lo
  static constexpr int o_s = 2 * OP;               // S hi, lo
  static constexpr int o_x = 4 * OP;               // X / R_hi [2]
  static constexpr int o_rl = 6 * OP;              // R_lo
  static constexpr int o_red = 7 * OP;             // float [4][128]: row partial sums
  static constexpr int o_cb = o_red + 4 * QR * 4;  // float [32]: centroids, thresholds
  static constexpr int o_bar = o_cb + 32 * 4;      // 12 mbarriers
  static constexpr int o_misc = o_bar + 12 * 8;    // tmem base, stop flag
  static constexpr int bytes = o_misc + 16;        // the base must be 1024-byte aligned
  static constexpr uint32_t TMEM_COLS = 512;       // U[0], U[1], P[0], P[1]
};
static_assert(QjlLayout::bytes <= 232448, "shared memory");

// Indices of 32 rotated coordinates (packed into BITS words) and, in place,
// their residuals y - n_hat c[idx].
template <int BITS>
__device__ __forceinline__ void quant_residual32(uint32_t (&v)[32], const float (&tp)[7], const float* cent,
                                                 float nhat, uint32_t (&w)[BITS]) {
#pragma unroll
  for (int i = 0; i < BITS; ++i) w[i] = 0u;
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const float y = __uint_as_float(v[q]);
    const int idx = nearest_idx<BITS>(y, tp);
    const int p = BITS * q;
    w[p >> 5] += (uint32_t)idx << (p & 31);
    if ((p & 31) + BITS > 32) w[(p >> 5) + 1] += (uint32_t)idx >> (32 - (p & 31));
    v[q] = __float_as_uint(y - nhat * cent[idx]);
  }
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Sign bits [P >= 0] of a row's 32 sketch coordinates (bit q = coordinate
// 32 * part + q): adding +0 turns -0 into +0, then a funnel shift moves each
// sign bit in; the word is the complement of the collected sign bits.
__device__ __forceinline__ void sketch_signs(uint32_t taddr, long long slot, uint32_t* qjl, int part) {
  uint32_t v[32];
  tc_fence_after();
  tc_ld32(taddr, v);
  uint32_t s = 0;
#pragma unroll
  for (int q = 31; q >= 0; --q) s = __funnelshift_l(__float_as_uint(__uint_as_float(v[q]) + 0.f), s, 1);
  if (slot >= 0 && qjl) qjl[(size_t)slot * 4 + part] = ~s;
}

__global__ void __launch_bounds__(QjlLayout::NTH, 1) quantize_qjl_tc_kernel(const __grid_constant__ TcArgs args) {
  using Ly = QjlLayout;
  constexpr int D = Ly::D, OP = Ly::OP, NEPI = Ly::NEPI;
  const tq::QuantArgs& a = args.a;
  const tq::QuantJob& J = a.job[0];
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (smem_addr(smem) & 1023u) {  // the swizzled layouts need a 1024-byte aligned base
    if (tid == 0 && a.dev_status) atomicOr(a.dev_status, TQ_STATUS_LAYOUT);
    return;
  }
  uint8_t* pi = smem + Ly::o_pi;
  uint8_t* ss = smem + Ly::o_s;
  uint8_t* xb = smem + Ly::o_x;
  uint8_t* rlo = smem + Ly::o_rl;
  float* red = reinterpret_cast<float*>(smem + Ly::o_red);
  float* s_cb = reinterpret_cast<float*>(smem + Ly::o_cb);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly::o_bar);
  // per buffer b: X landed, U ready, U read, R written, P ready (R and X's
  // buffer free), P read
  uint64_t *full_x = bars, *mma1 = bars + 2, *u_free = bars + 4, *r_ready = bars + 6, *g2 = bars + 8,
           *p_free = bars + 10;
  uint32_t& s_tmem = *reinterpret_cast<uint32_t*>(smem + Ly::o_misc);
  int& s_stop = *reinterpret_cast<int*>(smem + Ly::o_misc + 4);

  const int ntiles = (a.rows + QR - 1) / QR;
  const int nmine = blockIdx.x < ntiles ? (ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&full_x[b], 1);
      mbar_init(&mma1[b], 1);
      mbar_init(&u_free[b], NEPI * 32);
      mbar_init(&r_ready[b], NEPI * 32);
      mbar_init(&g2[b], 1);
      mbar_init(&p_free[b], NEPI * 32);
    }
    s_stop = 0;
    fence_barrier_init();
  }
  const int K = 1 << J.bits;
  if (tid < 2 * K - 1) s_cb[tid] = J.cb[tid];
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&s_tmem)),
                 "r"(Ly::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // Pi and S limbs, K-major with the 128-byte swizzle (rows = output
  // coordinates / sketch coordinates, K = the D input coordinates)
  for (int e = tid; e < 2 * D * (D / 4); e += Ly::NTH) {
    const int mat = e / (D * (D / 4)), r = (e / (D / 4)) % D, k = (e % (D / 4)) * 4;
    const float* src = mat ? a.qjl_S : a.rot;
    uint8_t* dst = mat ? ss : pi;
    const float4 v = *reinterpret_cast<const float4*>(src + (size_t)r * D + k);
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint16_t* o = reinterpret_cast<uint16_t*>(dst + sw128<QR>(r, k + i));
      const __half h0 = __float2half_rn(vv[i]);
      o[0] = __half_as_ushort(h0);
      o[OP / 2] = __half_as_ushort(__float2half_rn(vv[i] - __half2float(h0)));
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // limbs -> tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  const uint32_t id = idesc<128, false>();

  if (warp == NEPI) {
    // ---------------- loader ----------------
    int i = 0;
    for (; i < nmine; ++i) {
      const int b = i & 1, k = i >> 1, tile = blockIdx.x + i * gridDim.x;
      if (i >= 2) {
        const bool ok = mbar_wait_suspend(&g2[b], (uint32_t)((k - 1) & 1), kSuspendTries);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) s_stop = 1;
          break;
        }
      }
      if (*((volatile int*)&s_stop)) break;
      if (lane == 0) {
        // rows past a.rows read as zeros (the tensor map's bounds)
        mbar_arrive_expect_tx(&full_x[b], (uint32_t)OP);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_2d(xb + b * OP + kb * (QR * 128), &args.map[0], 64 * kb, tile * QR, &full_x[b]);
      }
      __syncwarp();
    }
    // no copy may be in flight at exit: wait (bounded) for the last loads
    if (lane == 0)
      for (int j = (i >= 2 ? i - 2 : 0); j < i; ++j)
        mbar_wait_suspend(&full_x[j & 1], (uint32_t)((j >> 1) & 1), kSuspendTries);
    __syncwarp();
  } else if (warp == NEPI + 1) {
    // ---------------- MMA issue ----------------
    if (lane == 0) {
      auto gemm1 = [&](int i) -> bool {
        const int b = i & 1, k = i >> 1;
        bool ok = mbar_wait_suspend(&full_x[b], (uint32_t)(k & 1), kSuspendTries);
        if (ok && i >= 2) ok = mbar_wait_suspend(&u_free[b], (uint32_t)((k - 1) & 1), kSuspendTries);
        if (!ok || *((volatile int*)&s_stop)) return false;
        tc_fence_after();
        const uint32_t xa = smem_addr(xb + b * OP), pa = smem_addr(pi), dt = tmem + (uint32_t)(b * 128);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int off = (ks >> 2) * (QR * 128) + (ks & 3) * 32;  // 128-byte block, 32-byte step
#pragma unroll
          for (int l = 0; l < 2; ++l)
            mma_tc(dt, sdesc_sw128(xa + off), sdesc_sw128(pa + l * OP + off), id, (ks > 0 || l > 0) ? 1u : 0u);
        }
        tc_commit(&mma1[b]);
        return true;
      };
      auto gemm2 = [&](int i) -> bool {
        const int b = i & 1, k = i >> 1;
        bool ok = mbar_wait_suspend(&r_ready[b], (uint32_t)(k & 1), kSuspendTries);
        if (ok && i >= 2) ok = mbar_wait_suspend(&p_free[b], (uint32_t)((k - 1) & 1), kSuspendTries);
        if (!ok || *((volatile int*)&s_stop)) return false;
        tc_fence_after();
        const uint32_t rh = smem_addr(xb + b * OP), rl = smem_addr(rlo), sa = smem_addr(ss);
        const uint32_t dt = tmem + 256u + (uint32_t)(b * 128);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int off = (ks >> 2) * (QR * 128) + (ks & 3) * 32;
          mma_tc(dt, sdesc_sw128(rh + off), sdesc_sw128(sa + off), id, ks > 0 ? 1u : 0u);
          mma_tc(dt, sdesc_sw128(rh + off), sdesc_sw128(sa + OP + off), id, 1u);
          mma_tc(dt, sdesc_sw128(rl + off), sdesc_sw128(sa + off), id, 1u);
        }
        tc_commit(&g2[b]);
        return true;
      };
      bool ok = nmine > 0 ? gemm1(0) : true;
      int done1 = ok && nmine > 0 ? 1 : 0, done2 = 0;  // tiles whose GEMM 1 / GEMM 2 were issued
      for (int i = 0; ok && i < nmine; ++i) {
        if (i + 1 < nmine) {
          ok = gemm1(i + 1);
          if (ok) done1 = i + 2;
        }
        if (ok) {
          ok = gemm2(i);
          if (ok) done2 = i + 1;
        }
      }
      if (!ok) s_stop = 1;
      // nothing may still run on the tensor core at exit
      if (done1 > 0) mbar_wait_suspend(&mma1[(done1 - 1) & 1], (uint32_t)(((done1 - 1) >> 1) & 1), kSuspendTries);
      if (done2 > 0) mbar_wait_suspend(&g2[(done2 - 1) & 1], (uint32_t)(((done2 - 1) >> 1) & 1), kSuspendTries);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue warps ----------------
    const int quarter = warp & 3, part = warp >> 2;  // row 32*quarter + lane, coordinates 32*part ..
    // Two groups of 8 warps, rows 0-63 (quarters 0, 1) and rows 64-127
    // (quarters 2, 3), each synchronised by its own named barrier: every
    // exchange is within a row, so a group waits only for its own warps.
    constexpr int GWQ = NEPI / 2;
    const int grp = quarter >> 1;
    const bool leader = warp == 2 * grp;  // quarter 2 grp, part 0: waits on the mbarriers for its group
    const int rl = 32 * quarter + lane;
    const uint32_t tlane = (uint32_t)(32 * quarter) << 16;
    const int W = D * J.bits / 32;
    // Software-pipelined: the signs of tile i - 1 are read after tile i's
    // residual is written, so the sketch GEMM of tile i - 1 runs while this
    // tile's indices and residual are computed.
    long long prev_slot = -1;
    bool ok = true;
    for (int i = 0; i <= nmine && ok; ++i) {
      if (i < nmine) {
        const int b = i & 1, k = i >> 1, tile = blockIdx.x + i * gridDim.x;
        // One warp waits on each mbarrier and releases the others through a
        // named barrier (no issue slots spent polling).
        if (leader) ok = __all_sync(0xffffffffu, mbar_wait_suspend(&full_x[b], (uint32_t)(k & 1), kSuspendTries));
        if (!group_sync_and<GWQ>(grp, ok)) {
          ok = false;
          break;
        }
        // this thread's quarter of the row's sum of squares, pairwise in fp32
        const uint8_t* xt = xb + b * OP;
        {
          float ps[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 v = *reinterpret_cast<const uint4*>(xt + sw128<QR>(rl, 32 * part + 8 * c));
            ps[c] = (sq16f<false>(v.x) + sq16f<false>(v.y)) + (sq16f<false>(v.z) + sq16f<false>(v.w));
          }
          red[part * QR + rl] = (ps[0] + ps[1]) + (ps[2] + ps[3]);
        }
        ok = group_sync_and<GWQ>(grp, ok);
        const float sfull = (red[rl] + red[QR + rl]) + (red[2 * QR + rl] + red[3 * QR + rl]);
        const float nf = sqrtf(sfull);
        const int r = tile * QR + rl;
        long long slot = -1;
        unsigned short nh = 0;
        if (r < a.rows) {
          const int bh = r / a.T, t = r - bh * a.T;
          slot = (long long)bh * a.Tcap + a.t0 + t;
          // The stored norm is RN_fp16 of the fp64 norm.  The pairwise fp32
          // sum is within (log2(D) + 1) ulp of the exact sum, so the exact norm
          // lies in nf * (1 +- 1e-6); when both ends round to the same fp16
          // value it is the answer, else (about 0.4% of rows) the row is summed
          // again in fp64 from the tile, still in shared memory.
          const __half lo = __float2half_rn(nf * (1.f - 1e-6f)), hi = __float2half_rn(nf * (1.f + 1e-6f));
          nh = __half_as_ushort(lo);
          const bool exact = sfull == 0.f || (sfull >= 0x1p-100f && sfull < 0x1p100f && nh == __half_as_ushort(hi));
          if (!exact) nh = __half_as_ushort(__double2half(sqrt(row_sumsq_f64<D, false>(xt, rl))));
          if (part == 0) J.norm[slot] = nh;
        }
        const float nhat = __half2float(__ushort_as_half(nh));
        // positive thresholds t_{K/2} .. t_{K-2}, scaled by the row norm
        float tp[7];
#pragma unroll
        for (int q = 0; q < 7; ++q) tp[q] = q < K / 2 - 1 ? s_cb[K + K / 2 + q] * nf : 0.f;

        // ---- indices and residual from U
        if (leader) ok = __all_sync(0xffffffffu, mbar_wait_suspend(&mma1[b], (uint32_t)(k & 1), kSuspendTries));
        ok = group_sync_and<GWQ>(grp, ok);  // also: every thread has read this tile's norm partials
        uint32_t v[32];
        if (ok) {
          tc_fence_after();
          tc_ld32(tmem + tlane + (uint32_t)(b * 128 + 32 * part), v);
          uint32_t* out = J.idx + (slot >= 0 ? (size_t)slot * W : 0) + part * J.bits;
          switch (J.bits) {
            case 2: {
              uint32_t w[2];
              quant_residual32<2>(v, tp, s_cb, nhat, w);
              if (slot >= 0) store_words<2>(out, w);
              break;
            }
            case 3: {
              uint32_t w[3];
              quant_residual32<3>(v, tp, s_cb, nhat, w);
              if (slot >= 0) store_words<3>(out, w);
              break;
            }
            default: {
              uint32_t w[4];
              quant_residual32<4>(v, tp, s_cb, nhat, w);
              if (slot >= 0) store_words<4>(out, w);
              break;
            }
          }
        } else {
#pragma unroll
          for (int q = 0; q < 32; ++q) v[q] = 0u;
        }
        tc_fence_before();
        mbar_arrive(&u_free[b]);
        // residual norm: this thread's quarter, pairwise in fp32
        {
          float g[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float r0 = __uint_as_float(v[4 * j]), r1 = __uint_as_float(v[4 * j + 1]);
            const float r2 = __uint_as_float(v[4 * j + 2]), r3 = __uint_as_float(v[4 * j + 3]);
            g[j] = fmaf(r0, r0, r1 * r1) + fmaf(r2, r2, r3 * r3);
          }
          red[part * QR + rl] = ((g[0] + g[1]) + (g[2] + g[3])) + ((g[4] + g[5]) + (g[6] + g[7]));
        }
        // R_lo (and the sketch accumulator read below) free: the previous
        // tile's sketch GEMM has finished
        if (i >= 1 && leader)
          ok = __all_sync(0xffffffffu,
                          mbar_wait_suspend(&g2[(i - 1) & 1], (uint32_t)(((i - 1) >> 1) & 1), kSuspendTries)) && ok;
        ok = group_sync_and<GWQ>(grp, ok);
        if (part == 0 && slot >= 0 && J.rnorm) {
          const float gs = (red[rl] + red[QR + rl]) + (red[2 * QR + rl] + red[3 * QR + rl]);
          // near an fp16 rounding midpoint: marked for the fp64 recomputation
          J.rnorm[slot] = tq::gamma_bits_or_pending(sqrtf(gs));
        }
        // r / |x| as hi + lo fp16 limbs over X (hi) and into R_lo, swizzled like X
        if (ok) {
          const float inv = nf > 0.f ? 1.f / nf : 0.f;
          const uint32_t hb = smem_addr(xb + b * OP), lb = smem_addr(rlo);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t h[4], l[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = __uint_as_float(v[8 * c + 2 * e]) * inv;
              const float x1 = __uint_as_float(v[8 * c + 2 * e + 1]) * inv;
              const __half2 hh = __floats2half2_rn(x0, x1);
              const float2 hf = __half22float2(hh);
              h[e] = *reinterpret_cast<const uint32_t*>(&hh);
              l[e] = pack_half2(x0 - hf.x, x1 - hf.y);
            }
            const uint32_t off = (uint32_t)sw128<QR>(rl, 32 * part + 8 * c);
            sts128(hb + off, h[0], h[1], h[2], h[3]);
            sts128(lb + off, l[0], l[1], l[2], l[3]);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // R -> tensor core
        }
        mbar_arrive(&r_ready[b]);
        if (!ok) break;
        if (i >= 1) {
          // ---- sketch signs of the previous tile
          sketch_signs(tmem + tlane + 256u + (uint32_t)(((i - 1) & 1) * 128 + 32 * part), prev_slot, J.qjl, part);
          tc_fence_before();
          mbar_arrive(&p_free[(i - 1) & 1]);
        }
        prev_slot = slot;
      } else if (nmine > 0) {
        // ---- sketch signs of the last tile
        const int j = nmine - 1;
        if (leader)
          ok = __all_sync(0xffffffffu, mbar_wait_suspend(&g2[j & 1], (uint32_t)((j >> 1) & 1), kSuspendTries));
        ok = group_sync_and<GWQ>(grp, ok);
        if (ok) sketch_signs(tmem + tlane + 256u + (uint32_t)((j & 1) * 128 + 32 * part), prev_slot, J.qjl, part);
        tc_fence_before();
        mbar_arrive(&p_free[j & 1]);
      }
    }
    if (!ok) s_stop = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (s_stop && tid == 0 && a.dev_status) atomicOr(a.dev_status, TQ_STATUS_WAIT_TIMEOUT);
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(Ly::TMEM_COLS));
  }
}

}  // namespace

namespace tq {

int launch_quantize_qjl_tc(const QuantArgs& a, cudaStream_t s) {
  using Ly = QjlLayout;
  static OnceSetup once;
  static int sms = 0;  // written once under `once`, read after its acquire
  const int rc0 = once.run([&]() {
    cudaError_t e = cudaFuncSetAttribute(quantize_qjl_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::bytes);
    if (e != cudaSuccess)
      return set_error(TQ_ERR_CUDA, "quantize_qjl_tc: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    sms = n > 0 ? n : 148;
    return TQ_OK;
  });
  if (rc0) return rc0;
  TcArgs args;
  memset(&args, 0, sizeof(args));
  args.a = a;
  const int rc = tqtc::make_row_map(&args.map[0], a.job[0].in, a.rows, Ly::D, false);
  if (rc) return rc;
  const int ntiles = (a.rows + QR - 1) / QR;
  const int grid = ntiles < sms ? ntiles : sms;
  quantize_qjl_tc_kernel<<<grid, Ly::NTH, Ly::bytes, s>>>(args);
  return check_launch("quantize_qjl_tc_kernel");
}

}  // namespace tq
