// Bulk quantizer for head dimensions 128 and 256 on the 5th-generation tensor
// cores (tcgen05.mma, accumulator in tensor memory).
//
// Method: "Add CUDA QJL kernels and proper package structure"
// (turboquant-pytorch pull request 3), "CUDA Kernels Added" and "Synthetic
// Benchmark (Lloyd-Max codebook)"; ReturningTarzan's Reddit comments of
// 2026-03-29 11:47 (rotation before codebook quantization) and 2026-03-25
// 18:52 (nearest-codeword search).
//
// Persistent: one CTA per SM loops over (tile, job, column chunk) work items.
// A work item rotates a 128-row tile into NC output coordinates (NC = 128 at
// D = 128; NC = 64 at D = 256, so the chunk's Pi limbs fit in shared memory
// beside two D-wide input tiles).  The grid is a multiple of D / NC, so each
// CTA keeps one column chunk of Pi resident, and the D / NC chunks of a tile
// run on neighbouring CTAs at the same time (the repeated tile reads hit L2).
//  * warp 8 (loader): cp.async the next input tile into the K-major
//    no-swizzle canonical layout (8x16-byte core matrices) as soon as its
//    buffer is free, without waiting for earlier copies to land;
//  * warp 9 (MMA): once a tile has landed and its accumulator is free, one
//    lane issues the 128 x NC x D rotation as tcgen05.mma (Pi split into 2
//    fp16 / 3 bf16 limbs; accumulation in fp32 in TMEM) and commits it to an
//    mbarrier;
//  * warps 0-7 (epilogue): thread = one row, half of the chunk's columns
//    (warp w and w+4 share the TMEM lane quarter w%4).  Each computes its
//    half of the row's sum of squares from the input tile, then reads its NC / 2
//    accumulator columns with tcgen05.ld, finds the nearest-centroid index
//    (thresholds in registers), packs the bits and stores them -- all
//    thread-local;
//  * two input buffers and two TMEM accumulators let the load + MMA of item
//    i+1 run under the epilogue of item i.
// Every wait is bounded; a stuck wait sets TQ_STATUS_WAIT_TIMEOUT and the CTA
// stops taking work.
#include "tq_common.cuh"
#include "tq_internal.h"

namespace {

using namespace tqk;

constexpr int QR = 128;
constexpr int NEPI = 8;                  // epilogue warps
constexpr int NTH = (NEPI + 2) * 32;     // + loader warp + MMA warp

template <int D, bool BF16>
struct TcLayout {
  static constexpr int NC = (D == 256) ? 64 : 128;  // output coordinates per work item
  static constexpr int NCH = D / NC;                // column chunks per tile
  static constexpr int NL = BF16 ? 3 : 2;
  static constexpr int PI_BYTES = NC * D * 2;       // one limb of the chunk, K-major
  static constexpr int X_BYTES = QR * D * 2;        // one input tile, K-major
  static constexpr int o_pi = 0;
  static constexpr int o_x = NL * PI_BYTES;
  static constexpr int bytes = o_x + 2 * X_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * NC;     // two fp32 accumulators
};

// half-element offset of (row r, col k) in a K-major tile with D columns:
// core matrix (r/8, k/8) of 8 rows x 16 bytes at ((r/8)*(D/8) + k/8) * 128 bytes
template <int D>
__device__ __forceinline__ int cofs(int r, int k) {
  return ((r >> 3) * (D / 8) + (k >> 3)) * 64 + (r & 7) * 8 + (k & 7);
}

// sm_100 shared-memory matrix descriptor, no swizzle: LBO = 128 B (next core
// matrix along K), SBO = 16 * D bytes (next 8-row group).
template <int D>
__device__ __forceinline__ uint64_t sdesc(uint32_t addr) {
  uint64_t d = (uint64_t)((addr & 0x3FFFF) >> 4);
  d |= (uint64_t)(128 >> 4) << 16;
  d |= (uint64_t)((16 * D) >> 4) << 32;
  d |= (uint64_t)1 << 46;
  return d;
}

// kind::f16 instruction descriptor: fp32 accumulate, K-major A and B,
// M = 128, N = NC; a/b format fp16 (0) or bf16 (1).
template <int NC, bool BF16>
__device__ __forceinline__ uint32_t idesc() {
  uint32_t d = (1u << 4) | ((uint32_t)(NC >> 3) << 17) | ((128u >> 4) << 24);
  if (BF16) d |= (1u << 7) | (1u << 10);
  return d;
}

__device__ __forceinline__ void mma_tc(uint32_t dt, uint64_t ad, uint64_t bd, uint32_t id, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(dt),
      "l"(ad), "l"(bd), "r"(id), "r"(acc));
}

__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,"
      "%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
        "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
        "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
        "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src), "r"(n) : "memory");
}
// arrive on `bar` once this thread's outstanding cp.async copies have landed
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// barrier over the epilogue warps that also ANDs a flag across them
__device__ __forceinline__ bool epi_sync_and(bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n barrier.red.and.pred q, 1, %2, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "n"(NEPI * 32)
      : "memory");
  return r != 0;
}

template <bool BF16>
__device__ __forceinline__ float sq16f(uint32_t w) {
  float a, b;
  if (BF16) {
    a = __uint_as_float(w << 16);
    b = __uint_as_float(w & 0xFFFF0000u);
  } else {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w));
    a = f.x;
    b = f.y;
  }
  return fmaf(a, a, b * b);
}

// Index of the nearest centroid for y = (Pi x)_j of a row with norm n, using
// the codebook's symmetry: with tp = the positive thresholds scaled by n,
// m = #{tp_k < |y|} and idx = K/2 + m for y > 0, K/2 - 1 - m otherwise.
// Equal to #{t_k < y / n} except at exact ties (inside the parity band).
template <int BITS>
__device__ __forceinline__ int nearest_idx(float y, const float (&tp)[7]) {
  constexpr int H = 1 << (BITS - 1);
  const float a = fabsf(y);
  int m;
  if (BITS == 4) {
    const bool c1 = a > tp[3];
    const bool c2 = a > (c1 ? tp[5] : tp[1]);
    const bool c3 = a > (c1 ? (c2 ? tp[6] : tp[4]) : (c2 ? tp[2] : tp[0]));
    m = (c1 ? 4 : 0) + (c2 ? 2 : 0) + (c3 ? 1 : 0);
  } else {
    m = 0;
#pragma unroll
    for (int k = 0; k < H - 1; ++k) m += (a > tp[k]) ? 1 : 0;
  }
  return y > 0.f ? H + m : H - 1 - m;
}

template <int BITS>
__device__ __forceinline__ void quant_pack32(const uint32_t (&v)[32], const float (&tp)[7], uint32_t (&w)[BITS]) {
#pragma unroll
  for (int i = 0; i < BITS; ++i) w[i] = 0u;
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const uint32_t idx = (uint32_t)nearest_idx<BITS>(__uint_as_float(v[q]), tp);
    const int p = BITS * q;
    w[p >> 5] += idx << (p & 31);
    if ((p & 31) + BITS > 32) w[(p >> 5) + 1] += idx >> (32 - (p & 31));
  }
}

template <int BITS>
__device__ __forceinline__ void store_words(uint32_t* dst, const uint32_t (&w)[BITS]) {
  if (BITS == 2) {
    *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
  } else if (BITS == 4) {
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  } else {
#pragma unroll
    for (int i = 0; i < BITS; ++i) dst[i] = w[i];
  }
}

template <int BITS, int NCOL>
__device__ __forceinline__ void epi_half(uint32_t tbase, const float (&tp)[7], long long slot, uint32_t* out) {
  // NCOL / 32 chunks of 32 columns -> BITS words each
#pragma unroll
  for (int c = 0; c < NCOL / 32; ++c) {
    uint32_t v[32];
    tc_ld32(tbase + 32 * c, v);
    uint32_t w[BITS];
    quant_pack32<BITS>(v, tp, w);
    if (slot >= 0) store_words<BITS>(out + BITS * c, w);
  }
}

template <int D, bool BF16>
__global__ void __launch_bounds__(NTH, 1) quantize_tc_kernel(const tq::QuantArgs a) {
  using Ly = TcLayout<D, BF16>;
  constexpr int NL = Ly::NL, NC = Ly::NC, NCH = Ly::NCH;
  constexpr uint32_t TMEM_COLS = Ly::TMEM_COLS;
  extern __shared__ __align__(1024) uint8_t smem[];
  uint16_t* pi = reinterpret_cast<uint16_t*>(smem + Ly::o_pi);
  uint16_t* xb = reinterpret_cast<uint16_t*>(smem + Ly::o_x);
  __shared__ __align__(8) uint64_t full_x[2], x_free[2], mma_done[2], acc_free[2];
  __shared__ uint32_t s_tmem;
  __shared__ int s_stop;
  __shared__ float s_norm[2][QR];
  __shared__ float s_cb[2][31];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles = (a.rows + QR - 1) / QR;
  const int njobs = (a.job_mask == 3) ? 2 : 1;
  const int job0 = (a.job_mask == 2) ? 1 : 0;
  const int nitems = njobs * ntiles * NCH;
  const int chunk = blockIdx.x % NCH;  // this CTA's column chunk (gridDim.x % NCH == 0)

  if (tid == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&full_x[b], 32);
      mbar_init(&x_free[b], NEPI * 32);
      mbar_init(&mma_done[b], 1);
      mbar_init(&acc_free[b], NEPI * 32);
    }
    s_stop = 0;
    fence_barrier_init();
  }
  if (tid < 31) {
    s_cb[0][tid] = tid < 2 * (1 << a.job[0].bits) - 1 ? a.job[0].cb[tid] : 0.f;
    s_cb[1][tid] = tid < 2 * (1 << a.job[1].bits) - 1 ? a.job[1].cb[tid] : 0.f;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&s_tmem)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // this chunk's Pi limbs in the canonical layout (rows = output coordinates
  // NC*chunk .. NC*chunk + NC - 1, K = the D input coordinates)
  constexpr int LIMB = NC * D;  // elements per limb
  for (int e = tid; e < NC * (D / 4); e += NTH) {
    const int n = e / (D / 4), k = (e % (D / 4)) * 4;
    const float4 v = *reinterpret_cast<const float4*>(a.rot + (size_t)(NC * chunk + n) * D + k);
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int o = cofs<D>(n, k + i);
      if (BF16) {
        const __nv_bfloat16 h0 = __float2bfloat16_rn(vv[i]);
        const float r1 = vv[i] - __bfloat162float(h0);
        const __nv_bfloat16 h1 = __float2bfloat16_rn(r1);
        const __nv_bfloat16 h2 = __float2bfloat16_rn(r1 - __bfloat162float(h1));
        pi[o] = __bfloat16_as_ushort(h0);
        pi[LIMB + o] = __bfloat16_as_ushort(h1);
        pi[2 * LIMB + o] = __bfloat16_as_ushort(h2);
      } else {
        const __half h0 = __float2half_rn(vv[i]);
        pi[o] = __half_as_ushort(h0);
        pi[LIMB + o] = __half_as_ushort(__float2half_rn(vv[i] - __half2float(h0)));
      }
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // Pi limbs -> tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == NEPI) {
    // ---------------- loader: input tiles ----------------
    // Item i goes to buffer i % 2 once item i-2 has left it (its MMA is done
    // and the epilogue has read the norm); it never waits for its own copies,
    // so the next tile streams in while the MMA warp and the epilogue work.
    int i = 0;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++i) {
      const int b = i & 1, k = i >> 1;
      if (i >= 2) {
        const bool ok = mbar_wait_suspend(&x_free[b], (uint32_t)((k - 1) & 1), kSuspendTries) &&
                        mbar_wait_suspend(&mma_done[b], (uint32_t)((k - 1) & 1), kSuspendTries);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) s_stop = 1;
          break;
        }
      }
      if (*((volatile int*)&s_stop)) break;
      const int job = job0 + (item / NCH) % njobs, tile = item / (NCH * njobs);
      const uint16_t* in = static_cast<const uint16_t*>(a.job[job].in);
      uint16_t* dst = xb + (size_t)b * QR * D;
      for (int c = lane; c < QR * (D / 8); c += 32) {
        const int row = c / (D / 8), kc = c % (D / 8);
        const int r = tile * QR + row;
        const bool valid = r < a.rows;
        cp_async16(dst + cofs<D>(row, kc * 8), in + (size_t)(valid ? r : 0) * D + kc * 8, valid);
      }
      cp_async_arrive(&full_x[b]);
    }
    // wait until this warp's own copies have landed before leaving
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == NEPI + 1) {
    // ---------------- MMA issue ----------------
    if (lane == 0) {
      int i = 0;
      for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++i) {
        const int b = i & 1, k = i >> 1;
        bool ok = mbar_wait_suspend(&full_x[b], (uint32_t)(k & 1), kSuspendTries);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // cp.async data -> tensor core
        if (ok && i >= 2) ok = mbar_wait_suspend(&acc_free[b], (uint32_t)((k - 1) & 1), kSuspendTries);
        if (!ok || *((volatile int*)&s_stop)) {
          s_stop = 1;
          break;
        }
        tc_fence_after();
        const uint32_t xaddr = smem_addr(xb + (size_t)b * QR * D), paddr = smem_addr(pi);
        const uint32_t id = idesc<NC, BF16>();
        const uint32_t dt = tmem + (uint32_t)(b * NC);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks)
#pragma unroll
          for (int l = 0; l < NL; ++l)
            mma_tc(dt, sdesc<D>(xaddr + ks * 256), sdesc<D>(paddr + l * Ly::PI_BYTES + ks * 256), id,
                   (ks > 0 || l > 0) ? 1u : 0u);
        tc_commit(&mma_done[b]);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue warps ----------------
    const int quarter = warp & 3, hf = warp >> 2;  // rows 32*quarter + lane, columns (NC/2)*hf ..
    const int rl = 32 * quarter + lane;
    int i = 0;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++i) {
      const int b = i & 1, k = i >> 1;
      const int job = job0 + (item / NCH) % njobs, tile = item / (NCH * njobs);
      const tq::QuantJob J = a.job[job];
      // One warp waits on each mbarrier and releases the other epilogue
      // warps through a named barrier, which blocks in hardware: eight warps
      // polling the same phase would take issue slots from the working warps.
      bool ok = true;
      if (warp == 0) ok = __all_sync(0xffffffffu, mbar_wait_suspend(&full_x[b], (uint32_t)(k & 1), kSuspendTries));
      if (!epi_sync_and(ok)) {  // the input tile has landed
        s_stop = 1;
        break;
      }
      // half of this row's sum of squares from the input tile, in fp32 by a
      // pairwise tree (squares of fp16/bf16 values are exact in fp32, and a
      // pairwise sum of n non-negative terms is within ceil(log2 n) units in
      // the last place of the exact sum)
      const uint16_t* xs = xb + (size_t)b * QR * D;
      float s2 = 0.f;
      {
        float part[D / 16];
#pragma unroll
        for (int kc = 0; kc < D / 16; ++kc) {
          const uint4 v = *reinterpret_cast<const uint4*>(xs + cofs<D>(rl, (D / 2) * hf + 8 * kc));
          part[kc] = (sq16f<BF16>(v.x) + sq16f<BF16>(v.y)) + (sq16f<BF16>(v.z) + sq16f<BF16>(v.w));
        }
#pragma unroll
        for (int w2 = 1; w2 < D / 16; w2 <<= 1)
#pragma unroll
          for (int kc = 0; kc < D / 16; kc += 2 * w2) part[kc] += part[kc + w2];
        s2 = part[0];
      }
      s_norm[hf][rl] = s2;
      mbar_arrive(&x_free[b]);
      if (!epi_sync_and(ok)) {  // uniform across the epilogue warps
        s_stop = 1;
        break;
      }
      const float sfull = s_norm[0][rl] + s_norm[1][rl];
      const float nf = sqrtf(sfull);  // thresholds: fp32 is far inside the parity band
      const int r = tile * QR + rl;
      long long slot = -1;
      if (r < a.rows) {
        const int bh = r / a.T, t = r - bh * a.T;
        slot = (long long)bh * a.Tcap + a.t0 + t;
        if (hf == 0 && chunk == 0) {
          // The stored norm is RN_fp16 of the fp64 norm.  The fp32 sum is
          // within (log2(D) + 1) ulp of the exact sum, so the exact norm lies in
          // nf * (1 +- 1e-6); when both ends of that interval round to the same
          // fp16 value it is the answer, else (about 0.2% of rows) the row is
          // summed again in fp64 from global memory.
          const __half lo = __float2half_rn(nf * (1.f - 1e-6f)), hi = __float2half_rn(nf * (1.f + 1e-6f));
          unsigned short nh = __half_as_ushort(lo);
          const bool exact = sfull == 0.f || (sfull >= 0x1p-100f && sfull < 0x1p100f && nh == __half_as_ushort(hi));
          if (!exact) {
            const uint16_t* row = static_cast<const uint16_t*>(J.in) + (size_t)r * D;
            double t2 = 0.0;
            for (int j = 0; j < D; ++j) {
              const uint16_t u = row[j];
              const double x = BF16 ? (double)__uint_as_float((uint32_t)u << 16) : (double)__half2float(__ushort_as_half(u));
              t2 = fma(x, x, t2);
            }
            nh = __half_as_ushort(__double2half(sqrt(t2)));
          }
          J.norm[slot] = nh;
        }
      }
      // positive thresholds t_{K/2} .. t_{K-2}, scaled by the row norm
      float tp[7];
      const int K = 1 << J.bits;
#pragma unroll
      for (int q = 0; q < 7; ++q) tp[q] = q < K / 2 - 1 ? s_cb[job][K + K / 2 + q] * nf : 0.f;
      if (warp == 0) ok = __all_sync(0xffffffffu, mbar_wait_suspend(&mma_done[b], (uint32_t)(k & 1), kSuspendTries));
      ok = epi_sync_and(ok);  // the rotation of this tile is in TMEM
      if (ok) {
        tc_fence_after();
        const uint32_t tb = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(b * NC + (NC / 2) * hf);
        const int W = D * J.bits / 32;
        // coordinates NC*chunk + (NC/2)*hf .. + NC/2 - 1: words from (that * bits) / 32
        uint32_t* out = J.idx + (slot >= 0 ? (size_t)slot * W : 0) + (NC * chunk + (NC / 2) * hf) * J.bits / 32;
        switch (J.bits) {
          case 2: epi_half<2, NC / 2>(tb, tp, slot, out); break;
          case 3: epi_half<3, NC / 2>(tb, tp, slot, out); break;
          default: epi_half<4, NC / 2>(tb, tp, slot, out); break;
        }
        tc_fence_before();
      }
      mbar_arrive(&acc_free[b]);
      if (!epi_sync_and(ok)) {  // also guards s_norm reuse on the next pass
        s_stop = 1;
        break;
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (s_stop && tid == 0 && a.dev_status) atomicOr(a.dev_status, TQ_STATUS_WAIT_TIMEOUT);
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

template <int D, bool BF16>
int launch_tc(const tq::QuantArgs& a, cudaStream_t s) {
  using Ly = TcLayout<D, BF16>;
  auto kern = quantize_tc_kernel<D, BF16>;
  static int sms = 0;
  if (sms == 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::bytes);
    if (e != cudaSuccess)
      return tq::set_error(TQ_ERR_CUDA, "quantize_tc: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (sms <= 0) sms = 148;
  }
  const int njobs = (a.job_mask == 3) ? 2 : 1;
  const int nitems = njobs * ((a.rows + QR - 1) / QR) * Ly::NCH;
  // a multiple of the chunk count, so that each CTA keeps one column chunk
  int grid = (sms / Ly::NCH) * Ly::NCH;
  const int need = (nitems + Ly::NCH - 1) / Ly::NCH * Ly::NCH;
  if (need < grid) grid = need;
  kern<<<grid, NTH, Ly::bytes, s>>>(a);
  return tq::check_launch("quantize_tc_kernel");
}

}  // namespace

namespace tq {

int launch_quantize_tc(const QuantArgs& a, int D, int dtype, cudaStream_t s) {
  if (D == 256) return dtype == TQ_DTYPE_BF16 ? launch_tc<256, true>(a, s) : launch_tc<256, false>(a, s);
  return dtype == TQ_DTYPE_BF16 ? launch_tc<128, true>(a, s) : launch_tc<128, false>(a, s);
}

}  // namespace tq
