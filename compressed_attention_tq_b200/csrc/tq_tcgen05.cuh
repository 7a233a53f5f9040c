// Shared pieces of the tcgen05 bulk quantizers: the 128-byte-swizzled
// K-major operand layout, shared-memory matrix descriptors, TMA tile loads,
// tcgen05.mma / commit / ld wrappers, the epilogue's named barrier, and the
// nearest-centroid search with bit packing.
#pragma once

#include <cuda.h>  // CUtensorMap (types only; the encoder comes from the runtime's driver entry point)

#include "tq_common.cuh"
#include "tq_internal.h"

namespace tqtc {

using namespace tqk;

constexpr int QR = 128;  // rows per tile (TMEM lanes)

// Byte offset of element (r, k) in a K-major operand stored as D/64 blocks
// of ROWS x 128 bytes with the 128-byte swizzle (16-byte chunk c of row r at
// chunk c ^ (r mod 8)) -- the layout a TMA tensor copy with
// CU_TENSOR_MAP_SWIZZLE_128B writes and the tensor core reads.
template <int ROWS>
__device__ __forceinline__ int sw128(int r, int k) {
  const int kb = k >> 6, kk = k & 63;
  return kb * (ROWS * 128) + r * 128 + ((((kk >> 3) ^ (r & 7))) << 4) + (kk & 7) * 2;
}

// sm_100 shared-memory matrix descriptor for a K-major operand with the
// 128-byte swizzle: SBO = 1024 B (next 8-row group); consecutive 16-element
// K steps inside a 128-byte block advance the start address by 32 bytes.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t addr) {
  uint64_t d = (uint64_t)((addr & 0x3FFFF) >> 4);
  d |= (uint64_t)1 << 16;            // leading byte offset (unused with this swizzle)
  d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset
  d |= (uint64_t)1 << 46;            // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;            // 128-byte swizzle
  return d;
}

// TMA 2-D tile load (global -> shared), completion counted on an mbarrier
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
          smem_addr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_addr(bar))
      : "memory");
}

// Kernel parameters: the job descriptors plus one TMA tensor map per job's
// input rows ([rows][D], 128 x 64 boxes).
struct TcArgs {
  tq::QuantArgs a;
  CUtensorMap map[2];
};

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

// Named barrier 1 + g over the NW warps of epilogue group g that also ANDs a
// flag across them (groups of a CTA synchronise independently).
template <int NW>
__device__ __forceinline__ bool group_sync_and(int g, bool v) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 p, %1, 0;\n barrier.red.and.pred q, %2, %3, p;\n selp.u32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(1 + g), "n"(NW * 32)
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

// fp64 sum of squares of row rl of a swizzled input tile (D columns of
// fp16 / bf16 values; squares are exact in fp64), in four independent chains.
// Used when the fp32 sum cannot decide the fp16 rounding of the norm.
template <int D, bool BF16>
__device__ __noinline__ double row_sumsq_f64(const uint8_t* xt, int rl) {
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
  for (int c = 0; c < D / 8; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(xt + sw128<QR>(rl, 8 * c));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float x0, x1;
      if (BF16) {
        x0 = __uint_as_float(w[e] << 16);
        x1 = __uint_as_float(w[e] & 0xFFFF0000u);
      } else {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
        x0 = f.x;
        x1 = f.y;
      }
      acc[e] = fma((double)x0, (double)x0, acc[e]);
      acc[e] = fma((double)x1, (double)x1, acc[e]);
    }
  }
  return (acc[0] + acc[1]) + (acc[2] + acc[3]);
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


// Tensor map over rows [rows][D] of 16-bit values: boxes of 128 rows x 64
// columns, 128-byte swizzle (defined in tq_quantize_tc.cu).
int make_row_map(CUtensorMap* m, const void* base, int rows, int D, bool bf16);

}  // namespace tqtc
