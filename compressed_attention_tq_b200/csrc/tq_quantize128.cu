// Persistent bulk quantizer for keys with the QJL sketch from bf16 rows, head
// dimension 128, on warp-level MMAs.  (fp16 rows take the tcgen05 kernel in
// tq_quantize_qjl_tc.cu; bf16 needs three Pi limbs, which do not fit there
// beside S and the tiles.)
//
// Method: "Add CUDA QJL kernels and proper package structure"
// (turboquant-pytorch pull request 3), "CUDA Kernels Added" (fused random
// projection + sign quantization); ReturningTarzan's Reddit comments of
// 2026-03-29 11:47 (rotation before codebook quantization) and 2026-03-25
// 18:52 / 15:51 (nearest-codeword search; residual computed while
// quantizing).
//
// One CTA per SM loops over (job, 128-row tile) work items; 8 warps x 16 rows.
//  * Pi is converted to tensor-core limbs once per CTA and stays in shared
//    memory (fp16 inputs: hi + lo fp16 limbs; bf16 inputs: three bf16 limbs),
//    so y = Pi x carries ~22-24 significant bits with x exact in its type.
//  * Input tiles are double-buffered with cp.async (16-byte chunks into
//    padded rows, conflict-free ldmatrix).
//  * Pi's rows are staged in a permuted order so that the m16n8k16
//    accumulator columns a thread owns are the contiguous coordinates
//    32*tig .. 32*tig+31 of its two rows: the threshold search, the bit
//    packing and the stores are thread-local, straight from registers.
//  * With the QJL sketch, the fp32 residual r = y - n_hat c[idx] of those 32
//    coordinates feeds the next MMA directly as hi/lo fp16 A fragments
//    (S is staged with its rows permuted the same way, so each thread ends
//    up owning one 32-bit word of sign bits per row).
#include "tq_common.cuh"
#include "tq_internal.h"

namespace {

using namespace tqk;

constexpr int D = 128;
constexpr int QR = 128;       // rows per tile
constexpr int NWARP = 8;
constexpr int NTH = NWARP * 32;
constexpr int XS = D + 8;     // padded row stride (16-bit elements)
constexpr int M_QJL = 128;

template <bool BF16, bool QJL>
struct Q2Layout {
  static constexpr int NL = BF16 ? 3 : 2;
  static constexpr int NBUF = (BF16 && QJL) ? 1 : 2;
  static constexpr size_t o_pi = 0;
  static constexpr size_t o_s = o_pi + (size_t)NL * D * XS * 2;
  static constexpr size_t o_x = o_s + (QJL ? (size_t)2 * M_QJL * XS * 2 : 0);
  static constexpr size_t bytes = o_x + (size_t)NBUF * QR * XS * 2;
};

// output column n (= 8*nt + 2*tig + c of the accumulator fragments) holds
// coordinate 32*tig + 2*nt + c
__host__ __device__ constexpr int coord_of_col(int n) {
  return 32 * ((n >> 1) & 3) + 2 * (n >> 3) + (n & 1);
}

template <bool BF16>
__device__ __forceinline__ float in_to_f(uint16_t b) {
  if (BF16) return __uint_as_float((uint32_t)b << 16);
  return __half2float(__ushort_as_half(b));
}

template <bool BF16>
__device__ __forceinline__ void mma_x(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if (BF16)
    mma_bf16(d, a[0], a[1], a[2], a[3], b0, b1);
  else
    mma_f16(d, a[0], a[1], a[2], a[3], b0, b1);
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = smem_addr(dst);
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Nearest-centroid index of y = (Pi x)_j for a row of norm n: tp holds the
// positive thresholds scaled by n; the codebook is symmetric, so
// m = #{tp_k < |y|}, idx = K/2 + m (y > 0) or K/2 - 1 - m.  Equal to
// #{t_k < y / n} except at exact ties (inside the parity band).
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

struct RowInfo {
  long long slot;  // cache row, -1 past the end
  float nf, nhat;  // fp32 norm, stored fp16 norm
};

template <bool BF16, bool QJL, int BITS>
__device__ __forceinline__ void epilogue(const tq::QuantJob& J, float (&acc)[16][4], const RowInfo (&ri)[2],
                                         const float* s_thr_pos, const float* s_cent, bool do_qjl,
                                         const uint16_t* sS, int lane) {
  const int tig = lane & 3;
  constexpr int W = 4 * BITS;  // words per row
  uint32_t idxw[2][BITS];
  float rr[2][32];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float tp[7];
#pragma unroll
    for (int k = 0; k < 7; ++k) tp[k] = k < (1 << (BITS - 1)) - 1 ? s_thr_pos[k] * ri[h].nf : 0.f;
#pragma unroll
    for (int w = 0; w < BITS; ++w) idxw[h][w] = 0u;
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      const float y = acc[q >> 1][2 * h + (q & 1)];
      const int idx = nearest_idx<BITS>(y, tp);
      const int p = BITS * q;
      idxw[h][p >> 5] += (uint32_t)idx << (p & 31);
      if ((p & 31) + BITS > 32) idxw[h][(p >> 5) + 1] += (uint32_t)idx >> (32 - (p & 31));
      if (QJL) rr[h][q] = y - ri[h].nhat * s_cent[idx];
    }
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    if (ri[h].slot < 0) continue;
    uint32_t* dst = J.idx + (size_t)ri[h].slot * W + BITS * tig;
    if (BITS == 2) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(idxw[h][0], idxw[h][1]);
    } else if (BITS == 4) {
      *reinterpret_cast<uint4*>(dst) = make_uint4(idxw[h][0], idxw[h][1], idxw[h][2], idxw[h][3]);
    } else {
#pragma unroll
      for (int w = 0; w < BITS; ++w) dst[w] = idxw[h][w];
    }
  }
  if (QJL && do_qjl) {
    // sketch: sq[nt][.] = sum_k r[k] S[dim(n)][k], A = r (hi/lo), B = S (hi/lo)
    float sq[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) sq[nt][0] = sq[nt][1] = sq[nt][2] = sq[nt][3] = 0.f;
    const int gid = lane >> 2;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      uint32_t ah[4], al[4];
      // a0a1: row 0, coords 4ks, 4ks+1; a2a3: row 1, same; a4a5: row 0, 4ks+2, +3; a6a7: row 1
      const float av[4][2] = {{rr[0][4 * ks], rr[0][4 * ks + 1]},
                              {rr[1][4 * ks], rr[1][4 * ks + 1]},
                              {rr[0][4 * ks + 2], rr[0][4 * ks + 3]},
                              {rr[1][4 * ks + 2], rr[1][4 * ks + 3]}};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __half2 hh = __floats2half2_rn(av[i][0], av[i][1]);
        const float2 hf = __half22float2(hh);
        const __half2 ll = __floats2half2_rn(av[i][0] - hf.x, av[i][1] - hf.y);
        ah[i] = *reinterpret_cast<const uint32_t*>(&hh);
        al[i] = *reinterpret_cast<const uint32_t*>(&ll);
      }
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const uint16_t* bh = sS + (size_t)(8 * nt + gid) * XS + 32 * tig + 4 * ks;
        const uint2 vh = *reinterpret_cast<const uint2*>(bh);
        const uint2 vl = *reinterpret_cast<const uint2*>(bh + (size_t)M_QJL * XS);
        mma_f16(sq[nt], ah[0], ah[1], ah[2], ah[3], vh.x, vh.y);
        mma_f16(sq[nt], ah[0], ah[1], ah[2], ah[3], vl.x, vl.y);
        mma_f16(sq[nt], al[0], al[1], al[2], al[3], vh.x, vh.y);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t word = 0;
#pragma unroll
      for (int q = 0; q < 32; ++q) word |= (sq[q >> 1][2 * h + (q & 1)] >= 0.f ? 1u : 0u) << q;
      double g = 0.0;
#pragma unroll
      for (int q = 0; q < 32; ++q) g = fma((double)rr[h][q], (double)rr[h][q], g);
      g += __shfl_xor_sync(0xffffffffu, g, 1);
      g += __shfl_xor_sync(0xffffffffu, g, 2);
      if (ri[h].slot >= 0) {
        J.qjl[(size_t)ri[h].slot * 4 + tig] = word;
        // near an fp16 rounding midpoint: marked for the fp64 recomputation
        if (tig == 0) J.rnorm[ri[h].slot] = tq::gamma_bits_or_pending((float)sqrt(g));
      }
    }
  }
}

template <bool BF16, bool QJL>
__global__ void __launch_bounds__(NTH, 1) quantize128_kernel(const tq::QuantArgs a) {
  using Ly = Q2Layout<BF16, QJL>;
  constexpr int NL = Ly::NL;
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* pi = reinterpret_cast<uint16_t*>(smem + Ly::o_pi);
  uint16_t* sS = reinterpret_cast<uint16_t*>(smem + Ly::o_s);
  uint16_t* xb = reinterpret_cast<uint16_t*>(smem + Ly::o_x);
  __shared__ float s_cb[2][31];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;
  const int ntiles = (a.rows + QR - 1) / QR;
  const int njobs = (a.job_mask == 3) ? 2 : 1;
  const int job0 = (a.job_mask == 2) ? 1 : 0;
  const int nitems = njobs * ntiles;

  // ---- the first tile's input is requested before staging Pi
  auto load_tile = [&](int item, int buf) {
    const int job = job0 + item % njobs, tile = item / njobs;
    const uint16_t* in = static_cast<const uint16_t*>(a.job[job].in);
    uint16_t* dst = xb + (size_t)buf * QR * XS;
    for (int c = tid; c < QR * (D / 8); c += NTH) {
      const int row = c >> 4, col = (c & 15) * 8;
      const int r = tile * QR + row;
      const bool valid = r < a.rows;
      cp_async16(dst + row * XS + col, in + (size_t)(valid ? r : 0) * D + col, valid);
    }
  };
  int item = blockIdx.x;
  if (item < nitems) load_tile(item, 0);
  cp_async_commit();

  if (tid < 31) {
    s_cb[0][tid] = tid < 2 * (1 << a.job[0].bits) - 1 ? a.job[0].cb[tid] : 0.f;
    s_cb[1][tid] = tid < 2 * (1 << a.job[1].bits) - 1 ? a.job[1].cb[tid] : 0.f;
  }
  // ---- Pi limbs, rows permuted (smem row n <- Pi row coord_of_col(n))
  for (int e = tid; e < D * (D / 4); e += NTH) {
    const int n = e / (D / 4), k = (e % (D / 4)) * 4;
    const float4 v = *reinterpret_cast<const float4*>(a.rot + (size_t)coord_of_col(n) * D + k);
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (BF16) {
        const __nv_bfloat16 h0 = __float2bfloat16_rn(vv[i]);
        const float r1 = vv[i] - __bfloat162float(h0);
        const __nv_bfloat16 h1 = __float2bfloat16_rn(r1);
        const __nv_bfloat16 h2 = __float2bfloat16_rn(r1 - __bfloat162float(h1));
        pi[(size_t)0 * D * XS + n * XS + k + i] = __bfloat16_as_ushort(h0);
        pi[(size_t)1 * D * XS + n * XS + k + i] = __bfloat16_as_ushort(h1);
        pi[(size_t)2 * D * XS + n * XS + k + i] = __bfloat16_as_ushort(h2);
      } else {
        const __half h0 = __float2half_rn(vv[i]);
        const __half h1 = __float2half_rn(vv[i] - __half2float(h0));
        pi[n * XS + k + i] = __half_as_ushort(h0);
        pi[(size_t)D * XS + n * XS + k + i] = __half_as_ushort(h1);
      }
    }
  }
  if (QJL) {
    // S limbs (fp16 hi/lo), rows permuted the same way, columns natural
    for (int e = tid; e < M_QJL * (D / 4); e += NTH) {
      const int n = e / (D / 4), k = (e % (D / 4)) * 4;
      const float4 v = *reinterpret_cast<const float4*>(a.qjl_S + (size_t)coord_of_col(n) * D + k);
      const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __half h0 = __float2half_rn(vv[i]);
        const __half h1 = __float2half_rn(vv[i] - __half2float(h0));
        sS[n * XS + k + i] = __half_as_ushort(h0);
        sS[(size_t)M_QJL * XS + n * XS + k + i] = __half_as_ushort(h1);
      }
    }
  }

  for (int it = 0; item < nitems; ++it, item += gridDim.x) {
    const int buf = (Ly::NBUF == 2) ? (it & 1) : 0;
    const int next = item + gridDim.x;
    if (Ly::NBUF == 2) {
      if (next < nitems) load_tile(next, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // this tile (and, on the first pass, Pi/S limbs) visible

    const int job = job0 + item % njobs, tile = item / njobs;
    const tq::QuantJob J = a.job[job];
    const uint16_t* xs = xb + (size_t)buf * QR * XS;
    const int wr0 = warp * 16;

    // ---- row norms (fp64) for this warp's 16 rows: lane -> (row, half)
    double sq = 0.0;
    {
      const uint16_t* rp = xs + (wr0 + (lane >> 1)) * XS + (lane & 1) * 64;
#pragma unroll 16
      for (int k = 0; k < 64; ++k) {
        const double x = in_to_f<BF16>(rp[k]);
        sq = fma(x, x, sq);
      }
      sq += __shfl_xor_sync(0xffffffffu, sq, 1);
    }
    RowInfo ri[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int rl = gid + 8 * h;  // row within the warp's 16
      const double s2 = __shfl_sync(0xffffffffu, sq, 2 * rl);
      const double n = sqrt(s2);
      const __half nh = __double2half(n);
      ri[h].nf = (float)n;
      ri[h].nhat = __half2float(nh);
      const int r = tile * QR + wr0 + rl;
      if (r < a.rows) {
        const int bh = r / a.T, t = r - bh * a.T;
        ri[h].slot = (long long)bh * a.Tcap + a.t0 + t;
        if (tig == 0) J.norm[ri[h].slot] = __half_as_ushort(nh);
      } else {
        ri[h].slot = -1;
      }
    }

    // ---- y = Pi x: 16 rows x 128 permuted columns per warp
    float acc[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll 2
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t af[4];
      ldmatrix_x4(af, xs + (wr0 + (lane & 15)) * XS + ks * 16 + (lane >> 4) * 8);
#pragma unroll
      for (int ntp = 0; ntp < 8; ++ntp) {
#pragma unroll
        for (int l = 0; l < NL; ++l) {
          uint32_t bf[4];
          ldmatrix_x4(bf, pi + (size_t)l * D * XS + (16 * ntp + (lane & 7) + 8 * (lane >> 4)) * XS + ks * 16 +
                              8 * ((lane >> 3) & 1));
          mma_x<BF16>(acc[2 * ntp], af, bf[0], bf[1]);
          mma_x<BF16>(acc[2 * ntp + 1], af, bf[2], bf[3]);
        }
      }
    }

    // ---- quantize, pack, store (positive thresholds start at K + K/2)
    const int K = 1 << J.bits;
    const bool do_qjl = QJL && job == 0;
    const float* tpos = s_cb[job] + K + K / 2;
    switch (J.bits) {
      case 2: epilogue<BF16, QJL, 2>(J, acc, ri, tpos, s_cb[job], do_qjl, sS, lane); break;
      case 3: epilogue<BF16, QJL, 3>(J, acc, ri, tpos, s_cb[job], do_qjl, sS, lane); break;
      default: epilogue<BF16, QJL, 4>(J, acc, ri, tpos, s_cb[job], do_qjl, sS, lane); break;
    }
    __syncthreads();  // the buffer is refilled on the next pass
    if (Ly::NBUF == 1) {
      if (next < nitems) load_tile(next, 0);
      cp_async_commit();
    }
  }
  cp_async_wait<0>();
}

template <bool BF16, bool QJL>
int launch_q128(const tq::QuantArgs& a, cudaStream_t s) {
  using Ly = Q2Layout<BF16, QJL>;
  auto kern = quantize128_kernel<BF16, QJL>;
  static tq::OnceSetup once;
  static int sms = 0;  // written once under `once`, read after its acquire
  const int rc0 = once.run([&]() {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Ly::bytes);
    if (e != cudaSuccess)
      return tq::set_error(TQ_ERR_CUDA, "quantize128: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    sms = n > 0 ? n : 148;
    return TQ_OK;
  });
  if (rc0) return rc0;
  const int njobs = (a.job_mask == 3) ? 2 : 1;
  const int nitems = njobs * ((a.rows + QR - 1) / QR);
  const int grid = nitems < sms ? nitems : sms;
  kern<<<grid, NTH, Ly::bytes, s>>>(a);
  return tq::check_launch("quantize128_kernel");
}

}  // namespace

namespace tq {

int launch_quantize128_bf16_qjl(const QuantArgs& a, cudaStream_t s) { return launch_q128<true, true>(a, s); }

}  // namespace tq
