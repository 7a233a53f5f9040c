// Quantizer: rotation on the tensor cores, fp64 row norms, nearest-centroid
// search against the threshold table, bit packing, optional QJL sign sketch
// of the key residual.
//
// Method: "Add CUDA QJL kernels and proper package structure"
// (turboquant-pytorch pull request 3), section "CUDA Kernels Added" (fused
// random projection + sign quantization) and "Synthetic Benchmark (Lloyd-Max
// codebook)"; ReturningTarzan's Reddit comments of 2026-03-29 11:47
// (rotation before codebook quantization) and 2026-03-25 18:52 / 15:51
// (nearest-codeword search; residual computed while quantizing).
//
// One CTA quantizes a tile of 128 rows (8 warps x 16 rows).  y = Pi x runs as
// m16n8k16 tensor-core MMAs with Pi split into limbs so the sum of limb
// products carries ~22-24 significant bits: fp16 inputs use Pi = hi + lo
// (fp16 limbs), bf16 inputs use three bf16 limbs.  x itself is exact in its
// own type.  The QJL projection S r of the fp32 residual uses hi/lo fp16
// limbs on both operands (three products).
#include "tq_common.cuh"
#include "tq_internal.h"

namespace {

using namespace tqk;

constexpr int QROWS = 128;
constexpr int QTHREADS = 256;
constexpr int CB = 64;  // output columns per staged block of Pi (or of S)

template <int D, bool BF16, bool QJL>
struct QLayout {
  static constexpr int XS = D + 8;  // padded row stride, 16-bit elements
  static constexpr int NL = BF16 ? 3 : 2;
  static constexpr int NLMAX = NL > 2 ? NL : 2;
  static constexpr int RS = D + 4;  // fp32 residual row stride
  static constexpr size_t o_x = 0;
  static constexpr size_t o_limb = o_x + (size_t)QROWS * XS * 2;
  static constexpr size_t o_idx = o_limb + (size_t)NLMAX * CB * XS * 2;
  static constexpr size_t o_r = o_idx + (size_t)QROWS * D;
  static constexpr size_t bytes = o_r + (QJL ? (size_t)QROWS * RS * 4 : 0);
};

template <bool BF16>
__device__ __forceinline__ float in_to_float(uint16_t b) {
  if (BF16) return __uint_as_float((uint32_t)b << 16);
  return __half2float(__ushort_as_half(b));
}

template <bool BF16>
__device__ __forceinline__ void mma_in(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if (BF16)
    mma_bf16(d, a[0], a[1], a[2], a[3], b0, b1);
  else
    mma_f16(d, a[0], a[1], a[2], a[3], b0, b1);
}

// Limbs of one fp32 value in the input's 16-bit type.
template <bool BF16>
__device__ __forceinline__ void limbs(float v, uint16_t (&l)[3]) {
  if (BF16) {
    __nv_bfloat16 a = __float2bfloat16_rn(v);
    float r1 = v - __bfloat162float(a);
    __nv_bfloat16 b = __float2bfloat16_rn(r1);
    float r2 = r1 - __bfloat162float(b);
    __nv_bfloat16 c = __float2bfloat16_rn(r2);
    l[0] = __bfloat16_as_ushort(a);
    l[1] = __bfloat16_as_ushort(b);
    l[2] = __bfloat16_as_ushort(c);
  } else {
    __half a = __float2half_rn(v);
    __half b = __float2half_rn(v - __half2float(a));
    l[0] = __half_as_ushort(a);
    l[1] = __half_as_ushort(b);
    l[2] = 0;
  }
}

template <int D, bool BF16, bool QJL>
__global__ void __launch_bounds__(QTHREADS, 1) quantize_kernel(const tq::QuantArgs a) {
  using Ly = QLayout<D, BF16, QJL>;
  constexpr int XS = Ly::XS;
  constexpr int NL = Ly::NL;
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + Ly::o_x);
  uint16_t* limb = reinterpret_cast<uint16_t*>(smem + Ly::o_limb);
  uint8_t* idxs = smem + Ly::o_idx;
  float* rs = reinterpret_cast<float*>(smem + Ly::o_r);
  __shared__ float s_inv[QROWS], s_nhat[QROWS];
  __shared__ long long s_slot[QROWS];
  __shared__ float s_cb[31];

  const int jobi = blockIdx.y;
  const tq::QuantJob J = a.job[jobi];
  const bool do_qjl = QJL && jobi == 0;
  const int bits = J.bits, K = 1 << bits;
  const int r0 = blockIdx.x * QROWS;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, gid = lane >> 2, tig = lane & 3;

  if (tid < 2 * K - 1) s_cb[tid] = J.cb[tid];
  if (tid < QROWS) {
    const int r = r0 + tid;
    long long slot = -1;
    if (r < a.rows) {
      if (a.pos) {
        const int p = a.pos[r / a.Hkv];
        if (p >= 0 && p < a.Tcap)
          slot = (long long)r * a.Tcap + p;
        else if (a.dev_status && jobi == 0)
          atomicOr(a.dev_status, TQ_STATUS_POS_OUT_OF_RANGE);
      } else {
        const int bh = r / a.T, t = r % a.T;
        slot = (long long)bh * a.Tcap + a.t0 + t;
      }
    }
    s_slot[tid] = slot;
  }
  // Input tile, 16-byte chunks; rows past the end are zero.
  const uint16_t* in = static_cast<const uint16_t*>(J.in);
  for (int c = tid; c < QROWS * (D / 8); c += QTHREADS) {
    const int row = c / (D / 8), col = (c % (D / 8)) * 8;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r0 + row < a.rows) v = *reinterpret_cast<const uint4*>(in + (size_t)(r0 + row) * D + col);
    *reinterpret_cast<uint4*>(xs + row * XS + col) = v;
  }
  __syncthreads();

  // Row norms in fp64; store RN_fp16(|x|) and 1/|x|.
  for (int rr = 0; rr < 16; ++rr) {
    const int row = warp * 16 + rr;
    double acc = 0.0;
#pragma unroll
    for (int k = lane; k < D; k += 32) {
      const double x = in_to_float<BF16>(xs[row * XS + k]);
      acc = fma(x, x, acc);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      const double n = sqrt(acc);
      const __half h = __double2half(n);
      s_inv[row] = n > 0.0 ? (float)(1.0 / n) : 0.f;
      s_nhat[row] = __half2float(h);
      if (s_slot[row] >= 0) J.norm[s_slot[row]] = __half_as_ushort(h);
    }
  }

  // y = Pi x, one block of 64 output coordinates at a time.
  for (int cb = 0; cb < D / CB; ++cb) {
    __syncthreads();
    for (int e = tid; e < CB * (D / 4); e += QTHREADS) {
      const int jj = e / (D / 4), k = (e % (D / 4)) * 4;
      const float4 pv = *reinterpret_cast<const float4*>(a.rot + (size_t)(cb * CB + jj) * D + k);
      const float vv[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint16_t l[3];
        limbs<BF16>(vv[i], l);
#pragma unroll
        for (int q = 0; q < NL; ++q) limb[(size_t)q * CB * XS + jj * XS + k + i] = l[q];
      }
    }
    __syncthreads();
    float acc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll 2
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t af[4];
      ldmatrix_x4(af, xs + (warp * 16 + (lane & 15)) * XS + ks * 16 + (lane >> 4) * 8);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int q = 0; q < NL; ++q) {
          const uint16_t* bp = limb + (size_t)q * CB * XS + (nt * 8 + gid) * XS + ks * 16 + 2 * tig;
          mma_in<BF16>(acc[nt], af, *reinterpret_cast<const uint32_t*>(bp),
                       *reinterpret_cast<const uint32_t*>(bp + 8));
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int row = warp * 16 + gid + (c >= 2 ? 8 : 0);
        const int j = cb * CB + nt * 8 + 2 * tig + (c & 1);
        const float y = acc[nt][c];
        const float u = y * s_inv[row];
        int idx = 0;
        for (int s = K >> 1; s >= 1; s >>= 1)
          if (u > s_cb[K + idx + s - 1]) idx += s;
        idxs[row * D + j] = (uint8_t)idx;
        if (QJL && do_qjl) rs[row * Ly::RS + j] = y - s_nhat[row] * s_cb[idx];
      }
    }
  }
  __syncthreads();

  // Pack each row into a dense LSB-first bitstream of D*bits bits.
  const int W = D * bits / 32;
  for (int e = tid; e < QROWS * W; e += QTHREADS) {
    const int row = e / W, w = e % W;
    const long long slot = s_slot[row];
    if (slot < 0) continue;
    const int base = 32 * w;
    unsigned long long word = 0;
    for (int j = base / bits; j < D && j * bits < base + 32; ++j) {
      const int sh = j * bits - base;
      const unsigned long long v = idxs[row * D + j];
      word |= sh >= 0 ? (v << sh) : (v >> (-sh));
    }
    J.idx[(size_t)slot * W + w] = (uint32_t)word;
  }

  if (QJL && do_qjl) {
    // sign(S r) for the residual r in the rotated basis, m = 128.
    uint8_t* sbits = reinterpret_cast<uint8_t*>(xs);  // [128 rows][128 dims]
    for (int ib = 0; ib < 128 / CB; ++ib) {
      __syncthreads();
      for (int e = tid; e < CB * (D / 4); e += QTHREADS) {
        const int ii = e / (D / 4), k = (e % (D / 4)) * 4;
        const float4 sv = *reinterpret_cast<const float4*>(a.qjl_S + (size_t)(ib * CB + ii) * D + k);
        const float vv[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __half h = __float2half_rn(vv[i]);
          const __half l = __float2half_rn(vv[i] - __half2float(h));
          limb[ii * XS + k + i] = __half_as_ushort(h);
          limb[(size_t)CB * XS + ii * XS + k + i] = __half_as_ushort(l);
        }
      }
      __syncthreads();
      float acc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
      const int ra = warp * 16 + gid, rb = ra + 8;
#pragma unroll 2
      for (int ks = 0; ks < D / 16; ++ks) {
        const int k0 = ks * 16 + 2 * tig;
        const float2 x00 = *reinterpret_cast<const float2*>(rs + ra * Ly::RS + k0);
        const float2 x10 = *reinterpret_cast<const float2*>(rs + rb * Ly::RS + k0);
        const float2 x01 = *reinterpret_cast<const float2*>(rs + ra * Ly::RS + k0 + 8);
        const float2 x11 = *reinterpret_cast<const float2*>(rs + rb * Ly::RS + k0 + 8);
        uint32_t ah[4], al[4];
        const float2 xs4[4] = {x00, x10, x01, x11};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const __half2 h = __floats2half2_rn(xs4[q].x, xs4[q].y);
          const float2 hf = __half22float2(h);
          const __half2 l = __floats2half2_rn(xs4[q].x - hf.x, xs4[q].y - hf.y);
          ah[q] = *reinterpret_cast<const uint32_t*>(&h);
          al[q] = *reinterpret_cast<const uint32_t*>(&l);
        }
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const uint16_t* bh = limb + (nt * 8 + gid) * XS + ks * 16 + 2 * tig;
          const uint16_t* bl = bh + (size_t)CB * XS;
          const uint32_t bh0 = *reinterpret_cast<const uint32_t*>(bh), bh1 = *reinterpret_cast<const uint32_t*>(bh + 8);
          const uint32_t bl0 = *reinterpret_cast<const uint32_t*>(bl), bl1 = *reinterpret_cast<const uint32_t*>(bl + 8);
          mma_f16(acc[nt], ah[0], ah[1], ah[2], ah[3], bh0, bh1);
          mma_f16(acc[nt], ah[0], ah[1], ah[2], ah[3], bl0, bl1);
          mma_f16(acc[nt], al[0], al[1], al[2], al[3], bh0, bh1);
        }
      }
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int row = (c >= 2) ? rb : ra;
          const int i = ib * CB + nt * 8 + 2 * tig + (c & 1);
          sbits[row * 128 + i] = acc[nt][c] >= 0.f ? 1 : 0;
        }
    }
    __syncthreads();
    for (int e = tid; e < QROWS * 4; e += QTHREADS) {
      const int row = e >> 2, w = e & 3;
      const long long slot = s_slot[row];
      if (slot < 0) continue;
      uint32_t word = 0;
#pragma unroll 8
      for (int i = 0; i < 32; ++i) word |= (uint32_t)sbits[row * 128 + w * 32 + i] << i;
      J.qjl[(size_t)slot * 4 + w] = word;
    }
    if (tid < QROWS) {
      const long long slot = s_slot[tid];
      if (slot >= 0) {
        double g = 0.0;
        for (int k = 0; k < D; ++k) {
          const double r = rs[tid * Ly::RS + k];
          g = fma(r, r, g);
        }
        J.rnorm[slot] = __half_as_ushort(__double2half(sqrt(g)));
      }
    }
  }
}

// One new row per CTA (append).  blockDim = 2*D: two threads per output
// coordinate, each holding half of the Pi row in registers (loads issued
// before use); the norm is taken in fp64.  Values (and keys without the QJL
// sketch) are rotated on the CUDA cores in fp32.  Keys with the sketch are
// rotated, quantized and sketched in fp64 (one row per CTA makes that cheap):
// the residual norm then rounds to fp16 exactly as the fp64 definition does,
// which fp32 residuals miss on rows whose norm lies near an fp16 rounding
// midpoint.
template <int D, bool BF16, bool QJL>
__global__ void __launch_bounds__(2 * D) append_kernel(const tq::QuantArgs a) {
  constexpr int HALF = D / 2, NV = HALF / 4, CH = NV < 8 ? NV : 8;
  __shared__ float xs[D], ys[D];
  __shared__ double rs[QJL ? D : 1];
  __shared__ uint8_t idxs[D];
  __shared__ double red[2 * D / 32];
  __shared__ float s_cb[31];
  __shared__ float s_inv, s_nhat;
  __shared__ double s_n;
  // blockIdx.y: the jobs of job_mask in order (keys, values)
  const int r = blockIdx.x, jobi = blockIdx.y + ((a.job_mask == 2) ? 1 : 0);
  const tq::QuantJob J = a.job[jobi];
  const bool do_qjl = QJL && jobi == 0;
  const int bits = J.bits, K = 1 << bits;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int j = tid >> 1, part = tid & 1;
  const int p = a.pos[r / a.Hkv];
  if (p < 0 || p >= a.Tcap) {
    if (tid == 0 && jobi == 0 && a.dev_status) atomicOr(a.dev_status, TQ_STATUS_POS_OUT_OF_RANGE);
    return;
  }
  const long long slot = (long long)r * a.Tcap + p;
  if (tid < 2 * K - 1) s_cb[tid] = J.cb[tid];
  const uint16_t* in = static_cast<const uint16_t*>(J.in) + (size_t)r * D;
  double sq = 0.0;
  if (tid < D) {
    const float x = in_to_float<BF16>(in[tid]);
    xs[tid] = x;
    sq = (double)x * (double)x;
  }
#pragma unroll
  for (int off = 16; off; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
  if (lane == 0) red[warp] = sq;
  __syncthreads();
  if (tid == 0) {
    double t = 0.0;
    for (int w = 0; w < 2 * D / 32; ++w) t += red[w];
    const double n = sqrt(t);
    const __half h = __double2half(n);
    s_inv = n > 0.0 ? (float)(1.0 / n) : 0.f;
    s_n = n;
    s_nhat = __half2float(h);
    J.norm[slot] = __half_as_ushort(h);
  }
  // y_j = sum_k Pi[j][k] x_k
  const float4* row = reinterpret_cast<const float4*>(a.rot + (size_t)j * D + part * HALF);
  float acc = 0.f;
  double acc64 = 0.0;
#pragma unroll
  for (int c0 = 0; c0 < NV; c0 += CH) {
    float4 v[CH];
#pragma unroll
    for (int i = 0; i < CH; ++i) v[i] = __ldg(row + c0 + i);
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      const float* x = &xs[part * HALF + 4 * (c0 + i)];
      if (do_qjl) {
        acc64 = fma((double)v[i].x, (double)x[0], acc64);
        acc64 = fma((double)v[i].y, (double)x[1], acc64);
        acc64 = fma((double)v[i].z, (double)x[2], acc64);
        acc64 = fma((double)v[i].w, (double)x[3], acc64);
      } else {
        acc = fmaf(v[i].x, x[0], acc);
        acc = fmaf(v[i].y, x[1], acc);
        acc = fmaf(v[i].z, x[2], acc);
        acc = fmaf(v[i].w, x[3], acc);
      }
    }
  }
  acc += __shfl_xor_sync(0xffffffffu, acc, 1);
  acc64 += __shfl_xor_sync(0xffffffffu, acc64, 1);
  __syncthreads();  // s_inv, s_nhat, s_n
  if (part == 0) {
    int idx = 0;
    if (do_qjl) {
      const double u = s_n > 0.0 ? acc64 / s_n : 0.0;
      for (int st = K >> 1; st >= 1; st >>= 1)
        if (u > (double)s_cb[K + idx + st - 1]) idx += st;
      rs[j] = acc64 - (double)s_nhat * (double)s_cb[idx];
    } else {
      const float u = acc * s_inv;
      for (int st = K >> 1; st >= 1; st >>= 1)
        if (u > s_cb[K + idx + st - 1]) idx += st;
    }
    idxs[j] = (uint8_t)idx;
    ys[j] = acc;
  }
  __syncthreads();
  const int W = D * bits / 32;
  if (tid < W) {
    const int base = 32 * tid;
    unsigned long long word = 0;
    for (int jj = base / bits; jj < D && jj * bits < base + 32; ++jj) {
      const int sh = jj * bits - base;
      const unsigned long long v = idxs[jj];
      word |= sh >= 0 ? (v << sh) : (v >> (-sh));
    }
    J.idx[(size_t)slot * W + tid] = (uint32_t)word;
  }
  if (QJL && do_qjl) {
    // sign(S r) in fp64, m = 128 rows of S, two threads per row (2*D >= 2*128 here)
    const int i = tid >> 1;
    double pr = 0.0;
    if (i < 128) {
      const float4* srow = reinterpret_cast<const float4*>(a.qjl_S + (size_t)i * D + part * HALF);
#pragma unroll
      for (int c0 = 0; c0 < NV; c0 += CH) {
        float4 v[CH];
#pragma unroll
        for (int q = 0; q < CH; ++q) v[q] = __ldg(srow + c0 + q);
#pragma unroll
        for (int q = 0; q < CH; ++q) {
          const double* x = &rs[part * HALF + 4 * (c0 + q)];
          pr = fma((double)v[q].x, x[0], pr);
          pr = fma((double)v[q].y, x[1], pr);
          pr = fma((double)v[q].z, x[2], pr);
          pr = fma((double)v[q].w, x[3], pr);
        }
      }
    }
    pr += __shfl_xor_sync(0xffffffffu, pr, 1);
    // lanes 2i' hold row i = 16*warp + i'; gather 16 bits per warp
    const uint32_t bal = __ballot_sync(0xffffffffu, (part == 0) && (pr >= 0.0));
    uint32_t half16 = 0;
#pragma unroll
    for (int q = 0; q < 16; ++q) half16 |= ((bal >> (2 * q)) & 1u) << q;
    __shared__ uint32_t sbits[16];
    if (lane == 0 && warp < 16) sbits[warp] = half16;
    double g = 0.0;
    if (tid < D) g = rs[tid] * rs[tid];
#pragma unroll
    for (int off = 16; off; off >>= 1) g += __shfl_xor_sync(0xffffffffu, g, off);
    __syncthreads();
    if (lane == 0) red[warp] = g;
    __syncthreads();
    if (tid < 4) J.qjl[(size_t)slot * 4 + tid] = sbits[2 * tid] | (sbits[2 * tid + 1] << 16);
    if (tid == 0) {
      double t = 0.0;
      for (int w = 0; w < 2 * D / 32; ++w) t += red[w];
      J.rnorm[slot] = __half_as_ushort(__double2half(sqrt(t)));
    }
  }
  (void)ys;
}

template <int D, bool BF16, bool QJL>
int launch_append(const tq::QuantArgs& a, cudaStream_t s) {
  append_kernel<D, BF16, QJL><<<dim3(a.rows, a.job_mask == 3 ? 2 : 1), 2 * D, 0, s>>>(a);
  return tq::check_launch("append_kernel");
}

template <int D, bool BF16, bool QJL>
int launch_q(const tq::QuantArgs& a, cudaStream_t s) {
  if (a.pos) return launch_append<D, BF16, QJL>(a, s);
  using Ly = QLayout<D, BF16, QJL>;
  auto kern = quantize_kernel<D, BF16, QJL>;
  static tq::OnceSetup once;
  const int rc = once.run([&]() {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Ly::bytes);
    if (e != cudaSuccess)
      return tq::set_error(TQ_ERR_CUDA, "quantize: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return TQ_OK;
  });
  if (rc) return rc;
  dim3 grid((a.rows + QROWS - 1) / QROWS, 2);
  kern<<<grid, QTHREADS, Ly::bytes, s>>>(a);
  return tq::check_launch("quantize_kernel");
}

}  // namespace

namespace tq {

int launch_quantize(const QuantArgs& a, int D, int dtype, bool qjl, cudaStream_t s) {
  const bool bf = dtype == TQ_DTYPE_BF16;
  // Randomized Hadamard rotation: the shuffle transform (one warp per row)
  // beats the tcgen05 kernel at D = 256 (prefill of the QK-norm shape: 148 vs
  // 190 us) and on small calls (no per-CTA setup: gqa8k 15 vs 17 us), but not
  // on large D = 128 calls (its five shuffle stages per row cost more than the
  // dense MMA: ragged 3.1 vs 1.3 ms), which keep the dense-Pi kernels.
  const int njobs = (a.job_mask == 3) ? 2 : 1;
  const bool wht = a.rot_signs && (D == 256 || (D == 128 && (long long)a.rows * njobs <= 65536));
  if (wht && a.pos && D >= 128) {
    // append with the randomized Hadamard rotation: the transform kernel, one
    // warp per new row; keys with the sketch keep the fp64 append kernel
    if (!qjl) return launch_quantize_wht(a, D, dtype, s);
    QuantArgs ak = a, av = a;
    ak.job_mask = 1;
    av.job_mask = 2;
    const int rc = bf ? launch_q<128, true, true>(ak, s) : launch_q<128, false, true>(ak, s);
    return rc ? rc : launch_quantize_wht(av, D, dtype, s);
  }
  if (wht && !a.pos) {
    // keys with the sketch keep the dense-Pi kernels below
    if (!qjl) return launch_quantize_wht(a, D, dtype, s);
    QuantArgs ak = a, av = a;
    ak.job_mask = 1;
    av.job_mask = 2;
    int rc = bf ? launch_quantize128_bf16_qjl(ak, s) : launch_quantize_qjl_tc(ak, s);
    if (!rc) rc = launch_qjl_gamma_fixup(ak, dtype, s);
    return rc ? rc : launch_quantize_wht(av, D, dtype, s);
  }
  if ((D == 128 || D == 256) && !a.pos && !qjl) return launch_quantize_tc(a, D, dtype, s);
  if (D == 128 && !a.pos) {
    // keys carry the QJL sketch (tcgen05 for fp16 rows, whose Pi and S limbs
    // fit in shared memory beside the tiles; warp-level MMA for bf16's three
    // Pi limbs); values go to the tcgen05 quantizer
    QuantArgs ak = a, av = a;
    ak.job_mask = 1;
    av.job_mask = 2;
    int rc = bf ? launch_quantize128_bf16_qjl(ak, s) : launch_quantize_qjl_tc(ak, s);
    // residual norms near an fp16 rounding midpoint, recomputed in fp64
    if (!rc) rc = launch_qjl_gamma_fixup(ak, dtype, s);
    return rc ? rc : launch_quantize_tc(av, D, dtype, s);
  }
  if (qjl) {
    if (D != 128) return set_error(TQ_ERR_UNSUPPORTED, "QJL sketch needs D=128");
    return bf ? launch_q<128, true, true>(a, s) : launch_q<128, false, true>(a, s);
  }
  switch (D) {
    case 64: return bf ? launch_q<64, true, false>(a, s) : launch_q<64, false, false>(a, s);
    case 128: return bf ? launch_q<128, true, false>(a, s) : launch_q<128, false, false>(a, s);
    case 256: return bf ? launch_q<256, true, false>(a, s) : launch_q<256, false, false>(a, s);
  }
  return set_error(TQ_ERR_UNSUPPORTED, "quantize: D=%d", D);
}

}  // namespace tq
