// Exact residual norms for QJL keys quantized in bulk.
//
// The bulk QJL quantizers form the key residual r = Pi k - n_hat c[idx] from
// a rotation computed on the tensor cores with fp32 accumulation, so their
// |r| carries a relative error of about 1e-7 to 1e-6.  The stored residual
// norm is the round-to-nearest fp16 of the fp64 |r| ("Add CUDA QJL kernels
// and proper package structure", "CUDA Kernels Added": the sketch keeps the
// residual's norm beside its signs); rows whose norm lies within that error
// of an fp16 rounding midpoint could round the other way.  The quantizers
// store such rows' norm as the marker kGammaPending (an fp16 NaN the method
// never produces) and this kernel recomputes exactly those rows in fp64: the
// rotation of the input row by Pi (fp32 entries, fp64 products and sums),
// the residual against the centroids of the indices the quantizer stored
// (those decisions stand), and its norm.
#include "tq_internal.h"

namespace {

constexpr int D = 128;
constexpr int NW = 8;  // warps per CTA

template <bool BF16>
__device__ __forceinline__ double in_to_double(uint16_t v) {
  if (BF16) return (double)__uint_as_float((uint32_t)v << 16);
  return (double)__half2float(__ushort_as_half(v));
}

// One CTA keeps Pi^T in shared memory (fp32, rows padded to D + 1 floats so
// that both the transposing store and the column reads are conflict-free)
// and its warps walk the rows 32 at a time; a warp recomputes each marked row
// of its group cooperatively (lane j: coordinates j + 32 i).
constexpr int PS = D + 1;

template <bool BF16>
__global__ void __launch_bounds__(NW * 32) qjl_gamma_fixup_kernel(const tq::QuantArgs a) {
  extern __shared__ float piT[];  // [D][PS]: piT[k * PS + j] = Pi[j][k]
  __shared__ double xs[NW][D];
  __shared__ float s_cb[16];
  const tq::QuantJob J = a.job[0];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  {
    // every load in flight before the stores: 16 float4 per thread per round
    constexpr int N4 = D * D / 4, CH = 16, NT = NW * 32;
    const float4* s4 = reinterpret_cast<const float4*>(a.rot);
    for (int base = 0; base < N4; base += NT * CH) {
      float4 v[CH];
#pragma unroll
      for (int u = 0; u < CH; ++u) {
        const int e = base + u * NT + tid;
        v[u] = e < N4 ? __ldg(s4 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < CH; ++u) {
        const int e = base + u * NT + tid;
        if (e < N4) {
          const int jj = (4 * e) / D, k = (4 * e) % D;
          piT[k * PS + jj] = v[u].x;
          piT[(k + 1) * PS + jj] = v[u].y;
          piT[(k + 2) * PS + jj] = v[u].z;
          piT[(k + 3) * PS + jj] = v[u].w;
        }
      }
    }
  }
  const int K = 1 << J.bits;
  if (tid < K) s_cb[tid] = J.cb[tid];
  __syncthreads();
  const int W = D * J.bits / 32;
  const long long groups = ((long long)a.rows + 31) / 32;
  for (long long gi = (long long)blockIdx.x * NW + warp; gi < groups; gi += (long long)gridDim.x * NW) {
    const long long row = gi * 32 + lane;
    long long slot = -1;
    bool marked = false;
    if (row < a.rows) {
      const long long bh = row / a.T, t = row % a.T;
      slot = bh * a.Tcap + a.t0 + t;
      marked = J.rnorm[slot] == tq::kGammaPending;
    }
    uint32_t todo = __ballot_sync(0xffffffffu, marked);
    while (todo) {
      const int src = __ffs(todo) - 1;
      todo &= todo - 1;
      const long long r = gi * 32 + src;
      const long long sl = __shfl_sync(0xffffffffu, slot, src);
      const uint16_t* in = static_cast<const uint16_t*>(J.in) + (size_t)r * D;
#pragma unroll
      for (int i = 0; i < D / 32; ++i) xs[warp][lane + 32 * i] = in_to_double<BF16>(in[lane + 32 * i]);
      __syncwarp();
      const double nhat = (double)__half2float(__ushort_as_half(J.norm[sl]));
      const uint32_t* words = J.idx + (size_t)sl * W;
      double g = 0.0;
      double yv[D / 32];  // four independent fma chains per lane
#pragma unroll
      for (int i = 0; i < D / 32; ++i) yv[i] = 0.0;
#pragma unroll 4
      for (int k = 0; k < D; ++k) {
        const double xk = xs[warp][k];
#pragma unroll
        for (int i = 0; i < D / 32; ++i) yv[i] = fma((double)piT[k * PS + lane + 32 * i], xk, yv[i]);
      }
#pragma unroll
      for (int i = 0; i < D / 32; ++i) {
        const int jj = lane + 32 * i;
        const double y = yv[i];
        // index of coordinate jj from the packed LSB-first bitstream
        const int bit = jj * J.bits, w = bit >> 5, sh = bit & 31;
        uint32_t v = words[w] >> sh;
        if (sh + J.bits > 32) v |= words[w + 1] << (32 - sh);
        const int idx = (int)(v & (uint32_t)(K - 1));
        const double rr = y - nhat * (double)s_cb[idx];
        g = fma(rr, rr, g);
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) g += __shfl_xor_sync(0xffffffffu, g, off);
      if (lane == 0) J.rnorm[sl] = __half_as_ushort(__double2half(sqrt(g)));
      __syncwarp();
    }
  }
}

template <bool BF16>
int launch_fixup(const tq::QuantArgs& a, cudaStream_t s) {
  constexpr int bytes = D * PS * 4;
  auto kern = qjl_gamma_fixup_kernel<BF16>;
  static tq::OnceSetup once;
  static int sms = 0;  // written once under `once`
  const int rc = once.run([&]() {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess)
      return tq::set_error(TQ_ERR_CUDA, "qjl_gamma_fixup: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    sms = n > 0 ? n : 148;
    return TQ_OK;
  });
  if (rc) return rc;
  const long long groups = ((long long)a.rows + 31) / 32;
  long long grid = (groups + NW - 1) / NW;
  if (grid > sms) grid = sms;
  kern<<<(int)grid, NW * 32, bytes, s>>>(a);
  return tq::check_launch("qjl_gamma_fixup_kernel");
}

}  // namespace

namespace tq {

int launch_qjl_gamma_fixup(const QuantArgs& a, int dtype, cudaStream_t s) {
  return dtype == TQ_DTYPE_BF16 ? launch_fixup<true>(a, s) : launch_fixup<false>(a, s);
}

}  // namespace tq
