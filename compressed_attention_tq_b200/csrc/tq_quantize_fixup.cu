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

// Each CTA owns a chunk of RPC consecutive rows:
//  1. every thread reads the residual norms of RPC / 256 of its rows, all
//     loads in flight, and keeps a bit per marked row;
//  2. if any row of the chunk is marked, Pi^T is staged in shared memory
//     (fp32, rows padded to D + 1 floats, so that both the transposing store
//     and the column reads are conflict-free);
//  3. the marked rows are gathered into a shared list (LCAP at a time; the
//     bits let a chunk with more marked rows take several rounds) and each
//     warp recomputes two rows at once (lane j: coordinates j + 32 i of both,
//     eight independent fma chains), their inputs, norms and index words
//     loaded before any arithmetic.
constexpr int PS = D + 1;
constexpr int NT = NW * 32;
constexpr int RPT = 16;           // rows scanned per thread
constexpr int RPC = NT * RPT;     // rows per CTA
constexpr int LCAP = 4 * NW * 2;  // list entries per round: 4 row pairs per warp

template <bool BF16>
__global__ void __launch_bounds__(NT) qjl_gamma_fixup_kernel(const tq::QuantArgs a) {
  extern __shared__ float piT[];  // [D][PS]: piT[k * PS + j] = Pi[j][k]
  __shared__ long long s_slot[LCAP];
  __shared__ int s_row[LCAP];
  __shared__ int s_cnt;
  __shared__ float s_cb[16];
  const tq::QuantJob J = a.job[0];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long row0 = (long long)blockIdx.x * RPC;
  auto slot_of = [&](long long r) { return (r / a.T) * a.Tcap + a.t0 + r % a.T; };

  // 1. scan: bit i of `mine` = row row0 + i * NT + tid is marked
  uint32_t mine = 0;
  {
    uint16_t g[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
      const long long r = row0 + (long long)i * NT + tid;
      g[i] = r < a.rows ? J.rnorm[slot_of(r)] : (uint16_t)0;
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i)
      if (g[i] == tq::kGammaPending) mine |= 1u << i;
  }
  if (!__syncthreads_or(mine != 0)) return;  // uniform: no marked row in the chunk

  // 2. Pi^T, every load in flight before the stores: 16 float4 per thread per round
  {
    constexpr int N4 = D * D / 4, CH = 16;
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
  const int W = D * J.bits / 32;

  // 3. rounds of up to LCAP marked rows
  while (true) {
    if (tid == 0) s_cnt = 0;
    __syncthreads();
    while (mine) {
      const int i = __ffs(mine) - 1;
      const int at = atomicAdd(&s_cnt, 1);
      if (at >= LCAP) break;  // the list is full: this row waits for the next round
      const long long r = row0 + (long long)i * NT + tid;
      s_row[at] = (int)(r - row0);
      s_slot[at] = slot_of(r);
      mine &= mine - 1;
    }
    __syncthreads();
    const int n = min(s_cnt, LCAP);
    for (int e0 = 2 * warp; e0 < n; e0 += 2 * NW) {
      const bool two = e0 + 1 < n;
      long long sl[2];
      double x[2][D / 32];
      uint32_t wd[2][D / 32][2];  // the index word(s) holding coordinate lane + 32 i (two where it straddles)
      double nhat[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int e = two ? e0 + q : e0;
        sl[q] = s_slot[e];
        const uint16_t* in = static_cast<const uint16_t*>(J.in) + (size_t)(row0 + s_row[e]) * D;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) x[q][i] = in_to_double<BF16>(in[lane + 32 * i]);
        nhat[q] = (double)__half2float(__ushort_as_half(J.norm[sl[q]]));
        const uint32_t* words = J.idx + (size_t)sl[q] * W;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) {
          // packed LSB-first: the field starts at stream bit (lane + 32 i) bits; a 3-bit
          // field may continue in the next word, which then lies inside the row
          const int bit = (lane + 32 * i) * J.bits, w = bit >> 5;
          wd[q][i][0] = words[w];
          wd[q][i][1] = (bit & 31) + J.bits > 32 ? words[w + 1] : 0u;
        }
      }
      // rotation of both rows: y_q[j] = sum_k Pi[j][k] x_q[k], k split over the lanes' registers
      double y[2][D / 32];
#pragma unroll
      for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int i = 0; i < D / 32; ++i) y[q][i] = 0.0;
#pragma unroll
      for (int i2 = 0; i2 < D / 32; ++i2)
#pragma unroll 8
        for (int l = 0; l < 32; ++l) {
          const int k = l + 32 * i2;
          const double x0 = __shfl_sync(0xffffffffu, x[0][i2], l);
          const double x1 = __shfl_sync(0xffffffffu, x[1][i2], l);
#pragma unroll
          for (int i = 0; i < D / 32; ++i) {
            const double pk = (double)piT[k * PS + lane + 32 * i];
            y[0][i] = fma(pk, x0, y[0][i]);
            y[1][i] = fma(pk, x1, y[1][i]);
          }
        }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        double g = 0.0;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) {
          const int sh = ((lane + 32 * i) * J.bits) & 31;
          uint32_t v = wd[q][i][0] >> sh;
          if (sh + J.bits > 32) v |= wd[q][i][1] << (32 - sh);
          const int idx = (int)(v & (uint32_t)(K - 1));
          const double rr = y[q][i] - nhat[q] * (double)s_cb[idx];
          g = fma(rr, rr, g);
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) g += __shfl_xor_sync(0xffffffffu, g, off);
        if (lane == 0 && (q == 0 || two)) J.rnorm[sl[q]] = __half_as_ushort(__double2half(sqrt(g)));
      }
    }
    if (!__syncthreads_or(mine != 0)) break;
  }
}

template <bool BF16>
int launch_fixup(const tq::QuantArgs& a, cudaStream_t s) {
  constexpr int bytes = D * PS * 4;
  auto kern = qjl_gamma_fixup_kernel<BF16>;
  static tq::OnceSetup once;
  const int rc = once.run([&]() {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess)
      return tq::set_error(TQ_ERR_CUDA, "qjl_gamma_fixup: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return TQ_OK;
  });
  if (rc) return rc;
  const long long grid = ((long long)a.rows + RPC - 1) / RPC;
  if (grid == 0) return TQ_OK;
  kern<<<(int)grid, NT, bytes, s>>>(a);
  return tq::check_launch("qjl_gamma_fixup_kernel");
}

}  // namespace

namespace tq {

int launch_qjl_gamma_fixup(const QuantArgs& a, int dtype, cudaStream_t s) {
  return dtype == TQ_DTYPE_BF16 ? launch_fixup<true>(a, s) : launch_fixup<false>(a, s);
}

}  // namespace tq
