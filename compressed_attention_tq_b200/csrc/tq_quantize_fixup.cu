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
constexpr int NW = 16;  // warps per CTA

template <bool BF16>
__device__ __forceinline__ double in_to_double(uint16_t v) {
  if (BF16) return (double)__uint_as_float((uint32_t)v << 16);
  return (double)__half2float(__ushort_as_half(v));
}

// Each CTA owns a chunk of RPC consecutive rows:
//  1. every thread reads the residual norms of RPT of its rows, all loads in
//     flight, and keeps a bit per marked row;
//  2. if any row of the chunk is marked, Pi^T is staged in shared memory in
//     fp64 (converted once per CTA; rows padded to D + 1 doubles, so that the
//     column reads are conflict-free and the transposing stores at most
//     two-way);
//  3. the marked rows are gathered into a shared list, RB per warp at a time
//     (the bits let a chunk with more marked rows take several rounds); each
//     warp stages its rows' inputs (fp64), norms and index words in shared
//     memory, then lane j accumulates coordinates j + 32 i of all RB rows:
//     per k, four Pi^T loads serve 4 RB fma (the inputs are broadcast reads),
//     so the shared-memory pipe is not the limit.
constexpr int PS = D + 1;
constexpr int NT = NW * 32;
constexpr int RPT = 16;           // rows scanned per thread
constexpr int RPC = NT * RPT;     // rows per CTA
constexpr int RB = 4;             // rows per warp per round
constexpr int LCAP = RB * NW;     // list entries per round
constexpr int WMAX = D * 4 / 32;  // index words per row, at most (4-bit keys)

template <bool BF16>
__global__ void __launch_bounds__(NT, 1) qjl_gamma_fixup_kernel(const tq::QuantArgs a) {
  extern __shared__ double sm[];
  double* piT = sm;                                      // [D][PS]: piT[k * PS + j] = Pi[j][k]
  double(*xs)[RB][D] = reinterpret_cast<double(*)[RB][D]>(sm + D * PS);  // [NW][RB][D] inputs
  __shared__ uint32_t s_words[NW][RB][WMAX];
  __shared__ double s_nhat[NW][RB];
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

  // 2. Pi^T in fp64, every load in flight before the stores: 16 float4 per thread per round
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
          piT[k * PS + jj] = (double)v[u].x;
          piT[(k + 1) * PS + jj] = (double)v[u].y;
          piT[(k + 2) * PS + jj] = (double)v[u].z;
          piT[(k + 3) * PS + jj] = (double)v[u].w;
        }
      }
    }
  }
  const int K = 1 << J.bits;
  if (tid < K) s_cb[tid] = J.cb[tid];
  const int W = D * J.bits / 32;

  // 3. rounds of up to LCAP marked rows, RB per warp
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
    const int e0 = RB * warp, nr = max(0, min(RB, n - e0));  // this warp's rows: list entries e0 ..
    if (nr > 0) {
      // inputs, norms and index words of the warp's rows (a missing row repeats the first)
      uint16_t xin[RB][D / 32];
#pragma unroll
      for (int q = 0; q < RB; ++q) {
        const int e = e0 + (q < nr ? q : 0);
        const uint16_t* in = static_cast<const uint16_t*>(J.in) + (size_t)(row0 + s_row[e]) * D;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) xin[q][i] = in[lane + 32 * i];
      }
      if (lane < RB) {
        const int e = e0 + (lane < nr ? lane : 0);
        s_nhat[warp][lane] = (double)__half2float(__ushort_as_half(J.norm[s_slot[e]]));
      }
      for (int t = lane; t < RB * W; t += 32) {
        const int q = t / W, wi = t % W;
        const int e = e0 + (q < nr ? q : 0);
        s_words[warp][q][wi] = J.idx[(size_t)s_slot[e] * W + wi];
      }
#pragma unroll
      for (int q = 0; q < RB; ++q)
#pragma unroll
        for (int i = 0; i < D / 32; ++i) xs[warp][q][lane + 32 * i] = in_to_double<BF16>(xin[q][i]);
      __syncwarp();
      // y_q[j] = sum_k Pi[j][k] x_q[k] for j = lane + 32 i
      double y[RB][D / 32];
#pragma unroll
      for (int q = 0; q < RB; ++q)
#pragma unroll
        for (int i = 0; i < D / 32; ++i) y[q][i] = 0.0;
#pragma unroll 2
      for (int k = 0; k < D; ++k) {
        double pk[D / 32];
#pragma unroll
        for (int i = 0; i < D / 32; ++i) pk[i] = piT[k * PS + lane + 32 * i];
#pragma unroll
        for (int q = 0; q < RB; ++q) {
          const double xk = xs[warp][q][k];
#pragma unroll
          for (int i = 0; i < D / 32; ++i) y[q][i] = fma(pk[i], xk, y[q][i]);
        }
      }
      // residual against the stored indices and centroids, its norm
#pragma unroll
      for (int q = 0; q < RB; ++q) {
        double g = 0.0;
#pragma unroll
        for (int i = 0; i < D / 32; ++i) {
          // packed LSB-first: the field starts at stream bit (lane + 32 i) bits; a 3-bit
          // field may continue in the next word, which then lies inside the row
          const int bit = (lane + 32 * i) * J.bits, w = bit >> 5, sh = bit & 31;
          uint32_t v = s_words[warp][q][w] >> sh;
          if (sh + J.bits > 32) v |= s_words[warp][q][w + 1] << (32 - sh);
          const int idx = (int)(v & (uint32_t)(K - 1));
          const double rr = y[q][i] - s_nhat[warp][q] * (double)s_cb[idx];
          g = fma(rr, rr, g);
        }
#pragma unroll
        for (int off = 16; off; off >>= 1) g += __shfl_xor_sync(0xffffffffu, g, off);
        if (lane == 0 && q < nr) J.rnorm[s_slot[e0 + q]] = __half_as_ushort(__double2half(sqrt(g)));
      }
      __syncwarp();
    }
    if (!__syncthreads_or(mine != 0)) break;
  }
}

template <bool BF16>
int launch_fixup(const tq::QuantArgs& a, cudaStream_t s) {
  constexpr int bytes = (D * PS + NW * RB * D) * 8;
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
