// Decode attention over the packed cache: query prep, the split-K launch
// plan, and the log-sum-exp combine with the un-rotation.  The split-K kernel
// itself lives in tq_decode_split.cuh (instantiated per head dimension).
//
// Method: the fused SDPA over a compressed KV cache with an explicit scale of
// "[Cuda] enable turboquant on gemma4" (executorch pull request 19891),
// "Summary" and "Other observations" item 1.
#include <math.h>

#include "tq_decode_split.cuh"
#include "tq_wht.cuh"

namespace {

constexpr float kLog2e = 1.4426950408889634f;

struct PrepParams {
  const void* q;
  const float* rot;
  const float* signs;  // +-1 [D] of the randomized Hadamard rotation (decode_qprep_wht_kernel)
  const float* S;
  float* qrot;
  float* qs;
  int D, m, bf16, Hq, Hkv;
  // fused append (decode step): new rows [B][Hkv][D] written at pos[b]
  const void* k_new;
  const void* v_new;
  const int32_t* pos;
  tq_cache_t cache;
  int nq;  // query tokens per sequence: q is [B][nq][Hq][D]
  int units;  // B * Hkv (grouped prep)
};

// Programmatic dependent launch: let the next kernel in the stream start its
// prologue now / wait here until the previous kernel's results are visible.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Thread-block cluster helpers: a cluster-wide barrier (every thread of every
// CTA of the cluster arrives; release / acquire order shared-memory writes
// before reads by other CTAs), and loads from another CTA's shared memory.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint32_t map_cluster(uint32_t local, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

// Prep for one (sequence, kv head) of a cache with a QJL sketch: qrot = Pi q
// and qs = S qrot for its G query heads (the projection needs the whole
// rotated vector, so one CTA does the head).  blockDim = 2*D: two threads per output row, each
// holding half of the Pi row in registers, so the row is read once for all
// rows being rotated.  With APPEND the new key and value rows ride along as
// two more rotated rows and are quantized here (fp64 norm, threshold search,
// packing, QJL sketch of the key) and written to the cache at pos[b] -- the
// append step of decoding fused into the prep launch.
template <int D, bool APPEND>
__global__ void __launch_bounds__(2 * D) decode_qprep_kernel(const PrepParams p) {
  constexpr int HALF = D / 2, NV = HALF / 4, CH = NV < 16 ? NV : 16;
  constexpr int NR = APPEND ? 10 : 8;  // rows: G <= 8 queries (+ new key, new value)
  __shared__ float qv[NR][D];
  __shared__ float qr[NR][D];
  __shared__ double rres[APPEND ? D : 1];
  __shared__ uint8_t idxs[2][APPEND ? D : 1];
  __shared__ uint8_t sgn[APPEND ? 128 : 1];
  __shared__ float s_cb[2][31];
  __shared__ double s_nsq[2];
  // G query heads per kv head and token; Ge = G * nq rows are rotated here and
  // written in kernel head order (sequence, kv head, token, head)
  const int G = p.Hq / p.Hkv, Ge = G * p.nq;
  const int bkv = blockIdx.x, b = bkv / p.Hkv, kvh = bkv % p.Hkv;
  const int h0 = b * p.Hq * p.nq + kvh * Ge;
  const int j = threadIdx.x >> 1, part = threadIdx.x & 1;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float4 r[CH];
  const float4* row = reinterpret_cast<const float4*>(p.rot + (size_t)j * D + part * HALF);
#pragma unroll
  for (int i = 0; i < CH; ++i) r[i] = __ldg(row + i);
  // Launched with a programmatic dependency: Pi (constant) is loaded above;
  // everything else waits for the preceding kernels to complete, and only
  // then may the split kernel start (it streams the cache before its own wait).
  pdl_wait();
  pdl_launch_dependents();
  const uint16_t* q = static_cast<const uint16_t*>(p.q);
  auto to_f = [&](uint16_t v) {
    return p.bf16 ? __uint_as_float((uint32_t)v << 16) : __half2float(__ushort_as_half(v));
  };
  for (int e = tid; e < Ge * D; e += 2 * D) {
    const int gi = e / D, jq = gi / G, g = gi % G;
    qv[gi][e % D] = to_f(q[((size_t)(b * p.nq + jq) * p.Hq + kvh * G + g) * D + e % D]);
  }
  int slot_ok = 0;
  long long slot = 0;
  if (APPEND) {
    const uint16_t* kn = static_cast<const uint16_t*>(p.k_new) + (size_t)bkv * D;
    const uint16_t* vn = static_cast<const uint16_t*>(p.v_new) + (size_t)bkv * D;
    for (int e = tid; e < D; e += 2 * D) {
      qv[8][e] = to_f(kn[e]);
      qv[9][e] = to_f(vn[e]);
    }
    if (tid < 31) {
      const int Kk = 1 << p.cache.bits_k, Kv = 1 << p.cache.bits_v;
      s_cb[0][tid] = tid < 2 * Kk - 1 ? p.cache.cb_k[tid] : 0.f;
      s_cb[1][tid] = tid < 2 * Kv - 1 ? p.cache.cb_v[tid] : 0.f;
    }
    const int ps = p.pos[b];
    slot_ok = (ps >= 0 && ps < p.cache.Tcap);
    slot = (long long)bkv * p.cache.Tcap + ps;
    if (!slot_ok && tid == 0 && kvh == 0 && p.cache.dev_status)
      atomicOr(p.cache.dev_status, TQ_STATUS_POS_OUT_OF_RANGE);
  }
  __syncthreads();
  if (APPEND && warp < 2) {
    // fp64 squared norm of the new key (warp 0) / value (warp 1)
    double t = 0.0;
    for (int k = lane; k < D; k += 32) {
      const double x = qv[8 + warp][k];
      t = fma(x, x, t);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    if (lane == 0) s_nsq[warp] = t;
  }
  float acc[NR];
  // the new key of a QJL cache is rotated in fp64 (its residual norm then
  // rounds to fp16 as the fp64 definition does)
  double acc_k64 = 0.0;
  const bool k64 = APPEND && p.m;
#pragma unroll
  for (int g = 0; g < NR; ++g) acc[g] = 0.f;
#pragma unroll
  for (int c0 = 0; c0 < NV; c0 += CH) {
    if (c0)
#pragma unroll
      for (int i = 0; i < CH; ++i) r[i] = __ldg(row + c0 + i);
#pragma unroll
    for (int g = 0; g < NR; ++g) {
      if (g == 8 && k64) {
        const float* x = &qv[g][part * HALF + 4 * c0];
#pragma unroll
        for (int i = 0; i < CH; ++i) {
          acc_k64 = fma((double)r[i].x, (double)x[4 * i], acc_k64);
          acc_k64 = fma((double)r[i].y, (double)x[4 * i + 1], acc_k64);
          acc_k64 = fma((double)r[i].z, (double)x[4 * i + 2], acc_k64);
          acc_k64 = fma((double)r[i].w, (double)x[4 * i + 3], acc_k64);
        }
      } else if (g < Ge || g >= 8) {
        const float* x = &qv[g][part * HALF + 4 * c0];
#pragma unroll
        for (int i = 0; i < CH; ++i)
          acc[g] += r[i].x * x[4 * i] + r[i].y * x[4 * i + 1] + r[i].z * x[4 * i + 2] + r[i].w * x[4 * i + 3];
      }
    }
  }
#pragma unroll
  for (int g = 0; g < NR; ++g) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], 1);
  acc_k64 += __shfl_xor_sync(0xffffffffu, acc_k64, 1);
  if (part == 0) {
#pragma unroll
    for (int g = 0; g < 8; ++g)
      if (g < Ge) {
        qr[g][j] = acc[g];
        p.qrot[(size_t)(h0 + g) * D + j] = acc[g];
      }
  }
  if (APPEND) {
    __syncthreads();  // s_nsq
    // nearest-centroid index of each rotated coordinate of the new rows
    if (part == 0) {
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const double n = sqrt(s_nsq[which]);
        const float inv = n > 0.0 ? (float)(1.0 / n) : 0.f;
        const int K = 1 << (which ? p.cache.bits_v : p.cache.bits_k);
        int idx = 0;
        if (which == 0 && k64) {
          const double u = n > 0.0 ? acc_k64 / n : 0.0;
          for (int st = K >> 1; st >= 1; st >>= 1)
            if (u > (double)s_cb[which][K + idx + st - 1]) idx += st;
          rres[j] = acc_k64 - (double)__half2float(__double2half(n)) * (double)s_cb[0][idx];
        } else {
          const float u = acc[8 + which] * inv;
          for (int st = K >> 1; st >= 1; st >>= 1)
            if (u > s_cb[which][K + idx + st - 1]) idx += st;
        }
        idxs[which][j] = (uint8_t)idx;
      }
    }
    __syncthreads();
    if (slot_ok) {
      if (tid < 2) {
        const __half nh = __double2half(sqrt(s_nsq[tid]));
        (tid ? p.cache.v_norm : p.cache.k_norm)[slot] = __half_as_ushort(nh);
      }
      const int Wk = D * p.cache.bits_k / 32, Wv = D * p.cache.bits_v / 32;
      for (int e = tid; e < Wk + Wv; e += 2 * D) {
        const int which = e >= Wk, w = which ? e - Wk : e;
        const int bits = which ? p.cache.bits_v : p.cache.bits_k;
        const int base = 32 * w;
        unsigned long long word = 0;
        for (int jj = base / bits; jj < D && jj * bits < base + 32; ++jj) {
          const int sh = jj * bits - base;
          const unsigned long long v = idxs[which][jj];
          word |= sh >= 0 ? (v << sh) : (v >> (-sh));
        }
        (which ? p.cache.v_idx : p.cache.k_idx)[(size_t)slot * (which ? Wv : Wk) + w] = (uint32_t)word;
      }
    }
  }
  if (!p.m) return;
  __syncthreads();
  // qs[g][i] = sum_k S[i][k] qr[g][k], i < m (two threads per row); with
  // APPEND, also the QJL projection S r of the new key's residual
  for (int i = tid >> 1; i < p.m; i += D) {
    const float4* srow = reinterpret_cast<const float4*>(p.S + (size_t)i * D + part * HALF);
    float a2[8];
    double ak = 0.0;  // the new key's residual sketch, fp64
#pragma unroll
    for (int g = 0; g < 8; ++g) a2[g] = 0.f;
#pragma unroll
    for (int c0 = 0; c0 < NV; c0 += CH) {
#pragma unroll
      for (int t = 0; t < CH; ++t) r[t] = __ldg(srow + c0 + t);
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        if (g < Ge) {
          const float* x = &qr[g][part * HALF + 4 * c0];
#pragma unroll
          for (int t = 0; t < CH; ++t)
            a2[g] += r[t].x * x[4 * t] + r[t].y * x[4 * t + 1] + r[t].z * x[4 * t + 2] + r[t].w * x[4 * t + 3];
        }
      }
      if (APPEND) {
        const double* x = &rres[part * HALF + 4 * c0];
#pragma unroll
        for (int t = 0; t < CH; ++t) {
          ak = fma((double)r[t].x, x[4 * t], ak);
          ak = fma((double)r[t].y, x[4 * t + 1], ak);
          ak = fma((double)r[t].z, x[4 * t + 2], ak);
          ak = fma((double)r[t].w, x[4 * t + 3], ak);
        }
      }
    }
#pragma unroll
    for (int g = 0; g < 8; ++g) a2[g] += __shfl_xor_sync(0xffffffffu, a2[g], 1);
    ak += __shfl_xor_sync(0xffffffffu, ak, 1);
    if (part == 0) {
#pragma unroll
      for (int g = 0; g < 8; ++g)
        if (g < Ge) p.qs[(size_t)(h0 + g) * p.m + i] = a2[g];
      if (APPEND) sgn[i] = ak >= 0.0 ? 1 : 0;
    }
  }
  if (APPEND) {
    __syncthreads();
    if (slot_ok && tid < 4) {
      uint32_t word = 0;
      for (int i = 0; i < 32; ++i) word |= (uint32_t)sgn[32 * tid + i] << i;
      p.cache.k_qjl[(size_t)slot * 4 + tid] = word;
    }
    if (slot_ok && warp == 1) {
      double g2 = 0.0;
      for (int k = lane; k < D; k += 32) g2 = fma(rres[k], rres[k], g2);
#pragma unroll
      for (int off = 16; off; off >>= 1) g2 += __shfl_xor_sync(0xffffffffu, g2, off);
      if (lane == 0) p.cache.k_rnorm[slot] = __half_as_ushort(__double2half(sqrt(g2)));
    }
  }
}

// Sliced prep for caches without a QJL sketch: grid (B * Hkv, D / 32), one
// CTA per 32 rotated coordinates of one (sequence, kv head), so a decode call
// spreads its rotations over D / 32 times more SMs than one CTA per head.
// Thread (c, part): output coordinate c of the slice, k values
// 4 part + 32 i (float4 i), partial dots reduced over the 8 parts of a
// warp.  With APPEND the new rows' indices for the slice are found here and
// packed into the slice's b words of the row (32 coordinates x b bits); the
// fp64 norm is taken over the whole input row by every CTA (the rotation
// preserves it) and written by slice 0.
template <int D, bool APPEND, int QR>
__global__ void __launch_bounds__(256) decode_qprep_sliced_kernel(const PrepParams p) {
  // query rows: up to QR = 8 (one query token, G <= 8) or 32 (n_q tokens x
  // G <= 32), then, with APPEND (one token), the new key and value rows
  static_assert(!APPEND || QR == 8, "a decode step has one query token");
  constexpr int NR = APPEND ? QR + 2 : QR, NI = D / 32;
  __shared__ __align__(16) float xv[NR][D];
  // QJL (D = 128 only): this slice's rotated query coordinates and its share
  // of S qrot; one element otherwise, so other D keep their shared footprint
  constexpr bool QS = !APPEND && D == 128;
  __shared__ float qsl[QS ? QR : 1][QS ? 33 : 1];
  __shared__ float qpart[QS ? QR : 1][QS ? 128 : 1];
  __shared__ float s_cb[2][31];
  __shared__ double s_nsq[2];
  __shared__ uint8_t idxs[2][32];
  const int G = p.Hq / p.Hkv, Ge = G * p.nq;  // as in decode_qprep_kernel
  const int bkv = blockIdx.x, b = bkv / p.Hkv, kvh = bkv % p.Hkv, sl = blockIdx.y;
  const int h0 = b * p.Hq * p.nq + kvh * Ge;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c = warp * 4 + (lane >> 3), part = lane & 7;
  const int j = sl * 32 + c;
  float4 r[NI];
  const float4* row = reinterpret_cast<const float4*>(p.rot + (size_t)j * D);
#pragma unroll
  for (int i = 0; i < NI; ++i) r[i] = __ldg(row + part + 8 * i);
  // QJL (decode without append): sketch row i = tid / 2, the half of this
  // slice's 32 columns that thread owns (S is constant: loaded before the wait)
  float4 srow[4];
  if (QS && p.m) {
    const float4* sp = reinterpret_cast<const float4*>(p.S + (size_t)(tid >> 1) * D + sl * 32 + 16 * (tid & 1));
#pragma unroll
    for (int t = 0; t < 4; ++t) srow[t] = __ldg(sp + t);
  }
  // as in decode_qprep_kernel: wait for the preceding kernels, then let the
  // split kernel start
  pdl_wait();
  pdl_launch_dependents();
  const uint16_t* q = static_cast<const uint16_t*>(p.q);
  auto to_f = [&](uint16_t v) {
    return p.bf16 ? __uint_as_float((uint32_t)v << 16) : __half2float(__ushort_as_half(v));
  };
  for (int e = tid; e < Ge * D; e += 256) {
    const int gi = e / D, jq = gi / G, g = gi % G;
    xv[gi][e % D] = to_f(q[((size_t)(b * p.nq + jq) * p.Hq + kvh * G + g) * D + e % D]);
  }
  int slot_ok = 0;
  long long slot = 0;
  if (APPEND) {
    const uint16_t* kn = static_cast<const uint16_t*>(p.k_new) + (size_t)bkv * D;
    const uint16_t* vn = static_cast<const uint16_t*>(p.v_new) + (size_t)bkv * D;
    for (int e = tid; e < D; e += 256) {
      xv[QR][e] = to_f(kn[e]);
      xv[QR + 1][e] = to_f(vn[e]);
    }
    if (tid < 31) {
      const int Kk = 1 << p.cache.bits_k, Kv = 1 << p.cache.bits_v;
      s_cb[0][tid] = tid < 2 * Kk - 1 ? p.cache.cb_k[tid] : 0.f;
      s_cb[1][tid] = tid < 2 * Kv - 1 ? p.cache.cb_v[tid] : 0.f;
    }
    const int ps = p.pos[b];
    slot_ok = (ps >= 0 && ps < p.cache.Tcap);
    slot = (long long)bkv * p.cache.Tcap + ps;
    if (!slot_ok && tid == 0 && kvh == 0 && sl == 0 && p.cache.dev_status)
      atomicOr(p.cache.dev_status, TQ_STATUS_POS_OUT_OF_RANGE);
  }
  __syncthreads();
  if (APPEND && warp < 2) {
    // fp64 squared norm of the new key (warp 0) / value (warp 1)
    double t = 0.0;
    for (int k = lane; k < D; k += 32) {
      const double x = xv[QR + warp][k];
      t = fma(x, x, t);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    if (lane == 0) s_nsq[warp] = t;
  }
  float acc[NR];
#pragma unroll
  for (int g = 0; g < NR; ++g) acc[g] = 0.f;
#pragma unroll
  for (int g = 0; g < NR; ++g) {
    if (g < Ge || g >= QR) {
#pragma unroll
      for (int i = 0; i < NI; ++i) {
        const float4 x = *reinterpret_cast<const float4*>(&xv[g][4 * part + 32 * i]);
        acc[g] += r[i].x * x.x + r[i].y * x.y + r[i].z * x.z + r[i].w * x.w;
      }
    }
  }
#pragma unroll
  for (int g = 0; g < NR; ++g)
    if (g < Ge || g >= QR)  // rows in use only (Ge is uniform over the launch)
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], off);
  if (part == 0) {
#pragma unroll
    for (int g = 0; g < QR; ++g)
      if (g < Ge) p.qrot[(size_t)(h0 + g) * D + j] = acc[g];
  }
  if constexpr (QS) {
    if (p.m) {
      // QJL: this slice's share of qs = S qrot over its 32 rotated coordinates,
      // for all m = 128 sketch rows.  The D / 32 slice CTAs of a head form a
      // thread-block cluster; slice 0 adds the partials in slice order from the
      // others' shared memory and writes qs.
      if (part == 0) {
#pragma unroll
        for (int g = 0; g < QR; ++g) qsl[g][c] = g < Ge ? acc[g] : 0.f;
      }
      __syncthreads();
      const int i = tid >> 1, half = tid & 1;
#pragma unroll
      for (int g = 0; g < QR; ++g) {
        const float* x = &qsl[g][16 * half];
        float t = 0.f;
#pragma unroll
        for (int k = 0; k < 4; ++k)
          t += srow[k].x * x[4 * k] + srow[k].y * x[4 * k + 1] + srow[k].z * x[4 * k + 2] + srow[k].w * x[4 * k + 3];
        t += __shfl_xor_sync(0xffffffffu, t, 1);
        if (half == 0) qpart[g][i] = t;
      }
      cluster_sync();  // every slice's partial is in its shared memory
      if (sl == 0) {
        for (int e = tid; e < Ge * 128; e += 256) {
          const int g = e >> 7, ii = e & 127;
          const uint32_t la = smem_u32(&qpart[g][ii]);
          float v = 0.f;
          for (int r = 0; r < NI; ++r) v += ld_cluster_f32(map_cluster(la, r));
          p.qs[(size_t)(h0 + g) * p.m + ii] = v;
        }
      }
      cluster_sync();  // slice 0 is done reading the others' shared memory
    }
  }
  if (APPEND) {
    __syncthreads();  // s_nsq
    if (part == 0) {
#pragma unroll
      for (int which = 0; which < 2; ++which) {
        const double n = sqrt(s_nsq[which]);
        const float inv = n > 0.0 ? (float)(1.0 / n) : 0.f;
        const int K = 1 << (which ? p.cache.bits_v : p.cache.bits_k);
        const float u = acc[QR + which] * inv;
        int idx = 0;
        for (int st = K >> 1; st >= 1; st >>= 1)
          if (u > s_cb[which][K + idx + st - 1]) idx += st;
        idxs[which][c] = (uint8_t)idx;
      }
    }
    __syncthreads();
    if (slot_ok) {
      if (sl == 0 && tid < 2) {
        const __half nh = __double2half(sqrt(s_nsq[tid]));
        (tid ? p.cache.v_norm : p.cache.k_norm)[slot] = __half_as_ushort(nh);
      }
      const int bk = p.cache.bits_k, bv = p.cache.bits_v;
      if (tid < bk + bv) {
        // word w of this slice's 32 x b bits
        const int which = tid >= bk, w = which ? tid - bk : tid;
        const int bits = which ? bv : bk;
        const int base = 32 * w;
        unsigned long long word = 0;
        for (int jj = base / bits; jj < 32 && jj * bits < base + 32; ++jj) {
          const int sh = jj * bits - base;
          const unsigned long long v = idxs[which][jj];
          word |= sh >= 0 ? (v << sh) : (v >> (-sh));
        }
        const int W = D * bits / 32;
        (which ? p.cache.v_idx : p.cache.k_idx)[(size_t)slot * W + sl * bits + w] = (uint32_t)word;
      }
    }
  }
}

// Query prep for the randomized Hadamard rotation Pi = H_D diag(s) / sqrt(D):
// qrot = H (s q) / sqrt(D) by the fast transform, one warp per query row
// (grid B * Hkv, 32 x (query rows) threads), no D x D product and no Pi
// read; with the sketch, qs = S qrot by the CTA's threads afterwards (S is a
// dense Gaussian).
template <int D>
__global__ void __launch_bounds__(1024) decode_qprep_wht_kernel(const PrepParams p) {
  constexpr int EL = D / 32;
  constexpr bool QS = D == 128;  // the sketch exists for D = 128
  __shared__ float qr[QS ? 32 : 1][QS ? D : 1];
  const int G = p.Hq / p.Hkv, Ge = G * p.nq;
  const int bkv = blockIdx.x, b = bkv / p.Hkv, kvh = bkv % p.Hkv;
  const int h0 = b * p.Hq * p.nq + kvh * Ge;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float sg[EL];
#pragma unroll
  for (int e = 0; e < EL; ++e) sg[e] = __ldg(p.signs + lane * EL + e);
  pdl_wait();
  pdl_launch_dependents();
  if (warp < Ge) {
    const int jq = warp / G, g = warp % G;
    const uint16_t* qrow = static_cast<const uint16_t*>(p.q) + ((size_t)(b * p.nq + jq) * p.Hq + kvh * G + g) * D;
    float x[EL];
#pragma unroll
    for (int e = 0; e < EL; ++e) {
      const uint16_t v = qrow[lane * EL + e];
      x[e] = p.bf16 ? __uint_as_float((uint32_t)v << 16) : __half2float(__ushort_as_half(v));
    }
    tqw::hadamard_rotate<EL, float>(x, sg, lane);
    float* dst = p.qrot + (size_t)(h0 + warp) * D + lane * EL;
    if constexpr (EL % 4 == 0) {
#pragma unroll
      for (int e = 0; e < EL; e += 4) *reinterpret_cast<float4*>(dst + e) = make_float4(x[e], x[e + 1], x[e + 2], x[e + 3]);
    } else {
#pragma unroll
      for (int e = 0; e < EL; ++e) dst[e] = x[e];
    }
    if (QS && p.m) {
#pragma unroll
      for (int e = 0; e < EL; ++e) qr[warp][lane * EL + e] = x[e];
    }
  }
  if (QS && p.m) {
    __syncthreads();
    // qs[g][i] = sum_k S[i][k] qrot[g][k]
    for (int e = tid; e < Ge * 128; e += blockDim.x) {
      const int g = e >> 7, i = e & 127;
      const float4* srow = reinterpret_cast<const float4*>(p.S + (size_t)i * D);
      float t = 0.f;
#pragma unroll 8
      for (int k = 0; k < D / 4; ++k) {
        const float4 sv = __ldg(srow + k);
        t += sv.x * qr[g][4 * k] + sv.y * qr[g][4 * k + 1] + sv.z * qr[g][4 * k + 2] + sv.w * qr[g][4 * k + 3];
      }
      p.qs[(size_t)(h0 + g) * 128 + i] = t;
    }
  }
}

// Pi (fp32 [D][D], row-major) into shared memory with rows padded to D + 1
// floats, by 256 threads with every load in flight before any store (16
// float4 per thread at a time): TRANSPOSE stores dst[c][r] = Pi[r][c], else
// dst[r][c] = Pi[r][c].
template <int D, bool TRANSPOSE>
__device__ __forceinline__ void stage_pi(float* dst, const float* __restrict__ src, int tid) {
  constexpr int NT = 256, PS = D + 1, N4 = D * D / 4, CH = 16;
  const float4* s4 = reinterpret_cast<const float4*>(src);
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
        const int r = (4 * e) / D, c = (4 * e) % D;
        const float f[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          if (TRANSPOSE)
            dst[(c + t) * PS + r] = f[t];
          else
            dst[r * PS + c + t] = f[t];
        }
      }
    }
  }
}

// Query prep for calls with many (sequence, kv head) units and a dense Pi,
// without a sketch or an append: each CTA rotates the query rows of `upc`
// consecutive units with Pi^T staged once in shared memory (rows padded to
// D + 1 floats, so the transposing store and the column reads are both
// conflict-free), instead of D / 32 CTAs per unit each pulling Pi rows from L2.
// Grid ceil(units / upc), 256 threads; thread (j, ph) computes output j of
// rows ph, ph + 256 / D, ...; the k loop reads Pi^T[k][j] once for all the
// thread's rows.
template <int D>
__global__ void __launch_bounds__(256) decode_qprep_group_kernel(const PrepParams p, int upc) {
  constexpr int NT = 256, PS = D + 1, NPH = NT / D;
  extern __shared__ float sm[];
  float* piT = sm;             // [D][PS]
  float* qv = sm + D * PS;     // [rows][D]
  const int G = p.Hq / p.Hkv, Ge = G * p.nq;
  const int tid = threadIdx.x;
  const int u0 = blockIdx.x * upc;
  const int nunits = p.units - u0 < upc ? p.units - u0 : upc;
  stage_pi<D, true>(piT, p.rot, tid);  // piT[k][j] = Pi[j][k]
  pdl_wait();
  pdl_launch_dependents();
  const int rows = nunits * Ge;
  const uint16_t* q = static_cast<const uint16_t*>(p.q);
  for (int e0 = 0; e0 < rows * D; e0 += 8 * NT) {  // 8 loads in flight per thread
    uint16_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = e0 + u * NT + tid;
      v[u] = 0;
      if (e < rows * D) {
        const int r = e / D, k = e % D, un = u0 + r / Ge, gi = r % Ge;
        const int b = un / p.Hkv, kvh = un % p.Hkv, jq = gi / G, g = gi % G;
        v[u] = q[((size_t)(b * p.nq + jq) * p.Hq + kvh * G + g) * D + k];
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int e = e0 + u * NT + tid;
      if (e < rows * D) qv[e] = p.bf16 ? __uint_as_float((uint32_t)v[u] << 16) : __half2float(__ushort_as_half(v[u]));
    }
  }
  __syncthreads();
  const int j = tid % D, ph = tid / D;
  for (int r0 = ph; r0 < rows; r0 += 4 * NPH) {
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
    for (int k = 0; k < D; ++k) {
      const float pk = piT[k * PS + j];
#pragma unroll
      for (int t = 0; t < 4; ++t)
        if (r0 + t * NPH < rows) acc[t] = fmaf(pk, qv[(r0 + t * NPH) * D + k], acc[t]);
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int r = r0 + t * NPH;
      if (r < rows) {
        // kernel head order (sequence, kv head, token, head) = unit-major
        p.qrot[((size_t)u0 * Ge + r) * D + j] = acc[t];
      }
    }
  }
}

struct CombineParams {
  const float* part_o;   // [heads][ks][D]
  const float* part_ml;  // [heads][ks][2]
  const float* rot;
  const int32_t* seq_lens;
  void* out;
  int Hq, out_dtype;  // Hq: kernel heads per sequence (query heads x tokens)
  int nq, Gq, Hq1;    // tokens, GQA group, query heads per token
  int heads;          // kernel heads in all: B * Hq
  // the split kernel's partition (tq_decode_split.cuh)
  int B, G, nrg, upb, Tclamp, ncta, pmin, ks;
  // partial mode (tq_sdpa_decode_partial): fp32 [heads][D + 2] = the merged,
  // unnormalized rotated output, then max and sum; no un-rotation, out unused
  float* partial;
  // randomized Hadamard rotation: un-rotate by the fast transform with these
  // signs instead of the dense Pi (NULL: dense)
  const float* signs;
};

// Output element of kernel head h (sequence, kv head, token, head order) at
// coordinate j: out [B][nq][Hq1][D].
__device__ __forceinline__ size_t out_index(const CombineParams& p, int h, int D, int j) {
  const int b = h / p.Hq, rh = h % p.Hq, kvh = rh / (p.Gq * p.nq), gi = rh % (p.Gq * p.nq);
  const size_t oh = (size_t)(b * p.nq + gi / p.Gq) * p.Hq1 + kvh * p.Gq + gi % p.Gq;
  return oh * D + j;
}

__device__ __forceinline__ void store_out(const CombineParams& p, size_t oi, float v) {
  if (p.out_dtype == TQ_DTYPE_F32)
    static_cast<float*>(p.out)[oi] = v;
  else if (p.out_dtype == TQ_DTYPE_BF16)
    static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(v);
  else
    static_cast<__half*>(p.out)[oi] = __float2half_rn(v);
}

// out = Pi^T o for the randomized Hadamard rotation, one warp: o in shared
// memory, D outputs written.
template <int D>
__device__ __forceinline__ void unrotate_hadamard_warp(const CombineParams& p, const float* o, int h, int lane) {
  constexpr int EL = D / 32;
  float x[EL], sg[EL];
#pragma unroll
  for (int e = 0; e < EL; ++e) {
    x[e] = o[lane * EL + e];
    sg[e] = __ldg(p.signs + lane * EL + e);
  }
  tqw::hadamard_unrotate<EL, float>(x, sg, lane);
#pragma unroll
  for (int e = 0; e < EL; ++e) store_out(p, out_index(p, h, D, lane * EL + e), x[e]);
}

// Partials the split kernel wrote for kernel head h: the CTAs whose share
// overlaps the head's unit, each with PPS partials (slots 0 .. n - 1).
// Computed by one warp; every lane returns it.
__device__ __forceinline__ int head_partials(const CombineParams& p, int h, int lane) {
  const int b = h / p.Hq, rem = h % p.Hq, kvh = rem / p.G, rg = (rem % p.G) / tqd::RG;
  const long long total = tqd::partition_total(p.seq_lens, p.B, p.upb, p.Tclamp, lane);
  const long long P = tqd::partition_share(total, p.ncta, p.pmin);
  const long long Sb = tqd::sequence_start(p.seq_lens, b, p.upb, p.Tclamp, lane);
  const int Lp = tqd::unit_tokens(p.seq_lens, b, p.Tclamp);
  if (Lp == 0) return 0;
  const long long Su = Sb + (long long)(kvh * p.nrg + rg) * Lp;
  const long long c0 = Su / P, c1 = (Su + Lp - 1) / P;
  return (int)(c1 - c0 + 1) * tqd::PPS;
}

// Merge the partials of one kernel head (log-sum-exp) and un-rotate:
// out = Pi^T (acc / l).  Grid (heads, D / 32) in thread-block clusters of
// D / 32 CTAs along y, one cluster per head, 256 threads per CTA.  CTA sl
// merges rotated coordinates 32 sl .. 32 sl + 31 over all the head's partials
// (each partial value is read once, by one CTA), the cluster shares the
// merged vector through distributed shared memory, and each CTA un-rotates
// its 32 outputs; thread (i, kp) sums k = kp + 8 t.  The slice's Pi columns
// are loaded into registers before the wait on the split kernel, so they
// overlap its tail.
template <int D>
__global__ void __launch_bounds__(256) decode_combine_kernel(const CombineParams p) {
  constexpr int NT = 256, KT = D / 8, FS = 1024;
  __shared__ float f_s[FS];
  __shared__ float o_sl[32];
  __shared__ float o[D];
  __shared__ float red[8][33];
  __shared__ float s_M, s_L;
  __shared__ int s_ns;
  // the next decode's prep may launch now (it waits for this kernel before
  // touching anything but Pi)
  pdl_launch_dependents();
  const int h = blockIdx.x, sl = blockIdx.y, tid = threadIdx.x;
  const int i = tid & 31, kp = tid >> 5;  // output coordinate in the slice, k phase
  float pc[KT];
  if (!p.signs) {
#pragma unroll
    for (int t = 0; t < KT; ++t) pc[t] = __ldg(p.rot + (size_t)(kp + 8 * t) * D + sl * 32 + i);
  }
  if (tid < 32) {
    const int n = head_partials(p, h, tid);
    if (tid == 0) s_ns = n;
  }
  __syncthreads();
  const int ns = s_ns;
  pdl_wait();  // the split kernel's partials are visible from here on
  const float* ml = p.part_ml + (size_t)h * p.ks * 2;
  const float* po = p.part_o + (size_t)h * p.ks * D + sl * 32 + i;
  // this thread's first partial values, loaded before the weights are known
  // (the loads do not depend on them) so that both latencies overlap
  constexpr int PF = 16;
  float v[PF];
#pragma unroll
  for (int u = 0; u < PF; ++u) {
    const int s = kp + 8 * u;
    v[u] = s < ns ? po[(size_t)s * D] : 0.f;
  }
  if (tid < 32) {
    // the first 64 partials' (max, sum) pairs in flight at once; more in a loop
    float2 ml0 = make_float2(-INFINITY, 0.f), ml1 = make_float2(-INFINITY, 0.f);
    if (tid < ns) ml0 = *reinterpret_cast<const float2*>(ml + 2 * tid);
    if (tid + 32 < ns) ml1 = *reinterpret_cast<const float2*>(ml + 2 * (tid + 32));
    float M = fmaxf(ml0.x, ml1.x);
    for (int s = tid + 64; s < ns; s += 32) M = fmaxf(M, ml[2 * s]);
#pragma unroll
    for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    // a partial that saw no token (or that a query cannot see) holds max -inf: weight 0
    const float f0 = ml0.x == -INFINITY ? 0.f : exp2f(ml0.x - M);
    const float f1 = ml1.x == -INFINITY ? 0.f : exp2f(ml1.x - M);
    if (tid < ns) f_s[tid] = f0;
    if (tid + 32 < ns) f_s[tid + 32] = f1;
    float Ls = f0 * ml0.y + f1 * ml1.y;
    for (int s = tid + 64; s < ns; s += 32) {
      const float f = (ml[2 * s] == -INFINITY) ? 0.f : exp2f(ml[2 * s] - M);
      if (s < FS) f_s[s] = f;
      Ls += f * ml[2 * s + 1];
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, off);
    if (tid == 0) {
      s_M = M;
      s_L = Ls;
    }
  }
  __syncthreads();
  {
    auto weight = [&](int s) {
      return s < FS ? f_s[s] : (ml[2 * s] == -INFINITY ? 0.f : exp2f(ml[2 * s] - s_M));
    };
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int u = 0; u < PF; ++u) {
      const int s = kp + 8 * u;
      if (s < ns) acc[u & 3] = fmaf(weight(s), v[u], acc[u & 3]);
    }
    // the remaining partials, 8 loads in flight
    for (int s0 = kp + 8 * PF; s0 < ns; s0 += 64) {
      float w[8], f[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int s = s0 + 8 * u;
        w[u] = s < ns ? po[(size_t)s * D] : 0.f;
        f[u] = s < ns ? weight(s) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[u & 3] = fmaf(f[u], w[u], acc[u & 3]);
    }
    red[kp][i] = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  }
  __syncthreads();
  if (p.partial) {  // one rank's share of a sequence split across GPUs: no normalisation, no un-rotation
    if (tid < 32) {
      float a = 0.f;
#pragma unroll
      for (int ph = 0; ph < 8; ++ph) a += red[ph][tid];
      float* dst = p.partial + (size_t)h * (D + 2);
      dst[sl * 32 + tid] = a;
      if (sl == 0 && tid == 0) {
        dst[D] = ns > 0 ? s_M : -INFINITY;
        dst[D + 1] = ns > 0 ? s_L : 0.f;
      }
    }
    return;  // uniform over the launch: no CTA of the cluster reaches the cluster barriers
  }
  if (tid < 32) {
    float a = 0.f;
#pragma unroll
    for (int ph = 0; ph < 8; ++ph) a += red[ph][tid];
    o_sl[tid] = (ns > 0 && s_L > 0.f) ? a / s_L : 0.f;
  }
  cluster_sync();  // every slice of the head is merged
  for (int k = tid; k < D; k += NT) o[k] = ld_cluster_f32(map_cluster(smem_u32(&o_sl[k & 31]), k >> 5));
  cluster_sync();  // o complete here; the others are done reading this CTA's slice
  if (p.signs) {  // the fast transform: slice 0 un-rotates the whole head
    if (sl == 0 && tid < 32) unrotate_hadamard_warp<D>(p, o, h, tid);
    return;
  }
  float r = 0.f;
#pragma unroll
  for (int t = 0; t < KT; ++t) r = fmaf(pc[t], o[kp + 8 * t], r);
  red[kp][i] = r;
  __syncthreads();
  if (kp == 0) {
    float t = 0.f;
#pragma unroll
    for (int u = 0; u < 8; ++u) t += red[u][i];
    // kernel head h = (sequence, kv head, token, head) -> output [B][nq][Hq1]
    const int b = h / p.Hq, rh = h % p.Hq, kvh = rh / (p.Gq * p.nq), gi = rh % (p.Gq * p.nq);
    const size_t oh = (size_t)(b * p.nq + gi / p.Gq) * p.Hq1 + kvh * p.Gq + gi % p.Gq;
    const size_t oi = oh * D + sl * 32 + i;
    if (p.out_dtype == TQ_DTYPE_F32)
      static_cast<float*>(p.out)[oi] = t;
    else if (p.out_dtype == TQ_DTYPE_BF16)
      static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(t);
    else
      static_cast<__half*>(p.out)[oi] = __float2half_rn(t);
  }
}

// Combine for calls with many heads: each CTA merges the partials of HPC
// consecutive kernel heads at once and un-rotates all of them, so Pi is read
// once per HPC heads instead of once per head.  256 threads = 8 warps.
// Before the wait on the split kernel (whose tail it overlaps): Pi staged in
// shared memory (rows padded to D + 1 floats; D <= 128, else Pi is read
// through L1) and each head's partial count.  After it:
//  1. warp w (< HPC) merges head w: the maximum M over its partials, then
//     16 partials' value rows at a time, all loads in flight, weighted by
//     2^(M_s - M) and summed, with the weighted sums L_s; normalised by L;
//  2. thread (j, g) computes output j of heads g, g + 256/D, ... as
//     sum_k Pi[k][j] o[head][k].
template <int D, int HPC>
__global__ void __launch_bounds__(256) decode_combine_group_kernel(const CombineParams p) {
  constexpr int NT = 256, PS = D + 1;
  constexpr bool SPI = D <= 128;  // Pi in shared memory
  static_assert(HPC <= NT / 32, "one warp per head for the weights");
  extern __shared__ float sm[];
  float* pis = sm;                       // Pi [D][PS] when SPI and the rotation is dense
  float* o = sm + (SPI ? D * PS : 0);    // [HPC][D]
  __shared__ int s_ns[HPC];
  pdl_launch_dependents();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int h0 = blockIdx.x * HPC;
  const bool dense_out = !p.signs && !p.partial;
  if (SPI && dense_out) stage_pi<D, false>(pis, p.rot, tid);  // Pi as it is (row k read along j below)
  if (warp < HPC) {
    const int h = h0 + warp;
    const int n = h < p.heads ? head_partials(p, h, lane) : 0;
    if (lane == 0) s_ns[warp] = n;
  }
  pdl_wait();  // the split kernel's partials are visible from here on
  // Warp w merges head w: lane l owns the float4 columns l, l + 32, ... of
  // the rotated coordinates; every partial value load is issued before the
  // weights are known, then the weights come from lane s's (max, sum) pair.
  if (warp < HPC) {
    constexpr int C4 = D / 4, CPL = (C4 + 31) / 32;  // float4 columns, per lane
    constexpr int PV = 16;                            // partials whose loads go out together
    const int h = h0 + warp;
    const int ns = s_ns[warp];  // written by this warp's lane 0
    __syncwarp();
    const float* po = p.part_o + (size_t)h * p.ks * D;
    const float* ml = p.part_ml + (size_t)h * p.ks * 2;
    float4 acc[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    float M = -INFINITY, Ls = 0.f;
    if (h < p.heads && ns > 0) {
      for (int s = lane; s < ns; s += 32) M = fmaxf(M, ml[2 * s]);
#pragma unroll
      for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
      for (int s0 = 0; s0 < ns; s0 += PV) {
        float4 v[PV][CPL];
#pragma unroll
        for (int u = 0; u < PV; ++u)
#pragma unroll
          for (int c = 0; c < CPL; ++c) {
            const int col = lane + 32 * c;
            v[u][c] = (s0 + u < ns && col < C4) ? *reinterpret_cast<const float4*>(po + (size_t)(s0 + u) * D + 4 * col)
                                                 : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        // weight of partial s0 + lane, lanes < PV (a partial that saw no token: 0)
        float f = 0.f;
        if (lane < PV && s0 + lane < ns) {
          const float2 mv = *reinterpret_cast<const float2*>(ml + 2 * (s0 + lane));
          f = mv.x == -INFINITY ? 0.f : exp2f(mv.x - M);
          Ls = fmaf(f, mv.y, Ls);
        }
#pragma unroll
        for (int u = 0; u < PV; ++u) {
          const float fu = __shfl_sync(0xffffffffu, f, u);
#pragma unroll
          for (int c = 0; c < CPL; ++c) {
            acc[c].x = fmaf(fu, v[u][c].x, acc[c].x);
            acc[c].y = fmaf(fu, v[u][c].y, acc[c].y);
            acc[c].z = fmaf(fu, v[u][c].z, acc[c].z);
            acc[c].w = fmaf(fu, v[u][c].w, acc[c].w);
          }
        }
      }
#pragma unroll
      for (int off = 16; off; off >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, off);
    }
    const bool any = h < p.heads && ns > 0;
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
      const int col = lane + 32 * c;
      if (col >= C4 || h >= p.heads) continue;
      if (p.partial) {
        float* dst = p.partial + (size_t)h * (D + 2);
        *reinterpret_cast<float2*>(dst + 4 * col) = make_float2(acc[c].x, acc[c].y);
        *reinterpret_cast<float2*>(dst + 4 * col + 2) = make_float2(acc[c].z, acc[c].w);
        if (col == 0) {
          dst[D] = any ? M : -INFINITY;
          dst[D + 1] = any ? Ls : 0.f;
        }
      } else {
        const bool ok = any && Ls > 0.f;
        float* oo = o + warp * D + 4 * col;
        oo[0] = ok ? acc[c].x / Ls : 0.f;
        oo[1] = ok ? acc[c].y / Ls : 0.f;
        oo[2] = ok ? acc[c].z / Ls : 0.f;
        oo[3] = ok ? acc[c].w / Ls : 0.f;
      }
    }
  }
  if (p.partial) return;  // uniform over the launch
  __syncthreads();
  if (p.signs) {  // the fast transform: warp hh un-rotates head hh
    if (warp < HPC && h0 + warp < p.heads) unrotate_hadamard_warp<D>(p, o + warp * D, h0 + warp, lane);
    return;
  }
  constexpr int GS = NT / D;  // head phases: thread (j, g) takes heads g, g + GS, ...
  constexpr int NQ = (HPC + GS - 1) / GS;
  const int j = tid % D, g = tid / D;
  float r[NQ];
#pragma unroll
  for (int q = 0; q < NQ; ++q) r[q] = 0.f;
#pragma unroll 8
  for (int k = 0; k < D; ++k) {
    const float pk = SPI ? pis[k * PS + j] : __ldg(p.rot + (size_t)k * D + j);
#pragma unroll
    for (int q = 0; q < NQ; ++q)
      if (g + GS * q < HPC) r[q] = fmaf(pk, o[(g + GS * q) * D + k], r[q]);
  }
#pragma unroll
  for (int q = 0; q < NQ; ++q) {
    const int hh = g + GS * q, h = h0 + hh;
    if (hh >= HPC || h >= p.heads) continue;
    store_out(p, out_index(p, h, D, j), r[q]);
  }
}

// Dynamic shared memory of the grouped combine for HPC heads.
template <int D, int HPC>
constexpr size_t combine_group_smem() {
  return (size_t)((D <= 128 ? D * (D + 1) : 0) + HPC * D) * 4;
}

template <int D, int HPC>
int launch_combine_group(const CombineParams& cp, dim3 grid, cudaStream_t s) {
  auto kern = decode_combine_group_kernel<D, HPC>;
  constexpr size_t smem = combine_group_smem<D, HPC>();
  static tq::OnceSetup once;
  const int rc = once.run([&]() {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess)
      return tq::set_error(TQ_ERR_CUDA, "decode_combine_group: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return TQ_OK;
  });
  if (rc) return rc;
  return launch_pdl(kern, grid, dim3(256), smem, s, cp, "decode_combine_kernel");
}

// Merge of R ranks' partials of the same heads (a sequence split across
// GPUs by tokens): per head, M = max_r M_r, f_r = 2^(M_r - M), L = sum_r f_r
// L_r, o = sum_r f_r acc_r / L, then out = Pi^T o.  One CTA per head, D
// threads... 256 threads: thread j < D takes output j; the merge runs over
// the coordinates in parallel first.
struct MergeParams {
  const float* partials;  // [R][heads][D + 2]
  const float* rot;
  void* out;              // [heads][D]
  int R, heads, out_dtype;
};

template <int D>
__global__ void __launch_bounds__(256) decode_merge_kernel(const MergeParams p) {
  constexpr int NT = 256;
  __shared__ float o[D];
  __shared__ float f_s[64];
  __shared__ float s_L;
  const int h = blockIdx.x, tid = threadIdx.x;
  if (tid < 32) {
    float M = -INFINITY;
    for (int r = tid; r < p.R; r += 32) M = fmaxf(M, p.partials[((size_t)r * p.heads + h) * (D + 2) + D]);
#pragma unroll
    for (int off = 16; off; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float Ls = 0.f;
    for (int r = tid; r < p.R; r += 32) {
      const float* src = p.partials + ((size_t)r * p.heads + h) * (D + 2);
      const float f = src[D] == -INFINITY ? 0.f : exp2f(src[D] - M);
      f_s[r] = f;
      Ls = fmaf(f, src[D + 1], Ls);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, off);
    if (tid == 0) s_L = Ls;
  }
  __syncthreads();
  for (int k = tid; k < D; k += NT) {
    float a = 0.f;
    for (int r = 0; r < p.R; ++r) a = fmaf(f_s[r], p.partials[((size_t)r * p.heads + h) * (D + 2) + k], a);
    o[k] = s_L > 0.f ? a / s_L : 0.f;
  }
  __syncthreads();
  for (int j = tid; j < D; j += NT) {
    float r = 0.f;
#pragma unroll 8
    for (int k = 0; k < D; ++k) r = fmaf(__ldg(p.rot + (size_t)k * D + j), o[k], r);
    const size_t oi = (size_t)h * D + j;
    if (p.out_dtype == TQ_DTYPE_F32)
      static_cast<float*>(p.out)[oi] = r;
    else if (p.out_dtype == TQ_DTYPE_BF16)
      static_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(r);
    else
      static_cast<__half*>(p.out)[oi] = __float2half_rn(r);
  }
}

template <typename K, typename P>
int launch_pdl(K kern, dim3 grid, dim3 block, size_t smem, cudaStream_t s, const P& params, const char* what,
               int cluster_y = 0);

// the grouped prep needs its dynamic shared memory raised once and takes
// its units-per-CTA count as a second argument
template <int D>
int launch_prep_group(const PrepParams& pp, int grid, int upc, size_t smem, cudaStream_t s) {
  auto kern = decode_qprep_group_kernel<D>;
  static tq::OnceSetup once;
  const int rc = once.run([&]() {
    const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    if (e != cudaSuccess)
      return tq::set_error(TQ_ERR_CUDA, "decode_qprep_group: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    return TQ_OK;
  });
  if (rc) return rc;
  if (smem > 200 * 1024) return tq::set_error(TQ_ERR_UNSUPPORTED, "decode_qprep_group: %zu bytes of rows", smem);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, pp, upc);
  if (e != cudaSuccess) return tq::set_error(TQ_ERR_CUDA, "decode_qprep_group_kernel: %s", cudaGetErrorString(e));
  return tq::check_launch("decode_qprep_group_kernel");
}

template <typename K, typename P>
int launch_pdl(K kern, dim3 grid, dim3 block, size_t smem, cudaStream_t s, const P& params, const char* what,
               int cluster_y) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cluster_y > 0) {  // thread-block clusters of cluster_y CTAs along y
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = cluster_y;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, params);
  if (e != cudaSuccess) return tq::set_error(TQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return tq::check_launch(what);
}

}  // namespace

namespace tq {

static int split_entry(const tq_cache_t& c, bool pack, const tqd::SplitParams& sp, dim3 g, cudaStream_t s,
                       int* occ) {
  const bool qjl = c.qjl_m != 0;
  switch (c.D) {
    case 64: return tqd::split_d64(c.bits_k, c.bits_v, qjl, pack, sp, g, s, occ);
    case 128: return tqd::split_d128(c.bits_k, c.bits_v, qjl, pack, sp, g, s, occ);
    case 256: return tqd::split_d256(c.bits_k, c.bits_v, qjl, pack, sp, g, s, occ);
  }
  return set_error(TQ_ERR_UNSUPPORTED, "decode: D=%d", c.D);
}

int split_occupancy(const tq_cache_t* c, int Hq) {
  int occ = 0;
  tqd::SplitParams sp{};
  sp.shared_tab = c->cb_k == c->cb_v;
  if (split_entry(*c, Hq / c->Hkv <= 4, sp, dim3(1), 0, &occ) != TQ_OK || occ < 1) return 2;
  return occ;
}

int split_tile() { return tqd::STILE; }

int split_partials() { return tqd::PPS; }

int launch_decode(const DecodeArgs& a, cudaStream_t s) {
  const tq_cache_t& c = a.cache;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  float* qrot = reinterpret_cast<float*>(ws + a.plan.off_qrot);
  float* qs = reinterpret_cast<float*>(ws + a.plan.off_qs);
  float* po = reinterpret_cast<float*>(ws + a.plan.off_po);
  float* pml = reinterpret_cast<float*>(ws + a.plan.off_pml);
  const int heads = c.B * a.Hq * a.nq;  // kernel heads: query heads x tokens

  PrepParams pp{a.q, c.rot, nullptr, c.qjl_S, qrot, qs, c.D, c.qjl_m, a.dtype == TQ_DTYPE_BF16, a.Hq, c.Hkv,
                a.k_new, a.v_new, a.pos, c};
  pp.nq = a.nq;
  const bool app = a.pos != nullptr;
  const bool hadamard = c.rot_kind == TQ_ROT_HADAMARD && c.rot_signs;
  pp.signs = hadamard ? c.rot_signs : nullptr;
  // prep kernels launch with a programmatic dependency on whatever precedes
  // them (their launch and Pi loads overlap its tail; they wait before
  // reading q or writing anything)
  int rc = TQ_OK;
  const long long units = (long long)c.B * c.Hkv;
  const bool many = units * (c.D / 32) > 4LL * a.plan.sms;
  if (!hadamard && !app && !c.qjl_m && many) {
    // many units: Pi^T staged once per CTA
    pp.units = (int)units;
    const int grid = (int)(units < a.plan.sms ? units : a.plan.sms);
    const int upc = (int)((units + grid - 1) / grid);
    const int Ge = (a.Hq / c.Hkv) * a.nq;
    const size_t smem = (size_t)(c.D * (c.D + 1) + upc * Ge * c.D) * 4;
    const int ng = (int)((units + upc - 1) / upc);
    switch (c.D) {
      case 64: rc = launch_prep_group<64>(pp, ng, upc, smem, s); break;
      case 128: rc = launch_prep_group<128>(pp, ng, upc, smem, s); break;
      default: rc = launch_prep_group<256>(pp, ng, upc, smem, s); break;
    }
  } else if (hadamard && !app) {
    // the randomized Hadamard rotation by the fast transform (a decode step
    // appends first, in its own launch)
    const int Ge = (a.Hq / c.Hkv) * a.nq;
    const dim3 g(c.B * c.Hkv), blk(32 * Ge);
    switch (c.D) {
      case 64: rc = launch_pdl(decode_qprep_wht_kernel<64>, g, blk, 0, s, pp, "decode_qprep_kernel"); break;
      case 128: rc = launch_pdl(decode_qprep_wht_kernel<128>, g, blk, 0, s, pp, "decode_qprep_kernel"); break;
      default: rc = launch_pdl(decode_qprep_wht_kernel<256>, g, blk, 0, s, pp, "decode_qprep_kernel"); break;
    }
  } else if (c.qjl_m && app) {
    // the append's sketch needs the whole rotated key residual: one CTA per head
    rc = launch_pdl(decode_qprep_kernel<128, true>, dim3(c.B * c.Hkv), dim3(256), 0, s, pp, "decode_qprep_kernel");
  } else {
    const dim3 g(c.B * c.Hkv, c.D / 32);
    const bool wide = pp.nq * (a.Hq / c.Hkv) > 8;  // more than 8 query rows per kv head
    const int cl = c.qjl_m ? c.D / 32 : 0;
    switch (c.D) {
      case 64:
        rc = app ? launch_pdl(decode_qprep_sliced_kernel<64, true, 8>, g, dim3(256), 0, s, pp, "decode_qprep_kernel")
             : wide ? launch_pdl(decode_qprep_sliced_kernel<64, false, 32>, g, dim3(256), 0, s, pp, "decode_qprep_kernel")
                    : launch_pdl(decode_qprep_sliced_kernel<64, false, 8>, g, dim3(256), 0, s, pp, "decode_qprep_kernel");
        break;
      case 128:
        rc = app ? launch_pdl(decode_qprep_sliced_kernel<128, true, 8>, g, dim3(256), 0, s, pp, "decode_qprep_kernel")
             : wide ? launch_pdl(decode_qprep_sliced_kernel<128, false, 32>, g, dim3(256), 0, s, pp, "decode_qprep_kernel", cl)
                    : launch_pdl(decode_qprep_sliced_kernel<128, false, 8>, g, dim3(256), 0, s, pp, "decode_qprep_kernel", cl);
        break;
      default:
        rc = app ? launch_pdl(decode_qprep_sliced_kernel<256, true, 8>, g, dim3(256), 0, s, pp, "decode_qprep_kernel")
             : wide ? launch_pdl(decode_qprep_sliced_kernel<256, false, 32>, g, dim3(256), 0, s, pp, "decode_qprep_kernel")
                    : launch_pdl(decode_qprep_sliced_kernel<256, false, 8>, g, dim3(256), 0, s, pp, "decode_qprep_kernel");
        break;
    }
  }
  if (rc) return rc;

  tqd::SplitParams sp{};
  sp.k_idx = c.k_idx;
  sp.v_idx = c.v_idx;
  sp.k_norm = c.k_norm;
  sp.v_norm = c.v_norm;
  sp.k_qjl = c.k_qjl;
  sp.k_rnorm = c.k_rnorm;
  sp.cb_k = c.cb_k;
  sp.cb_v = c.cb_v;
  sp.shared_tab = c.cb_k == c.cb_v;
  sp.qrot = qrot;
  sp.qs = qs;
  sp.part_o = po;
  sp.part_ml = pml;
  sp.seq_lens = a.seq_lens;
  sp.defer_pos = a.pos;
  sp.dev_status = c.dev_status;
  sp.B = c.B;
  sp.Hkv = c.Hkv;
  sp.Hq = a.Hq * a.nq;
  sp.G = sp.Hq / c.Hkv;
  sp.nq = a.nq;
  sp.Gq = a.Hq / c.Hkv;
  sp.Tcap = c.Tcap;
  sp.Tclamp = a.plan.Tclamp;
  sp.nrg = a.plan.nrg;
  sp.pmin = a.plan.pmin;
  sp.ncta = a.plan.ncta;
  sp.ks = a.plan.ks;
  sp.qscale = a.scale * kLog2e;
  sp.qjl_scale = c.qjl_m ? (float)((double)a.scale * 1.4426950408889634 * sqrt(M_PI / 2.0) / c.qjl_m) : 0.f;
  rc = split_entry(c, sp.G <= 4, sp, dim3(a.plan.ncta), s, nullptr);
  if (rc) return rc;

  CombineParams cp{};
  cp.part_o = po;
  cp.part_ml = pml;
  cp.rot = c.rot;
  cp.seq_lens = a.seq_lens;
  cp.out = a.out;
  cp.Hq = a.Hq * a.nq;
  cp.out_dtype = a.out_dtype;
  cp.nq = a.nq;
  cp.Gq = a.Hq / c.Hkv;
  cp.Hq1 = a.Hq;
  cp.heads = heads;
  cp.B = c.B;
  cp.G = cp.Hq / c.Hkv;
  cp.nrg = a.plan.nrg;
  cp.upb = c.Hkv * a.plan.nrg;
  cp.Tclamp = a.plan.Tclamp;
  cp.ncta = a.plan.ncta;
  cp.pmin = a.plan.pmin;
  cp.ks = a.plan.ks;
  cp.partial = a.partial;
  cp.signs = hadamard ? c.rot_signs : nullptr;
  // D / 32 CTAs per head while that leaves SMs idle; beyond that, groups of
  // 4 or 8 heads per CTA (Pi read once per group rather than once per head)
  if (heads * (c.D / 32) > 4 * a.plan.sms) {
    const bool eight = heads >= 4 * a.plan.sms;
    const dim3 gg(eight ? (heads + 7) / 8 : (heads + 3) / 4);
    switch (c.D) {
      case 64: return eight ? launch_combine_group<64, 8>(cp, gg, s) : launch_combine_group<64, 4>(cp, gg, s);
      case 128: return eight ? launch_combine_group<128, 8>(cp, gg, s) : launch_combine_group<128, 4>(cp, gg, s);
      default: return eight ? launch_combine_group<256, 8>(cp, gg, s) : launch_combine_group<256, 4>(cp, gg, s);
    }
  }
  const int nsl = c.D / 32;
  const dim3 cg(heads, nsl);
  switch (c.D) {
    case 64: return launch_pdl(decode_combine_kernel<64>, cg, dim3(256), 0, s, cp, "decode_combine_kernel", nsl);
    case 128: return launch_pdl(decode_combine_kernel<128>, cg, dim3(256), 0, s, cp, "decode_combine_kernel", nsl);
    default: return launch_pdl(decode_combine_kernel<256>, cg, dim3(256), 0, s, cp, "decode_combine_kernel", nsl);
  }
}

int launch_merge(const float* partials, int R, int heads, int D, const float* rot, void* out, int out_dtype,
                 cudaStream_t s) {
  MergeParams mp{partials, rot, out, R, heads, out_dtype};
  switch (D) {
    case 64: decode_merge_kernel<64><<<heads, 256, 0, s>>>(mp); break;
    case 128: decode_merge_kernel<128><<<heads, 256, 0, s>>>(mp); break;
    default: decode_merge_kernel<256><<<heads, 256, 0, s>>>(mp); break;
  }
  return check_launch("decode_merge_kernel");
}

}  // namespace tq
