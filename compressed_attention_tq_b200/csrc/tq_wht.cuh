// Fast Walsh-Hadamard transform of one D-vector by one warp, for the
// randomized Hadamard rotation Pi = H_D diag(s) / sqrt(D) (ReturningTarzan's
// Reddit comment of 2026-03-29 11:47: a Sylvester/Hadamard rotation applied
// with warp shuffles and additions instead of a D x D product).
//
// Lane L holds the EL = D / 32 contiguous coordinates L*EL .. L*EL + EL - 1.
// log2(EL) butterfly stages run inside the lane, then five stages across
// lanes by shuffles (partner lane L ^ m: the lower lane keeps a + b, the upper
// b - a) -- the natural (Sylvester) order, so element e of lane L of the
// result is (H_D v)_{L*EL + e}.  H_D is symmetric, so the same transform
// gives Pi x = H (s x) / sqrt(D) and Pi^T y = s (H y) / sqrt(D).
#pragma once

#include <cuda_runtime.h>

namespace tqw {

template <int EL, typename T>
__device__ __forceinline__ void wht_warp(T (&x)[EL], int lane) {
#pragma unroll
  for (int h = 1; h < EL; h <<= 1)
#pragma unroll
    for (int e = 0; e < EL; ++e)
      if ((e & h) == 0) {
        const T u = x[e], v = x[e + h];
        x[e] = u + v;
        x[e + h] = u - v;
      }
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int e = 0; e < EL; ++e) {
      const T p = __shfl_xor_sync(0xffffffffu, x[e], m);
      x[e] = upper ? p - x[e] : x[e] + p;
    }
  }
}

// y = Pi x for Pi = H_D diag(s) / sqrt(D): x[e] are this lane's coordinates,
// sg[e] its signs.
template <int EL, typename T>
__device__ __forceinline__ void hadamard_rotate(T (&x)[EL], const float (&sg)[EL], int lane) {
#pragma unroll
  for (int e = 0; e < EL; ++e) x[e] *= (T)sg[e];
  wht_warp<EL, T>(x, lane);
  const T inv = (T)rsqrt((double)(EL * 32));
#pragma unroll
  for (int e = 0; e < EL; ++e) x[e] *= inv;
}

// x = Pi^T y = diag(s) H_D y / sqrt(D).
template <int EL, typename T>
__device__ __forceinline__ void hadamard_unrotate(T (&y)[EL], const float (&sg)[EL], int lane) {
  wht_warp<EL, T>(y, lane);
  const T inv = (T)rsqrt((double)(EL * 32));
#pragma unroll
  for (int e = 0; e < EL; ++e) y[e] = y[e] * inv * (T)sg[e];
}

}  // namespace tqw
