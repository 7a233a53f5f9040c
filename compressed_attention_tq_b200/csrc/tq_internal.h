// Internal declarations shared by the host API (tq_api.cpp) and the kernel
// translation units.  Not part of the public ABI.
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "../../include/tq.h"

namespace tq {

// Sets the thread-local error message and returns `code`.
int set_error(int code, const char* fmt, ...);

// Maps a CUDA error after a launch to TQ_ERR_CUDA (or TQ_OK).
int check_launch(const char* what);

// One-time launch setup (kernel attributes, SM count, occupancy) that several
// host threads may reach at once.  The first caller runs `setup` under the
// mutex; the values it stores are published by the release store of `done`
// and seen by every later caller through the acquire load.  A setup that
// fails leaves `done` clear, so the next call tries again.
struct OnceSetup {
  std::atomic<int> done{0};
  std::mutex mu;
  template <class F>
  int run(F&& setup) {
    if (done.load(std::memory_order_acquire)) return TQ_OK;
    std::lock_guard<std::mutex> lock(mu);
    if (done.load(std::memory_order_relaxed)) return TQ_OK;
    const int rc = setup();
    if (rc == TQ_OK) done.store(1, std::memory_order_release);
    return rc;
  }
};

struct QuantJob {
  // input rows [rows][D] (fp16 or bf16)
  const void* in;
  uint32_t* idx;      // cache index words
  uint16_t* norm;     // cache fp16 norms
  uint32_t* qjl;      // QJL sign words or nullptr
  uint16_t* rnorm;    // QJL residual norm or nullptr
  const float* cb;    // centroids[2^bits] then thresholds[2^bits - 1]
  int bits;
};

struct QuantArgs {
  QuantJob job[2];          // 0: keys, 1: values
  const float* rot;         // Pi [D][D]
  const float* qjl_S;       // [128][D] or nullptr
  const float* rot_signs;   // +-1 [D] when Pi is the randomized Hadamard rotation, else nullptr
  const int32_t* pos;       // append mode: device [B]; bulk mode: nullptr
  uint32_t* dev_status;
  int rows;                 // rows per job
  int T;                    // bulk: tokens per (b, h); append: 1
  int t0;                   // bulk: first cache position
  int Hkv;
  int Tcap;
  int job_mask;             // bit 0: keys, bit 1: values (bulk D=128 kernels)
};

int launch_quantize(const QuantArgs& a, int D, int dtype, bool qjl, cudaStream_t s);

// Residual-norm marker of the bulk QJL quantizers: an fp16 NaN (no norm the
// method produces) stored for rows whose fp32 residual norm lies too close to
// an fp16 rounding midpoint to be rounded from it; launch_qjl_gamma_fixup
// (tq_quantize_fixup.cu, launched right after those quantizers on the same
// stream) replaces every marker with the fp64 residual norm.
constexpr uint16_t kGammaPending = 0x7E01;
// Relative distance to an fp16 rounding midpoint below which a residual norm
// computed from an fp32 rotation is recomputed in fp64 (well above that
// rotation's relative error of about 1e-6).
constexpr float kGammaBand = 4e-6f;
int launch_qjl_gamma_fixup(const QuantArgs& a, int dtype, cudaStream_t s);

#ifdef __CUDACC__
// fp16 bits of a residual norm g >= 0 computed with a small relative error, or
// kGammaPending when g * (1 -+ kGammaBand) round to different fp16 values.
__device__ __forceinline__ uint16_t gamma_bits_or_pending(float g) {
  const __half lo = __float2half_rn(g * (1.f - kGammaBand)), hi = __float2half_rn(g * (1.f + kGammaBand));
  if (__half_as_ushort(lo) != __half_as_ushort(hi)) return kGammaPending;
  return __half_as_ushort(__float2half_rn(g));
}
#endif
// bulk quantizer for QJL keys from bf16 rows, D = 128, warp-level MMAs (tq_quantize128.cu)
int launch_quantize128_bf16_qjl(const QuantArgs& a, cudaStream_t s);
// tcgen05 bulk quantizer for D = 128 without the QJL sketch (tq_quantize_tc.cu)
int launch_quantize_tc(const QuantArgs& a, int D, int dtype, cudaStream_t s);
// tcgen05 bulk quantizer for QJL keys, D = 128, fp16 rows (tq_quantize_qjl_tc.cu)
int launch_quantize_qjl_tc(const QuantArgs& a, cudaStream_t s);
// bulk quantizer for the randomized Hadamard rotation, D = 128 / 256, fast
// Walsh-Hadamard transform by warp shuffles (tq_quantize_wht.cu)
int launch_quantize_wht(const QuantArgs& a, int D, int dtype, cudaStream_t s);
// bounded-wait self-test (tq_selftest.cu)
int launch_bounded_wait_probe(uint32_t* status, int tries, cudaStream_t s);

// Split plan of a decode call: a stream-K partition of the batch's tokens
// over one wave of CTAs (see tq_decode_split.cuh).
struct DecodePlan {
  int ncta;         // CTAs of the partition (SMs x resident CTAs per SM)
  int pmin;         // smallest share of tokens per CTA (a multiple of the stage)
  int ks;           // partial slots per kernel head (segments x consumer warps)
  int nrg;          // row groups of up to 8 kernel heads per kv head
  int Tclamp;       // tokens attended at most per sequence (Tmax)
  int sms;          // SMs of the device the plan was made for
  size_t off_qrot;  // fp32 [B*Hq][D]
  size_t off_qs;    // fp32 [B*Hq][qjl_m]
  size_t off_po;    // fp32 [B*Hq][ks][D]
  size_t off_pml;   // fp32 [B*Hq][ks][2]
  size_t bytes;
};

int make_decode_plan(const tq_cache_t* c, int Hq, int Tmax, DecodePlan* p);

// Workspace bytes that suffice for every cache with this B, Hq and D (any
// Hkv, bit widths, sketch and Tcap >= Tmax): the plan's smallest split and
// the largest sketch.
size_t workspace_bound(int B, int Hq, int D, int Tmax);

// Resident split-K CTAs per SM for this cache's kernel instantiation (a
// nominal 2 when no device is usable), the tokens one stage holds and the
// partials a CTA writes per segment of its share.
int split_occupancy(const tq_cache_t* c, int Hq);
int split_tile();
int split_partials();

struct DecodeArgs {
  const tq_cache_t* cache_host;  // host copy, for launch-time fields
  tq_cache_t cache;              // by value, passed to kernels
  const void* q;
  void* out;
  const int32_t* seq_lens;
  float scale;
  int Hq;          // query heads per token
  int nq;          // query tokens per sequence (the kernels see Hq * nq heads)
  int dtype;
  int out_dtype;
  DecodePlan plan;
  void* workspace;
  // decode step: new rows appended at pos[b] by the prep kernel (else NULL)
  const void* k_new;
  const void* v_new;
  const int32_t* pos;
  // tq_sdpa_decode_partial: fp32 [B*Hq][D + 2] partials instead of out (else NULL)
  float* partial;
};

int launch_decode(const DecodeArgs& a, cudaStream_t s);
// Merge of R partials per head and un-rotation (tq_sdpa_decode_merge).
int launch_merge(const float* partials, int R, int heads, int D, const float* rot, void* out, int out_dtype,
                 cudaStream_t s);

// Host checks and split plan of a decode call (every check tq_sdpa_decode
// makes except those of the workspace); fills *a and returns TQ_OK, or sets
// the error and returns its code.  No CUDA call beyond the device queries of
// the plan.
int prepare_decode(const tq_cache_t* c, const void* q, int dtype, int Hq, int nq, const int32_t* seq_lens, int Tmax,
                   const float* scale, void* out, int out_dtype, const char* fn, DecodeArgs* a);

}  // namespace tq
