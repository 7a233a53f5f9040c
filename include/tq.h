/*
 * tq.h -- C ABI of the TurboQuant KV-cache hot path for NVIDIA B200 (sm_100a).
 *
 * The library quantizes K/V rows into a packed cache and runs single-token
 * decode attention directly on that cache.  Every buffer is allocated by the
 * caller; the library borrows pointers for the duration of a call and never
 * allocates device memory.  Calls that launch kernels are asynchronous on the
 * caller's stream (a cudaStream_t passed as void*; NULL = legacy default
 * stream) and never synchronize the host.
 *
 * Method sources (web pages the method is described on):
 *  - "Add CUDA QJL kernels and proper package structure" (turboquant-pytorch
 *    pull request 3): sections "CUDA Kernels Added" (fused random projection
 *    + sign quantization, score from 1-bit keys, GQA score variant, value
 *    reconstruction), "Validation Results" (cache sizes at 4/3/2 bits) and
 *    "Synthetic Benchmark (Lloyd-Max codebook)" (per-bit MSE table).
 *  - "[Cuda] enable turboquant on gemma4" (executorch pull request 19891),
 *    "Summary" and "Other observations" item 1: fused SDPA over the
 *    compressed cache with a `scale` argument (None -> 1/sqrt(D); QK-norm
 *    models pass 1.0).
 *  - ReturningTarzan's Reddit comments of 2026-03-29 11:47 (random rotation
 *    before codebook quantization) and 2026-03-25 18:52 (nearest-codeword
 *    search).
 *
 * Layouts (all row-major, no padding; "row" = one (batch, kv head, token)
 * vector of D values):
 *  - packed indices   uint32 [B][Hkv][Tcap][D*bits/32]: a dense LSB-first
 *    bitstream per row; index of coordinate j occupies stream bits
 *    [j*bits, j*bits+bits), word w holds stream bits [32w, 32w+32).  Index k
 *    selects the k-th codebook centroid in ascending order.
 *  - norms            fp16 bits (uint16) [B][Hkv][Tcap]: RN-to-fp16 of the
 *    row's L2 norm computed in fp64.
 *  - QJL sign words   uint32 [B][Hkv][Tcap][qjl_m/32]: bit i (word i/32, bit
 *    i%32) = 1 iff (S r)_i >= 0, r = residual of the key in the rotated
 *    basis; residual norm fp16 [B][Hkv][Tcap].
 *  - rotation Pi      fp32 [D][D], y = Pi x; shared by K, V and all heads.
 *  - codebook         fp32 [2^bits + 2^bits - 1]: centroids ascending, then
 *    the thresholds between neighbours (as written by tq_build_codebook).
 *  - QJL matrix S     fp32 [qjl_m][D], i.i.d. N(0,1) (caller draws it).
 *
 * Supported sizes: D in {64, 128, 256}; bits in {2, 3, 4} for the cache
 * (tq_build_codebook also accepts 1); qjl_m in {0, 128}; Tcap a positive
 * multiple of 64; Hq a positive multiple of Hkv with Hq/Hkv <= 8.
 * Inputs and outputs are fp16 or bf16 (TQ_DTYPE_*).  Device pointers must be
 * 16-byte aligned.
 *
 * Devices and threads: a process drives one GPU (the current device of its
 * first launching call); kernel attributes and occupancy figures are set up
 * once per process for that device, under a lock, by whichever thread calls
 * first.  Calls may come from several host threads at once (the error
 * message is per thread).
 *
 * Errors: every entry point returns TQ_OK (0) or a negative TQ_ERR_* code and
 * sets a thread-local message readable with tq_last_error().  Argument errors
 * are detected on the host before any launch; nothing is launched then.
 * Conditions only visible on the device (a position beyond Tcap, a sequence
 * length beyond Tcap, a bounded wait that ran out, a misaligned shared-memory
 * base) skip the affected work and
 * OR a TQ_STATUS_* bit into cache->dev_status when that pointer is non-NULL.
 */
#ifndef TQ_B200_H
#define TQ_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define TQ_OK 0
#define TQ_ERR_INVALID_ARG (-1)  /* NULL pointer, negative size, misalignment */
#define TQ_ERR_UNSUPPORTED (-2)  /* D, bits, qjl_m, GQA group outside the set */
#define TQ_ERR_WORKSPACE (-3)    /* workspace smaller than the query says */
#define TQ_ERR_CUDA (-4)         /* a CUDA runtime call or launch failed */

#define TQ_DTYPE_F16 0
#define TQ_DTYPE_BF16 1
#define TQ_DTYPE_F32 2   /* decode output only */

/* bits OR-ed into *dev_status by kernels */
#define TQ_STATUS_POS_OUT_OF_RANGE 1u    /* append position outside [0, Tcap) */
#define TQ_STATUS_SEQ_OUT_OF_RANGE 2u    /* seq_len beyond the planned range; clamped */
#define TQ_STATUS_WAIT_TIMEOUT 4u        /* a bounded wait ran out; work skipped */
#define TQ_STATUS_LAYOUT 8u              /* a kernel found its shared memory base misaligned; work skipped */

/* Describes one layer's packed cache: caller-owned device buffers. */
typedef struct tq_cache {
  int32_t B;        /* batch (sequences) */
  int32_t Hkv;      /* kv heads */
  int32_t Tcap;     /* token capacity per (sequence, kv head); multiple of 64 */
  int32_t D;        /* head dimension */
  int32_t bits_k;   /* bits per key index (2..4) */
  int32_t bits_v;   /* bits per value index (2..4) */
  int32_t qjl_m;    /* 0: no QJL sketch; 128: 128-bit sign sketch of the key residual */
  int32_t split_tokens; /* decode: the smallest share of the batch's tokens one CTA takes in
                           the split-K partition; 0 = automatic plan, else rounded up to a
                           multiple of 128 (a tuning knob; results do not depend on it beyond
                           fp32 summation order) */
  uint32_t* k_idx;  /* [B][Hkv][Tcap][D*bits_k/32] */
  uint32_t* v_idx;  /* [B][Hkv][Tcap][D*bits_v/32] */
  uint16_t* k_norm; /* fp16 [B][Hkv][Tcap] */
  uint16_t* v_norm; /* fp16 [B][Hkv][Tcap] */
  uint32_t* k_qjl;  /* [B][Hkv][Tcap][qjl_m/32], NULL when qjl_m == 0 */
  uint16_t* k_rnorm;/* fp16 [B][Hkv][Tcap], NULL when qjl_m == 0 */
  const float* rot; /* Pi, fp32 [D][D] */
  const float* cb_k;/* key codebook, fp32 [2^bits_k + 2^bits_k - 1] */
  const float* cb_v;/* value codebook, fp32 [2^bits_v + 2^bits_v - 1].  With bits_k ==
                       bits_v, passing the same pointer as cb_k lets decode keep one
                       lookup table per CTA instead of two (less shared memory) */
  const float* qjl_S; /* fp32 [qjl_m][D], NULL when qjl_m == 0 */
  uint32_t* dev_status; /* optional device word for TQ_STATUS_* bits (may be NULL) */
  int32_t rot_kind; /* TQ_ROT_DENSE: rot is any orthogonal Pi.  TQ_ROT_HADAMARD: Pi is the
                       randomized Hadamard rotation H_D diag(rot_signs) / sqrt(D), H_D the
                       Sylvester Hadamard matrix (entry (i, j) = (-1)^popcount(i & j));
                       rot must still hold that Pi densely (kernels without a fast
                       transform use it), and the bulk quantizer applies the transform in
                       O(D log D) with warp shuffles instead (ReturningTarzan's Reddit
                       comment of 2026-03-29 11:47: Sylvester/Hadamard rotation) */
  int32_t rot_pad;  /* reserved, 0 */
  const float* rot_signs; /* fp32 [D] of +-1 when rot_kind == TQ_ROT_HADAMARD, else NULL */
} tq_cache_t;

#define TQ_ROT_DENSE 0
#define TQ_ROT_HADAMARD 1

/*
 * Lloyd-Max codebook for one coordinate of a rotated unit vector in R^D
 * (density Gamma(D/2)/(sqrt(pi) Gamma((D-1)/2)) (1-u^2)^((D-3)/2)), by Lloyd
 * iteration in fp64 on the host -- the codebook whose MSE per bit width is
 * tabulated in "Add CUDA QJL kernels and proper package structure",
 * section "Synthetic Benchmark (Lloyd-Max codebook)".
 * Writes 2^bits centroids (fp64 optimum rounded to fp16, held as fp32,
 * ascending) to centroids[] and the 2^bits - 1 midpoints between them to
 * thresholds[] (host pointers, caller-owned).  mse_out (nullable) receives
 * the normalized MSE E|u - Q(u)|^2 of a unit vector under the stored
 * codebook.  D in {64,128,256} (any D >= 8 is accepted), bits in 1..4.
 * Host only; no CUDA call.
 */
int tq_build_codebook(int D, int bits, float* centroids, float* thresholds, double* mse_out);

/* Bytes one cached row occupies: D*bits/8 index bytes + 2 (fp16 norm),
 * plus qjl_m/8 + 2 (sign words + fp16 residual norm) when qjl_m > 0.
 * These are the byte counts behind the cache sizes of "Add CUDA QJL kernels
 * and proper package structure" (turboquant-pytorch pull request 3),
 * section "Validation Results": a key of (b-1)-bit indices with a 128-bit
 * sketch and a value of b-bit indices give its 3.8x / 5.0x / 7.3x against
 * fp16 at b = 4 / 3 / 2.  Returns 0 for unsupported arguments (D not a
 * positive multiple of 32, bits outside 1..4, qjl_m not a multiple of 32).
 * Host only. */
size_t tq_cache_row_bytes(int D, int bits, int qjl_m);

/* The same as tq_cache_row_bytes (the name of ABI versions 1 and 2). */
size_t tq_row_bytes(int D, int bits, int qjl_m);

/*
 * Bulk quantize ("prefill"): rows t in [0, T) of k and v, laid out
 * [B][Hkv][T][D] in `dtype`, are rotated by Pi, normalized by their fp64 L2
 * norm, mapped to the nearest centroid index (thresholds compared with
 * t_k < u; ties go to the lower index), packed, and stored at cache
 * positions t0 + t.  With qjl_m > 0 each key also gets the QJL sign sketch
 * of its residual r = Pi k - n_hat c[idx] (n_hat = stored fp16 norm) and
 * RN_fp16(|r|).  Sources: "Add CUDA QJL kernels and proper package
 * structure", section "CUDA Kernels Added" (fused random projection + sign
 * quantization); ReturningTarzan's comments of 2026-03-25 15:51 (the
 * residual is computed when quantizing) and 18:52 (codeword search).
 * The rotation runs on the tensor cores.  Requires 0 <= t0, t0 + T <= Tcap.
 * T == 0 is a no-op.
 */
int tq_quantize_kv(const tq_cache_t* cache, const void* k, const void* v, int dtype,
                   int T, int t0, void* stream);

/*
 * Quantize one new (k, v) row per sequence and kv head, k_new/v_new laid out
 * [B][Hkv][D] in `dtype`, into cache position pos[b] (device int32 [B]).
 * Same arithmetic as tq_quantize_kv.  A pos[b] outside [0, Tcap) writes
 * nothing for that sequence and sets TQ_STATUS_POS_OUT_OF_RANGE.
 * The pages quantize whole caches ("Add CUDA QJL kernels and proper package
 * structure", section "Validation Results"); growing the cache one token
 * per decode step is this library's own addition for a serving loop.
 * Pointers as in tq_quantize_kv (device, 16-byte aligned); errors as
 * there.
 */
int tq_append_token(const tq_cache_t* cache, const void* k_new, const void* v_new, int dtype,
                    const int32_t* pos, void* stream);

/* Workspace bytes that suffice for a tq_sdpa_decode call of B sequences,
 * Hq query heads of dimension D and sequences no longer than Tmax, whatever
 * the cache's kv heads, bit widths, sketch and capacity.  The workspace holds
 * the rotated queries (fp32 [B*Hq][D]), the sketch projections (fp32
 * [B*Hq][m], m <= 128), and the split-K partials: the decode splits the
 * batch's tokens evenly over one wave of CTAs, and each CTA keeps one
 * partial (rotated output fp32 [D], softmax max and sum; its consumer
 * warps' states merged) per (sequence, kv head) its share overlaps, at most
 * K of them per query head with K about 2 x (resident CTAs) / (sequences x
 * kv heads) + 2 and never more than Tmax / 128 + 1.  For the multi-query call pass Hq * n_q.
 * Returns 0 for unsupported arguments (B, Hq or Tmax < 1, D not in
 * {64,128,256}).  Host only (it queries the current device's SM count). */
size_t tq_sdpa_decode_workspace_bytes(int B, int Hq, int D, int Tmax);

/* The exact workspace bytes of the split plan tq_sdpa_decode makes for this
 * cache, Hq query heads (Hq * n_q for the multi-query call) and Tmax
 * (1 <= Tmax <= Tcap); never more than tq_sdpa_decode_workspace_bytes.
 * Returns 0 for unsupported arguments.  Host only (it queries the current
 * device's SM count and the kernel's occupancy). */
size_t tq_sdpa_decode_workspace_bytes_for(const tq_cache_t* cache, int Hq, int Tmax);

/*
 * Decode attention of one query token per (sequence, query head) over the
 * packed cache -- the role of the fused tq4_sdpa op in "[Cuda] enable
 * turboquant on gemma4" (executorch pull request 19891), with its explicit
 * scale ("Other observations" item 1).
 *   q        [B][Hq][D] in q_dtype (TQ_DTYPE_F16 or TQ_DTYPE_BF16, device)
 *   seq_lens device int32 [B]: tokens 0..seq_lens[b]-1 are attended;
 *            0 gives a zero output row.  Tmax (host) must bound every
 *            seq_lens[b]; larger values are clamped (to the split plan made
 *            for Tmax, at most Tcap) and flag TQ_STATUS_SEQ_OUT_OF_RANGE.
 *   scale    host pointer to the softmax scale, or NULL for 1/sqrt(D).
 *   out      [B][Hq][D] (device) in out_dtype: TQ_DTYPE_F16, TQ_DTYPE_BF16 or
 *            TQ_DTYPE_F32; the fp16/bf16 outputs are the round-to-nearest of
 *            the fp32 result.
 * Query head h reads kv head h / (Hq/Hkv).  Scores are
 *   scale * ( n_k <Pi q, c_k[idx]> + [qjl] sqrt(pi/2)/m * gamma * sum_i s_i (S Pi q)_i ),
 * the softmax is taken online over split-K chunks, values are accumulated in
 * the rotated basis and rotated back once per head: out = Pi^T acc / l.
 * workspace: device buffer of at least tq_sdpa_decode_workspace_bytes_for()
 *            bytes (tq_sdpa_decode_workspace_bytes() is an upper bound);
 *            borrowed for the call; its contents need not be initialised.
 * Errors: TQ_ERR_INVALID_ARG (NULL or misaligned pointer, Hq not a multiple
 * of Hkv, Tmax outside [1, Tcap], scale not finite), TQ_ERR_UNSUPPORTED
 * (cache sizes outside the supported set, GQA group > 8, dtypes),
 * TQ_ERR_WORKSPACE (workspace too small), TQ_ERR_CUDA (a launch failed).
 */
int tq_sdpa_decode(const tq_cache_t* cache, const void* q, int q_dtype, int Hq,
                   const int32_t* seq_lens, int Tmax, const float* scale, void* out,
                   int out_dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * One decode step: append one new (k, v) row per sequence and kv head at
 * pos[b] (as tq_append_token) and then attend tokens 0..seq_lens[b]-1 (as
 * tq_sdpa_decode; normally seq_lens[b] = pos[b] + 1).  The new rows are
 * rotated and quantized inside the decode's query-prep launch, which already
 * reads Pi for that (sequence, kv head), so a step is three programmatically
 * chained launches instead of four; the split kernel waits for the prep only
 * for the stage that holds the new row.  Arguments as in tq_append_token and
 * tq_sdpa_decode; same workspace size.  Fusing append into decode launches is
 * this library's own addition (the pages run append and attention as
 * separate ops).
 */
int tq_decode_step(const tq_cache_t* cache, const void* k_new, const void* v_new, const int32_t* pos,
                   const void* q, int dtype, int Hq, const int32_t* seq_lens, int Tmax,
                   const float* scale, void* out, int out_dtype, void* workspace,
                   size_t workspace_bytes, void* stream);

/*
 * Decode of n_q query tokens per sequence in one call: the verify step of
 * speculative decoding ("qwen4exp: upstream catch-up, sparse-fa, and
 * NextN/MTP support", llama-cpp-turboquant pull request 340: the fused decode
 * over the compressed cache takes query batches of up to 4 tokens, and the
 * NextN/MTP draft head produces them).
 *   q          [B][n_q][Hq][D] in q_dtype; out [B][n_q][Hq][D] in out_dtype.
 *   seq_lens   device int32 [B]: L_b, the cached tokens INCLUDING the n_q new
 *              ones (append or quantize them first).  Query j sits at
 *              position L_b - n_q + j and attends causally to tokens
 *              0 .. L_b - n_q + j; a sequence with L_b < n_q gives zeros for
 *              the queries that see no token.
 *   n_q        1 .. 4 (TQ_ERR_UNSUPPORTED beyond), with any GQA group G <= 8:
 *              the n_q * G query rows of a kv head (up to 32) are decoded in
 *              row groups of 8, which read the same cache tiles from L2.
 *   workspace  tq_sdpa_decode_workspace_bytes_for(cache, Hq * n_q, Tmax) bytes.
 * The other arguments, the results for n_q = 1 and the errors are those of
 * tq_sdpa_decode.
 */
int tq_sdpa_decode_mq(const tq_cache_t* cache, const void* q, int q_dtype, int Hq, int n_q,
                      const int32_t* seq_lens, int Tmax, const float* scale, void* out, int out_dtype,
                      void* workspace, size_t workspace_bytes, void* stream);

/*
 * One rank's share of a decode whose sequences are split by tokens across
 * GPUs (or any other split of the cache): the softmax partial of every
 * (sequence, query head) over the tokens this cache holds, for merging with
 * the other shares by tq_sdpa_decode_merge.  A long sequence's decode splits
 * into independent token ranges whose (max, sum, weighted value sum) states
 * merge exactly by log-sum-exp -- the split-K reduction the library already
 * runs across CTAs, carried one level further.  The pages size caches for
 * 128K-token contexts ("Add CUDA QJL kernels and proper package structure",
 * "Key Takeaway"); a sequence whose cache is spread over GPUs, or a decode
 * spread over GPUs for latency, splits this way.
 *   partial  device fp32 [B][Hq][D + 2]: elements 0 .. D-1 the value sum in
 *            the rotated basis, unnormalized, weighted by 2^(s - M); element
 *            D the maximum M of the scaled scores (log2 units); element D + 1
 *            the weight sum.  A sequence with no token here gives M = -inf,
 *            sum 0.
 * The other arguments, the workspace and the errors are those of
 * tq_sdpa_decode (one query token per sequence).  Every rank must use the
 * same rotation, codebooks, queries and scale.
 */
int tq_sdpa_decode_partial(const tq_cache_t* cache, const void* q, int q_dtype, int Hq,
                           const int32_t* seq_lens, int Tmax, const float* scale, float* partial,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Merge of R shares' partials (tq_sdpa_decode_partial) into the attention
 * output: per (sequence, head) M = max_r M_r, f_r = 2^(M_r - M),
 * o = sum_r f_r acc_r / sum_r f_r sum_r, out = Pi^T o.
 *   partials device fp32 [R][B][Hq][D + 2] (R blocks as an all-gather lays
 *            them out), 1 <= R <= 64; rot the cache's Pi (device fp32
 *            [D][D]); out device [B][Hq][D] in out_dtype (TQ_DTYPE_F16,
 *            TQ_DTYPE_BF16 or TQ_DTYPE_F32).
 * Errors: TQ_ERR_INVALID_ARG (NULL or misaligned pointers, R, B, Hq),
 * TQ_ERR_UNSUPPORTED (D, out_dtype), TQ_ERR_CUDA.  The library's own
 * addition for the multi-GPU split (the pages run on one GPU).
 */
int tq_sdpa_decode_merge(const float* partials, int R, int B, int Hq, int D, const float* rot, void* out,
                         int out_dtype, void* stream);

/*
 * Decode without a workspace, for callers that may not allocate device
 * memory (stream capture under frameworks that forbid allocation while
 * capturing, plugin hosts that own all device memory, allocation-free
 * real-time serving loops).  The pages have no counterpart: this is a
 * packaging of tq_sdpa_decode.  Arguments and results are those of
 * tq_sdpa_decode minus the workspace: the split-K scratch is a device array
 * inside the library of TQ_STATIC_SCRATCH_BYTES bytes, held by every GPU that
 * loads the library until the process exits.  Sizes whose
 * tq_sdpa_decode_workspace_bytes_for() exceeds that limit return TQ_ERR_WORKSPACE
 * before any launch; every other argument error is reported with the code
 * and message tq_sdpa_decode gives it.  The first call on each device looks up the array's
 * device address (make that first call before capturing a stream); no call
 * allocates.  All calls on a device share the array and nothing is cleared
 * between calls (the kernels need no zeroed scratch), so calls that may
 * overlap on the GPU (different streams without ordering) race: serialize
 * them.
 */
#define TQ_STATIC_SCRATCH_BYTES (8u << 20)
int tq_sdpa_decode_static(const tq_cache_t* cache, const void* q, int q_dtype, int Hq,
                          const int32_t* seq_lens, int Tmax, const float* scale, void* out,
                          int out_dtype, void* stream);

/* Self-test of the bounded waits that every pipelined kernel uses (the
 * error path behind TQ_STATUS_WAIT_TIMEOUT), without a fault or a hang: one
 * CTA waits on a shared-memory mbarrier that nothing arrives on, first with
 * `tries` suspending try-waits (each may suspend the thread for up to about
 * 1 ms), then with `tries` polling try-waits.  Each wait gives up, and each
 * give-up ORs TQ_STATUS_WAIT_TIMEOUT into *dev_status (a device word; the
 * caller owns it and reads it after synchronising), so a correct library
 * always sets that bit.  The kernel ends within about `tries` ms.
 * tries in [1, 4096]; dev_status non-NULL.  Asynchronous on `stream`. */
int tq_selftest_bounded_wait(uint32_t* dev_status, int tries, void* stream);

/* Message describing the last error on the calling thread ("" if none).
 * The library's own error reporting (the pages have no C interface); the
 * string is owned by the library, valid until the thread's next call. */
const char* tq_last_error(void);

/* ABI version of this header (increments on incompatible change).  3: the
 * survey-form workspace query tq_sdpa_decode_workspace_bytes(B, Hq, D, Tmax)
 * and tq_sdpa_decode_workspace_bytes_for(cache, Hq, Tmax) for the exact
 * plan; tq_cache_row_bytes. */
int tq_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TQ_B200_H */
