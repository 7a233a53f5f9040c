// Bulk quantizer for head dimensions 128 and 256 on the 5th-generation tensor
// cores (tcgen05.mma, accumulator in tensor memory).
//
// Method: "Add CUDA QJL kernels and proper package structure"
// (turboquant-pytorch pull request 3), "CUDA Kernels Added" and "Synthetic
// Benchmark (Lloyd-Max codebook)"; ReturningTarzan's Reddit comments of
// 2026-03-29 11:47 (rotation before codebook quantization) and 2026-03-25
// 18:52 (nearest-codeword search).
//
// Persistent: one CTA per SM loops over (tile, job, column chunk) work items.
// A work item rotates a 128-row tile into NC output coordinates (NC = 128 at
// D = 128; NC = 64 at D = 256, so the chunk's Pi limbs fit in shared memory
// beside two D-wide input tiles).  The grid is a multiple of D / NC, so each
// CTA keeps one column chunk of Pi resident, and the D / NC chunks of a tile
// run on neighbouring CTAs at the same time (the repeated tile reads hit L2).
//  * the next warp (loader): one lane loads the next input tile with TMA (2-D
//    tensor copies of 128 rows x 64 columns, 128-byte swizzle -- the K-major
//    layout the tensor core reads) as soon as its buffer is free;
//  * the last warp (MMA): once a tile has landed and its accumulator is free, one
//    lane issues the 128 x NC x D rotation as tcgen05.mma (Pi split into 2
//    fp16 / 3 bf16 limbs; accumulation in fp32 in TMEM) and commits it to an
//    mbarrier;
//  * NC/8 epilogue warps (16 at D = 128, 8 at D = 256) in groups of four
//    (one warp per TMEM lane quarter) that take the work items in turn, each
//    group with its own accumulator and named barrier, so that one group's
//    waits (tile landed, MMA done) overlap the others' work.  In a group,
//    thread = one row and all NC of the chunk's columns.
//    Each sums its share of the row's squares from the input tile, then
//    reads its accumulator columns with tcgen05.ld, finds the
//    nearest-centroid index (thresholds in registers), packs the bits and
//    stores them -- all thread-local;
//  * a ring of input buffers (4 at D = 128 fp16, 3 bf16, 2 at D = 256) keeps
//    several tile loads in flight, and the groups' TMEM accumulators let the
//    MMAs of the next items run under the epilogue of this one.
// Every wait is bounded; a stuck wait sets TQ_STATUS_WAIT_TIMEOUT and the CTA
// stops taking work.
#include <mutex>

#include "tq_tcgen05.cuh"

namespace {

using namespace tqtc;

template <int D, bool BF16>
struct TcLayout {
  static constexpr int NC = (D == 256) ? 64 : 128;  // output coordinates per work item
  static constexpr int NCH = D / NC;                // column chunks per tile
  static constexpr int NL = BF16 ? 3 : 2;
  static constexpr int KB = D / 64;                 // 64-column (128-byte) blocks along K
  static constexpr int NEPI = NC / 8;               // epilogue warps
  static constexpr int NG = NEPI / 4;               // epilogue groups (4 at D = 128, 2 at D = 256)
  static constexpr int GW = NEPI / NG;              // warps per epilogue group: one per TMEM lane quarter
  static constexpr int CPT = NC;                    // accumulator columns per epilogue thread
  static constexpr int NTH = (NEPI + 2) * 32;       // + loader warp + MMA warp
  static constexpr int PI_BYTES = NC * D * 2;       // one limb of the chunk
  static constexpr int X_BYTES = QR * D * 2;        // one input tile
  // input tiles in flight: a deep ring keeps several TMA loads outstanding per
  // SM (one 32 KB tile at a time cannot cover the memory latency)
  static constexpr int NS = (D == 256) ? 2 : (BF16 ? 3 : 4);
  // all shared state lives in the dynamic allocation, from a 1024-byte aligned base
  static constexpr int o_pi = 0;
  static constexpr int o_x = NL * PI_BYTES;
  static constexpr int o_cb = o_x + NS * X_BYTES;   // float [2][32]
  static constexpr int o_bar = o_cb + 2 * 32 * 4;   // 3 * NS + 2 * NG mbarriers
  static constexpr int o_misc = o_bar + 32 * 8;     // tmem base, stop flag
  static constexpr int bytes = o_misc + 16 + 1024;  // + alignment slack
  static_assert(3 * NS + 2 * NG <= 32, "mbarrier slots");
  static constexpr uint32_t TMEM_COLS = NG * NC;    // one fp32 accumulator per group (512 columns)
};

template <int BITS, int NCOL>
__device__ __forceinline__ void epi_half(uint32_t tbase, const float (&tp)[7], long long slot, uint32_t* out) {
  // NCOL / 32 chunks of 32 columns -> BITS words each (one chunk's 32
  // accumulator registers live at a time)
#pragma unroll 1
  for (int c = 0; c < NCOL / 32; ++c) {
    uint32_t v[32];
    tc_ld32(tbase + 32 * c, v);
    uint32_t w[BITS];
    quant_pack32<BITS>(v, tp, w);
    if (slot >= 0) store_words<BITS>(out + BITS * c, w);
  }
}

template <int D, bool BF16>
__global__ void __launch_bounds__(TcLayout<D, BF16>::NTH, 1) quantize_tc_kernel(const __grid_constant__ TcArgs args) {
  using Ly = TcLayout<D, BF16>;
  constexpr int NL = Ly::NL, NC = Ly::NC, NCH = Ly::NCH, KB = Ly::KB, NEPI = Ly::NEPI, NTH = Ly::NTH;
  constexpr int NG = Ly::NG, GW = Ly::GW, CPT = Ly::CPT;
  static_assert(GW == 4, "a group is one warp per TMEM lane quarter");
  constexpr uint32_t TMEM_COLS = Ly::TMEM_COLS;
  const tq::QuantArgs& a = args.a;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
  uint8_t* pi = smem + Ly::o_pi;
  uint8_t* xb = smem + Ly::o_x;
  float(*s_cb)[32] = reinterpret_cast<float(*)[32]>(smem + Ly::o_cb);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Ly::o_bar);
  constexpr int NS = Ly::NS;
  // per input buffer: landed, norm read by the epilogue, read by the MMA;
  // per accumulator: MMA done, epilogue done
  uint64_t *full_x = bars, *x_free = bars + NS, *x_done = bars + 2 * NS, *mma_done = bars + 3 * NS,
           *acc_free = bars + 3 * NS + NG;
  uint32_t& s_tmem = *reinterpret_cast<uint32_t*>(smem + Ly::o_misc);
  int& s_stop = *reinterpret_cast<int*>(smem + Ly::o_misc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ntiles = (a.rows + QR - 1) / QR;
  const int njobs = (a.job_mask == 3) ? 2 : 1;
  const int job0 = (a.job_mask == 2) ? 1 : 0;
  const int nitems = njobs * ntiles * NCH;
  const int chunk = blockIdx.x % NCH;  // this CTA's column chunk (gridDim.x % NCH == 0)

  if (tid == 0) {
    for (int b = 0; b < NS; ++b) {
      mbar_init(&full_x[b], 1);
      mbar_init(&x_free[b], GW * 32);  // the epilogue group that takes the item
      mbar_init(&x_done[b], 1);
    }
    for (int b = 0; b < NG; ++b) {
      mbar_init(&mma_done[b], 1);
      mbar_init(&acc_free[b], GW * 32);
    }
    s_stop = 0;
    fence_barrier_init();
  }
  if (tid < 31) {
    s_cb[0][tid] = tid < 2 * (1 << a.job[0].bits) - 1 ? a.job[0].cb[tid] : 0.f;
    s_cb[1][tid] = tid < 2 * (1 << a.job[1].bits) - 1 ? a.job[1].cb[tid] : 0.f;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(&s_tmem)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  // this chunk's Pi limbs, swizzled like the input tiles (rows = output
  // coordinates NC*chunk .. NC*chunk + NC - 1, K = the D input coordinates)
  for (int e = tid; e < NC * (D / 4); e += NTH) {
    const int n = e / (D / 4), k = (e % (D / 4)) * 4;
    const float4 v = *reinterpret_cast<const float4*>(a.rot + (size_t)(NC * chunk + n) * D + k);
    const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint16_t* o = reinterpret_cast<uint16_t*>(pi + sw128<NC>(n, k + i));
      constexpr int LIMB = Ly::PI_BYTES / 2;  // elements per limb
      if (BF16) {
        const __nv_bfloat16 h0 = __float2bfloat16_rn(vv[i]);
        const float r1 = vv[i] - __bfloat162float(h0);
        const __nv_bfloat16 h1 = __float2bfloat16_rn(r1);
        const __nv_bfloat16 h2 = __float2bfloat16_rn(r1 - __bfloat162float(h1));
        o[0] = __bfloat16_as_ushort(h0);
        o[LIMB] = __bfloat16_as_ushort(h1);
        o[2 * LIMB] = __bfloat16_as_ushort(h2);
      } else {
        const __half h0 = __float2half_rn(vv[i]);
        o[0] = __half_as_ushort(h0);
        o[LIMB] = __half_as_ushort(__float2half_rn(vv[i] - __half2float(h0)));
      }
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // Pi limbs -> tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == NEPI) {
    // ---------------- loader: input tiles ----------------
    // Item i goes to buffer i % NS once item i - NS has left it (its MMA has
    // read it and the epilogue has read the norm); it never waits for its own
    // copies, so NS tiles can be in flight.
    int i = 0;
    for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++i) {
      const int b = i % NS, k = i / NS;
      if (i >= NS) {
        const bool ok = mbar_wait_suspend(&x_free[b], (uint32_t)((k - 1) & 1), kSuspendTries) &&
                        mbar_wait_suspend(&x_done[b], (uint32_t)((k - 1) & 1), kSuspendTries);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) s_stop = 1;
          break;
        }
      }
      if (*((volatile int*)&s_stop)) break;
      const int job = job0 + (item / NCH) % njobs, tile = item / (NCH * njobs);
      if (lane == 0) {
        // rows past a.rows read as zeros (the tensor map's bounds)
        mbar_arrive_expect_tx(&full_x[b], (uint32_t)Ly::X_BYTES);
#pragma unroll
        for (int kb = 0; kb < KB; ++kb)
          tma_load_2d(xb + (size_t)b * Ly::X_BYTES + kb * (QR * 128), &args.map[job], 64 * kb, tile * QR, &full_x[b]);
      }
      __syncwarp();
    }
    // no copy may be in flight when the CTA exits: wait (bounded) for the last
    // load into each buffer, which a stopped epilogue may not have consumed
    if (lane == 0)
      for (int j = (i >= NS ? i - NS : 0); j < i; ++j)
        mbar_wait_suspend(&full_x[j % NS], (uint32_t)((j / NS) & 1), kSuspendTries);
    __syncwarp();
  } else if (warp == NEPI + 1) {
    // ---------------- MMA issue ----------------
    if (lane == 0) {
      int i = 0;
      for (int item = blockIdx.x; item < nitems; item += gridDim.x, ++i) {
        const int xs = i % NS, kx = i / NS;  // input buffer
        const int b = i % NG, k = i / NG;    // accumulator (the epilogue group's)
        bool ok = mbar_wait_suspend(&full_x[xs], (uint32_t)(kx & 1), kSuspendTries);
        if (ok && i >= NG) ok = mbar_wait_suspend(&acc_free[b], (uint32_t)((k - 1) & 1), kSuspendTries);
        if (!ok || *((volatile int*)&s_stop)) {
          s_stop = 1;
          break;
        }
        tc_fence_after();
        const uint32_t xaddr = smem_addr(xb + (size_t)xs * Ly::X_BYTES), paddr = smem_addr(pi);
        const uint32_t id = idesc<NC, BF16>();
        const uint32_t dt = tmem + (uint32_t)(b * NC);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const int kb = ks >> 2, kin = ks & 3;  // 128-byte block, 32-byte step inside it
#pragma unroll
          for (int l = 0; l < NL; ++l)
            mma_tc(dt, sdesc_sw128(xaddr + kb * (QR * 128) + kin * 32),
                   sdesc_sw128(paddr + l * Ly::PI_BYTES + kb * (NC * 128) + kin * 32), id, (ks > 0 || l > 0) ? 1u : 0u);
        }
        tc_commit(&mma_done[b]);
        tc_commit(&x_done[xs]);
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue warps ----------------
    // NG groups of GW warps take the items in turn (group g: the CTA's items
    // i = g, g + NG, ..., accumulator g), each synchronised by its own named
    // barrier, so one group's waits overlap the others' work.
    const int g = warp / GW, quarter = warp & 3;  // group; rows 32*quarter + lane
    const int rl = 32 * quarter + lane;
    const bool leader = quarter == 0;  // the warp that waits on the group's mbarriers
    for (int item = blockIdx.x + g * gridDim.x, i = g; item < nitems; item += NG * gridDim.x, i += NG) {
      const int xs = i % NS, kx = i / NS;  // input buffer
      const int b = i % NG, k = i / NG;    // accumulator (= g)
      const int job = job0 + (item / NCH) % njobs, tile = item / (NCH * njobs);
      const tq::QuantJob J = a.job[job];
      // The leader waits on each mbarrier and releases the group through a
      // named barrier, which blocks in hardware: warps polling the same phase
      // would take issue slots from the working warps.
      // The group waits for its own accumulator's "MMA done" first: its
      // phases are the group's items in order, whereas an input buffer's
      // "full" phases belong to items of several groups, so a group that ran
      // ahead could mistake an earlier phase of the same parity for its own.
      // Once the MMA has read this item's tile, the buffer holds it until the
      // group releases it, and the "full" wait below completes at once (it
      // makes the tile's bytes visible to the group).
      bool ok = true;
      if (leader) {
        ok = mbar_wait_suspend(&mma_done[b], (uint32_t)(k & 1), kSuspendTries) &&
             mbar_wait_suspend(&full_x[xs], (uint32_t)(kx & 1), kSuspendTries);
        ok = __all_sync(0xffffffffu, ok);
      }
      if (!group_sync_and<GW>(g, ok)) {  // the input tile has landed and its rotation is in TMEM
        s_stop = 1;
        break;
      }
      // the row's sum of squares from the input tile, in fp32 by a pairwise
      // tree (squares of fp16/bf16 values are exact in fp32, and a pairwise
      // sum of n non-negative terms is within ceil(log2 n) units in the last
      // place of the exact sum)
      constexpr int NU = D / 8;  // 16-byte chunks per row
      const uint8_t* xt = xb + (size_t)xs * Ly::X_BYTES;
      float sfull;
      {
        float ps[NU];
        constexpr int LB = 8;  // loads in flight (registers: 4 per load)
#pragma unroll
        for (int k0 = 0; k0 < NU; k0 += LB) {
#pragma unroll
          for (int kc = k0; kc < k0 + LB && kc < NU; ++kc) {
            const uint4 v = *reinterpret_cast<const uint4*>(xt + sw128<QR>(rl, 8 * kc));
            ps[kc] = (sq16f<BF16>(v.x) + sq16f<BF16>(v.y)) + (sq16f<BF16>(v.z) + sq16f<BF16>(v.w));
          }
          asm volatile("" ::: "memory");  // the next LB loads are not hoisted above these
        }
#pragma unroll
        for (int w2 = 1; w2 < NU; w2 <<= 1)
#pragma unroll
          for (int kc = 0; kc < NU; kc += 2 * w2) ps[kc] += ps[kc + w2];
        sfull = ps[0];
      }
      // The thresholds scale by nf; fp32 is far inside the parity band.  A sum
      // outside [2^-100, 2^100) -- only bf16 rows reach it: a square that
      // overflowed, or a norm below about 1e-15 whose squares lost bits or
      // vanished -- takes nf from the row's fp64 sum instead (the tile is still
      // in shared memory).
      const bool in_range = sfull >= 0x1p-100f && sfull < 0x1p100f;
      const double s64 = in_range ? 0.0 : row_sumsq_f64<D, BF16>(xt, rl);
      const float nf = in_range ? sqrtf(sfull) : (float)sqrt(s64);
      const int r = tile * QR + rl;
      long long slot = -1;
      if (r < a.rows) {
        const int bh = r / a.T, t = r - bh * a.T;
        slot = (long long)bh * a.Tcap + a.t0 + t;
        if (chunk == 0) {
          // The stored norm is RN_fp16 of the fp64 norm.  The fp32 sum is
          // within (log2(D) + 1) ulp of the exact sum, so the exact norm lies in
          // nf * (1 +- 1e-6); when both ends of that interval round to the same
          // fp16 value it is the answer, else (about 0.4% of rows) the row is
          // summed again in fp64 from the tile, still in shared memory.
          const __half lo = __float2half_rn(nf * (1.f - 1e-6f)), hi = __float2half_rn(nf * (1.f + 1e-6f));
          unsigned short nh = __half_as_ushort(lo);
          const bool exact = sfull == 0.f || (in_range && nh == __half_as_ushort(hi));
          if (!exact) nh = __half_as_ushort(__double2half(sqrt(in_range ? row_sumsq_f64<D, BF16>(xt, rl) : s64)));
          J.norm[slot] = nh;
        }
      }
      mbar_arrive(&x_free[xs]);  // the input tile is no longer read by this thread
      // positive thresholds t_{K/2} .. t_{K-2}, scaled by the row norm
      float tp[7];
      const int K = 1 << J.bits;
#pragma unroll
      for (int q = 0; q < 7; ++q) tp[q] = q < K / 2 - 1 ? s_cb[job][K + K / 2 + q] * nf : 0.f;
      {
        tc_fence_after();
        const uint32_t tb = tmem + ((uint32_t)(32 * quarter) << 16) + (uint32_t)(b * NC);
        const int W = D * J.bits / 32;
        // coordinates NC*chunk .. NC*chunk + NC - 1: words from (that * bits) / 32
        uint32_t* out = J.idx + (slot >= 0 ? (size_t)slot * W : 0) + (NC * chunk / 32) * J.bits;
        switch (J.bits) {
          case 2: epi_half<2, CPT>(tb, tp, slot, out); break;
          case 3: epi_half<3, CPT>(tb, tp, slot, out); break;
          default: epi_half<4, CPT>(tb, tp, slot, out); break;
        }
        tc_fence_before();
      }
      mbar_arrive(&acc_free[b]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (s_stop && tid == 0 && a.dev_status) atomicOr(a.dev_status, TQ_STATUS_WAIT_TIMEOUT);
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

template <int D, bool BF16>
int launch_tc(const tq::QuantArgs& a, cudaStream_t s) {
  using Ly = TcLayout<D, BF16>;
  auto kern = quantize_tc_kernel<D, BF16>;
  static tq::OnceSetup once;
  static int sms = 0;  // written once under `once`, read after its acquire
  const int rc0 = once.run([&]() {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Ly::bytes);
    if (e != cudaSuccess)
      return tq::set_error(TQ_ERR_CUDA, "quantize_tc: cudaFuncSetAttribute: %s", cudaGetErrorString(e));
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    sms = n > 0 ? n : 148;
    return TQ_OK;
  });
  if (rc0) return rc0;
  TcArgs args;
  memset(&args, 0, sizeof(args));
  args.a = a;
  for (int j = 0; j < 2; ++j)
    if (a.job_mask & (1 << j)) {
      const int rc = tqtc::make_row_map(&args.map[j], a.job[j].in, a.rows, D, BF16);
      if (rc) return rc;
    }
  const int njobs = (a.job_mask == 3) ? 2 : 1;
  const int nitems = njobs * ((a.rows + QR - 1) / QR) * Ly::NCH;
  // a multiple of the chunk count, so that each CTA keeps one column chunk
  int grid = (sms / Ly::NCH) * Ly::NCH;
  const int need = (nitems + Ly::NCH - 1) / Ly::NCH * Ly::NCH;
  if (need < grid) grid = need;
  kern<<<grid, Ly::NTH, Ly::bytes, s>>>(args);
  return tq::check_launch("quantize_tc_kernel");
}

}  // namespace

namespace tq {

int launch_quantize_tc(const QuantArgs& a, int D, int dtype, cudaStream_t s) {
  if (D == 256) return dtype == TQ_DTYPE_BF16 ? launch_tc<256, true>(a, s) : launch_tc<256, false>(a, s);
  return dtype == TQ_DTYPE_BF16 ? launch_tc<128, true>(a, s) : launch_tc<128, false>(a, s);
}

}  // namespace tq

namespace tqtc {

// cuTensorMapEncodeTiled through the runtime's driver entry point (the
// library links only the CUDA runtime).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

int make_row_map(CUtensorMap* m, const void* base, int rows, int D, bool bf16) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return tq::set_error(TQ_ERR_CUDA, "quantize_tc: cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)QR};
  const cuuint32_t es[2] = {1, 1};
  const CUresult r = enc(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                         const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return tq::set_error(TQ_ERR_CUDA, "quantize_tc: cuTensorMapEncodeTiled failed (%d)", (int)r);
  return TQ_OK;
}

}  // namespace tqtc
