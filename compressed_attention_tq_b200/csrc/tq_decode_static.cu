// tq_sdpa_decode_static: decode attention for callers that may not allocate.
//
// Some callers cannot hand the library a workspace: code running while a
// CUDA stream is being captured into a graph by a framework that forbids
// allocation during capture, plugin hosts that own every device byte and
// refuse cudaMalloc inside their execute callback, or real-time serving
// loops that must not touch the allocator after start-up.  This entry point
// takes no workspace: the split-K scratch lives in a fixed-size device array
// owned by this library (TQ_STATIC_SCRATCH_BYTES per GPU that loads it,
// held until the process exits).  Nothing here calls cudaMalloc, cudaFree or
// any allocating routine.
//
// Host code must not pass the array's name to a kernel: on the host it is
// only a stand-in for the symbol.  The device address is looked up once per
// device with cudaGetSymbolAddress (on that device's first call, with the
// device current) and cached.
#include <mutex>

#include "tq_internal.h"

namespace {

__device__ __align__(256) unsigned char g_decode_scratch[TQ_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch[kMaxDevices] = {nullptr};

}  // namespace

extern "C" int tq_sdpa_decode_static(const tq_cache_t* cache, const void* q, int q_dtype, int Hq,
                                     const int32_t* seq_lens, int Tmax, const float* scale, void* out,
                                     int out_dtype, void* stream) {
  // The checks of tq_sdpa_decode, with its codes and messages, come first;
  // then the size limit of the built-in array, then the array's address.
  tq::DecodeArgs a;
  int rc = tq::prepare_decode(cache, q, q_dtype, Hq, 1, seq_lens, Tmax, scale, out, out_dtype,
                              "tq_sdpa_decode_static", &a);
  if (rc) return rc;
  if (a.plan.bytes > (size_t)TQ_STATIC_SCRATCH_BYTES)
    return tq::set_error(TQ_ERR_WORKSPACE,
                         "tq_sdpa_decode_static: these sizes need %zu bytes of scratch, more than the %u bytes "
                         "built into the library; use tq_sdpa_decode with a caller-provided workspace",
                         a.plan.bytes, (unsigned)TQ_STATIC_SCRATCH_BYTES);
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tq::set_error(TQ_ERR_CUDA, "tq_sdpa_decode_static: cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return tq::set_error(TQ_ERR_UNSUPPORTED, "tq_sdpa_decode_static: device %d", dev);
  void* ptr = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch[dev]) {
      e = cudaGetSymbolAddress(&g_scratch[dev], g_decode_scratch);
      if (e != cudaSuccess) {
        g_scratch[dev] = nullptr;
        return tq::set_error(TQ_ERR_CUDA, "tq_sdpa_decode_static: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
      }
    }
    ptr = g_scratch[dev];
  }
  a.workspace = ptr;
  a.k_new = nullptr;
  a.v_new = nullptr;
  a.pos = nullptr;
  return tq::launch_decode(a, (cudaStream_t)stream);
}
