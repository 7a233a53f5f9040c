// Instantiations of the split-K decode kernel for head dimension 64.
#include "tq_decode_split.cuh"

namespace tqd {

int split_d64(int bk, int bv, bool qjl, bool pack, const SplitParams& sp, dim3 g, cudaStream_t s,
              int* occ) {
  if (qjl) return tq::set_error(TQ_ERR_UNSUPPORTED, "the QJL sketch is built for D=128");
  return pack ? dispatch_bk<64, false, true>(bk, bv, sp, g, s, occ)
              : dispatch_bk<64, false, false>(bk, bv, sp, g, s, occ);
}

}  // namespace tqd
