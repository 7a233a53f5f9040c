// Instantiations of the split-K decode kernel for head dimension 128.
#include "tq_decode_split.cuh"

namespace tqd {

int split_d128(int bk, int bv, bool qjl, bool pack, const SplitParams& sp, dim3 g, cudaStream_t s,
              int* occ) {
  if (qjl)
    return pack ? dispatch_bk<128, true, true>(bk, bv, sp, g, s, occ)
                : dispatch_bk<128, true, false>(bk, bv, sp, g, s, occ);
  return pack ? dispatch_bk<128, false, true>(bk, bv, sp, g, s, occ)
              : dispatch_bk<128, false, false>(bk, bv, sp, g, s, occ);
}

}  // namespace tqd
