// Instantiations of the decode split kernel's staged (bulk-copy ring) variant
// (tq_decode_split.cuh), compiled apart from the other so that the two sets
// build in parallel.

#include "tq_decode_split.cuh"

namespace tq {
namespace dec {

cudaError_t launch_split_staged(int kbm, bool kprod, int vbm, bool pack, const SplitParams &sp, cudaStream_t s) {
  return launch_split_variant<true>(kbm, kprod, vbm, pack, sp, s);
}

}  // namespace dec
}  // namespace tq
