// Fused tensor-core path (placeholder until the tcgen05 kernel lands).
#include "gdr_internal.h"

namespace gdr {

bool fused_tc_applies(const Problem &) { return false; }

cudaError_t fused_tc_run(const Problem &, cudaStream_t) {
  return cudaErrorNotSupported;
}

cudaError_t fused_tc_read_error(unsigned *word, bool) {
  *word = 0;
  return cudaSuccess;
}

}  // namespace gdr
