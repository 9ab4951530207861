// Lightning-indexer scores on the 5th-generation tensor cores (placeholder: the
// tcgen05 kernel is not built yet, so every shape goes to the CUDA-core kernel).
#include "common.cuh"
#include "kernels.h"

namespace dsa {

bool index_scores_tc_supported(int, int, int) { return false; }

cudaError_t launch_index_scores_tc(const void*, const void*, const float*, float, int, int, int,
                                   int, int, int, int, float*, int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace dsa
