// chunkwise_tc.cu -- tcgen05 tensor-core chunkwise retention kernel (bf16 inputs).
#include "launch.h"

namespace retnet {

bool tc_chunkwise_supported(const RetentionCall&) { return false; }

cudaError_t launch_tc_chunkwise(const RetentionCall&, const HeadParams&, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace retnet
