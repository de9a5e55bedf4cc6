// Chunked prefill (placeholder until the tcgen05 kernel lands).
#include "common.cuh"

namespace kvattn {

cudaError_t prepare_prefill_kernels() { return cudaSuccess; }

}  // namespace kvattn
