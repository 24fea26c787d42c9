// Chunked prefill on tcgen05 tensor cores (bf16, head_dim 128, block 16).
// Until this kernel is enabled the dispatcher uses the generic kernel.
#include "common.cuh"
#include "launch.hpp"

namespace pa {

bool prefill_fast_supported(int, int, int, int) { return false; }

cudaError_t launch_prefill_fast(const CUtensorMap*, const CUtensorMap*,
                                const PrefillArgs&, int, cudaStream_t) {
  return cudaErrorNotSupported;
}

}  // namespace pa
