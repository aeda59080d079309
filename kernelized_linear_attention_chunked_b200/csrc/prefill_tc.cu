// Causal chunked prefill on the tcgen05 tensor cores (bf16 operands, fp32
// accumulation in tensor memory). Not built yet: every shape goes to the
// CUDA-core path.
#include "kata_internal.h"

namespace kata {

bool prefill_tc_supported(const PrefillArgs &) { return false; }

size_t prefill_tc_workspace_bytes(int, int, int, int, int) { return 0; }

cudaError_t prefill_tc(const PrefillArgs &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace kata
