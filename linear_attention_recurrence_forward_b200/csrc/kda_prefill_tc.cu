// Placeholder for the tcgen05 chunkwise prefill kernel (not yet built).
#include "kda_internal.cuh"

namespace kda {
bool prefill_tc_supports(const PrefillArgs&) { return false; }
cudaError_t launch_prefill_tc(const PrefillArgs&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace kda
