// Tensor-core (tcgen05) chunked prefill: not built yet.
#include "kda_internal.cuh"

namespace kda {
bool prefill_tc_supported(int, int, int, int) { return false; }
cudaError_t launch_prefill_tc(const PrefillArgs &) { return cudaErrorNotSupported; }
size_t prefill_tc_workspace(const PrefillArgs &) { return 0; }
int prefill_tc_launches(const PrefillArgs &) { return 0; }
}  // namespace kda
