// Placeholder until the tensor-core chunked kernel lands: route to the exact
// recurrent kernel.
#include "gdn_internal.cuh"
namespace gdn {
cudaError_t launch_prefill_tc(const PrefillArgs &a, cudaStream_t s) { return launch_prefill_recurrent(a, s); }
}  // namespace gdn
