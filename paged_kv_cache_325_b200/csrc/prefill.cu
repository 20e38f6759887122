// Varlen causal prefill over the paged cache (placeholder until the tcgen05 kernel lands).
#include "pa_internal.h"

namespace pa {
cudaError_t launch_prefill(const PrefillArgs &, const CUtensorMap &, const CUtensorMap &, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace pa
