// Causal prefill on tcgen05 tensor cores (placeholder until the kernel lands).
#include "tpa_internal.h"
namespace tpa {
bool prefill_tc_supported(const Shape&) { return false; }
cudaError_t launch_prefill_tc(const Shape&, const tpa_factors&, const tpa_cache&, int, int,
                              const SeqParams&, void*, int*, uint32_t, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace tpa
