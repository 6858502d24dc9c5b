// Factor projection on tcgen05 tensor cores (placeholder until the kernel lands).
#include "tpa_internal.h"
namespace tpa {
bool project_tc_supported(const Shape&, int) { return false; }
cudaError_t launch_project_tc(const Shape&, const void*, const void*, int, int, const SeqParams&,
                              const float*, const ProjLayout&, int*, uint32_t, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace tpa
