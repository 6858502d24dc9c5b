// Decode on tcgen05 tensor cores (placeholder until the kernel lands).
#include "tpa_internal.h"
namespace tpa {
bool decode_tc_supported(const Shape&) { return false; }
cudaError_t launch_decode_tc(const Shape&, const void*, const void*, const tpa_cache&,
                             const SeqParams&, int, const DecodeSchedule&, float*, int*, uint32_t,
                             cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace tpa
