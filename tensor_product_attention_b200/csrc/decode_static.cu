// tpa_decode_static: tpa_decode for callers that cannot allocate device memory.
//
// Some callers have no way to allocate device memory for a workspace.  Examples are a
// plug-in inside a host application that owns every allocation, or a process that
// must never call cudaMalloc once it is serving.  This entry point gives them decode
// without a caller-supplied workspace.  The split-K scratch lives in the file-scope
// device array below.  The array is sized once at compile time.  Every GPU on which
// the library is loaded holds it until the process exits.
//
// Behaviour:
//  - Set-up: the first call on each device looks up the array's device address with
//    cudaGetSymbolAddress while that device is current, then caches it.  Make that
//    first call before any stream capture.  The cached address belongs to the
//    device's current context: after cudaDeviceReset (or anything else that destroys
//    and re-creates the primary context) the module is loaded again and the array may
//    move, so the library must not be used across a device reset.
//  - Arguments: checked exactly as tpa_decode checks them, so both calls return the
//    same status for the same arguments; then calls needing more than
//    TPA_DECODE_STATIC_SCRATCH_BYTES of scratch are rejected with TPA_ERR_WORKSPACE.
//    Both checks come before any CUDA call.
//  - Contents: the array keeps whatever the previous call left.  Nothing needs
//    clearing, because a call that completes without a device error writes every
//    partial state it later reads.  If tpa_get_device_error reports an error (a
//    bounded wait gave up), that call's output is undefined: it may mix in partial
//    states an earlier call left in the array.
//  - Concurrency: all calls on a device share the one array, so calls that overlap on
//    the GPU (other streams, other threads) race.  Order them on one stream.
//  - No cudaMalloc, cudaFree or allocating library routine is called.
#include <mutex>

#include "tpa_internal.h"

namespace tpa {
namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[TPA_DECODE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (host code must not use
// the symbol itself: on the host it is only a stand-in, not a device address).
void* scratch_on_current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess) return nullptr;
        g_scratch_ptr[dev] = p;
    }
    return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace tpa

extern "C" tpa_status tpa_decode_static(const tpa_dims* dims, const void* q_a, const void* q_b,
                                        const tpa_cache* cache, const int32_t* lengths,
                                        int32_t batch, void* out, tpa_stream_t stream) {
    tpa_status st = tpa::validate_decode(dims, q_a, q_b, cache, lengths, batch, out);
    if (st != TPA_OK) return st;
    const size_t need = tpa_decode_workspace_bytes(dims, lengths, batch);
    if (need == 0) return TPA_ERR_INVALID;
    if (need > (size_t)TPA_DECODE_STATIC_SCRATCH_BYTES) return TPA_ERR_WORKSPACE;
    void* scratch = tpa::scratch_on_current_device();
    if (!scratch) return TPA_ERR_CUDA;
    return tpa_decode(dims, q_a, q_b, cache, lengths, batch, out, scratch,
                      (size_t)TPA_DECODE_STATIC_SCRATCH_BYTES, stream);
}
