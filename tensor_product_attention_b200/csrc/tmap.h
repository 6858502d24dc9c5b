// Host-side creation of TMA tensor maps through the driver entry point (no libcuda link).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

namespace tpa {

// 2-D (or 3-D) bf16 tensor map, 128-byte swizzle unless swizzle_bytes says 64, 32 or 0;
// dims/strides innermost first,
// strides in bytes for dims 1.. .  Returns false if the driver rejects it.
bool make_tmap_bf16(CUtensorMap* map, const void* base, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, int swizzle_bytes = 128);

int sm_count();

// Raise `func`'s dynamic shared-memory limit to at least `bytes` on the current
// device.  Remembered per (kernel, device), so repeated launches skip the call.
cudaError_t allow_smem(const void* func, int bytes);

}  // namespace tpa
