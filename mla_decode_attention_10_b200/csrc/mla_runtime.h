// mla_runtime.h -- host-side helpers shared by the library's launchers
// (internal; not part of the C ABI).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "mla_epilogue.h"

namespace mla {

constexpr int kMaxDevices = 64;

// Records `e` as this host thread's last CUDA error (what mla_last_cuda_error
// returns), clears the runtime's non-sticky error state and returns
// MLA_ERR_CUDA.  Every launcher returns MLA_ERR_CUDA through this.
mla_status cuda_failure(cudaError_t e);

// The current device and its SM count.  The count is queried once per device
// and cached (a relaxed atomic per device, so concurrent callers are safe).
mla_status current_device(int* dev, int32_t* sm_count);

}  // namespace mla
