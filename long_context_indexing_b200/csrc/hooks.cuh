// hooks.cuh -- test hooks of liblsa (not part of the method).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace lsa {

// Polls each bounded wait of the tensor-core centroid scorer makes before it
// gives up and records DEV_TIMEOUT; polls < 0 restores the default.
cudaError_t set_score_wait_polls(int64_t polls);

}  // namespace lsa
