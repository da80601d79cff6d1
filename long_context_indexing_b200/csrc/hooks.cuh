// hooks.cuh -- test hooks of liblsa (not part of the method).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace lsa {

// Polls each bounded wait of the tensor-core centroid scorer makes before it
// gives up and records DEV_TIMEOUT; polls < 0 restores the default.
cudaError_t set_score_wait_polls(int64_t polls);
// The same for the tensor-core attention tile kernel (bucket_attn_tc_kernel)
// and for the per-query bf16 attention kernel (attn_bf16_kernel: decode
// splits, prefill rows attended key by key, lsa_sparse_attn).
cudaError_t set_tile_wait_polls(int64_t polls);
cudaError_t set_attn_wait_polls(int64_t polls);

}  // namespace lsa
