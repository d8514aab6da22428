// KV write: copy each new token's [Hk][D] row of k and v into its slot of the
// paged pool ("vLLM and PagedAttention", ai.zenoagi.com, §2 "The PagedAttention
// Solution": blocks are filled on demand; "How vLLM Works?", peterindia.net, §03).
//
// A token row is contiguous both in the input ([T][Hk][D]) and in the pool
// (row `slot` of the pool viewed as [NB*16][Hk][D]), so the copy is a set of
// 16-byte vector moves. Consecutive threads move consecutive 16-byte pieces
// of one row, so loads and stores coalesce. The kernel is HBM-bound: it moves
// 2 * (read + write) * T * Hk * D * elem bytes.
#pragma once

#include "pa_common.cuh"

namespace pa {

__global__ void __launch_bounds__(256) reshape_and_cache_kernel(const uint4 *__restrict__ k,
                                                                const uint4 *__restrict__ v,
                                                                uint4 *__restrict__ k_cache,
                                                                uint4 *__restrict__ v_cache,
                                                                const int64_t *__restrict__ slot_mapping,
                                                                int64_t num_tokens, int64_t num_slots,
                                                                int row_vecs) {
    const int64_t total = num_tokens * row_vecs;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t t = i / row_vecs;
        const int c = static_cast<int>(i - t * row_vecs);
        const int64_t slot = __ldg(slot_mapping + t);
        if (slot < 0) continue;  // padding token
        if (slot >= num_slots) {
            if (c == 0) flag_status(PA_STATUS_BAD_SLOT);
            continue;
        }
        const uint4 kv = __ldcs(k + i);
        const uint4 vv = __ldcs(v + i);
        k_cache[slot * row_vecs + c] = kv;
        v_cache[slot * row_vecs + c] = vv;
    }
}

}  // namespace pa
