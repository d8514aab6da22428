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
    // The attention kernel that follows is a programmatic dependent: let it be
    // scheduled now; it waits for this grid to finish before reading the cache.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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

// FP8 E4M3 cache: each thread quantizes 8 bf16 (16 bytes in) to 8 codes (8
// bytes out): fp32(x) * inv_scale in fp32, then nearest code, ties to even,
// saturating at +-448.
__global__ void __launch_bounds__(256) reshape_and_cache_fp8_kernel(const uint4 *__restrict__ k,
                                                                    const uint4 *__restrict__ v,
                                                                    uint2 *__restrict__ k_cache,
                                                                    uint2 *__restrict__ v_cache,
                                                                    const int64_t *__restrict__ slot_mapping,
                                                                    int64_t num_tokens, int64_t num_slots,
                                                                    int row_vecs, float k_inv, float v_inv) {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t total = num_tokens * row_vecs;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t t = i / row_vecs;
        const int c = static_cast<int>(i - t * row_vecs);
        const int64_t slot = __ldg(slot_mapping + t);
        if (slot < 0) continue;
        if (slot >= num_slots) {
            if (c == 0) flag_status(PA_STATUS_BAD_SLOT);
            continue;
        }
        const uint4 kv = __ldcs(k + i), vv = __ldcs(v + i);
        const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w}, vw[4] = {vv.x, vv.y, vv.z, vv.w};
        uint32_t kq[4], vq[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {  // bf16 pair e -> two codes
            kq[e] = f32x2_to_e4m3x2(__uint_as_float(kw[e] << 16) * k_inv, __uint_as_float(kw[e] & 0xffff0000u) * k_inv);
            vq[e] = f32x2_to_e4m3x2(__uint_as_float(vw[e] << 16) * v_inv, __uint_as_float(vw[e] & 0xffff0000u) * v_inv);
        }
        k_cache[slot * row_vecs + c] = make_uint2(kq[0] | (kq[1] << 16), kq[2] | (kq[3] << 16));
        v_cache[slot * row_vecs + c] = make_uint2(vq[0] | (vq[1] << 16), vq[2] | (vq[3] << 16));
    }
}

}  // namespace pa
