// Whole-block copies for the paged pool.
//
// Copy-on-write: sequences that share a prefix point at the same physical
// blocks, and a shared block is copied before a sequence writes into it
// ("vLLM — PagedAttention and Continuous Batching", s-samarth.github.io,
// §2.3; "vLLM and PagedAttention", ai.zenoagi.com, §2 "The PagedAttention
// Solution"; "How vLLM Works?", peterindia.net, §03). Preemption swaps a
// request's blocks out to host memory and back ("vLLM and PagedAttention" §3;
// "How vLLM Works?" §04).
//
// One kernel serves both: pair i copies block pairs[2i] of src to block
// pairs[2i+1] of dst. Each CTA owns pairs in a grid-stride loop and moves the
// block in 16-byte vectors, so consecutive threads touch consecutive bytes.
// The pools may be device memory or pinned host memory (reached through its
// device mapping, so a swap is one launch rather than one copy per block).
// HBM-bound for device pools (2 x block bytes per pair), link-bound for host.
#pragma once

#include "pa_common.cuh"

namespace pa {

__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4 *__restrict__ dst, const uint4 *__restrict__ src,
                                                          const int64_t *__restrict__ pairs, int64_t num_pairs,
                                                          int64_t src_blocks, int64_t dst_blocks, int block_vecs) {
    for (int64_t i = blockIdx.x; i < num_pairs; i += gridDim.x) {
        const int64_t s = __ldg(pairs + 2 * i), d = __ldg(pairs + 2 * i + 1);
        if (s < 0 || s >= src_blocks || d < 0 || d >= dst_blocks) {
            if (threadIdx.x == 0) flag_status(PA_STATUS_BAD_BLOCK_ID);
            continue;
        }
        const uint4 *sp = src + s * block_vecs;
        uint4 *dp = dst + d * block_vecs;
        // eight loads of each thread in flight before its stores (a 32 KB block is 8 per thread)
        for (int v0 = threadIdx.x; v0 < block_vecs; v0 += 8 * blockDim.x) {
            uint4 r[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int v = v0 + u * blockDim.x;
                if (v < block_vecs) r[u] = __ldcs(sp + v);
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int v = v0 + u * blockDim.x;
                if (v < block_vecs) __stcs(dp + v, r[u]);
            }
        }
    }
}

}  // namespace pa
