// Chunked-prefill attention on tcgen05 tensor cores (in progress).
#pragma once

#include "pa_common.cuh"

namespace pa {

inline int launch_prefill(void *, const void *, const void *, const void *, const int32_t *, int32_t,
                          const int32_t *, const int32_t *, int32_t, int32_t, int32_t, float, const pa_shape *,
                          cudaStream_t) {
    return PA_ERR_UNSUPPORTED;
}

}  // namespace pa
