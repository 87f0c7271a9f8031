// prefill.cuh -- chunked prefill over the paged cache (tensor-core kernel).
#pragma once

#include "pa_device.cuh"

namespace pa {

inline pa_status launch_prefill(void *, const void *, const void *, const void *, const int32_t *,
                                const int32_t *, const int32_t *, int, int, int, int, int, int,
                                int, int, float, cudaStream_t) {
    return PA_ERR_UNSUPPORTED;
}

}  // namespace pa
