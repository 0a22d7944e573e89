// Chunked WY/UT delta-rule kernel (tcgen05 + TMA + TMEM). Placeholder: not yet built.
#pragma once

#include "common.cuh"

namespace drscan {

inline bool chunked_supported(int, int, int) { return false; }

inline int launch_chunked(const void*, const void*, const void*, const float*, const float*,
                          const float*, void*, float*, int, int, int, int, int, cudaStream_t) {
    return DR_ERR_UNSUPPORTED;
}

}  // namespace drscan
