// fa_bwd.cuh -- backward kernels (placeholder until the kernels land).
#pragma once
#include "fa_common.cuh"
#include "fa.h"

namespace fa {
inline size_t bwd_workspace_bytes(long long BH, int N, int d) {
    return static_cast<size_t>(BH) * N * 4 + static_cast<size_t>(BH) * N * d * 4 + 256;
}
inline int bwd_entry(const void *, const void *, const void *, const void *, const void *, const float *, void *,
                     void *, void *, void *, size_t, const uint8_t *, int, int, int, int, float, int, int, void *) {
    return FA_ERR_UNSUPPORTED;
}
}  // namespace fa
