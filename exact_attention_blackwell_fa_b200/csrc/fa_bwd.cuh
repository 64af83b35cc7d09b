// fa_bwd.cuh -- exact attention backward for sm_100a (placeholder until the kernels land).
#pragma once

#include "fa_common.cuh"

namespace fa {

inline size_t bwd_round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

inline size_t bwd_workspace_bytes(int B, int Sq, int Hq, int d)
{
    const size_t sq_pad = (static_cast<size_t>(Sq) + 127) / 128 * 128;
    const size_t rows = static_cast<size_t>(B) * Hq * sq_pad;
    return 2 * bwd_round256(rows * 4) + bwd_round256(rows * d * 4);
}

inline fa_status launch_bwd(const void*, const void*, const void*, const void*, const float*,
                            const void*, void*, void*, void*, int, int, int, int, int, int, bool,
                            float, bool, void*, int, cudaStream_t)
{
    return FA_ERR_UNSUPPORTED;
}

}  // namespace fa
