// Instantiations of the lane-block pass (bf16 operands by magnitude,
// full-width rows with k a multiple of 64).
#include "pass_lane_block.cuh"

namespace ss24 {
const void *stream_lb_kernel_bf16(int pattern, int score, int fmt)
{
    if (pattern == kDense)
        return stream_lb_for_fmt<kDense>(fmt);
    if (score != kMag)
        return nullptr;
    if (pattern == kSparse24)
        return stream_lb_for_fmt<kSparse24>(fmt);
    if (pattern == kSparse48)
        return stream_lb_for_fmt<kSparse48>(fmt);
    return nullptr;
}
} // namespace ss24
