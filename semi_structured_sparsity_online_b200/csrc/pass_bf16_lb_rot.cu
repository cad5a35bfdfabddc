// Instantiations of the lane-block pass over the operand rotated along k
// (bf16, magnitude score, full-width rows with k a multiple of 64; block
// Hadamard in registers before the selection, "Is 2:4 Sparsity Still Worth
// It?" §4).
#include "pass_lane_block.cuh"

namespace ss24 {

namespace {

template <int PAT> const void *rot_for_fmt(int fmt)
{
    switch (fmt) {
    case kNone:
        if constexpr (PAT != kDense)
            return reinterpret_cast<const void *>(&stream_lb_kernel<PAT, kNone, true>);
        break;
    case kFp8:
        return reinterpret_cast<const void *>(&stream_lb_kernel<PAT, kFp8, true>);
    case kNvfp4:
        return reinterpret_cast<const void *>(&stream_lb_kernel<PAT, kNvfp4, true>);
    case kMxfp4:
        return reinterpret_cast<const void *>(&stream_lb_kernel<PAT, kMxfp4, true>);
    case kInt:
        if constexpr (PAT == kSparse24)
            return reinterpret_cast<const void *>(&stream_lb_kernel<PAT, kInt, true>);
        break;
    }
    return nullptr;
}

} // namespace

const void *stream_lb_amax_kernel_bf16_rot(int pattern)
{
    if (pattern == kDense)
        return reinterpret_cast<const void *>(&stream_lb_amax_rot_kernel<kDense>);
    if (pattern == kSparse24)
        return reinterpret_cast<const void *>(&stream_lb_amax_rot_kernel<kSparse24>);
    if (pattern == kSparse48)
        return reinterpret_cast<const void *>(&stream_lb_amax_rot_kernel<kSparse48>);
    return nullptr;
}

const void *stream_lb_kernel_bf16_rot(int pattern, int fmt)
{
    if (pattern == kDense)
        return rot_for_fmt<kDense>(fmt);
    if (pattern == kSparse24)
        return rot_for_fmt<kSparse24>(fmt);
    if (pattern == kSparse48)
        return rot_for_fmt<kSparse48>(fmt);
    return nullptr;
}

} // namespace ss24
