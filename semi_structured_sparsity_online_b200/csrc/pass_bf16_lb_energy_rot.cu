// Instantiations of the lane-block energy pass over the operand rotated along
// k (2:4 by magnitude, bf16, full-width rows with k a multiple of 64; block
// Hadamard in registers before the selection, "Is 2:4 Sparsity Still Worth
// It?" §4).
#include "pass_lane_energy.cuh"

namespace ss24 {
const void *stream_lb_energy_kernel_bf16_rot(int sparse_fmt, int dense_fmt)
{
    switch (sparse_fmt) {
    case kNone:
        return stream_lb_energy_for_dense<kNone, true>(dense_fmt);
    case kFp8:
        return stream_lb_energy_for_dense<kFp8, true>(dense_fmt);
    case kNvfp4:
        return stream_lb_energy_for_dense<kNvfp4, true>(dense_fmt);
    case kMxfp4:
        return stream_lb_energy_for_dense<kMxfp4, true>(dense_fmt);
    case kInt:
        return stream_lb_energy_for_dense<kInt, true>(dense_fmt);
    }
    return nullptr;
}
} // namespace ss24
