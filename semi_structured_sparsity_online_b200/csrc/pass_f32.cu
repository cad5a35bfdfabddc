// Instantiations of the pass kernels for fp32 operands.
#include "pass_dispatch.cuh"

namespace ss24 {
const void *tile_kernel_f32(int pattern, int score, int fmt)
{
    return tile_kernel<float>(pattern, score, fmt);
}
const void *row_kernel_f32(int pattern, int score)
{
    return row_kernel_ptr<float>(pattern, score);
}
const void *rowreg_kernel_f32(int pattern, int score, int nch)
{
    return rowreg_kernel_ptr<float>(pattern, score, nch);
}
const void *axis0_kernel_f32(int pattern, int score, int fmt)
{
    return axis0_kernel_ptr<float>(pattern, score, fmt);
}
} // namespace ss24
