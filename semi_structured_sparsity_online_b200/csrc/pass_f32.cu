// Instantiations of the pass kernels for fp32 operands.
#include "pass_dispatch.cuh"

namespace ss24 {
const void *stream_kernel_f32(int pattern, int score, int fmt, bool fw)
{
    return stream_kernel_ptr<float>(pattern, score, fmt, fw);
}
const void *rowsweep_kernel_f32(int pattern, int score)
{
    return rowsweep_kernel_ptr<float>(pattern, score);
}
const void *axis0_kernel_f32(int pattern, int score, int fmt)
{
    return axis0_kernel_ptr<float>(pattern, score, fmt);
}
const void *rowblock_kernel_f32(int pattern, int score, int cpt)
{
    return rowblock_kernel_ptr<float>(pattern, score, cpt);
}
} // namespace ss24
