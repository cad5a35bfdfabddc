// Instantiations of the pass kernels for bf16 operands.
#include "pass_dispatch.cuh"

namespace ss24 {
const void *tile_kernel_bf16(int pattern, int score, int fmt)
{
    return tile_kernel<__nv_bfloat16>(pattern, score, fmt);
}
const void *row_kernel_bf16(int pattern, int score)
{
    return row_kernel_ptr<__nv_bfloat16>(pattern, score);
}
const void *rowreg_kernel_bf16(int pattern, int score, int nch)
{
    return rowreg_kernel_ptr<__nv_bfloat16>(pattern, score, nch);
}
const void *axis0_kernel_bf16(int pattern, int score, int fmt)
{
    return axis0_kernel_ptr<__nv_bfloat16>(pattern, score, fmt);
}
} // namespace ss24
