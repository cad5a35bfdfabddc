// Instantiations of the pass kernels for bf16 operands.
#include "pass_dispatch.cuh"

namespace ss24 {
const void *stream_kernel_bf16(int pattern, int score, int fmt, bool fw)
{
    return stream_kernel_ptr<__nv_bfloat16>(pattern, score, fmt, fw);
}
const void *rowsweep_kernel_bf16(int pattern, int score)
{
    return rowsweep_kernel_ptr<__nv_bfloat16>(pattern, score);
}
const void *axis0_kernel_bf16(int pattern, int score, int fmt)
{
    return axis0_kernel_ptr<__nv_bfloat16>(pattern, score, fmt);
}
const void *rowblock_kernel_bf16(int pattern, int score, int cpt)
{
    return rowblock_kernel_ptr<__nv_bfloat16>(pattern, score, cpt);
}
} // namespace ss24
