// Instantiations of the stream kernel for passes over the rotated operand
// (bf16, magnitude score; block Hadamard along k in registers before the
// selection, "Is 2:4 Sparsity Still Worth It?" §4).
#include "pass_dispatch.cuh"

namespace ss24 {

namespace {

template <bool FW> const void *rot_pat(int pattern, int fmt)
{
    constexpr int SC = kMag | kRotated;
    if (pattern == kDense)
        return stream_kernel_for_fmt<__nv_bfloat16, kDense, SC, FW>(fmt);
    if (pattern == kSparse24)
        return stream_kernel_for_fmt<__nv_bfloat16, kSparse24, SC, FW>(fmt);
    if (pattern == kSparse48)
        return stream_kernel_for_fmt<__nv_bfloat16, kSparse48, SC, FW>(fmt);
    return nullptr;
}

} // namespace

const void *stream_kernel_bf16_rot(int pattern, int fmt, bool fw)
{
    return fw ? rot_pat<true>(pattern, fmt) : rot_pat<false>(pattern, fmt);
}

} // namespace ss24
