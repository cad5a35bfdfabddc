// Kernel tables for one element type: maps (pattern, score, format) to the
// instantiated stream (axis 1), row-sweep or axis-0 kernel.
#pragma once

#include "pass_impl.cuh"

namespace ss24 {

template <typename T, int PAT, int SC, bool FW> const void *stream_kernel_for_fmt(int fmt)
{
    switch (fmt) {
    case kNone:
        if constexpr (PAT != kDense)
            return reinterpret_cast<const void *>(&stream_kernel<T, PAT, SC, kNone, FW>);
        break;
    case kFp8:
        return reinterpret_cast<const void *>(&stream_kernel<T, PAT, SC, kFp8, FW>);
    case kInt:
        return reinterpret_cast<const void *>(&stream_kernel<T, PAT, SC, kInt, FW>);
    case kIntRows:
        return reinterpret_cast<const void *>(&stream_kernel<T, PAT, SC, kIntRows, FW>);
    case kNvfp4:
        return reinterpret_cast<const void *>(&stream_kernel<T, PAT, SC, kNvfp4, FW>);
    case kMxfp4:
        return reinterpret_cast<const void *>(&stream_kernel<T, PAT, SC, kMxfp4, FW>);
    case kAmax:
        return reinterpret_cast<const void *>(&stream_kernel<T, PAT, SC, kAmax, FW>);
    case kEnergy:
        if constexpr (PAT != kDense)
            return reinterpret_cast<const void *>(&stream_kernel<T, PAT, SC, kEnergy, FW>);
        break;
    }
    return nullptr;
}

template <typename T, bool FW> const void *stream_kernel_pat(int pattern, int score, int fmt)
{
    if (pattern == kDense)
        return stream_kernel_for_fmt<T, kDense, kMag, FW>(fmt);
    if (pattern == kSparse24)
        return score == kWanda ? stream_kernel_for_fmt<T, kSparse24, kWanda, FW>(fmt)
                               : stream_kernel_for_fmt<T, kSparse24, kMag, FW>(fmt);
    if (pattern == kSparse48)
        return score == kWanda ? stream_kernel_for_fmt<T, kSparse48, kWanda, FW>(fmt)
                               : stream_kernel_for_fmt<T, kSparse48, kMag, FW>(fmt);
    return nullptr;
}

template <typename T> const void *stream_kernel_ptr(int pattern, int score, int fmt, bool fw)
{
    return fw ? stream_kernel_pat<T, true>(pattern, score, fmt) : stream_kernel_pat<T, false>(pattern, score, fmt);
}

template <typename T> const void *rowsweep_kernel_ptr(int pattern, int score)
{
    if (pattern == kDense)
        return reinterpret_cast<const void *>(&rowsweep_kernel<T, kDense, kMag>);
    if (pattern == kSparse24)
        return score == kWanda ? reinterpret_cast<const void *>(&rowsweep_kernel<T, kSparse24, kWanda>)
                               : reinterpret_cast<const void *>(&rowsweep_kernel<T, kSparse24, kMag>);
    if (pattern == kSparse48)
        return score == kWanda ? reinterpret_cast<const void *>(&rowsweep_kernel<T, kSparse48, kWanda>)
                               : reinterpret_cast<const void *>(&rowsweep_kernel<T, kSparse48, kMag>);
    return nullptr;
}

template <typename T, int PAT, int SC> const void *rowblock_for_cpt(int cpt)
{
    switch (cpt) {
    case 1:
        return reinterpret_cast<const void *>(&rowblock_kernel<T, PAT, SC, 1>);
    case 4:
        return reinterpret_cast<const void *>(&rowblock_kernel<T, PAT, SC, 4>);
    case 8:
        return reinterpret_cast<const void *>(&rowblock_kernel<T, PAT, SC, 8>);
    }
    return nullptr;
}

template <typename T> const void *rowblock_kernel_ptr(int pattern, int score, int cpt)
{
    if (pattern == kDense)
        return rowblock_for_cpt<T, kDense, kMag>(cpt);
    if (pattern == kSparse24)
        return score == kWanda ? rowblock_for_cpt<T, kSparse24, kWanda>(cpt) : rowblock_for_cpt<T, kSparse24, kMag>(cpt);
    if (pattern == kSparse48)
        return score == kWanda ? rowblock_for_cpt<T, kSparse48, kWanda>(cpt) : rowblock_for_cpt<T, kSparse48, kMag>(cpt);
    return nullptr;
}

template <typename T, int PAT, int SC> const void *axis0_for_fmt(int fmt)
{
    switch (fmt) {
    case kNone:
        if constexpr (PAT != kDense)
            return reinterpret_cast<const void *>(&axis0_kernel<T, PAT, SC, kNone>);
        break;
    case kFp8:
        return reinterpret_cast<const void *>(&axis0_kernel<T, PAT, SC, kFp8>);
    case kInt:
        return reinterpret_cast<const void *>(&axis0_kernel<T, PAT, SC, kInt>);
    case kNvfp4:
        return reinterpret_cast<const void *>(&axis0_kernel<T, PAT, SC, kNvfp4>);
    case kMxfp4:
        return reinterpret_cast<const void *>(&axis0_kernel<T, PAT, SC, kMxfp4>);
    case kAmax:
        return reinterpret_cast<const void *>(&axis0_kernel<T, PAT, SC, kAmax>);
    case kEnergy:
        if constexpr (PAT != kDense)
            return reinterpret_cast<const void *>(&axis0_kernel<T, PAT, SC, kEnergy>);
        break;
    }
    return nullptr;
}

template <typename T> const void *axis0_kernel_ptr(int pattern, int score, int fmt)
{
    if (pattern == kDense)
        return axis0_for_fmt<T, kDense, kMag>(fmt);
    if (pattern == kSparse24)
        return score == kWanda ? axis0_for_fmt<T, kSparse24, kWanda>(fmt) : axis0_for_fmt<T, kSparse24, kMag>(fmt);
    if (pattern == kSparse48)
        return score == kWanda ? axis0_for_fmt<T, kSparse48, kWanda>(fmt) : axis0_for_fmt<T, kSparse48, kMag>(fmt);
    return nullptr;
}

} // namespace ss24
