// Dequantization: the stored outputs of a pass back to the dense fp32 operand
// they stand for ("Is 2:4 Sparsity Still Worth It?" §4: the 2:4 error of an
// element is x - x_hat, with x_hat the dequantized value on kept positions and
// 0 on dropped ones). The dequantized values are the products the pass forms,
// decode(code) * scale rounded once, so x_hat is exactly the pass's own
// reconstruction. One thread per 8 output elements (one chunk); the outputs of
// a batch are packed operand after operand, as the pass writes them.
#include "device.cuh"
#include "internal.cuh"

namespace ss24 {

struct DequantParams {
    int64_t rows, k, n;           // per operand; n: quantized row length (k / 2 sparse, k dense)
    int32_t store;                // INT code width (IntStore)
    int32_t lg;                   // INT: log2 of the group (group 0: the whole row, lg < 0)
    int32_t none_f32;             // format NONE: kept values are fp32 (else bf16)
    int32_t batch;
    const uint8_t *values, *scales, *meta;
    const float *tensor_scale;    // [batch] (FP8, NVFP4)
    float *xhat;                  // [batch][rows][k]
    int64_t values_bstride, scales_bstride, meta_bstride; // bytes per operand
};

// Entry j of quantized row r of one operand (the operand's base pointers).
template <int FMT>
__device__ __forceinline__ float dq_entry(const DequantParams &p, const uint8_t *vals, const uint8_t *sc, float st,
                                          int64_t r, int64_t j)
{
    const int64_t off = r * p.n + j;
    if constexpr (FMT == kNone) {
        if (p.none_f32)
            return reinterpret_cast<const float *>(vals)[off];
        return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t *>(vals)[off]) << 16);
    } else if constexpr (FMT == kFp8) {
        return __fmul_rn(e4m3_to_f32(vals[off]), st);
    } else if constexpr (FMT == kInt) {
        int code;
        if (p.store == kInt8) {
            code = static_cast<int8_t>(vals[off]);
        } else if (p.store == kInt16) {
            code = reinterpret_cast<const int16_t *>(vals)[off];
        } else {
            const int nib = (vals[off >> 1] >> (4 * (off & 1))) & 0xF;
            code = nib >= 8 ? nib - 16 : nib;
        }
        const int64_t gi = p.lg >= 0 ? (r * (p.n >> p.lg) + (j >> p.lg)) : r;
        return __fmul_rn(static_cast<float>(code), reinterpret_cast<const float *>(sc)[gi]);
    } else if constexpr (FMT == kNvfp4) {
        const float denom = __fmul_rn(e4m3_to_f32(sc[r * (p.n / 16) + j / 16]), st);
        const uint32_t code = (vals[off >> 1] >> (4 * (off & 1))) & 0xFu;
        return __fmul_rn(e2m1x2_to_f32(code).x, denom);
    } else { // kMxfp4
        const int e = static_cast<int>(sc[r * (p.n / 32) + j / 32]) - 127;
        const uint32_t code = (vals[off >> 1] >> (4 * (off & 1))) & 0xFu;
        return __fmul_rn(e2m1x2_to_f32(code).x, exp2_int(e));
    }
}

template <int PAT, int FMT>
__global__ void __launch_bounds__(256) dequant_kernel(const __grid_constant__ DequantParams p)
{
    grid_dependency_wait();
    grid_dependents_launch();
    const int64_t cpr = p.k / 8; // chunks per row
    const int64_t per_op = p.rows * cpr;
    const int64_t total = per_op * p.batch;
    for (int64_t c = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; c < total;
         c += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int op = static_cast<int>(c / per_op);
        const int64_t rc = c - op * per_op;
        const int64_t r = rc / cpr, c8 = rc - r * cpr;
        const uint8_t *vals = p.values + op * p.values_bstride;
        const uint8_t *sc = p.scales ? p.scales + op * p.scales_bstride : nullptr;
        const float st = p.tensor_scale ? p.tensor_scale[op] : 0.0f;
        float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if constexpr (PAT == kDense) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
                o[i] = dq_entry<FMT>(p, vals, sc, st, r, 8 * c8 + i);
        } else if constexpr (PAT == kSparse24) {
            const uint32_t byte = (p.meta + op * p.meta_bstride)[r * (p.k / 8) + c8];
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                const uint32_t nib = (byte >> (4 * g)) & 0xFu;
                o[4 * g + (nib & 3u)] = dq_entry<FMT>(p, vals, sc, st, r, 4 * c8 + 2 * g);
                o[4 * g + (nib >> 2)] = dq_entry<FMT>(p, vals, sc, st, r, 4 * c8 + 2 * g + 1);
            }
        } else {
            const uint32_t byte = (p.meta + op * p.meta_bstride)[r * (p.k / 16) + c8 / 2];
            const uint32_t nib = (byte >> (4 * (c8 & 1))) & 0xFu;
            const uint32_t p0 = nib & 3u, p1 = nib >> 2;
            o[2 * p0] = dq_entry<FMT>(p, vals, sc, st, r, 4 * c8);
            o[2 * p0 + 1] = dq_entry<FMT>(p, vals, sc, st, r, 4 * c8 + 1);
            o[2 * p1] = dq_entry<FMT>(p, vals, sc, st, r, 4 * c8 + 2);
            o[2 * p1 + 1] = dq_entry<FMT>(p, vals, sc, st, r, 4 * c8 + 3);
        }
        float4 *dst = reinterpret_cast<float4 *>(p.xhat + c * 8);
        dst[0] = make_float4(o[0], o[1], o[2], o[3]);
        dst[1] = make_float4(o[4], o[5], o[6], o[7]);
    }
}

template <int PAT> const void *dequant_for_fmt(int fmt)
{
    switch (fmt) {
    case kNone:
        if constexpr (PAT != kDense)
            return reinterpret_cast<const void *>(&dequant_kernel<PAT, kNone>);
        break;
    case kFp8:
        return reinterpret_cast<const void *>(&dequant_kernel<PAT, kFp8>);
    case kInt:
        return reinterpret_cast<const void *>(&dequant_kernel<PAT, kInt>);
    case kNvfp4:
        return reinterpret_cast<const void *>(&dequant_kernel<PAT, kNvfp4>);
    case kMxfp4:
        return reinterpret_cast<const void *>(&dequant_kernel<PAT, kMxfp4>);
    }
    return nullptr;
}

cudaError_t launch_dequant(int pattern, int fmt, int32_t store, int32_t lg, int32_t none_f32, int64_t rows,
                           int64_t k, int32_t batch, const void *values, const void *scales, const float *tscale,
                           const uint8_t *meta, float *xhat, int64_t values_bstride, int64_t scales_bstride,
                           int64_t meta_bstride, cudaStream_t stream)
{
    const void *kern = pattern == kDense      ? dequant_for_fmt<kDense>(fmt)
                       : pattern == kSparse24 ? dequant_for_fmt<kSparse24>(fmt)
                                              : dequant_for_fmt<kSparse48>(fmt);
    if (!kern)
        return cudaErrorInvalidValue;
    DequantParams p{};
    p.rows = rows;
    p.k = k;
    p.n = pattern == kDense ? k : k / 2;
    p.store = store;
    p.lg = lg;
    p.none_f32 = none_f32;
    p.batch = batch;
    p.values = static_cast<const uint8_t *>(values);
    p.scales = static_cast<const uint8_t *>(scales);
    p.meta = meta;
    p.tensor_scale = tscale;
    p.xhat = xhat;
    p.values_bstride = values_bstride;
    p.scales_bstride = scales_bstride;
    p.meta_bstride = meta_bstride;
    const int64_t chunks = rows * (k / 8) * batch;
    if (chunks == 0)
        return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (chunks + 255) / 256, cap = static_cast<int64_t>(sms) * 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(want < cap ? want : cap));
    cfg.blockDim = dim3(256);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *args[1] = {&p};
    return cudaLaunchKernelExC(&cfg, kern, args);
}

} // namespace ss24
