// Dequantization: the stored outputs of a pass back to the dense fp32 operand
// they stand for ("Is 2:4 Sparsity Still Worth It?" §4: the 2:4 error of an
// element is x - x_hat, with x_hat the dequantized value on kept positions and
// 0 on dropped ones). The dequantized values are the products the pass forms,
// decode(code) * scale rounded once, so x_hat is exactly the pass's own
// reconstruction.
//
// Work is cut into quads, 4 consecutive outputs of a row (k is a multiple of 8,
// so a row holds a whole number of quads and of metadata bytes). The outputs of
// a batch are packed operand after operand, so every stored index is linear in
// the global quad index Q: the quad's codes start at entry 4Q (dense), 2Q (2:4)
// or 4(Q >> 1) (4:8), its metadata nibble is Q (2:4) or Q >> 1 (4:8), and the
// group or block scale follows from the entry index. Only a per-row INT scale
// (the row of Q) and a per-tensor scale (the operand of Q) need a division;
// both come from a grid-stride tracker plus a multiply-shift division of a
// small remainder (Granlund and Montgomery, "Division by Invariant Integers
// using Multiplication": with s = 31 + ceil(log2 d) and m = floor(2^s / d) + 1,
// floor(n / d) = (n * m) >> s for every n < 2^31).
//
// A CTA takes units of kUnitQuads quads; each thread loads the codes, metadata
// and scales of its four quads first and then writes four float4, every store
// instruction of a warp covering 512 contiguous bytes. The write of x_hat
// (16 bytes per quad) dominates the traffic: the kernel is HBM-bound.
#include "device.cuh"
#include "internal.cuh"

namespace ss24 {

namespace {

constexpr int kDqThreads = 256;
constexpr int kDqPerThread = 4;
constexpr int kUnitQuads = kDqThreads * kDqPerThread;

struct DequantParams {
    int64_t quads;              // output quads over the batch
    int64_t qpo;                // quads per operand
    uint32_t qpr;               // quads per row (k / 4)
    uint32_t qpr_m;             // multiply-shift reciprocal of qpr
    int32_t qpr_s;
    uint32_t qpo_m;             // of qpo when qpo < 2^30 (qpo_s >= 0); else qpo_s = -1
    int32_t qpo_s;
    int32_t lg;                 // INT: log2 of the group of quantized values; one scale per row: -1
    int64_t step_rows;          // gridDim.x * kUnitQuads = step_rows * qpr + step_rrem
    uint32_t step_rrem;
    int64_t step_ops;           // gridDim.x * kUnitQuads = step_ops * qpo + step_orem
    int64_t step_orem;
    const uint8_t *values, *scales, *meta;
    const float *tensor_scale;  // [batch] (FP8, NVFP4)
    float *xhat;                // [batch][rows][k]
};

__device__ __forceinline__ uint32_t mulshift_div(uint32_t n, uint32_t m, int s)
{
    return static_cast<uint32_t>((static_cast<uint64_t>(n) * m) >> s);
}

// The NE codes of CB bits each that start at entry e (e is a multiple of NE, so
// the load is naturally aligned), as little-endian words.
template <int CB, int NE> __device__ __forceinline__ uint4 load_codes(const uint8_t *vals, int64_t e)
{
    constexpr int kBytes = CB * NE / 8;
    const uint8_t *ptr = vals + e * CB / 8;
    uint4 w = make_uint4(0u, 0u, 0u, 0u);
    if constexpr (kBytes == 1) {
        w.x = __ldg(ptr);
    } else if constexpr (kBytes == 2) {
        w.x = __ldg(reinterpret_cast<const unsigned short *>(ptr));
    } else if constexpr (kBytes == 4) {
        w.x = __ldg(reinterpret_cast<const unsigned int *>(ptr));
    } else if constexpr (kBytes == 8) {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(ptr));
        w.x = v.x;
        w.y = v.y;
    } else {
        w = __ldg(reinterpret_cast<const uint4 *>(ptr));
    }
    return w;
}

template <int CB> __device__ __forceinline__ uint32_t code_at(const uint4 &w, int i)
{
    if constexpr (CB == 32) {
        return i == 0 ? w.x : i == 1 ? w.y : i == 2 ? w.z : w.w;
    } else if constexpr (CB == 16) {
        const uint32_t word = i < 2 ? w.x : w.y;
        return (word >> (16 * (i & 1))) & 0xffffu;
    } else if constexpr (CB == 8) {
        return (w.x >> (8 * i)) & 0xffu;
    } else {
        return (w.x >> (4 * i)) & 0xfu;
    }
}

// Decoded value of one code, times the quad's scale (rounded once).
template <int FMT, int CB> __device__ __forceinline__ float dq_value(uint32_t c, float scale)
{
    if constexpr (FMT == kNone) {
        return __uint_as_float(CB == 16 ? c << 16 : c);
    } else {
        static_assert(FMT == kInt, "FP8 and E2M1 codes are decoded in pairs");
        const int code = CB == 16 ? static_cast<int>(static_cast<int16_t>(c))
                         : CB == 8 ? static_cast<int>(static_cast<int8_t>(c))
                                   : static_cast<int>(c << 28) >> 28;
        return __fmul_rn(static_cast<float>(code), scale);
    }
}

template <int PAT> __host__ __device__ constexpr int entries_per_quad() { return PAT == kSparse24 ? 2 : 4; }

template <int PAT> __device__ __forceinline__ int64_t first_entry(int64_t q)
{
    if constexpr (PAT == kDense)
        return 4 * q;
    else if constexpr (PAT == kSparse24)
        return 2 * q;
    else
        return 4 * (q >> 1);
}

template <int PAT, int FMT, int CB>
__global__ void __launch_bounds__(kDqThreads) dequant_kernel(const __grid_constant__ DequantParams p)
{
    constexpr int NE = entries_per_quad<PAT>();
    constexpr bool kRowScale = FMT == kInt;       // per-row INT scale needs the row (lg < 0)
    constexpr bool kTensorScale = FMT == kFp8 || FMT == kNvfp4;
    grid_dependency_wait();
    grid_dependents_launch();
    const uint32_t base = blockIdx.x * static_cast<uint32_t>(kUnitQuads); // < 2^31
    // trackers: row0 = B / qpr, rrem = B % qpr; op0 = B / qpo, orem = B % qpo
    int64_t row0 = 0, op0 = 0, orem = 0;
    uint32_t rrem = 0;
    if constexpr (kRowScale) {
        row0 = mulshift_div(base, p.qpr_m, p.qpr_s);
        rrem = base - static_cast<uint32_t>(row0) * p.qpr;
    }
    if constexpr (kTensorScale) {
        if (p.qpo_s >= 0)
            op0 = mulshift_div(base, p.qpo_m, p.qpo_s);
        else
            op0 = static_cast<int64_t>(base) >= p.qpo ? 1 : 0;
        orem = static_cast<int64_t>(base) - op0 * p.qpo;
    }
    for (int64_t b = base; b < p.quads; b += static_cast<int64_t>(gridDim.x) * kUnitQuads) {
        uint4 raw[kDqPerThread];
        uint32_t nib[kDqPerThread];
        float scale[kDqPerThread];
#pragma unroll
        for (int i = 0; i < kDqPerThread; ++i) {
            const int d = i * kDqThreads + static_cast<int>(threadIdx.x);
            const int64_t q = b + d;
            raw[i] = make_uint4(0u, 0u, 0u, 0u);
            nib[i] = 0u;
            scale[i] = 1.0f;
            if (q >= p.quads)
                continue;
            const int64_t e = first_entry<PAT>(q);
            raw[i] = load_codes<CB, NE>(p.values, e);
            if constexpr (PAT == kSparse24)
                nib[i] = (__ldg(p.meta + (q >> 1)) >> (4 * (q & 1))) & 0xfu;
            else if constexpr (PAT == kSparse48)
                nib[i] = (__ldg(p.meta + (q >> 2)) >> (4 * ((q >> 1) & 1))) & 0xfu;
            float st = 1.0f;
            if constexpr (kTensorScale) {
                const int64_t t = orem + d;
                const int64_t op = op0 + (p.qpo_s >= 0 ? static_cast<int64_t>(
                                                             mulshift_div(static_cast<uint32_t>(t), p.qpo_m, p.qpo_s))
                                                       : (t >= p.qpo ? 1 : 0));
                st = __ldg(p.tensor_scale + op);
            }
            if constexpr (FMT == kFp8) {
                scale[i] = st;
            } else if constexpr (FMT == kInt) {
                const float *sc = reinterpret_cast<const float *>(p.scales);
                if (p.lg >= 0) {
                    scale[i] = __ldg(sc + (e >> p.lg));
                } else {
                    const uint32_t t = rrem + static_cast<uint32_t>(d);
                    scale[i] = __ldg(sc + row0 + mulshift_div(t, p.qpr_m, p.qpr_s));
                }
            } else if constexpr (FMT == kNvfp4) {
                scale[i] = __fmul_rn(e4m3_to_f32(__ldg(p.scales + (e >> 4))), st);
            } else if constexpr (FMT == kMxfp4) {
                scale[i] = exp2_int(static_cast<int>(__ldg(p.scales + (e >> 5))) - 127);
            }
        }
#pragma unroll
        for (int i = 0; i < kDqPerThread; ++i) {
            const int64_t q = b + i * kDqThreads + static_cast<int>(threadIdx.x);
            if (q >= p.quads)
                continue;
            float v[NE];
            if constexpr (FMT == kFp8 || FMT == kNvfp4 || FMT == kMxfp4) {
                // two codes per conversion: E4M3 pairs from 16 bits, E2M1 pairs from 8
#pragma unroll
                for (int j = 0; j < NE; j += 2) {
                    const float2 d2 = FMT == kFp8 ? e4m3x2_to_f32((raw[i].x >> (8 * j)) & 0xffffu)
                                                  : e2m1x2_to_f32((raw[i].x >> (4 * j)) & 0xffu);
                    v[j] = __fmul_rn(d2.x, scale[i]);
                    v[j + 1] = __fmul_rn(d2.y, scale[i]);
                }
            } else {
#pragma unroll
                for (int j = 0; j < NE; ++j)
                    v[j] = dq_value<FMT, CB>(code_at<CB>(raw[i], j), scale[i]);
            }
            float o[4];
            if constexpr (PAT == kDense) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    o[j] = v[j];
            } else if constexpr (PAT == kSparse24) {
                const uint32_t a = nib[i] & 3u, c = nib[i] >> 2;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    o[j] = c == static_cast<uint32_t>(j) ? v[1] : (a == static_cast<uint32_t>(j) ? v[0] : 0.0f);
            } else {
                // pairs 2h and 2h + 1 of the 8-block; kept pairs at p0 (entries 0, 1) and p1 (entries 2, 3)
                const uint32_t h = static_cast<uint32_t>(q & 1), p0 = nib[i] & 3u, p1 = nib[i] >> 2;
#pragma unroll
                for (int s = 0; s < 2; ++s) {
                    const uint32_t pair = 2 * h + s;
                    o[2 * s] = p1 == pair ? v[2] : (p0 == pair ? v[0] : 0.0f);
                    o[2 * s + 1] = p1 == pair ? v[3] : (p0 == pair ? v[1] : 0.0f);
                }
            }
            __stcs(reinterpret_cast<float4 *>(p.xhat) + q, make_float4(o[0], o[1], o[2], o[3]));
        }
        if constexpr (kRowScale) {
            row0 += p.step_rows;
            rrem += p.step_rrem;
            if (rrem >= p.qpr) {
                rrem -= p.qpr;
                ++row0;
            }
        }
        if constexpr (kTensorScale) {
            op0 += p.step_ops;
            orem += p.step_orem;
            if (orem >= p.qpo) {
                orem -= p.qpo;
                ++op0;
            }
        }
    }
}

template <int PAT, int FMT, int CB> const void *dq_ptr()
{
    return reinterpret_cast<const void *>(&dequant_kernel<PAT, FMT, CB>);
}

template <int PAT> const void *dequant_for_fmt(int fmt, int32_t store, bool none_f32)
{
    switch (fmt) {
    case kNone:
        if constexpr (PAT != kDense)
            return none_f32 ? dq_ptr<PAT, kNone, 32>() : dq_ptr<PAT, kNone, 16>();
        break;
    case kFp8:
        return dq_ptr<PAT, kFp8, 8>();
    case kInt:
        return store == kInt16 ? dq_ptr<PAT, kInt, 16>() : store == kInt8 ? dq_ptr<PAT, kInt, 8>()
                                                                           : dq_ptr<PAT, kInt, 4>();
    case kNvfp4:
        return dq_ptr<PAT, kNvfp4, 4>();
    case kMxfp4:
        return dq_ptr<PAT, kMxfp4, 4>();
    }
    return nullptr;
}

// s = 31 + ceil(log2 d), m = floor(2^s / d) + 1 (d <= 2^30, so m < 2^32)
void mulshift_for(uint64_t d, uint32_t *m, int32_t *s)
{
    int l = 0;
    while ((uint64_t{1} << l) < d)
        ++l;
    *s = 31 + l;
    *m = static_cast<uint32_t>((uint64_t{1} << *s) / d + 1);
}

} // namespace

cudaError_t launch_dequant(int pattern, int fmt, int32_t store, int32_t lg, int32_t none_f32, int64_t rows,
                           int64_t k, int32_t batch, const void *values, const void *scales, const float *tscale,
                           const uint8_t *meta, float *xhat, cudaStream_t stream)
{
    const void *kern = pattern == kDense      ? dequant_for_fmt<kDense>(fmt, store, none_f32 != 0)
                       : pattern == kSparse24 ? dequant_for_fmt<kSparse24>(fmt, store, none_f32 != 0)
                                              : dequant_for_fmt<kSparse48>(fmt, store, none_f32 != 0);
    if (!kern)
        return cudaErrorInvalidValue;
    const int64_t qpr = k / 4, qpo = rows * qpr, quads = qpo * batch;
    if (quads == 0)
        return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int per_sm = 0;
    cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kDqThreads, 0);
    if (err != cudaSuccess)
        return err;
    const int64_t units = (quads + kUnitQuads - 1) / kUnitQuads,
                  cap = static_cast<int64_t>(sms) * (per_sm > 0 ? per_sm : 1);
    const int64_t grid = units < cap ? units : cap;
    DequantParams p{};
    p.quads = quads;
    p.qpo = qpo;
    p.qpr = static_cast<uint32_t>(qpr);
    mulshift_for(static_cast<uint64_t>(qpr), &p.qpr_m, &p.qpr_s);
    p.qpo_s = -1;
    if (qpo < (int64_t{1} << 30))
        mulshift_for(static_cast<uint64_t>(qpo), &p.qpo_m, &p.qpo_s);
    p.lg = lg;
    const int64_t step = grid * kUnitQuads;
    p.step_rows = step / qpr;
    p.step_rrem = static_cast<uint32_t>(step % qpr);
    p.step_ops = step / qpo;
    p.step_orem = step % qpo;
    p.values = static_cast<const uint8_t *>(values);
    p.scales = static_cast<const uint8_t *>(scales);
    p.meta = meta;
    p.tensor_scale = tscale;
    p.xhat = xhat;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(kDqThreads);
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
