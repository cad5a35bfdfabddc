// Block Hadamard rotation along the reduction axis ("Is 2:4 Sparsity Still
// Worth It?" §4: before low-bit quantization a tensor is often multiplied by a
// Hadamard matrix, an orthogonal matrix of +-1 entries rescaled, which spreads
// outliers over many elements). Every block of b consecutive elements of a row
// (b a power of two, 2..256, dividing k) is multiplied by the Sylvester matrix
// H_b and by c_b = RN(1/sqrt(b)), in binary32: the fast Walsh-Hadamard
// butterflies in stage order h = 1, 2, 4, ..., b/2, each pair (y_i, y_i+h)
// with (i & h) == 0 becoming (y_i + y_i+h, y_i - y_i+h), each result rounded,
// then one rounded multiplication by c_b.
//
// A thread holds one chunk of 8 consecutive elements; a warp holds 32
// consecutive chunks of the flattened [batch, rows, k / 8] chunk index, so
// (k being a multiple of b) the partner of every butterfly with h >= 8 sits
// in lane ^ (h / 8) of the same warp: strides 1, 2, 4 run in registers and
// strides 8..128 through warp shuffles, the lower lane taking own + partner
// and the upper lane partner - own (the pair's y_i - y_i+h). The output is
// fp32, packed [batch, rows, k]. The launch reads 2 (bf16) or 4 (fp32) and
// writes 4 bytes per element: HBM-bound.
#include "device.cuh"
#include "internal.cuh"

namespace ss24 {

namespace {

constexpr int kRotThreads = 256;

struct RotParams {
    const uint8_t *x;
    float *out;
    int64_t rows, ld, bstride; // ld, bstride in elements
    int64_t cpr;               // chunks per row (k / 8)
    int64_t chunks;            // over the batch
    int32_t esize;             // 2 (bf16) or 4 (fp32)
    int32_t log2b;
    float cb;
};

__device__ __forceinline__ void bfly(float &a, float &c)
{
    const float s = __fadd_rn(a, c), d = __fsub_rn(a, c);
    a = s;
    c = d;
}

template <bool BF16> __global__ void __launch_bounds__(kRotThreads) hadamard_kernel(const __grid_constant__ RotParams p)
{
    grid_dependency_wait();
    grid_dependents_launch();
    const int lane = static_cast<int>(threadIdx.x & 31);
    const int64_t tiles = (p.chunks + 31) >> 5;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (kRotThreads / 32);
    for (int64_t t = blockIdx.x * static_cast<int64_t>(kRotThreads / 32) + (threadIdx.x >> 5); t < tiles;
         t += warps) {
        const int64_t c = t * 32 + lane;
        const bool ok = c < p.chunks;
        float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (ok) {
            const int64_t grow = c / p.cpr, c8 = c - grow * p.cpr;
            const int64_t op = grow / p.rows, r = grow - op * p.rows;
            const uint8_t *src = p.x + (op * p.bstride + r * p.ld + 8 * c8) * p.esize;
            if constexpr (BF16) {
                const uint4 w = *reinterpret_cast<const uint4 *>(src);
                const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    y[2 * i] = __uint_as_float(ws[i] << 16);
                    y[2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
                }
            } else {
                const float4 a = reinterpret_cast<const float4 *>(src)[0];
                const float4 b = reinterpret_cast<const float4 *>(src)[1];
                y[0] = a.x, y[1] = a.y, y[2] = a.z, y[3] = a.w;
                y[4] = b.x, y[5] = b.y, y[6] = b.z, y[7] = b.w;
            }
        }
        // strides 1, 2, 4 inside the chunk
#pragma unroll
        for (int s = 0; s < 3; ++s) {
            if (s >= p.log2b)
                break;
            const int h = 1 << s;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if ((i & h) == 0)
                    bfly(y[i], y[i + h]);
        }
        // strides 8 .. b/2 across lanes (the whole warp takes part)
        for (int s = 3; s < p.log2b; ++s) {
            const int m = 1 << (s - 3);
            const bool upper = (lane & m) != 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float o = __shfl_xor_sync(0xffffffffu, y[i], m);
                y[i] = upper ? __fsub_rn(o, y[i]) : __fadd_rn(y[i], o);
            }
        }
        if (ok) {
            float4 *dst = reinterpret_cast<float4 *>(p.out + 8 * c);
            dst[0] = make_float4(__fmul_rn(y[0], p.cb), __fmul_rn(y[1], p.cb), __fmul_rn(y[2], p.cb),
                                 __fmul_rn(y[3], p.cb));
            dst[1] = make_float4(__fmul_rn(y[4], p.cb), __fmul_rn(y[5], p.cb), __fmul_rn(y[6], p.cb),
                                 __fmul_rn(y[7], p.cb));
        }
    }
}

} // namespace

cudaError_t launch_hadamard(const void *x, int bf16, int64_t rows, int64_t k, int64_t ld, int64_t bstride,
                            int64_t batch, int32_t block, float *out, cudaStream_t stream)
{
    RotParams p{};
    p.x = static_cast<const uint8_t *>(x);
    p.out = out;
    p.rows = rows;
    p.ld = ld;
    p.bstride = bstride;
    p.cpr = k / 8;
    p.chunks = batch * rows * p.cpr;
    p.esize = bf16 ? 2 : 4;
    int l = 0;
    while ((1 << l) < block)
        ++l;
    p.log2b = l;
    p.cb = static_cast<float>(1.0 / sqrt(static_cast<double>(block)));
    if (p.chunks == 0)
        return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t tiles = (p.chunks + 31) / 32, want = (tiles + kRotThreads / 32 - 1) / (kRotThreads / 32);
    const int64_t cap = static_cast<int64_t>(sms) * 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(want < cap ? want : cap));
    cfg.blockDim = dim3(kRotThreads);
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void *args[1] = {&p};
    const void *kern = bf16 ? reinterpret_cast<const void *>(&hadamard_kernel<true>)
                            : reinterpret_cast<const void *>(&hadamard_kernel<false>);
    return cudaLaunchKernelExC(&cfg, kern, args);
}

} // namespace ss24
