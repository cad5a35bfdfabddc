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
// fp32, packed [batch, rows, k], each lane's 32 bytes in one 256-bit store when
// the output is 32-byte aligned. The launch reads 2 (bf16) or 4 (fp32) and
// writes 4 bytes per element: HBM-bound.
#include <type_traits>

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

// One 32-byte store of 8 floats (sm_100 256-bit vector store; dst 32-byte aligned).
__device__ __forceinline__ void st_v8(float *dst, const float (&v)[8])
{
    asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "f"(v[0]), "f"(v[1]),
                 "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7])
                 : "memory");
}

template <bool BF16, bool V8, bool LIN>
__global__ void __launch_bounds__(kRotThreads) hadamard_kernel(const __grid_constant__ RotParams p)
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
            // LIN: rows packed (ld == k) and operands packed, so chunk c starts
            // at element 8c; otherwise row and operand come from c
            int64_t e = 8 * c;
            if constexpr (!LIN) {
                const int64_t grow = c / p.cpr, c8 = c - grow * p.cpr;
                const int64_t op = grow / p.rows, r = grow - op * p.rows;
                e = op * p.bstride + r * p.ld + 8 * c8;
            }
            const uint8_t *src = p.x + e * p.esize;
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
        // strides 1, 2, 4 inside the chunk: two butterflies per packed add and subtract
#pragma unroll
        for (int s = 0; s < 3; ++s) {
            if (s >= p.log2b)
                break;
            const int h = 1 << s;
#pragma unroll
            for (int i0 = 0; i0 < 8; i0 += 2 * h) {
                if (h == 1 && (i0 & 2))
                    continue; // (stride 1 pairs two butterflies 2 apart)
#pragma unroll
                for (int j = 0; j < (h == 1 ? 1 : h); j += 2) {
                    // butterflies (a, a + h) and (b, b + h), a and b the pair's lower indices
                    const int a = h == 1 ? i0 : i0 + j, b = h == 1 ? i0 + 2 : i0 + j + 1;
                    const f32x2 lo = pack2(y[a], y[b]), hi = pack2(y[a + h], y[b + h]);
                    const f32x2 sm = add2(lo, hi), df = sub2(lo, hi);
                    y[a] = lo2(sm), y[b] = hi2(sm), y[a + h] = lo2(df), y[b + h] = hi2(df);
                }
            }
        }
        // strides 8 .. b/2 across lanes (the whole warp takes part): own * (+-1)
        // + partner is exactly the rounded own + partner (lower lane) or
        // partner - own (upper lane), one packed fused multiply-add per pair
        for (int s = 3; s < p.log2b; ++s) {
            const int m = 1 << (s - 3);
            const float sg = (lane & m) ? -1.0f : 1.0f;
            const f32x2 sg2 = pack2(sg, sg);
#pragma unroll
            for (int i = 0; i < 8; i += 2) {
                const float o0 = __shfl_xor_sync(0xffffffffu, y[i], m);
                const float o1 = __shfl_xor_sync(0xffffffffu, y[i + 1], m);
                const f32x2 r = fma2(pack2(y[i], y[i + 1]), sg2, pack2(o0, o1));
                y[i] = lo2(r), y[i + 1] = hi2(r);
            }
        }
        if (ok) {
            float o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                o[i] = __fmul_rn(y[i], p.cb);
            if constexpr (V8) {
                // a warp's 32 stores cover 1 KB of contiguous output
                st_v8(p.out + 8 * c, o);
            } else {
                float4 *dst = reinterpret_cast<float4 *>(p.out + 8 * c);
                dst[0] = make_float4(o[0], o[1], o[2], o[3]);
                dst[1] = make_float4(o[4], o[5], o[6], o[7]);
            }
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
    const bool v8 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
    const bool lin = ld == k && (batch == 1 || bstride == rows * k);
    const void *kern = nullptr;
    auto pick = [&](auto b16, auto vec) {
        constexpr bool B = decltype(b16)::value, V = decltype(vec)::value;
        kern = lin ? reinterpret_cast<const void *>(&hadamard_kernel<B, V, true>)
                   : reinterpret_cast<const void *>(&hadamard_kernel<B, V, false>);
    };
    using T_ = std::true_type;
    using F_ = std::false_type;
    if (bf16)
        v8 ? pick(T_{}, T_{}) : pick(T_{}, F_{});
    else
        v8 ? pick(F_{}, T_{}) : pick(F_{}, F_{});
    return cudaLaunchKernelExC(&cfg, kern, args);
}

} // namespace ss24
