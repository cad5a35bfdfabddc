// Small kernels: the predicted-ratio finalisation and the format converters.
#include "device.cuh"
#include "internal.cuh"

namespace ss24 {

// §4 of "Is 2:4 Sparsity Still Worth It?": loss = E_prune / E_total, the two
// relative errors, and R_hat = sqrt((E_prune + E_q,2m) / E_q,m+1), for `count`
// consecutive pairs of energy records.
__global__ void ratio_kernel(const double *sp, const double *de, double *out, int64_t count)
{
    grid_dependency_wait();
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < count;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const double et = sp[4 * i], ep = sp[4 * i + 1], eq = sp[4 * i + 2], ed = de[4 * i + 3];
        out[4 * i] = ep / et;
        out[4 * i + 1] = sqrt((ep + eq) / et);
        out[4 * i + 2] = sqrt(ed / et);
        out[4 * i + 3] = sqrt((ep + eq) / ed);
    }
}

cudaError_t launch_ratio(const double *sparse_side, const double *dense_side, double *out, int64_t count,
                         cudaStream_t stream)
{
    if (count <= 0)
        return cudaSuccess;
    const int64_t blocks = (count + 127) / 128;
    ratio_kernel<<<static_cast<unsigned>(blocks < 1024 ? blocks : 1024), 128, 0, stream>>>(sparse_side, dense_side,
                                                                                          out, count);
    return cudaGetLastError();
}

// op 0: f32 -> E4M3 byte; 1: E4M3 byte -> f32; 2: f32 -> E2M1 (low nibble);
// 3: E2M1 (low nibble) -> f32.
__global__ void convert_kernel(int op, const void *in, void *out, int64_t n)
{
    grid_dependency_wait();
    for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        switch (op) {
        case 0:
            static_cast<uint8_t *>(out)[i] =
                static_cast<uint8_t>(cvt_e4m3x2(static_cast<const float *>(in)[i], 0.0f) & 0xffu);
            break;
        case 1:
            static_cast<float *>(out)[i] = e4m3_to_f32(static_cast<const uint8_t *>(in)[i]);
            break;
        case 2:
            static_cast<uint8_t *>(out)[i] =
                static_cast<uint8_t>(cvt_e2m1x4(static_cast<const float *>(in)[i], 0.0f, 0.0f, 0.0f) & 0xfu);
            break;
        default:
            static_cast<float *>(out)[i] = e2m1x2_to_f32(static_cast<const uint8_t *>(in)[i] & 0xfu).x;
            break;
        }
    }
}

// Markstein's correction against IEEE division, in both forms the kernels
// use: div_fast (a / b) and the packed negated form neg_div_fast2, whose two
// lanes are checked as -(a / b) (negated back) and -(-a) / b.
// mode 0: b = 1 + (b_first + blockIdx.x) * 2^-23 against every a in [1, 2)
//         (all 2^23 significands); the full sweep over b covers every pair of
//         significands.
// mode 1: pseudo-random pairs with b in [2^-60, 2^60] and |a / b| in
//         [2^-40, 2^100] (the range where the kernels use the correction),
//         2^23 per block, from a counter-based hash of (block, index).
// result[0] += mismatches; result[1] = first mismatch as (a bits << 32 | b bits).
__device__ __forceinline__ uint32_t hash32(uint32_t x)
{
    x ^= x >> 16;
    x *= 0x7feb352du;
    x ^= x >> 15;
    x *= 0x846ca68bu;
    x ^= x >> 16;
    return x;
}

__global__ void selfcheck_division_kernel(int mode, uint32_t b_first, unsigned long long *result)
{
    unsigned long long bad = 0, first = ~0ull;
    if (mode == 0) {
        const float b = __uint_as_float(0x3f800000u | (b_first + blockIdx.x));
        const Recip rc = make_recip(b);
        for (uint32_t i = threadIdx.x; i < (1u << 23); i += blockDim.x) {
            const float a = __uint_as_float(0x3f800000u | i);
            const float q = div_fast(a, rc), ref = __fdiv_rn(a, b);
            const float qn = lo2(neg_div_fast2(pack2(a, -a), rc)), qp = hi2(neg_div_fast2(pack2(a, -a), rc));
            if (__float_as_uint(q) != __float_as_uint(ref) || __float_as_uint(-qn) != __float_as_uint(ref) ||
                __float_as_uint(qp) != __float_as_uint(ref)) {
                ++bad;
                first = min(first, (static_cast<unsigned long long>(__float_as_uint(a)) << 32) | __float_as_uint(b));
            }
        }
    } else if (mode == 1) {
        for (uint32_t i = threadIdx.x; i < (1u << 23); i += blockDim.x) {
            const uint32_t h1 = hash32(((b_first + blockIdx.x) << 23) ^ i), h2 = hash32(h1 ^ 0x9e3779b9u);
            const uint32_t h3 = hash32(h2 + 0x632be5abu);
            const int eb = static_cast<int>(h1 % 121u) - 60;            // b exponent in [-60, 60]
            const int eq = static_cast<int>(h2 % 141u) - 40;            // quotient exponent in [-40, 100]
            const float b = __uint_as_float((static_cast<uint32_t>(eb + 127) << 23) | (h3 & 0x7fffffu));
            int ea = eb + eq;
            if (ea > 127 || ea < -126)
                continue;
            const float a = __uint_as_float((h2 & 0x80000000u) | (static_cast<uint32_t>(ea + 127) << 23) |
                                            (hash32(h3) & 0x7fffffu));
            const Recip rc = make_recip(b);
            const float q = div_fast(a, rc), ref = __fdiv_rn(a, b);
            const f32x2 nq = neg_div_fast2(pack2(a, -a), rc);
            if (__float_as_uint(q) != __float_as_uint(ref) || __float_as_uint(-lo2(nq)) != __float_as_uint(ref) ||
                __float_as_uint(hi2(nq)) != __float_as_uint(ref)) {
                ++bad;
                first = min(first, (static_cast<unsigned long long>(__float_as_uint(a)) << 32) | __float_as_uint(b));
            }
        }
    } else {
        // mode 2: the packed bf16 operations of the selection and the amax,
        // for a = b_first + blockIdx.x against every b (magnitude bits < 2^15,
        // finite), signs taken from the low bits of the other operand
        const uint32_t a = b_first + blockIdx.x;
        for (uint32_t b = threadIdx.x; b < 32768u; b += blockDim.x) {
            if (((a >> 7) & 0xffu) == 0xffu || ((b >> 7) & 0xffu) == 0xffu)
                continue;
            const uint32_t sa = (b & 1u) << 15, sb = (a & 1u) << 15;
            const uint32_t ha = a | sa, hb = b | sb;
            const uint32_t u = ha | (hb << 16), v = hb | (ha << 16);   // lanes (a, b) and (b, a)
            const uint32_t gt = bf16x2_gt_abs(v, u);                    // lane 0: |b| > |a|; lane 1: |a| > |b|
            const uint32_t mx = bf16x2_maxabs(u, v);
            // the FP8 overflow guard's test of a larger magnitude against a limit
            const bool ge = bf16x2_max_ge_abs(hb | (hb << 16), 0u, a | (a << 16));
            const float fa = __uint_as_float(ha << 16), fb = __uint_as_float(hb << 16);
            bool ok = gt == ((b > a ? 0xffffu : 0u) | (a > b ? 0xffff0000u : 0u));
            ok = ok && ge == (b >= a);
            ok = ok && (mx & 0x7fffu) == max(a, b) && ((mx >> 16) & 0x7fffu) == max(a, b);
            ok = ok && bf16x2_hmax(u) == fmaxf(fabsf(fa), fabsf(fb));
            ok = ok && __float_as_uint(bf16_lo(u)) == __float_as_uint(fa) &&
                 __float_as_uint(bf16_hi(u)) == __float_as_uint(fb);
            const float c = __uint_as_float(hash32(a * 32768u + b) & 0xbf7fffffu);   // finite addend
            ok = ok && __float_as_uint(bf16_sq_lo(u, c)) == __float_as_uint(__fmaf_rn(fa, fa, c)) &&
                 __float_as_uint(bf16_sq_hi(u, c)) == __float_as_uint(__fmaf_rn(fb, fb, c));
            if (!ok) {
                ++bad;
                first = min(first, (static_cast<unsigned long long>(a) << 32) | b);
            }
        }
    }
    for (int off = 16; off >= 1; off >>= 1) {
        bad += __shfl_xor_sync(kFull, bad, off);
        first = min(first, __shfl_xor_sync(kFull, first, off));
    }
    if ((threadIdx.x & 31) == 0 && bad) {
        atomicAdd(result, bad);
        atomicMin(result + 1, first);
    }
}

cudaError_t launch_selfcheck_division(int mode, uint32_t b_first, uint32_t b_count, unsigned long long *result,
                                      cudaStream_t stream)
{
    if (b_count == 0)
        return cudaSuccess;
    selfcheck_division_kernel<<<b_count, 256, 0, stream>>>(mode, b_first, result);
    return cudaGetLastError();
}

// The kernels' encoders (cvt ... satfinite) against a step table: for the
// fp32 bit patterns (hi << 16) | lo, hi = hi_first + blockIdx.x, every lo,
// finite values only, the expected code of |x| is the number of bounds <= the
// magnitude bits (bounds ascending: bounds[i] is the smallest magnitude whose
// code is i + 1), with the sign bit (0x80 / 0x8) set for negative x, -0
// included. e2m1: 0 = E4M3 (126 bounds), 1 = E2M1 (7 bounds).
__global__ void selfcheck_encoder_kernel(int e2m1, const uint32_t *bounds, int n_bounds, uint32_t hi_first,
                                         unsigned long long *result)
{
    __shared__ uint32_t b[128];
    for (int i = threadIdx.x; i < n_bounds; i += blockDim.x)
        b[i] = bounds[i];
    __syncthreads();
    unsigned long long bad = 0, first = ~0ull;
    const uint32_t hi = hi_first + blockIdx.x;
    for (uint32_t lo = threadIdx.x; lo < 65536u; lo += blockDim.x) {
        const uint32_t bits = (hi << 16) | lo;
        if (((bits >> 23) & 0xffu) == 0xffu)
            continue;
        const uint32_t mag = bits & 0x7fffffffu;
        int lo_i = 0, hi_i = n_bounds; // count of bounds <= mag (upper bound search)
        while (lo_i < hi_i) {
            const int mid = (lo_i + hi_i) >> 1;
            if (b[mid] <= mag)
                lo_i = mid + 1;
            else
                hi_i = mid;
        }
        const float x = __uint_as_float(bits);
        uint32_t want, got;
        if (e2m1) {
            want = static_cast<uint32_t>(lo_i) | ((bits >> 31) << 3);
            got = cvt_e2m1x4(x, 0.0f, 0.0f, 0.0f) & 0xfu;
        } else {
            want = static_cast<uint32_t>(lo_i) | ((bits >> 31) << 7);
            got = cvt_e4m3x2(x, 0.0f) & 0xffu;
        }
        if (want != got) {
            ++bad;
            first = min(first, static_cast<unsigned long long>(bits));
        }
    }
    for (int off = 16; off >= 1; off >>= 1) {
        bad += __shfl_xor_sync(kFull, bad, off);
        first = min(first, __shfl_xor_sync(kFull, first, off));
    }
    if ((threadIdx.x & 31) == 0 && bad) {
        atomicAdd(result, bad);
        atomicMin(result + 1, first);
    }
}

cudaError_t launch_selfcheck_encoder(int e2m1, const uint32_t *bounds, int n_bounds, uint32_t hi_first,
                                     uint32_t hi_count, unsigned long long *result, cudaStream_t stream)
{
    if (hi_count == 0)
        return cudaSuccess;
    selfcheck_encoder_kernel<<<hi_count, 256, 0, stream>>>(e2m1, bounds, n_bounds, hi_first, result);
    return cudaGetLastError();
}

cudaError_t launch_convert(int op, const void *in, void *out, int64_t n, cudaStream_t stream)
{
    if (n <= 0)
        return cudaSuccess;
    const int threads = 256;
    const int64_t want = (n + threads - 1) / threads;
    const int blocks = static_cast<int>(want < 4096 ? want : 4096);
    convert_kernel<<<blocks, threads, 0, stream>>>(op, in, out, n);
    return cudaGetLastError();
}

} // namespace ss24
