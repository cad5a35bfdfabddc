// Small kernels: the predicted-ratio finalisation and the format converters.
#include "device.cuh"
#include "internal.cuh"

namespace ss24 {

// §4 of "Is 2:4 Sparsity Still Worth It?": loss = E_prune / E_total, the two
// relative errors, and R_hat = sqrt((E_prune + E_q,2m) / E_q,m+1).
__global__ void ratio_kernel(const double *sp, const double *de, double *out)
{
    const double et = sp[0], ep = sp[1], eq = sp[2], ed = de[3];
    out[0] = ep / et;
    out[1] = sqrt((ep + eq) / et);
    out[2] = sqrt(ed / et);
    out[3] = sqrt((ep + eq) / ed);
}

cudaError_t launch_ratio(const double *sparse_side, const double *dense_side, double *out, cudaStream_t stream)
{
    ratio_kernel<<<1, 1, 0, stream>>>(sparse_side, dense_side, out);
    return cudaGetLastError();
}

// op 0: f32 -> E4M3 byte; 1: E4M3 byte -> f32; 2: f32 -> E2M1 (low nibble);
// 3: E2M1 (low nibble) -> f32.
__global__ void convert_kernel(int op, const void *in, void *out, int64_t n)
{
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
