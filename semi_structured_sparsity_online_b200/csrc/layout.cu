// Consumer layouts: the NVFP4 / MXFP4 scale bytes of a pass rearranged into the
// 128 x 4 tiles in which the tensor cores' block-scaled MMA takes its scale
// factors (NVIDIA's documented "1D block scaling factors layout"): the scale
// matrix padded with zeros to multiples of 128 rows and 4 columns, 512-byte
// tiles row tile by row tile, and inside a tile row 32 a + b, column j at byte
// 16 b + 4 a + j.
//
// One thread writes one 16-byte line of a tile (rows b, 32 + b, 64 + b, 96 + b
// of the tile, its 4 columns), so consecutive threads store consecutive lines
// and a warp writes one whole tile. The scale bytes are 1/32 (NVFP4, 2:4) to
// 1/64 of a byte per operand element: the launch moves a few MB for a
// 4096 x 4096 batch of 8.
#include "device.cuh"
#include "internal.cuh"

namespace ss24 {

namespace {

struct TileParams {
    const uint8_t *in;
    uint8_t *out;
    int64_t rows, cols;
    int64_t ctiles;     // column tiles per operand (ceil(cols / 4))
    int64_t lines_op;   // 16-byte lines per operand (32 per tile)
    int64_t lines;      // over the batch
};

__global__ void __launch_bounds__(256) scale_tiles_kernel(const __grid_constant__ TileParams p)
{
    grid_dependency_wait();
    grid_dependents_launch();
    for (int64_t g = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; g < p.lines;
         g += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t op = g / p.lines_op, lo = g - op * p.lines_op;
        const int64_t tile = lo >> 5;
        const int b = static_cast<int>(lo & 31);
        const int64_t rt = tile / p.ctiles, ct = tile - rt * p.ctiles;
        const uint8_t *src = p.in + op * p.rows * p.cols;
        uint32_t w[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int64_t r = rt * 128 + 32 * a + b;
            uint32_t word = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int64_t c = ct * 4 + j;
                if (r < p.rows && c < p.cols)
                    word |= static_cast<uint32_t>(__ldg(src + r * p.cols + c)) << (8 * j);
            }
            w[a] = word;
        }
        reinterpret_cast<uint4 *>(p.out)[g] = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

} // namespace

int64_t scale_tiles_bytes(int64_t rows, int64_t cols)
{
    if (rows < 0 || cols < 0)
        return -1;
    return ((rows + 127) / 128) * ((cols + 3) / 4) * 512;
}

cudaError_t launch_scale_tiles(const uint8_t *in, int64_t rows, int64_t cols, int64_t batch, uint8_t *out,
                               cudaStream_t stream)
{
    TileParams p{};
    p.in = in;
    p.out = out;
    p.rows = rows;
    p.cols = cols;
    p.ctiles = (cols + 3) / 4;
    p.lines_op = scale_tiles_bytes(rows, cols) / 16;
    p.lines = p.lines_op * batch;
    if (p.lines == 0)
        return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t want = (p.lines + 255) / 256, cap = static_cast<int64_t>(sms) * 8;
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
    return cudaLaunchKernelExC(&cfg, reinterpret_cast<const void *>(&scale_tiles_kernel), args);
}

} // namespace ss24
