// Internal interface between the C ABI layer (abi.cu) and the kernels
// (pass_impl.cuh, instantiated in pass_bf16.cu / pass_f32.cu; misc.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace ss24 {

enum Pattern { kDense = 0, kSparse24 = 24, kSparse48 = 48 };
enum Score { kMag = 0, kWanda = 1 };
// A stream kernel's score parameter with this bit set: the magnitude score on
// the operand rotated along k (block Hadamard, rounded to bf16) in registers.
constexpr int kRotated = 2;
// Formats of the pass; kAmax is the read-only amax pass; kEnergy the
// read-only two-format energy pass; kIntRows is INT with one scale per row
// from a given per-row amax (the stream kernel).
enum Fmt { kNone = 0, kFp8 = 1, kInt = 2, kNvfp4 = 3, kMxfp4 = 4, kAmax = 5, kEnergy = 6, kIntRows = 7 };
enum IntStore { kInt8 = 0, kInt16 = 1, kPack4 = 2 };

// How long a kernel's wait on a barrier may take before the kernel gives up,
// records an error code in the workspace and returns (instead of spinning
// forever); and the shorter limit of the test hook (see ss24.h).
constexpr uint64_t kWaitLimitNs = 2000000000ull;
constexpr uint64_t kTestWaitLimitNs = 10000000ull;

// Consumer warps per CTA and the TMA stage ring (each stage 16 KiB).
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32; // + one producer warp
constexpr int kStageBytes = 16384;
constexpr int kStages = 4;
constexpr int kMaxGrid = 1024;            // bound on CTAs (workspace partials)
constexpr size_t kSmemBytes = kStages * kStageBytes + 4096;

// The axis-1 stream kernel: 8 warps per CTA, no shared-memory stages. The
// block reductions assume the same warp count as the tile kernels' consumers.
constexpr int kStreamWarps = kConsumerWarps;
constexpr int kStreamThreads = kStreamWarps * 32;

// One scale per long row: one warp per row, 8 warps per CTA.
constexpr int kRowThreads = 256;

// Strided reduction axis (axis 0: rows contiguous in memory). A stage holds a
// TMA box of 128 k x (64 bf16 | 32 fp32) rows, 16 KiB; consumers transpose it
// into a row-major buffer (row pitch 128 + 8 bf16 / 128 + 4 fp32 elements =
// 272 / 528 bytes) and process it like an axis-1 tile of width 128.
constexpr int kAxis0K = 128;
constexpr size_t kAxis0TBytes = 64 * 136 * 2; // >= 32 * 132 * 4
// (two transpose buffers, used by alternate tiles)
constexpr size_t kAxis0SmemBytes = kStages * kStageBytes + 2 * kAxis0TBytes + 4096;

// Workspace layout (bytes):
//   [0, 256)                 header: the error word at 0
//   energy tickets           kMaxGrid uint32, one per operand of a batch
//   amax tickets             kMaxGrid uint32, one per operand
//   energy partials          kMaxGrid x 4 doubles (one slot per CTA)
//   amax partials            kMaxGrid x 2 floats (one slot per CTA)
//   reduced amax             kMaxGrid x 2 floats per operand (kept values, all values)
// Tickets are left at zero by the CTA that finishes last; the header and the
// tickets (the first kWsClearBytes) must be zero before the first call.
constexpr size_t kWsErrOff = 0;
constexpr size_t kWsEnergyTicketOff = 256;
constexpr size_t kWsAmaxTicketOff = kWsEnergyTicketOff + 4 * kMaxGrid;
constexpr size_t kWsClearBytes = kWsAmaxTicketOff + 4 * kMaxGrid;
constexpr size_t kWsEnergyOff = kWsClearBytes;
constexpr size_t kWsAmaxOff = kWsEnergyOff + 32 * kMaxGrid;
constexpr size_t kWsAmaxReducedOff = kWsAmaxOff + 8 * kMaxGrid;
constexpr size_t kWsBytes = kWsAmaxReducedOff + 8 * kMaxGrid;

struct QuantSpec {
    int32_t fmt;       // Fmt (kNone .. kMxfp4)
    int32_t bits;      // INT
    int32_t group;     // INT: quantized values per scale (already resolved, > 0)
    int32_t lanes;     // lanes (chunks) per scale group
    int32_t store;     // IntStore
    float qmax;        // INT
    float qmax_inv;    // INT: RN(1 / qmax)
    float divisor;     // FP8: 448, NVFP4: 2688 (tensor scale = amax / divisor)
    const float *scale_in;     // given tensor scale (device) or nullptr
    const float *amax_reduced; // device float holding the amax when the scale is computed
    const float *row_amax_in;  // INT, one scale per row: the given amax of each row's quantized
                               // values, [batch][rows] (device), or nullptr
    float *scale_out;          // where to write the tensor scale used (device) or nullptr
};

struct PassParams {
    int64_t rows, k;           // logical operand A[rows][k] (each operand of a batch)
    int64_t n_tiles, n_col_tiles; // per operand
    int32_t R, W;              // tile rows and width (elements)
    int32_t log2_cpr;          // log2(chunks of 8 per tile row)
    int32_t cpt;               // chunks per consumer thread per tile
    int32_t axis;              // 1: k is the contiguous (TMA inner) dimension; 0: rows are
    uint32_t tile_bytes;
    // axis-1 stream kernel: the operand (elements ld apart between rows), the
    // unit grid units_a x units_b, a unit's extent (rows, columns) and the
    // step between its four slots (rows, columns)
    const void *x;
    int64_t ld;
    int32_t units_a, units_b, unit_rows, unit_cols, step_rows, step_cols;
    // outputs
    void *values;
    void *scales;
    uint8_t *meta;
    const float *norms;        // Wanda column norms
    QuantSpec q;               // the stored format (or the sparse side of kEnergy)
    QuantSpec qd;              // kEnergy: the dense side
    double *energy_partials;   // [grid][4] (workspace)
    double *energy_out;        // caller's ss24_energy records [batch] or nullptr: no energies
    float *amax_partials;      // kAmax: [grid][2] (workspace)
    float *amax_out;           // kAmax: [batch][2] (kept values, all values)
    float *amax_user;          // kAmax: caller's [batch] amax of the quantized values, or nullptr
    float *row_amax;           // kAmax: the amax of each row's quantized values, [batch][rows]
                               // (device, zero before the launch; atomic max), or nullptr
    uint32_t *energy_ticket;   // last-CTA-done counters, one per operand (workspace)
    uint32_t *amax_ticket;
    int32_t *err;              // workspace error word
    // batch of operands: CTAs [b * ctas_per_op, (b + 1) * ctas_per_op) serve
    // operand b, whose input starts x_bstride elements after operand b - 1's
    // and whose outputs start the given byte strides after operand b - 1's
    int32_t batch, ctas_per_op;
    int64_t x_bstride, values_bstride, scales_bstride, meta_bstride;
    // set per CTA by operand_view(): the operand served and the CTA's index
    // among that operand's CTAs
    int32_t op, cta;
    // rotated kernels: log2 of the Hadamard block and RN(1/sqrt(block))
    int32_t rot_log2b;
    float rot_scale;
    // the time limit of every barrier wait (ns); and a test hook: with
    // test_skip_tile = t >= 0 the first CTA of operand 0 of the strided-axis
    // kernel does not copy its t-th tile, so that its consumers' wait runs out
    uint64_t wait_limit_ns;
    int32_t test_skip_tile;
    // lane-block kernel: bit 0, a lane's 64 input bytes are read with two
    // 32-byte loads (the operand's rows 32-byte aligned); bit 1, its 32-byte
    // runs of output are written with one store (the values 32-byte aligned)
    int32_t lb_wide;
};

cudaError_t launch_ratio(const double *sparse_side, const double *dense_side, double *out, int64_t count,
                         cudaStream_t stream);
cudaError_t launch_selfcheck_division(int mode, uint32_t b_first, uint32_t b_count, unsigned long long *result,
                                      cudaStream_t stream);
cudaError_t launch_convert(int op, const void *in, void *out, int64_t n, cudaStream_t stream);
cudaError_t launch_dequant(int pattern, int fmt, int32_t store, int32_t lg, int32_t none_f32, int64_t rows,
                           int64_t k, int32_t batch, const void *values, const void *scales, const float *tscale,
                           const uint8_t *meta, float *xhat, cudaStream_t stream);
cudaError_t launch_hadamard(const void *x, int bf16, int64_t rows, int64_t k, int64_t ld, int64_t bstride,
                            int64_t batch, int32_t block, float *out, cudaStream_t stream);
// Rows of up to this many keys keep their values in shared memory.
constexpr int64_t kSoftmaxSmemKeys = 2048;
const void *softmax_prune_kernel_ptr(int bf16, int pattern, int fmt, bool smem);
int64_t scale_tiles_bytes(int64_t rows, int64_t cols);
cudaError_t launch_scale_tiles(const uint8_t *in, int64_t rows, int64_t cols, int64_t batch, uint8_t *out,
                               cudaStream_t stream);
cudaError_t launch_selfcheck_encoder(int e2m1, const uint32_t *bounds, int n_bounds, uint32_t hi_first,
                                     uint32_t hi_count, unsigned long long *result, cudaStream_t stream);
size_t sparse_gemm_smem_bytes();
cudaError_t launch_sparse_gemm_fp8(const uint8_t *a_values, const uint8_t *a_meta, const float *a_scale,
                                   const uint8_t *b, const float *b_scale, int64_t m, int64_t n, int64_t k, float *y,
                                   int32_t *err, uint64_t wait_limit_ns, cudaStream_t stream);

} // namespace ss24
