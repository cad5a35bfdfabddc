// The C ABI (include/ss24.h): host-side validation, tile geometry, TMA tensor
// maps and launches. Every check runs before anything is enqueued; a failed
// check returns its status and launches nothing.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "../../include/ss24.h"
#include "internal.cuh"

namespace ss24 {
const void *stream_kernel_bf16(int pattern, int score, int fmt, bool fw);
const void *stream_kernel_f32(int pattern, int score, int fmt, bool fw);
const void *stream_kernel_bf16_rot(int pattern, int fmt, bool fw);
const void *stream_lb_kernel_bf16(int pattern, int score, int fmt);
const void *stream_lb_energy_kernel_bf16(int sparse_fmt, int dense_fmt);
const void *stream_lb_kernel_bf16_rot(int pattern, int fmt);
const void *stream_lb_amax_kernel_bf16_rot(int pattern);
const void *stream_lb_energy_kernel_bf16_rot(int sparse_fmt, int dense_fmt);
const void *rowsweep_kernel_bf16(int pattern, int score);
const void *rowsweep_kernel_f32(int pattern, int score);
const void *rowblock_kernel_bf16(int pattern, int score, int cpt);
const void *rowblock_kernel_f32(int pattern, int score, int cpt);
const void *axis0_kernel_bf16(int pattern, int score, int fmt);
const void *axis0_kernel_f32(int pattern, int score, int fmt);
} // namespace ss24

using namespace ss24;

namespace {

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned32(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }
bool pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }
int64_t next_pow2(int64_t v)
{
    int64_t p = 1;
    while (p < v)
        p <<= 1;
    return p;
}
int ilog2(int64_t v)
{
    int l = 0;
    while ((int64_t(1) << l) < v)
        ++l;
    return l;
}
size_t esize(int dtype) { return dtype == SS24_BF16 ? 2 : 4; }

ss24_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SS24_OK : SS24_ERR_CUDA; }

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// Operands in a batch (batch 0 reads as 1) and the element stride between them.
int64_t nbatch(const ss24_operand *x) { return x->batch > 1 ? x->batch : 1; }
int64_t bstride_elems(const ss24_operand *x)
{
    if (x->batch > 1)
        return x->batch_stride;
    return (x->axis == 1 ? x->rows : x->k) * x->ld; // unused: one operand
}

// 3-D map over the operands' memory: {contiguous dimension, the other one,
// operand of the batch}.
bool make_map(CUtensorMap *map, const ss24_operand *x, int64_t inner, int64_t outer, uint32_t box_inner,
              uint32_t box_outer)
{
    auto fn = encode_fn();
    if (!fn)
        return false;
    const CUtensorMapDataType dt =
        x->dtype == SS24_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    const cuuint64_t es = esize(x->dtype);
    int64_t bs = bstride_elems(x);
    if (bs < 1)
        bs = x->ld; // an empty single operand never gets here; keep the stride valid
    cuuint64_t gdim[3] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer),
                          static_cast<cuuint64_t>(nbatch(x))};
    cuuint64_t gstride[2] = {static_cast<cuuint64_t>(x->ld) * es, static_cast<cuuint64_t>(bs) * es};
    cuuint32_t box[3] = {box_inner, box_outer, 1};
    cuuint32_t estride[3] = {1, 1, 1};
    const CUresult r = fn(map, dt, 3, const_cast<void *>(x->x), gdim, gstride, box, estride,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool current_ctx_id(unsigned long long *id);

// Kernel attributes (dynamic shared memory) and occupancy, once per kernel and
// context (a context created after a device reset starts without the
// attributes).
struct KernelInfo {
    int blocks_per_sm = 0;
    unsigned long long ctx_id = 0;
};

std::mutex g_mu;
std::unordered_map<const void *, KernelInfo> g_info;
int g_sms = 0;

cudaError_t kernel_info(const void *k, size_t smem, KernelInfo *out, int threads = kThreads)
{
    unsigned long long id = 0;
    const bool have_id = current_ctx_id(&id);
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = g_info.find(k);
    if (it != g_info.end() && have_id && it->second.ctx_id == id) {
        *out = it->second;
        return cudaSuccess;
    }
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess)
        return e;
    KernelInfo info;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&info.blocks_per_sm, k, threads, smem);
    if (e != cudaSuccess)
        return e;
    if (g_sms == 0) {
        int dev = 0;
        e = cudaGetDevice(&dev);
        if (e == cudaSuccess)
            e = cudaDeviceGetAttribute(&g_sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess)
            return e;
    }
    info.ctx_id = current_ctx_id(&id) ? id : 0;
    g_info[k] = info;
    *out = info;
    return cudaSuccess;
}

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel on the stream finishes; it waits for it
// (griddepcontrol.wait) before touching global memory.
cudaError_t launch_pdl(const void *k, unsigned grid, unsigned threads, size_t smem, cudaStream_t stream, void **args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, k, args);
}

// CTAs per operand: the persistent grid (SMs x resident CTAs, at most
// kMaxGrid) shared among the operands of the batch, at most one CTA per unit
// of work of an operand.
int64_t ctas_per_operand(const KernelInfo &info, int64_t batch, int64_t units)
{
    int64_t total = static_cast<int64_t>(g_sms) * (info.blocks_per_sm > 0 ? info.blocks_per_sm : 1);
    if (total > kMaxGrid)
        total = kMaxGrid;
    int64_t per = total / batch;
    if (per > units)
        per = units;
    return per < 1 ? 1 : per;
}

cudaError_t launch(const void *k, size_t smem, int64_t n_tiles, const CUtensorMap &map, const PassParams &p,
                   cudaStream_t stream)
{
    KernelInfo info;
    if (p.axis == 1) {
        // the stream kernel: no tensor map, no dynamic shared memory
        cudaError_t e = kernel_info(k, 0, &info, kStreamThreads);
        if (e != cudaSuccess)
            return e;
        PassParams pp = p;
        pp.ctas_per_op = static_cast<int32_t>(ctas_per_operand(info, p.batch, n_tiles));
        void *args[1] = {&pp};
        return launch_pdl(k, static_cast<unsigned>(p.batch * pp.ctas_per_op), kStreamThreads, 0, stream, args);
    }
    cudaError_t e = kernel_info(k, smem, &info);
    if (e != cudaSuccess)
        return e;
    PassParams pp = p;
    pp.ctas_per_op = static_cast<int32_t>(ctas_per_operand(info, p.batch, n_tiles));
    CUtensorMap m = map;
    void *args[2] = {&m, &pp};
    return launch_pdl(k, static_cast<unsigned>(p.batch * pp.ctas_per_op), kThreads, smem, stream, args);
}

// The one-scale-per-row kernel: no tensor map; one warp per row, 8 rows per CTA.
cudaError_t launch_rowsweep(const void *k, const ss24_operand *x, const PassParams &p, cudaStream_t stream)
{
    KernelInfo info;
    cudaError_t e = kernel_info(k, 0, &info, kRowThreads);
    if (e != cudaSuccess)
        return e;
    const int64_t rows_per_cta = kRowThreads / 32;
    PassParams pp = p;
    pp.ctas_per_op = static_cast<int32_t>(ctas_per_operand(info, p.batch, (x->rows + rows_per_cta - 1) / rows_per_cta));
    const void *xp = x->x;
    int64_t ld = x->ld;
    void *args[3] = {&xp, &ld, &pp};
    return launch_pdl(k, static_cast<unsigned>(p.batch * pp.ctas_per_op), kRowThreads, 0, stream, args);
}

// One scale per row with the row in registers: cpt chunks per thread, tpr
// threads per row (a power of two in [32, 256]), 256 / tpr rows per CTA step.
// Rows longer than 2048 chunks (k > 16384) take the two-sweep kernel instead.
bool rowblock_plan(int64_t k, int *cpt, int *log2_tpr)
{
    const int64_t nchunks = k / 8;
    int c;
    if (nchunks <= 32)
        c = 1;
    else if (nchunks <= 1024)
        c = 4;
    else if (nchunks <= 2048)
        c = 8;
    else
        return false;
    int64_t tpr = 32;
    while (tpr * c < nchunks)
        tpr *= 2;
    *cpt = c;
    *log2_tpr = ilog2(tpr);
    return true;
}

cudaError_t launch_rowblock(const void *k, const ss24_operand *x, int log2_tpr, const PassParams &p,
                            cudaStream_t stream)
{
    KernelInfo info;
    cudaError_t e = kernel_info(k, 0, &info, kRowThreads);
    if (e != cudaSuccess)
        return e;
    const int64_t rows_per_cta = kRowThreads >> log2_tpr;
    PassParams pp = p;
    pp.ctas_per_op = static_cast<int32_t>(ctas_per_operand(info, p.batch, (x->rows + rows_per_cta - 1) / rows_per_cta));
    const void *xp = x->x;
    int64_t ld = x->ld;
    int32_t lt = log2_tpr;
    void *args[4] = {&xp, &ld, &lt, &pp};
    return launch_pdl(k, static_cast<unsigned>(p.batch * pp.ctas_per_op), kRowThreads, 0, stream, args);
}

// ---------------------------------------------------------------------------
// validation
// ---------------------------------------------------------------------------

// An empty operand (rows == 0) may have a NULL data pointer.
ss24_status check_operand(const ss24_operand *x)
{
    if (!x || (!x->x && x->rows != 0))
        return SS24_ERR_NULL;
    if (x->dtype != SS24_BF16 && x->dtype != SS24_F32)
        return SS24_ERR_DTYPE;
    if (x->axis != 0 && x->axis != 1)
        return SS24_ERR_ARG;
    if (x->rows < 0 || x->k <= 0 || x->rows > INT32_MAX || x->k > INT32_MAX)
        return SS24_ERR_SHAPE;
    if (x->ld < (x->axis == 1 ? x->k : x->rows))
        return SS24_ERR_SHAPE;
    if (!aligned16(x->x) || (x->ld * static_cast<int64_t>(esize(x->dtype))) % 16 != 0)
        return SS24_ERR_ALIGN;
    if (x->batch < 0 || x->batch > kMaxGrid)
        return SS24_ERR_SHAPE;
    if (x->hadamard != 0) {
        // the rotated pass: bf16 along k, a power-of-two block of 2..256 dividing k
        const int32_t b = x->hadamard;
        if (b < 2 || b > 256 || (b & (b - 1)) != 0 || x->axis != 1 || x->dtype != SS24_BF16)
            return SS24_ERR_ARG;
        if (x->k % b != 0)
            return SS24_ERR_SHAPE;
    }
    if (x->batch > 1) {
        // operands must not overlap
        if (x->batch_stride < (x->axis == 1 ? x->rows : x->k) * x->ld)
            return SS24_ERR_SHAPE;
        if ((x->batch_stride * static_cast<int64_t>(esize(x->dtype))) % 16 != 0)
            return SS24_ERR_ALIGN;
    }
    return SS24_OK;
}

ss24_status check_ws(const void *ws, size_t ws_bytes)
{
    if (!ws || ws_bytes < kWsBytes || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return SS24_ERR_WORKSPACE;
    return SS24_OK;
}

ss24_status check_pattern_k(int pattern, int64_t k)
{
    if (pattern != SS24_DENSE && pattern != SS24_SPARSE_24 && pattern != SS24_SPARSE_48)
        return SS24_ERR_ARG;
    if (k % (pattern == SS24_SPARSE_48 ? 16 : 8) != 0)
        return SS24_ERR_SHAPE;
    return SS24_OK;
}

// Resolved quantization of the values a pass stores (n per row).
struct Resolved {
    QuantSpec q;
    bool row_mode = false;
};

// Validates `fmt` for rows of n quantized values (n = k/2 sparse, k dense) and
// fills the kernel's QuantSpec (without the scale pointers).
ss24_status resolve_format(ss24_format fmt, int pattern, int64_t k, bool allow_none, Resolved *r)
{
    const bool sparse = pattern != SS24_DENSE;
    const int64_t n = sparse ? k / 2 : k;
    const int vpc = sparse ? 4 : 8;
    QuantSpec q{};
    q.fmt = fmt.kind;
    switch (fmt.kind) {
    case SS24_FMT_NONE:
        if (!allow_none || !sparse)
            return SS24_ERR_FORMAT;
        break;
    case SS24_FMT_FP8_E4M3:
        q.divisor = 448.0f;
        break;
    case SS24_FMT_NVFP4:
        if (n % 16 != 0)
            return SS24_ERR_SHAPE;
        q.divisor = 2688.0f;
        break;
    case SS24_FMT_MXFP4:
        if (n % 32 != 0)
            return SS24_ERR_SHAPE;
        break;
    case SS24_FMT_INT: {
        if (fmt.bits < 2 || fmt.bits > 16)
            return SS24_ERR_FORMAT;
        if (fmt.pack4 && fmt.bits > 4)
            return SS24_ERR_FORMAT;
        q.bits = fmt.bits;
        q.qmax = static_cast<float>((1 << (fmt.bits - 1)) - 1);
        q.qmax_inv = 1.0f / q.qmax; // IEEE binary32 division: RN(1 / qmax)
        q.store = fmt.pack4 ? kPack4 : (fmt.bits > 8 ? kInt16 : kInt8);
        if (fmt.group < 0)
            return SS24_ERR_FORMAT;
        if (fmt.group == 0) {
            q.group = static_cast<int32_t>(n);
            // a whole row fits one warp's span only when k is a power of two <= 256
            r->row_mode = !(pow2(k) && k <= 256);
            q.lanes = r->row_mode ? 32 : static_cast<int32_t>(n / vpc);
        } else {
            const int64_t g_in = static_cast<int64_t>(fmt.group) * (sparse ? 2 : 1);
            if (!pow2(fmt.group) || g_in < 8 || g_in > 256)
                return SS24_ERR_FORMAT;
            if (n % fmt.group != 0)
                return SS24_ERR_SHAPE;
            q.group = fmt.group;
            q.lanes = fmt.group / vpc;
        }
        break;
    }
    default:
        return SS24_ERR_FORMAT;
    }
    r->q = q;
    return SS24_OK;
}

bool per_tensor(int kind) { return kind == SS24_FMT_FP8_E4M3 || kind == SS24_FMT_NVFP4; }

// ---------------------------------------------------------------------------
// geometry
// ---------------------------------------------------------------------------

struct Geometry {
    int32_t R, W, log2_cpr, cpt;
    int64_t n_tiles, n_col_tiles; // axis 1: n_tiles = work items of 8 units (one per warp of a CTA)
    uint32_t tile_bytes;
    int32_t units_a, units_b, unit_rows, unit_cols, step_rows, step_cols;
};

// Axis 1 (stream kernel). A slot is a row segment of W = min(256,
// next_pow2(k)) columns for 256 / W rows (one 16-byte chunk per lane); a unit
// is four slots. Four consecutive segments of the same rows when a row has at
// least 4 segments and a ragged last quad wastes little (nseg a multiple of 4
// or at least 16); otherwise the same segment of four consecutive row groups.
Geometry stream_geometry(const ss24_operand *x)
{
    Geometry g{};
    g.W = static_cast<int32_t>(x->k >= 256 ? 256 : next_pow2(x->k));
    g.log2_cpr = ilog2(g.W / 8);
    const int64_t rps = 256 / g.W;
    const int64_t nseg = (x->k + g.W - 1) / g.W;
    const int64_t n_rg = (x->rows + rps - 1) / rps;
    int64_t ua, ub;
    if (nseg >= 4 && (nseg % 4 == 0 || nseg >= 16)) {
        g.unit_rows = static_cast<int32_t>(rps);
        g.unit_cols = 4 * g.W;
        g.step_rows = 0;
        g.step_cols = g.W;
        ua = n_rg;
        ub = (nseg + 3) / 4;
    } else {
        g.unit_rows = static_cast<int32_t>(4 * rps);
        g.unit_cols = g.W;
        g.step_rows = static_cast<int32_t>(rps);
        g.step_cols = 0;
        ua = (n_rg + 3) / 4;
        ub = nseg;
    }
    g.units_a = static_cast<int32_t>(ua);
    g.units_b = static_cast<int32_t>(ub);
    g.n_tiles = (ua * ub + kStreamWarps - 1) / kStreamWarps;
    return g;
}

// Axis 0: a tile is 128 k x (64 bf16 | 32 fp32) rows, transposed in shared memory.
Geometry axis0_geometry(const ss24_operand *x)
{
    Geometry g{};
    const int64_t R = x->dtype == SS24_BF16 ? 64 : 32;
    g.W = kAxis0K;
    g.R = static_cast<int32_t>(R);
    g.log2_cpr = ilog2(kAxis0K / 8);
    g.cpt = static_cast<int32_t>((R * kAxis0K / 8) / kConsumers);
    g.n_col_tiles = (x->k + kAxis0K - 1) / kAxis0K;
    g.n_tiles = g.n_col_tiles * ((x->rows + R - 1) / R);
    g.tile_bytes = static_cast<uint32_t>(kStageBytes);
    return g;
}

// The largest quantization group, in input elements, an axis-0 tile holds.
bool axis0_format_ok(const ss24_format &fmt, int pattern, int64_t k)
{
    const bool sparse = pattern != SS24_DENSE;
    if (fmt.kind == SS24_FMT_MXFP4 && sparse)
        return true; // 64 input elements
    if (fmt.kind != SS24_FMT_INT)
        return true;
    if (fmt.group == 0)
        return pow2(k) && k <= kAxis0K;
    return static_cast<int64_t>(fmt.group) * (sparse ? 2 : 1) <= kAxis0K;
}

PassParams base_params(const ss24_operand *x, const Geometry &g, void *ws, ss24_energy *energy)
{
    PassParams p{};
    p.rows = x->rows;
    p.k = x->k;
    p.n_tiles = g.n_tiles;
    p.n_col_tiles = g.n_col_tiles;
    p.R = g.R;
    p.W = g.W;
    p.log2_cpr = g.log2_cpr;
    p.cpt = g.cpt;
    p.axis = x->axis;
    p.tile_bytes = g.tile_bytes;
    p.x = x->x;
    p.ld = x->ld;
    p.units_a = g.units_a;
    p.units_b = g.units_b;
    p.unit_rows = g.unit_rows;
    p.unit_cols = g.unit_cols;
    p.step_rows = g.step_rows;
    p.step_cols = g.step_cols;
    uint8_t *w = static_cast<uint8_t *>(ws);
    p.err = reinterpret_cast<int32_t *>(w + kWsErrOff);
    p.energy_ticket = reinterpret_cast<uint32_t *>(w + kWsEnergyTicketOff);
    p.amax_ticket = reinterpret_cast<uint32_t *>(w + kWsAmaxTicketOff);
    p.energy_partials = reinterpret_cast<double *>(w + kWsEnergyOff);
    p.amax_partials = reinterpret_cast<float *>(w + kWsAmaxOff);
    p.amax_out = reinterpret_cast<float *>(w + kWsAmaxReducedOff);
    p.energy_out = reinterpret_cast<double *>(energy);
    p.wait_limit_ns = kWaitLimitNs;
    p.test_skip_tile = -1;
    if (const char *t = std::getenv("SS24_TEST_SKIP_TILE")) {
        // test hook (ss24.h): one tile copy skipped, waits limited to 10 ms
        const long v = std::strtol(t, nullptr, 10);
        if (v >= 0 && v < INT32_MAX) {
            p.test_skip_tile = static_cast<int32_t>(v);
            p.wait_limit_ns = kTestWaitLimitNs;
        }
    }
    p.batch = static_cast<int32_t>(nbatch(x));
    p.x_bstride = bstride_elems(x);
    if (x->hadamard != 0) {
        int l = 0;
        while ((1 << l) < x->hadamard)
            ++l;
        p.rot_log2b = l;
        p.rot_scale = static_cast<float>(1.0 / std::sqrt(static_cast<double>(x->hadamard)));
    }
    return p;
}

// Per-operand byte strides of the outputs of a pass storing `fmt` (outputs of
// a batch are packed one operand after the other).
void output_strides(const ss24_operand *x, int pattern, ss24_format fmt, PassParams *p)
{
    const bool sparse = pattern != SS24_DENSE;
    const int64_t n = sparse ? x->k / 2 : x->k, rows = x->rows;
    switch (fmt.kind) {
    case SS24_FMT_NONE:
        p->values_bstride = rows * n * static_cast<int64_t>(esize(x->dtype));
        break;
    case SS24_FMT_FP8_E4M3:
        p->values_bstride = rows * n;
        break;
    case SS24_FMT_INT:
        p->values_bstride = fmt.pack4 ? rows * n / 2 : rows * n * (fmt.bits > 8 ? 2 : 1);
        p->scales_bstride = rows * (fmt.group ? n / fmt.group : 1) * 4;
        break;
    case SS24_FMT_NVFP4:
        p->values_bstride = rows * n / 2;
        p->scales_bstride = rows * n / 16;
        break;
    case SS24_FMT_MXFP4:
        p->values_bstride = rows * n / 2;
        p->scales_bstride = rows * n / 32;
        break;
    }
    if (sparse)
        p->meta_bstride = rows * x->k / (pattern == SS24_SPARSE_48 ? 16 : 8);
}

const void *stream_kernel(int dtype, int pattern, int score, int fmt, bool fw)
{
    return dtype == SS24_BF16 ? stream_kernel_bf16(pattern, score, fmt, fw)
                              : stream_kernel_f32(pattern, score, fmt, fw);
}

// Tile geometry, tensor map and kernel for a tile-mode pass along either axis.
struct TilePlan {
    Geometry g;
    CUtensorMap map;
    const void *kernel;
    size_t smem;
};

bool plan_tile(const ss24_operand *x, int pattern, int score, int mode, TilePlan *t)
{
    if (x->axis == 1) {
        t->g = stream_geometry(x);
        // full width: W = 256 with four segments per unit
        const bool fw = t->g.W == 256 && t->g.step_cols == 256;
        if (x->hadamard != 0) {
            t->kernel = nullptr;
            if (score == SS24_SCORE_MAG) {
                if (fw && x->k % 64 == 0)
                    t->kernel = stream_lb_kernel_bf16_rot(pattern, mode);
                if (!t->kernel)
                    t->kernel = stream_kernel_bf16_rot(pattern, mode, fw);
            }
        } else {
            // bf16 with rows a multiple of 64: one lane per 32 consecutive
            // elements (where that kernel has the format)
            t->kernel = nullptr;
            if (fw && x->dtype == SS24_BF16 && x->k % 64 == 0)
                t->kernel = stream_lb_kernel_bf16(pattern, score, mode);
            if (!t->kernel)
                t->kernel = stream_kernel(x->dtype, pattern, score, mode, fw);
        }
        t->smem = 0;
        return t->kernel != nullptr;
    }
    t->g = axis0_geometry(x);
    t->kernel = x->dtype == SS24_BF16 ? axis0_kernel_bf16(pattern, score, mode) : axis0_kernel_f32(pattern, score, mode);
    t->smem = kAxis0SmemBytes;
    return make_map(&t->map, x, x->rows, x->k, static_cast<uint32_t>(t->g.R), static_cast<uint32_t>(t->g.W));
}

// The read-only amax pass; leaves {amax of kept, amax of all} in the workspace.
// For 2:4 by magnitude the kept amax equals the amax of all values (a group's
// largest value is always kept), so the cheaper dense form is used; pairwise
// 4:8 can drop the largest value (its pair may rank third) and takes its own.
cudaError_t run_amax(const ss24_operand *x, int pattern, int score, const float *norms, void *ws,
                     cudaStream_t stream, float *scale_out = nullptr, float divisor = 1.0f,
                     float *amax_user = nullptr, float *row_amax = nullptr)
{
    const int pat = score == SS24_SCORE_MAG && pattern != SS24_SPARSE_48 ? SS24_DENSE : pattern;
    TilePlan t;
    if (!plan_tile(x, pat, score, kAmax, &t))
        return cudaErrorInvalidValue;
    // over the rotated operand on bf16 full-width rows (k a multiple of 64),
    // without per-row output: the lane-block amax kernel
    if (x->axis == 1 && x->hadamard != 0 && score == SS24_SCORE_MAG && !row_amax && t.g.W == 256 &&
        t.g.step_cols == 256 && x->k % 64 == 0) {
        if (const void *kl = stream_lb_amax_kernel_bf16_rot(pat)) {
            t.kernel = kl;
            t.smem = 0;
        }
    }
    PassParams p = base_params(x, t.g, ws, nullptr);
    p.norms = norms;
    p.q.scale_out = scale_out;
    p.q.divisor = divisor;
    p.amax_user = amax_user;
    p.row_amax = row_amax;
    return launch(t.kernel, t.smem, t.g.n_tiles, t.map, p, stream);
}

// Zero energy records / scales for empty operands (nothing to launch).
ss24_status empty_operand(const ss24_operand *x, ss24_energy *energy, const ss24_outputs *out, const float *scale_in,
                          cudaStream_t stream)
{
    const size_t nb = static_cast<size_t>(nbatch(x));
    cudaError_t e = cudaSuccess;
    if (energy)
        e = cudaMemsetAsync(energy, 0, nb * sizeof(ss24_energy), stream);
    if (e == cudaSuccess && out && out->tensor_scale) {
        if (scale_in)
            e = cudaMemcpyAsync(out->tensor_scale, scale_in, nb * sizeof(float), cudaMemcpyDeviceToDevice, stream);
        else
            e = cudaMemsetAsync(out->tensor_scale, 0, nb * sizeof(float), stream);
    }
    return cuda_status(e);
}

// The storing pass shared by the quantize / prune entry points.
// With launch false it only validates: it returns the status the call would
// return before enqueueing anything, and enqueues nothing.
ss24_status run_pass(const ss24_operand *x, int pattern, int score, const float *norms, ss24_format fmt,
                     bool allow_none, const float *scale_in, const ss24_outputs *out, ss24_energy *energy,
                     void *ws, size_t ws_bytes, cudaStream_t stream, const float *row_amax_in = nullptr,
                     bool launch_it = true)
{
    ss24_status st = check_operand(x);
    if (st != SS24_OK)
        return st;
    if ((st = check_pattern_k(pattern, x->k)) != SS24_OK)
        return st;
    if (score != SS24_SCORE_MAG && score != SS24_SCORE_WANDA)
        return SS24_ERR_ARG;
    if (x->hadamard != 0 && score != SS24_SCORE_MAG)
        return SS24_ERR_ARG; // a rotated pass selects by magnitude
    if (score == SS24_SCORE_WANDA && pattern != SS24_DENSE && (!norms || !aligned16(norms)))
        return norms ? SS24_ERR_ALIGN : SS24_ERR_NULL;
    if ((st = check_ws(ws, ws_bytes)) != SS24_OK)
        return st;
    Resolved r;
    if ((st = resolve_format(fmt, pattern, x->k, allow_none, &r)) != SS24_OK)
        return st;
    if (!out)
        return SS24_ERR_NULL;
    if (x->axis == 0 && !axis0_format_ok(fmt, pattern, x->k))
        return SS24_ERR_FORMAT; // a group longer than the 128-element axis-0 tile
    Geometry g;
    if (x->axis == 0) {
        r.row_mode = false;
        g = axis0_geometry(x);
    } else {
        g = stream_geometry(x); // (row mode uses only rows / k of it)
    }
    if (x->rows == 0)
        return launch_it ? empty_operand(x, energy, out, per_tensor(fmt.kind) ? scale_in : nullptr, stream)
                         : SS24_OK;
    if (!out->values)
        return SS24_ERR_NULL;
    if (!aligned16(out->values))
        return SS24_ERR_ALIGN;
    const bool needs_scales = fmt.kind == SS24_FMT_INT || fmt.kind == SS24_FMT_NVFP4 || fmt.kind == SS24_FMT_MXFP4;
    if (needs_scales && !out->scales)
        return SS24_ERR_NULL;
    if (needs_scales && !aligned16(out->scales))
        return SS24_ERR_ALIGN;
    if (per_tensor(fmt.kind) && !out->tensor_scale)
        return SS24_ERR_NULL;
    if (pattern != SS24_DENSE && (!out->meta))
        return SS24_ERR_NULL;
    if (pattern != SS24_DENSE && !aligned16(out->meta))
        return SS24_ERR_ALIGN;
    if (r.row_mode && x->hadamard != 0 && !row_amax_in)
        return SS24_ERR_ARG; // one INT scale per row over a rotated operand: amax_rows + quantize_int_rows
    if (!launch_it)
        return SS24_OK;

    // ---- launches ----
    PassParams p = base_params(x, g, ws, energy);
    output_strides(x, pattern, fmt, &p);
    {
        // lane-block kernel: 32-byte loads measured faster for pairwise 4:8
        // only; 32-byte stores wherever the values are aligned for them
        const int64_t es = static_cast<int64_t>(esize(x->dtype));
        const bool in32 = aligned32(x->x) && (x->ld * es) % 32 == 0 &&
                          (nbatch(x) == 1 || (x->batch_stride * es) % 32 == 0);
        const bool out32 = aligned32(out->values) && p.values_bstride % 32 == 0;
        p.lb_wide = (in32 && pattern == SS24_SPARSE_48 ? 1 : 0) | (out32 ? 2 : 0);
    }
    p.values = out->values;
    p.scales = out->scales;
    p.meta = out->meta;
    p.norms = norms;
    p.q = r.q;
    p.q.row_amax_in = row_amax_in;
    if (row_amax_in)
        r.row_mode = false; // the stream kernel, with the rows' scales from the given amax
    if (per_tensor(fmt.kind)) {
        p.q.scale_out = out->tensor_scale;
        p.q.scale_in = scale_in;
        if (!scale_in) {
            cudaError_t e = run_amax(x, pattern, score, norms, ws, stream);
            if (e != cudaSuccess)
                return SS24_ERR_CUDA;
            p.q.amax_reduced = p.amax_out; // [0] = amax of the quantized values
        }
    }
    cudaError_t e;
    int cpt = 0, log2_tpr = 0;
    if (r.row_mode && rowblock_plan(x->k, &cpt, &log2_tpr)) {
        const void *k = x->dtype == SS24_BF16 ? rowblock_kernel_bf16(pattern, score, cpt)
                                              : rowblock_kernel_f32(pattern, score, cpt);
        e = launch_rowblock(k, x, log2_tpr, p, stream);
    } else if (r.row_mode) {
        const void *k = x->dtype == SS24_BF16 ? rowsweep_kernel_bf16(pattern, score) : rowsweep_kernel_f32(pattern, score);
        e = launch_rowsweep(k, x, p, stream);
    } else {
        TilePlan t;
        if (!plan_tile(x, pattern, score, row_amax_in ? static_cast<int>(kIntRows) : fmt.kind, &t))
            return SS24_ERR_CUDA;
        e = launch(t.kernel, t.smem, t.g.n_tiles, t.map, p, stream);
    }
    return cuda_status(e);
}

// ---------------------------------------------------------------------------
// Library-owned scratch for callers that cannot allocate device memory
// ---------------------------------------------------------------------------

// The fused pass keeps a few partial sums per CTA (and an error word and two
// ticket counters) between its CTAs. For callers that cannot call cudaMalloc,
// that scratch lives in this file-scope device array: one copy per GPU that
// loads the library, held until the process exits. The pass needs the same
// fixed amount whatever the operand size (partials for at most kMaxGrid CTAs).
constexpr size_t kStaticScratchBytes = kWsBytes;
static_assert(kStaticScratchBytes >= kWsBytes, "the array must hold the pass's whole workspace");
static __device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_static_mu;
struct StaticScratch {
    unsigned long long ctx_id = 0; // context the address belongs to (0: none yet)
    void *ptr = nullptr;
};
StaticScratch g_static[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Process-unique ID of the current context (cuCtxGetId), through the driver
// entry points the runtime exposes; false if it cannot be read.
bool current_ctx_id(unsigned long long *id)
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx)
        return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the array in the current device's context. Host code must
// not use the symbol's host-side name as a pointer; the address comes from
// cudaGetSymbolAddress, taken with the device current, once per device and
// context: a context created after a device reset loads the module again, so
// the address is looked up again when the context's ID changes.
cudaError_t static_scratch(void **ptr)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    // (no current context yet, e.g. on a fresh thread: the lookup below makes
    // the device's primary context current, and the ID is read after it)
    unsigned long long id = 0;
    const bool have_id = current_ctx_id(&id);
    std::lock_guard<std::mutex> lock(g_static_mu);
    StaticScratch &s = g_static[dev];
    if (!s.ptr || !have_id || s.ctx_id != id) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess)
            return e;
        s.ptr = p;
        s.ctx_id = current_ctx_id(&id) ? id : 0;
    }
    *ptr = s.ptr;
    return cudaSuccess;
}

} // namespace

// ===========================================================================
// C ABI
// ===========================================================================

extern "C" {

size_t ss24_workspace_bytes(void) { return kWsBytes; }

ss24_status ss24_workspace_init(void *ws, size_t ws_bytes, ss24_stream stream)
{
    ss24_status st = check_ws(ws, ws_bytes);
    if (st != SS24_OK)
        return st;
    return cuda_status(cudaMemsetAsync(ws, 0, kWsClearBytes, reinterpret_cast<cudaStream_t>(stream)));
}

ss24_status ss24_workspace_error(const void *ws, int32_t *code, ss24_stream stream)
{
    if (!ws || !code)
        return SS24_ERR_NULL;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e == cudaSuccess)
        e = cudaMemcpy(code, ws, sizeof(int32_t), cudaMemcpyDeviceToHost);
    return cuda_status(e);
}

ss24_status ss24_prune24_compress(const ss24_operand *x, ss24_score score, const float *col_norms, void *kept,
                                  uint8_t *meta, ss24_energy *energy, void *ws, size_t ws_bytes,
                                  ss24_stream stream)
{
    ss24_outputs out{kept, nullptr, nullptr, meta};
    ss24_format none{SS24_FMT_NONE, 0, 0, 0};
    return run_pass(x, SS24_SPARSE_24, score, col_norms, none, true, nullptr, &out, energy, ws, ws_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
}

ss24_status ss24_quantize_fp8(const ss24_operand *x, const float *tensor_scale_in, ss24_outputs *out,
                              ss24_energy *energy, void *ws, size_t ws_bytes, ss24_stream stream)
{
    ss24_format f{SS24_FMT_FP8_E4M3, 8, 0, 0};
    return run_pass(x, SS24_DENSE, SS24_SCORE_MAG, nullptr, f, false, tensor_scale_in, out, energy, ws, ws_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
}

ss24_status ss24_quantize_int(const ss24_operand *x, ss24_format fmt, ss24_outputs *out, ss24_energy *energy,
                              void *ws, size_t ws_bytes, ss24_stream stream)
{
    if (fmt.kind != SS24_FMT_INT)
        return SS24_ERR_FORMAT;
    return run_pass(x, SS24_DENSE, SS24_SCORE_MAG, nullptr, fmt, false, nullptr, out, energy, ws, ws_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
}

ss24_status ss24_quantize_nvfp4(const ss24_operand *x, const float *tensor_scale_in, ss24_outputs *out,
                                ss24_energy *energy, void *ws, size_t ws_bytes, ss24_stream stream)
{
    ss24_format f{SS24_FMT_NVFP4, 4, 0, 0};
    return run_pass(x, SS24_DENSE, SS24_SCORE_MAG, nullptr, f, false, tensor_scale_in, out, energy, ws, ws_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
}

ss24_status ss24_quantize_mxfp4(const ss24_operand *x, ss24_outputs *out, ss24_energy *energy, void *ws,
                                size_t ws_bytes, ss24_stream stream)
{
    ss24_format f{SS24_FMT_MXFP4, 4, 0, 0};
    return run_pass(x, SS24_DENSE, SS24_SCORE_MAG, nullptr, f, false, nullptr, out, energy, ws, ws_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
}

ss24_status ss24_prune24_quant_fused(const ss24_operand *x, ss24_score score, const float *col_norms,
                                     ss24_format fmt, const float *tensor_scale_in, ss24_outputs *out,
                                     ss24_energy *energy, void *ws, size_t ws_bytes, ss24_stream stream)
{
    return run_pass(x, SS24_SPARSE_24, score, col_norms, fmt, true, tensor_scale_in, out, energy, ws, ws_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
}

ss24_status ss24_prune48_pairwise_quant_fused(const ss24_operand *x, ss24_score score, const float *col_norms,
                                              ss24_format fmt, const float *tensor_scale_in, ss24_outputs *out,
                                              ss24_energy *energy, void *ws, size_t ws_bytes, ss24_stream stream)
{
    return run_pass(x, SS24_SPARSE_48, score, col_norms, fmt, true, tensor_scale_in, out, energy, ws, ws_bytes,
                    reinterpret_cast<cudaStream_t>(stream));
}

ss24_status ss24_error_energy(const ss24_operand *x, ss24_pattern pattern, ss24_score score, const float *col_norms,
                              ss24_format sparse_fmt, ss24_format dense_fmt, const float *sparse_scale_in,
                              const float *dense_scale_in, ss24_energy *energy, void *ws, size_t ws_bytes,
                              ss24_stream stream)
{
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    ss24_status st = check_operand(x);
    if (st != SS24_OK)
        return st;
    if (pattern == SS24_DENSE)
        return SS24_ERR_ARG;
    if ((st = check_pattern_k(pattern, x->k)) != SS24_OK)
        return st;
    if (score != SS24_SCORE_MAG && score != SS24_SCORE_WANDA)
        return SS24_ERR_ARG;
    if (x->hadamard != 0 && score != SS24_SCORE_MAG)
        return SS24_ERR_ARG; // a rotated pass selects by magnitude
    if (score == SS24_SCORE_WANDA && (!col_norms || !aligned16(col_norms)))
        return col_norms ? SS24_ERR_ALIGN : SS24_ERR_NULL;
    if ((st = check_ws(ws, ws_bytes)) != SS24_OK)
        return st;
    if (!energy)
        return SS24_ERR_NULL;
    Resolved rs, rd;
    if ((st = resolve_format(sparse_fmt, pattern, x->k, true, &rs)) != SS24_OK)
        return st;
    if ((st = resolve_format(dense_fmt, SS24_DENSE, x->k, false, &rd)) != SS24_OK)
        return st;
    if (x->axis == 1 && (rs.row_mode || rd.row_mode))
        return SS24_ERR_FORMAT; // one scale per long row needs the storing row-mode pass
    if (x->axis == 0 && (!axis0_format_ok(sparse_fmt, pattern, x->k) || !axis0_format_ok(dense_fmt, SS24_DENSE, x->k)))
        return SS24_ERR_FORMAT;
    if (x->rows == 0)
        return empty_operand(x, energy, nullptr, nullptr, s);
    TilePlan t;
    if (!plan_tile(x, pattern, score, kEnergy, &t))
        return SS24_ERR_CUDA;
    // 2:4 by magnitude on bf16 full-width rows with k a multiple of 64: the
    // lane-block form with both formats fixed at compile time (rotated or not)
    if (x->axis == 1 && x->dtype == SS24_BF16 && score == SS24_SCORE_MAG && pattern == SS24_SPARSE_24 &&
        t.g.W == 256 && t.g.step_cols == 256 && x->k % 64 == 0) {
        const void *kl = x->hadamard != 0 ? stream_lb_energy_kernel_bf16_rot(rs.q.fmt, rd.q.fmt)
                                          : stream_lb_energy_kernel_bf16(rs.q.fmt, rd.q.fmt);
        if (kl)
            t.kernel = kl;
    }
    PassParams p = base_params(x, t.g, ws, energy);
    p.norms = col_norms;
    p.q = rs.q;
    p.qd = rd.q;
    const bool need_s = per_tensor(sparse_fmt.kind) && !sparse_scale_in;
    const bool need_d = per_tensor(dense_fmt.kind) && !dense_scale_in;
    if (need_s || need_d) {
        if (run_amax(x, pattern, score, col_norms, ws, s) != cudaSuccess)
            return SS24_ERR_CUDA;
    }
    p.q.scale_in = sparse_scale_in;
    p.q.amax_reduced = p.amax_out;     // [0]: amax of the kept values
    p.qd.scale_in = dense_scale_in;
    p.qd.amax_reduced = p.amax_out + 1; // [1]: amax of all values
    return cuda_status(launch(t.kernel, t.smem, t.g.n_tiles, t.map, p, s));
}

ss24_status ss24_amax(const ss24_operand *x, ss24_pattern pattern, ss24_score score, const float *col_norms,
                      float *amax_out, void *ws, size_t ws_bytes, ss24_stream stream)
{
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    ss24_status st = check_operand(x);
    if (st != SS24_OK)
        return st;
    if ((st = check_pattern_k(pattern, x->k)) != SS24_OK)
        return st;
    if (score != SS24_SCORE_MAG && score != SS24_SCORE_WANDA)
        return SS24_ERR_ARG;
    if (x->hadamard != 0 && score != SS24_SCORE_MAG)
        return SS24_ERR_ARG; // a rotated pass selects by magnitude
    if (score == SS24_SCORE_WANDA && pattern != SS24_DENSE && (!col_norms || !aligned16(col_norms)))
        return col_norms ? SS24_ERR_ALIGN : SS24_ERR_NULL;
    if ((st = check_ws(ws, ws_bytes)) != SS24_OK)
        return st;
    if (!amax_out)
        return SS24_ERR_NULL;
    if (x->rows == 0)
        return cuda_status(cudaMemsetAsync(amax_out, 0, nbatch(x) * sizeof(float), s));
    return cuda_status(run_amax(x, pattern, score, col_norms, ws, s, nullptr, 1.0f, amax_out));
}

ss24_status ss24_amax_rows(const ss24_operand *x, ss24_pattern pattern, ss24_score score, const float *col_norms,
                           float *row_amax, int32_t kind, float *scale_out, void *ws, size_t ws_bytes,
                           ss24_stream stream)
{
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    ss24_status st = check_operand(x);
    if (st != SS24_OK)
        return st;
    if (x->axis != 1)
        return SS24_ERR_ARG;
    if ((st = check_pattern_k(pattern, x->k)) != SS24_OK)
        return st;
    if (score != SS24_SCORE_MAG && score != SS24_SCORE_WANDA)
        return SS24_ERR_ARG;
    if (x->hadamard != 0 && score != SS24_SCORE_MAG)
        return SS24_ERR_ARG; // a rotated pass selects by magnitude
    if (score == SS24_SCORE_WANDA && pattern != SS24_DENSE && (!col_norms || !aligned16(col_norms)))
        return col_norms ? SS24_ERR_ALIGN : SS24_ERR_NULL;
    if (scale_out && !per_tensor(kind))
        return SS24_ERR_FORMAT;
    if ((st = check_ws(ws, ws_bytes)) != SS24_OK)
        return st;
    if (!row_amax && x->rows != 0) // an empty operand may give a NULL row array
        return SS24_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(row_amax) & 3u) != 0)
        return SS24_ERR_ALIGN;
    const size_t nb = static_cast<size_t>(nbatch(x));
    if (x->rows == 0)
        return scale_out ? cuda_status(cudaMemsetAsync(scale_out, 0, nb * sizeof(float), s)) : SS24_OK;
    // full-width rows are each reduced by one warp and stored; other shapes
    // reduce row segments with atomic maxima into a cleared array
    const Geometry g = stream_geometry(x);
    if (!(g.W == 256 && g.step_cols == 256)) {
        cudaError_t e = cudaMemsetAsync(row_amax, 0, nb * static_cast<size_t>(x->rows) * sizeof(float), s);
        if (e != cudaSuccess)
            return SS24_ERR_CUDA;
    }
    const float divisor = kind == SS24_FMT_FP8_E4M3 ? 448.0f : 2688.0f;
    return cuda_status(run_amax(x, pattern, score, col_norms, ws, s, scale_out, scale_out ? divisor : 1.0f, nullptr,
                                row_amax));
}

ss24_status ss24_quantize_int_rows(const ss24_operand *x, ss24_pattern pattern, ss24_score score,
                                   const float *col_norms, ss24_format fmt, const float *row_amax,
                                   ss24_outputs *out, ss24_energy *energy, void *ws, size_t ws_bytes,
                                   ss24_stream stream)
{
    if (fmt.kind != SS24_FMT_INT || fmt.group != 0)
        return SS24_ERR_FORMAT;
    if (!x)
        return SS24_ERR_NULL;
    if (x->axis != 1)
        return SS24_ERR_ARG;
    if (!row_amax && x->rows != 0)
        return SS24_ERR_NULL;
    if ((reinterpret_cast<uintptr_t>(row_amax) & 3u) != 0)
        return SS24_ERR_ALIGN;
    return run_pass(x, pattern, score, col_norms, fmt, false, nullptr, out, energy, ws, ws_bytes,
                    reinterpret_cast<cudaStream_t>(stream), row_amax);
}

ss24_status ss24_tensor_scale(const ss24_operand *x, ss24_pattern pattern, ss24_score score, const float *col_norms,
                              int32_t kind, float *scale_out, void *ws, size_t ws_bytes, ss24_stream stream)
{
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    ss24_status st = check_operand(x);
    if (st != SS24_OK)
        return st;
    if ((st = check_pattern_k(pattern, x->k)) != SS24_OK)
        return st;
    if (score != SS24_SCORE_MAG && score != SS24_SCORE_WANDA)
        return SS24_ERR_ARG;
    if (x->hadamard != 0 && score != SS24_SCORE_MAG)
        return SS24_ERR_ARG; // a rotated pass selects by magnitude
    if (score == SS24_SCORE_WANDA && pattern != SS24_DENSE && (!col_norms || !aligned16(col_norms)))
        return col_norms ? SS24_ERR_ALIGN : SS24_ERR_NULL;
    if (!per_tensor(kind))
        return SS24_ERR_FORMAT;
    if ((st = check_ws(ws, ws_bytes)) != SS24_OK)
        return st;
    if (!scale_out)
        return SS24_ERR_NULL;
    if (x->rows == 0)
        return cuda_status(cudaMemsetAsync(scale_out, 0, nbatch(x) * sizeof(float), s));
    const float divisor = kind == SS24_FMT_FP8_E4M3 ? 448.0f : 2688.0f;
    return cuda_status(run_amax(x, pattern, score, col_norms, ws, s, scale_out, divisor));
}

ss24_status ss24_dequantize(const ss24_operand *x, ss24_pattern pattern, ss24_format fmt, const ss24_outputs *in,
                            float *xhat, ss24_stream stream)
{
    if (!x || !in)
        return SS24_ERR_NULL;
    if (x->dtype != SS24_BF16 && x->dtype != SS24_F32)
        return SS24_ERR_DTYPE;
    if (x->rows < 0 || x->k <= 0 || x->rows > INT32_MAX || x->k > INT32_MAX)
        return SS24_ERR_SHAPE;
    if (x->batch < 0 || x->batch > kMaxGrid)
        return SS24_ERR_SHAPE;
    ss24_status st = check_pattern_k(pattern, x->k);
    if (st != SS24_OK)
        return st;
    Resolved r;
    if ((st = resolve_format(fmt, pattern, x->k, true, &r)) != SS24_OK)
        return st;
    if (x->rows == 0)
        return SS24_OK;
    const bool needs_scales = fmt.kind == SS24_FMT_INT || fmt.kind == SS24_FMT_NVFP4 || fmt.kind == SS24_FMT_MXFP4;
    if (!in->values || !xhat || (needs_scales && !in->scales) || (per_tensor(fmt.kind) && !in->tensor_scale) ||
        (pattern != SS24_DENSE && !in->meta))
        return SS24_ERR_NULL;
    if (!aligned16(xhat) || !aligned16(in->values))
        return SS24_ERR_ALIGN;
    // the outputs of a batch are packed operand after operand, each the exact size
    // of one operand's outputs (as the pass writes them)
    int32_t lg = -1; // INT: log2 of the group of quantized values; one scale per row: -1
    if (fmt.kind == SS24_FMT_INT && fmt.group != 0)
        lg = ilog2(fmt.group);
    return cuda_status(launch_dequant(pattern, fmt.kind, r.q.store, lg, x->dtype == SS24_F32 ? 1 : 0, x->rows, x->k,
                                      static_cast<int32_t>(nbatch(x)), in->values, in->scales, in->tensor_scale,
                                      in->meta, xhat, reinterpret_cast<cudaStream_t>(stream)));
}

ss24_status ss24_softmax_prune(const ss24_operand *s, float alpha, ss24_pattern pattern, ss24_format fmt,
                               const float *tensor_scale_in, ss24_outputs *out, ss24_energy *energy, void *ws,
                               size_t ws_bytes, ss24_stream stream)
{
    ss24_status st = check_operand(s);
    if (st != SS24_OK)
        return st;
    if (s->axis != 1 || !std::isfinite(alpha) || s->hadamard != 0)
        return SS24_ERR_ARG;
    if ((st = check_pattern_k(pattern, s->k)) != SS24_OK)
        return st;
    if (s->k % 256 != 0)
        return SS24_ERR_SHAPE;
    if ((st = check_ws(ws, ws_bytes)) != SS24_OK)
        return st;
    Resolved r;
    if ((st = resolve_format(fmt, pattern, s->k, true, &r)) != SS24_OK)
        return st;
    if (r.row_mode)
        return SS24_ERR_FORMAT; // one INT scale per row is not offered here
    if (!out)
        return SS24_ERR_NULL;
    if (per_tensor(fmt.kind) && !tensor_scale_in)
        return SS24_ERR_NULL; // the tensor scale of P must be given
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    if (s->rows == 0)
        return empty_operand(s, energy, out, per_tensor(fmt.kind) ? tensor_scale_in : nullptr, cs);
    const bool needs_scales = fmt.kind == SS24_FMT_INT || fmt.kind == SS24_FMT_NVFP4 || fmt.kind == SS24_FMT_MXFP4;
    if (!out->values || (needs_scales && !out->scales) || (per_tensor(fmt.kind) && !out->tensor_scale) ||
        (pattern != SS24_DENSE && !out->meta))
        return SS24_ERR_NULL;
    if (!aligned16(out->values) || (needs_scales && !aligned16(out->scales)) ||
        (pattern != SS24_DENSE && !aligned16(out->meta)))
        return SS24_ERR_ALIGN;
    PassParams p = base_params(s, stream_geometry(s), ws, energy);
    output_strides(s, pattern, fmt, &p);
    p.values = out->values;
    p.scales = out->scales;
    p.meta = out->meta;
    p.q = r.q;
    if (per_tensor(fmt.kind)) {
        p.q.scale_in = tensor_scale_in;
        p.q.scale_out = out->tensor_scale;
    }
    const bool smem = s->k <= kSoftmaxSmemKeys;
    const size_t smem_bytes = smem ? static_cast<size_t>(kStreamWarps) * s->k * sizeof(float) : 0;
    const void *k = softmax_prune_kernel_ptr(s->dtype == SS24_BF16 ? 1 : 0, pattern, fmt.kind, smem);
    if (!k)
        return SS24_ERR_FORMAT;
    KernelInfo info;
    // (the dynamic shared memory of the largest row, set once per kernel)
    cudaError_t e = kernel_info(k, smem ? static_cast<size_t>(kStreamWarps) * kSoftmaxSmemKeys * sizeof(float) : 0,
                                &info, kStreamThreads);
    if (e != cudaSuccess)
        return SS24_ERR_CUDA;
    if (smem) {
        int per_sm = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k, kStreamThreads, smem_bytes);
        if (e != cudaSuccess)
            return SS24_ERR_CUDA;
        info.blocks_per_sm = per_sm;
    }
    p.ctas_per_op = static_cast<int32_t>(ctas_per_operand(info, p.batch, (s->rows + kStreamWarps - 1) / kStreamWarps));
    float a = alpha;
    void *args[2] = {&p, &a};
    return cuda_status(
        launch_pdl(k, static_cast<unsigned>(p.batch * p.ctas_per_op), kStreamThreads, smem_bytes, cs, args));
}

ss24_status ss24_hadamard(const ss24_operand *x, int32_t block, float *out, ss24_stream stream)
{
    ss24_status st = check_operand(x);
    if (st != SS24_OK)
        return st;
    if (x->hadamard != 0)
        return SS24_ERR_ARG; // (the rotation is this call's own block)
    if (x->axis != 1)
        return SS24_ERR_ARG;
    if (block < 2 || block > 256 || (block & (block - 1)) != 0)
        return SS24_ERR_ARG;
    if (x->k % 8 != 0 || x->k % block != 0)
        return SS24_ERR_SHAPE;
    if (x->rows == 0)
        return SS24_OK;
    if (!out)
        return SS24_ERR_NULL;
    if (!aligned16(out))
        return SS24_ERR_ALIGN;
    return cuda_status(launch_hadamard(x->x, x->dtype == SS24_BF16 ? 1 : 0, x->rows, x->k, x->ld,
                                       nbatch(x) > 1 ? x->batch_stride : 0, nbatch(x), block, out,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

int64_t ss24_scale_tiles_bytes(int64_t rows, int64_t cols)
{
    return scale_tiles_bytes(rows, cols);
}

ss24_status ss24_scale_tiles(const uint8_t *scales, int64_t rows, int64_t cols, int64_t batch, uint8_t *tiles,
                             ss24_stream stream)
{
    if (rows < 0 || cols < 0 || batch < 0 || batch > kMaxGrid)
        return SS24_ERR_SHAPE;
    const int64_t nb = batch > 1 ? batch : 1;
    if (scale_tiles_bytes(rows, cols) == 0)
        return SS24_OK;
    if (!tiles || (!scales && rows * cols > 0))
        return SS24_ERR_NULL;
    if (!aligned16(tiles))
        return SS24_ERR_ALIGN;
    return cuda_status(launch_scale_tiles(scales, rows, cols, nb, tiles, reinterpret_cast<cudaStream_t>(stream)));
}

ss24_status ss24_predicted_ratio(const ss24_energy *sparse_side, const ss24_energy *dense_side, ss24_ratio *out,
                                 int64_t count, ss24_stream stream)
{
    if (count < 0)
        return SS24_ERR_SHAPE;
    if (count > 0 && (!sparse_side || !dense_side || !out))
        return SS24_ERR_NULL;
    return cuda_status(launch_ratio(reinterpret_cast<const double *>(sparse_side),
                                    reinterpret_cast<const double *>(dense_side), reinterpret_cast<double *>(out),
                                    count, reinterpret_cast<cudaStream_t>(stream)));
}

double ss24_bits_per_element(ss24_format fmt, ss24_pattern pattern, int64_t k, int32_t with_scales)
{
    if (pattern != SS24_DENSE && pattern != SS24_SPARSE_24 && pattern != SS24_SPARSE_48)
        return -1.0;
    double vb;
    switch (fmt.kind) {
    case SS24_FMT_NONE:
        vb = 16.0;
        break;
    case SS24_FMT_FP8_E4M3:
        vb = 8.0;
        break;
    case SS24_FMT_INT:
        if (fmt.bits < 2 || fmt.bits > 16)
            return -1.0;
        vb = fmt.bits;
        break;
    case SS24_FMT_NVFP4:
    case SS24_FMT_MXFP4:
        vb = 4.0;
        break;
    default:
        return -1.0;
    }
    const double kept = pattern == SS24_DENSE ? 1.0 : 0.5;
    const double index = pattern == SS24_SPARSE_24 ? 1.0 : (pattern == SS24_SPARSE_48 ? 0.25 : 0.0);
    double bits = kept * vb + index;
    if (with_scales) {
        double per_value = 0.0;
        if (fmt.kind == SS24_FMT_INT)
            per_value = 32.0 / (fmt.group > 0 ? static_cast<double>(fmt.group) : kept * static_cast<double>(k));
        else if (fmt.kind == SS24_FMT_NVFP4)
            per_value = 8.0 / 16.0;
        else if (fmt.kind == SS24_FMT_MXFP4)
            per_value = 8.0 / 32.0;
        bits += kept * per_value;
    }
    return bits;
}

const char *ss24_status_string(ss24_status status)
{
    switch (status) {
    case SS24_OK:
        return "ok";
    case SS24_ERR_NULL:
        return "a required pointer is NULL";
    case SS24_ERR_SHAPE:
        return "shape does not fit the pattern or format";
    case SS24_ERR_ALIGN:
        return "pointer or row stride not 16-byte aligned";
    case SS24_ERR_DTYPE:
        return "unknown element type";
    case SS24_ERR_FORMAT:
        return "unsupported quantization format";
    case SS24_ERR_WORKSPACE:
        return "workspace missing, too small or misaligned";
    case SS24_ERR_CUDA:
        return "CUDA call or launch failed";
    case SS24_ERR_ARG:
        return "unknown score, axis or pattern";
    }
    return "unknown status";
}

ss24_status ss24_selfcheck_division(int32_t mode, uint32_t b_first, uint32_t b_count, unsigned long long *result,
                                    ss24_stream stream)
{
    if (!result)
        return SS24_ERR_NULL;
    if (mode < 0 || mode > 2)
        return SS24_ERR_ARG;
    if (mode == 0 && (b_first >= (1u << 23) || b_count > (1u << 23) - b_first))
        return SS24_ERR_SHAPE;
    if (mode == 2 && (b_first >= (1u << 15) || b_count > (1u << 15) - b_first))
        return SS24_ERR_SHAPE;
    if (b_count > 65535u * 32u)
        return SS24_ERR_SHAPE;
    return cuda_status(launch_selfcheck_division(mode, b_first, b_count, result, reinterpret_cast<cudaStream_t>(stream)));
}

ss24_status ss24_selfcheck_encoder(int32_t kind, const uint32_t *bounds, int32_t n_bounds, uint32_t hi_first,
                                   uint32_t hi_count, unsigned long long *result, ss24_stream stream)
{
    if (!bounds || !result)
        return SS24_ERR_NULL;
    int e2m1;
    if (kind == SS24_FMT_FP8_E4M3)
        e2m1 = 0;
    else if (kind == SS24_FMT_NVFP4 || kind == SS24_FMT_MXFP4)
        e2m1 = 1;
    else
        return SS24_ERR_FORMAT;
    if (n_bounds != (e2m1 ? 7 : 126))
        return SS24_ERR_SHAPE;
    if (hi_first >= 65536u || hi_count > 65536u - hi_first)
        return SS24_ERR_SHAPE;
    return cuda_status(launch_selfcheck_encoder(e2m1, bounds, n_bounds, hi_first, hi_count, result,
                                                reinterpret_cast<cudaStream_t>(stream)));
}

ss24_status ss24_encode_e4m3(const float *in, uint8_t *out, int64_t n, ss24_stream stream)
{
    if ((!in || !out) && n > 0)
        return SS24_ERR_NULL;
    if (n < 0)
        return SS24_ERR_SHAPE;
    return cuda_status(launch_convert(0, in, out, n, reinterpret_cast<cudaStream_t>(stream)));
}

ss24_status ss24_decode_e4m3(const uint8_t *in, float *out, int64_t n, ss24_stream stream)
{
    if ((!in || !out) && n > 0)
        return SS24_ERR_NULL;
    if (n < 0)
        return SS24_ERR_SHAPE;
    return cuda_status(launch_convert(1, in, out, n, reinterpret_cast<cudaStream_t>(stream)));
}

ss24_status ss24_encode_e2m1(const float *in, uint8_t *out, int64_t n, ss24_stream stream)
{
    if ((!in || !out) && n > 0)
        return SS24_ERR_NULL;
    if (n < 0)
        return SS24_ERR_SHAPE;
    return cuda_status(launch_convert(2, in, out, n, reinterpret_cast<cudaStream_t>(stream)));
}

ss24_status ss24_decode_e2m1(const uint8_t *in, float *out, int64_t n, ss24_stream stream)
{
    if ((!in || !out) && n > 0)
        return SS24_ERR_NULL;
    if (n < 0)
        return SS24_ERR_SHAPE;
    return cuda_status(launch_convert(3, in, out, n, reinterpret_cast<cudaStream_t>(stream)));
}

ss24_status ss24_sparse_gemm_fp8(const uint8_t *a_values, const uint8_t *a_meta, const float *a_scale,
                                 const uint8_t *b, const float *b_scale, int64_t m, int64_t n, int64_t k, float *y,
                                 void *ws, size_t ws_bytes, ss24_stream stream)
{
    if (m < 0 || n < 0 || k <= 0 || m % 128 != 0 || n % 128 != 0 || k % 256 != 0 || m > INT32_MAX ||
        n > INT32_MAX || k > INT32_MAX)
        return SS24_ERR_SHAPE;
    ss24_status st = check_ws(ws, ws_bytes);
    if (st != SS24_OK)
        return st;
    if (m == 0 || n == 0)
        return SS24_OK;
    if (!a_values || !a_meta || !a_scale || !b || !b_scale || !y)
        return SS24_ERR_NULL;
    if (!aligned16(a_values) || !aligned16(a_meta) || !aligned16(b) || !aligned16(y))
        return SS24_ERR_ALIGN;
    int32_t *err = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(ws) + kWsErrOff);
    return cuda_status(launch_sparse_gemm_fp8(a_values, a_meta, a_scale, b, b_scale, m, n, k, y, err, kWaitLimitNs,
                                              reinterpret_cast<cudaStream_t>(stream)));
}

ss24_status ss24_prune24_quant_fused_noalloc(const ss24_operand *x, ss24_score score, const float *col_norms,
                                             ss24_format fmt, const float *tensor_scale_in, ss24_outputs *out,
                                             ss24_energy *energy, ss24_stream stream)
{
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // the strided-axis kernel waits on its copies with a time limit and records
    // a wait that gave up in the scratch's error word, which a caller of this
    // entry point cannot read: only the axis-1 kernels (no such waits) run here
    if (x && x->axis != 1)
        return SS24_ERR_ARG;
    void *scratch = nullptr;
    if (static_scratch(&scratch) != cudaSuccess)
        return SS24_ERR_CUDA;
    // every check first: a rejected call enqueues nothing, not even the clear
    ss24_status st = run_pass(x, SS24_SPARSE_24, score, col_norms, fmt, true, tensor_scale_in, out, energy, scratch,
                              kStaticScratchBytes, s, nullptr, false);
    if (st != SS24_OK)
        return st;
    // the error word and the ticket counters must start at zero for this call
    if (cudaMemsetAsync(scratch, 0, kWsClearBytes, s) != cudaSuccess)
        return SS24_ERR_CUDA;
    return run_pass(x, SS24_SPARSE_24, score, col_norms, fmt, true, tensor_scale_in, out, energy, scratch,
                    kStaticScratchBytes, s);
}

} // extern "C"
