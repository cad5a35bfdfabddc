// The consumer of the online pass: a 2:4-sparse GEMM on the 5th-generation
// tensor cores that reads the pass's outputs as they are stored.
//
// "Is 2:4 Sparsity Still Worth It? Semi-Structured Sparsity versus
// Quantization in LLM Inference" §1 (operands computed on the fly are pruned
// and compressed before every GEMM), §3 (the sparse GEMM reads the kept values
// and their indices; FP8 as the 2x tier). Y[m][n] = s_a s_b sum_k A[m][k] B[n][k]
// with A the 2:4 operand (FP8 E4M3 kept values [m][k/2] and metadata [m][k/8]
// from ss24_prune24_quant_fused, tensor scale s_a) and B a dense FP8 E4M3
// operand [n][k] (tensor scale s_b), accumulated in binary32 in tensor memory.
//
// The metadata bytes of the pass (one nibble i0 | i1 << 2 per group of four,
// two groups per byte, even group in the low nibble, rows of k/8 bytes) are the
// operand the sparse MMA of kind f8f6f4 takes: per row of A, 8 bytes for each
// 64 values of k, copied into tensor memory as 128 rows x 16 bytes (two MMA k
// steps) per copy. A 2-D TMA box of 16 bytes x 128 rows cuts them out of the
// row-major array; no reordering pass is needed.
//
// Kernel. One CTA per 128 x BN output tile, 128 threads. Lane 0 of warp 0
// streams k tiles of BK into a ring of stages by TMA (A: 128 rows x BK/2
// bytes with 128- or 64-byte swizzle, B: BN rows x BK bytes as boxes of 128
// bytes with 128-byte swizzle; metadata: 128 rows x BK/8 bytes); lane 0 of
// warp 1 copies each stage's metadata into tensor memory and issues BK/64
// sparse MMAs (k = 64 each, N = BN) per stage, releasing the stage with a
// commit; the four warps then read the accumulator (warp w: rows 32w .. 32w +
// 31) and write Y. Two shapes: BN = 256 with BK = 128 and five stages where n
// is a multiple of 256 (each A and B byte brought to the SM serves twice the
// products of the other shape), else BN = 128 with BK = 256 and four stages.
// Every barrier wait is bounded: a wait that gives up records an error code
// in the workspace, and the kernel still drains its copies and frees its
// tensor memory.
#include <cudaTypedefs.h>

#include "device.cuh"
#include "internal.cuh"

namespace ss24 {

namespace {

constexpr int kGemmBM = 128;
constexpr int kGemmThreads = 128;

// A tile shape: BN output columns, BK logical k per stage, STAGES stages.
template <int BN, int BK, int STAGES> struct GemmShape {
    static constexpr uint32_t kABytes = kGemmBM * BK / 2; // compressed A: 128 rows x BK/2 bytes
    static constexpr uint32_t kBBytes = BN * BK;          // BK/128 boxes of BN rows x 128 bytes
    static constexpr uint32_t kEBytes = kGemmBM * BK / 8; // BK/128 boxes of 128 rows x 16 bytes
    static constexpr uint32_t kStageBytes = kABytes + kBBytes + kEBytes;
    static constexpr int kBoxes = BK / 128;               // B and metadata boxes per stage
    static constexpr int kSteps = BK / 64;                // MMAs per stage
    static constexpr uint32_t kMetaCols = BK / 32;        // tensor-memory columns of a stage's metadata
    // accumulator BN columns + the stages' metadata, rounded up to a power of two
    static constexpr uint32_t kTmemCols = BN + STAGES * kMetaCols <= 256 ? 256 : 512;
    static constexpr size_t kSmemBytes = STAGES * kStageBytes + 1024 + 256;
    static_assert(kStageBytes % 1024 == 0, "stages on 1024-byte boundaries");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
};

// Shared-memory matrix descriptor (tcgen05): start address, leading and stride
// byte offsets (in 16-byte units), version 1, layout type.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout)
{
    uint64_t d = 0;
    d |= static_cast<uint64_t>((addr >> 4) & 0x3fffu);
    d |= static_cast<uint64_t>(lbo & 0x3fffu) << 16;
    d |= static_cast<uint64_t>(sbo & 0x3fffu) << 32;
    d |= static_cast<uint64_t>(1u) << 46; // descriptor version
    d |= static_cast<uint64_t>(layout & 7u) << 61;
    return d;
}
constexpr uint32_t kLayoutNone = 0, kLayoutSw128 = 2;

constexpr uint32_t kLayoutSw64 = 4;

// K-major operand with 128-byte swizzle: rows of 128 bytes, 8-row groups
// 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t addr) { return smem_desc(addr, 1, 64, kLayoutSw128); }
// K-major operand with 64-byte swizzle: rows of 64 bytes, 8-row groups 512
// bytes apart.
__device__ __forceinline__ uint64_t desc_sw64(uint32_t addr) { return smem_desc(addr, 1, 32, kLayoutSw64); }

// Instruction descriptor: sparse, binary32 accumulator, E4M3 x E4M3, both
// K-major, N = BN, M = 128.
template <int BN>
constexpr uint32_t kGemmIdesc = (1u << 2)                                     // sparse
                                | (1u << 4)                                   // D: f32
                                | (0u << 7) | (0u << 10)                      // A, B: e4m3
                                | (static_cast<uint32_t>(BN >> 3) << 17)      // N / 8
                                | (static_cast<uint32_t>(kGemmBM >> 4) << 24); // M / 16

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t cols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(cols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() { asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::); }
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_cp_128x128b(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tc_mma_sp(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t e_tmem,
                                          uint32_t idesc, uint32_t accumulate)
{
    const uint32_t z = 0;
    asm volatile("{\n"
                 " .reg .pred p;\n"
                 " setp.ne.b32 p, %4, 0;\n"
                 " tcgen05.mma.sp.cta_group::1.kind::f8f6f4 [%0], %1, %2, [%3], %5, {%6, %6, %6, %6}, p;\n"
                 "}\n" ::"r"(d_tmem),
                 "l"(adesc), "l"(bdesc), "r"(e_tmem), "r"(accumulate), "r"(idesc), "r"(z)
                 : "memory");
}
// 32 consecutive accumulator columns of this thread's row (lane base in taddr)
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, "
                 "%14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                   "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                   "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                   "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]),
                   "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 2-D tiled TMA load of one box (no cache hint), completing on `bar`.
__device__ __forceinline__ void tma_box(void *dst, const CUtensorMap *map, int32_t c_inner, int32_t c_outer,
                                        uint64_t *bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(c_inner), "r"(c_outer), "r"(smem_u32(bar))
                 : "memory");
}

struct GemmParams {
    int64_t m, n, k;
    const float *a_scale, *b_scale;
    float *y;
    int32_t *err;
    uint64_t wait_limit_ns;
};

template <int BN, int BK, int STAGES>
__global__ void __launch_bounds__(kGemmThreads, 1)
    sparse_gemm_fp8_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                           const __grid_constant__ CUtensorMap map_e, const GemmParams p)
{
    using S = GemmShape<BN, BK, STAGES>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    // stages start on a 1024-byte boundary (swizzle atoms)
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *stages = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(stages + STAGES * S::kStageBytes);
    uint64_t *empty = full + STAGES;
    uint64_t *accbar = empty + STAGES;
    uint32_t *tmem_base_smem = reinterpret_cast<uint32_t *>(accbar + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t n0 = static_cast<int64_t>(blockIdx.x) * BN, m0 = static_cast<int64_t>(blockIdx.y) * kGemmBM;
    const int nk = static_cast<int>(p.k / BK);

    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accbar, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(tmem_base_smem, S::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_smem;
    grid_dependency_wait();

    if (warp == 0 && lane == 0) {
        // producer: one stage per k tile
        int issued = 0;
        bool failed = false;
        for (int kt = 0; kt < nk; ++kt) {
            const int s = kt % STAGES;
            if (kt >= STAGES && !mbar_wait(&empty[s], ((kt / STAGES) - 1) & 1, p.wait_limit_ns)) {
                atomicCAS(p.err, 0, 11);
                failed = true;
                break;
            }
            uint8_t *sa = stages + s * S::kStageBytes, *sb = sa + S::kABytes, *se = sb + S::kBBytes;
            mbar_arrive_expect_tx(&full[s], S::kStageBytes);
            const int32_t ka = static_cast<int32_t>(kt * (BK / 2)), kb = kt * BK, ke = kt * (BK / 8);
            tma_box(sa, &map_a, ka, static_cast<int32_t>(m0), &full[s]);
#pragma unroll
            for (int h = 0; h < S::kBoxes; ++h) {
                tma_box(sb + h * (BN * 128), &map_b, kb + 128 * h, static_cast<int32_t>(n0), &full[s]);
                tma_box(se + h * (kGemmBM * 16), &map_e, ke + 16 * h, static_cast<int32_t>(m0), &full[s]);
            }
            ++issued;
        }
        if (failed) {
            // the copies already issued land before the CTA can exit
            for (int kt = issued > STAGES ? issued - STAGES : 0; kt < issued; ++kt)
                (void)mbar_wait(&full[kt % STAGES], (kt / STAGES) & 1, p.wait_limit_ns);
        }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer
        const uint32_t acc = tmem;
        for (int kt = 0; kt < nk; ++kt) {
            const int s = kt % STAGES;
            if (!mbar_wait(&full[s], (kt / STAGES) & 1, p.wait_limit_ns)) {
                atomicCAS(p.err, 0, 12);
                break;
            }
            tc_fence_after();
            uint8_t *sa = stages + s * S::kStageBytes, *sb = sa + S::kABytes, *se = sb + S::kBBytes;
            // metadata: 128-row x 16-byte tiles into this stage's columns
            const uint32_t ecol = BN + S::kMetaCols * s;
#pragma unroll
            for (int h = 0; h < S::kBoxes; ++h)
                tc_cp_128x128b(tmem + ecol + 4 * h, smem_desc(smem_u32(se + h * (kGemmBM * 16)), 128, 8, kLayoutNone));
#pragma unroll
            for (int j = 0; j < S::kSteps; ++j) {
                // k step j: 64 values of k = 32 bytes of compressed A, 64 bytes of B
                const uint64_t ad = BK == 256 ? desc_sw128(smem_u32(sa) + 32 * j) : desc_sw64(smem_u32(sa) + 32 * j);
                const uint64_t bd = desc_sw128(smem_u32(sb) + (j >> 1) * (BN * 128) + 64 * (j & 1));
                tc_mma_sp(acc, ad, bd, tmem + ecol + 2 * j, kGemmIdesc<BN>, (kt | j) != 0 ? 1u : 0u);
            }
            tc_commit(&empty[s]); // the stage is free once these MMAs have read it
        }
        tc_commit(accbar); // the accumulator is complete once every MMA issued has finished
    }
    __syncwarp();

    // epilogue: warp w reads accumulator rows 32w .. 32w + 31
    const bool ok = mbar_wait(accbar, 0, p.wait_limit_ns);
    if (!ok && lane == 0)
        atomicCAS(p.err, 0, 13);
    tc_fence_after();
    const float sc = __fmul_rn(*p.a_scale, *p.b_scale);
    const int64_t row = m0 + 32 * warp + lane;
    float *yr = p.y + row * p.n + n0;
#pragma unroll 1
    for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32];
        tmem_ld32(tmem + (static_cast<uint32_t>(32 * warp) << 16) + c0, v);
#pragma unroll
        for (int i = 0; i < 32; i += 4)
            *reinterpret_cast<float4 *>(yr + c0 + i) =
                make_float4(__fmul_rn(__uint_as_float(v[i]), sc), __fmul_rn(__uint_as_float(v[i + 1]), sc),
                            __fmul_rn(__uint_as_float(v[i + 2]), sc), __fmul_rn(__uint_as_float(v[i + 3]), sc));
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, S::kTmemCols);
    }
}

bool encode_u8(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer, uint64_t row_bytes,
               uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle)
{
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !fn)
        return false;
    auto encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    cuuint64_t gdim[2] = {inner, outer};
    cuuint64_t gstride[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estride[2] = {1, 1};
    return encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), gdim, gstride, box, estride,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

using GemmWide = GemmShape<256, 128, 5>;
using GemmNarrow = GemmShape<128, 256, 4>;

template <int BN, int BK, int STAGES>
cudaError_t launch_shape(const uint8_t *a_values, const uint8_t *a_meta, const float *a_scale, const uint8_t *b,
                         const float *b_scale, int64_t m, int64_t n, int64_t k, float *y, int32_t *err,
                         uint64_t wait_limit_ns, cudaStream_t stream)
{
    using S = GemmShape<BN, BK, STAGES>;
    CUtensorMap ma, mb, me;
    if (!encode_u8(&ma, a_values, k / 2, m, k / 2, BK / 2, kGemmBM,
                   BK == 256 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B) ||
        !encode_u8(&mb, b, k, n, k, 128, BN, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_u8(&me, a_meta, k / 8, m, k / 8, 16, kGemmBM, CU_TENSOR_MAP_SWIZZLE_NONE))
        return cudaErrorInvalidValue;
    auto kern = sparse_gemm_fp8_kernel<BN, BK, STAGES>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(S::kSmemBytes));
    if (e != cudaSuccess)
        return e;
    GemmParams p{m, n, k, a_scale, b_scale, y, err, wait_limit_ns};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(n / BN), static_cast<unsigned>(m / kGemmBM));
    cfg.blockDim = dim3(kGemmThreads);
    cfg.dynamicSmemBytes = S::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, ma, mb, me, p);
}

} // namespace

size_t sparse_gemm_smem_bytes() { return GemmWide::kSmemBytes > GemmNarrow::kSmemBytes ? GemmWide::kSmemBytes : GemmNarrow::kSmemBytes; }

cudaError_t launch_sparse_gemm_fp8(const uint8_t *a_values, const uint8_t *a_meta, const float *a_scale,
                                   const uint8_t *b, const float *b_scale, int64_t m, int64_t n, int64_t k, float *y,
                                   int32_t *err, uint64_t wait_limit_ns, cudaStream_t stream)
{
    if (n % 256 == 0)
        return launch_shape<256, 128, 5>(a_values, a_meta, a_scale, b, b_scale, m, n, k, y, err, wait_limit_ns,
                                         stream);
    return launch_shape<128, 256, 4>(a_values, a_meta, a_scale, b, b_scale, m, n, k, y, err, wait_limit_ns, stream);
}

} // namespace ss24
