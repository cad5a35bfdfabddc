// Attention probabilities pruned in their producer: P = softmax(alpha * s)
// computed per row from the logits s and handed, as the bf16 operand it is,
// straight to the pass's chunk routine (2:4 / 4:8 selection, compression,
// quantization, energies), so P is never written to or read from HBM
// ("Is 2:4 Sparsity Still Worth It?" §3: P is pruned along the key axis; §1:
// an operand computed on the fly must be pruned before every GEMM).
//
// The arithmetic is fixed so that it can be reproduced bit for bit (the pages
// leave it open):
//   v_j = RN(alpha * s_j); m = max_j v_j; e_j = exp_ss(RN(v_j - m));
//   S = the row's 256-element slice sums added left to right, each slice
//       summed pairwise in index order;
//   p_j = RN(e_j / S), rounded to bf16 (nearest even).
// exp_ss (x <= 0): Cody and Waite's reduction x = n ln2 + r (ln2 split into an
// exact high part and a rounded low part), e^r by the degree-7 Taylor
// polynomial (coefficients RN(1/k!)) in Horner form with fused multiply-adds,
// then q * 2^n rounded once; arguments below -104 are taken as -104, where the
// result rounds to 0.
//
// One warp per row: lane L holds columns 256 t + 8 L .. + 7 of slice t, so a
// chunk's 8 values are summed in-lane as a pairwise tree and the 32 chunk sums
// of a slice by butterflies over lane distances 1, 2, ..., 16 (adjacent chunks
// first: the pairwise order). Three sweeps over the row: the maximum, the sum,
// then P and the pass. For rows of up to 2048 keys the warp keeps the row in
// shared memory (v, then e in place), so the logits are read once and e is
// computed once; longer rows are read again (from L2) and e recomputed.
#include "pass_impl.cuh"

namespace ss24 {

namespace {

// exp_ss of two values with packed arithmetic (fma2 rounds each lane once,
// like a scalar fused multiply-add): x' = max(x, -104); t = RN(x' log2e);
// n = RN(RN(t + 1.5 * 2^23) - 1.5 * 2^23) (t rounded to an integer, ties to
// even); r = fma(-n, ln2_hi, x'), r = fma(-n, ln2_lo, r); q = the degree-7
// Taylor polynomial of e^r in fused multiply-add Horner form; the result
// RN(RN(q * 2^(n + 64)) * 2^-64), q * 2^n rounded once. The bits of
// t + 1.5 * 2^23 are those of 1.5 * 2^23 plus n, and 1.5 * 2^23's bits shifted
// left by 23 vanish modulo 2^32, so one integer multiply-add gives the bits of
// 2^(n + 64).
__device__ __forceinline__ f32x2 exp_ss2(float x0, float x1)
{
    const f32x2 xc = pack2(fmaxf(x0, -104.0f), fmaxf(x1, -104.0f));
    const f32x2 t = mul2(xc, pack2(1.44269502162933349609375f, 1.44269502162933349609375f));
    const f32x2 magic = pack2(12582912.0f, 12582912.0f);
    const f32x2 tm = add2(t, magic);
    const f32x2 n = sub2(tm, magic);
    f32x2 r = fma2(n, pack2(-0.693145751953125f, -0.693145751953125f), xc);
    r = fma2(n, pack2(-1.428606765330187e-06f, -1.428606765330187e-06f), r);
    f32x2 q = pack2(1.98412701138295233249664306640625e-04f, 1.98412701138295233249664306640625e-04f);
    q = fma2(q, r, pack2(1.38888892251998186111450195312500e-03f, 1.38888892251998186111450195312500e-03f));
    q = fma2(q, r, pack2(8.33333376795053482055664062500000e-03f, 8.33333376795053482055664062500000e-03f));
    q = fma2(q, r, pack2(4.16666679084300994873046875000000e-02f, 4.16666679084300994873046875000000e-02f));
    q = fma2(q, r, pack2(1.66666671633720397949218750000000e-01f, 1.66666671633720397949218750000000e-01f));
    q = fma2(q, r, pack2(0.5f, 0.5f));
    q = fma2(q, r, pack2(1.0f, 1.0f));
    q = fma2(q, r, pack2(1.0f, 1.0f));
    const uint32_t s0 = __float_as_uint(lo2(tm)) * (1u << 23) + (191u << 23);
    const uint32_t s1 = __float_as_uint(hi2(tm)) * (1u << 23) + (191u << 23);
    const f32x2 up = mul2(q, pack2(__uint_as_float(s0), __uint_as_float(s1)));
    return mul2(up, pack2(0x1p-64f, 0x1p-64f));
}

// The 8 logits of one chunk as binary32 (bf16 widened exactly).
template <typename TL> __device__ __forceinline__ void load_logits(const TL *p, float (&v)[8]);
template <> __device__ __forceinline__ void load_logits<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[8])
{
    const uint4 w = ld_stream(p, true);
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(ws[i] << 16);
        v[2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
    }
}
template <> __device__ __forceinline__ void load_logits<float>(const float *p, float (&v)[8])
{
    const uint4 a = ld_stream(p, true), b = ld_stream(p + 4, true);
    v[0] = __uint_as_float(a.x), v[1] = __uint_as_float(a.y), v[2] = __uint_as_float(a.z),
    v[3] = __uint_as_float(a.w);
    v[4] = __uint_as_float(b.x), v[5] = __uint_as_float(b.y), v[6] = __uint_as_float(b.z),
    v[7] = __uint_as_float(b.w);
}

// P of one chunk as four bf16x2 words (lower value in the low half):
// p = RN(e / S) by Markstein's corrected reciprocal on packed pairs (div_fast:
// exact for quotients >= 2^-40, S being in [1, 2^31]; e >= 0 keeps the sign),
// the IEEE division for a chunk holding a smaller quotient; then the bf16
// rounding to nearest even of the conversion instruction (the reading's).
__device__ __forceinline__ uint4 p_chunk(const float (&e)[8], const Recip &rs, float tiny)
{
    const float mn = fminf(fminf(fminf(e[0], e[1]), fminf(e[2], e[3])), fminf(fminf(e[4], e[5]), fminf(e[6], e[7])));
    float q[8];
    if (mn >= tiny) {
        const f32x2 y2 = pack2(rs.y, rs.y), nb2 = pack2(rs.nb, rs.nb);
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
            const f32x2 a = pack2(e[j], e[j + 1]);
            const f32x2 q0 = mul2(a, y2);
            const f32x2 qq = fma2(fma2(q0, nb2, a), y2, q0);
            q[j] = lo2(qq);
            q[j + 1] = hi2(qq);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; ++j)
            q[j] = __fdiv_rn(e[j], rs.b);
    }
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(q[2 * j], q[2 * j + 1]);
        w[j] = *reinterpret_cast<const uint32_t *>(&h);
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// One row's 8 values of e for slice t: packed exp of RN(v - m).
__device__ __forceinline__ void slice_exp(const float (&v)[8], float m, float (&e)[8])
{
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
        const f32x2 r = exp_ss2(__fsub_rn(v[j], m), __fsub_rn(v[j + 1], m));
        e[j] = lo2(r);
        e[j + 1] = hi2(r);
    }
}

// SMEM: the warp keeps v = RN(alpha s) and then e in k floats of dynamic shared
// memory (each lane only its own columns), so the logits are read once; else
// the row is read three times (from L2 after the first) and e recomputed.
template <typename TL, int PAT, int FMT, bool SMEM>
__global__ void __launch_bounds__(kStreamThreads) softmax_prune_kernel(const __grid_constant__ PassParams pk,
                                                                        const float alpha)
{
    const PassParams &p = pk;
    const int op = static_cast<int>(blockIdx.x) / pk.ctas_per_op;
    const int cta = static_cast<int>(blockIdx.x) - op * pk.ctas_per_op;
    __shared__ double red[kStreamWarps * 4];
    __shared__ uint32_t flag;
    __shared__ float nvt[FMT == kNvfp4 ? 512 : 4];
    extern __shared__ float4 rowbuf[]; // SMEM: [kStreamWarps][k / 4]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    grid_dependency_wait();
    grid_dependents_launch();
    const PassConsts c = make_consts<FMT>(operand_view(pk), tid, kStreamThreads, nvt);
    const OutBase ob = out_base(pk, op);
    const TL *x = static_cast<const TL *>(p.x) + op * p.x_bstride;
    const int slices = static_cast<int>(p.k / 256);
    float4 *wb = rowbuf + (SMEM ? warp * (p.k / 4) + 2 * lane : 0); // this lane's 8 floats of slice 0
    double e_total = 0.0, e_prune = 0.0, e_q = 0.0, e_qd = 0.0;
    Acc acc{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int64_t row = static_cast<int64_t>(cta) * kStreamWarps + warp; row < p.rows;
         row += static_cast<int64_t>(p.ctas_per_op) * kStreamWarps) {
        const TL *xr = x + row * p.ld + 8 * lane;
        // sweep 1: the row maximum of v = alpha * s
        float m = -INFINITY;
        for (int t = 0; t < slices; ++t) {
            float v[8];
            load_logits<TL>(xr + 256 * t, v);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                v[j] = __fmul_rn(alpha, v[j]);
                m = fmaxf(m, v[j]);
            }
            if constexpr (SMEM) {
                wb[64 * t] = make_float4(v[0], v[1], v[2], v[3]);
                wb[64 * t + 1] = make_float4(v[4], v[5], v[6], v[7]);
            }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
        // sweep 2: e and the row sum, slice by slice
        float total = 0.0f;
        for (int t = 0; t < slices; ++t) {
            float v[8], e[8];
            if constexpr (SMEM) {
                const float4 a = wb[64 * t], b = wb[64 * t + 1];
                v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
            } else {
                load_logits<TL>(xr + 256 * t, v);
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    v[j] = __fmul_rn(alpha, v[j]);
            }
            slice_exp(v, m, e);
            if constexpr (SMEM) {
                wb[64 * t] = make_float4(e[0], e[1], e[2], e[3]);
                wb[64 * t + 1] = make_float4(e[4], e[5], e[6], e[7]);
            }
            float cs = __fadd_rn(__fadd_rn(__fadd_rn(e[0], e[1]), __fadd_rn(e[2], e[3])),
                                 __fadd_rn(__fadd_rn(e[4], e[5]), __fadd_rn(e[6], e[7])));
#pragma unroll
            for (int off = 1; off <= 16; off <<= 1)
                cs = __fadd_rn(cs, __shfl_xor_sync(kFull, cs, off));
            total = t == 0 ? cs : __fadd_rn(total, cs);
        }
        const Recip rs = make_recip(total);
        const float tiny = __fmul_rn(total, 0x1p-40f); // quotients below 2^-40 take the IEEE division
        // sweep 3: P in bf16, through the pass's chunk routine, four slices at a time
        for (int t0 = 0; t0 < slices; t0 += 4) {
            acc.et = acc.ep = acc.eq = acc.eqd = 0.0f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int t = t0 + i;
                if (t >= slices) // (the same for the whole warp)
                    break;
                float e[8];
                if constexpr (SMEM) {
                    const float4 a = wb[64 * t], b = wb[64 * t + 1];
                    e[0] = a.x, e[1] = a.y, e[2] = a.z, e[3] = a.w, e[4] = b.x, e[5] = b.y, e[6] = b.z, e[7] = b.w;
                } else {
                    float v[8];
                    load_logits<TL>(xr + 256 * t, v);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        v[j] = __fmul_rn(alpha, v[j]);
                    slice_exp(v, m, e);
                }
                typename Elem<__nv_bfloat16>::Raw raw;
                raw.v = p_chunk(e, rs, tiny);
                const ChunkOut o = make_out<__nv_bfloat16, PAT, FMT>(p, ob, row, 256 * t + 8 * lane, true, lane);
                process_chunk<__nv_bfloat16, PAT, kMag, FMT>(p, raw, o, c, acc);
            }
            e_total += acc.et;
            if constexpr (PAT != kDense)
                e_prune += acc.ep;
            if constexpr (FMT != kNone && PAT != kDense)
                e_q += acc.eq;
            if constexpr (FMT == kFp8 && PAT == kSparse24) {
                e_q += lo2(acc.eq2) + hi2(acc.eq2);
                acc.eq2 = 0ull;
            }
            if constexpr (FMT != kNone && PAT == kDense)
                e_qd += acc.eqd;
        }
    }
    const PassParams v = operand_view(pk);
    if (!v.energy_out)
        return;
    grid_reduce_energy(v, e_total, e_prune, e_q, e_qd, red, &flag, tid, lane, warp);
}

template <typename TL, int PAT, bool SMEM> const void *softmax_for_fmt(int fmt)
{
    switch (fmt) {
    case kNone:
        if constexpr (PAT != kDense)
            return reinterpret_cast<const void *>(&softmax_prune_kernel<TL, PAT, kNone, SMEM>);
        break;
    case kFp8:
        return reinterpret_cast<const void *>(&softmax_prune_kernel<TL, PAT, kFp8, SMEM>);
    case kInt:
        return reinterpret_cast<const void *>(&softmax_prune_kernel<TL, PAT, kInt, SMEM>);
    case kNvfp4:
        return reinterpret_cast<const void *>(&softmax_prune_kernel<TL, PAT, kNvfp4, SMEM>);
    case kMxfp4:
        return reinterpret_cast<const void *>(&softmax_prune_kernel<TL, PAT, kMxfp4, SMEM>);
    }
    return nullptr;
}

template <typename TL, bool SMEM> const void *softmax_for(int pattern, int fmt)
{
    return pattern == kDense      ? softmax_for_fmt<TL, kDense, SMEM>(fmt)
           : pattern == kSparse24 ? softmax_for_fmt<TL, kSparse24, SMEM>(fmt)
                                  : softmax_for_fmt<TL, kSparse48, SMEM>(fmt);
}

} // namespace

const void *softmax_prune_kernel_ptr(int bf16, int pattern, int fmt, bool smem)
{
    if (smem)
        return bf16 ? softmax_for<__nv_bfloat16, true>(pattern, fmt) : softmax_for<float, true>(pattern, fmt);
    return bf16 ? softmax_for<__nv_bfloat16, false>(pattern, fmt) : softmax_for<float, false>(pattern, fmt);
}

} // namespace ss24
