// The online pass (tile mode): one read of the operand, selection, quantization,
// stores and error energies, in a persistent warp-specialised kernel.
//
// Method: "Is 2:4 Sparsity Still Worth It? Semi-Structured Sparsity versus
// Quantization in LLM Inference" — intro (2:4 along the reduction axis), §2
// (scores, round-to-nearest), §3 (formats; a fused kernel that reads the input
// once and writes kept values and indices once), §4 (disjoint error energies),
// §6 (pairwise 4:8).
//
// Structure. The CTAs serving one operand of a batch own its tiles t = cta,
// cta + ctas_per_op, ... A tile is a TMA box of R rows x W columns of the operand (W a power of two
// <= 256 along k, out-of-range parts zero-filled). One producer lane streams
// tiles into a ring of kStages shared-memory stages (mbarrier full/empty
// pairs); 8 consumer warps each read 16-byte chunks of 8 consecutive elements
// from the stage, release it, then select / quantize / store from registers.
// A warp's 32 lanes hold 32 consecutive chunks of one tile row segment, so a
// quantization group (at most 256 input elements) is a power-of-two run of
// lanes reduced with xor shuffles. Energies are summed per chunk in binary32
// trees, accumulated per thread in binary64, reduced per CTA, and the last CTA
// to finish (a ticket counter) reduces the per-CTA partials in fixed order.
#pragma once

#include <type_traits>

#include "device.cuh"
#include "internal.cuh"

namespace ss24 {

// ---------------------------------------------------------------------------
// element access: a chunk is 8 consecutive elements of one row
// ---------------------------------------------------------------------------

template <typename T> struct Elem;

template <> struct Elem<__nv_bfloat16> {
    struct Raw {
        uint4 v;
    };
    static constexpr int kChunkBytes = 16;
    __device__ __forceinline__ static Raw load(const uint8_t *tile, int j)
    {
        Raw r;
        r.v = *reinterpret_cast<const uint4 *>(tile + j * 16);
        return r;
    }
    __device__ __forceinline__ static void unpack(const Raw &r, float (&x)[8])
    {
        const uint32_t w[4] = {r.v.x, r.v.y, r.v.z, r.v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = bf16_lo(w[i]);
            x[2 * i + 1] = bf16_hi(w[i]);
        }
    }
};

template <> struct Elem<float> {
    struct Raw {
        float4 a, b;
    };
    static constexpr int kChunkBytes = 32;
    __device__ __forceinline__ static Raw load(const uint8_t *tile, int j)
    {
        Raw r;
        r.a = *reinterpret_cast<const float4 *>(tile + j * 32);
        r.b = *reinterpret_cast<const float4 *>(tile + j * 32 + 16);
        return r;
    }
    __device__ __forceinline__ static void unpack(const Raw &r, float (&x)[8])
    {
        x[0] = r.a.x; x[1] = r.a.y; x[2] = r.a.z; x[3] = r.a.w;
        x[4] = r.b.x; x[5] = r.b.y; x[6] = r.b.z; x[7] = r.b.w;
    }
};

// ---------------------------------------------------------------------------
// quantizers of one chunk's values (VPC = 4 kept or 8 dense values); every
// lane of the warp calls them (group reductions shuffle across lanes)
// ---------------------------------------------------------------------------

// Where one chunk's results go: its first output value, its group's scale
// entry, its metadata byte (4:8: the byte of its pair of chunks, written by the
// even lane) and, for the Wanda score, the norms of its eight columns.
struct ChunkOut {
    uint8_t *val;
    uint8_t *scale;
    uint8_t *meta;
    const float *norms;
    bool valid;
    int lane;
};

template <int VPC> __device__ __forceinline__ float local_amax(const float (&v)[VPC])
{
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < VPC; ++i)
        m = fmaxf(m, fabsf(v[i]));
    return m;
}

__device__ __forceinline__ float group_amax(float m, int lanes)
{
    for (int off = 1; off < lanes; off <<= 1)
        m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
    return m;
}

// Sum of the squares of N packed pairs: one packed multiply, then packed fused
// multiply-adds, then the two lanes (binary32; the energies are sums compared
// within 1e-6 relative, and each term and partial sum is rounded once).
template <int N> __device__ __forceinline__ float sq_sum2(const f32x2 (&e)[N])
{
    f32x2 t = mul2(e[0], e[0]);
#pragma unroll
    for (int i = 1; i < N; ++i)
        t = fma2(e[i], e[i], t);
    return lo2(t) + hi2(t);
}

// Sum of (v - d)^2 over a chunk's values (packed differences, sq_sum2).
template <int VPC> __device__ __forceinline__ float err_energy(const float (&v)[VPC], const float (&d)[VPC])
{
    f32x2 e[VPC / 2];
#pragma unroll
    for (int i = 0; i < VPC / 2; ++i)
        e[i] = sub2(pack2(v[2 * i], v[2 * i + 1]), pack2(d[2 * i], d[2 * i + 1]));
    return sq_sum2<VPC / 2>(e);
}

// The same with the dequantized values given negated (dn = -d): the terms
// v + dn equal v - d, rounding included.
template <int VPC> __device__ __forceinline__ float err_energy_neg(const float (&v)[VPC], const float (&dn)[VPC])
{
    f32x2 e[VPC / 2];
#pragma unroll
    for (int i = 0; i < VPC / 2; ++i)
        e[i] = add2(pack2(v[2 * i], v[2 * i + 1]), pack2(dn[2 * i], dn[2 * i + 1]));
    return sq_sum2<VPC / 2>(e);
}

// True when the fast division applies to every value of a chunk or group
// whose largest magnitude is vmax: the scale is in [2^-60, 2^60] and no
// quotient can overflow (vmax * y < 2^126).
__device__ __forceinline__ bool quot_fast(const Recip &rc, float vmax)
{
    return rc.fast && __fmul_rn(vmax, rc.y) < 0x1p126f;
}

// Negated quotients -v / s of a chunk: neg_div_fast2 on the fast path,
// otherwise IEEE division; a zero scale gives negated zero quotients. Callers encode -q and flip the sign of the codes,
// which is exact because every rounding to a format is symmetric.
template <int VPC>
__device__ __forceinline__ void neg_quotients(const float (&v)[VPC], const Recip &rc, bool fast, float (&qn)[VPC])
{
    if (fast) {
#pragma unroll
        for (int i = 0; i < VPC / 2; ++i) {
            const f32x2 qq = neg_div_fast2(pack2(v[2 * i], v[2 * i + 1]), rc);
            qn[2 * i] = lo2(qq);
            qn[2 * i + 1] = hi2(qq);
        }
    } else {
#pragma unroll
        for (int i = 0; i < VPC; ++i)
            qn[i] = rc.b != 0.0f ? __fdiv_rn(-v[i], rc.b) : -0.0f;
    }
}

// A packed product rounded once, as fma(a, b, -0): RN(a b), sign of zero
// included. Products that feed an add or a subtract are written this way so
// that no code generator can contract them into the following operation (the
// readings round every product and every sum separately).
__device__ __forceinline__ f32x2 mul2_rn(f32x2 a, f32x2 b, float z)
{
    // z: a zero the code generator cannot see as a constant (it is computed
    // from run-time data), so the fused multiply-add is not rewritten as a
    // multiply and then merged with its consumer
    return fma2(a, b, pack2(z, z));
}

// Dequantized values code_value * s of a chunk (binary32 products).
template <int VPC>
__device__ __forceinline__ void scale_values(const float (&c)[VPC], float s, float (&d)[VPC])
{
    const f32x2 s2 = pack2(s, s);
    const float z = __fmul_rn(-0.0f, s); // -0 for the scales (s >= 0)
#pragma unroll
    for (int i = 0; i < VPC / 2; ++i) {
        const f32x2 r = mul2_rn(pack2(c[2 * i], c[2 * i + 1]), s2, z);
        d[2 * i] = lo2(r);
        d[2 * i + 1] = hi2(r);
    }
}

// FP8 E4M3, per-tensor scale s: code = E4M3(v / s); deq = E4M3(code) * s.
// With `guard` false the caller knows that no quotient can overflow (the scale
// was derived from the amax of the values quantized).
template <int VPC, bool STORE>
__device__ __forceinline__ float quant_fp8_as(const float (&v)[VPC], bool fast, const Recip &rc, const ChunkOut &o);

template <int VPC, bool STORE>
__device__ __forceinline__ float quant_fp8(const float (&v)[VPC], float vmax, const Recip &rc, bool guard,
                                           const ChunkOut &o)
{
    bool fast = rc.fast;
    if (guard)
        fast = quot_fast(rc, vmax);
    return quant_fp8_as<VPC, STORE>(v, fast, rc, o);
}

// quant_fp8 with the division path decided by the caller (fast: every
// quotient of the chunk is in range for neg_div_fast2).
template <int VPC, bool STORE>
__device__ __forceinline__ float quant_fp8_as(const float (&v)[VPC], bool fast, const Recip &rc, const ChunkOut &o)
{
    float qn[VPC], decn[VPC], dn[VPC];
    neg_quotients<VPC>(v, rc, fast, qn);
    // codes of -q, decoded as they come from the conversion: dn = -deq exactly
    uint16_t h[VPC / 2];
#pragma unroll
    for (int t = 0; t < VPC / 2; ++t) {
        h[t] = cvt_e4m3x2h(qn[2 * t], qn[2 * t + 1]);
        const float2 f = e4m3x2h_to_f32(h[t]);
        decn[2 * t] = f.x;
        decn[2 * t + 1] = f.y;
    }
    scale_values<VPC>(decn, rc.b, dn);
    uint32_t c[VPC / 4]; // the codes of q: the sign bits flipped back
#pragma unroll
    for (int t = 0; t < VPC / 4; ++t)
        c[t] = (static_cast<uint32_t>(h[2 * t]) | (static_cast<uint32_t>(h[2 * t + 1]) << 16)) ^ 0x80808080u;
    if (STORE && o.valid) {
        if constexpr (VPC == 4)
            *reinterpret_cast<uint32_t *>(o.val) = c[0];
        else
            *reinterpret_cast<uint2 *>(o.val) = make_uint2(c[0], c[1]);
    }
    return err_energy_neg<VPC>(v, dn);
}

// quant_fp8_as (STORE, fast division decided by the caller) that adds the
// squared errors to the packed chains acc2 instead of returning their sum:
// the same terms, summed in two chains across the tile's chunks.
template <int VPC>
__device__ __forceinline__ void quant_fp8_acc(const float (&v)[VPC], bool fast, const Recip &rc, const ChunkOut &o,
                                              f32x2 &acc2)
{
    float qn[VPC], decn[VPC], dn[VPC];
    neg_quotients<VPC>(v, rc, fast, qn);
    uint16_t h[VPC / 2];
#pragma unroll
    for (int t = 0; t < VPC / 2; ++t) {
        h[t] = cvt_e4m3x2h(qn[2 * t], qn[2 * t + 1]);
        const float2 f = e4m3x2h_to_f32(h[t]);
        decn[2 * t] = f.x;
        decn[2 * t + 1] = f.y;
    }
    scale_values<VPC>(decn, rc.b, dn);
    uint32_t c[VPC / 4];
#pragma unroll
    for (int t = 0; t < VPC / 4; ++t)
        c[t] = (static_cast<uint32_t>(h[2 * t]) | (static_cast<uint32_t>(h[2 * t + 1]) << 16)) ^ 0x80808080u;
    if (o.valid) {
        if constexpr (VPC == 4)
            *reinterpret_cast<uint32_t *>(o.val) = c[0];
        else
            *reinterpret_cast<uint2 *>(o.val) = make_uint2(c[0], c[1]);
    }
#pragma unroll
    for (int i = 0; i < VPC / 2; ++i) {
        const f32x2 e = add2(pack2(v[2 * i], v[2 * i + 1]), pack2(dn[2 * i], dn[2 * i + 1]));
        acc2 = fma2(e, e, acc2);
    }
}

// Integer rounding by the magic constant 1.5 * 2^23: for |q| < 2^22 the sum
// q + M rounds q to the nearest integer (ties to even) in its low mantissa
// bits, and (q + M) - M is that integer exactly.
constexpr float kMagic = 12582912.0f; // 1.5 * 2^23, bits 0x4B400000

// Symmetric INT-b, one fp32 scale per q.group quantized values (q.lanes
// lanes). row_amax >= 0 supplies the group amax (row mode: the whole row) and
// leaves the scale store to the caller. The scale comes from the group amax:
// for a normal scale |v / scale| <= qmax (1 + 2^-23), so the rounded code never
// leaves [-qmax, qmax] and the clamp of the definition is only needed on the
// IEEE-division path (scales outside [2^-60, 2^60]).
// The scale of an INT group, amax / qmax (qmax in [1, 32767]): Markstein's
// correction is exact for quotients >= 2^-40; tinier ones take the IEEE division.
__device__ __forceinline__ float int_scale(float amax, const QuantSpec &q)
{
    Recip rq;
    rq.b = q.qmax;
    rq.nb = -q.qmax;
    rq.y = q.qmax_inv;
    rq.fast = true;
    return amax >= 0x1p-25f ? div_fast(amax, rq) : __fdiv_rn(amax, q.qmax);
}

// A whole-row INT scale computed once by the caller (row kernels).
struct RowScale {
    bool given;
    float amax, scale;
    Recip rc;
    bool fast; // quot_fast(rc, amax)
};

template <int VPC, bool STORE>
__device__ __forceinline__ float quant_int(const float (&v)[VPC], float vmax, const QuantSpec &q, const ChunkOut &o,
                                           float row_amax = -1.0f, const RowScale *rs = nullptr,
                                           float gamax = -1.0f)
{
    float amax, scale;
    Recip rc;
    bool fast;
    if (rs && rs->given) {
        amax = rs->amax;
        scale = rs->scale;
        rc = rs->rc;
        fast = rs->fast;
    } else {
        amax = row_amax >= 0.0f ? row_amax : (gamax >= 0.0f ? gamax : group_amax(vmax, q.lanes));
        scale = int_scale(amax, q);
        rc = make_recip(scale);
        fast = quot_fast(rc, amax);
    }
    float qn[VPC];
    neg_quotients<VPC>(v, rc, fast, qn);
    if (!fast) {
        // a scale outside [2^-60, 2^60] (e.g. subnormal) can put |v / scale|
        // above qmax: apply the clamp of the definition
#pragma unroll
        for (int i = 0; i < VPC; ++i)
            qn[i] = fminf(fmaxf(qn[i], -q.qmax), q.qmax);
    }
    // M - (-q) = M + q rounds q to an integer (ties to even) held in the low
    // bits of the sum; (M + q) - M is that integer exactly
    float t[VPC], cf[VPC], d[VPC];
    const f32x2 m2 = pack2(kMagic, kMagic);
#pragma unroll
    for (int i = 0; i < VPC / 2; ++i) {
        const f32x2 tt = sub2(m2, pack2(qn[2 * i], qn[2 * i + 1]));
        const f32x2 cc = sub2(tt, m2);
        t[2 * i] = lo2(tt);
        t[2 * i + 1] = hi2(tt);
        cf[2 * i] = lo2(cc);
        cf[2 * i + 1] = hi2(cc);
    }
    scale_values<VPC>(cf, scale, d);
    if (STORE && o.valid) {
        uint32_t b[VPC]; // low bits of M + q hold the two's-complement code
#pragma unroll
        for (int i = 0; i < VPC; ++i)
            b[i] = __float_as_uint(t[i]);
        if (q.store == kInt8) {
            uint32_t w[VPC / 4];
#pragma unroll
            for (int k = 0; k < VPC / 4; ++k)
                w[k] = __byte_perm(__byte_perm(b[4 * k], b[4 * k + 1], 0x0040), __byte_perm(b[4 * k + 2], b[4 * k + 3], 0x0040),
                                   0x5410);
            if constexpr (VPC == 4)
                *reinterpret_cast<uint32_t *>(o.val) = w[0];
            else
                *reinterpret_cast<uint2 *>(o.val) = make_uint2(w[0], w[1]);
        } else if (q.store == kInt16) {
            uint32_t w[VPC / 2];
#pragma unroll
            for (int k = 0; k < VPC / 2; ++k)
                w[k] = __byte_perm(b[2 * k], b[2 * k + 1], 0x5410);
            if constexpr (VPC == 4)
                *reinterpret_cast<uint2 *>(o.val) = make_uint2(w[0], w[1]);
            else
                *reinterpret_cast<uint4 *>(o.val) = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
            uint32_t w = 0;
#pragma unroll
            for (int i = 0; i < VPC; ++i)
                w |= (b[i] & 0xfu) << (4 * i);
            if constexpr (VPC == 4)
                *reinterpret_cast<uint16_t *>(o.val) = static_cast<uint16_t>(w);
            else
                *reinterpret_cast<uint32_t *>(o.val) = w;
        }
        if (row_amax < 0.0f && !(rs && rs->given) && (o.lane & (q.lanes - 1)) == 0)
            *reinterpret_cast<float *>(o.scale) = scale;
    }
    return err_energy<VPC>(v, d);
}

template <int VPC> __device__ __forceinline__ uint32_t pack_e2m1(const float (&q)[VPC])
{
    if constexpr (VPC == 4)
        return cvt_e2m1x4(q[0], q[1], q[2], q[3]);
    else
        return cvt_e2m1x4(q[0], q[1], q[2], q[3]) | (cvt_e2m1x4(q[4], q[5], q[6], q[7]) << 16);
}

template <int VPC>
__device__ __forceinline__ void unpack_e2m1(uint32_t codes, float mult, float (&d)[VPC])
{
    float dec[VPC];
#pragma unroll
    for (int t = 0; t < VPC / 2; ++t) {
        const float2 f = e2m1x2_to_f32((codes >> (8 * t)) & 0xffu);
        dec[2 * t] = f.x;
        dec[2 * t + 1] = f.y;
    }
    scale_values<VPC>(dec, mult, d);
}

template <int VPC, bool STORE>
__device__ __forceinline__ void store_fp4(uint32_t codes, const ChunkOut &o)
{
    if (STORE && o.valid) {
        if constexpr (VPC == 4)
            *reinterpret_cast<uint16_t *>(o.val) = static_cast<uint16_t>(codes);
        else
            *reinterpret_cast<uint32_t *>(o.val) = codes;
    }
}

// NVFP4: block of 16 values (16 / VPC lanes), E4M3 block scale over a fp32
// tensor scale st.
// Per-CTA NVFP4 table over the 128 non-negative E4M3 block-scale codes c:
// den[c] = E4M3(c) * s_t (the block's divisor) and inv[c] = RN(1 / den[c]).
struct NvTable {
    const float *den, *inv;
};

// Fills den / inv (256 floats at `t`) for tensor scale st; threads 0..127.
__device__ __forceinline__ void build_nv_table(float *t, float st, int tid)
{
    if (tid < 128) {
        const float d = __fmul_rn(e4m3_to_f32(static_cast<uint32_t>(tid)), st);
        t[tid] = d;
        t[128 + tid] = d != 0.0f ? __frcp_rn(d) : 0.0f;
    }
}

// The E4M3 code of an NVFP4 block scale, E4M3((amax / 6) / st): two
// correctly rounded divisions, by Markstein's correction when both are in its
// exact range (zero amax included), else by IEEE division; one branch in the
// common case.
__device__ __forceinline__ uint32_t nv_block_code(float amax, const Recip &rst)
{
    const float st = rst.b;
    Recip r6;
    r6.b = 6.0f;
    r6.nb = -6.0f;
    r6.y = 0x1.555556p-3f; // RN(1/6)
    r6.fast = true;
    float a6 = div_fast(amax, r6);
    float bs = div_fast(a6, rst);
    const bool ok = (amax == 0.0f || amax >= 0x1p-30f) && rst.fast &&
                    (a6 == 0.0f || (a6 >= 0x1p-40f * st && __fmul_rn(a6, rst.y) < 0x1p126f));
    if (!ok) {
        a6 = __fdiv_rn(amax, 6.0f);
        bs = st != 0.0f ? __fdiv_rn(a6, st) : 0.0f;
    }
    return cvt_e4m3x2(bs, 0.0f) & 0xffu;
}

// A block's divisor and its reciprocal, when the caller computed them (the
// block scale byte is then stored by the caller too).
struct NvBlock {
    float den, inv;
};

template <int VPC, bool STORE>
__device__ __forceinline__ float quant_nvfp4(const float (&v)[VPC], float vmax, const Recip &rst,
                                             const ChunkOut &o, const NvTable &tb, float gamax = -1.0f,
                                             const NvBlock *blk = nullptr)
{
    constexpr int kLanes = 16 / VPC;
    uint32_t sb = 0;
    Recip rd;
    bool fast;
    if (blk) {
        // the block's owner took quot_fast once: a non-positive reciprocal
        // marks a block for the IEEE division
        rd.b = blk->den;
        rd.y = blk->inv;
        rd.nb = -rd.b;
        rd.fast = true;
        fast = blk->inv > 0.0f;
    } else {
        const float amax = gamax >= 0.0f ? gamax : group_amax(vmax, kLanes);
        sb = nv_block_code(amax, rst);
        rd.b = tb.den[sb];
        rd.y = tb.inv[sb];
        rd.nb = -rd.b;
        rd.fast = rd.b >= 0x1p-60f && rd.b <= 0x1p60f;
        fast = quot_fast(rd, amax);
    }
    const float denom = rd.b;
    float qn[VPC], d[VPC];
    neg_quotients<VPC>(v, rd, fast, qn);
    const uint32_t codes = pack_e2m1<VPC>(qn) ^ (VPC == 4 ? 0x8888u : 0x88888888u);
    unpack_e2m1<VPC>(codes, denom, d);
    store_fp4<VPC, STORE>(codes, o);
    if (STORE && !blk && o.valid && (o.lane & (kLanes - 1)) == 0)
        *o.scale = static_cast<uint8_t>(sb);
    return err_energy<VPC>(v, d);
}

// MXFP4: block of 32 values (32 / VPC lanes), power-of-two scale 2^e stored as
// the E8M0 byte e + 127; v / 2^e is computed as v * 2^-e (the same correctly
// rounded value, since both scale factors are exact powers of two).
template <int VPC, bool STORE>
__device__ __forceinline__ float quant_mxfp4(const float (&v)[VPC], float vmax, const ChunkOut &o,
                                             float gamax = -1.0f)
{
    constexpr int kLanes = 32 / VPC;
    const float amax = gamax >= 0.0f ? gamax : group_amax(vmax, kLanes);
    uint32_t byte = 0;
    float inv = 0.0f, mult = 0.0f;
    if (amax != 0.0f) {
        const int e = mx_shared_exponent(amax);
        byte = static_cast<uint32_t>(e + 127);
        inv = exp2_int(-e);
        mult = exp2_int(e);
    }
    float q[VPC], d[VPC];
    scale_values<VPC>(v, inv, q);
    const uint32_t codes = pack_e2m1<VPC>(q);
    unpack_e2m1<VPC>(codes, mult, d);
    store_fp4<VPC, STORE>(codes, o);
    if (STORE && o.valid && (o.lane & (kLanes - 1)) == 0)
        *o.scale = static_cast<uint8_t>(byte);
    return err_energy<VPC>(v, d);
}

// Runtime-dispatched quantizer without stores (the energy-only pass).
template <int VPC>
__device__ __forceinline__ float quant_energy_only(const float (&v)[VPC], float vmax, const QuantSpec &q,
                                                   const Recip &rst, bool guard, const NvTable &tb)
{
    const ChunkOut o{nullptr, nullptr, nullptr, nullptr, false, 0};
    switch (q.fmt) {
    case kFp8:
        return quant_fp8<VPC, false>(v, vmax, rst, guard, o);
    case kInt:
        return quant_int<VPC, false>(v, vmax, q, o);
    case kNvfp4:
        return quant_nvfp4<VPC, false>(v, vmax, rst, o, tb);
    case kMxfp4:
        return quant_mxfp4<VPC, false>(v, vmax, o);
    default:
        return 0.0f;
    }
}

// ---------------------------------------------------------------------------
// one chunk: score, select, quantize, store, energies
// ---------------------------------------------------------------------------

struct Acc {
    float et, ep, eq, eqd; // energies of the current tile (binary32)
    float amax_kept, amax_all;
    // FP8 of a packed 2:4 selection: the squared errors' two packed chains
    // over the tile (added to eq where the tile's energies are taken)
    f32x2 eq2 = 0ull;
};

// Per-CTA constants of a pass: the tensor scales (as reciprocals), the NVFP4
// tables, and whether a per-tensor FP8 quotient must be checked for overflow
// (a scale the caller gave; a scale derived from the amax never overflows).
struct PassConsts {
    Recip rst, rstd;
    NvTable tb, tbd;
    bool guard, guardd;
    uint32_t lim2; // FP8 with a given scale: bf16x2 of fast_limit(rst), see fp8_fast_limit
};

// The smallest bf16 magnitude m with RN(m * y) >= 2^126 for the reciprocal y
// of a per-tensor scale (+inf when no finite bf16 reaches it). RN(m * y) is
// non-decreasing in m, so a chunk's quotients all suit neg_div_fast2 (see
// quot_fast) exactly when every kept magnitude is below this limit.
__device__ __forceinline__ uint32_t fp8_fast_limit(const Recip &rc)
{
    uint32_t lo = 0u, hi = 0x7f80u; // f(lo) false, the answer in (lo, hi]
    while (hi - lo > 1u) {
        const uint32_t mid = (lo + hi) >> 1;
        if (__fmul_rn(__uint_as_float(mid << 16), rc.y) >= 0x1p126f)
            hi = mid;
        else
            lo = mid;
    }
    return hi | (hi << 16);
}

template <int SCORE>
__device__ __forceinline__ void scores(const float (&x)[8], const ChunkOut &o, float (&s)[8])
{
    if constexpr (SCORE == kWanda) {
        float4 n0 = make_float4(0.f, 0.f, 0.f, 0.f), n1 = n0;
        if (o.valid) {
            n0 = __ldg(reinterpret_cast<const float4 *>(o.norms));
            n1 = __ldg(reinterpret_cast<const float4 *>(o.norms + 4));
        }
        const float n[8] = {n0.x, n0.y, n0.z, n0.w, n1.x, n1.y, n1.z, n1.w};
#pragma unroll
        for (int i = 0; i < 8; ++i)
            s[i] = __fmul_rn(fabsf(x[i]), n[i]);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            s[i] = fabsf(x[i]);
    }
}

// The largest magnitude of a chunk's eight input values: packed bf16 lanes for
// bf16 operands, else from the unpacked values.
template <typename T>
__device__ __forceinline__ float chunk_amax(const typename Elem<T>::Raw &raw, const float (&x)[8])
{
    if constexpr (sizeof(T) == 2) {
        const uint4 w = raw.v;
        return bf16x2_hmax(bf16x2_maxabs(bf16x2_maxabs(w.x, w.y), bf16x2_maxabs(w.z, w.w)));
    } else {
        return local_amax<8>(x);
    }
}

// The selection half of a chunk: scores, the kept values (all values for the
// dense pattern), their largest magnitude, the metadata and the chunk's
// energies E_total and E_prune.
template <int VPC> struct Sel {
    float v[VPC];
    float vmax;
    uint32_t meta;
    uint32_t kept_bits[2]; // bf16 2:4 by magnitude: kept values as bf16x2 (group 0, group 1)
    uint32_t k0, k1;       // the same values as selected: lower-index kept value of each group, then the other
    float et, ep;
};

template <typename T, int PAT, int SCORE>
__device__ __forceinline__ Sel<PAT == kDense ? 8 : 4> select_chunk(const typename Elem<T>::Raw &raw,
                                                                   const ChunkOut &o)
{
    constexpr int VPC = PAT == kDense ? 8 : 4;
    // two groups of bf16 values selected by magnitude with packed lanes
    constexpr bool kPair = sizeof(T) == 2 && PAT == kSparse24 && SCORE == kMag;
    float x[8]; // (unused values are not computed)
    Elem<T>::unpack(raw, x);
    float v[VPC];
    float vmax;   // max |v| over the chunk's values to quantize
    uint32_t meta = 0;
    uint32_t kept_bits[2] = {0u, 0u};
    uint32_t kw0 = 0u, kw1 = 0u;
    float et, ep = 0.0f;

    if constexpr (PAT == kDense) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            v[i] = x[i];
        vmax = chunk_amax<T>(raw, x);
        f32x2 t[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            t[i] = pack2(x[2 * i], x[2 * i + 1]);
        et = sq_sum2<4>(t);
    } else if constexpr (kPair) {
        const uint4 w = raw.v;
        const Pair24 g = pair24_bf16(w.x, w.y, w.z, w.w);
        v[0] = bf16_lo(g.k0);
        v[1] = bf16_lo(g.k1);
        v[2] = bf16_hi(g.k0);
        v[3] = bf16_hi(g.k1);
        vmax = bf16x2_hmax(bf16x2_maxabs(g.k0, g.k1));
        kept_bits[0] = __byte_perm(g.k0, g.k1, 0x5410);
        kept_bits[1] = __byte_perm(g.k0, g.k1, 0x7632);
        kw0 = g.k0;
        kw1 = g.k1;
        meta = g.meta;
        et = g.e_all;
        ep = g.e_drop;
    } else if constexpr (PAT == kSparse24) {
        Group24 g0, g1;
        if constexpr (SCORE == kWanda) {
            float s[8];
            scores<SCORE>(x, o, s);
            g0 = group24<false>(x[0], x[1], x[2], x[3], s[0], s[1], s[2], s[3]);
            g1 = group24<false>(x[4], x[5], x[6], x[7], s[4], s[5], s[6], s[7]);
        } else {
            g0 = group24<true>(x[0], x[1], x[2], x[3], 0.f, 0.f, 0.f, 0.f);
            g1 = group24<true>(x[4], x[5], x[6], x[7], 0.f, 0.f, 0.f, 0.f);
        }
        v[0] = g0.k0;
        v[1] = g0.k1;
        v[2] = g1.k0;
        v[3] = g1.k1;
        vmax = local_amax<4>(v);
        meta = g0.nib | (g1.nib << 4);
        et = g0.e_all + g1.e_all;
        ep = g0.e_drop + g1.e_drop;
    } else {
        // pairwise 4:8: pair p ranked by s_2p^2 + s_2p+1^2 (each product and
        // the sum rounded); for the magnitude score these are also the
        // pairs' energies
        const float zq = __fmul_rn(-0.0f, fabsf(x[0])); // a run-time -0 (see mul2_rn)
        f32x2 a = mul2_rn(pack2(x[0], x[2]), pack2(x[0], x[2]), zq);
        f32x2 b = mul2_rn(pack2(x[1], x[3]), pack2(x[1], x[3]), zq);
        const f32x2 e01 = add2(a, b);
        a = mul2_rn(pack2(x[4], x[6]), pack2(x[4], x[6]), zq);
        b = mul2_rn(pack2(x[5], x[7]), pack2(x[5], x[7]), zq);
        const f32x2 e23 = add2(a, b);
        float e[4] = {lo2(e01), hi2(e01), lo2(e23), hi2(e23)};
        float rank[4] = {e[0], e[1], e[2], e[3]};
        if constexpr (SCORE == kWanda) {
            float s[8];
            scores<SCORE>(x, o, s);
            a = mul2_rn(pack2(s[0], s[2]), pack2(s[0], s[2]), zq);
            b = mul2_rn(pack2(s[1], s[3]), pack2(s[1], s[3]), zq);
            const f32x2 r01 = add2(a, b);
            a = mul2_rn(pack2(s[4], s[6]), pack2(s[4], s[6]), zq);
            b = mul2_rn(pack2(s[5], s[7]), pack2(s[5], s[7]), zq);
            const f32x2 r23 = add2(a, b);
            rank[0] = lo2(r01);
            rank[1] = hi2(r01);
            rank[2] = lo2(r23);
            rank[3] = hi2(r23);
        }
        // the tournament over the four pairs: kept first elements, kept second
        // elements, and (through e) the dropped pairs' energy
        const Group24 f = group24<false>(x[0], x[2], x[4], x[6], rank[0], rank[1], rank[2], rank[3]);
        const Group24 sc = group24<false>(x[1], x[3], x[5], x[7], rank[0], rank[1], rank[2], rank[3]);
        const Group24 en = group24<false>(e[0], e[1], e[2], e[3], rank[0], rank[1], rank[2], rank[3]);
        v[0] = f.k0;
        v[1] = sc.k0;
        v[2] = f.k1;
        v[3] = sc.k1;
        meta = f.nib;
        et = (e[0] + e[1]) + (e[2] + e[3]);
        ep = en.d0 + en.d1;
        vmax = local_amax<4>(v);
    }


    Sel<VPC> r;
#pragma unroll
    for (int i = 0; i < VPC; ++i)
        r.v[i] = v[i];
    r.vmax = vmax;
    r.meta = meta;
    r.kept_bits[0] = kept_bits[0];
    r.kept_bits[1] = kept_bits[1];
    r.k0 = kw0;
    r.k1 = kw1;
    r.et = et;
    r.ep = ep;
    return r;
}

// The rest of a chunk: metadata and value stores, quantization, energies.
// gamax >= 0: the group / block amax of the values to quantize, already
// reduced across the group's lanes by the caller.
template <typename T, int PAT, int SCORE, int FMT>
__device__ __forceinline__ void finish_chunk(const PassParams &p, const typename Elem<T>::Raw &raw,
                                             const Sel<PAT == kDense ? 8 : 4> &sl, const ChunkOut &o,
                                             const PassConsts &c, Acc &acc, float row_amax = -1.0f,
                                             const RowScale *rs = nullptr, float gamax = -1.0f,
                                             const NvBlock *blk = nullptr)
{
    constexpr int VPC = PAT == kDense ? 8 : 4;
    constexpr bool kPair = sizeof(T) == 2 && PAT == kSparse24 && SCORE == kMag;
    float x[8]; // (unused values are not computed)
    Elem<T>::unpack(raw, x);
    float v[VPC];
#pragma unroll
    for (int i = 0; i < VPC; ++i)
        v[i] = sl.v[i];
    const float vmax = sl.vmax;
    const uint32_t meta = sl.meta;
    const uint32_t kept_bits[2] = {sl.kept_bits[0], sl.kept_bits[1]};
    const float et = sl.et, ep = sl.ep;

    if constexpr (FMT == kAmax) {
        acc.amax_all = fmaxf(acc.amax_all, chunk_amax<T>(raw, x));
        if constexpr (PAT != kDense)
            acc.amax_kept = fmaxf(acc.amax_kept, vmax);
        return;
    }
    acc.et += et;
    acc.ep += ep;

    // metadata
    if constexpr (PAT == kSparse24) {
        if (FMT != kEnergy && o.valid)
            *o.meta = static_cast<uint8_t>(meta);
    } else if constexpr (PAT == kSparse48) {
        const uint32_t other = __shfl_down_sync(kFull, meta, 1);
        if (FMT != kEnergy && o.valid && (o.lane & 1) == 0)
            *o.meta = static_cast<uint8_t>(meta | (other << 4));
    }

    float eq = 0.0f;
    if constexpr (FMT == kNone) {
        if (o.valid) {
            if constexpr (kPair) {
                *reinterpret_cast<uint2 *>(o.val) = make_uint2(kept_bits[0], kept_bits[1]);
            } else if constexpr (sizeof(T) == 2) {
                const uint32_t w0 = (__float_as_uint(v[0]) >> 16) | (__float_as_uint(v[1]) & 0xffff0000u);
                const uint32_t w1 = (__float_as_uint(v[2]) >> 16) | (__float_as_uint(v[3]) & 0xffff0000u);
                *reinterpret_cast<uint2 *>(o.val) = make_uint2(w0, w1);
            } else {
                *reinterpret_cast<float4 *>(o.val) = make_float4(v[0], v[1], v[2], v[3]);
            }
        }
    } else if constexpr (FMT == kFp8) {
        if constexpr (kPair) {
            // the overflow guard as two packed comparisons of the kept values
            // with the CTA's limit (equivalent to quot_fast on their maximum)
            const bool fast = c.rst.fast && !(c.guard && bf16x2_max_ge_abs(sl.k0, sl.k1, c.lim2));
            quant_fp8_acc<VPC>(v, fast, c.rst, o, acc.eq2);
        } else {
            eq = quant_fp8<VPC, true>(v, vmax, c.rst, c.guard, o);
        }
    } else if constexpr (FMT == kInt || FMT == kIntRows) {
        eq = quant_int<VPC, true>(v, vmax, p.q, o, row_amax, rs, gamax);
    } else if constexpr (FMT == kNvfp4) {
        eq = quant_nvfp4<VPC, true>(v, vmax, c.rst, o, c.tb, gamax, blk);
    } else if constexpr (FMT == kMxfp4) {
        eq = quant_mxfp4<VPC, true>(v, vmax, o, gamax);
    } else if constexpr (FMT == kEnergy) {
        eq = quant_energy_only<VPC>(v, vmax, p.q, c.rst, c.guard, c.tb);
        acc.eqd += quant_energy_only<8>(x, chunk_amax<T>(raw, x), p.qd, c.rstd, c.guardd, c.tbd);
    }
    if constexpr (PAT == kDense)
        acc.eqd += eq;
    else
        acc.eq += eq;
}

template <typename T, int PAT, int SCORE, int FMT>
__device__ __forceinline__ void process_chunk(const PassParams &p, const typename Elem<T>::Raw &raw,
                                              const ChunkOut &o, const PassConsts &c, Acc &acc,
                                              float row_amax = -1.0f, const RowScale *rs = nullptr)
{
    const auto sl = select_chunk<T, PAT, SCORE>(raw, o);
    finish_chunk<T, PAT, SCORE, FMT>(p, raw, sl, o, c, acc, row_amax, rs);
}

// Dense INT-b codes of one chunk with its row's scale, straight-line on
// binary32 pairs: the same operations, roundings and summation order as
// quant_int / err_energy and the dense energy in select_chunk, with the code
// width (STORE) and the fast-division decision (FAST, one per row) fixed.
template <typename T, int STORE, bool FAST>
__device__ __forceinline__ void dense_int_chunk(const typename Elem<T>::Raw &raw, const RowScale &rs, float qmax,
                                                uint8_t *val, bool valid, Acc &acc)
{
    float x[8];
    Elem<T>::unpack(raw, x);
    f32x2 x2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        x2[i] = pack2(x[2 * i], x[2 * i + 1]);
    acc.et += sq_sum2<4>(x2);
    const f32x2 m2 = pack2(kMagic, kMagic), s2 = pack2(rs.scale, rs.scale);
    f32x2 tt[4], e[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f32x2 qn;
        if constexpr (FAST) {
            qn = neg_div_fast2(x2[i], rs.rc);
        } else {
            float a = rs.rc.b != 0.0f ? __fdiv_rn(-x[2 * i], rs.rc.b) : -0.0f;
            float b = rs.rc.b != 0.0f ? __fdiv_rn(-x[2 * i + 1], rs.rc.b) : -0.0f;
            qn = pack2(fminf(fmaxf(a, -qmax), qmax), fminf(fmaxf(b, -qmax), qmax));
        }
        tt[i] = sub2(m2, qn);
        const f32x2 d = mul2_rn(sub2(tt[i], m2), s2, __fmul_rn(-0.0f, rs.scale));
        e[i] = sub2(x2[i], d);
    }
    acc.eqd += sq_sum2<4>(e);
    if (valid) {
        uint32_t b[8]; // low bits of M + q hold the two's-complement code
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            b[2 * i] = __float_as_uint(lo2(tt[i]));
            b[2 * i + 1] = __float_as_uint(hi2(tt[i]));
        }
        if constexpr (STORE == kInt8) {
            *reinterpret_cast<uint2 *>(val) =
                make_uint2(__byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410),
                           __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040), 0x5410));
        } else if constexpr (STORE == kInt16) {
            *reinterpret_cast<uint4 *>(val) = make_uint4(__byte_perm(b[0], b[1], 0x5410), __byte_perm(b[2], b[3], 0x5410),
                                                         __byte_perm(b[4], b[5], 0x5410), __byte_perm(b[6], b[7], 0x5410));
        } else {
            uint32_t w = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i)
                w |= (b[i] & 0xfu) << (4 * i);
            *reinterpret_cast<uint32_t *>(val) = w;
        }
    }
}

// The CPT chunks of a thread in one row (dense operand), chunk j at val0 + j * cval.
template <typename T, int CPT, int STORE, bool FAST>
__device__ __forceinline__ void dense_int_row(const typename Elem<T>::Raw (&raw)[CPT], const RowScale &rs, float qmax,
                                              uint8_t *val0, int64_t cval, int t, int tpr, int nchunks, bool rv,
                                              Acc &acc)
{
#pragma unroll
    for (int j = 0; j < CPT; ++j)
        dense_int_chunk<T, STORE, FAST>(raw[j], rs, qmax, val0 + j * cval, rv && t + j * tpr < nchunks, acc);
}

// ---------------------------------------------------------------------------
// kernel
// ---------------------------------------------------------------------------

__device__ __forceinline__ void record_error(int32_t *err, int32_t code)
{
    atomicCAS(err, 0, code);
}

// The parameters as seen by the CTAs serving one operand of a batch: every
// per-operand pointer offset to that operand, and the CTA's index among the
// operand's CTAs.
__device__ __forceinline__ PassParams operand_view(const PassParams &p)
{
    PassParams q = p;
    const int b = static_cast<int>(blockIdx.x) / p.ctas_per_op;
    q.op = b;
    q.cta = static_cast<int>(blockIdx.x) - b * p.ctas_per_op;
    if (p.values)
        q.values = static_cast<uint8_t *>(p.values) + b * p.values_bstride;
    if (p.scales)
        q.scales = static_cast<uint8_t *>(p.scales) + b * p.scales_bstride;
    if (p.meta)
        q.meta = p.meta + b * p.meta_bstride;
    if (p.energy_out)
        q.energy_out = p.energy_out + 4 * b;
    if (p.amax_user)
        q.amax_user = p.amax_user + b;
    q.energy_partials = p.energy_partials + 4 * static_cast<int64_t>(b) * p.ctas_per_op;
    q.amax_partials = p.amax_partials + 2 * static_cast<int64_t>(b) * p.ctas_per_op;
    q.amax_out = p.amax_out + 2 * b;
    q.energy_ticket = p.energy_ticket + b;
    q.amax_ticket = p.amax_ticket + b;
    QuantSpec *qs[2] = {&q.q, &q.qd};
    for (int i = 0; i < 2; ++i) {
        if (qs[i]->scale_in)
            qs[i]->scale_in += b;
        if (qs[i]->scale_out)
            qs[i]->scale_out += b;
        if (qs[i]->amax_reduced)
            qs[i]->amax_reduced += 2 * b;
    }
    return q;
}

// Tensor scale of a per-tensor format: the given one, or amax / divisor.
__device__ __forceinline__ float tensor_scale(const QuantSpec &q)
{
    if (q.fmt != kFp8 && q.fmt != kNvfp4)
        return 0.0f;
    if (q.scale_in)
        return *q.scale_in;
    return __fdiv_rn(*q.amax_reduced, q.divisor);
}

// Energy reduction over the CTAs of one operand: per-CTA binary64 partials go
// to the workspace; the CTA that takes the operand's last ticket sums them in
// fixed order, writes the caller's 4-double record and resets the ticket.
// Called by all consumers, with the operand's view of the parameters.
__device__ __forceinline__ void grid_reduce_energy(const PassParams &p, double e_total, double e_prune, double e_q,
                                                   double e_qd, double *red, uint32_t *flag, int tid, int lane,
                                                   int warp)
{
    double e[4] = {e_total, e_prune, e_q, e_qd};
#pragma unroll
    for (int f = 0; f < 4; ++f)
        for (int off = 16; off >= 1; off >>= 1)
            e[f] += __shfl_xor_sync(kFull, e[f], off);
    if (lane == 0)
#pragma unroll
        for (int f = 0; f < 4; ++f)
            red[warp * 4 + f] = e[f];
    named_barrier_sync(1, kConsumers);
    if (tid == 0) {
        double sum[4] = {0.0, 0.0, 0.0, 0.0};
        for (int w = 0; w < kConsumerWarps; ++w)
#pragma unroll
            for (int f = 0; f < 4; ++f)
                sum[f] += red[w * 4 + f];
#pragma unroll
        for (int f = 0; f < 4; ++f)
            p.energy_partials[p.cta * 4 + f] = sum[f];
        __threadfence();
        const uint32_t ticket = atomicAdd(p.energy_ticket, 1u);
        *flag = ticket == static_cast<uint32_t>(p.ctas_per_op - 1);
    }
    named_barrier_sync(1, kConsumers);
    if (*flag) {
        __threadfence();
        // thread tid sums field (tid & 3) over CTAs (tid >> 2), (tid >> 2) + 64, ...
        const int f = tid & 3;
        double acc_f = 0.0;
        for (int i = tid >> 2; i < p.ctas_per_op; i += kConsumers / 4)
            acc_f += __ldcg(p.energy_partials + 4 * i + f);
        // lanes holding the same field differ in lane bits 2..4
        for (int off = 16; off >= 4; off >>= 1)
            acc_f += __shfl_xor_sync(kFull, acc_f, off);
        named_barrier_sync(1, kConsumers);
        if (lane < 4)
            red[warp * 4 + lane] = acc_f;
        named_barrier_sync(1, kConsumers);
        if (tid < 4) {
            double total = 0.0;
            for (int w = 0; w < kConsumerWarps; ++w)
                total += red[w * 4 + tid];
            p.energy_out[tid] = total;
        }
        if (tid == 0)
            *p.energy_ticket = 0;
    }
}

// Amax reduction over the CTAs of one operand, of the kept values (a) and of
// all values (b): the same last-CTA scheme as the energies. Writes amax_out[0]
// (the amax of the values the pass quantizes), amax_out[1] (all values) and,
// when asked, the caller's amax and the per-tensor scale amax / divisor.
template <int PAT>
__device__ __forceinline__ void grid_reduce_amax(const PassParams &p, float a, float b, float *fred, uint32_t *flag,
                                                 int tid, int lane, int warp)
{
    for (int off = 16; off >= 1; off >>= 1) {
        a = fmaxf(a, __shfl_xor_sync(kFull, a, off));
        b = fmaxf(b, __shfl_xor_sync(kFull, b, off));
    }
    if (lane == 0) {
        fred[warp * 2] = a;
        fred[warp * 2 + 1] = b;
    }
    named_barrier_sync(1, kConsumers);
    if (tid == 0) {
        for (int w = 1; w < kConsumerWarps; ++w) {
            a = fmaxf(a, fred[w * 2]);
            b = fmaxf(b, fred[w * 2 + 1]);
        }
        p.amax_partials[p.cta * 2] = a;
        p.amax_partials[p.cta * 2 + 1] = b;
        __threadfence();
        const uint32_t ticket = atomicAdd(p.amax_ticket, 1u);
        *flag = ticket == static_cast<uint32_t>(p.ctas_per_op - 1);
    }
    named_barrier_sync(1, kConsumers);
    if (*flag) {
        __threadfence();
        float ka = 0.0f, kb = 0.0f;
        for (int i = tid; i < p.ctas_per_op; i += kConsumers) {
            ka = fmaxf(ka, __ldcg(p.amax_partials + 2 * i));
            kb = fmaxf(kb, __ldcg(p.amax_partials + 2 * i + 1));
        }
        for (int off = 16; off >= 1; off >>= 1) {
            ka = fmaxf(ka, __shfl_xor_sync(kFull, ka, off));
            kb = fmaxf(kb, __shfl_xor_sync(kFull, kb, off));
        }
        named_barrier_sync(1, kConsumers);
        if (lane == 0) {
            fred[warp * 2] = ka;
            fred[warp * 2 + 1] = kb;
        }
        named_barrier_sync(1, kConsumers);
        if (tid == 0) {
            for (int w = 1; w < kConsumerWarps; ++w) {
                ka = fmaxf(ka, fred[w * 2]);
                kb = fmaxf(kb, fred[w * 2 + 1]);
            }
            const float a0 = PAT == kDense ? kb : ka;
            p.amax_out[0] = a0;
            p.amax_out[1] = kb;
            if (p.amax_user)
                *p.amax_user = a0;
            if (p.q.scale_out)
                *p.q.scale_out = __fdiv_rn(a0, p.q.divisor);
            *p.amax_ticket = 0;
        }
    }
}

__device__ __forceinline__ void producer(const CUtensorMap *map, const PassParams &p, uint8_t *stages,
                                         uint64_t *full, uint64_t *empty)
{
    const uint64_t policy = l2_evict_first_policy();
    uint32_t it = 0;
    bool failed = false;
    for (int64_t t = p.cta; t < p.n_tiles; t += p.ctas_per_op, ++it) {
        const int s = it % kStages;
        const uint32_t use = it / kStages;
        if (p.test_skip_tile >= 0 && p.op == 0 && p.cta == 0 && it == static_cast<uint32_t>(p.test_skip_tile)) {
            // test hook: this tile is never copied, so its consumers' wait runs
            // out; nothing more is issued, and the copies already issued are
            // drained below
            failed = true;
            break;
        }
        if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1, p.wait_limit_ns)) {
            record_error(p.err, 1);
            failed = true;
            break;
        }
        mbar_arrive_expect_tx(&full[s], p.tile_bytes);
        const int64_t rt = t / p.n_col_tiles, ct = t - rt * p.n_col_tiles;
        const int32_t ck = static_cast<int32_t>(ct * p.W), cr = static_cast<int32_t>(rt * p.R);
        // TMA coordinates are {inner (contiguous), outer, operand}
        if (p.axis == 1)
            tma_load_3d(stages + s * kStageBytes, map, ck, cr, p.op, &full[s], policy);
        else
            tma_load_3d(stages + s * kStageBytes, map, cr, ck, p.op, &full[s], policy);
    }
    if (failed) {
        // let the copies already issued land before the CTA can exit
        for (int s = 0; s < kStages && s < static_cast<int>(it); ++s) {
            const uint32_t last_use = (it - 1 - ((it - 1 - s) % kStages)) / kStages;
            (void)mbar_wait(&full[s], last_use & 1, p.wait_limit_ns);
        }
    }
}

// Output pointers of the chunk at (row, col) (col: first input column of the
// chunk); nothing is dereferenced unless `valid`.
// Output base pointers of one operand of a batch.
struct OutBase {
    uint8_t *values, *scales, *meta;
};

__device__ __forceinline__ OutBase out_base(const PassParams &pk, int op)
{
    OutBase b;
    b.values = static_cast<uint8_t *>(pk.values) + op * pk.values_bstride;
    b.scales = static_cast<uint8_t *>(pk.scales) + op * pk.scales_bstride;
    b.meta = pk.meta + op * pk.meta_bstride;
    return b;
}

template <typename T, int PAT, int FMT>
__device__ __forceinline__ ChunkOut make_out(const PassParams &p, const OutBase &ob, int64_t row, int64_t col,
                                             bool valid, int lane)
{
    const int64_t n = PAT == kDense ? p.k : p.k / 2;
    const int64_t colq = PAT == kDense ? col : col / 2;
    const int64_t off = row * n + colq; // index of the chunk's first quantized value
    uint8_t *vals = ob.values;
    uint8_t *sc = ob.scales;
    ChunkOut o{nullptr, nullptr, nullptr, nullptr, valid, lane};
    if constexpr (FMT == kNone) {
        o.val = vals + off * static_cast<int64_t>(sizeof(T));
    } else if constexpr (FMT == kFp8) {
        o.val = vals + off;
    } else if constexpr (FMT == kInt || FMT == kIntRows) {
        o.val = vals + (p.q.store == kInt8 ? off : (p.q.store == kInt16 ? 2 * off : off / 2));
        const int lg = __ffs(p.q.group) - 1; // tile-mode groups are powers of two
        o.scale = sc + 4 * (row * (n >> lg) + (colq >> lg));
    } else if constexpr (FMT == kNvfp4) {
        o.val = vals + off / 2;
        o.scale = sc + row * (n / 16) + colq / 16;
    } else if constexpr (FMT == kMxfp4) {
        o.val = vals + off / 2;
        o.scale = sc + row * (n / 32) + colq / 32;
    }
    if constexpr (PAT == kSparse24 && FMT != kAmax && FMT != kEnergy)
        o.meta = ob.meta + row * (p.k / 8) + col / 8;
    else if constexpr (PAT == kSparse48 && FMT != kAmax && FMT != kEnergy)
        o.meta = ob.meta + row * (p.k / 16) + col / 16;
    if (p.norms)
        o.norms = p.norms + col;
    return o;
}

// make_out for kernels whose parameters are already an operand's view.
template <typename T, int PAT, int FMT>
__device__ __forceinline__ ChunkOut make_out(const PassParams &p, int64_t row, int64_t col, bool valid, int lane)
{
    const OutBase ob{static_cast<uint8_t *>(p.values), static_cast<uint8_t *>(p.scales), p.meta};
    return make_out<T, PAT, FMT>(p, ob, row, col, valid, lane);
}

// Tensor scales, reciprocals and NVFP4 tables of a pass (every thread of the
// CTA calls it; `nvt` is 512 floats of shared memory for the tables).
template <int FMT>
__device__ __forceinline__ PassConsts make_consts(const PassParams &p, int tid, int nthreads, float *nvt)
{
    float st = 0.0f, std_ = 0.0f;
    if constexpr (FMT == kFp8 || FMT == kNvfp4 || FMT == kEnergy) {
        st = tensor_scale(p.q);
        if (p.cta == 0 && tid == 0 && p.q.scale_out)
            *p.q.scale_out = st;
    }
    if constexpr (FMT == kEnergy)
        std_ = tensor_scale(p.qd);
    PassConsts c;
    c.rst = make_recip(st);
    c.rstd = make_recip(std_);
    c.guard = p.q.scale_in != nullptr;
    c.guardd = p.qd.scale_in != nullptr;
    c.lim2 = 0x7f807f80u;
    if constexpr (FMT == kFp8)
        if (c.guard)
            c.lim2 = fp8_fast_limit(c.rst);
    c.tb = NvTable{nvt, nvt + 128};
    c.tbd = NvTable{nvt + 256, nvt + 384};
    if constexpr (FMT == kNvfp4 || FMT == kEnergy) {
        build_nv_table(nvt, st, tid);
        build_nv_table(nvt + 256, std_, tid);
        named_barrier_sync(1, nthreads);
    }
    return c;
}

// 16-byte global load that bypasses L1 (each input byte is read once),
// predicated: zeros and no memory access when !ok (no branch).
__device__ __forceinline__ uint4 ld_stream(const void *p, bool ok)
{
    uint4 r = make_uint4(0u, 0u, 0u, 0u);
    asm volatile("{\n"
                 " .reg .pred q;\n"
                 " setp.ne.b32 q, %5, 0;\n"
                 " @q ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];\n"
                 "}\n"
                 : "+r"(r.x), "+r"(r.y), "+r"(r.z), "+r"(r.w)
                 : "l"(p), "r"(static_cast<int>(ok)));
    return r;
}

// 32-byte global load (two 16-byte halves) that bypasses L1, predicated like
// ld_stream; p must be 32-byte aligned. A warp's 32 loads then cover whole
// 32-byte sectors, where 16-byte loads 32 or 64 bytes apart would fetch each
// sector twice.
__device__ __forceinline__ void ld_stream32(const void *p, bool ok, uint4 &a, uint4 &b)
{
    a = make_uint4(0u, 0u, 0u, 0u);
    b = a;
    asm volatile("{\n"
                 " .reg .pred q;\n"
                 " setp.ne.b32 q, %9, 0;\n"
                 " @q ld.global.nc.L1::no_allocate.v8.u32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n"
                 "}\n"
                 : "+r"(a.x), "+r"(a.y), "+r"(a.z), "+r"(a.w), "+r"(b.x), "+r"(b.y), "+r"(b.z), "+r"(b.w)
                 : "l"(p), "r"(static_cast<int>(ok)));
}

// 32-byte global store; p must be 32-byte aligned.
__device__ __forceinline__ void st32(void *p, const uint4 &a, const uint4 &b)
{
    asm volatile("st.global.v8.u32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x), "r"(a.y), "r"(a.z),
                 "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
}

template <typename T> struct Stream;
template <> struct Stream<__nv_bfloat16> {
    __device__ __forceinline__ static Elem<__nv_bfloat16>::Raw load(const __nv_bfloat16 *p, bool ok)
    {
        Elem<__nv_bfloat16>::Raw r;
        r.v = ld_stream(p, ok);
        return r;
    }
};
template <> struct Stream<float> {
    __device__ __forceinline__ static Elem<float>::Raw load(const float *p, bool ok)
    {
        Elem<float>::Raw r;
        const uint4 a = ld_stream(p, ok);
        const uint4 b = ld_stream(p + 4, ok);
        r.a = make_float4(__uint_as_float(a.x), __uint_as_float(a.y), __uint_as_float(a.z), __uint_as_float(a.w));
        r.b = make_float4(__uint_as_float(b.x), __uint_as_float(b.y), __uint_as_float(b.z), __uint_as_float(b.w));
        return r;
    }
};

// Resident CTAs per SM the stream kernel is compiled for (register budget).
// (Four CTAs where the kernel fits 64 registers without spilling, else three.)
template <typename T, int PAT, int SCORE, int FMT, bool FW, bool ROT = false> struct StreamOcc {
    // (INT holds four selected chunks across its group reduction; a rotated
    // pass holds its rotation's temporaries)
    static constexpr bool light =
        !ROT && (FMT == kAmax || (sizeof(T) == 2 && SCORE == kMag && PAT != kSparse48 &&
                                  (FMT == kNone || FMT == kMxfp4 || (FMT == kFp8 && (FW || PAT == kDense)))));
    static constexpr int value = light ? 4 : 3;
};

// Block Hadamard rotation, in place, of the bf16 chunk a lane holds, for
// rotated passes. The lanes of a warp hold consecutive chunks of a row
// segment, so the partner of a butterfly of stride h >= 8 is lane ^ (h / 8).
// Binary32 arithmetic in stage order h = 1, 2, 4, ..., b/2: inside the lane
// packed adds and subtracts of the pairs (y_i, y_i+h); across lanes
// own * (+-1) + partner, which is exactly the rounded y_i + y_i+h (lower lane)
// or y_i - y_i+h (upper lane); then times RN(1/sqrt(b)) and rounded to bf16
// (nearest even). The whole warp calls it.
__device__ __forceinline__ void rotate_chunk(uint4 &w, int log2b, float cb, int lane)
{
    float y[8];
    const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        y[2 * i] = __uint_as_float(ws[i] << 16);
        y[2 * i + 1] = __uint_as_float(ws[i] & 0xffff0000u);
    }
#pragma unroll
    for (int s = 0; s < 3; ++s) {
        if (s >= log2b)
            break;
        const int h = 1 << s;
#pragma unroll
        for (int i0 = 0; i0 < 8; i0 += 2 * h) {
            if (h == 1 && (i0 & 2))
                continue; // (stride 1 pairs two butterflies 2 apart)
#pragma unroll
            for (int j = 0; j < (h == 1 ? 1 : h); j += 2) {
                const int a = h == 1 ? i0 : i0 + j, b = h == 1 ? i0 + 2 : i0 + j + 1;
                const f32x2 lo = pack2(y[a], y[b]), hi = pack2(y[a + h], y[b + h]);
                const f32x2 sm = add2(lo, hi), df = sub2(lo, hi);
                y[a] = lo2(sm), y[b] = hi2(sm), y[a + h] = lo2(df), y[b + h] = hi2(df);
            }
        }
    }
    for (int s = 3; s < log2b; ++s) {
        const int m = 1 << (s - 3);
        const float sg = (lane & m) ? -1.0f : 1.0f;
        const f32x2 sg2 = pack2(sg, sg);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
            const float o0 = __shfl_xor_sync(kFull, y[i], m);
            const float o1 = __shfl_xor_sync(kFull, y[i + 1], m);
            const f32x2 r = fma2(pack2(y[i], y[i + 1]), sg2, pack2(o0, o1));
            y[i] = lo2(r), y[i + 1] = hi2(r);
        }
    }
    uint32_t o[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 h2 = __floats2bfloat162_rn(__fmul_rn(y[2 * i], cb), __fmul_rn(y[2 * i + 1], cb));
        o[i] = *reinterpret_cast<const uint32_t *>(&h2);
    }
    w = make_uint4(o[0], o[1], o[2], o[3]);
}

// Byte advance of each output between consecutive slots of a full-width unit
// (slots 256 input columns apart); -1 where it depends on runtime fields (INT
// code width and group).
template <typename T, int PAT, int FMT> struct FwStep {
    static constexpr int64_t q = PAT == kDense ? 256 : 128; // quantized values per slot
    static constexpr int64_t val = FMT == kNone   ? q * static_cast<int64_t>(sizeof(T))
                                   : FMT == kFp8  ? q
                                   : (FMT == kNvfp4 || FMT == kMxfp4) ? q / 2
                                                  : -1;
    static constexpr int64_t scale = FMT == kNvfp4 ? q / 16 : FMT == kMxfp4 ? q / 32 : -1;
    static constexpr int64_t meta = PAT == kSparse24 ? 32 : PAT == kSparse48 ? 16 : 0;
};

// The largest magnitude among a chunk's values a pass quantizes (all values
// for the dense pattern, the kept ones otherwise).
template <typename T, int PAT, int SCORE>
__device__ __forceinline__ float quantized_amax(const typename Elem<T>::Raw &raw, const ChunkOut &o)
{
    if constexpr (PAT == kDense || (PAT == kSparse24 && SCORE == kMag)) {
        float xv[8];
        Elem<T>::unpack(raw, xv);
        return chunk_amax<T>(raw, xv);
    } else {
        return select_chunk<T, PAT, SCORE>(raw, o).vmax;
    }
}

// A full-width unit of the amax pass, wholly inside the operand: the amax of
// all values and of the kept values into acc, and the lane's largest
// quantized magnitude returned (for the row amax).
template <typename T, int PAT, int SCORE, bool ROT = false>
__device__ __forceinline__ float amax_unit_fw(const PassParams &p, const T *xp, const ChunkOut &o, Acc &acc)
{
    typename Elem<T>::Raw raw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        raw[i] = Stream<T>::load(xp + i * 256, true);
    if constexpr (ROT) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            rotate_chunk(raw[i].v, p.rot_log2b, p.rot_scale, static_cast<int>(threadIdx.x & 31));
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float xv[8];
        Elem<T>::unpack(raw[i], xv);
        const float all = chunk_amax<T>(raw[i], xv);
        acc.amax_all = fmaxf(acc.amax_all, all);
        if constexpr (PAT == kDense) {
            m = fmaxf(m, all);
        } else {
            ChunkOut oi = o;
            if constexpr (SCORE == kWanda)
                oi.norms = o.norms + i * 256;
            // (2:4 by magnitude keeps every group's largest value; pairwise 4:8
            // can drop it: its pair may rank third)
            const float kept = (PAT == kSparse24 && SCORE == kMag) ? all : select_chunk<T, PAT, SCORE>(raw[i], oi).vmax;
            acc.amax_kept = fmaxf(acc.amax_kept, kept);
            m = fmaxf(m, kept);
        }
    }
    return m;
}

// One unit: four 16-byte loads per lane first, then the four chunks. FULL:
// every chunk of the unit lies inside the operand (no per-chunk checks).
template <typename T, int PAT, int SCORE, int FMT, bool FULL, bool ROT = false>
__device__ __forceinline__ void stream_unit(const PassParams &p, const PassConsts &c, const T *xp, int64_t step_x,
                                            int64_t step_c, const ChunkOut &o, int64_t dval, int64_t dscale,
                                            int64_t dmeta, int64_t row0, int64_t col0, Acc &acc,
                                            float *rowa = nullptr, const float *rowa_in = nullptr,
                                            float *rscales = nullptr)
{
    using E = Elem<T>;
    typename E::Raw raw[4];
    bool ok[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        ok[i] = FULL || (row0 + i * p.step_rows < p.rows && col0 + i * p.step_cols < p.k);
        raw[i] = Stream<T>::load(xp + i * step_x, ok[i]);
    }
    if constexpr (ROT) {
        // (a chunk outside the operand is zero, and so is its whole block: k is
        // a multiple of the block and blocks never straddle rows)
#pragma unroll
        for (int i = 0; i < 4; ++i)
            rotate_chunk(raw[i].v, p.rot_log2b, p.rot_scale, static_cast<int>(threadIdx.x & 31));
    }
    auto out_i = [&](int i) {
        ChunkOut oi = o;
        oi.val += i * dval;
        oi.scale += i * dscale;
        oi.meta += i * dmeta;
        if constexpr (SCORE == kWanda)
            oi.norms = o.norms + i * step_c;
        oi.valid = ok[i];
        return oi;
    };
    const int lane = static_cast<int>(threadIdx.x & 31);
    if constexpr (FMT == kIntRows) {
        {
            // one scale per row from the given row amax: the chunks' rows are
            // row0 + i * step_rows; the first lane of a row's first segment
            // stores the row's scale
            if constexpr (PAT == kDense) {
                if (p.step_rows == 0) {
                    // one row for the whole unit: one scale, the straight-line
                    // chunk quantizer with the code width fixed
                    const bool rv = row0 < p.rows;
                    RowScale rs;
                    rs.given = true;
                    rs.amax = rv ? rowa_in[row0] : 0.0f;
                    rs.scale = int_scale(rs.amax, p.q);
                    rs.rc = make_recip(rs.scale);
                    rs.fast = quot_fast(rs.rc, rs.amax);
                    const float qm = p.q.qmax;
                    auto run = [&](auto store_tag, auto fast_tag) {
                        constexpr int S = decltype(store_tag)::value;
                        constexpr bool F = decltype(fast_tag)::value;
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            dense_int_chunk<T, S, F>(raw[i], rs, qm, o.val + i * dval, ok[i], acc);
                    };
                    using I8 = std::integral_constant<int, kInt8>;
                    using I16 = std::integral_constant<int, kInt16>;
                    using P4 = std::integral_constant<int, kPack4>;
                    using Y = std::true_type;
                    using N = std::false_type;
                    const int st = p.q.store;
                    if (rs.fast) {
                        if (st == kInt8)
                            run(I8{}, Y{});
                        else if (st == kInt16)
                            run(I16{}, Y{});
                        else
                            run(P4{}, Y{});
                    } else {
                        if (st == kInt8)
                            run(I8{}, N{});
                        else if (st == kInt16)
                            run(I16{}, N{});
                        else
                            run(P4{}, N{});
                    }
                    if (rv && col0 == 0)
                        rscales[row0] = rs.scale;
                    return;
                }
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int64_t row = row0 + i * p.step_rows;
                const bool rv = row < p.rows;
                RowScale rs;
                rs.given = true;
                rs.amax = rv ? rowa_in[row] : 0.0f;
                rs.scale = int_scale(rs.amax, p.q);
                rs.rc = make_recip(rs.scale);
                rs.fast = quot_fast(rs.rc, rs.amax);
                const ChunkOut oi = out_i(i);
                process_chunk<T, PAT, SCORE, FMT>(p, raw[i], oi, c, acc, rs.amax, &rs);
                if (rv && col0 + i * p.step_cols == 0)
                    rscales[row] = rs.scale;
            }
            return;
        }
    }
    if constexpr (FMT == kInt) {
        // INT groups (up to 32 lanes): select all four chunks, then reduce
        // their group amaxes across lanes together (four independent shuffle
        // chains instead of four dependent ones), then quantize. The short
        // NVFP4 / MXFP4 reductions gain less than the registers cost.
        constexpr int VPC = PAT == kDense ? 8 : 4;
        Sel<VPC> sl[4];
        float g[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            sl[i] = select_chunk<T, PAT, SCORE>(raw[i], out_i(i));
            g[i] = sl[i].vmax;
        }
        const int lanes = p.q.lanes;
        for (int off = 1; off < lanes; off <<= 1)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                g[i] = fmaxf(g[i], __shfl_xor_sync(kFull, g[i], off));
#pragma unroll
        for (int i = 0; i < 4; ++i)
            finish_chunk<T, PAT, SCORE, FMT>(p, raw[i], sl[i], out_i(i), c, acc, -1.0f, nullptr, g[i]);
    } else if (FMT == kNvfp4 && PAT != kDense && p.step_rows == 0) {
        // 2:4 / 4:8 + NVFP4: a unit holds 4 chunks x 8 blocks of 16 kept
        // values = 32 blocks; lane L computes the scale of block L % 8 of
        // chunk L / 8 once (instead of each chunk's lanes computing their
        // block's) and stores its byte; the chunks' lanes fetch the divisor
        // and its reciprocal. (Full-width units: one row per slot, so block
        // j's scale byte is j - lane / 4 bytes from this lane's own.)
        constexpr int VPC = PAT == kDense ? 8 : 4;
        // bf16 2:4 by magnitude: the block maxima on packed kept pairs (one
        // conversion per block instead of one per chunk)
        constexpr bool kPk = sizeof(T) == 2 && PAT == kSparse24 && SCORE == kMag;
        Sel<VPC> sl[4];
        const int bs_ = lane >> 3, bj = lane & 7;
        float am;
        if constexpr (kPk) {
            uint32_t g2[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                sl[i] = select_chunk<T, PAT, SCORE>(raw[i], out_i(i));
                g2[i] = bf16x2_maxabs(sl[i].k0, sl[i].k1);
            }
#pragma unroll
            for (int off = 1; off < 4; off <<= 1)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    g2[i] = bf16x2_maxabs(g2[i], __shfl_xor_sync(kFull, g2[i], off));
            uint32_t t2[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                t2[i] = __shfl_sync(kFull, g2[i], 4 * bj);
            am = bf16x2_hmax(bs_ == 0 ? t2[0] : bs_ == 1 ? t2[1] : bs_ == 2 ? t2[2] : t2[3]);
        } else {
            float g[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                sl[i] = select_chunk<T, PAT, SCORE>(raw[i], out_i(i));
                g[i] = sl[i].vmax;
            }
#pragma unroll
            for (int off = 1; off < 4; off <<= 1)
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    g[i] = fmaxf(g[i], __shfl_xor_sync(kFull, g[i], off));
            float t[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                t[i] = __shfl_sync(kFull, g[i], 4 * bj);
            am = bs_ == 0 ? t[0] : bs_ == 1 ? t[1] : bs_ == 2 ? t[2] : t[3];
        }
        const uint32_t sb = nv_block_code(am, c.rst);
        const float den = c.tb.den[sb];
        // quot_fast for the block, once: its chunks' lanes read the verdict
        // from the reciprocal's sign
        const bool bfast = den >= 0x1p-60f && den <= 0x1p60f && __fmul_rn(am, c.tb.inv[sb]) < 0x1p126f;
        const float inv = bfast ? c.tb.inv[sb] : -1.0f;
        {
            // the block's scale byte: block bj of chunk bs_, 8 bytes per chunk slot
            const ChunkOut ob_ = out_i(bs_);
            const bool bvalid = FULL || col0 - 8 * lane + bs_ * step_c + 32 * bj < p.k;
            if (bvalid && row0 + bs_ * p.step_rows < p.rows)
                ob_.scale[bj - (lane >> 2)] = static_cast<uint8_t>(sb);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            NvBlock b;
            const int src = 8 * i + (lane >> 2);
            b.den = __shfl_sync(kFull, den, src);
            b.inv = __shfl_sync(kFull, inv, src);
            finish_chunk<T, PAT, SCORE, FMT>(p, raw[i], sl[i], out_i(i), c, acc, -1.0f, nullptr, 0.0f, &b);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            process_chunk<T, PAT, SCORE, FMT>(p, raw[i], out_i(i), c, acc);
        if constexpr (FMT == kAmax) {
            if (rowa) {
                // per-row amax of the values to quantize: reduced over the
                // lanes sharing a row segment, then an atomic max (non-negative
                // floats order like their bit patterns)
                const int segl = 1 << p.log2_cpr;
                float cm[4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    cm[i] = quantized_amax<T, PAT, SCORE>(raw[i], out_i(i));
                if (p.step_rows == 0) {
                    // the four chunks share the lane's row
                    float m = fmaxf(fmaxf(cm[0], cm[1]), fmaxf(cm[2], cm[3]));
                    m = group_amax(m, segl);
                    if ((lane & (segl - 1)) == 0 && row0 < p.rows)
                        atomicMax(reinterpret_cast<int *>(rowa + row0), __float_as_int(m));
                } else {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float m = group_amax(cm[i], segl);
                        const int64_t row = row0 + i * p.step_rows;
                        if ((lane & (segl - 1)) == 0 && row < p.rows)
                            atomicMax(reinterpret_cast<int *>(rowa + row), __float_as_int(m));
                    }
                }
            }
        }
    }
}

// The pass along axis 1 (k contiguous). A slot is 32 chunks, one per lane: a
// row segment of W = 8 * cpr columns for each of 32 / cpr rows (lane = row
// offset * cpr + chunk). A unit is four slots, either four consecutive
// segments of the same rows (step_cols = W) or the same segment of four
// consecutive row groups (step_rows = 32 / cpr); a warp loads the unit's
// four chunks per lane (16-byte loads, 512 contiguous bytes per slot) before
// processing them. The warps serving an operand take units u = warp index,
// warp index + number of warps, ... The CTA count per operand and the layout
// are chosen by the host. FW: the full-width case W = 256 with four segments
// per unit, where the slot offsets are compile-time constants and a unit
// wholly inside the operand skips the per-chunk checks.
template <typename T, int PAT, int SC, int FMT, bool FW>
__global__ void __launch_bounds__(kStreamThreads, (StreamOcc<T, PAT, (SC & 1), FMT, FW, (SC & kRotated) != 0>::value))
    stream_kernel(const __grid_constant__ PassParams pk)
{
    // SC: the score, with kRotated set for a pass over the rotated operand
    constexpr int SCORE = SC & 1;
    constexpr bool ROT = (SC & kRotated) != 0;
    static_assert(!ROT || (sizeof(T) == 2 && SCORE == kMag), "rotated passes: bf16, magnitude score");
    // the loop reads the (operand-independent) parameters in place and keeps
    // only this operand's output bases; the operand's full view is built for
    // the constants and again for the final reductions
    const PassParams &p = pk;
    const int op = static_cast<int>(blockIdx.x) / pk.ctas_per_op;
    const int cta = static_cast<int>(blockIdx.x) - op * pk.ctas_per_op;
    __shared__ double red[kStreamWarps * 4];
    __shared__ float fred[kStreamWarps * 2];
    __shared__ uint32_t flag;
    __shared__ float nvt[(FMT == kNvfp4 || FMT == kEnergy) ? 512 : 4];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    grid_dependency_wait();
    grid_dependents_launch();
    const PassConsts c = make_consts<FMT>(operand_view(pk), tid, kStreamThreads, nvt);
    const OutBase ob = out_base(pk, op);
    // per-row amax out (amax pass) or in (INT with one scale per row)
    float *rowa = FMT == kAmax && p.row_amax ? p.row_amax + op * p.rows : nullptr;
    const float *rowa_in = FMT == kIntRows ? p.q.row_amax_in + op * p.rows : nullptr;
    float *rscales = reinterpret_cast<float *>(ob.scales);

    const T *x = static_cast<const T *>(p.x) + op * p.x_bstride;
    const int log2_cpr = FW ? 5 : p.log2_cpr;
    const int lrow = lane >> log2_cpr;
    const int lcol = (lane & ((1 << log2_cpr) - 1)) << 3;
    const int64_t step_x = FW ? 256 : static_cast<int64_t>(p.step_rows) * p.ld + p.step_cols;
    const int64_t step_c = FW ? 256 : p.step_cols;
    // pointer advance per slot of a unit (the output offsets are linear in
    // row and column, and a step never splits a scale group)
    const ChunkOut z0 = make_out<T, PAT, FMT>(p, ob, 0, 0, false, lane);
    const ChunkOut z1 = make_out<T, PAT, FMT>(p, ob, FW ? 0 : p.step_rows, FW ? 256 : p.step_cols, false, lane);
    using FS = FwStep<T, PAT, FMT>;
    const int64_t dval = (FW && FS::val >= 0) ? FS::val : z1.val - z0.val;
    const int64_t dscale = (FW && FS::scale >= 0) ? FS::scale : z1.scale - z0.scale;
    const int64_t dmeta = FW ? FS::meta : z1.meta - z0.meta;
    const int unit_rows = FW ? 1 : p.unit_rows;
    const int unit_cols = FW ? 1024 : p.unit_cols;

    const int tw = p.ctas_per_op * kStreamWarps;
    const int u0 = cta * kStreamWarps + warp;
    int ua = u0 / p.units_b, ub = u0 - ua * p.units_b;
    const int sa = tw / p.units_b, sb = tw - sa * p.units_b;
    double e_total = 0.0, e_prune = 0.0, e_q = 0.0, e_qd = 0.0;
    Acc acc{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if constexpr (FMT == kAmax && FW) {
        if (rowa) {
            // whole rows per warp (rows = units_a here): the row amax is the
            // warp's own, stored without atomics; units wholly inside the
            // operand take the fast path, the last partial quad the general one
            for (int64_t row = u0; row < p.units_a; row += tw) {
                float rm = 0.0f;
                for (int b = 0; b < p.units_b; ++b) {
                    const int64_t col0 = static_cast<int64_t>(b) * 1024 + lcol;
                    const T *xp = x + row * p.ld + col0;
                    const ChunkOut o = make_out<T, PAT, FMT>(p, ob, row, col0, true, lane);
                    if (static_cast<int64_t>(b + 1) * 1024 <= p.k) {
                        rm = fmaxf(rm, amax_unit_fw<T, PAT, SCORE, ROT>(p, xp, o, acc));
                    } else {
                        Acc a{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                        stream_unit<T, PAT, SCORE, FMT, false, ROT>(p, c, xp, step_x, step_c, o, dval, dscale, dmeta,
                                                                    row, col0, a);
                        acc.amax_all = fmaxf(acc.amax_all, a.amax_all);
                        acc.amax_kept = fmaxf(acc.amax_kept, a.amax_kept);
                        rm = fmaxf(rm, PAT == kDense ? a.amax_all : a.amax_kept);
                    }
                }
                rm = group_amax(rm, 32);
                if (lane == 0)
                    rowa[row] = rm;
            }
            ua = p.units_a; // skip the unit loop
        }
    }
    while (ua < p.units_a) {
        const int64_t row0 = static_cast<int64_t>(ua) * unit_rows + lrow;
        const int64_t col0 = static_cast<int64_t>(ub) * unit_cols + lcol;
        const T *xp = x + row0 * p.ld + col0;
        const ChunkOut o = make_out<T, PAT, FMT>(p, ob, row0, col0, true, lane);
        acc.et = acc.ep = acc.eq = acc.eqd = 0.0f;
        // full-width units lie inside the operand except in the last quad
        // of a row (rows are whole: one row per unit)
        if (FW && static_cast<int64_t>(ub + 1) * 1024 <= p.k)
            stream_unit<T, PAT, SCORE, FMT, true, ROT>(p, c, xp, step_x, step_c, o, dval, dscale, dmeta, row0, col0,
                                                  acc, rowa, rowa_in, rscales);
        else
            stream_unit<T, PAT, SCORE, FMT, false, ROT>(p, c, xp, step_x, step_c, o, dval, dscale, dmeta, row0, col0,
                                                   acc, rowa, rowa_in, rscales);
        // only the energies this pass produces (the others stay zero)
        if constexpr (FMT != kAmax)
            e_total += acc.et;
        if constexpr (FMT != kAmax && PAT != kDense)
            e_prune += acc.ep;
        if constexpr (FMT != kAmax && FMT != kNone && PAT != kDense)
            e_q += acc.eq;
        if constexpr (FMT == kFp8 && PAT == kSparse24) {
            e_q += lo2(acc.eq2) + hi2(acc.eq2);
            acc.eq2 = 0ull;
        }
        if constexpr (FMT != kAmax && FMT != kNone && (PAT == kDense || FMT == kEnergy))
            e_qd += acc.eqd;
        ua += sa;
        ub += sb;
        if (ub >= p.units_b) {
            ub -= p.units_b;
            ++ua;
        }
    }

    const PassParams v = operand_view(pk);
    if constexpr (FMT == kAmax) {
        grid_reduce_amax<PAT>(v, acc.amax_kept, acc.amax_all, fred, &flag, tid, lane, warp);
    } else {
        if (!v.energy_out)
            return;
        grid_reduce_energy(v, e_total, e_prune, e_q, e_qd, red, &flag, tid, lane, warp);
    }
}

// ---------------------------------------------------------------------------
// one scale per row (INT with group 0) when a row does not fit one warp's
// 256-element span. One warp per row, two sweeps over the row in global
// memory: the first streams it through L1-caching loads (eight 16-byte chunks
// per lane in flight) and takes the amax of the values to quantize; the second
// reads it again (from L1 or L2; HBM sees one read) and quantizes with the
// row's scale. The code stays small and registers few, so many warps are
// resident to cover the load latency.
// ---------------------------------------------------------------------------

// Chunk c of a row through the read-only cache path (the row is read again in
// the second sweep, from L1 or L2); zeros when !ok.
template <typename T> struct RowChunk;
template <> struct RowChunk<__nv_bfloat16> {
    __device__ __forceinline__ static Elem<__nv_bfloat16>::Raw load(const void *row, int c, bool ok)
    {
        Elem<__nv_bfloat16>::Raw r;
        r.v = ok ? __ldg(reinterpret_cast<const uint4 *>(row) + c) : make_uint4(0u, 0u, 0u, 0u);
        return r;
    }
};
template <> struct RowChunk<float> {
    __device__ __forceinline__ static Elem<float>::Raw load(const void *row, int c, bool ok)
    {
        Elem<float>::Raw r;
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        r.a = ok ? __ldg(reinterpret_cast<const float4 *>(row) + 2 * c) : z;
        r.b = ok ? __ldg(reinterpret_cast<const float4 *>(row) + 2 * c + 1) : z;
        return r;
    }
};

template <typename T, int PAT, int SCORE>
__global__ void __launch_bounds__(kRowThreads) rowsweep_kernel(const T *__restrict__ x, int64_t ld,
                                                               const PassParams pk)
{
    const PassParams p = operand_view(pk);
    __shared__ double red[kConsumerWarps * 4];
    __shared__ uint32_t flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    grid_dependency_wait();
    grid_dependents_launch();
    const int nchunks = static_cast<int>(p.k / 8);
    const PassConsts nc{make_recip(0.0f), make_recip(0.0f), NvTable{nullptr, nullptr}, NvTable{nullptr, nullptr},
                        false, false};
    double e_total = 0.0, e_prune = 0.0, e_q = 0.0, e_qd = 0.0;
    for (int64_t row = static_cast<int64_t>(p.cta) * kConsumerWarps + warp; row < p.rows;
         row += static_cast<int64_t>(p.ctas_per_op) * kConsumerWarps) {
        const T *xr = x + p.op * p.x_bstride + row * ld;
        // sweep 1: the row amax of the values to quantize (for 2:4 by
        // magnitude the kept amax equals the amax of all values)
        float amax = 0.0f;
        for (int c0 = 0; c0 < nchunks; c0 += 256) {
            typename Elem<T>::Raw buf[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                buf[u] = RowChunk<T>::load(xr, c0 + 32 * u + lane, c0 + 32 * u + lane < nchunks);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int c = c0 + 32 * u + lane;
                if (c < nchunks) {
                    if constexpr (PAT == kDense || (PAT == kSparse24 && SCORE == kMag)) {
                        float xv[8];
                        Elem<T>::unpack(buf[u], xv);
                        amax = fmaxf(amax, chunk_amax<T>(buf[u], xv));
                    } else {
                        Acc a{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                        process_chunk<T, PAT, SCORE, kAmax>(
                            p, buf[u], make_out<T, PAT, kAmax>(p, row, static_cast<int64_t>(c) * 8, true, lane), nc,
                            a);
                        amax = fmaxf(amax, a.amax_kept);
                    }
                }
            }
        }
        amax = group_amax(amax, 32);
        RowScale rs;
        rs.given = true;
        rs.amax = amax;
        rs.scale = int_scale(amax, p.q);
        rs.rc = make_recip(rs.scale);
        rs.fast = quot_fast(rs.rc, amax);
        // sweep 2: codes, metadata and energies; every lane takes part in each
        // step (4:8 metadata pairs lanes through a shuffle)
        Acc acc{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int c0 = 0; c0 < nchunks; c0 += 64) {
            typename Elem<T>::Raw buf[2];
#pragma unroll
            for (int u = 0; u < 2; ++u)
                buf[u] = RowChunk<T>::load(xr, c0 + 32 * u + lane, c0 + 32 * u + lane < nchunks);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int c = c0 + 32 * u + lane;
                if (c0 + 32 * u < nchunks)
                    process_chunk<T, PAT, SCORE, kInt>(
                        p, buf[u], make_out<T, PAT, kInt>(p, row, static_cast<int64_t>(c) * 8, c < nchunks, lane), nc,
                        acc, amax, &rs);
            }
        }
        if (lane == 0)
            static_cast<float *>(p.scales)[row] = rs.scale;
        e_total += acc.et;
        e_prune += acc.ep;
        e_q += acc.eq;
        e_qd += acc.eqd;
    }
    if (!p.energy_out)
        return;
    grid_reduce_energy(p, e_total, e_prune, e_q, e_qd, red, &flag, tid, lane, warp);
}

// ---------------------------------------------------------------------------
// one scale per row with the row held in registers (k <= 8 * 256 * CPT):
// tpr threads (a power of two, 32..256) share a row, each holding CPT chunks
// (chunk c = t + j * tpr of the row, so a warp's loads are contiguous); a CTA
// of 256 threads takes 256 / tpr rows per step. The row amax is reduced with
// shuffles and, across the row's warps, through shared memory (one named
// barrier per row and step, over that row's warps only; the buffer alternates
// between steps); the codes are then computed from the registers, so the
// operand is read once.
// ---------------------------------------------------------------------------

// Resident CTAs per SM the row-block kernel is compiled for (register budget:
// the row's CPT chunks per thread stay in registers).
template <typename T, int PAT, int SCORE, int CPT> struct RowblockOcc {
    static constexpr bool light = sizeof(T) == 2 && (PAT == kDense || (PAT == kSparse24 && SCORE == kMag));
    static constexpr int value = CPT == 1 ? 4 : CPT == 4 ? (light ? 4 : 3) : 2;
};

template <typename T, int PAT, int SCORE, int CPT>
__global__ void __launch_bounds__(kRowThreads, (RowblockOcc<T, PAT, SCORE, CPT>::value))
    rowblock_kernel(const T *__restrict__ x, int64_t ld, int32_t log2_tpr, const __grid_constant__ PassParams pk)
{
    const PassParams &p = pk;
    const int op = static_cast<int>(blockIdx.x) / pk.ctas_per_op;
    const int cta = static_cast<int>(blockIdx.x) - op * pk.ctas_per_op;
    __shared__ double red[kConsumerWarps * 4];
    __shared__ float wmax[2][kConsumerWarps];
    __shared__ uint32_t flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    grid_dependency_wait();
    grid_dependents_launch();
    const int tpr = 1 << log2_tpr, rpc = kRowThreads >> log2_tpr;
    const int t = tid & (tpr - 1), rin = tid >> log2_tpr;
    const int wpr = tpr >> 5 > 0 ? tpr >> 5 : 1; // warps per row
    const int w0 = (rin * tpr) >> 5;               // first warp of this thread's row
    const int nchunks = static_cast<int>(p.k / 8);
    const PassConsts nc{make_recip(0.0f), make_recip(0.0f), NvTable{nullptr, nullptr}, NvTable{nullptr, nullptr},
                        false, false};
    const OutBase ob = out_base(pk, op);
    const T *xo = x + op * p.x_bstride;
    // output offsets are linear in the column: the advance of each pointer
    // per chunk step (tpr chunks)
    const ChunkOut z = make_out<T, PAT, kInt>(p, ob, 0, 8 * t, true, lane);
    const ChunkOut zc = make_out<T, PAT, kInt>(p, ob, 0, 8 * (t + tpr), true, lane);
    const int64_t cval = zc.val - z.val, cmeta = zc.meta - z.meta;
    float *scales = reinterpret_cast<float *>(ob.scales); // one per row
    double e_total = 0.0, e_prune = 0.0, e_q = 0.0, e_qd = 0.0;
    int buf = 0;
    for (int64_t base = static_cast<int64_t>(cta) * rpc; base < p.rows;
         base += static_cast<int64_t>(p.ctas_per_op) * rpc, buf ^= 1) {
        const int64_t row = base + rin;
        const bool rv = row < p.rows;
        const T *xr = xo + row * ld;
        typename Elem<T>::Raw raw[CPT];
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const int c = t + j * tpr;
            raw[j] = Stream<T>::load(xr + 8 * c, rv && c < nchunks);
        }
        const ChunkOut o = make_out<T, PAT, kInt>(p, ob, row, 8 * t, rv, lane);
        // the row amax of the values to quantize (for 2:4 by magnitude the
        // kept amax equals the amax of all values)
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            if constexpr (PAT == kDense || (PAT == kSparse24 && SCORE == kMag)) {
                float xv[8];
                Elem<T>::unpack(raw[j], xv);
                m = fmaxf(m, chunk_amax<T>(raw[j], xv));
            } else {
                ChunkOut oj = o;
                oj.norms = o.norms + 8 * j * tpr;
                oj.valid = rv && t + j * tpr < nchunks;
                Acc a{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                process_chunk<T, PAT, SCORE, kAmax>(p, raw[j], oj, nc, a);
                m = fmaxf(m, a.amax_kept);
            }
        }
        m = group_amax(m, 32);
        if (wpr > 1) {
            // the row's warps only: a named barrier per row, ids 2.. (id 1
            // belongs to the CTA-wide reduction at the end)
            if (lane == 0)
                wmax[buf][warp] = m;
            named_barrier_sync(2 + rin, tpr);
            for (int w = 0; w < wpr; ++w)
                m = fmaxf(m, wmax[buf][w0 + w]);
        }
        RowScale rs;
        rs.given = true;
        rs.amax = m;
        rs.scale = int_scale(m, p.q);
        rs.rc = make_recip(rs.scale);
        rs.fast = quot_fast(rs.rc, m);
        Acc acc{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if constexpr (PAT == kDense) {
            const float qm = p.q.qmax;
            const int st = p.q.store;
            if (rs.fast) {
                if (st == kInt8)
                    dense_int_row<T, CPT, kInt8, true>(raw, rs, qm, o.val, cval, t, tpr, nchunks, rv, acc);
                else if (st == kInt16)
                    dense_int_row<T, CPT, kInt16, true>(raw, rs, qm, o.val, cval, t, tpr, nchunks, rv, acc);
                else
                    dense_int_row<T, CPT, kPack4, true>(raw, rs, qm, o.val, cval, t, tpr, nchunks, rv, acc);
            } else {
                if (st == kInt8)
                    dense_int_row<T, CPT, kInt8, false>(raw, rs, qm, o.val, cval, t, tpr, nchunks, rv, acc);
                else if (st == kInt16)
                    dense_int_row<T, CPT, kInt16, false>(raw, rs, qm, o.val, cval, t, tpr, nchunks, rv, acc);
                else
                    dense_int_row<T, CPT, kPack4, false>(raw, rs, qm, o.val, cval, t, tpr, nchunks, rv, acc);
            }
        } else {
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                ChunkOut oj = o;
                oj.val += j * cval;
                oj.meta += j * cmeta;
                if constexpr (SCORE == kWanda)
                    oj.norms = o.norms + 8 * j * tpr;
                oj.valid = rv && t + j * tpr < nchunks;
                process_chunk<T, PAT, SCORE, kInt>(p, raw[j], oj, nc, acc, m, &rs);
            }
        }
        if (rv && t == 0)
            scales[row] = rs.scale;
        e_total += acc.et;
        if constexpr (PAT != kDense) {
            e_prune += acc.ep;
            e_q += acc.eq;
        } else {
            e_qd += acc.eqd;
        }
    }
    const PassParams v = operand_view(pk);
    if (!v.energy_out)
        return;
    grid_reduce_energy(v, e_total, e_prune, e_q, e_qd, red, &flag, tid, lane, warp);
}

// ---------------------------------------------------------------------------
// strided reduction axis (axis 0): A[r][c] at x[c * ld + r]. The TMA box is
// 128 k (outer) x Rr rows (inner, contiguous): Rr = 64 for bf16, 32 for fp32,
// a 16 KiB stage S laid out [k][Rr]. Consumers transpose S through registers
// into T[Rr][k + pad] (row pitch 272 / 528 bytes, 16 mod 128), then read
// 8-element chunks of T exactly as an axis-1 tile of width 128 is read.
//
// Transpose blocks: bf16 8 k x 8 rows (threads 0..127), fp32 4 k x 4 rows
// (threads 0..255). Thread t takes row block b = t & 7 and k block
// a = ((t >> 3) + b) mod (number of k blocks): the eight lanes of a shared-
// memory phase then read eight different 16-byte columns of S and write eight
// different 16-byte bank groups of T (the pitch is 16 mod 128), so neither side
// has bank conflicts.
// ---------------------------------------------------------------------------

template <typename T> struct Axis0;

// Component c (a constant after unrolling) of a uint4.
__device__ __forceinline__ uint32_t word(const uint4 &v, int c)
{
    switch (c) {
    case 0:
        return v.x;
    case 1:
        return v.y;
    case 2:
        return v.z;
    default:
        return v.w;
    }
}

template <> struct Axis0<__nv_bfloat16> {
    static constexpr int kRows = 64;   // rows per tile
    static constexpr int kPitch = 136; // elements per T row
    __device__ __forceinline__ static void transpose(const uint8_t *S, uint8_t *Tb, int tid)
    {
        if (tid >= 128)
            return;
        const int b = tid & 7, a = ((tid >> 3) + b) & 15;
        uint4 in[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            in[i] = *reinterpret_cast<const uint4 *>(S + ((8 * a + i) * kRows + 8 * b) * 2);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            // row 8b + j gathers the j-th bf16 of each of the eight k rows
            const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;
            uint4 o;
            o.x = __byte_perm(word(in[0], j >> 1), word(in[1], j >> 1), sel);
            o.y = __byte_perm(word(in[2], j >> 1), word(in[3], j >> 1), sel);
            o.z = __byte_perm(word(in[4], j >> 1), word(in[5], j >> 1), sel);
            o.w = __byte_perm(word(in[6], j >> 1), word(in[7], j >> 1), sel);
            *reinterpret_cast<uint4 *>(Tb + ((8 * b + j) * kPitch + 8 * a) * 2) = o;
        }
    }
    __device__ __forceinline__ static Elem<__nv_bfloat16>::Raw load(const uint8_t *Tb, int trow, int c)
    {
        Elem<__nv_bfloat16>::Raw r;
        r.v = *reinterpret_cast<const uint4 *>(Tb + (trow * kPitch + 8 * c) * 2);
        return r;
    }
};

template <> struct Axis0<float> {
    static constexpr int kRows = 32;
    static constexpr int kPitch = 132;
    __device__ __forceinline__ static void transpose(const uint8_t *S, uint8_t *Tb, int tid)
    {
        const int b = tid & 7, a = ((tid >> 3) + b) & 31;
        float4 in[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            in[i] = *reinterpret_cast<const float4 *>(S + ((4 * a + i) * kRows + 4 * b) * 4);
        const float4 o0 = make_float4(in[0].x, in[1].x, in[2].x, in[3].x);
        const float4 o1 = make_float4(in[0].y, in[1].y, in[2].y, in[3].y);
        const float4 o2 = make_float4(in[0].z, in[1].z, in[2].z, in[3].z);
        const float4 o3 = make_float4(in[0].w, in[1].w, in[2].w, in[3].w);
        *reinterpret_cast<float4 *>(Tb + ((4 * b + 0) * kPitch + 4 * a) * 4) = o0;
        *reinterpret_cast<float4 *>(Tb + ((4 * b + 1) * kPitch + 4 * a) * 4) = o1;
        *reinterpret_cast<float4 *>(Tb + ((4 * b + 2) * kPitch + 4 * a) * 4) = o2;
        *reinterpret_cast<float4 *>(Tb + ((4 * b + 3) * kPitch + 4 * a) * 4) = o3;
    }
    __device__ __forceinline__ static Elem<float>::Raw load(const uint8_t *Tb, int trow, int c)
    {
        Elem<float>::Raw r;
        r.a = *reinterpret_cast<const float4 *>(Tb + (trow * kPitch + 8 * c) * 4);
        r.b = *reinterpret_cast<const float4 *>(Tb + (trow * kPitch + 8 * c) * 4 + 16);
        return r;
    }
};

// Two CTAs per SM (2 x 86 KB of shared memory; the register cap this sets,
// 96, spills a few bytes in some instantiations): the second CTA's tiles
// overlap the first's barriers and transposes, 20 - 23% faster than one.
template <typename T, int PAT, int SCORE, int FMT>
__global__ void __launch_bounds__(kThreads, 2) axis0_kernel(const __grid_constant__ CUtensorMap map,
                                                            const PassParams pk)
{
    const PassParams p = operand_view(pk);
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *stages = smem;
    uint8_t *Tb = smem + kStages * kStageBytes; // two transpose buffers
    uint64_t *full = reinterpret_cast<uint64_t *>(Tb + 2 * kAxis0TBytes);
    uint64_t *empty = full + kStages;
    double *red = reinterpret_cast<double *>(empty + kStages);
    float *fred = reinterpret_cast<float *>(red + kConsumerWarps * 4);
    uint32_t *flag = reinterpret_cast<uint32_t *>(fred + kConsumerWarps * 2);
    uint32_t *ready = flag + 1;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_barrier_init();
    }
    __syncthreads();
    grid_dependency_wait();
    grid_dependents_launch();
    if (warp == kConsumerWarps) {
        if (lane == 0)
            producer(&map, p, stages, full, empty);
        return;
    }

    float *nvt = reinterpret_cast<float *>(ready + 4); // 2 x 256 floats
    const PassConsts c = make_consts<FMT>(p, tid, kConsumers, nvt);
    using A0 = Axis0<T>;
    double e_total = 0.0, e_prune = 0.0, e_q = 0.0, e_qd = 0.0;
    Acc acc{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    uint32_t it = 0;
    for (int64_t t = p.cta; t < p.n_tiles; t += p.ctas_per_op, ++it) {
        const int s = it % kStages;
        // one thread waits for the stage and tells the others, so that every
        // consumer leaves the loop together if the wait gives up
        if (tid == 0) {
            const bool ok = mbar_wait(&full[s], (it / kStages) & 1, p.wait_limit_ns);
            if (!ok)
                record_error(p.err, 5);
            *ready = ok;
        }
        named_barrier_sync(1, kConsumers);
        if (!*ready)
            break;
        // this tile's transpose buffer: the other one may still be read by
        // threads finishing the previous tile; a buffer is written again only
        // two tiles later, after every thread has passed the next tile's
        // first barrier (and so has read it)
        uint8_t *Tc = Tb + (it & 1) * kAxis0TBytes;
        A0::transpose(stages + s * kStageBytes, Tc, tid);
        named_barrier_sync(1, kConsumers); // S is read, T is written
        if (lane == 0)
            mbar_arrive(&empty[s]);
        typename Elem<T>::Raw raw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (i < p.cpt) {
                const int j = tid + i * kConsumers;
                raw[i] = A0::load(Tc, j >> 4, j & 15);
            }
        const int64_t rt = t / p.n_col_tiles, ct = t - rt * p.n_col_tiles;
        const int64_t row0 = rt * A0::kRows, col0 = ct * kAxis0K;
        acc.et = acc.ep = acc.eq = acc.eqd = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (i < p.cpt) {
                const int j = tid + i * kConsumers;
                const int64_t row = row0 + (j >> 4), col = col0 + ((j & 15) << 3);
                process_chunk<T, PAT, SCORE, FMT>(
                    p, raw[i], make_out<T, PAT, FMT>(p, row, col, row < p.rows && col < p.k, lane), c, acc);
            }
        }
        if constexpr (FMT != kAmax) {
            e_total += acc.et;
            e_prune += acc.ep;
            e_q += acc.eq;
            e_qd += acc.eqd;
        }
        if constexpr (FMT == kFp8 && PAT == kSparse24) {
            e_q += lo2(acc.eq2) + hi2(acc.eq2);
            acc.eq2 = 0ull;
        }
    }
    if constexpr (FMT == kAmax) {
        grid_reduce_amax<PAT>(p, acc.amax_kept, acc.amax_all, fred, flag, tid, lane, warp);
    } else {
        if (!p.energy_out)
            return;
        grid_reduce_energy(p, e_total, e_prune, e_q, e_qd, red, flag, tid, lane, warp);
    }
}

} // namespace ss24
