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
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
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

__device__ __forceinline__ float sq(float a) { return a * a; }

// ---------------------------------------------------------------------------
// quantizers of one chunk's values (VPC = 4 kept or 8 dense values); every
// lane of the warp calls them (group reductions shuffle across lanes)
// ---------------------------------------------------------------------------

struct QOut {
    void *values;
    void *scales;
    int64_t row, colq, n; // quantized row length n, column of the chunk's first value
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

// Sum of (v - d)^2 over a chunk's values: packed differences and squares,
// summed as a binary tree (each term and each partial sum rounded once).
template <int VPC> __device__ __forceinline__ float err_energy(const float (&v)[VPC], const float (&d)[VPC])
{
    f32x2 t[VPC / 2];
#pragma unroll
    for (int i = 0; i < VPC / 2; ++i) {
        const f32x2 e = sub2(pack2(v[2 * i], v[2 * i + 1]), pack2(d[2 * i], d[2 * i + 1]));
        t[i] = mul2(e, e);
    }
#pragma unroll
    for (int w = VPC / 4; w >= 1; w /= 2)
#pragma unroll
        for (int i = 0; i < w; ++i)
            t[i] = add2(t[i], t[i + w]);
    return lo2(t[0]) + hi2(t[0]);
}

// Quotients v / s of a chunk: Markstein's correction when the scale is in the
// fast range and no quotient can overflow (max|v| * y < 2^126), IEEE division
// otherwise; zero scale gives zero quotients.
template <int VPC>
__device__ __forceinline__ void quotients(const float (&v)[VPC], const Recip &rc, float vmax, float (&q)[VPC])
{
    if (rc.fast && __fmul_rn(vmax, rc.y) < 0x1p126f) {
#pragma unroll
        for (int i = 0; i < VPC / 2; ++i) {
            const f32x2 qq = div_fast2(pack2(v[2 * i], v[2 * i + 1]), rc);
            q[2 * i] = with_sign_of(lo2(qq), v[2 * i]);
            q[2 * i + 1] = with_sign_of(hi2(qq), v[2 * i + 1]);
        }
    } else {
#pragma unroll
        for (int i = 0; i < VPC; ++i)
            q[i] = rc.b != 0.0f ? __fdiv_rn(v[i], rc.b) : 0.0f;
    }
}

// Dequantized values code_value * s of a chunk (binary32 products).
template <int VPC>
__device__ __forceinline__ void scale_values(const float (&c)[VPC], float s, float (&d)[VPC])
{
    const f32x2 s2 = pack2(s, s);
#pragma unroll
    for (int i = 0; i < VPC / 2; ++i) {
        const f32x2 r = mul2(pack2(c[2 * i], c[2 * i + 1]), s2);
        d[2 * i] = lo2(r);
        d[2 * i + 1] = hi2(r);
    }
}

// FP8 E4M3, per-tensor scale s: code = E4M3(v / s); deq = E4M3(code) * s.
template <int VPC, bool STORE>
__device__ __forceinline__ float quant_fp8(const float (&v)[VPC], const Recip &rc, const QOut &o)
{
    float q[VPC], dec[VPC], d[VPC];
    quotients<VPC>(v, rc, local_amax<VPC>(v), q);
    uint32_t c[VPC / 4];
#pragma unroll
    for (int t = 0; t < VPC / 4; ++t) {
        c[t] = cvt_e4m3x2(q[4 * t], q[4 * t + 1]) | (cvt_e4m3x2(q[4 * t + 2], q[4 * t + 3]) << 16);
        const float2 lo = e4m3x2_to_f32(c[t] & 0xffffu), hi = e4m3x2_to_f32(c[t] >> 16);
        dec[4 * t + 0] = lo.x;
        dec[4 * t + 1] = lo.y;
        dec[4 * t + 2] = hi.x;
        dec[4 * t + 3] = hi.y;
    }
    scale_values<VPC>(dec, rc.b, d);
    if (STORE && o.valid) {
        uint8_t *dst = static_cast<uint8_t *>(o.values) + o.row * o.n + o.colq;
        if constexpr (VPC == 4)
            *reinterpret_cast<uint32_t *>(dst) = c[0];
        else
            *reinterpret_cast<uint2 *>(dst) = make_uint2(c[0], c[1]);
    }
    return err_energy<VPC>(v, d);
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
};

template <int VPC, bool STORE>
__device__ __forceinline__ float quant_int(const float (&v)[VPC], const QuantSpec &q, const QOut &o,
                                           float row_amax = -1.0f, const RowScale *rs = nullptr)
{
    float amax, scale;
    Recip rc;
    if (rs && rs->given) {
        amax = rs->amax;
        scale = rs->scale;
        rc = rs->rc;
    } else {
        amax = row_amax >= 0.0f ? row_amax : group_amax(local_amax<VPC>(v), q.lanes);
        scale = int_scale(amax, q);
        rc = make_recip(scale);
    }
    float qv[VPC];
    quotients<VPC>(v, rc, amax, qv);
    if (!rc.fast) {
        // a scale outside [2^-60, 2^60] (e.g. subnormal) can put |v / scale|
        // above qmax: apply the clamp of the definition
#pragma unroll
        for (int i = 0; i < VPC; ++i)
            qv[i] = fminf(fmaxf(qv[i], -q.qmax), q.qmax);
    }
    float t[VPC], cf[VPC], d[VPC];
    const f32x2 m2 = pack2(kMagic, kMagic);
#pragma unroll
    for (int i = 0; i < VPC / 2; ++i) {
        const f32x2 tt = add2(pack2(qv[2 * i], qv[2 * i + 1]), m2);
        const f32x2 cc = sub2(tt, m2);
        t[2 * i] = lo2(tt);
        t[2 * i + 1] = hi2(tt);
        cf[2 * i] = lo2(cc);
        cf[2 * i + 1] = hi2(cc);
    }
    scale_values<VPC>(cf, scale, d);
    if (STORE && o.valid) {
        const int64_t off = o.row * o.n + o.colq;
        uint32_t b[VPC]; // low bits of q + M hold the two's-complement code
#pragma unroll
        for (int i = 0; i < VPC; ++i)
            b[i] = __float_as_uint(t[i]);
        if (q.store == kInt8) {
            uint32_t w[VPC / 4];
#pragma unroll
            for (int k = 0; k < VPC / 4; ++k)
                w[k] = __byte_perm(__byte_perm(b[4 * k], b[4 * k + 1], 0x0040), __byte_perm(b[4 * k + 2], b[4 * k + 3], 0x0040),
                                   0x5410);
            uint8_t *dst = static_cast<uint8_t *>(o.values) + off;
            if constexpr (VPC == 4)
                *reinterpret_cast<uint32_t *>(dst) = w[0];
            else
                *reinterpret_cast<uint2 *>(dst) = make_uint2(w[0], w[1]);
        } else if (q.store == kInt16) {
            uint32_t w[VPC / 2];
#pragma unroll
            for (int k = 0; k < VPC / 2; ++k)
                w[k] = __byte_perm(b[2 * k], b[2 * k + 1], 0x5410);
            int16_t *dst = static_cast<int16_t *>(o.values) + off;
            if constexpr (VPC == 4)
                *reinterpret_cast<uint2 *>(dst) = make_uint2(w[0], w[1]);
            else
                *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        } else {
            uint32_t w = 0;
#pragma unroll
            for (int i = 0; i < VPC; ++i)
                w |= (b[i] & 0xfu) << (4 * i);
            uint8_t *dst = static_cast<uint8_t *>(o.values) + off / 2;
            if constexpr (VPC == 4)
                *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(w);
            else
                *reinterpret_cast<uint32_t *>(dst) = w;
        }
        if (row_amax < 0.0f && !(rs && rs->given) && (o.lane & (q.lanes - 1)) == 0)
            static_cast<float *>(o.scales)[o.row * (o.n / q.group) + o.colq / q.group] = scale;
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
__device__ __forceinline__ void store_fp4(uint32_t codes, const QOut &o)
{
    if (STORE && o.valid) {
        uint8_t *dst = static_cast<uint8_t *>(o.values) + (o.row * o.n + o.colq) / 2;
        if constexpr (VPC == 4)
            *reinterpret_cast<uint16_t *>(dst) = static_cast<uint16_t>(codes);
        else
            *reinterpret_cast<uint32_t *>(dst) = codes;
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

template <int VPC, bool STORE>
__device__ __forceinline__ float quant_nvfp4(const float (&v)[VPC], const Recip &rst, const QOut &o,
                                             const NvTable &tb)
{
    constexpr int kLanes = 16 / VPC;
    const float st = rst.b;
    const float amax = group_amax(local_amax<VPC>(v), kLanes);
    uint32_t sb = 0;
    if (st != 0.0f) {
        // (amax / 6) / st: two correctly rounded divisions
        Recip r6;
        r6.b = 6.0f;
        r6.nb = -6.0f;
        r6.y = 0x1.555556p-3f; // RN(1/6)
        r6.fast = true;
        const float a6 = amax >= 0x1p-30f ? div_fast(amax, r6) : __fdiv_rn(amax, 6.0f);
        const float bs = (rst.fast && a6 >= 0x1p-40f * st && __fmul_rn(a6, rst.y) < 0x1p126f)
                             ? div_fast(a6, rst)
                             : __fdiv_rn(a6, st);
        sb = cvt_e4m3x2(bs, 0.0f) & 0xffu;
    }
    Recip rd;
    rd.b = tb.den[sb];
    rd.nb = -rd.b;
    rd.y = tb.inv[sb];
    rd.fast = rd.b >= 0x1p-60f && rd.b <= 0x1p60f;
    const float denom = rd.b;
    float q[VPC], d[VPC];
    quotients<VPC>(v, rd, amax, q);
    const uint32_t codes = pack_e2m1<VPC>(q);
    unpack_e2m1<VPC>(codes, denom, d);
    store_fp4<VPC, STORE>(codes, o);
    if (STORE && o.valid && (o.lane & (kLanes - 1)) == 0)
        static_cast<uint8_t *>(o.scales)[o.row * (o.n / 16) + o.colq / 16] = static_cast<uint8_t>(sb);
    return err_energy<VPC>(v, d);
}

// MXFP4: block of 32 values (32 / VPC lanes), power-of-two scale 2^e stored as
// the E8M0 byte e + 127; v / 2^e is computed as v * 2^-e (the same correctly
// rounded value, since both scale factors are exact powers of two).
template <int VPC, bool STORE>
__device__ __forceinline__ float quant_mxfp4(const float (&v)[VPC], const QOut &o)
{
    constexpr int kLanes = 32 / VPC;
    const float amax = group_amax(local_amax<VPC>(v), kLanes);
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
        static_cast<uint8_t *>(o.scales)[o.row * (o.n / 32) + o.colq / 32] = static_cast<uint8_t>(byte);
    return err_energy<VPC>(v, d);
}

// Runtime-dispatched quantizer without stores (the energy-only pass).
template <int VPC>
__device__ __forceinline__ float quant_energy_only(const float (&v)[VPC], const QuantSpec &q, const Recip &rst,
                                                   const NvTable &tb)
{
    QOut o{nullptr, nullptr, 0, 0, 1, false, 0};
    switch (q.fmt) {
    case kFp8:
        return quant_fp8<VPC, false>(v, rst, o);
    case kInt:
        return quant_int<VPC, false>(v, q, o);
    case kNvfp4:
        return quant_nvfp4<VPC, false>(v, rst, o, tb);
    case kMxfp4:
        return quant_mxfp4<VPC, false>(v, o);
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
};

template <int SCORE>
__device__ __forceinline__ void scores(const float (&x)[8], const float *norms, int64_t col, bool in_k,
                                       float (&s)[8])
{
    if constexpr (SCORE == kWanda) {
        float4 n0 = make_float4(0.f, 0.f, 0.f, 0.f), n1 = n0;
        if (in_k) {
            n0 = __ldg(reinterpret_cast<const float4 *>(norms + col));
            n1 = __ldg(reinterpret_cast<const float4 *>(norms + col + 4));
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

template <typename T, int PAT, int SCORE, int FMT>
__device__ __forceinline__ void process_chunk(const PassParams &p, const float (&x)[8], int64_t row,
                                              int64_t col, int lane, const Recip &rst, const Recip &rstd,
                                              Acc &acc, float row_amax = -1.0f, const RowScale *rs = nullptr,
                                              const NvTable &tb = NvTable{nullptr, nullptr},
                                              const NvTable &tbd = NvTable{nullptr, nullptr})
{
    constexpr int VPC = PAT == kDense ? 8 : 4;
    const bool in_k = col < p.k;
    const bool valid = in_k && row < p.rows;
    float v[VPC];
    uint32_t meta = 0;
    float et, ep = 0.0f;

    if constexpr (PAT == kDense) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            v[i] = x[i];
        f32x2 t[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            t[i] = mul2(pack2(x[2 * i], x[2 * i + 1]), pack2(x[2 * i], x[2 * i + 1]));
        t[0] = add2(add2(t[0], t[1]), add2(t[2], t[3]));
        et = lo2(t[0]) + hi2(t[0]);
    } else if constexpr (PAT == kSparse24) {
        Group24 g0, g1;
        if constexpr (SCORE == kWanda) {
            float s[8];
            scores<SCORE>(x, p.norms, col, in_k, s);
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
        meta = g0.nib | (g1.nib << 4);
        et = g0.e_all + g1.e_all;
        ep = g0.e_drop + g1.e_drop;
    } else {
        // pairwise 4:8: pair p ranked by s_2p^2 + s_2p+1^2 (each product and
        // the sum rounded); for the magnitude score these are also the
        // pairs' energies
        f32x2 a = mul2(pack2(x[0], x[2]), pack2(x[0], x[2]));
        f32x2 b = mul2(pack2(x[1], x[3]), pack2(x[1], x[3]));
        const f32x2 e01 = add2(a, b);
        a = mul2(pack2(x[4], x[6]), pack2(x[4], x[6]));
        b = mul2(pack2(x[5], x[7]), pack2(x[5], x[7]));
        const f32x2 e23 = add2(a, b);
        float e[4] = {lo2(e01), hi2(e01), lo2(e23), hi2(e23)};
        float rank[4] = {e[0], e[1], e[2], e[3]};
        if constexpr (SCORE == kWanda) {
            float s[8];
            scores<SCORE>(x, p.norms, col, in_k, s);
            a = mul2(pack2(s[0], s[2]), pack2(s[0], s[2]));
            b = mul2(pack2(s[1], s[3]), pack2(s[1], s[3]));
            const f32x2 r01 = add2(a, b);
            a = mul2(pack2(s[4], s[6]), pack2(s[4], s[6]));
            b = mul2(pack2(s[5], s[7]), pack2(s[5], s[7]));
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
    }

    if constexpr (FMT == kAmax) {
        acc.amax_all = fmaxf(acc.amax_all, local_amax<8>(x));
        if constexpr (PAT != kDense)
            acc.amax_kept = fmaxf(acc.amax_kept, local_amax<4>(v));
        return;
    }
    acc.et += et;
    acc.ep += ep;

    // metadata
    if constexpr (PAT == kSparse24) {
        if (FMT != kEnergy && valid)
            p.meta[row * (p.k / 8) + col / 8] = static_cast<uint8_t>(meta);
    } else if constexpr (PAT == kSparse48) {
        const uint32_t other = __shfl_down_sync(kFull, meta, 1);
        if (FMT != kEnergy && valid && (lane & 1) == 0)
            p.meta[row * (p.k / 16) + col / 16] = static_cast<uint8_t>(meta | (other << 4));
    }

    const int64_t n = PAT == kDense ? p.k : p.k / 2;
    const QOut o{p.values, p.scales, row, PAT == kDense ? col : col / 2, n, valid, lane};
    float eq = 0.0f;
    if constexpr (FMT == kNone) {
        if (valid) {
            if constexpr (sizeof(T) == 2) {
                const uint32_t w0 = (__float_as_uint(v[0]) >> 16) | (__float_as_uint(v[1]) & 0xffff0000u);
                const uint32_t w1 = (__float_as_uint(v[2]) >> 16) | (__float_as_uint(v[3]) & 0xffff0000u);
                *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(p.values) + row * n + col / 2) =
                    make_uint2(w0, w1);
            } else {
                *reinterpret_cast<float4 *>(static_cast<float *>(p.values) + row * n + col / 2) =
                    make_float4(v[0], v[1], v[2], v[3]);
            }
        }
    } else if constexpr (FMT == kFp8) {
        eq = quant_fp8<VPC, true>(v, rst, o);
    } else if constexpr (FMT == kInt) {
        eq = quant_int<VPC, true>(v, p.q, o, row_amax, rs);
    } else if constexpr (FMT == kNvfp4) {
        eq = quant_nvfp4<VPC, true>(v, rst, o, tb);
    } else if constexpr (FMT == kMxfp4) {
        eq = quant_mxfp4<VPC, true>(v, o);
    } else if constexpr (FMT == kEnergy) {
        eq = quant_energy_only<VPC>(v, p.q, rst, tb);
        acc.eqd += quant_energy_only<8>(x, p.qd, rstd, tbd);
    }
    if constexpr (PAT == kDense)
        acc.eqd += eq;
    else
        acc.eq += eq;
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
        if (use > 0 && !mbar_wait(&empty[s], (use - 1) & 1)) {
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
            (void)mbar_wait(&full[s], last_use & 1);
        }
    }
}

template <typename T, int PAT, int SCORE, int FMT>
__global__ void __launch_bounds__(kThreads, 3) pass_kernel(const __grid_constant__ CUtensorMap map,
                                                           const PassParams pk)
{
    const PassParams p = operand_view(pk);
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *stages = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + kStages * kStageBytes);
    uint64_t *empty = full + kStages;
    double *red = reinterpret_cast<double *>(empty + kStages); // [kConsumerWarps][4]
    float *fred = reinterpret_cast<float *>(red + kConsumerWarps * 4); // [kConsumerWarps][2]
    uint32_t *flag = reinterpret_cast<uint32_t *>(fred + kConsumerWarps * 2);

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

    // ---- consumers ----
    float st = 0.0f, std_ = 0.0f;
    if constexpr (FMT == kFp8 || FMT == kNvfp4 || FMT == kEnergy) {
        st = tensor_scale(p.q);
        if (p.cta == 0 && tid == 0 && p.q.scale_out)
            *p.q.scale_out = st;
    }
    if constexpr (FMT == kEnergy)
        std_ = tensor_scale(p.qd);
    const Recip rst = make_recip(st), rstd = make_recip(std_);
    float *nvt = reinterpret_cast<float *>(flag + 4); // 2 x 256 floats
    if constexpr (FMT == kNvfp4 || FMT == kEnergy) {
        build_nv_table(nvt, st, tid);
        build_nv_table(nvt + 256, std_, tid);
        named_barrier_sync(1, kConsumers);
    }
    const NvTable tb{nvt, nvt + 128}, tbd{nvt + 256, nvt + 384};

    using E = Elem<T>;
    const int cpr_mask = (1 << p.log2_cpr) - 1;
    const bool energies = p.energy_out != nullptr;
    double e_total = 0.0, e_prune = 0.0, e_q = 0.0, e_qd = 0.0;
    Acc acc{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    uint32_t it = 0;
    for (int64_t t = p.cta; t < p.n_tiles; t += p.ctas_per_op, ++it) {
        const int s = it % kStages;
        if (!mbar_wait(&full[s], (it / kStages) & 1)) {
            record_error(p.err, 2);
            break;
        }
        const uint8_t *tile = stages + s * kStageBytes;
        typename E::Raw raw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (i < p.cpt)
                raw[i] = E::load(tile, tid + i * kConsumers);
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[s]);

        const int64_t rt = t / p.n_col_tiles, ct = t - rt * p.n_col_tiles;
        const int64_t row0 = rt * p.R, col0 = ct * p.W;
        acc.et = acc.ep = acc.eq = acc.eqd = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (i < p.cpt) {
                const int j = tid + i * kConsumers;
                const int64_t row = row0 + (j >> p.log2_cpr);
                const int64_t col = col0 + ((j & cpr_mask) << 3);
                float x[8];
                E::unpack(raw[i], x);
                process_chunk<T, PAT, SCORE, FMT>(p, x, row, col, lane, rst, rstd, acc, -1.0f, nullptr, tb, tbd);
            }
        }
        if constexpr (FMT != kAmax) {
            e_total += acc.et;
            e_prune += acc.ep;
            e_q += acc.eq;
            e_qd += acc.eqd;
        }
    }

    // ---- grid reductions (last CTA to finish reduces the partials) ----
    if constexpr (FMT == kAmax) {
        grid_reduce_amax<PAT>(p, acc.amax_kept, acc.amax_all, fred, flag, tid, lane, warp);
        return;
    } else {
        if (!energies)
            return;
        grid_reduce_energy(p, e_total, e_prune, e_q, e_qd, red, flag, tid, lane, warp);
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

template <typename T> struct RowChunk;
template <> struct RowChunk<__nv_bfloat16> {
    uint4 v;
    __device__ __forceinline__ void load(const void *row, int c)
    {
        v = __ldg(reinterpret_cast<const uint4 *>(row) + c);
    }
    __device__ __forceinline__ void unpack(float (&x)[8]) const
    {
        Elem<__nv_bfloat16>::Raw r{v};
        Elem<__nv_bfloat16>::unpack(r, x);
    }
};
template <> struct RowChunk<float> {
    float4 a, b;
    __device__ __forceinline__ void load(const void *row, int c)
    {
        a = __ldg(reinterpret_cast<const float4 *>(row) + 2 * c);
        b = __ldg(reinterpret_cast<const float4 *>(row) + 2 * c + 1);
    }
    __device__ __forceinline__ void unpack(float (&x)[8]) const
    {
        Elem<float>::Raw r{a, b};
        Elem<float>::unpack(r, x);
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
    const Recip no_recip = make_recip(0.0f);
    double e_total = 0.0, e_prune = 0.0, e_q = 0.0, e_qd = 0.0;
    for (int64_t row = static_cast<int64_t>(p.cta) * kConsumerWarps + warp; row < p.rows;
         row += static_cast<int64_t>(p.ctas_per_op) * kConsumerWarps) {
        const T *xr = x + p.op * p.x_bstride + row * ld;
        // sweep 1: the row amax of the values to quantize (for the magnitude
        // score the kept amax equals the amax of all values)
        float amax = 0.0f;
        for (int c0 = 0; c0 < nchunks; c0 += 256) {
            RowChunk<T> buf[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (c0 + 32 * u + lane < nchunks)
                    buf[u].load(xr, c0 + 32 * u + lane);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int c = c0 + 32 * u + lane;
                if (c < nchunks) {
                    float xv[8];
                    buf[u].unpack(xv);
                    if constexpr (PAT == kDense || SCORE == kMag) {
                        amax = fmaxf(amax, local_amax<8>(xv));
                    } else {
                        Acc a{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                        process_chunk<T, PAT, SCORE, kAmax>(p, xv, row, static_cast<int64_t>(c) * 8, lane,
                                                            no_recip, no_recip, a);
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
        // sweep 2: codes, metadata and energies; every lane takes part in each
        // step (4:8 metadata pairs lanes through a shuffle)
        Acc acc{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int c0 = 0; c0 < nchunks; c0 += 64) {
            RowChunk<T> buf[2];
#pragma unroll
            for (int u = 0; u < 2; ++u)
                if (c0 + 32 * u + lane < nchunks)
                    buf[u].load(xr, c0 + 32 * u + lane);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int c = c0 + 32 * u + lane;
                if (c0 + 32 * u < nchunks) {
                    float xv[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                    if (c < nchunks)
                        buf[u].unpack(xv);
                    process_chunk<T, PAT, SCORE, kInt>(p, xv, row, static_cast<int64_t>(c) * 8, lane, no_recip,
                                                       no_recip, acc, amax, &rs);
                }
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

template <typename T, int PAT, int SCORE, int FMT>
__global__ void __launch_bounds__(kThreads, 1) axis0_kernel(const __grid_constant__ CUtensorMap map,
                                                            const PassParams pk)
{
    const PassParams p = operand_view(pk);
    extern __shared__ __align__(1024) uint8_t smem[];
    uint8_t *stages = smem;
    uint8_t *Tb = smem + kStages * kStageBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(Tb + kAxis0TBytes);
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

    float st = 0.0f, std_ = 0.0f;
    if constexpr (FMT == kFp8 || FMT == kNvfp4 || FMT == kEnergy) {
        st = tensor_scale(p.q);
        if (p.cta == 0 && tid == 0 && p.q.scale_out)
            *p.q.scale_out = st;
    }
    if constexpr (FMT == kEnergy)
        std_ = tensor_scale(p.qd);
    const Recip rst = make_recip(st), rstd = make_recip(std_);
    float *nvt = reinterpret_cast<float *>(ready + 4); // 2 x 256 floats
    if constexpr (FMT == kNvfp4 || FMT == kEnergy) {
        build_nv_table(nvt, st, tid);
        build_nv_table(nvt + 256, std_, tid);
        named_barrier_sync(1, kConsumers);
    }
    const NvTable tb{nvt, nvt + 128}, tbd{nvt + 256, nvt + 384};
    using A0 = Axis0<T>;
    double e_total = 0.0, e_prune = 0.0, e_q = 0.0, e_qd = 0.0;
    Acc acc{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    uint32_t it = 0;
    for (int64_t t = p.cta; t < p.n_tiles; t += p.ctas_per_op, ++it) {
        const int s = it % kStages;
        // one thread waits for the stage and tells the others, so that every
        // consumer leaves the loop together if the wait gives up
        if (tid == 0) {
            const bool ok = mbar_wait(&full[s], (it / kStages) & 1);
            if (!ok)
                record_error(p.err, 5);
            *ready = ok;
        }
        named_barrier_sync(1, kConsumers);
        if (!*ready)
            break;
        A0::transpose(stages + s * kStageBytes, Tb, tid);
        named_barrier_sync(1, kConsumers); // S is read, T is written
        if (lane == 0)
            mbar_arrive(&empty[s]);
        typename Elem<T>::Raw raw[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (i < p.cpt) {
                const int j = tid + i * kConsumers;
                raw[i] = A0::load(Tb, j >> 4, j & 15);
            }
        named_barrier_sync(1, kConsumers); // T is read: the next tile may overwrite it
        const int64_t rt = t / p.n_col_tiles, ct = t - rt * p.n_col_tiles;
        const int64_t row0 = rt * A0::kRows, col0 = ct * kAxis0K;
        acc.et = acc.ep = acc.eq = acc.eqd = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (i < p.cpt) {
                const int j = tid + i * kConsumers;
                float x[8];
                Elem<T>::unpack(raw[i], x);
                process_chunk<T, PAT, SCORE, FMT>(p, x, row0 + (j >> 4), col0 + ((j & 15) << 3), lane, rst,
                                                  rstd, acc, -1.0f, nullptr, tb, tbd);
            }
        }
        if constexpr (FMT != kAmax) {
            e_total += acc.et;
            e_prune += acc.ep;
            e_q += acc.eq;
            e_qd += acc.eqd;
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
