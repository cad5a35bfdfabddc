// The pass along axis 1 for bf16 operands selected by magnitude, full-width
// rows (k a multiple of 64 and at least 1024), with one lane per 32
// consecutive elements, for the formats listed at stream_lb_for_fmt.
//
// Method: "Is 2:4 Sparsity Still Worth It? Semi-Structured Sparsity versus
// Quantization in LLM Inference" — intro (2:4 along the reduction axis), §2
// (magnitude score, round-to-nearest), §3 (formats; one read of the input, the
// kept values and indices written once), §4 (error energies), §6 (pairwise
// 4:8). The arithmetic of every value is that of the stream kernel
// (pass_impl.cuh); only the assignment of elements to lanes differs (MXFP4
// forms its error terms in quotient units and scales them by 2^2e, the same
// values in the normal range). The same kernel serves the passes over the
// operand rotated along k (rotate_lane32, the stream kernel's rotation value
// by value), and its loads run one unit ahead for the formats where that
// measured faster (LbPipe).
//
// Layout. A unit is 1024 consecutive columns of one row, served by one warp;
// lane L holds columns 32L .. 32L + 31 of it (four consecutive 16-byte
// chunks). The lane's 16 kept values (2:4, 4:8) or 32 values (dense) are then
// a whole NVFP4 block (2:4, 4:8), two NVFP4 blocks or one MXFP4 block (dense),
// or half an MXFP4 block (2:4, 4:8: two lanes): block maxima need no more than
// one shuffle. Each output of the lane is contiguous, so it is written with one
// or two vector stores instead of one small store per chunk. The division of a
// unit takes Markstein's correction when it applies to every lane of the warp
// (one vote per unit), else IEEE division for the whole warp: no per-chunk
// branches in the common case.
#pragma once

#include "pass_impl.cuh"

namespace ss24 {

// Whether a unit's loads are issued one unit ahead (a software pipeline, 16
// more registers), and the resident CTAs per SM that the register budget then
// allows: 3 (80 registers) with the pipeline, else 4 (64). The pipeline
// measured faster for the NVFP4 and MXFP4 passes of the 2:4 and dense
// patterns, slower for 4:8 and for INT (whose group reductions need the
// registers). Value 1: the next unit's words are copied into the current
// unit's registers each step; 2: two register buffers used in turn (the loop
// body twice), faster for NVFP4 (dense 146.2 -> 141.3 us on 16384 x 14336)
// and for 2:4 INT (INT8 g128 on 8 x 4096^2: 115.1 -> 112.4 us), slower for
// MXFP4 (dense 107.8 -> 112.1 us) and for 4:8 (NVFP4 154.6 -> 159.8 us).
template <int PAT, int FMT, bool ROT = false> struct LbPipe {
    static constexpr int value = ROT || !(PAT == kSparse24 || PAT == kDense) ? 0
                                 : (FMT == kNvfp4 || FMT == kInt)            ? 2
                                 : FMT == kMxfp4                             ? 1
                                                                             : 0;
};
// (the rotated passes hold a lane's 32 values as binary32 during the
// rotation: 3 CTAs)
template <int PAT, int FMT, bool ROT = false> struct LbOcc {
    static constexpr int value = (LbPipe<PAT, FMT, ROT>::value != 0 || ROT) ? 3 : 4;
};

// Block Hadamard rotation (block b = 2^log2b, 2 <= b <= 256), in place, of
// the 32 consecutive bf16 values a lane holds: the stream kernel's
// rotate_chunk for the lane-block layout. Binary32 arithmetic in stage order
// h = 1, 2, 4, ..., b/2 on the pairs (y_i, y_i+h): inside the lane for h <= 16
// (packed adds and subtracts), across lanes for h >= 32 with the partner lane
// ^ (h / 32), own * (+-1) + partner (exactly the rounded y_i + y_i+h in the
// lower lane, y_i - y_i+h in the upper); then times RN(1/sqrt(b)) and rounded
// to bf16 (nearest even). The same operations as rotate_chunk, value by
// value. The whole warp calls it.
// The in-lane stages h = 1 .. 2^(NS-1) of rotate_lane32 (NS <= 5), fully
// unrolled so that every index is a constant.
template <int NS> __device__ __forceinline__ void rotate_in_lane(float (&y)[32])
{
#pragma unroll
    for (int s = 0; s < NS; ++s) {
        const int h = 1 << s;
        // the 16 butterflies (i, i + h) with bit h of i clear, two per packed
        // add and subtract: the t-th such i is (t & (h - 1)) | ((t & ~(h - 1)) << 1)
#pragma unroll
        for (int t = 0; t < 16; t += 2) {
            const int a = (t & (h - 1)) | ((t & ~(h - 1)) << 1);
            const int b = ((t + 1) & (h - 1)) | (((t + 1) & ~(h - 1)) << 1);
            const f32x2 lo = pack2(y[a], y[b]), hi = pack2(y[a + h], y[b + h]);
            const f32x2 sm = add2(lo, hi), df = sub2(lo, hi);
            y[a] = lo2(sm), y[b] = hi2(sm), y[a + h] = lo2(df), y[b + h] = hi2(df);
        }
    }
}

__device__ __forceinline__ void rotate_lane32(uint4 (&w)[4], int log2b, float cb, int lane)
{
    float y[32];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t ws[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            y[8 * i + 2 * j] = __uint_as_float(ws[j] << 16);
            y[8 * i + 2 * j + 1] = __uint_as_float(ws[j] & 0xffff0000u);
        }
    }
    switch (log2b < 5 ? log2b : 5) {
    case 1:
        rotate_in_lane<1>(y);
        break;
    case 2:
        rotate_in_lane<2>(y);
        break;
    case 3:
        rotate_in_lane<3>(y);
        break;
    case 4:
        rotate_in_lane<4>(y);
        break;
    default:
        rotate_in_lane<5>(y);
        break;
    }
    for (int s = 5; s < log2b; ++s) {
        const int m = 1 << (s - 5);
        const float sg = (lane & m) ? -1.0f : 1.0f;
        const f32x2 sg2 = pack2(sg, sg);
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
            const float o0 = __shfl_xor_sync(kFull, y[i], m);
            const float o1 = __shfl_xor_sync(kFull, y[i + 1], m);
            const f32x2 r = fma2(pack2(y[i], y[i + 1]), sg2, pack2(o0, o1));
            y[i] = lo2(r), y[i + 1] = hi2(r);
        }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const __nv_bfloat162 h2 =
                __floats2bfloat162_rn(__fmul_rn(y[8 * i + 2 * j], cb), __fmul_rn(y[8 * i + 2 * j + 1], cb));
            o[j] = *reinterpret_cast<const uint32_t *>(&h2);
        }
        w[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

// The four values of a packed 2:4 selection in output order (group 0's kept
// values, then group 1's), as binary32.
__device__ __forceinline__ void kept4(uint32_t k0, uint32_t k1, float (&v)[4])
{
    v[0] = bf16_lo(k0);
    v[1] = bf16_lo(k1);
    v[2] = bf16_hi(k0);
    v[3] = bf16_hi(k1);
}

// FP8 codes of four values (bits 0..31, value 0 lowest) with the per-tensor
// scale rc; FAST: Markstein's correction for every quotient, else IEEE
// division (a zero scale giving zero codes). Adds the squared errors of the
// dequantized values to eq. The operations are quant_fp8_as's.
template <bool FAST>
__device__ __forceinline__ uint32_t fp8_codes4(const float (&v)[4], const Recip &rc, float &eq)
{
    float qn[4], decn[4], dn[4];
    neg_quotients<4>(v, rc, FAST, qn);
    uint16_t h[2];
#pragma unroll
    for (int t = 0; t < 2; ++t) {
        h[t] = cvt_e4m3x2h(qn[2 * t], qn[2 * t + 1]);
        const float2 f = e4m3x2h_to_f32(h[t]);
        decn[2 * t] = f.x;
        decn[2 * t + 1] = f.y;
    }
    scale_values<4>(decn, rc.b, dn);
    eq += err_energy_neg<4>(v, dn);
    return (static_cast<uint32_t>(h[0]) | (static_cast<uint32_t>(h[1]) << 16)) ^ 0x80808080u;
}

// E2M1 codes of four values of an NVFP4 block with divisor den and its
// reciprocal inv (bits 0..15); FAST as above. The operations are
// quant_nvfp4's: the codes are formed for the negated quotients and their sign
// bits flipped, the code values come decoded from the same conversion (-c),
// and the squared errors of v - RN(c den) are added to eq.
template <bool FAST>
__device__ __forceinline__ uint32_t nv_codes4(const float (&v)[4], float den, float inv, float &eq)
{
    Recip rd;
    rd.b = den;
    rd.y = inv;
    rd.nb = -den;
    rd.fast = true;
    float qn[4], dn[4];
    neg_quotients<4>(v, rd, FAST, qn);
    uint32_t d01, d23;
    const uint32_t codes = cvt_e2m1x4_dec(qn[0], qn[1], qn[2], qn[3], d01, d23);
    const float2 c01 = f16x2_to_f32(d01), c23 = f16x2_to_f32(d23);
    const float cn[4] = {c01.x, c01.y, c23.x, c23.y};
    scale_values<4>(cn, den, dn); // -RN(c den)
    eq += err_energy_neg<4>(v, dn);
    return codes ^ 0x8888u;
}

// The sum of a block's squared errors from the sum rs of its squared
// quotient-unit errors (q - c)^2, for a power-of-two scale f: v - c f = f (q -
// c) and every step scales exactly (normal range).
__device__ __forceinline__ float block_err(f32x2 rs, float f) { return f * (f * (lo2(rs) + hi2(rs))); }

// E2M1 codes of four values of an MXFP4 block (quotients v inv, inv = 2^-e,
// exact), adding (c - q)^2 to rs: the block's squared error is 2^2e times the
// sum, as v - c 2^e = 2^e (q - c) exactly. The codes are quant_mxfp4's.
__device__ __forceinline__ uint32_t mx_codes4(const float (&v)[4], float inv, f32x2 &rs)
{
    float q[4];
    scale_values<4>(v, inv, q);
    uint32_t d01, d23;
    const uint32_t codes = cvt_e2m1x4_dec(q[0], q[1], q[2], q[3], d01, d23);
    const f32x2 r01 = f16x2_sub_f32(d01, q[0], q[1]), r23 = f16x2_sub_f32(d23, q[2], q[3]);
    rs = fma2(r23, r23, fma2(r01, r01, rs));
    return codes;
}

// The NVFP4 scale of a block with amax am: its E4M3 code, divisor and
// reciprocal, and whether Markstein's correction applies to all its quotients.
struct NvScale {
    uint32_t code;
    float den, inv;
    bool fast;
};

__device__ __forceinline__ NvScale nv_scale(float am, const PassConsts &c)
{
    NvScale s;
    s.code = nv_block_code(am, c.rst);
    s.den = c.tb.den[s.code];
    s.inv = c.tb.inv[s.code];
    s.fast = s.den >= 0x1p-60f && s.den <= 0x1p60f && __fmul_rn(am, s.inv) < 0x1p126f;
    return s;
}

// The MXFP4 scale of a block with amax am: E8M0 byte, 2^-e and 2^e (zero
// block: byte 0, zero factors), as quant_mxfp4 takes them.
struct MxScale {
    uint32_t byte;
    float inv, mult;
};

__device__ __forceinline__ MxScale mx_scale(float am)
{
    MxScale s{0u, 0.0f, 0.0f};
    if (am != 0.0f) {
        const int e = mx_shared_exponent(am);
        s.byte = static_cast<uint32_t>(e + 127);
        s.inv = exp2_int(-e);
        s.mult = exp2_int(e);
    }
    return s;
}

// An INT group's scale (amax / qmax), its reciprocal and its division path,
// as quant_int forms them.
struct IntScale {
    float scale;
    Recip rc;
    bool fast;
};

__device__ __forceinline__ IntScale int_group_scale(float amax, const QuantSpec &q)
{
    IntScale s;
    s.scale = int_scale(amax, q);
    s.rc = make_recip(s.scale);
    s.fast = quot_fast(s.rc, amax);
    return s;
}

// INT codes of four values with their group's scale, as quant_int forms them:
// the two's-complement codes in the low bits of b[0..3] (the bits of M + q,
// M the rounding constant), and the squared errors added to eq. FAST:
// Markstein's correction for every quotient, else IEEE division and the clamp
// to [-qmax, qmax].
template <bool FAST>
__device__ __forceinline__ void int_codes4(const float (&v)[4], const IntScale &s, float qmax, uint32_t (&b)[4],
                                           float &eq)
{
    float qn[4], d[4], cf[4];
    neg_quotients<4>(v, s.rc, FAST, qn);
    if constexpr (!FAST) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            qn[i] = fminf(fmaxf(qn[i], -qmax), qmax);
    }
    const f32x2 m2 = pack2(kMagic, kMagic);
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const f32x2 tt = sub2(m2, pack2(qn[2 * i], qn[2 * i + 1]));
        const f32x2 cc = sub2(tt, m2);
        b[2 * i] = __float_as_uint(lo2(tt));
        b[2 * i + 1] = __float_as_uint(hi2(tt));
        cf[2 * i] = lo2(cc);
        cf[2 * i + 1] = hi2(cc);
    }
    scale_values<4>(cf, s.scale, d);
    eq += err_energy<4>(v, d);
}

// The INT part of a lane-block unit. The lane holds NQ quads of four values
// (the kept values of four chunks: NQ = 4); values(j, v) gives quad j, qm[j]
// its largest magnitude. A group of g values spans g / 4 quads: inside the
// lane when that is at most NQ, else over g / (4 NQ) lanes (an xor reduction
// of their maxima). With STORE, codes are stored contiguously per lane (int8,
// int16 or packed nibbles) and a group's scale by the lane holding its first
// quad; without, only the energy is formed.
template <int NQ, bool STORE, typename Values>
__device__ __forceinline__ void lb_int(const QuantSpec &q, const Values &values, const float (&qm)[NQ], bool valid,
                                       bool wide, const ChunkOut &o, float &eq)
{
    float gm[NQ];
    const int gq = q.group >> 2; // quads per group
#pragma unroll
    for (int j = 0; j < NQ; ++j)
        gm[j] = qm[j];
#pragma unroll
    for (int span = 1; span < NQ; span <<= 1)
        if (span < gq)
#pragma unroll
            for (int j = 0; j < NQ; ++j)
                gm[j] = fmaxf(gm[j], gm[j ^ span]);
    if (gq > NQ) {
        float m = gm[0];
        for (int off = 1; off < gq / NQ; off <<= 1)
            m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
#pragma unroll
        for (int j = 0; j < NQ; ++j)
            gm[j] = m;
    }
    // one scale per group (a group's quads share its first quad's)
    IntScale sc[NQ];
    bool fast = true;
#pragma unroll
    for (int j = 0; j < NQ; ++j) {
        if (j == 0 || j % gq == 0)
            sc[j] = int_group_scale(gm[j], q);
        else
            sc[j] = sc[j - 1];
        fast = fast && sc[j].fast;
    }
    uint32_t b[NQ][4];
    if (__all_sync(kFull, fast || !valid)) {
#pragma unroll
        for (int j = 0; j < NQ; ++j) {
            float v[4];
            values(j, v);
            int_codes4<true>(v, sc[j], q.qmax, b[j], eq);
        }
    } else {
#pragma unroll
        for (int j = 0; j < NQ; ++j) {
            float v[4];
            values(j, v);
            if (sc[j].fast)
                int_codes4<true>(v, sc[j], q.qmax, b[j], eq);
            else
                int_codes4<false>(v, sc[j], q.qmax, b[j], eq);
        }
    }
    if (!STORE || !valid)
        return;
    if (q.store == kInt8) {
        uint32_t wd[NQ];
#pragma unroll
        for (int j = 0; j < NQ; ++j)
            wd[j] = __byte_perm(__byte_perm(b[j][0], b[j][1], 0x0040), __byte_perm(b[j][2], b[j][3], 0x0040), 0x5410);
        if constexpr (NQ == 4) {
            *reinterpret_cast<uint4 *>(o.val) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        } else {
            const uint4 a = make_uint4(wd[0], wd[1], wd[2], wd[3]), c2 = make_uint4(wd[4], wd[5], wd[6], wd[7]);
            if (wide) {
                st32(o.val, a, c2);
            } else {
                reinterpret_cast<uint4 *>(o.val)[0] = a;
                reinterpret_cast<uint4 *>(o.val)[1] = c2;
            }
        }
    } else if (q.store == kInt16) {
        uint32_t wd[2 * NQ];
#pragma unroll
        for (int j = 0; j < NQ; ++j) {
            wd[2 * j] = __byte_perm(b[j][0], b[j][1], 0x5410);
            wd[2 * j + 1] = __byte_perm(b[j][2], b[j][3], 0x5410);
        }
#pragma unroll
        for (int h = 0; h < NQ / 4; ++h) {
            const uint4 a = make_uint4(wd[8 * h], wd[8 * h + 1], wd[8 * h + 2], wd[8 * h + 3]);
            const uint4 c2 = make_uint4(wd[8 * h + 4], wd[8 * h + 5], wd[8 * h + 6], wd[8 * h + 7]);
            if (wide) {
                st32(o.val + 32 * h, a, c2);
            } else {
                reinterpret_cast<uint4 *>(o.val + 32 * h)[0] = a;
                reinterpret_cast<uint4 *>(o.val + 32 * h)[1] = c2;
            }
        }
    } else {
        uint32_t hw[NQ];
#pragma unroll
        for (int j = 0; j < NQ; ++j)
            hw[j] = (b[j][0] & 0xfu) | ((b[j][1] & 0xfu) << 4) | ((b[j][2] & 0xfu) << 8) | ((b[j][3] & 0xfu) << 12);
        if constexpr (NQ == 4)
            *reinterpret_cast<uint2 *>(o.val) = make_uint2(hw[0] | (hw[1] << 16), hw[2] | (hw[3] << 16));
        else
            *reinterpret_cast<uint4 *>(o.val) =
                make_uint4(hw[0] | (hw[1] << 16), hw[2] | (hw[3] << 16), hw[4] | (hw[5] << 16), hw[6] | (hw[7] << 16));
    }
    float *scales = reinterpret_cast<float *>(o.scale);
    if (gq >= NQ) {
        if ((o.lane & (gq / NQ - 1)) == 0)
            *scales = sc[0].scale;
    } else {
        // NQ / gq groups in the lane, their scales consecutive
#pragma unroll
        for (int j = 0; j < NQ; ++j)
            if (j % gq == 0)
                scales[j / gq] = sc[j].scale;
    }
}

// One unit's lane: the four chunks w[0..3] (columns 32L .. 32L + 31 of the
// unit), valid when the lane's columns lie inside the operand (then all 32
// do). o points at the lane's first output bytes. The whole warp calls it.
template <int PAT, int FMT>
__device__ __forceinline__ void lb_unit(const PassConsts &c, const QuantSpec &q, const uint4 (&w)[4], bool valid,
                                        bool wide, const ChunkOut &o, Acc &acc)
{
    // a lane's 32 output bytes: one 32-byte store where aligned, else two
    auto store32 = [&](const uint4 &a, const uint4 &b) {
        if (wide) {
            st32(o.val, a, b);
        } else {
            reinterpret_cast<uint4 *>(o.val)[0] = a;
            reinterpret_cast<uint4 *>(o.val)[1] = b;
        }
    };
    float eq = 0.0f;
    if constexpr (PAT == kSparse24 || PAT == kSparse48) {
        // selection: kept values (as packed bf16 pairs for 2:4 by magnitude,
        // else binary32), metadata and the chunks' energies
        constexpr bool kPk = PAT == kSparse24;
        uint32_t k0[4], k1[4];
        float v48[4][4];
        float cmax[4];
        uint32_t meta = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if constexpr (kPk) {
                const Pair24 g = pair24_bf16(w[i].x, w[i].y, w[i].z, w[i].w);
                k0[i] = g.k0;
                k1[i] = g.k1;
                meta |= g.meta << (8 * i);
                acc.et += g.e_all;
                acc.ep += g.e_drop;
            } else {
                Elem<__nv_bfloat16>::Raw raw;
                raw.v = w[i];
                const ChunkOut none{nullptr, nullptr, nullptr, nullptr, false, 0};
                const Sel<4> s = select_chunk<__nv_bfloat16, PAT, kMag>(raw, none);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    v48[i][j] = s.v[j];
                cmax[i] = s.vmax;
                meta |= s.meta << ((PAT == kSparse24 ? 8 : 4) * i);
                acc.et += s.et;
                acc.ep += s.ep;
            }
        }
        auto values = [&](int i, float (&v)[4]) {
            if constexpr (kPk) {
                kept4(k0[i], k1[i], v);
            } else {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    v[j] = v48[i][j];
            }
        };
        // the largest kept magnitude of the lane (16 values)
        auto lane_amax = [&]() {
            if constexpr (kPk) {
                const uint32_t m = bf16x2_maxabs(bf16x2_maxabs(bf16x2_maxabs(k0[0], k1[0]), bf16x2_maxabs(k0[1], k1[1])),
                                                 bf16x2_maxabs(bf16x2_maxabs(k0[2], k1[2]), bf16x2_maxabs(k0[3], k1[3])));
                return bf16x2_hmax(m);
            } else {
                return fmaxf(fmaxf(cmax[0], cmax[1]), fmaxf(cmax[2], cmax[3]));
            }
        };
        if constexpr (FMT == kNone) {
            uint32_t kw[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if constexpr (kPk) {
                    kw[2 * i] = __byte_perm(k0[i], k1[i], 0x5410);
                    kw[2 * i + 1] = __byte_perm(k0[i], k1[i], 0x7632);
                } else {
                    kw[2 * i] = (__float_as_uint(v48[i][0]) >> 16) | (__float_as_uint(v48[i][1]) & 0xffff0000u);
                    kw[2 * i + 1] = (__float_as_uint(v48[i][2]) >> 16) | (__float_as_uint(v48[i][3]) & 0xffff0000u);
                }
            }
            if (valid)
                store32(make_uint4(kw[0], kw[1], kw[2], kw[3]), make_uint4(kw[4], kw[5], kw[6], kw[7]));
        } else if constexpr (FMT == kFp8) {
            bool bad = false;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if constexpr (kPk)
                    bad |= c.guard && bf16x2_max_ge_abs(k0[i], k1[i], c.lim2);
                else
                    bad |= c.guard && !(__fmul_rn(cmax[i], c.rst.y) < 0x1p126f);
            }
            uint32_t codes[4];
            if (c.rst.fast && !__any_sync(kFull, bad)) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float v[4];
                    values(i, v);
                    codes[i] = fp8_codes4<true>(v, c.rst, eq);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float v[4];
                    values(i, v);
                    bool fi;
                    if constexpr (kPk)
                        fi = c.rst.fast && !(c.guard && bf16x2_max_ge_abs(k0[i], k1[i], c.lim2));
                    else
                        fi = c.guard ? quot_fast(c.rst, cmax[i]) : c.rst.fast;
                    codes[i] = fi ? fp8_codes4<true>(v, c.rst, eq) : fp8_codes4<false>(v, c.rst, eq);
                }
            }
            if (valid)
                *reinterpret_cast<uint4 *>(o.val) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
        } else if constexpr (FMT == kNvfp4) {
            const float am = lane_amax();
            const NvScale s = nv_scale(am, c);
            uint32_t codes[4];
            if (__all_sync(kFull, s.fast || !valid)) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float v[4];
                    values(i, v);
                    codes[i] = nv_codes4<true>(v, s.den, s.inv, eq);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float v[4];
                    values(i, v);
                    codes[i] = nv_codes4<false>(v, s.den, s.inv, eq);
                }
            }
            if (valid) {
                *reinterpret_cast<uint2 *>(o.val) =
                    make_uint2(codes[0] | (codes[1] << 16), codes[2] | (codes[3] << 16));
                *o.scale = static_cast<uint8_t>(s.code);
            }
        } else if constexpr (FMT == kMxfp4) {
            // a block of 32 kept values: this lane and its neighbour
            float am = lane_amax();
            am = fmaxf(am, __shfl_xor_sync(kFull, am, 1));
            const MxScale s = mx_scale(am);
            uint32_t codes[4];
            f32x2 rs = pack2(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v[4];
                values(i, v);
                codes[i] = mx_codes4(v, s.inv, rs);
            }
            eq = block_err(rs, s.mult);
            if (valid) {
                *reinterpret_cast<uint2 *>(o.val) =
                    make_uint2(codes[0] | (codes[1] << 16), codes[2] | (codes[3] << 16));
                if ((o.lane & 1) == 0)
                    *o.scale = static_cast<uint8_t>(s.byte);
            }
        } else if constexpr (FMT == kInt) {
            float qm[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                if constexpr (kPk)
                    qm[i] = bf16x2_hmax(bf16x2_maxabs(k0[i], k1[i]));
                else
                    qm[i] = cmax[i];
            }
            lb_int<4, true>(q, values, qm, valid, wide, o, eq);
        }
        // (a lane outside the operand holds zeros; its scale may be zero and
        // its quotients then not finite: it contributes no energy)
        if (!valid)
            eq = 0.0f;
        if (valid) {
            if constexpr (PAT == kSparse24)
                *reinterpret_cast<uint32_t *>(o.meta) = meta;
            else
                *reinterpret_cast<uint16_t *>(o.meta) = static_cast<uint16_t>(meta);
        }
        acc.eq += eq;
    } else {
        // dense: the 32 values of the lane
        auto values = [&](int i, int half, float (&v)[4]) {
            const uint32_t a = half ? w[i].z : w[i].x, b = half ? w[i].w : w[i].y;
            v[0] = bf16_lo(a);
            v[1] = bf16_hi(a);
            v[2] = bf16_lo(b);
            v[3] = bf16_hi(b);
        };
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float x[8];
            Elem<__nv_bfloat16>::Raw raw;
            raw.v = w[i];
            Elem<__nv_bfloat16>::unpack(raw, x);
            f32x2 t[4];
#pragma unroll
            for (int j = 0; j < 4; ++j)
                t[j] = pack2(x[2 * j], x[2 * j + 1]);
            acc.et += sq_sum2<4>(t);
        }
        auto chunk_max2 = [&](int i) { return bf16x2_maxabs(bf16x2_maxabs(w[i].x, w[i].y), bf16x2_maxabs(w[i].z, w[i].w)); };
        if constexpr (FMT == kFp8) {
            bool bad = false;
#pragma unroll
            for (int i = 0; i < 4; ++i)
                bad |= c.guard && (bf16x2_any_ge_abs(w[i].x, w[i].y, c.lim2) || bf16x2_any_ge_abs(w[i].z, w[i].w, c.lim2));
            uint32_t codes[8];
            if (c.rst.fast && !__any_sync(kFull, bad)) {
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float v[4];
                        values(i, h, v);
                        codes[2 * i + h] = fp8_codes4<true>(v, c.rst, eq);
                    }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const bool fi = c.guard ? quot_fast(c.rst, bf16x2_hmax(chunk_max2(i))) : c.rst.fast;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        float v[4];
                        values(i, h, v);
                        codes[2 * i + h] = fi ? fp8_codes4<true>(v, c.rst, eq) : fp8_codes4<false>(v, c.rst, eq);
                    }
                }
            }
            if (valid)
                store32(make_uint4(codes[0], codes[1], codes[2], codes[3]), make_uint4(codes[4], codes[5], codes[6], codes[7]));
        } else if constexpr (FMT == kNvfp4) {
            // two blocks of 16: chunks 0-1 and 2-3
            const NvScale s0 = nv_scale(bf16x2_hmax(bf16x2_maxabs(chunk_max2(0), chunk_max2(1))), c);
            const NvScale s1 = nv_scale(bf16x2_hmax(bf16x2_maxabs(chunk_max2(2), chunk_max2(3))), c);
            uint32_t codes[4];
            if (__all_sync(kFull, (s0.fast && s1.fast) || !valid)) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const NvScale &s = i < 2 ? s0 : s1;
                    float v[4], u[4];
                    values(i, 0, v);
                    values(i, 1, u);
                    codes[i] = nv_codes4<true>(v, s.den, s.inv, eq) | (nv_codes4<true>(u, s.den, s.inv, eq) << 16);
                }
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const NvScale &s = i < 2 ? s0 : s1;
                    float v[4], u[4];
                    values(i, 0, v);
                    values(i, 1, u);
                    codes[i] = nv_codes4<false>(v, s.den, s.inv, eq) | (nv_codes4<false>(u, s.den, s.inv, eq) << 16);
                }
            }
            if (valid) {
                *reinterpret_cast<uint4 *>(o.val) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
                *reinterpret_cast<uint16_t *>(o.scale) = static_cast<uint16_t>(s0.code | (s1.code << 8));
            }
        } else if constexpr (FMT == kMxfp4) {
            // one block of 32: the lane
            const MxScale s = mx_scale(bf16x2_hmax(
                bf16x2_maxabs(bf16x2_maxabs(chunk_max2(0), chunk_max2(1)), bf16x2_maxabs(chunk_max2(2), chunk_max2(3)))));
            uint32_t codes[4];
            f32x2 rs = pack2(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v[4], u[4];
                values(i, 0, v);
                values(i, 1, u);
                codes[i] = mx_codes4(v, s.inv, rs) | (mx_codes4(u, s.inv, rs) << 16);
            }
            eq = block_err(rs, s.mult);
            if (valid) {
                *reinterpret_cast<uint4 *>(o.val) = make_uint4(codes[0], codes[1], codes[2], codes[3]);
                *o.scale = static_cast<uint8_t>(s.byte);
            }
        }
        acc.eqd += valid ? eq : 0.0f;
    }
}

// The kernel: persistent, 8 warps per CTA, a warp per unit (1024 columns of
// one row), units u = warp index, warp index + number of warps, ... among the
// CTAs serving one operand of a batch; energies reduced as in stream_kernel.
//
// ROT: the pass over the operand rotated along k (rotate_lane32 right after
// the loads).
template <int PAT, int FMT, bool ROT = false>
__global__ void __launch_bounds__(kStreamThreads, (LbOcc<PAT, FMT, ROT>::value))
    stream_lb_kernel(const __grid_constant__ PassParams pk)
{
    using T = __nv_bfloat16;
    const PassParams &p = pk;
    const int op = static_cast<int>(blockIdx.x) / pk.ctas_per_op;
    const int cta = static_cast<int>(blockIdx.x) - op * pk.ctas_per_op;
    __shared__ double red[kStreamWarps * 4];
    __shared__ uint32_t flag;
    __shared__ float nvt[FMT == kNvfp4 ? 512 : 4];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    grid_dependency_wait();
    grid_dependents_launch();
    const PassConsts c = make_consts<FMT>(operand_view(pk), tid, kStreamThreads, nvt);
    const OutBase ob = out_base(pk, op);
    const T *x = static_cast<const T *>(p.x) + op * p.x_bstride;

    const int tw = p.ctas_per_op * kStreamWarps;
    const int u0 = cta * kStreamWarps + warp;
    int ua = u0 / p.units_b, ub = u0 - ua * p.units_b;
    const int sa = tw / p.units_b, sb = tw - sa * p.units_b;
    double e_total = 0.0, e_prune = 0.0, e_q = 0.0, e_qd = 0.0;
    Acc acc{0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    // a unit's loads (k is a multiple of 64: a lane is wholly in or out)
    auto load = [&](int a, int b, uint4 (&w)[4]) {
        const int64_t col = static_cast<int64_t>(b) * 1024 + 32 * lane;
        const bool ok = a < p.units_a && col < p.k;
        const T *xp = x + static_cast<int64_t>(a) * p.ld + col;
        if (PAT == kSparse48 && (p.lb_wide & 1)) {
            ld_stream32(xp, ok, w[0], w[1]);
            ld_stream32(xp + 16, ok, w[2], w[3]);
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i)
                w[i] = ld_stream(xp + 8 * i, ok);
        }
    };
    // one unit: its arithmetic and stores, and its energies added up
    auto unit = [&](uint4 (&w)[4], int a, int b) {
        const int64_t row = a;
        const int64_t col = static_cast<int64_t>(b) * 1024 + 32 * lane;
        const bool valid = col < p.k;
        if constexpr (ROT)
            rotate_lane32(w, p.rot_log2b, p.rot_scale, lane);
        const ChunkOut o = make_out<T, PAT, FMT>(p, ob, row, col, valid, lane);
        acc.et = acc.ep = acc.eq = acc.eqd = 0.0f;
        lb_unit<PAT, FMT>(c, p.q, w, valid, (p.lb_wide & 2) != 0, o, acc);
        e_total += acc.et;
        if constexpr (PAT != kDense)
            e_prune += acc.ep;
        if constexpr (FMT != kNone && PAT != kDense)
            e_q += acc.eq;
        if constexpr (FMT != kNone && PAT == kDense)
            e_qd += acc.eqd;
    };
    auto advance = [&](int &a, int &b) {
        a += sa;
        b += sb;
        if (b >= p.units_b) {
            b -= p.units_b;
            ++a;
        }
    };
    // (with the pipeline, a unit past the end loads nothing)
    constexpr int kPipe = LbPipe<PAT, FMT, ROT>::value;
    if constexpr (kPipe == 2) {
        uint4 wa[4], wb[4];
        load(ua, ub, wa);
        while (ua < p.units_a) {
            int na = ua, nb = ub;
            advance(na, nb);
            load(na, nb, wb);
            unit(wa, ua, ub);
            ua = na;
            ub = nb;
            if (ua >= p.units_a)
                break;
            advance(na, nb);
            load(na, nb, wa);
            unit(wb, ua, ub);
            ua = na;
            ub = nb;
        }
    } else if constexpr (kPipe == 1) {
        uint4 wn[4];
        load(ua, ub, wn);
        while (ua < p.units_a) {
            uint4 w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
                w[i] = wn[i];
            int na = ua, nb = ub;
            advance(na, nb);
            load(na, nb, wn);
            unit(w, ua, ub);
            ua = na;
            ub = nb;
        }
    } else {
        while (ua < p.units_a) {
            uint4 w[4];
            load(ua, ub, w);
            unit(w, ua, ub);
            advance(ua, ub);
        }
    }
    const PassParams v = operand_view(pk);
    if (!v.energy_out)
        return;
    grid_reduce_energy(v, e_total, e_prune, e_q, e_qd, red, &flag, tid, lane, warp);
}

// The amax pass over the rotated operand in the lane-block layout (bf16, by
// magnitude, full-width rows with k a multiple of 64, no per-row output): the
// largest magnitude of all rotated values and of the kept ones (2:4 keeps
// every group's largest value; pairwise 4:8 can drop it and takes the
// selection's own maximum), reduced over the grid as the stream kernel's amax
// mode does (grid_reduce_amax: the operand's two maxima, the tensor scale or
// the caller's amax).
template <int PAT>
__global__ void __launch_bounds__(kStreamThreads, 3) stream_lb_amax_rot_kernel(const __grid_constant__ PassParams pk)
{
    using T = __nv_bfloat16;
    const PassParams &p = pk;
    const int op = static_cast<int>(blockIdx.x) / pk.ctas_per_op;
    const int cta = static_cast<int>(blockIdx.x) - op * pk.ctas_per_op;
    __shared__ float fred[kStreamWarps * 2];
    __shared__ uint32_t flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    grid_dependency_wait();
    grid_dependents_launch();
    const T *x = static_cast<const T *>(p.x) + op * p.x_bstride;
    const int tw = p.ctas_per_op * kStreamWarps;
    const int u0 = cta * kStreamWarps + warp;
    int ua = u0 / p.units_b, ub = u0 - ua * p.units_b;
    const int sa = tw / p.units_b, sb = tw - sa * p.units_b;
    float amax_all = 0.0f, amax_kept = 0.0f;
    while (ua < p.units_a) {
        const int64_t col = static_cast<int64_t>(ub) * 1024 + 32 * lane;
        const bool valid = col < p.k; // (a lane outside the row holds zeros)
        const T *xp = x + static_cast<int64_t>(ua) * p.ld + col;
        uint4 w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = ld_stream(xp + 8 * i, valid);
        rotate_lane32(w, p.rot_log2b, p.rot_scale, lane);
        uint32_t m2 = bf16x2_maxabs(bf16x2_maxabs(w[0].x, w[0].y), bf16x2_maxabs(w[0].z, w[0].w));
#pragma unroll
        for (int i = 1; i < 4; ++i)
            m2 = bf16x2_maxabs(m2, bf16x2_maxabs(bf16x2_maxabs(w[i].x, w[i].y), bf16x2_maxabs(w[i].z, w[i].w)));
        const float all = bf16x2_hmax(m2);
        amax_all = fmaxf(amax_all, all);
        if constexpr (PAT == kSparse48) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                Elem<T>::Raw raw;
                raw.v = w[i];
                const ChunkOut none{nullptr, nullptr, nullptr, nullptr, false, 0};
                amax_kept = fmaxf(amax_kept, select_chunk<T, PAT, kMag>(raw, none).vmax);
            }
        } else {
            amax_kept = fmaxf(amax_kept, all);
        }
        ua += sa;
        ub += sb;
        if (ub >= p.units_b) {
            ub -= p.units_b;
            ++ua;
        }
    }
    const PassParams v = operand_view(pk);
    grid_reduce_amax<PAT>(v, amax_kept, amax_all, fred, &flag, tid, lane, warp);
}

// The lane-block kernel for (pattern, format), or nullptr where it has none.
// The lane-block kernel serves the (pattern, score, format) combinations where
// it measured faster than the stream kernel on 16384 x 14336 and 8 x 4096^2
// operands: NVFP4 and MXFP4 (2:4 and dense), pairwise 4:8 with FP8 or bf16
// kept values, and 2:4 INT with groups, all by magnitude. The others stay with
// the stream kernel: bf16 and FP8 of 2:4 and of the dense pattern (few
// instructions per chunk: bound by memory, where the stream kernel's loads of
// 512 contiguous bytes per warp instruction are faster), dense INT (its eight
// quads per lane need more than 64 registers; at 3 CTAs per SM it measured 8%
// slower), INT with one scale per row, and the Wanda score (a lane's 32 column
// norms are 128 scattered bytes per load; staged in shared memory instead,
// with conflict-free reads, the 2:4 Wanda passes still measured 9 - 40%
// slower).
template <int PAT, bool ROT = false> const void *stream_lb_for_fmt(int fmt)
{
    switch (fmt) {
    case kNone:
    case kFp8:
        if constexpr (PAT == kSparse48)
            return fmt == kNone ? reinterpret_cast<const void *>(&stream_lb_kernel<PAT, kNone, ROT>)
                                : reinterpret_cast<const void *>(&stream_lb_kernel<PAT, kFp8, ROT>);
        break;
    case kNvfp4:
        return reinterpret_cast<const void *>(&stream_lb_kernel<PAT, kNvfp4, ROT>);
    case kMxfp4:
        return reinterpret_cast<const void *>(&stream_lb_kernel<PAT, kMxfp4, ROT>);
    case kInt:
        if constexpr (PAT == kSparse24)
            return reinterpret_cast<const void *>(&stream_lb_kernel<PAT, kInt, ROT>);
        break;
    }
    return nullptr;
}

} // namespace ss24
