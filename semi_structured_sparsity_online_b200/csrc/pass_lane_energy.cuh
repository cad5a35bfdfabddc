// The read-only energy pass in the lane-block form: bf16 operands by
// magnitude, full-width rows with k a multiple of 64, the 2:4 side's format
// and the dense side's format fixed at compile time.
//
// Method: "Is 2:4 Sparsity Still Worth It?" §4 — the energies of both sides of
// the comparison from one read of the operand: E_total, E_prune (the dropped
// values), E_q of the kept values quantized to the 2:4 side's format (2m
// bits), E_q,dense of every value quantized to the dense side's format (m + 1
// bits). Nothing but the energies is written. The arithmetic of every value is
// that of the stream kernel's energy pass (MXFP4's error terms formed in
// quotient units and scaled by 2^2e, the same values in the normal range); it
// also serves the operand rotated along k (ROT). A lane holds 32 consecutive
// elements as in the lane-block pass (pass_lane_block.cuh), so each side's
// blocks and groups are reduced inside the lane or over a few lanes, and
// each side's division path is voted once per unit.
#pragma once

#include "pass_lane_block.cuh"

namespace ss24 {

// The 2:4 side's quantization error energy of a lane's kept values (four
// quads: kept4 of each chunk's packed selection).
template <int SF>
__device__ __forceinline__ float lb_sparse_energy(const PassConsts &c, const QuantSpec &q, const uint32_t (&k0)[4],
                                                  const uint32_t (&k1)[4], bool valid)
{
    float eq = 0.0f;
    auto values = [&](int i, float (&v)[4]) { kept4(k0[i], k1[i], v); };
    auto quad_amax = [&](int i) { return bf16x2_hmax(bf16x2_maxabs(k0[i], k1[i])); };
    if constexpr (SF == kFp8) {
        bool fast[4], all = true;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            fast[i] = c.guard ? quot_fast(c.rst, quad_amax(i)) : c.rst.fast;
            all = all && fast[i];
        }
        if (__all_sync(kFull, all || !valid)) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v[4];
                values(i, v);
                (void)fp8_codes4<true>(v, c.rst, eq);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v[4];
                values(i, v);
                if (fast[i])
                    (void)fp8_codes4<true>(v, c.rst, eq);
                else
                    (void)fp8_codes4<false>(v, c.rst, eq);
            }
        }
    } else if constexpr (SF == kNvfp4) {
        float am = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            am = fmaxf(am, quad_amax(i));
        const NvScale s = nv_scale(am, c);
        if (__all_sync(kFull, s.fast || !valid)) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v[4];
                values(i, v);
                (void)nv_codes4<true>(v, s.den, s.inv, eq);
            }
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                float v[4];
                values(i, v);
                (void)nv_codes4<false>(v, s.den, s.inv, eq);
            }
        }
    } else if constexpr (SF == kMxfp4) {
        float am = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i)
            am = fmaxf(am, quad_amax(i));
        am = fmaxf(am, __shfl_xor_sync(kFull, am, 1)); // a block of 32 kept values: two lanes
        const MxScale s = mx_scale(am);
        f32x2 rs = pack2(0.0f, 0.0f);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float v[4];
            values(i, v);
            (void)mx_codes4(v, s.inv, rs);
        }
        eq = block_err(rs, s.mult);
    } else if constexpr (SF == kInt) {
        float qm[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            qm[i] = quad_amax(i);
        const ChunkOut none{nullptr, nullptr, nullptr, nullptr, false, 0};
        lb_int<4, false>(q, values, qm, valid, false, none, eq);
    }
    return eq;
}

// The dense side's quantization error energy of a lane's 32 values (eight
// quads: the halves of its four chunks).
template <int DF>
__device__ __forceinline__ float lb_dense_energy(const PassConsts &c, const QuantSpec &qd, const uint4 (&w)[4],
                                                 bool valid)
{
    float eq = 0.0f;
    auto values = [&](int j, float (&v)[4]) {
        const uint32_t a = (j & 1) ? w[j >> 1].z : w[j >> 1].x, b = (j & 1) ? w[j >> 1].w : w[j >> 1].y;
        v[0] = bf16_lo(a);
        v[1] = bf16_hi(a);
        v[2] = bf16_lo(b);
        v[3] = bf16_hi(b);
    };
    auto quad_max2 = [&](int j) {
        return (j & 1) ? bf16x2_maxabs(w[j >> 1].z, w[j >> 1].w) : bf16x2_maxabs(w[j >> 1].x, w[j >> 1].y);
    };
    if constexpr (DF == kFp8) {
        bool fast[4], all = true;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            fast[i] = c.guardd ? quot_fast(c.rstd, bf16x2_hmax(bf16x2_maxabs(quad_max2(2 * i), quad_max2(2 * i + 1))))
                               : c.rstd.fast;
            all = all && fast[i];
        }
        if (__all_sync(kFull, all || !valid)) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float v[4];
                values(j, v);
                (void)fp8_codes4<true>(v, c.rstd, eq);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float v[4];
                values(j, v);
                if (fast[j >> 1])
                    (void)fp8_codes4<true>(v, c.rstd, eq);
                else
                    (void)fp8_codes4<false>(v, c.rstd, eq);
            }
        }
    } else if constexpr (DF == kNvfp4) {
        // two blocks of 16: quads 0-3 and 4-7 (the dense side's table)
        PassConsts cd = c;
        cd.rst = c.rstd;
        cd.tb = c.tbd;
        const NvScale s0 = nv_scale(bf16x2_hmax(bf16x2_maxabs(bf16x2_maxabs(quad_max2(0), quad_max2(1)),
                                                              bf16x2_maxabs(quad_max2(2), quad_max2(3)))), cd);
        const NvScale s1 = nv_scale(bf16x2_hmax(bf16x2_maxabs(bf16x2_maxabs(quad_max2(4), quad_max2(5)),
                                                              bf16x2_maxabs(quad_max2(6), quad_max2(7)))), cd);
        if (__all_sync(kFull, (s0.fast && s1.fast) || !valid)) {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const NvScale &s = j < 4 ? s0 : s1;
                float v[4];
                values(j, v);
                (void)nv_codes4<true>(v, s.den, s.inv, eq);
            }
        } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const NvScale &s = j < 4 ? s0 : s1;
                float v[4];
                values(j, v);
                (void)nv_codes4<false>(v, s.den, s.inv, eq);
            }
        }
    } else if constexpr (DF == kMxfp4) {
        uint32_t m2 = quad_max2(0);
#pragma unroll
        for (int j = 1; j < 8; ++j)
            m2 = bf16x2_maxabs(m2, quad_max2(j));
        const MxScale s = mx_scale(bf16x2_hmax(m2));
        f32x2 rs = pack2(0.0f, 0.0f);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float v[4];
            values(j, v);
            (void)mx_codes4(v, s.inv, rs);
        }
        eq = block_err(rs, s.mult);
    } else if constexpr (DF == kInt) {
        float qm[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            qm[j] = bf16x2_hmax(quad_max2(j));
        const ChunkOut none{nullptr, nullptr, nullptr, nullptr, false, 0};
        lb_int<8, false>(qd, values, qm, valid, false, none, eq);
    }
    return eq;
}

// ROT: over the operand rotated along k (rotate_lane32 right after the loads).
template <int SF, int DF, bool ROT = false>
__global__ void __launch_bounds__(kStreamThreads, 3) stream_lb_energy_kernel(const __grid_constant__ PassParams pk)
{
    using T = __nv_bfloat16;
    const PassParams &p = pk;
    const int op = static_cast<int>(blockIdx.x) / pk.ctas_per_op;
    const int cta = static_cast<int>(blockIdx.x) - op * pk.ctas_per_op;
    __shared__ double red[kStreamWarps * 4];
    __shared__ uint32_t flag;
    __shared__ float nvt[512];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    grid_dependency_wait();
    grid_dependents_launch();
    const PassConsts c = make_consts<kEnergy>(operand_view(pk), tid, kStreamThreads, nvt);
    const T *x = static_cast<const T *>(p.x) + op * p.x_bstride;
    const int tw = p.ctas_per_op * kStreamWarps;
    const int u0 = cta * kStreamWarps + warp;
    int ua = u0 / p.units_b, ub = u0 - ua * p.units_b;
    const int sa = tw / p.units_b, sb = tw - sa * p.units_b;
    double e_total = 0.0, e_prune = 0.0, e_q = 0.0, e_qd = 0.0;
    while (ua < p.units_a) {
        const int64_t col = static_cast<int64_t>(ub) * 1024 + 32 * lane;
        const bool valid = col < p.k; // (k is a multiple of 64: a lane is wholly in or out)
        const T *xp = x + static_cast<int64_t>(ua) * p.ld + col;
        uint4 w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            w[i] = ld_stream(xp + 8 * i, valid);
        if constexpr (ROT)
            rotate_lane32(w, p.rot_log2b, p.rot_scale, lane);
        uint32_t k0[4], k1[4];
        float et = 0.0f, ep = 0.0f;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const Pair24 g = pair24_bf16(w[i].x, w[i].y, w[i].z, w[i].w);
            k0[i] = g.k0;
            k1[i] = g.k1;
            et += g.e_all;
            ep += g.e_drop;
        }
        const float eq = SF == kNone ? 0.0f : lb_sparse_energy<SF>(c, p.q, k0, k1, valid);
        const float eqd = lb_dense_energy<DF>(c, p.qd, w, valid);
        // (a lane outside the operand holds zeros; its scales may be zero and
        // its quotients then not finite: it contributes no energy)
        if (valid) {
            e_total += et;
            e_prune += ep;
            e_q += eq;
            e_qd += eqd;
        }
        ua += sa;
        ub += sb;
        if (ub >= p.units_b) {
            ub -= p.units_b;
            ++ua;
        }
    }
    const PassParams v = operand_view(pk);
    grid_reduce_energy(v, e_total, e_prune, e_q, e_qd, red, &flag, tid, lane, warp);
}

// The lane-block energy kernel for 2:4 by magnitude with the 2:4 side's format
// sf (NONE, FP8, NVFP4, MXFP4, INT) and the dense side's format df (FP8,
// NVFP4, MXFP4, INT), or nullptr.
template <int SF, bool ROT = false> const void *stream_lb_energy_for_dense(int df)
{
    switch (df) {
    case kFp8:
        return reinterpret_cast<const void *>(&stream_lb_energy_kernel<SF, kFp8, ROT>);
    case kNvfp4:
        return reinterpret_cast<const void *>(&stream_lb_energy_kernel<SF, kNvfp4, ROT>);
    case kMxfp4:
        return reinterpret_cast<const void *>(&stream_lb_energy_kernel<SF, kMxfp4, ROT>);
    case kInt:
        return reinterpret_cast<const void *>(&stream_lb_energy_kernel<SF, kInt, ROT>);
    }
    return nullptr;
}

} // namespace ss24
