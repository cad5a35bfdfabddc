// Device building blocks of the ss24 kernels (sm_100a): PTX wrappers for
// mbarriers and TMA tile loads, bounded waits, the FP8 / FP4 converters, and
// the 2:4 / 4:8 selection tournaments.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace ss24 {

constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------------------
// shared-memory barriers and TMA (PTX ISA: mbarrier, cp.async.bulk.tensor)
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Makes barrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n"
        " .reg .pred p;\n"
        " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n"
        "}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits until the barrier phase with the given parity has completed.
// Returns false (without having waited forever) if that takes longer than
// limit_ns; the kernel then records an error code and returns.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    for (;;) {
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(bar, parity))
                return true;
        if (global_timer_ns() - t0 > limit_ns)
            return false;
    }
}

// 3-D tiled TMA load: {inner, outer, operand of a batch}.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int32_t c0, int32_t c1, int32_t c2,
                                            uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// L2 policy for data read exactly once: evict it first.
__device__ __forceinline__ uint64_t l2_evict_first_policy()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Programmatic dependent launch (PTX griddepcontrol): a kernel launched with
// programmatic stream serialization may start while the previous kernel on the
// stream is finishing; it must wait for that kernel's completion (and memory)
// before touching global memory. Every pass kernel waits right after its
// shared-memory set-up, so only launch latency and set-up overlap.
__device__ __forceinline__ void grid_dependency_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Lets the next kernel on the stream be scheduled (it still waits as above).
__device__ __forceinline__ void grid_dependents_launch()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void named_barrier_sync(int id, int threads)
{
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---------------------------------------------------------------------------
// number formats (PTX cvt forms for e4m3x2 / e2m1x2; rounding is the
// instruction's own .rn with .satfinite)
// ---------------------------------------------------------------------------

// Two binary32 -> two E4M3 bytes; `lo` lands in bits 0..7, `hi` in 8..15.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two E4M3 bytes (bits 0..7 and 8..15) -> two binary32 (exact).
// Two fp16 lanes -> two binary32 (exact), on the multiply-add pipe: a
// mixed-precision add of -0, which leaves every value unchanged.
__device__ __forceinline__ float2 f16x2_to_f32(uint32_t h2)
{
    float lo, hi;
    asm("{ .reg .b16 l, h; mov.b32 {l, h}, %2;\n"
        " add.rn.f32.f16 %0, l, 0f80000000;\n"
        " add.rn.f32.f16 %1, h, 0f80000000; }"
        : "=f"(lo), "=f"(hi)
        : "r"(h2));
    return make_float2(lo, hi);
}

// Two E4M3 codes in a 16-bit register -> their values as f16x2 (exact).
__device__ __forceinline__ uint32_t e4m3x2h_to_f16x2(uint16_t h)
{
    uint32_t h2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(h));
    return h2;
}
// Two E4M3 codes in a 16-bit register -> two binary32 (exact).
__device__ __forceinline__ float2 e4m3x2h_to_f32(uint16_t h) { return f16x2_to_f32(e4m3x2h_to_f16x2(h)); }
// Two binary32 -> two E4M3 codes (lo in the low byte), saturating, in a 16-bit register.
__device__ __forceinline__ uint16_t cvt_e4m3x2h(float lo, float hi)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t two_bytes)
{
    uint32_t h2;
    const uint16_t b = static_cast<uint16_t>(two_bytes);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(b));
    return f16x2_to_f32(h2); // .x from the low byte
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t byte)
{
    return e4m3x2_to_f32(byte & 0xffu).x;
}

// Four binary32 -> four E2M1 nibbles (v0 in bits 0..3, ..., v3 in 12..15).
__device__ __forceinline__ uint32_t cvt_e2m1x4(float v0, float v1, float v2, float v3)
{
    uint16_t r;
    asm("{\n"
        " .reg .b8 b0, b1;\n"
        " cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
        " cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
        " mov.b16 %0, {b0, b1};\n"
        "}\n"
        : "=h"(r)
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3));
    return r;
}

// cvt_e2m1x4 that also gives the code values it writes, decoded exactly as
// f16x2 words (values 0 and 1 in d01, 2 and 3 in d23; the low lane first).
__device__ __forceinline__ uint32_t cvt_e2m1x4_dec(float v0, float v1, float v2, float v3, uint32_t &d01,
                                                   uint32_t &d23)
{
    uint16_t r;
    asm("{\n"
        " .reg .b8 b0, b1;\n"
        " cvt.rn.satfinite.e2m1x2.f32 b0, %4, %3;\n"
        " cvt.rn.satfinite.e2m1x2.f32 b1, %6, %5;\n"
        " mov.b16 %0, {b0, b1};\n"
        " cvt.rn.f16x2.e2m1x2 %1, b0;\n"
        " cvt.rn.f16x2.e2m1x2 %2, b1;\n"
        "}\n"
        : "=h"(r), "=r"(d01), "=r"(d23)
        : "f"(v0), "f"(v1), "f"(v2), "f"(v3));
    return r;
}

// Two E2M1 nibbles (bits 0..3 and 4..7 of `byte`) -> two binary32 (exact).
__device__ __forceinline__ float2 e2m1x2_to_f32(uint32_t byte)
{
    uint32_t h2;
    const uint16_t h = static_cast<uint16_t>(byte & 0xffu);
    asm("{\n"
        " .reg .b8 lo, hi;\n"
        " mov.b16 {lo, hi}, %1;\n"
        " cvt.rn.f16x2.e2m1x2 %0, lo;\n"
        "}\n"
        : "=r"(h2)
        : "h"(h));
    return f16x2_to_f32(h2); // .x from the low nibble
}

// MXFP4 shared exponent of a block with amax > 0: floor(log2(amax)) - 2,
// read from the bits of amax (subnormals included), clamped to [-127, 127].
__device__ __forceinline__ int mx_shared_exponent(float amax)
{
    const uint32_t b = __float_as_uint(amax);
    const int ebits = static_cast<int>(b >> 23);
    const int fl = ebits ? ebits - 127 : (31 - __clz(static_cast<int>(b))) - 149;
    return max(-127, min(127, fl - 2));
}

// 2^e as a binary32 for e in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float exp2_int(int e)
{
    return e >= -126 ? __uint_as_float(static_cast<uint32_t>(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// ---------------------------------------------------------------------------
// packed binary32 pairs (sm_100 f32x2 arithmetic, each lane rounded to nearest)
// ---------------------------------------------------------------------------

typedef unsigned long long f32x2;

__device__ __forceinline__ f32x2 pack2(float lo, float hi)
{
    f32x2 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
// element 0 of a pair is its low 32 bits
__device__ __forceinline__ float lo2(f32x2 v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi2(f32x2 v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ f32x2 mul2(f32x2 a, f32x2 b)
{
    f32x2 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f32x2 add2(f32x2 a, f32x2 b)
{
    f32x2 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ f32x2 sub2(f32x2 a, f32x2 b)
{
    f32x2 d;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// (h.lo - a, h.hi - b) for the f16 lanes of h: mixed-precision subtractions,
// the f16 operand taken exactly and each difference rounded once.
__device__ __forceinline__ f32x2 f16x2_sub_f32(uint32_t h, float a, float b)
{
    float lo, hi;
    asm("{ .reg .b16 l, h; mov.b32 {l, h}, %2;\n"
        " sub.rn.f32.f16 %0, l, %3;\n"
        " sub.rn.f32.f16 %1, h, %4; }"
        : "=f"(lo), "=f"(hi)
        : "r"(h), "f"(a), "f"(b));
    return pack2(lo, hi);
}
__device__ __forceinline__ f32x2 fma2(f32x2 a, f32x2 b, f32x2 c)
{
    f32x2 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// ---------------------------------------------------------------------------
// packed bf16 pairs (two 16-bit lanes of a 32-bit word, lane 0 in the low half)
// ---------------------------------------------------------------------------

// bf16 lane -> binary32 (exact) computed on the FMA pipe: a mixed-precision
// add of -0, which leaves every value (signed zeros included) unchanged.
__device__ __forceinline__ float bf16_lo(uint32_t w)
{
    float r;
    asm("{ .reg .b16 l, h; mov.b32 {l, h}, %1; add.rn.f32.bf16 %0, l, 0f80000000; }" : "=f"(r) : "r"(w));
    return r;
}
__device__ __forceinline__ float bf16_hi(uint32_t w)
{
    float r;
    asm("{ .reg .b16 l, h; mov.b32 {l, h}, %1; add.rn.f32.bf16 %0, h, 0f80000000; }" : "=f"(r) : "r"(w));
    return r;
}
// RN(l * l + c) and RN(h * h + c) for the lanes of w (products of bf16 values
// are exact in binary32, so these equal the binary32 fused multiply-add)
__device__ __forceinline__ float bf16_sq_lo(uint32_t w, float c)
{
    float r;
    asm("{ .reg .b16 l, h; mov.b32 {l, h}, %1; fma.rn.f32.bf16 %0, l, l, %2; }" : "=f"(r) : "r"(w), "f"(c));
    return r;
}
__device__ __forceinline__ float bf16_sq_hi(uint32_t w, float c)
{
    float r;
    asm("{ .reg .b16 l, h; mov.b32 {l, h}, %1; fma.rn.f32.bf16 %0, h, h, %2; }" : "=f"(r) : "r"(w), "f"(c));
    return r;
}

// Per lane: a value whose magnitude is max(|a|, |b|) (its sign is not
// meaningful). Exact: a maximum selects one of its inputs.
__device__ __forceinline__ uint32_t bf16x2_maxabs(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
// The larger magnitude of the two lanes as binary32 (magnitude bit patterns
// of non-NaN values order like the values).
__device__ __forceinline__ float bf16x2_hmax(uint32_t m)
{
    return __uint_as_float(max(m & 0x7fffu, (m >> 16) & 0x7fffu) << 16);
}

// Per lane: all ones where |b| > |a|, else zero: a packed bf16 comparison of
// the magnitudes whose unsigned result is a 16-bit mask per lane (|-0| = |+0|
// is not greater; subnormals compare by value).
__device__ __forceinline__ uint32_t bf16x2_gt_abs(uint32_t b, uint32_t a)
{
    uint32_t m;
    asm("{ .reg .b32 aa, bb; abs.bf16x2 aa, %1; abs.bf16x2 bb, %2; set.gt.u32.bf16x2 %0, bb, aa; }"
        : "=r"(m)
        : "r"(a), "r"(b));
    return m;
}
__device__ __forceinline__ uint32_t sel_mask(uint32_t m, uint32_t a, uint32_t b) { return (a & m) | (b & ~m); }

// True when the larger magnitude of some lane of a and b is >= the bf16 value
// lim (both lanes of lim2 hold it): bf16x2_any_ge_abs from one packed maximum
// of the magnitudes and one comparison.
__device__ __forceinline__ bool bf16x2_max_ge_abs(uint32_t a, uint32_t b, uint32_t lim2)
{
    uint32_t m;
    asm("{ .reg .b32 mx; max.xorsign.abs.bf16x2 mx, %1, %2; and.b32 mx, mx, 0x7fff7fff;\n"
        " set.ge.u32.bf16x2 %0, mx, %3; }"
        : "=r"(m)
        : "r"(a), "r"(b), "r"(lim2));
    return m != 0u;
}

// True when some lane of a or b has a magnitude >= the bf16 value lim (both
// lanes of lim2 hold it): two packed comparisons.
__device__ __forceinline__ bool bf16x2_any_ge_abs(uint32_t a, uint32_t b, uint32_t lim2)
{
    uint32_t m;
    asm("{ .reg .b32 aa, bb, ma, mb; abs.bf16x2 aa, %1; abs.bf16x2 bb, %2;\n"
        " set.ge.u32.bf16x2 ma, aa, %3; set.ge.u32.bf16x2 mb, bb, %3; or.b32 %0, ma, mb; }"
        : "=r"(m)
        : "r"(a), "r"(b), "r"(lim2));
    return m != 0u;
}

// ---------------------------------------------------------------------------
// division by a scale
// ---------------------------------------------------------------------------

// Quotients a / b rounded to nearest-even, as an IEEE binary32 division gives
// them. For a scale b in [2^-60, 2^60] the library uses Markstein's one-step
// correction (P. Markstein, "Computation of elementary functions on the IBM
// RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): with
// y = RN(1/b), q0 = RN(a y), r = a - q0 b (exact through the fused
// multiply-add), q = RN(q0 + r y). Both significands range over [1, 2) without
// loss of generality (power-of-two factors scale every step exactly while
// operands and intermediates stay normal); ss24_selfcheck_division compares
// this against IEEE division for every pair of significands. With b in the
// range, y, q0 and the residual stay normal whenever |a / b| >= 2^-40, so the
// result is exact there; below that the residual may lose bits, but every
// format's code of such a quotient is the signed zero either way, and the sign
// is kept. A quotient that overflows is ruled out by the callers (a group,
// block or chunk amax times y stays below 2^126). Outside the range, IEEE
// division is used.
struct Recip {
    float b, y, nb; // scale, RN(1/b), -b
    bool fast;
};

__device__ __forceinline__ Recip make_recip(float b)
{
    Recip r;
    r.b = b;
    r.nb = -b;
    r.y = __frcp_rn(b);
    r.fast = b >= 0x1p-60f && b <= 0x1p60f;
    return r;
}

// The sign of a / b for b > 0 is the sign of a. The correction step can lose
// it for a signed zero (-0 * y - (-0) * b rounds to +0), so it is copied back.
__device__ __forceinline__ float with_sign_of(float q, float a)
{
    return __uint_as_float((__float_as_uint(q) & 0x7fffffffu) | (__float_as_uint(a) & 0x80000000u));
}

__device__ __forceinline__ float div_fast(float a, const Recip &r)
{
    const float q0 = __fmul_rn(a, r.y);
    const float res = __fmaf_rn(q0, r.nb, a);
    return with_sign_of(__fmaf_rn(res, r.y, q0), a);
}

// Negated quotients -(a / b) of two values: Markstein's correction run with
// -y in place of y (q0 = RN(a (-y)), r = a + q0 b exact, RN(q0 + r (-y))).
// Because rounding to nearest is symmetric this is exactly -RN(a / b) where
// div_fast is exact, with the signed zeros right as well: a = -0 gives +0 and
// a = +0 gives -0, so no sign fix-up is needed.
__device__ __forceinline__ f32x2 neg_div_fast2(f32x2 a, const Recip &r)
{
    const f32x2 ny2 = pack2(-r.y, -r.y), b2 = pack2(r.b, r.b);
    const f32x2 q0 = mul2(a, ny2);
    const f32x2 res = fma2(q0, b2, a);
    return fma2(res, ny2, q0);
}

// ---------------------------------------------------------------------------
// selection
// ---------------------------------------------------------------------------

// Top-2 of four by score with ties to the lower index. After the pairs (0,1)
// and (2,3) are decided, the kept pair is (0,1) when (0,1)'s loser beats
// (2,3)'s winner, (2,3) when (2,3)'s loser beats (0,1)'s winner, and the two
// winners otherwise: four comparisons in all. A later index wins a comparison
// only when its score is strictly larger.
//
// One 2:4 group: the kept values in index order, the dropped values, the
// group's energy, the energy of its dropped pair and the metadata nibble. With
// kAbs the scores are the magnitudes of the values themselves (compared
// through |.|); otherwise s0..s3 are the scores.
struct Group24 {
    float k0, k1, d0, d1, e_all, e_drop;
    uint32_t nib;
};

template <bool kAbs>
__device__ __forceinline__ Group24 group24(float x0, float x1, float x2, float x3, float s0, float s1, float s2,
                                           float s3)
{
    bool p, q, ta, tb;
    float w01, l01, w23, l23;
    if constexpr (kAbs) {
        p = fabsf(x1) > fabsf(x0);
        q = fabsf(x3) > fabsf(x2);
        w01 = p ? x1 : x0;
        l01 = p ? x0 : x1;
        w23 = q ? x3 : x2;
        l23 = q ? x2 : x3;
        ta = fabsf(w23) > fabsf(l01);
        tb = fabsf(l23) > fabsf(w01);
    } else {
        p = s1 > s0;
        q = s3 > s2;
        w01 = p ? x1 : x0;
        l01 = p ? x0 : x1;
        w23 = q ? x3 : x2;
        l23 = q ? x2 : x3;
        const float sw01 = p ? s1 : s0, sl01 = p ? s0 : s1;
        const float sw23 = q ? s3 : s2, sl23 = q ? s2 : s3;
        ta = sw23 > sl01;
        tb = sl23 > sw01;
    }
    // ties keep the lower index: l01 beats w23 exactly when both kept values
    // come from (0, 1); l23 beats w01 exactly when both come from (2, 3)
    const bool both01 = !ta, both23 = tb;
    Group24 g;
    g.k0 = both01 ? x0 : (both23 ? x2 : w01);
    g.k1 = both01 ? x1 : (both23 ? x3 : w23);
    g.d0 = both01 ? x2 : (both23 ? x0 : l01);
    g.d1 = both01 ? x3 : (both23 ? x1 : l23);
    const f32x2 e = fma2(pack2(x1, x3), pack2(x1, x3), mul2(pack2(x0, x2), pack2(x0, x2)));
    const float e01 = lo2(e), e23 = hi2(e);
    const float el = __fmaf_rn(l23, l23, l01 * l01);
    g.e_all = e01 + e23;
    g.e_drop = both01 ? e23 : (both23 ? e01 : el);
    const uint32_t mixed = (p ? 1u : 0u) + (q ? 12u : 8u);
    g.nib = both01 ? 0x4u : (both23 ? 0xEu : mixed);
    return g;
}

// The two 2:4 groups of a chunk of eight bf16 values (words w0..w3, element
// 2i in the low half of word i) by magnitude, both at once: lane 0 of every
// packed word below is group 0, lane 1 group 1. The same top-2 as group24
// (ties keep the lower index), from four comparisons (bf16x2_gt_abs) and bit
// selects. Results: kept values k0 (lower index) and k1 per lane, the
// metadata byte (group 0 in the low nibble), the chunk's energy and the
// energy of its dropped values.
struct Pair24 {
    uint32_t k0, k1, meta;
    float e_all, e_drop;
};

__device__ __forceinline__ Pair24 pair24_bf16(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t w3)
{
    const uint32_t A = __byte_perm(w0, w2, 0x5410), B = __byte_perm(w0, w2, 0x7632); // x0 | x4, x1 | x5
    const uint32_t C = __byte_perm(w1, w3, 0x5410), D = __byte_perm(w1, w3, 0x7632); // x2 | x6, x3 | x7
    const uint32_t mp = bf16x2_gt_abs(B, A);            // p: |x1| > |x0|
    const uint32_t mq = bf16x2_gt_abs(D, C);            // q: |x3| > |x2|
    const uint32_t w01 = sel_mask(mp, B, A), l01 = sel_mask(mp, A, B);
    const uint32_t w23 = sel_mask(mq, D, C), l23 = sel_mask(mq, C, D);
    // With the tie rule (the lower index wins), l01 beats w23 exactly when both
    // kept values come from (0, 1), and l23 beats w01 exactly when both come
    // from (2, 3); otherwise w01 and w23 are kept (already in index order). The
    // winners' own comparison is implied and not needed.
    const uint32_t ta = bf16x2_gt_abs(w23, l01);        // not both from (0, 1)
    const uint32_t tb = bf16x2_gt_abs(l23, w01);        // both from (2, 3)
    Pair24 g;
    g.k0 = sel_mask(ta, sel_mask(tb, C, w01), A);
    g.k1 = sel_mask(ta, sel_mask(tb, D, w23), B);
    const uint32_t d0 = sel_mask(ta, sel_mask(tb, A, l01), C);
    const uint32_t d1 = sel_mask(ta, sel_mask(tb, B, l23), D);
    // nibble i0 | i1 << 2: (0,1) -> 4, (2,3) -> 14, otherwise p | (2 + q) << 2
    const uint32_t mixed = 0x00080008u | (mp & 0x00010001u) | (mq & 0x00040004u);
    const uint32_t nib = sel_mask(ta, sel_mask(tb, 0x000E000Eu, mixed), 0x00040004u);
    g.meta = (nib | (nib >> 12)) & 0xffu;
    // energies: the dropped values' squares, and the chunk's energy as the kept
    // values' squares plus the dropped ones (binary32 chains of fused
    // multiply-adds; the energies are sums, compared within 1e-6 relative)
    g.e_drop = bf16_sq_hi(d1, bf16_sq_hi(d0, bf16_sq_lo(d1, bf16_sq_lo(d0, -0.0f))));
    g.e_all = bf16_sq_hi(g.k1, bf16_sq_hi(g.k0, bf16_sq_lo(g.k1, bf16_sq_lo(g.k0, g.e_drop))));
    return g;
}

} // namespace ss24
