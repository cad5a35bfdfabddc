/*
 * ss24 oracle: a plain, slow CPU statement of the online 2:4 prune / compress /
 * quantize pass and of its error energies.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg load this library. The product path (the CUDA
 * library and its Python binding) never calls, links or imports it, and this
 * file includes nothing from the product path.
 *
 * Style: every step is a scalar loop, in the order the method states it. A
 * decision that yields an integer (which elements are kept, which code a value
 * gets) is taken in IEEE binary32 with round-to-nearest-even and no
 * contraction, because that is the precision the kernels decide in. Error
 * energies are accumulated in binary64, row-major, one element at a time.
 * Build with -ffp-contract=off and without fast-math.
 *
 * Sources. "Is 2:4 Sparsity Still Worth It? Semi-Structured Sparsity versus
 * Quantization in LLM Inference" (English digest on paper-daily.com):
 *   intro .......... 2:4 keeps two non-zeros of every four along the reduction axis
 *   §1 ............. online operands are pruned and compressed before every GEMM
 *   §2 ............. equal bits (a 1-bit index per original element), the
 *                    magnitude and Wanda scores, round-to-nearest quantization
 *   §3 ............. the formats: FP8, INT8 with one scale per row, NVFP4
 *                    (FP8 scale per 16 plus one per tensor), MXFP4 (one
 *                    power-of-two scale per 32); the fused read-once kernel
 *   §4 ............. 2:4 energy loss, disjoint pruning / quantization error
 *                    energies, predicted R
 *   §6 ............. pairwise 4:8 (keep two of four adjacent pairs per eight)
 * Where the pages leave a format detail open the oracle follows the OCP 8-bit
 * Floating Point (OFP8) and OCP Microscaling (MX) v1.0 definitions.
 *
 * Readings of points the pages leave open (tie rule, metadata nibble layout,
 * scales over the compressed row, symmetric integer range, NVFP4 two-level
 * recipe, MX shared exponent) are stated at the function that takes them.
 *
 * Parity status: every function here is pinned by a CPU test against
 * something other than itself (brute force, a library routine, a closed form
 * or a figure printed on the pages). None is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Enumerations. Same numeric values as the product's C header; restated here
 * because the oracle shares no header with the product. */
enum { OR_BF16 = 0, OR_F32 = 1 };
enum { OR_SCORE_MAG = 0, OR_SCORE_WANDA = 1 };
enum { OR_DENSE = 0, OR_SPARSE_24 = 24, OR_SPARSE_48 = 48 };
enum { OR_FMT_NONE = 0, OR_FMT_FP8 = 1, OR_FMT_INT = 2, OR_FMT_NVFP4 = 3, OR_FMT_MXFP4 = 4 };

typedef struct {
    const void *x;        /* operand bytes (bf16 as raw uint16, or fp32)              */
    int32_t dtype;        /* OR_BF16 / OR_F32                                           */
    int32_t axis;         /* 1: element (r,c) at x[r*ld + c]; 0: at x[c*ld + r]         */
    int64_t rows, k, ld;  /* logical operand A[rows][k], reduction along k             */
    int32_t pattern;      /* OR_DENSE, OR_SPARSE_24, OR_SPARSE_48                       */
    int32_t score;        /* OR_SCORE_MAG, OR_SCORE_WANDA                               */
    const float *norms;   /* Wanda per-input-channel norms, length k (or NULL)          */
    int32_t fmt, bits, group, pack4;
    const float *tensor_scale_in; /* host pointer to a given per-tensor scale, or NULL   */
} oracle_args;

typedef struct {
    void *values;         /* kept values (format NONE) or codes                        */
    void *scales;         /* INT: fp32 per group; NVFP4: E4M3 bytes; MXFP4: E8M0 bytes  */
    float *tensor_scale;  /* FP8 / NVFP4: the per-tensor scale used                     */
    uint8_t *meta;        /* 2:4 / 4:8 position metadata                                */
} oracle_outputs;

/* ------------------------------------------------------------------------- */
/* Number formats                                                             */
/* ------------------------------------------------------------------------- */

/* bf16 is the upper half of a binary32; widening is exact. */
float oracle_bf16_to_f32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Exact floor(log2(a)) for finite a > 0, subnormals included (frexpf is exact). */
int oracle_floor_log2(float a)
{
    int e;
    (void)frexpf(a, &e); /* a = f * 2^e with f in [0.5, 1) */
    return e - 1;
}

/* Round a non-negative magnitude to the nearest multiple of `step` (a power of
 * two), ties to the even multiple. a/step is exact (power-of-two scaling). */
static float round_to_step(float a, float step)
{
    float q = a / step;
    float n = nearbyintf(q); /* default mode: round half to even */
    return n * step;
}

/* OCP FP8 E4M3 ("fn"): 1 sign, 4 exponent bits with bias 7, 3 mantissa bits;
 * no infinities; S.1111.111 is NaN; largest finite 448 = 1.75 * 2^8; smallest
 * normal 2^-6; subnormal step 2^-9. */
float oracle_e4m3_decode(uint8_t c)
{
    int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    float mag;
    if (e == 15 && m == 7)
        return s ? -NAN : NAN;
    if (e == 0)
        mag = ldexpf((float)m, -9); /* m/8 * 2^-6 */
    else
        mag = ldexpf(1.0f + (float)m / 8.0f, e - 7);
    return s ? -mag : mag;
}

/* Encode a binary32 to E4M3 with one rounding, nearest-even, saturating to
 * +-448 ("satfinite"); NaN stays NaN. The sign of a result that rounds to zero
 * is kept (so -0 and tiny negatives give 0x80). */
uint8_t oracle_e4m3_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    float a = fabsf(v);
    if (isnan(v))
        return sign | 0x7F;
    if (a >= 448.0f)
        return sign | 0x7E;
    /* Grid spacing: 2^(E-3) inside binade [2^E, 2^(E+1)) for E >= -6, and the
     * subnormal spacing 2^-9 below 2^-6. */
    float step;
    if (a < ldexpf(1.0f, -6))
        step = ldexpf(1.0f, -9);
    else
        step = ldexpf(1.0f, oracle_floor_log2(a) - 3);
    float r = round_to_step(a, step); /* may round up into the next binade */
    if (r > 448.0f)
        r = 448.0f;
    if (r == 0.0f)
        return sign;
    if (r < ldexpf(1.0f, -6))
        return sign | (uint8_t)(r / ldexpf(1.0f, -9)); /* subnormal: e = 0 */
    int E = oracle_floor_log2(r);
    int m = (int)(ldexpf(r, -E) * 8.0f) - 8; /* r = (1 + m/8) * 2^E */
    return sign | (uint8_t)(((E + 7) << 3) | m);
}

/* OCP E2M1 (FP4): 1 sign, 2 exponent bits with bias 1, 1 mantissa bit; the
 * magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6; no infinities or NaN. */
float oracle_e2m1_decode(uint8_t c)
{
    static const float mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    float m = mag[c & 7];
    return (c & 8) ? -m : m;
}

/* Encode to E2M1, nearest-even, saturating to +-6; the sign of zero is kept. */
uint8_t oracle_e2m1_encode(float v)
{
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    float a = fabsf(v);
    if (a >= 6.0f)
        return sign | 0x7;
    /* Spacing 0.5 below 2 (subnormal 0..0.5 and binade [1,2)), 1 in [2,4), 2 in [4,8). */
    float step = (a < 2.0f) ? 0.5f : (a < 4.0f ? 1.0f : 2.0f);
    float r = round_to_step(a, step);
    if (r > 6.0f)
        r = 6.0f;
    uint8_t code = 0;
    for (uint8_t c = 0; c < 8; ++c)
        if (oracle_e2m1_decode(c) == r)
            code = c;
    return sign | code;
}

/* ------------------------------------------------------------------------- */
/* Selection                                                                  */
/* ------------------------------------------------------------------------- */

/* Top-2 of a group of 4 scores (intro and §2: keep the two largest of every
 * four). Tie rule (the pages give none): element i beats element j iff
 * s_i > s_j, or s_i == s_j and i < j; an element is kept when fewer than two
 * others beat it. Returns the metadata nibble i0 | i1 << 2 with i0 < i1. */
int oracle_select24(const float s[4])
{
    int kept[2], nk = 0;
    for (int i = 0; i < 4; ++i) {
        int beaten = 0;
        for (int j = 0; j < 4; ++j)
            if (j != i && (s[j] > s[i] || (s[j] == s[i] && j < i)))
                beaten++;
        if (beaten < 2)
            kept[nk++] = i;
    }
    return kept[0] | (kept[1] << 2);
}

/* Pairwise 4:8 (§6): eight elements form four adjacent pairs; a pair's rank is
 * its energy e_p = s_{2p}^2 + s_{2p+1}^2 (binary32, multiply then add). The
 * same beats-rule picks two pairs; returns the nibble p0 | p1 << 2. */
int oracle_select48(const float s[8])
{
    float e[4];
    for (int p = 0; p < 4; ++p) {
        float a = s[2 * p] * s[2 * p];
        float b = s[2 * p + 1] * s[2 * p + 1];
        e[p] = a + b;
    }
    return oracle_select24(e);
}

/* ------------------------------------------------------------------------- */
/* Row access and scores                                                      */
/* ------------------------------------------------------------------------- */

static float element(const oracle_args *a, int64_t r, int64_t c)
{
    int64_t off = (a->axis == 0) ? c * a->ld + r : r * a->ld + c;
    if (a->dtype == OR_BF16)
        return oracle_bf16_to_f32(((const uint16_t *)a->x)[off]);
    return ((const float *)a->x)[off];
}

/* Score of element (r, c) (§2): magnitude |x|, or Wanda |x| * n_c where n_c is
 * the norm of input channel c (product rounded to binary32). */
static float score_of(const oracle_args *a, float x, int64_t c)
{
    if (a->score == OR_SCORE_WANDA)
        return fabsf(x) * a->norms[c];
    return fabsf(x);
}

/* Prune one row. Writes the kept values (in index order) to kept[k/2], their
 * source indices to kidx, the metadata bytes to meta_row (when not NULL), and
 * adds the row's energies: e_total += sum x^2, e_prune += sum over dropped x^2. */
static void prune_row(const oracle_args *a, const float *xr, float *kept, int64_t *kidx,
                      uint8_t *meta_row, double *e_total, double *e_prune)
{
    int64_t k = a->k;
    int gsize = (a->pattern == OR_SPARSE_48) ? 8 : 4;
    int64_t nk = 0;
    for (int64_t g0 = 0; g0 < k; g0 += gsize) {
        float s[8];
        int keep[8] = {0};
        int nib;
        for (int i = 0; i < gsize; ++i)
            s[i] = score_of(a, xr[g0 + i], g0 + i);
        if (gsize == 4) {
            nib = oracle_select24(s);
            keep[nib & 3] = 1;
            keep[nib >> 2] = 1;
        } else {
            nib = oracle_select48(s);
            int p0 = nib & 3, p1 = nib >> 2;
            keep[2 * p0] = keep[2 * p0 + 1] = 1;
            keep[2 * p1] = keep[2 * p1 + 1] = 1;
        }
        if (meta_row) {
            int64_t gi = g0 / gsize; /* group index: two groups share a byte */
            if (gi % 2 == 0)
                meta_row[gi / 2] = (uint8_t)nib;
            else
                meta_row[gi / 2] |= (uint8_t)(nib << 4);
        }
        for (int i = 0; i < gsize; ++i) {
            double xd = (double)xr[g0 + i];
            *e_total += xd * xd;
            if (keep[i]) {
                kept[nk] = xr[g0 + i];
                kidx[nk] = g0 + i;
                nk++;
            } else {
                *e_prune += xd * xd;
            }
        }
    }
}

/* The vector that gets quantized for row r: the kept row (sparse) or the whole
 * row (dense). Returns its length. */
static int64_t quantized_row(const oracle_args *a, int64_t r, float *xr, float *v, int64_t *kidx,
                             uint8_t *meta_row, double *e_total, double *e_prune)
{
    for (int64_t c = 0; c < a->k; ++c)
        xr[c] = element(a, r, c);
    if (a->pattern == OR_DENSE) {
        for (int64_t c = 0; c < a->k; ++c) {
            double xd = (double)xr[c];
            *e_total += xd * xd;
            v[c] = xr[c];
        }
        return a->k;
    }
    prune_row(a, xr, v, kidx, meta_row, e_total, e_prune);
    return a->k / 2;
}

/* ------------------------------------------------------------------------- */
/* Quantizers (round to nearest, §2; the formats, §3).                        */
/* Each writes codes for one row vector v[n] and its dequantized values.      */
/* ------------------------------------------------------------------------- */


typedef struct {
    const oracle_args *a;
    oracle_outputs *o;
    int64_t n;          /* length of the quantized row (k/2 sparse, k dense) */
    float tensor_scale; /* FP8 / NVFP4 per-tensor scale */
} qctx;

/* Symmetric INT-b with one fp32 scale per `group` consecutive values of the
 * quantized row; group 0 means one scale per row (the "INT8 with a single
 * scale per row" of §3). Reading: restricted range +-(2^(b-1) - 1);
 * scale = amax / qmax; code = clamp(round_half_even(v / scale)); a zero scale
 * gives all-zero codes. Codes are stored as int8 (b <= 8), int16 (b > 8), or,
 * with pack4 and b <= 4, as two's-complement nibbles two per byte, the lower
 * index in the low nibble. */
static void quant_int_row(const qctx *q, int64_t r, const float *v, float *deq)
{
    const oracle_args *a = q->a;
    int64_t n = q->n;
    int64_t g = a->group ? a->group : n;
    float qmax = (float)((1 << (a->bits - 1)) - 1);
    for (int64_t j0 = 0; j0 < n; j0 += g) {
        float amax = 0.0f;
        for (int64_t j = j0; j < j0 + g; ++j)
            if (fabsf(v[j]) > amax)
                amax = fabsf(v[j]);
        float scale = amax / qmax;
        if (q->o->scales)
            ((float *)q->o->scales)[r * (n / g) + j0 / g] = scale;
        for (int64_t j = j0; j < j0 + g; ++j) {
            int code = 0;
            if (scale != 0.0f) {
                float t = nearbyintf(v[j] / scale);
                if (t > qmax)
                    t = qmax;
                if (t < -qmax)
                    t = -qmax;
                code = (int)t;
            }
            deq[j] = (float)code * scale;
            if (!q->o->values)
                continue;
            if (a->pack4) {
                uint8_t *p = (uint8_t *)q->o->values + r * (n / 2) + j / 2;
                if (j % 2 == 0)
                    *p = (uint8_t)(code & 0xF);
                else
                    *p |= (uint8_t)((code & 0xF) << 4);
            } else if (a->bits > 8) {
                ((int16_t *)q->o->values)[r * n + j] = (int16_t)code;
            } else {
                ((int8_t *)q->o->values)[r * n + j] = (int8_t)code;
            }
        }
    }
}

/* FP8 E4M3 with one scale per tensor (§3 names FP8; the pages fix no granularity,
 * per-tensor is the reading): s = amax / 448; code = E4M3(v / s);
 * deq = decode(code) * s; s == 0 gives zero codes. */
static void quant_fp8_row(const qctx *q, int64_t r, const float *v, float *deq)
{
    float s = q->tensor_scale;
    for (int64_t j = 0; j < q->n; ++j) {
        uint8_t code = 0;
        if (s != 0.0f)
            code = oracle_e4m3_encode(v[j] / s);
        deq[j] = oracle_e4m3_decode(code) * s;
        if (q->o->values)
            ((uint8_t *)q->o->values)[r * q->n + j] = code;
    }
}

/* NVFP4 (§3: 4-bit float, an FP8 scale per 16 elements plus one scale per
 * tensor). Reading of the two-level recipe: s_t = amax / (6 * 448); for each
 * block of 16, sb = E4M3((amax_block / 6) / s_t) (two divisions in that
 * order); denom = decode(sb) * s_t; code = E2M1(v / denom); a zero s_t or
 * denom gives zero codes. Codes two per byte, lower index in the low nibble. */
static void quant_nvfp4_row(const qctx *q, int64_t r, const float *v, float *deq)
{
    float st = q->tensor_scale;
    int64_t n = q->n;
    for (int64_t j0 = 0; j0 < n; j0 += 16) {
        float amax = 0.0f;
        for (int64_t j = j0; j < j0 + 16; ++j)
            if (fabsf(v[j]) > amax)
                amax = fabsf(v[j]);
        uint8_t sb = 0;
        if (st != 0.0f)
            sb = oracle_e4m3_encode((amax / 6.0f) / st);
        float denom = oracle_e4m3_decode(sb) * st;
        if (q->o->scales)
            ((uint8_t *)q->o->scales)[r * (n / 16) + j0 / 16] = sb;
        for (int64_t j = j0; j < j0 + 16; ++j) {
            uint8_t code = 0;
            if (denom != 0.0f)
                code = oracle_e2m1_encode(v[j] / denom);
            deq[j] = oracle_e2m1_decode(code) * denom;
            if (q->o->values) {
                uint8_t *p = (uint8_t *)q->o->values + r * (n / 2) + j / 2;
                if (j % 2 == 0)
                    *p = code;
                else
                    *p |= (uint8_t)(code << 4);
            }
        }
    }
}

/* MXFP4 (§3: 32 elements share one power-of-two scale). Reading, from OCP MX
 * v1.0: shared exponent e = floor(log2(amax_block)) - 2 (2 = largest E2M1
 * exponent), clamped to [-127, 127], stored as the E8M0 byte e + 127;
 * code = E2M1(v / 2^e); an all-zero block stores byte 0 and zero codes. */
static void quant_mxfp4_row(const qctx *q, int64_t r, const float *v, float *deq)
{
    int64_t n = q->n;
    for (int64_t j0 = 0; j0 < n; j0 += 32) {
        float amax = 0.0f;
        for (int64_t j = j0; j < j0 + 32; ++j)
            if (fabsf(v[j]) > amax)
                amax = fabsf(v[j]);
        uint8_t byte = 0;
        float scale = 0.0f;
        if (amax != 0.0f) {
            int e = oracle_floor_log2(amax) - 2;
            if (e < -127)
                e = -127;
            if (e > 127)
                e = 127;
            byte = (uint8_t)(e + 127);
            scale = ldexpf(1.0f, e);
        }
        if (q->o->scales)
            ((uint8_t *)q->o->scales)[r * (n / 32) + j0 / 32] = byte;
        for (int64_t j = j0; j < j0 + 32; ++j) {
            uint8_t code = 0;
            if (scale != 0.0f)
                code = oracle_e2m1_encode(v[j] / scale);
            deq[j] = oracle_e2m1_decode(code) * scale;
            if (q->o->values) {
                uint8_t *p = (uint8_t *)q->o->values + r * (n / 2) + j / 2;
                if (j % 2 == 0)
                    *p = code;
                else
                    *p |= (uint8_t)(code << 4);
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* The pass                                                                   */
/* ------------------------------------------------------------------------- */

/* Largest |value| among the values that get quantized: the kept values for a
 * sparse pattern (reading: a per-tensor scale is taken over what is stored),
 * every value for the dense pattern. */
float oracle_amax(const oracle_args *a)
{
    int64_t k = a->k;
    float *xr = malloc(sizeof(float) * k), *v = malloc(sizeof(float) * k);
    int64_t *kidx = malloc(sizeof(int64_t) * k);
    double et = 0.0, ep = 0.0;
    float amax = 0.0f;
    for (int64_t r = 0; r < a->rows; ++r) {
        int64_t n = quantized_row(a, r, xr, v, kidx, NULL, &et, &ep);
        for (int64_t j = 0; j < n; ++j)
            if (fabsf(v[j]) > amax)
                amax = fabsf(v[j]);
    }
    free(xr);
    free(v);
    free(kidx);
    return amax;
}

/* Argument checks the oracle needs to run at all (it does not restate the
 * product's validation). Returns 0 when the arguments are usable. */
static int check_args(const oracle_args *a)
{
    if (!a->x || a->rows < 0 || a->k <= 0)
        return 1;
    if (a->pattern == OR_SPARSE_24 && a->k % 8)
        return 2;
    if (a->pattern == OR_SPARSE_48 && a->k % 16)
        return 2;
    if (a->score == OR_SCORE_WANDA && !a->norms)
        return 3;
    int64_t n = a->pattern == OR_DENSE ? a->k : a->k / 2;
    switch (a->fmt) {
    case OR_FMT_NONE:
        return a->pattern == OR_DENSE ? 4 : 0;
    case OR_FMT_FP8:
        return 0;
    case OR_FMT_INT:
        if (a->bits < 2 || a->bits > 16)
            return 4;
        if (a->group && n % a->group)
            return 4;
        if (a->pack4 && (a->bits > 4 || n % 2))
            return 4;
        return 0;
    case OR_FMT_NVFP4:
        return n % 16 ? 4 : 0;
    case OR_FMT_MXFP4:
        return n % 32 ? 4 : 0;
    }
    return 4;
}

/* One pass of the method over the operand: score, select, compress (sparse
 * patterns), quantize the stored values, and the error energies
 *   energy[0] = E_total = sum over all elements of x^2
 *   energy[1] = E_prune = sum over dropped elements of x^2
 *   energy[2] = E_q     = sum over kept elements of (x - deq)^2  (sparse)
 *   energy[3] = E_q,dense = sum over all elements of (x - deq)^2 (dense)
 * (§4: dropped elements carry only pruning error, kept ones only quantization
 * error). Format NONE stores the kept values unchanged and has E_q = 0.
 * Output layouts (all rows of the logical operand, k contiguous):
 *   values: NONE -> kept values in the input dtype [rows][k/2];
 *           FP8 -> u8 [rows][n]; INT -> int8/int16 [rows][n] or packed [rows][n/2];
 *           NVFP4 / MXFP4 -> u8 [rows][n/2]
 *   scales: INT fp32 [rows][n/group]; NVFP4 u8 [rows][n/16]; MXFP4 u8 [rows][n/32]
 *   meta:   2:4 -> u8 [rows][k/8], group g's nibble i0 | i1 << 2 in byte g/2,
 *           even g in the low nibble; 4:8 -> u8 [rows][k/16], same per octet.
 * Returns 0 on success, nonzero when the arguments are unusable. */
int oracle_run(const oracle_args *a, oracle_outputs *o, double *energy)
{
    int bad = check_args(a);
    if (bad)
        return bad;
    int64_t k = a->k, n = a->pattern == OR_DENSE ? k : k / 2;
    qctx q = {a, o, n, 0.0f};
    if (a->fmt == OR_FMT_FP8 || a->fmt == OR_FMT_NVFP4) {
        if (a->tensor_scale_in) {
            q.tensor_scale = *a->tensor_scale_in;
        } else {
            float amax = oracle_amax(a);
            q.tensor_scale = a->fmt == OR_FMT_FP8 ? amax / 448.0f : amax / 2688.0f;
        }
        if (o->tensor_scale)
            *o->tensor_scale = q.tensor_scale;
    }
    float *xr = malloc(sizeof(float) * k), *v = malloc(sizeof(float) * k);
    float *deq = malloc(sizeof(float) * k);
    int64_t *kidx = malloc(sizeof(int64_t) * k);
    double e_total = 0.0, e_prune = 0.0, e_q = 0.0;
    int64_t meta_bytes = a->pattern == OR_SPARSE_48 ? k / 16 : k / 8;
    for (int64_t r = 0; r < a->rows; ++r) {
        uint8_t *meta_row = (o->meta && a->pattern != OR_DENSE) ? o->meta + r * meta_bytes : NULL;
        quantized_row(a, r, xr, v, kidx, meta_row, &e_total, &e_prune);
        switch (a->fmt) {
        case OR_FMT_NONE:
            for (int64_t j = 0; j < n; ++j) {
                deq[j] = v[j];
                if (!o->values)
                    continue;
                if (a->dtype == OR_BF16) {
                    /* the kept value is stored bit-for-bit */
                    int64_t off = a->axis == 0 ? kidx[j] * a->ld + r : r * a->ld + kidx[j];
                    ((uint16_t *)o->values)[r * n + j] = ((const uint16_t *)a->x)[off];
                } else {
                    ((float *)o->values)[r * n + j] = v[j];
                }
            }
            break;
        case OR_FMT_FP8:
            quant_fp8_row(&q, r, v, deq);
            break;
        case OR_FMT_INT:
            quant_int_row(&q, r, v, deq);
            break;
        case OR_FMT_NVFP4:
            quant_nvfp4_row(&q, r, v, deq);
            break;
        case OR_FMT_MXFP4:
            quant_mxfp4_row(&q, r, v, deq);
            break;
        }
        for (int64_t j = 0; j < n; ++j) {
            double d = (double)v[j] - (double)deq[j];
            e_q += d * d;
        }
    }
    if (energy) {
        energy[0] = e_total;
        energy[1] = e_prune;
        energy[2] = a->pattern == OR_DENSE ? 0.0 : e_q;
        energy[3] = a->pattern == OR_DENSE ? e_q : 0.0;
    }
    free(xr);
    free(v);
    free(deq);
    free(kidx);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Derived quantities (§4) and equal-bit accounting (§2)                      */
/* ------------------------------------------------------------------------- */

/* From the sparse side's energies (E_total, E_prune, E_q at 2m bits) and the
 * dense side's (E_q,dense at m+1 bits):
 *   out[0] = 2:4 energy loss          = E_prune / E_total
 *   out[1] = sparse relative error    = sqrt((E_prune + E_q) / E_total)
 *   out[2] = dense relative error     = sqrt(E_q,dense / E_total)
 *   out[3] = predicted R              = sqrt((E_prune + E_q) / E_q,dense)
 * E_total is taken from the sparse side (both sides see the same tensor). */
void oracle_ratio(const double *sparse_e, const double *dense_e, double *out)
{
    double et = sparse_e[0], ep = sparse_e[1], eq = sparse_e[2], ed = dense_e[3];
    out[0] = ep / et;
    out[1] = sqrt((ep + eq) / et);
    out[2] = sqrt(ed / et);
    out[3] = sqrt((ep + eq) / ed);
}

/* Stored bits per ORIGINAL element (§2: every stored bit is charged, values,
 * indices and scales). Value bits: NONE -> 16 (bf16); FP8 -> 8; INT -> bits;
 * NVFP4 / MXFP4 -> 4. A sparse pattern keeps half the values and adds its
 * position index: 2:4 -> 2 bits per kept value = 1 bit per original element;
 * 4:8 -> 2 bits per 8 elements = 0.25. Scale bits (with_scales): INT 32 bits
 * per group (group 0: per row of k_q values), NVFP4 8 per 16 plus 32 per
 * tensor (ignored, O(1/size)), MXFP4 8 per 32 quantized values. */
double oracle_bits_per_element(int32_t fmt, int32_t bits, int32_t group, int32_t pattern,
                               int64_t k, int32_t with_scales)
{
    double vb = fmt == OR_FMT_NONE ? 16.0
              : fmt == OR_FMT_FP8 ? 8.0
              : fmt == OR_FMT_INT ? (double)bits
              : 4.0;
    double kept_frac = pattern == OR_DENSE ? 1.0 : 0.5;
    double index_bits = pattern == OR_SPARSE_24 ? 1.0 : pattern == OR_SPARSE_48 ? 0.25 : 0.0;
    double total = kept_frac * vb + index_bits;
    if (with_scales) {
        double nq = kept_frac * (double)k; /* quantized values per row */
        double per_q = 0.0;
        if (fmt == OR_FMT_INT)
            per_q = 32.0 / (group ? (double)group : nq);
        else if (fmt == OR_FMT_NVFP4)
            per_q = 8.0 / 16.0;
        else if (fmt == OR_FMT_MXFP4)
            per_q = 8.0 / 32.0;
        total += kept_frac * per_q;
    }
    return total;
}

/* The per-tensor scale a pass derives when none is given (§3): FP8
 * s = amax / 448, NVFP4 s_t = amax / (6 * 448), over the values that get
 * quantized. Lets a test check sampled rows of a large operand with the scale
 * of the whole tensor. */
float oracle_scale_of_amax(float amax, int32_t fmt)
{
    return fmt == OR_FMT_FP8 ? amax / 448.0f : amax / 2688.0f;
}

float oracle_tensor_scale(const oracle_args *a)
{
    return oracle_scale_of_amax(oracle_amax(a), a->fmt);
}

/* ------------------------------------------------------------------------- */
/* Dequantization: the stored outputs back to a dense operand                 */
/* ------------------------------------------------------------------------- */

/* The dequantized value of entry j of quantized row r, from the stored codes
 * and scales, formed exactly as the pass forms it (decode(code) * scale, one
 * binary32 product); format NONE returns the kept value itself. */
static float dequant_entry(const oracle_args *a, const oracle_outputs *o, int64_t r, int64_t n, int64_t j)
{
    switch (a->fmt) {
    case OR_FMT_NONE:
        if (a->dtype == OR_BF16)
            return oracle_bf16_to_f32(((const uint16_t *)o->values)[r * n + j]);
        return ((const float *)o->values)[r * n + j];
    case OR_FMT_FP8:
        return oracle_e4m3_decode(((const uint8_t *)o->values)[r * n + j]) * o->tensor_scale[0];
    case OR_FMT_INT: {
        int64_t g = a->group ? a->group : n;
        int code;
        if (a->pack4) {
            int nib = (((const uint8_t *)o->values)[(r * n + j) / 2] >> (4 * ((r * n + j) % 2))) & 0xF;
            code = nib >= 8 ? nib - 16 : nib; /* two's-complement nibble */
        } else if (a->bits > 8) {
            code = ((const int16_t *)o->values)[r * n + j];
        } else {
            code = ((const int8_t *)o->values)[r * n + j];
        }
        return (float)code * ((const float *)o->scales)[r * (n / g) + j / g];
    }
    case OR_FMT_NVFP4: {
        uint8_t sb = ((const uint8_t *)o->scales)[r * (n / 16) + j / 16];
        float denom = oracle_e4m3_decode(sb) * o->tensor_scale[0];
        uint8_t code = (((const uint8_t *)o->values)[(r * n + j) / 2] >> (4 * ((r * n + j) % 2))) & 0xF;
        return oracle_e2m1_decode(code) * denom;
    }
    default: { /* OR_FMT_MXFP4 */
        uint8_t byte = ((const uint8_t *)o->scales)[r * (n / 32) + j / 32];
        float scale = ldexpf(1.0f, (int)byte - 127);
        uint8_t code = (((const uint8_t *)o->values)[(r * n + j) / 2] >> (4 * ((r * n + j) % 2))) & 0xF;
        return oracle_e2m1_decode(code) * scale;
    }
    }
}

/* The dense operand the stored outputs stand for (§4: the 2:4 error of an
 * element is x - x_hat, with x_hat the dequantized value on kept positions and
 * 0 on dropped ones): xhat[r * k + c] for the operand's rows and columns (row
 * major, axis-1 layout). Sparse patterns place the quantized row's entries at
 * the positions the metadata records (2:4: nibble i0 | i1 << 2 per group of 4,
 * two groups per byte, even group low; 4:8: nibble p0 | p1 << 2 per 8, the
 * pairs 2p, 2p + 1). Returns 0, or -1 for arguments it does not support. */
int oracle_dequantize(const oracle_args *a, const oracle_outputs *o, float *xhat)
{
    if (!a || !o || !xhat || a->rows < 0 || a->k <= 0)
        return -1;
    int sparse = a->pattern != OR_DENSE;
    int64_t k = a->k, n = sparse ? k / 2 : k;
    for (int64_t r = 0; r < a->rows; ++r) {
        float *row = xhat + r * k;
        for (int64_t c = 0; c < k; ++c)
            row[c] = 0.0f;
        if (!sparse) {
            for (int64_t c = 0; c < k; ++c)
                row[c] = dequant_entry(a, o, r, n, c);
            continue;
        }
        int gsize = a->pattern == OR_SPARSE_48 ? 8 : 4;
        int64_t mrow = k / (2 * gsize); /* metadata bytes per row */
        for (int64_t gi = 0; gi < k / gsize; ++gi) {
            uint8_t byte = o->meta[r * mrow + gi / 2];
            int nib = (gi % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            int64_t j = gi * 2 * (gsize / 4); /* first quantized entry of the group */
            int64_t c0 = gi * gsize;
            if (gsize == 4) {
                row[c0 + (nib & 3)] = dequant_entry(a, o, r, n, j);
                row[c0 + (nib >> 2)] = dequant_entry(a, o, r, n, j + 1);
            } else {
                int p0 = nib & 3, p1 = nib >> 2;
                row[c0 + 2 * p0] = dequant_entry(a, o, r, n, j);
                row[c0 + 2 * p0 + 1] = dequant_entry(a, o, r, n, j + 1);
                row[c0 + 2 * p1] = dequant_entry(a, o, r, n, j + 2);
                row[c0 + 2 * p1 + 1] = dequant_entry(a, o, r, n, j + 3);
            }
        }
    }
    return 0;
}

/* Block-scale tiles: the layout in which the tensor cores' block-scaled MMA
 * takes its scale factors (one byte each, E4M3 for NVFP4, E8M0 for MXFP4).
 * This is not in the pages: it is the layout NVIDIA documents for block-scaled
 * GEMM operands (cuBLAS library documentation, "1D block scaling factors
 * layout"). The scale matrix of rows x cols bytes (cols = scale blocks along
 * the reduction axis) is padded with zero bytes to a multiple of 128 rows and
 * 4 columns and cut into 128 x 4 tiles. Tiles are stored row-tile major
 * (column tiles inner), 512 bytes each. Inside a tile, row r = 32 a + b and
 * column j go to byte 16 b + 4 a + j.
 * A batch is stored operand after operand, the input packed (rows * cols
 * bytes per operand), the output tiles_bytes(rows, cols) per operand.
 * Returns 0, or -1 for arguments it does not support. */
int64_t oracle_scale_tiles_bytes(int64_t rows, int64_t cols)
{
    if (rows < 0 || cols < 0)
        return -1;
    int64_t rt = (rows + 127) / 128, ct = (cols + 3) / 4;
    return rt * ct * 512;
}

int oracle_scale_tiles(const uint8_t *in, int64_t rows, int64_t cols, int64_t batch, uint8_t *out)
{
    if (rows < 0 || cols < 0 || batch < 1 || (!in && rows * cols > 0) || !out)
        return -1;
    int64_t ct = (cols + 3) / 4;
    int64_t per_op = oracle_scale_tiles_bytes(rows, cols);
    for (int64_t b = 0; b < batch; ++b) {
        const uint8_t *src = in ? in + b * rows * cols : NULL;
        uint8_t *dst = out + b * per_op;
        for (int64_t i = 0; i < per_op; ++i)
            dst[i] = 0;
        for (int64_t r = 0; r < rows; ++r) {
            for (int64_t c = 0; c < cols; ++c) {
                int64_t tile = (r / 128) * ct + c / 4;
                int64_t rr = r % 128;
                int64_t within = 16 * (rr % 32) + 4 * (rr / 32) + c % 4;
                dst[tile * 512 + within] = src[r * cols + c];
            }
        }
    }
    return 0;
}

/* Block Hadamard rotation along the reduction axis. The pages (§4) note that
 * tensors are often multiplied by a Hadamard matrix (an orthogonal matrix of
 * +-1 entries, rescaled) before low-bit quantization, which spreads outliers
 * over many elements and, by their analysis, raises R. They do not fix the
 * block size. Reading taken: block-diagonal along k with block size b (a power
 * of two from 2 to 256 dividing k); each block of b consecutive elements of a
 * row is multiplied by the Sylvester matrix H_b (H_1 = [1],
 * H_2m = [[H_m, H_m], [H_m, -H_m]]) and by 1/sqrt(b).
 * Arithmetic, binary32: the fast Walsh-Hadamard butterflies in stage order
 * h = 1, 2, 4, ..., b/2, each pair (y_i, y_i+h) with (i & h) == 0 becoming
 * (y_i + y_i+h, y_i - y_i+h), each result rounded; then every element times
 * c_b = RN(1/sqrt(b)) (exact when b is a power of 4).
 * x: rows x k values with row stride ld (>= k); out: rows x k, packed.
 * Returns 0, or -1 for arguments it does not support. */
float oracle_hadamard_scale(int32_t b)
{
    return (float)(1.0 / sqrt((double)b));
}

int oracle_hadamard(const float *x, int64_t rows, int64_t k, int64_t ld, int32_t b, float *out)
{
    if (!x || !out || rows < 0 || k <= 0 || ld < k || b < 2 || b > 256 || (b & (b - 1)) != 0 || k % b != 0)
        return -1;
    float y[256];
    const float cb = oracle_hadamard_scale(b);
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t c0 = 0; c0 < k; c0 += b) {
            for (int32_t i = 0; i < b; ++i)
                y[i] = x[r * ld + c0 + i];
            for (int32_t h = 1; h < b; h *= 2) {
                for (int32_t i = 0; i < b; ++i) {
                    if (i & h)
                        continue;
                    float a = y[i], c = y[i + h];
                    y[i] = a + c;
                    y[i + h] = a - c;
                }
            }
            for (int32_t i = 0; i < b; ++i)
                out[r * k + c0 + i] = y[i] * cb;
        }
    }
    return 0;
}

/* ---- attention probabilities: P = softmax(alpha * s) per row ----------------
 * The producer of an attention operand (§3: P pruned along the key axis;
 * the pages build it as softmax(N(0, 3) logits / sqrt(128))). A fused
 * producer computes P and prunes it in the same pass; for its results to be
 * reproducible bit for bit, the exponential and the order of the row sum are
 * fixed here (the pages leave both open):
 *   v_j = RN(alpha * s_j); m = max_j v_j; e_j = exp_ss(RN(v_j - m));
 *   S = sum of the 256-element slices' sums, left to right, each slice summed
 *       pairwise in index order (adjacent pairs, then adjacent pairs of pairs);
 *   p_j = RN(e_j / S), then rounded to bf16 (nearest even): the bf16 operand
 *   the pass prunes.
 * exp_ss(x), x <= 0, binary32, after Cody and Waite's argument reduction
 * (W. J. Cody, W. Waite, "Software Manual for the Elementary Functions", 1980):
 *   x' = max(x, -104); t = RN(x' log2e); n = RN(RN(t + 1.5 * 2^23) - 1.5 * 2^23)
 *   (t rounded to an integer, ties to even); r = fma(-n, ln2_hi, x'),
 *   r = fma(-n, ln2_lo, r) (ln2_hi = 0.693145751953125 exactly,
 *   ln2_lo = RN(ln 2 - ln2_hi)); q = the Taylor polynomial of e^r of degree 7
 *   in Horner form with fused multiply-adds (coefficients RN(1/k!));
 *   exp_ss = RN(RN(q * 2^(n + 64)) * 2^-64), i.e. q * 2^n rounded once (the
 *   first product is exact). At x' = -104 the result rounds to 0. */
float oracle_exp_ss(float x)
{
    const float xc = x < -104.0f ? -104.0f : x;
    const float log2e = 1.44269502162933349609375f; /* RN(log2 e), 0x3fb8aa3b */
    const float ln2_hi = 0.693145751953125f;          /* 0x3f317200 */
    const float ln2_lo = 1.428606765330187e-06f;      /* 0x35bfbe8e */
    const float magic = 12582912.0f;                  /* 1.5 * 2^23 */
    float t = xc * log2e;
    float tm = t + magic;
    float n = tm - magic;
    float r = fmaf(-n, ln2_hi, xc);
    r = fmaf(-n, ln2_lo, r);
    const float c7 = 1.98412701138295233249664306640625e-04f; /* RN(1/5040) */
    const float c6 = 1.38888892251998186111450195312500e-03f; /* RN(1/720) */
    const float c5 = 8.33333376795053482055664062500000e-03f; /* RN(1/120) */
    const float c4 = 4.16666679084300994873046875000000e-02f; /* RN(1/24) */
    const float c3 = 1.66666671633720397949218750000000e-01f; /* RN(1/6) */
    float q = c7;
    q = fmaf(q, r, c6);
    q = fmaf(q, r, c5);
    q = fmaf(q, r, c4);
    q = fmaf(q, r, c3);
    q = fmaf(q, r, 0.5f);
    q = fmaf(q, r, 1.0f);
    q = fmaf(q, r, 1.0f);
    const int ni = (int)n; /* in [-150, 0] */
    union {
        uint32_t u;
        float f;
    } s2;
    s2.u = (uint32_t)(ni + 64 + 127) << 23; /* 2^(n + 64), normal */
    float up = q * s2.f;
    return up * 0x1p-64f;
}

static uint16_t f32_to_bf16_rne(float f)
{
    union {
        float f;
        uint32_t u;
    } v;
    v.f = f;
    return (uint16_t)((v.u + 0x7fffu + ((v.u >> 16) & 1u)) >> 16); /* finite inputs */
}

/* s: rows x k logits (row stride ld), fp32 values (a bf16 operand widened
 * exactly); k a multiple of 256. p_bits: rows x k bf16 bit patterns. */
int oracle_softmax_bf16(const float *s, int64_t rows, int64_t k, int64_t ld, float alpha, uint16_t *p_bits)
{
    if (!s || !p_bits || rows < 0 || k <= 0 || k % 256 != 0 || ld < k)
        return -1;
    float *e = (float *)malloc((size_t)k * sizeof(float));
    if (!e)
        return -1;
    for (int64_t r = 0; r < rows; ++r) {
        const float *row = s + r * ld;
        float m = alpha * row[0];
        for (int64_t j = 1; j < k; ++j) {
            float v = alpha * row[j];
            if (v > m)
                m = v;
        }
        for (int64_t j = 0; j < k; ++j) {
            float v = alpha * row[j];
            e[j] = oracle_exp_ss(v - m);
        }
        float total = 0.0f;
        for (int64_t t0 = 0; t0 < k; t0 += 256) {
            float buf[256];
            for (int i = 0; i < 256; ++i)
                buf[i] = e[t0 + i];
            for (int w = 256; w > 1; w /= 2) /* pairwise: adjacent pairs first */
                for (int i = 0; i < w / 2; ++i)
                    buf[i] = buf[2 * i] + buf[2 * i + 1];
            total = t0 == 0 ? buf[0] : total + buf[0];
        }
        for (int64_t j = 0; j < k; ++j)
            p_bits[r * k + j] = f32_to_bf16_rne(e[j] / total);
    }
    free(e);
    return 0;
}

/* The same probabilities as the plain definition, without the fixed choices
 * above: v_j = RN(alpha * s_j) (the binary32 scaling of the logits), then in
 * binary64 e_j = exp(v_j - m) with libm's exp, S = sum of e_j in index order,
 * p_j = e_j / S, and p_j rounded once from binary64 to bf16 (nearest, ties to
 * even). An exponential within an ulp of e^x and any accurate order of the row
 * sum give a binary32 p within a few binary32 ulps of this p_j, so their bf16
 * roundings differ by at most one bf16 ulp from the bf16 p_j here. Same
 * arguments and layout as oracle_softmax_bf16 (k a multiple of 256 is not
 * required). */
static uint16_t f64_to_bf16_rne(double d)
{
    /* d >= 0 finite. bf16 has an 8-bit significand; below 2^-126 its steps
     * are 2^-133 (subnormal). q = d / step is exact (a power-of-two scaling);
     * nearbyint rounds it to an integer, ties to even. */
    if (d == 0.0)
        return 0;
    int e;
    (void)frexp(d, &e); /* d = f * 2^e, f in [0.5, 1) */
    int step_exp = e - 8;
    if (step_exp < -133)
        step_exp = -133;
    const double q = ldexp(d, -step_exp);
    const double r = ldexp(nearbyint(q), step_exp); /* exactly a bf16 value */
    union {
        float f;
        uint32_t u;
    } v;
    v.f = (float)r; /* exact */
    return (uint16_t)(v.u >> 16);
}

int oracle_softmax_f64_bf16(const float *s, int64_t rows, int64_t k, int64_t ld, float alpha, uint16_t *p_bits)
{
    if (!s || !p_bits || rows < 0 || k <= 0 || ld < k)
        return -1;
    double *e = (double *)malloc((size_t)k * sizeof(double));
    if (!e)
        return -1;
    for (int64_t r = 0; r < rows; ++r) {
        const float *row = s + r * ld;
        float m = alpha * row[0];
        for (int64_t j = 1; j < k; ++j) {
            float v = alpha * row[j];
            if (v > m)
                m = v;
        }
        double total = 0.0;
        for (int64_t j = 0; j < k; ++j) {
            float v = alpha * row[j];
            e[j] = exp((double)v - (double)m);
            total += e[j];
        }
        for (int64_t j = 0; j < k; ++j)
            p_bits[r * k + j] = f64_to_bf16_rne(e[j] / total);
    }
    free(e);
    return 0;
}

/* The rotation as a fused pass applies it: oracle_hadamard's binary32 result
 * rounded to bf16 (nearest even), the operand dtype the pass then prunes and
 * quantizes (an online rotation feeding a bf16 GEMM stores bf16). out_bits:
 * rows x k bf16 bit patterns. Returns 0, or -1 as oracle_hadamard. */
int oracle_hadamard_bf16(const float *x, int64_t rows, int64_t k, int64_t ld, int32_t b, uint16_t *out_bits)
{
    if (!x || !out_bits || rows < 0)
        return -1;
    float *tmp = (float *)malloc((size_t)(rows > 0 ? rows : 1) * (size_t)k * sizeof(float));
    if (!tmp)
        return -1;
    int rc = oracle_hadamard(x, rows, k, ld, b, tmp);
    if (rc == 0)
        for (int64_t i = 0; i < rows * k; ++i)
            out_bits[i] = f32_to_bf16_rne(tmp[i]);
    free(tmp);
    return rc;
}
