/*
 * ss24.h — C ABI of the online 2:4 prune / compress / quantize / error-energy
 * library for NVIDIA B200 (sm_100a).
 *
 * What it computes. "Is 2:4 Sparsity Still Worth It? Semi-Structured Sparsity
 * versus Quantization in LLM Inference" (English digest, paper-daily.com):
 *   intro  2:4 keeps two non-zeros of every four along a GEMM operand's
 *          reduction axis.
 *   §1     operands computed on the fly (activations, Q, K, V, P) must be
 *          pruned and compressed before every GEMM, and that cost counts.
 *   §2     the pruners' scores (magnitude; Wanda = |W| times the activation
 *          size of the input channel), plain round-to-nearest quantization,
 *          and equal-bit accounting (a 1-bit index per original element).
 *   §3     the formats (FP8, INT8 with one scale per row, NVFP4, MXFP4) and the
 *          fused kernel that reads the input once and writes kept values and
 *          indices once.
 *   §4     the 2:4 energy loss, the disjoint pruning / quantization error
 *          energies and the predicted ratio R.
 *   §6     pairwise 4:8 (keep two of the four adjacent pairs of each eight).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Operand. A logical matrix A[rows][k]; k is the reduction axis, along which
 * groups of 4 (2:4) or 8 (4:8) consecutive elements are formed. Memory:
 *   axis = 1: A[r][c] is at x[r * ld + c]   (k contiguous; ld >= k)
 *   axis = 0: A[r][c] is at x[c * ld + r]   (rows contiguous, e.g. V pruned
 *             along the key axis; ld >= rows)
 * Element type bf16 or fp32. Inputs are finite; NaN / Inf give unspecified
 * codes. Energies are accurate for |x| below 2^60 (binary32 squares).
 *
 * Outputs are always row-major with k (or the kept half of it) contiguous,
 * one row per logical row, no padding. With n = k/2 for a sparse pattern and
 * n = k for the dense pattern:
 *   kept values (format NONE)  input dtype [rows][n]
 *   FP8 E4M3 codes             u8 [rows][n]
 *   INT codes                  int8 [rows][n] (bits <= 8), int16 [rows][n]
 *                              (bits > 8), or with pack4 (bits <= 4) u8
 *                              [rows][n/2], two's-complement nibbles, element
 *                              2j in the low nibble
 *   INT scales                 fp32 [rows][n/group] (group 0: [rows][1])
 *   NVFP4 codes / scales       u8 [rows][n/2] (element 2j in the low nibble) /
 *                              E4M3 u8 [rows][n/16], plus fp32 tensor scale
 *   MXFP4 codes / scales       u8 [rows][n/2] / E8M0 u8 [rows][n/32]
 *   2:4 metadata               u8 [rows][k/8]: group g's nibble i0 | i1 << 2
 *                              (kept positions, i0 < i1) in byte g/2, even g in
 *                              the low nibble
 *   4:8 metadata               u8 [rows][k/16]: octet o's nibble p0 | p1 << 2
 *                              (kept pairs) in byte o/2, even o in the low nibble
 * Scales of the kept values are taken over the compressed row: an INT group of
 * g covers g kept values (2g original positions), an NVFP4 block 16 kept
 * values, an MXFP4 block 32.
 *
 * Batches. An operand descriptor with batch = B > 1 describes B operands of the
 * same shape, operand b at x + b * batch_stride. One call then processes all
 * of them (one launch per kernel instead of B), each exactly as a call on that
 * operand alone would: per-tensor scales, amaxes and energies are per operand.
 * Every output holds the B operands' outputs one after the other (the
 * per-operand layouts above, packed): values, scales and metadata as
 * [B][rows][...], tensor scales as float[B], tensor_scale_in as float[B],
 * energy records as ss24_energy[B], amax outputs as float[B]. col_norms is
 * shared by all operands.
 *
 * Selection. Element i beats element j when s_i > s_j, or s_i == s_j and
 * i < j; the two elements beaten by fewer than two others are kept (ties keep
 * the lower index). Scores: SS24_SCORE_MAG s = |x|; SS24_SCORE_WANDA
 * s = |x| * col_norms[c] rounded to binary32 (col_norms: fp32 [k], >= 0).
 * Pairwise 4:8 ranks pair p by s_{2p}*s_{2p} + s_{2p+1}*s_{2p+1} (binary32,
 * each product and the sum rounded) with the same rule over the four pairs.
 *
 * Quantization (round to nearest, ties to even; every division is an IEEE
 * binary32 division, every product one binary32 rounding, no contraction):
 *   FP8    s = amax / 448; code = E4M3satfinite(v / s); deq = E4M3(code) * s
 *   INT-b  qmax = 2^(b-1) - 1; scale = amax_group / qmax;
 *          code = clamp(rint(v / scale), -qmax, qmax); deq = code * scale
 *   NVFP4  s_t = amax / 2688; sb = E4M3satfinite((amax_block / 6) / s_t);
 *          denom = E4M3(sb) * s_t; code = E2M1satfinite(v / denom);
 *          deq = E2M1(code) * denom
 *   MXFP4  e = clamp(floor(log2(amax_block)) - 2, -127, 127); byte = e + 127;
 *          code = E2M1satfinite(v / 2^e); deq = E2M1(code) * 2^e
 * A zero scale (or zero block amax for MXFP4, which then stores byte 0) gives
 * all-zero codes. The per-tensor amax of a sparse pattern is taken over the
 * kept values (equal to the amax of all values for the magnitude score).
 *
 * Energies. ss24_energy holds binary64 sums (§4):
 *   e_total        sum over all elements of x^2
 *   e_prune        sum over dropped elements of x^2
 *   e_quant        sum over kept elements of (x - deq)^2 (sparse side)
 *   e_quant_dense  sum over all elements of (x - deq)^2 (dense side)
 * Fields a call does not compute are written as 0. Per-element terms are
 * formed in binary32 and summed in short binary32 trees before binary64
 * accumulation; the sums match a binary64 reference to about 5e-7 relative.
 * Results are deterministic run to run (fixed reduction order, no atomics).
 *
 * Memory and ownership. Every pointer argument except the descriptor structs
 * is DEVICE memory owned by the caller; the library allocates nothing and
 * keeps no state between calls. The descriptor structs (ss24_operand,
 * ss24_outputs) are read on the host during the call and may be reused
 * immediately. Data pointers must be 16-byte aligned and, for axis 1,
 * ld * sizeof(dtype) must be a multiple of 16 (axis 0: likewise).
 *
 * Workspace. Calls take a device workspace of ss24_workspace_bytes() bytes,
 * 256-byte aligned, that must have been cleared once with
 * ss24_workspace_init(). Concurrent calls need distinct workspaces.
 *
 * Asynchrony and errors. Every call validates its arguments on the host and,
 * if they are invalid, returns an SS24_ERR_* status and launches nothing.
 * Otherwise it enqueues its kernels on `stream` (NULL: the legacy default
 * stream) and returns SS24_OK, or SS24_ERR_CUDA if a launch failed. Results
 * are valid once the stream is synchronized. Kernels never trap: an internal
 * wait that exceeds about two seconds records a nonzero code in the
 * workspace (read with ss24_workspace_error) and the kernel returns; its
 * outputs and energies are then incomplete. The only kernels with such waits
 * are those of the strided axis (axis 0), which wait on their tile copies.
 *
 * Test hook. When the environment variable SS24_TEST_SKIP_TILE holds a
 * number t >= 0 at the time of a call, the first CTA of that call's
 * strided-axis kernel does not copy its t-th tile and every wait of the
 * kernel gives up after 10 ms instead of two seconds: a wait runs out on
 * purpose, and the error word shows it. For tests of that path only.
 */
#ifndef SS24_H
#define SS24_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st *ss24_stream;

typedef enum {
    SS24_OK = 0,
    SS24_ERR_NULL = 1,      /* a required pointer is NULL                            */
    SS24_ERR_SHAPE = 2,     /* rows / k / ld do not fit the pattern or format        */
    SS24_ERR_ALIGN = 3,     /* a pointer or the row stride is not 16-byte aligned    */
    SS24_ERR_DTYPE = 4,     /* unknown element type                                  */
    SS24_ERR_FORMAT = 5,    /* unknown format, bits out of range, bad group / pack4  */
    SS24_ERR_WORKSPACE = 6, /* workspace missing, too small or misaligned            */
    SS24_ERR_CUDA = 7,      /* a CUDA runtime call or a launch failed                */
    SS24_ERR_ARG = 8        /* unknown score, axis or pattern                        */
} ss24_status;

typedef enum { SS24_BF16 = 0, SS24_F32 = 1 } ss24_dtype;
typedef enum { SS24_SCORE_MAG = 0, SS24_SCORE_WANDA = 1 } ss24_score;
typedef enum { SS24_DENSE = 0, SS24_SPARSE_24 = 24, SS24_SPARSE_48 = 48 } ss24_pattern;
typedef enum {
    SS24_FMT_NONE = 0,     /* kept values stored unchanged (sparse patterns only) */
    SS24_FMT_FP8_E4M3 = 1, /* per-tensor scale                                    */
    SS24_FMT_INT = 2,      /* bits 2..16, per-group or per-row fp32 scales        */
    SS24_FMT_NVFP4 = 3,
    SS24_FMT_MXFP4 = 4
} ss24_fmt_kind;

/* Quantization format. `bits`, `group`, `pack4` are read for SS24_FMT_INT only:
 * bits in [2, 16]; group = 0 (one scale per row) or a power of two g with
 * 8 <= g * (2 for sparse, 1 for dense) <= 256 dividing the quantized row;
 * pack4 = 1 packs two codes per byte (bits <= 4). */
typedef struct {
    int32_t kind;
    int32_t bits;
    int32_t group;
    int32_t pack4;
} ss24_format;

typedef struct {
    const void *x;        /* device pointer to the (first) operand                */
    int32_t dtype;        /* ss24_dtype                                            */
    int32_t axis;         /* 1: k contiguous; 0: rows contiguous                   */
    int64_t rows;         /* logical rows (>= 0; 0 is a valid empty operand)       */
    int64_t k;            /* reduction length (> 0)                                */
    int64_t ld;           /* elements between consecutive rows (axis 1) or
                             consecutive k positions (axis 0)                      */
    int64_t batch;        /* operands in the call: 0 or 1 for one, up to 1024      */
    int64_t batch_stride; /* elements from one operand to the next (batch > 1);
                             at least rows * ld (axis 1) or k * ld (axis 0)       */
    int32_t hadamard;     /* 0, or a block size b (a power of two, 2..256, dividing
                             k): the pass takes the operand rotated along k, each
                             block of b elements times the Sylvester matrix H_b and
                             RN(1/sqrt(b)) as ss24_hadamard computes it, then
                             rounded to bf16 (nearest even); §4 (rotation before
                             quantization). bf16, axis 1, magnitude score only,
                             and not the row-block INT pass (one scale per row
                             without a given row amax): SS24_ERR_ARG otherwise. */
    int32_t reserved;     /* 0                                                     */
} ss24_operand;

typedef struct {
    double e_total, e_prune, e_quant, e_quant_dense;
} ss24_energy;

typedef struct {
    double loss;           /* e_prune / e_total                                   */
    double rel_err_sparse; /* sqrt((e_prune + e_quant) / e_total)                 */
    double rel_err_dense;  /* sqrt(e_quant_dense / e_total)                       */
    double r_hat;          /* sqrt((e_prune + e_quant) / e_quant_dense), §4       */
} ss24_ratio;

typedef struct {
    void *values;        /* kept values or codes (layout above)                 */
    void *scales;        /* INT / NVFP4 / MXFP4 scales; NULL for NONE and FP8    */
    float *tensor_scale; /* FP8 / NVFP4: receives the per-tensor scale used     */
    uint8_t *meta;       /* metadata (sparse patterns); NULL for dense           */
} ss24_outputs;

/* ---- workspace ----------------------------------------------------------- */

/* Bytes of device workspace every computing call needs (a constant). */
size_t ss24_workspace_bytes(void);

/* Clears the workspace's error word and ticket counters (a stream-ordered
 * memset of its first 8,448 bytes). Call once after allocating the workspace,
 * and again to reset a recorded error. */
ss24_status ss24_workspace_init(void *ws, size_t ws_bytes, ss24_stream stream);

/* Synchronizes `stream`, then copies the workspace's error word to *code
 * (0: no kernel gave up on a wait). */
ss24_status ss24_workspace_error(const void *ws, int32_t *code, ss24_stream stream);

/* ---- the pass -------------------------------------------------------------- */

/* 2:4 prune + compress (intro, §2 scores, §3 fused read-once / write-once
 * kernel). Writes the kept values in the input dtype to `kept` [rows][k/2] and
 * the metadata to `meta` [rows][k/8]. `energy` (may be NULL) receives e_total
 * and e_prune. col_norms is required for SS24_SCORE_WANDA, ignored otherwise.
 * k must be a multiple of 8. */
ss24_status ss24_prune24_compress(const ss24_operand *x, ss24_score score, const float *col_norms,
                                  void *kept, uint8_t *meta, ss24_energy *energy, void *ws,
                                  size_t ws_bytes, ss24_stream stream);

/* Dense FP8 E4M3 with one scale per tensor (§3). tensor_scale_in: device
 * pointer to a given scale s, or NULL to compute s = amax / 448 (an extra
 * read-only pass). out->values u8 [rows][k]; out->tensor_scale receives s.
 * energy (may be NULL) receives e_total and e_quant_dense. k % 8 == 0. */
ss24_status ss24_quantize_fp8(const ss24_operand *x, const float *tensor_scale_in,
                              ss24_outputs *out, ss24_energy *energy, void *ws, size_t ws_bytes,
                              ss24_stream stream);

/* Dense symmetric INT-b with per-group or per-row scales (§3: INT8 with one
 * scale per row; §2 equal-bit partners INT3 ... INT9). fmt.kind must be
 * SS24_FMT_INT. energy receives e_total and e_quant_dense. */
ss24_status ss24_quantize_int(const ss24_operand *x, ss24_format fmt, ss24_outputs *out,
                              ss24_energy *energy, void *ws, size_t ws_bytes, ss24_stream stream);

/* Dense NVFP4 (§3: FP8 scale per 16 plus one per tensor). tensor_scale_in as
 * for FP8 (NULL: s_t = amax / 2688). k % 16 == 0. */
ss24_status ss24_quantize_nvfp4(const ss24_operand *x, const float *tensor_scale_in,
                                ss24_outputs *out, ss24_energy *energy, void *ws, size_t ws_bytes,
                                ss24_stream stream);

/* Dense MXFP4 (§3: one power-of-two scale per 32). k % 32 == 0. */
ss24_status ss24_quantize_mxfp4(const ss24_operand *x, ss24_outputs *out, ss24_energy *energy,
                                void *ws, size_t ws_bytes, ss24_stream stream);

/* The fused online pass (§3): one read of the operand, 2:4 selection, and the
 * kept values written once, quantized to `fmt` (NONE: unchanged), with the
 * metadata; energy receives e_total, e_prune and e_quant (§4).
 * tensor_scale_in is read for FP8 / NVFP4 (NULL: computed from the amax of
 * the kept values by an extra read-only pass). Constraints: k % 8 == 0 and the
 * format's unit on the kept row (NVFP4 k % 32, MXFP4 k % 64, INT k % (2g)). */
ss24_status ss24_prune24_quant_fused(const ss24_operand *x, ss24_score score,
                                     const float *col_norms, ss24_format fmt,
                                     const float *tensor_scale_in, ss24_outputs *out,
                                     ss24_energy *energy, void *ws, size_t ws_bytes,
                                     ss24_stream stream);

/* Pairwise 4:8 variant of the fused pass (§6: keep two of the four adjacent
 * pairs of each eight, ranked by pair energy). meta is u8 [rows][k/16];
 * k % 16 == 0. Otherwise as ss24_prune24_quant_fused. */
ss24_status ss24_prune48_pairwise_quant_fused(const ss24_operand *x, ss24_score score,
                                              const float *col_norms, ss24_format fmt,
                                              const float *tensor_scale_in, ss24_outputs *out,
                                              ss24_energy *energy, void *ws, size_t ws_bytes,
                                              ss24_stream stream);

/* Read-only analysis pass (§4): in one read of the operand, the energies of
 * both sides of the comparison — pattern (2:4 or 4:8) with its kept values
 * quantized to sparse_fmt (2m bits; NONE allowed), and the whole operand
 * quantized to dense_fmt (m+1 bits; NONE not allowed). Nothing but `energy`
 * (all four fields) is written. sparse_scale_in / dense_scale_in: given
 * per-tensor scales, or NULL to compute them in an extra read-only pass. */
ss24_status ss24_error_energy(const ss24_operand *x, ss24_pattern pattern, ss24_score score,
                              const float *col_norms, ss24_format sparse_fmt,
                              ss24_format dense_fmt, const float *sparse_scale_in,
                              const float *dense_scale_in, ss24_energy *energy, void *ws,
                              size_t ws_bytes, ss24_stream stream);

/* Largest |value| among the values a pass would quantize (§3 per-tensor
 * scale): the kept values for a sparse pattern, all values for SS24_DENSE.
 * Writes one fp32 to the device pointer amax_out. */
ss24_status ss24_amax(const ss24_operand *x, ss24_pattern pattern, ss24_score score,
                      const float *col_norms, float *amax_out, void *ws, size_t ws_bytes,
                      ss24_stream stream);

/* The per-tensor scale a pass derives when it is given none (§3): FP8
 * s = amax / 448, NVFP4 s_t = amax / 2688, the amax taken over the values the
 * pass would quantize (kept values for a sparse pattern). One read-only pass;
 * writes one fp32 to the device pointer scale_out. Computing the scale ahead
 * of the quantizing pass and passing it as tensor_scale_in gives the same
 * codes as letting that pass compute it. kind: SS24_FMT_FP8_E4M3 or
 * SS24_FMT_NVFP4 (anything else: SS24_ERR_FORMAT). */
ss24_status ss24_tensor_scale(const ss24_operand *x, ss24_pattern pattern, ss24_score score,
                              const float *col_norms, int32_t kind, float *scale_out, void *ws,
                              size_t ws_bytes, ss24_stream stream);

/* Per-row amax in the same read as the per-tensor scale (§3: INT with one
 * scale per row needs the amax of each row before its codes; a pass that reads
 * the operand for the tensor scale can produce them at no extra read). Writes
 * row_amax[b * rows + r] = max |value| over the values of row r of operand b
 * that a pass with this pattern and score quantizes (the kept values for a
 * sparse pattern). row_amax: device, batch x rows fp32, 4-byte aligned (NULL
 * allowed when rows is 0); every entry is written. If scale_out is not
 * NULL it also writes the per-tensor scale of kind (SS24_FMT_FP8_E4M3 or
 * SS24_FMT_NVFP4) as ss24_tensor_scale does. Axis 1 only (SS24_ERR_ARG
 * otherwise). */
ss24_status ss24_amax_rows(const ss24_operand *x, ss24_pattern pattern, ss24_score score, const float *col_norms,
                           float *row_amax, int32_t kind, float *scale_out, void *ws, size_t ws_bytes,
                           ss24_stream stream);

/* INT-b with one scale per row (fmt.kind SS24_FMT_INT, fmt.group 0) from a
 * given per-row amax, as ss24_amax_rows writes it for the same pattern and
 * score: scale = amax / qmax per row, then the codes, metadata, scales and
 * energies of ss24_prune24_quant_fused / ss24_prune48_pairwise_quant_fused
 * (sparse patterns) or ss24_quantize_int (SS24_DENSE), identical to them when
 * row_amax holds the rows' amax. One streaming pass (the rows need not fit a
 * block of threads). row_amax: device, batch x rows fp32, 4-byte aligned.
 * Axis 1 only. */
ss24_status ss24_quantize_int_rows(const ss24_operand *x, ss24_pattern pattern, ss24_score score,
                                   const float *col_norms, ss24_format fmt, const float *row_amax,
                                   ss24_outputs *out, ss24_energy *energy, void *ws, size_t ws_bytes,
                                   ss24_stream stream);

/* Derived quantities (§4) from sparse-side energy records (e_total, e_prune,
 * e_quant) and dense-side records (e_quant_dense): count consecutive pairs,
 * sparse_side[i] with dense_side[i] -> out[i]. Device pointers; the two inputs
 * may be the same records (as ss24_error_energy writes them). One small
 * kernel; count 0 enqueues nothing. */
ss24_status ss24_predicted_ratio(const ss24_energy *sparse_side, const ss24_energy *dense_side,
                                 ss24_ratio *out, int64_t count, ss24_stream stream);

/* ---- without caller-supplied scratch ----------------------------------------- */

/* The fused 2:4 pass of ss24_prune24_quant_fused (same arguments, same results,
 * axis 1 only) for callers that cannot allocate device memory: code that runs
 * where cudaMalloc is not allowed (inside a caching allocator's own callbacks,
 * or a host that hands the library only the operand and the output buffers)
 * and so cannot provide a workspace. No counterpart in the paper: it exists for
 * such callers only.
 *
 * Scratch. The pass's scratch (per-CTA partial sums, two ticket counters and
 * an error word, 57,600 bytes: enough for the at most 1024 CTAs the pass
 * launches, whatever the operand size) lives in a device array owned by the
 * library: one copy on every GPU that loads the library, kept until the
 * process exits. The entry point allocates nothing and frees nothing.
 *
 * Errors. Every argument is checked before anything is enqueued, as for the
 * other entry points: a rejected call enqueues nothing, and leaves the array
 * as it was. An operand with axis 0 is rejected (SS24_ERR_ARG): the strided-
 * axis kernel waits on its tile copies with a time limit and records a wait
 * that gave up in the array, where the caller could not see it; the axis-1
 * kernels this entry point launches contain no such wait.
 *
 * First call on a device: it looks up the array's device address (once per
 * device and context, with that device current; a context created after a
 * device reset gets a fresh lookup); make that first call before any stream
 * capture. Every accepted call then clears the array's counters with a
 * stream-ordered memset before its first launch.
 *
 * Concurrency. All calls on a device share the one array, which keeps the
 * last call's contents: calls that overlap on the GPU (on different streams,
 * or from different host threads without ordering) race and may return wrong
 * energies. Order them on one stream. */
ss24_status ss24_prune24_quant_fused_noalloc(const ss24_operand *x, ss24_score score,
                                             const float *col_norms, ss24_format fmt,
                                             const float *tensor_scale_in, ss24_outputs *out,
                                             ss24_energy *energy, ss24_stream stream);

/* ---- host-only helpers ------------------------------------------------------ */

/* Stored bits per ORIGINAL element (§2: values, indices and, with with_scales,
 * scales are all charged). Value bits: NONE 16, FP8 8, INT bits, NVFP4 /
 * MXFP4 4; 2:4 adds 1 index bit per element, 4:8 adds 0.25. Scales: INT 32
 * bits per group (per row of the quantized length when group is 0), NVFP4
 * 8 per 16 values, MXFP4 8 per 32; the single NVFP4 / FP8 tensor scale is not
 * charged. Returns a negative value for an invalid format. */
double ss24_bits_per_element(ss24_format fmt, ss24_pattern pattern, int64_t k, int32_t with_scales);

/* Static string naming a status. */
const char *ss24_status_string(ss24_status status);

/* ---- format conversion primitives (the kernels' own converters) ------------ */

/* Encode n binary32 values to E4M3 (nearest-even, satfinite), one byte each. */
ss24_status ss24_encode_e4m3(const float *in, uint8_t *out, int64_t n, ss24_stream stream);
/* Decode n E4M3 bytes to binary32. */
ss24_status ss24_decode_e4m3(const uint8_t *in, float *out, int64_t n, ss24_stream stream);
/* Encode n binary32 values to E2M1 (nearest-even, satfinite), one code per
 * byte in the low nibble. */
ss24_status ss24_encode_e2m1(const float *in, uint8_t *out, int64_t n, ss24_stream stream);
/* Decode n E2M1 codes (low nibble of each byte) to binary32. */
ss24_status ss24_decode_e2m1(const uint8_t *in, float *out, int64_t n, ss24_stream stream);

/* ---- dequantization ------------------------------------------------------ */

/* The dense operand the outputs of a pass stand for (§4: the 2:4 error of an
 * element is x - x_hat, x_hat being the dequantized value on kept positions
 * and 0 on dropped ones). Writes xhat[b][r][c] (fp32, row major, batch x rows x
 * k, 16-byte aligned) from the outputs `in` that a pass with this pattern and
 * format wrote for an operand of x's shape (x->rows, x->k, x->batch; x->dtype
 * is the type of the kept values for SS24_FMT_NONE; x->x and the strides are
 * not read). Dequantized values are decode(code) * scale rounded once, the
 * products the pass forms, so sum (x - xhat)^2 reproduces the pass's
 * E_prune + E_quant (sparse) or E_quant_dense (dense). Layouts: those the
 * pass writes (see ss24_outputs), the operands of a batch packed one after the
 * other. Errors: SS24_ERR_NULL for a missing buffer the format needs, and the
 * shape / format checks of the passes. */
ss24_status ss24_dequantize(const ss24_operand *x, ss24_pattern pattern, ss24_format fmt, const ss24_outputs *in,
                            float *xhat, ss24_stream stream);

/* ---- self-check of the kernels' division -------------------------------- */

/* The kernels divide by a scale with Markstein's one-step correction of a
 * reciprocal (P. Markstein, IBM J. Res. Dev. 34(1), 1990) instead of an IEEE
 * division, for scales in [2^-60, 2^60]: as a / b, and in a packed form that
 * yields -(a / b) directly (the correction run with -1/b) so that codes come out
 * with their signs flipped back exactly. This entry point checks that both
 * forms agree bit for bit with IEEE division on the running GPU. mode 0: b = 1 + (b_first + j) 2^-23
 * for j < b_count, against every a in [1, 2) (2^23 significands each; b_first +
 * b_count <= 2^23 — all 2^23 values of b together cover every pair of
 * significands, which by exact power-of-two scaling covers every a and b the
 * kernels divide with the correction). mode 1: 2^23 pseudo-random pairs per
 * unit of b_count, exponents across the corrected range. mode 2 checks the
 * packed bf16 operations the 2:4 selection and the amax use (magnitude
 * comparison through a rounded bf16 difference, magnitude maximum and its
 * test against a limit, bf16 to binary32 conversion and squares on the
 * multiply-add unit) for the magnitude
 * bits a = b_first + j, j < b_count (b_first + b_count <= 2^15), against every
 * magnitude b < 2^15, finite values only, both signs; a mismatch is reported as
 * (a << 32 | b). Adds the number of
 * mismatches to result[0] and lowers result[1] to the first mismatch
 * (a bits << 32 | b bits); result is a device array of two uint64 the caller
 * initialises to {0, UINT64_MAX}. */
ss24_status ss24_selfcheck_division(int32_t mode, uint32_t b_first, uint32_t b_count,
                                    unsigned long long *result, ss24_stream stream);

/* ---- self-check of the kernels' encoders ------------------------------- */

/* The E4M3 (kind SS24_FMT_FP8_E4M3) or E2M1 (kind SS24_FMT_NVFP4 or
 * SS24_FMT_MXFP4) encoder the kernels use (round to nearest even,
 * saturating to the largest finite code) against a step table, for every fp32
 * bit pattern (hi << 16) | lo with hi in [hi_first, hi_first + hi_count) and
 * every lo, NaN and infinity excluded. bounds (device, ascending, 126 values
 * for E4M3, 7 for E2M1): bounds[i] is the smallest magnitude bit pattern whose
 * code is i + 1; the expected code of x is the number of bounds <= |x|'s bits,
 * with the sign bit (0x80, E2M1 0x8) set when x is negative (-0 included).
 * The caller derives the table from an independent encoder. Adds the number of
 * mismatches to result[0] and lowers result[1] to the first mismatching bit
 * pattern; result is a device array of two uint64 the caller initialises to
 * {0, UINT64_MAX}. Errors: SS24_ERR_NULL, SS24_ERR_FORMAT (other kinds),
 * SS24_ERR_SHAPE (wrong table length or hi range beyond 2^16). */
ss24_status ss24_selfcheck_encoder(int32_t kind, const uint32_t *bounds, int32_t n_bounds, uint32_t hi_first,
                                   uint32_t hi_count, unsigned long long *result, ss24_stream stream);

/* ---- pruning in the producer: attention probabilities ------------------------ */

/* P = softmax(alpha * s) per row, pruned and compressed along the key axis in
 * the same pass (§3: P pruned along the key axis; §1: an operand computed on
 * the fly is pruned before every GEMM): P is never stored. s: logits, bf16 or
 * fp32, axis 1 (keys contiguous), k (keys) a multiple of 256, ld and batch as
 * for the passes. The arithmetic, fixed so that results reproduce bit for bit
 * (the pages leave it open): v = RN(alpha s); m = the row max; e = exp_ss(RN(v -
 * m)); S = the row's 256-key slice sums added left to right, each slice summed
 * pairwise in index order; p = RN(e / S) rounded to bf16 (nearest even).
 * exp_ss: arguments below -104 taken as -104; Cody-Waite reduction (n = t
 * rounded to an integer, ties to even; ln 2 split into an exact high part and
 * a rounded low part), the degree-7 Taylor polynomial with coefficients
 * RN(1/k!) in fused multiply-add Horner form, times 2^n rounded once. The
 * bf16 P then goes through exactly what ss24_prune24_quant_fused (2:4), the
 * pairwise 4:8 pass or a dense quantization does to a bf16 operand by
 * magnitude: same outputs (layouts of ss24_outputs), same energies. Formats:
 * NONE (sparse patterns), FP8 and NVFP4 with the tensor scale GIVEN
 * (tensor_scale_in, device, one per operand; P <= 1, so 1/448 suits FP8),
 * MXFP4, INT with groups. Errors: the operand and output checks of the passes,
 * SS24_ERR_ARG (axis 0, alpha not finite), SS24_ERR_SHAPE (k not a multiple of
 * 256), SS24_ERR_FORMAT (INT with one scale per row), SS24_ERR_NULL (no
 * tensor scale for FP8 / NVFP4). */
ss24_status ss24_softmax_prune(const ss24_operand *s, float alpha, ss24_pattern pattern, ss24_format fmt,
                               const float *tensor_scale_in, ss24_outputs *out, ss24_energy *energy, void *ws,
                               size_t ws_bytes, ss24_stream stream);

/* ---- rotation ----------------------------------------------------------------- */

/* Block Hadamard rotation along k (§4: a Hadamard matrix, orthogonal with
 * +-1 entries rescaled, applied before low-bit quantization spreads outliers
 * and, by the pages' analysis, raises R; they do not fix the block size).
 * Every block of `block` consecutive elements of a row (block a power of two
 * from 2 to 256 dividing k; k a multiple of 8) is multiplied by the Sylvester
 * matrix H_b (H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]]) and by
 * RN(1/sqrt(block)). Arithmetic in binary32: fast Walsh-Hadamard butterflies
 * in stage order h = 1, 2, 4, ..., block/2, the pair (y_i, y_i+h) with
 * (i & h) == 0 becoming (y_i + y_i+h, y_i - y_i+h), each rounded, then one
 * rounded multiplication. x: bf16 or fp32, axis 1 only (ld >= k, batch as for
 * the passes). out (device, 16-byte aligned, owned by the caller): fp32,
 * packed [batch][rows][k]; it is the operand to hand to the passes (as fp32)
 * for a rotated pass. Errors: the operand checks of the passes, SS24_ERR_ARG
 * (axis 0, block not a power of two in [2, 256]), SS24_ERR_SHAPE (k not a
 * multiple of 8 and of block), SS24_ERR_NULL, SS24_ERR_ALIGN. */
ss24_status ss24_hadamard(const ss24_operand *x, int32_t block, float *out, ss24_stream stream);

/* ---- the consumer: 2:4-sparse GEMM on the tensor cores ---------------------- */

/* Y = s_a s_b A B^T on the 2:4-sparse FP8 MMA of the 5th-generation tensor
 * cores (§1: an operand computed on the fly is pruned and compressed before
 * every GEMM; §3: the sparse GEMM reads the kept values and their indices). A
 * is the 2:4 operand as ss24_prune24_quant_fused writes it with FP8: a_values
 * the E4M3 kept values u8 [m][k/2], a_meta the metadata u8 [m][k/8] (the
 * pass's layout is the one the sparse MMA takes, read in 128-row x 16-byte
 * tiles), a_scale its tensor scale (device fp32). B is a dense E4M3 operand u8
 * [n][k] (k contiguous; e.g. a weight through ss24_quantize_fp8) with tensor
 * scale b_scale (device fp32). y (device fp32 [m][n], row major) receives
 * RN(acc * RN(s_a * s_b)), acc the binary32 accumulation of the products.
 * Shapes: m and n multiples of 128, k a multiple of 256 (a zero m or n is an
 * empty product: nothing is launched). Pointers 16-byte aligned. The workspace
 * carries the error word of the kernel's bounded waits (ss24_workspace_error).
 * Errors: SS24_ERR_SHAPE, SS24_ERR_NULL, SS24_ERR_ALIGN, SS24_ERR_WORKSPACE,
 * SS24_ERR_CUDA. */
ss24_status ss24_sparse_gemm_fp8(const uint8_t *a_values, const uint8_t *a_meta, const float *a_scale,
                                 const uint8_t *b, const float *b_scale, int64_t m, int64_t n, int64_t k, float *y,
                                 void *ws, size_t ws_bytes, ss24_stream stream);

/* ---- consumer layouts ------------------------------------------------------ */

/* Bytes of the block-scale tiles of a rows x cols scale matrix (one operand):
 * ceil(rows / 128) * ceil(cols / 4) * 512; -1 for negative sizes. */
int64_t ss24_scale_tiles_bytes(int64_t rows, int64_t cols);

/* The NVFP4 (E4M3) or MXFP4 (E8M0) scale bytes a pass wrote, rearranged into
 * the layout in which the tensor cores' block-scaled MMA takes its scale
 * factors (NVIDIA's documented "1D block scaling factors layout"; the pages
 * give no layout, §3 only the scale granularity). `scales` holds batch
 * operands packed one after the other, each rows x cols bytes row major
 * (cols = scale blocks per row: n / 16 for NVFP4, n / 32 for MXFP4, n the
 * quantized row length), on the device. `tiles` (device, 16-byte aligned)
 * receives ss24_scale_tiles_bytes(rows, cols) bytes per operand: the matrix
 * padded with zero bytes to multiples of 128 rows and 4 columns, cut into
 * 128 x 4 tiles of 512 bytes stored row tile by row tile (column tiles
 * inner); inside a tile, row 32 a + b and column j sit at byte 16 b + 4 a + j.
 * Every byte of `tiles` is written. batch: 0 or 1 for one operand, up to
 * 1024. Errors: SS24_ERR_NULL, SS24_ERR_SHAPE (negative sizes, batch out of
 * range), SS24_ERR_ALIGN (tiles not 16-byte aligned). */
ss24_status ss24_scale_tiles(const uint8_t *scales, int64_t rows, int64_t cols, int64_t batch, uint8_t *tiles,
                             ss24_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* SS24_H */
