/*
 * fp8qgg — FP8 training quantisation for MoE expert GEMMs and the FP8 scaled
 * grouped GEMM that consumes it, for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Every tensor argument is a DEVICE pointer owned by the caller; the
 * library keeps no data between calls (only per-device caches of device
 * properties and kernel attributes, and the setting of the failure-detection
 * test hook), and every call is enqueued on `stream`
 * (a cudaStream_t passed as void*; NULL = the legacy default stream) with no
 * implicit synchronisation.  Unless a function says otherwise it allocates no
 * device memory.
 *
 * Sources, cited by page title and section:
 *  [AIR] "FP8 su GPU AMD: i guadagni di TorchTitan e TorchAO ora sono nel
 *        mainline PyTorch" (ai-radar.it)
 *  [ABP] "AMD Boosts PyTorch FP8 Training on Instinct GPUs" (latestnews.news)
 *  [PRI] "AMD Primus adds FP8/MXFP8 kernels, megakernel fusion and DeepSeek-V3
 *        training at 1024 GPUs" (fosswire.org)
 *
 * Conventions shared by every entry point
 *  - Formats: FP8QGG_E4M3FN (largest finite 448, signed zero, NaN S.1111.111)
 *    is the default; FP8QGG_E4M3FNUZ (largest finite 240, single zero, only
 *    NaN 0x80) is the format of [AIR] section "La correttezza del formato viene
 *    prima del tuning" and [ABP] third paragraph.  Scaling against the wrong
 *    maximum clips silently; `scale_max` reproduces that case on purpose and
 *    `sat_count` makes it observable.
 *  - Quantisation chain ([AIR] section "Il guadagno vero è nel movimento dei
 *    dati", first paragraph), all in one pass over HBM:
 *        amax = max |x|                       (exact; NaN inputs are skipped)
 *        s    = fp32(Fmax / max(amax, 1e-12)) (IEEE round to nearest)
 *        y    = clamp(fp32(x * s), -Fmax, Fmax)
 *        q    = e4m3(y)   round to nearest, ties to even, one rounding from
 *                         fp32, saturating; e4m3fnuz maps every zero to 0x00.
 *    Fmax = scale_max when scale_max > 0, else the format's largest finite.
 *    The stored scale is s (dequantise with decode(q) / s).  Special inputs
 *    (the pages never meet them): an infinity saturates like any magnitude
 *    above Fmax, an infinite amax gives s = 0, and a NaN (also inf * 0)
 *    encodes to a NaN code (e4m3fn 0x7F or 0xFF, e4m3fnuz 0x80).
 *  - Offsets ([AIR] introduction, second paragraph: an offsets tensor routes
 *    tokens to experts): int32[num_groups] of CUMULATIVE group ends, no
 *    leading zero, device memory.  Group e spans rows [start_e, end_e) with
 *    start_0 = 0, start_e = end_{e-1}, end_e = clamp(offsets[e], start_e,
 *    rows_total).  Malformed offsets (decreasing, negative, beyond rows_total)
 *    are clamped that way on the device, so no access leaves the buffers, and
 *    FP8QGG_STATUS_BAD_OFFSETS is OR-ed into *dev_status when it is given.
 *    Rows past the last end belong to no group and are not written.
 *  - sat_count (nullable, device uint64): the kernel ADDS the number of
 *    elements whose pre-clamp |y| is more than one fp32 ulp above the
 *    encoding's largest finite value.  Zero it before the call.
 *  - dev_status (nullable, device int32): the kernel ORs FP8QGG_STATUS_* bits.
 *    Zero it before the call; read it after the stream has synchronised.
 *  - Return value: FP8QGG_OK or one of the negative FP8QGG_ERR_* codes below.
 *    Argument errors are detected on the host before anything is enqueued.
 */
#ifndef FP8QGG_H
#define FP8QGG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* return codes */
#define FP8QGG_OK 0
#define FP8QGG_ERR_NULL (-1)        /* a required pointer is NULL */
#define FP8QGG_ERR_SHAPE (-2)       /* bad size, leading dimension or group count */
#define FP8QGG_ERR_ALIGN (-3)       /* base pointer or leading dimension misaligned */
#define FP8QGG_ERR_UNSUPPORTED (-4) /* bad flag or unsupported combination */
#define FP8QGG_ERR_CUDA (-5)        /* a CUDA runtime/driver call failed */

/* formats */
#define FP8QGG_E4M3FN 0
#define FP8QGG_E4M3FNUZ 1

/* output layouts of the jagged column-wise quantisation */
#define FP8QGG_LAYOUT_SAME 0
#define FP8QGG_LAYOUT_TRANSPOSED 1
#define FP8QGG_LAYOUT_TRANSPOSED_PADDED 2 /* transposed, groups at 128-token boundaries */

/* grouped GEMM modes */
#define FP8QGG_M_JAGGED 0 /* groups split the rows of A and of the output */
#define FP8QGG_K_JAGGED 1 /* groups split the contraction axis */
#define FP8QGG_K_JAGGED_PADDED 2 /* the same, on FP8QGG_LAYOUT_TRANSPOSED_PADDED operands */

/* grouped GEMM output types */
#define FP8QGG_OUT_F32 0
#define FP8QGG_OUT_BF16 1

/* bits OR-ed into *dev_status */
#define FP8QGG_STATUS_BAD_OFFSETS 1  /* offsets had to be clamped */
#define FP8QGG_STATUS_TIMEOUT 2      /* a bounded device-side wait gave up */

/* The FP8 variant this device's tensor cores consume.  The pages add
 * automatic detection of the format because the wrong maximum corrupts
 * results silently ([AIR] "La correttezza del formato viene prima del
 * tuning"); on sm_100 the answer is always FP8QGG_E4M3FN. */
int fp8_native_format(void);

/* Short English text for a return code. */
const char *fp8qgg_error_string(int code);

/*
 * Encode step alone: q[i] = e4m3(y[i]), round to nearest, ties to even, one
 * rounding from fp32, saturating at the format's largest finite magnitude
 * (no scaling, no clamp).  It is the cast at the end of the chain of [AIR]
 * "Il guadagno vero è nel movimento dei dati", exposed for callers that bring
 * their own scales and for exhaustive checks of the device encoder.  NaN
 * inputs give unspecified codes.
 *   y fp32 [n] (4-byte aligned), q uint8 [n]; n >= 0 (0 is a no-op).
 */
int fp8_cast_f32(const float *y, int64_t n, uint8_t *q, int fmt, void *stream);

/*
 * Rowwise quantisation: one scale per row ([AIR] introduction: activations
 * take one scale per row).  Also the per-output-channel scale of a weight
 * stored [N, K] (rows = output channels).
 *   x      bf16 [rows, ld_x], row-major, read only.
 *   q      uint8 e4m3 codes [rows, ld_q], written for columns [0, cols).
 *   scales fp32 [rows], written.
 * Requirements: rows >= 0; cols in [1, 32768] and a multiple of 8;
 * ld_x >= cols and ld_x % 8 == 0; ld_q >= cols and ld_q % 8 == 0;
 * x and q 16-byte aligned, scales 4-byte aligned.  rows == 0 is a no-op.
 */
int fp8_quant_rowwise(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                      uint8_t *q, int64_t ld_q, float *scales,
                      int fmt, float scale_max, uint64_t *sat_count, void *stream);

/*
 * Bytes of device workspace fp8_quant_colwise_jagged needs, for every layout:
 * the larger of (a) the plain layouts' kernel: a task counter (256 bytes),
 * plus, for every (group, 64-column) unit that may be taller than 448 rows,
 * an arrival counter and 64 absmax words (at most min(num_groups,
 * rows_total / 432) groups can be that tall), and (b) the padded layout's
 * kernel: a task counter, one arrival counter per (group, 256-column panel)
 * and one absmax word per (group, column).  Always > 0 and a multiple of 256.
 */
size_t fp8_quant_colwise_jagged_workspace_size(int64_t rows_total, int64_t cols,
                                               int32_t num_groups);

/*
 * Jagged column-wise quantisation: for every expert group e and column c the
 * absmax runs over the group's rows only, giving one scale per (e, c)
 * ([AIR] introduction: one scale per column of each expert's weights; the
 * backward applies the same per-group column scaling to gradients,
 * [AIR] "Il guadagno vero è nel movimento dei dati", second paragraph).
 *   x        bf16 [rows_total, ld_x], row-major, read once from HBM.
 *   offsets  int32 [num_groups] cumulative group ends (device).
 *   layout   FP8QGG_LAYOUT_SAME:       q[r * ld_q + c], ld_q >= cols, ld_q % 8 == 0.
 *            FP8QGG_LAYOUT_TRANSPOSED: q[c * ld_q + r], ld_q >= rows_total,
 *            ld_q % 16 == 0.  Group e occupies columns [start_e, end_e) of
 *            every output row: the contraction axis of the weight-gradient
 *            GEMM comes out contiguous, with no separate transposed copy
 *            (the pages remove a .t().contiguous().t() round trip).
 *            FP8QGG_LAYOUT_TRANSPOSED_PADDED: as TRANSPOSED, but group e
 *            starts at column P_e = sum_{j<e} round_up(size_j, 128) of every
 *            output row and is followed by zero codes up to P_e +
 *            round_up(size_e, 128): the weight-gradient GEMM then meets no
 *            group edge inside a 128-token block (mode
 *            FP8QGG_K_JAGGED_PADDED).  ld_q >= rows_total + 128 * num_groups,
 *            ld_q % 16 == 0; columns past the last padded group are not
 *            written.  The codes of each 128-token block (zeros past the
 *            group's end included) leave the chip as one bulk tensor store.
 *            This layout is this library's choice: the pages do not
 *            describe one.
 *   scales   fp32 [num_groups, cols]; an empty group gets Fmax / 1e-12 in
 *            every column and no codes.
 *   workspace, workspace_bytes: device scratch of at least
 *            fp8_quant_colwise_jagged_workspace_size(...) bytes, 16-byte
 *            aligned, owned by the caller; its contents on entry do not
 *            matter (the call clears what it uses, on `stream`).  Calls that
 *            share one workspace must be ordered on the device.
 * Requirements: rows_total >= 0; cols in [1, 2^31) and a multiple of 8;
 * num_groups in [1, 1024]; ld_x >= cols, ld_x % 8 == 0; x, q and workspace
 * 16-byte aligned.  Groups of any height are handled: up to 448 rows a
 * (group, 64-column) block of x is read from HBM once and stays on chip for
 * the cast; a taller block is cut into chunks of at most 448 rows spread over
 * the SMs, whose absmax merge in the workspace, and each chunk is read a
 * second time for the cast, while it is still in L2.
 */
int fp8_quant_colwise_jagged(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                             const int32_t *offsets, int32_t num_groups,
                             uint8_t *q, int64_t ld_q, int layout, float *scales,
                             int fmt, float scale_max, uint64_t *sat_count,
                             int32_t *dev_status, void *workspace, size_t workspace_bytes,
                             void *stream);

/*
 * Bytes of device workspace fp8_quant_dual_jagged needs: a task counter (256
 * bytes), one arrival counter per group, the column absmax words
 * [num_groups, cols] and one row absmax word per row, each part rounded up to
 * 256 bytes.
 */
size_t fp8_quant_dual_jagged_workspace_size(int64_t rows_total, int64_t cols,
                                            int32_t num_groups);

/*
 * Dual-output quantisation for the backward pass: ONE read of x gives both
 * FP8 copies the two backward GEMMs of an expert layer need ([AIR] "Il
 * guadagno vero è nel movimento dei dati", second paragraph: the backward's
 * scale-and-cast fused and its transposed copy removed; [ABP] second
 * paragraph):
 *  - the rowwise quantisation (one scale per row) of every row of the groups,
 *    for the input-gradient GEMM (token-jagged, FP8QGG_M_JAGGED);
 *  - the jagged column-wise quantisation in FP8QGG_LAYOUT_TRANSPOSED_PADDED
 *    (one scale per (group, column)), for the weight-gradient GEMM
 *    (FP8QGG_K_JAGGED_PADDED).
 * The codes and scales are those of fp8_quant_rowwise on each row of a group
 * and of fp8_quant_colwise_jagged with the padded layout, bit for bit.
 *   x          bf16 [rows_total, ld_x], read once from HBM (each 128-row
 *              block is read a second time for the casts, from L2).
 *   offsets    int32 [num_groups] cumulative group ends (device).
 *   q_row      uint8 [rows_total, ld_qr]: columns [0, cols) of every row of
 *              a group; rows past the last group end are not written.
 *   scales_row fp32 [rows_total], written for the rows of the groups.
 *   q_col      uint8 [cols, ld_qc] in the padded transposed layout,
 *              ld_qc >= rows_total + 128 * num_groups, ld_qc % 16 == 0.
 *   scales_col fp32 [num_groups, cols]; an empty group gets Fmax / 1e-12.
 *   sat_count  (nullable) adds the saturated elements of both quantisations.
 *   workspace  at least fp8_quant_dual_jagged_workspace_size(...) bytes,
 *              16-byte aligned, cleared by the call on `stream`; calls that
 *              share one workspace must be ordered on the device.
 * Requirements: those of fp8_quant_colwise_jagged with the padded layout,
 * plus ld_qr >= cols, ld_qr % 8 == 0, q_row 16-byte aligned, scales_row
 * 4-byte aligned.
 */
int fp8_quant_dual_jagged(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                          const int32_t *offsets, int32_t num_groups,
                          uint8_t *q_row, int64_t ld_qr, float *scales_row,
                          uint8_t *q_col, int64_t ld_qc, float *scales_col,
                          int fmt, float scale_max, uint64_t *sat_count, int32_t *dev_status,
                          void *workspace, size_t workspace_bytes, void *stream);

/*
 * Same computation as fp8_quant_colwise_jagged, for callers that cannot
 * allocate device memory or supply a workspace (for example a runtime that
 * fixes its memory budget at start-up and forbids cudaMalloc later, or a
 * plugin interface that passes tensors but no scratch buffer).  The pages
 * have no counterpart to this entry point; it exists only for such callers.
 *
 * It calls no cudaMalloc/cudaFree and no allocating routine.  Its scratch is a
 * fixed device array of FP8QGG_NOALLOC_SCRATCH_BYTES inside the library, held
 * by every GPU that loads the library until the process exits.
 *  - Size limit: problems whose fp8_quant_colwise_jagged_workspace_size(...)
 *    exceeds FP8QGG_NOALLOC_SCRATCH_BYTES are rejected with FP8QGG_ERR_SHAPE
 *    before anything is enqueued.  2 MiB covers, for instance, 64 groups of
 *    a 98304 x 2048 tensor (532,736 bytes) or 256 groups of a 131072 x 1408
 *    tensor (1,464,576 bytes); it does not cover 64 groups of a 98304 x 8192
 *    tensor (2,130,176 bytes).
 *  - Set-up: the first call on each device looks up the array's device
 *    address with that device current (cudaGetSymbolAddress) and keeps it
 *    with the device's current context.  Make that first call before any
 *    stream capture on the device.  A later call made under another context
 *    (for instance after cudaDeviceReset, which unloads the library's device
 *    code with the old context) looks the address up again.
 *  - Errors: FP8QGG_ERR_CUDA when the current device ordinal is 64 or above
 *    (the set-up keeps one address per device for ordinals 0..63), when the
 *    address lookup fails, or when the clearing memset or the launch fails.
 *  - Sharing: every call uses the same array and clears the part it needs on
 *    `stream` first.  Calls on one device whose executions could overlap on
 *    the GPU race; order them (one stream, or events).
 * Arguments, layouts, requirements and errors are otherwise those of
 * fp8_quant_colwise_jagged without the workspace pair.
 */
#define FP8QGG_NOALLOC_SCRATCH_BYTES (2u * 1024u * 1024u)
int fp8_quant_colwise_jagged_noalloc(const void *x, int64_t rows_total, int64_t cols,
                                     int64_t ld_x, const int32_t *offsets, int32_t num_groups,
                                     uint8_t *q, int64_t ld_q, int layout, float *scales,
                                     int fmt, float scale_max, uint64_t *sat_count,
                                     int32_t *dev_status, void *stream);

/*
 * Test hook of the failure detection, not for production use.  Every device
 * wait of the library gives up after a time limit and ORs
 * FP8QGG_STATUS_TIMEOUT into *dev_status instead of spinning for ever.  This
 * call changes one of them, for the jagged column-wise calls that follow it in
 * the process: the wait of a tall unit's cast for the unit's merged absmax
 * also needs `extra_arrivals` chunk arrivals that never come, and gives up
 * after `limit_ns` nanoseconds (0 restores the normal limit of 2 s; at most
 * 2e9).  With extra_arrivals > 0 a call with a group taller than one chunk
 * therefore returns FP8QGG_OK, leaves FP8QGG_STATUS_TIMEOUT in *dev_status
 * and undefined codes and scales, and the device stays usable.  The waits for
 * copies in flight keep their normal limit.  (0, 0) restores normal calls.
 */
int fp8qgg_test_unit_wait(uint32_t extra_arrivals, uint64_t limit_ns);

/*
 * FP8 scaled grouped GEMM on the 5th-generation tensor cores (the pages run
 * the expert GEMMs as one grouped GEMM over FP8 operands: [ABP] third
 * paragraph; [PRI] "What Primus adds").  e4m3fn operands, fp32 accumulation.
 * Group boundaries are read from `offsets` ON THE DEVICE: no host
 * synchronisation on routing results.
 *
 * mode FP8QGG_M_JAGGED (forward, input gradient): rows of A and of the output
 * are split into groups; group e multiplies with its own B_e.
 *   out[m, n] = (sum_k A[m,k] * B_e[n,k]) / scale_a[m] / scale_b[e*sbs + n]
 *   a        e4m3 [m_total, ld_a]            (K contiguous)
 *   b        e4m3, B_e[n, k] at b[e*b_group_stride + n*ld_b + k]
 *   scale_a  fp32 [m_total]                  (scale_a_group_stride unused)
 *   scale_b  fp32, scale_b_group_stride (sbs) >= n
 *   out      [m_total, ld_out] of out_dtype; rows outside every group are
 *            not written (out_group_stride unused).
 * mode FP8QGG_K_JAGGED (weight gradient): the contraction axis (tokens) is
 * split into groups; one output matrix per group.
 *   out[e, i, j] = (sum_{t in group e} A[i,t] * B[j,t]) / scale_a[e*sas + i] / scale_b[e*sbs + j]
 *   a        e4m3 [n, ld_a], b e4m3 [k, ld_b]: the TRANSPOSED outputs of
 *            fp8_quant_colwise_jagged (tokens contiguous), m_total tokens.
 *   scale_a  fp32, group stride sas >= n;  scale_b fp32, group stride sbs >= k
 *   out      [num_groups, n, ld_out] with group stride out_group_stride
 *            (>= n * ld_out); an empty group's matrix is written as zeros.
 *   b_group_stride unused.
 * mode FP8QGG_K_JAGGED_PADDED: the same product on operands in
 * FP8QGG_LAYOUT_TRANSPOSED_PADDED (group e at tokens [P_e, P_e +
 * round_up(size_e, 128)), zeros past its size); m_total is the unpadded token
 * count, ld_a and ld_b >= m_total + 128 * num_groups.
 * Requirements: fmt == FP8QGG_E4M3FN (the tensor cores have no e4m3fnuz
 * input); m_total >= 0, n >= 1, k >= 1; num_groups in [1, 1024];
 * a, b 16-byte aligned; ld_a, ld_b, b_group_stride multiples of 16;
 * out 16-byte aligned; FP32 output needs n (M_JAGGED) or k (K_JAGGED) and
 * ld_out multiples of 4, BF16 output multiples of 8.  The call returns
 * FP8QGG_ERR_ALIGN or FP8QGG_ERR_SHAPE otherwise.
 */
int fp8_scaled_grouped_gemm(int mode,
                            const uint8_t *a, int64_t ld_a, const float *scale_a,
                            int64_t scale_a_group_stride,
                            const uint8_t *b, int64_t ld_b, int64_t b_group_stride,
                            const float *scale_b, int64_t scale_b_group_stride,
                            const int32_t *offsets, int32_t num_groups,
                            int64_t m_total, int64_t n, int64_t k,
                            void *out, int64_t ld_out, int64_t out_group_stride, int out_dtype,
                            int fmt, int32_t *dev_status, void *stream);

/* ------------------------------------------------------------------ MXFP8
 * Microscaled FP8: one scale per block of 32 consecutive elements along the
 * contraction axis ([PRI] "What Primus adds for MoE training on MI355X": MXFP8
 * grouped GEMM and quantisation kernels; [ABP] last paragraph; [AIR] section
 * "Cosa significa per chi gestisce cluster locali").  The pages do not define
 * the format; it is the OCP Microscaling (MX) v1.0 MXFP8 with e4m3fn
 * elements:
 *        amax = max |x| over the block        (NaN skipped)
 *        E    = floor(log2(amax)) - 8, clamped to [-127, 127]
 *               (amax = 0 gives -127, an infinite amax 127)
 *        scale byte (E8M0) = E + 127
 *        q    = e4m3fn(x / 2^E)  round to nearest even, saturating at 448
 *        value = decode(q) * 2^E
 * Scale layout (packed for the grouped GEMM): the contraction axis is cut
 * into groups of 128 elements (four blocks); one uint32 word per (group g,
 * row r) holds the four scale bytes, byte j = block 4g + j (bytes of blocks
 * past the end of the axis are 0), and the words of one group are
 * contiguous over the rows: scales[g * ld_sw + r].  Only e4m3fn exists in
 * this format.
 */

/*
 * MX quantisation along rows (activations; weights [E, N, K] viewed as
 * [E*N, K]): blocks of 32 consecutive columns.
 *   x       bf16 [rows, ld_x], 16-byte aligned, ld_x % 8 == 0.
 *   q       uint8 [rows, ld_q], 8-byte aligned, ld_q % 8 == 0.
 *   scales  uint32 [ceil(cols / 128), ld_sw], ld_sw >= rows, 4-byte aligned.
 * Requirements: cols >= 1, cols % 32 == 0 (FP8QGG_ERR_SHAPE otherwise).
 */
int fp8_mx_quant_rowwise(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                         uint8_t *q, int64_t ld_q, uint32_t *scales, int64_t ld_sw,
                         void *stream);

/*
 * MX quantisation along each expert group's tokens (the input and the output
 * gradient of the weight-gradient GEMM), written transposed in the padded
 * layout of FP8QGG_LAYOUT_TRANSPOSED_PADDED: token t of group e, column c goes
 * to q[c * ld_q + P_e + t], P_e = sum_{j<e} round_up(size_j, 128); the tokens
 * [size_e, round_up(size_e, 128)) of the group hold zero codes.  Blocks are
 * 32 consecutive tokens from the group's start (a group's last block may be
 * partial; its padding counts as zeros), so no block holds two groups.  The
 * scales follow the packed layout with the columns as rows and the padded
 * token axis as contraction axis: word (P_e / 128 + b, c) for the group's
 * 128-token groups b < round_up(size_e, 128) / 128 (padding-only blocks:
 * amax 0, byte 0).  Tokens past the last padded group are not written.
 *   x        bf16 [rows_total, ld_x], read once.
 *   offsets  int32 [num_groups] cumulative group ends (device).
 *   q        uint8 [cols, ld_q], ld_q >= rows_total + 128 * num_groups,
 *            ld_q % 16 == 0, 16-byte aligned.
 *   scales   uint32 [ld_q / 128, ld_sw], ld_sw >= cols, 4-byte aligned.
 * Requirements: cols % 8 == 0, ld_x % 8 == 0, x 16-byte aligned,
 * num_groups in [1, 1024].
 */
int fp8_mx_quant_colwise_padded(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                                const int32_t *offsets, int32_t num_groups,
                                uint8_t *q, int64_t ld_q, uint32_t *scales, int64_t ld_sw,
                                int32_t *dev_status, void *stream);

/*
 * Dual-output MX quantisation for the backward pass: ONE read of x gives the
 * MX rowwise quantisation of every row of the groups (blocks along the
 * columns, for the input-gradient GEMM) and the MX column-wise quantisation
 * in the padded transposed layout (blocks along each group's tokens, for the
 * weight-gradient GEMM): the codes and scale words of
 * fp8_mx_quant_rowwise on each grouped row and of
 * fp8_mx_quant_colwise_padded, bit for bit ([AIR] "Il guadagno vero è nel
 * movimento dei dati", second paragraph: the backward's quantisations fused;
 * [PRI] "What Primus adds…": MXFP8 kernels).  Rows past the last group end
 * are not written.
 *   q_row      uint8 [rows_total, ld_qr], ld_qr >= cols, ld_qr % 8 == 0,
 *              8-byte aligned.
 *   scales_row uint32 [cols / 128 rounded up, ld_swr], ld_swr >= rows_total.
 *   q_col, scales_col, ld_qc, ld_swc: as q, scales, ld_q, ld_sw of
 *              fp8_mx_quant_colwise_padded.
 * Requirements: those of fp8_mx_quant_colwise_padded, plus cols % 32 == 0.
 */
int fp8_mx_quant_dual_padded(const void *x, int64_t rows_total, int64_t cols, int64_t ld_x,
                             const int32_t *offsets, int32_t num_groups,
                             uint8_t *q_row, int64_t ld_qr, uint32_t *scales_row, int64_t ld_swr,
                             uint8_t *q_col, int64_t ld_qc, uint32_t *scales_col, int64_t ld_swc,
                             int32_t *dev_status, void *stream);

/*
 * MXFP8 grouped GEMM: block-scaled tensor-core products (each 32-element
 * block's partial sum times 2^(Ea + Eb)), fp32 accumulation.  Scales in the
 * packed layout above (ld_sa, ld_sb: words per 128-element group).
 * mode FP8QGG_M_JAGGED (forward, input gradient):
 *   out[m, n] = sum_k value_a[m, k] * value_b_e[n, k], e the group of row m
 *   a        e4m3 [m_total, ld_a]; scale_a word (g, m) at scale_a[g * ld_sa + m],
 *            ld_sa >= m_total
 *   b        B_e[n, k] at b[e*b_group_stride + n*ld_b + k]; scale_b word
 *            (g, e, n) at scale_b[g * ld_sb + e * scale_b_group_stride + n]
 *            (B quantised as one [E*N, K] matrix: scale_b_group_stride = n).
 *            The experts' matrices may be stacked (b_group_stride >= n*ld_b,
 *            ld_b >= k) or interleaved in the rows of one matrix (ld_b >=
 *            (E-1)*b_group_stride + k, b_group_stride >= k): the input
 *            gradient's B = W_e^T as fp8_mx_quant_colwise_padded writes it for
 *            W viewed [E*N, K] with groups of N rows (N % 128 == 0), where
 *            b_group_stride = N, ld_b = ld_q, and the scale words of expert e
 *            start at group e*N/128 (scale_b_group_stride = (N/128)*ld_sb).
 *            Their scale words: stacked (scale_b_group_stride >= n, ld_sb >=
 *            (E-1)*scale_b_group_stride + n) or in per-expert blocks (ld_sb >=
 *            n, scale_b_group_stride >= ceil(k/128) * ld_sb).
 *   out      [m_total, ld_out]; rows outside every group are not written.
 *   Requirements: k % 32 == 0; ld_sa >= m_total.
 * mode FP8QGG_K_JAGGED_PADDED (weight gradient, outputs of
 * fp8_mx_quant_colwise_padded):
 *   out[e, i, j] = sum_{t < size_e} value_a[i, P_e + t] * value_b[j, P_e + t]
 *   a        e4m3 [n, ld_a], scale_a words [.., ld_sa >= n];
 *   b        e4m3 [k, ld_b], scale_b words [.., ld_sb >= k];
 *            ld_a, ld_b >= m_total + 128 * num_groups (m_total: unpadded
 *            tokens).
 *   out      [num_groups, n, ld_out], group stride out_group_stride; an empty
 *            group's matrix is written as zeros.
 * (The plain K_JAGGED mode does not exist here: a 32-token block may not
 * hold two groups.)  Other requirements as fp8_scaled_grouped_gemm (a, b, out
 * 16-byte aligned; ld_a, ld_b, b_group_stride multiples of 16; output columns
 * and ld_out multiples of 4 (fp32) or 8 (bf16)); scale pointers 4-byte
 * aligned.  Returns FP8QGG_ERR_UNSUPPORTED for another mode or out_dtype.
 */
int fp8_mx_grouped_gemm(int mode,
                        const uint8_t *a, int64_t ld_a, const uint32_t *scale_a, int64_t ld_sa,
                        const uint8_t *b, int64_t ld_b, int64_t b_group_stride,
                        const uint32_t *scale_b, int64_t ld_sb, int64_t scale_b_group_stride,
                        const int32_t *offsets, int32_t num_groups,
                        int64_t m_total, int64_t n, int64_t k,
                        void *out, int64_t ld_out, int64_t out_group_stride, int out_dtype,
                        int32_t *dev_status, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* FP8QGG_H */
