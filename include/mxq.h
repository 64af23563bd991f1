/*
 * mxq.h -- C ABI of libmxq: block-scaled shared-exponent quantization on
 * NVIDIA B200 (sm_100a).
 *
 * A tensor of shape [rows, cols] (row-major, contiguous, cols % 32 == 0) is
 * cut into blocks of 32 consecutive values along the last dimension. Each
 * block gets one power-of-two scale 2^Es with
 *     Es = clamp(floor(log2(max_i |x_i|)) - emax, -127, 127)
 * stored as an E8M0 byte Es + 127, and every value is rounded to the element
 * format (round to nearest, ties to even, saturating at the largest finite
 * magnitude) and bit-packed.
 *   - "AXS-6: Adaptive eXponent Sharing", block figure: 8-bit shared exponent
 *     and 2-bit config once per 32 values, sign + 5-bit mantissa per value.
 *   - "Sonar: Online MXFP6", Start a model / Select the FP6 encoding: packed
 *     six-bit E2M3 or E3M2 data with an E8M0 scale per block of 32 values.
 *   - "EFQ-Softmax" explainer, Jargon and stage table: E2M1 (MXFP4) codes, an
 *     exponent-only block scale taken from the block's local maximum; the
 *     exp-then-quantize probability stage.
 *   - "eXmY" abstract: non-power-of-two widths packed densely, byte addressable.
 *
 * Element formats (emax = floor(log2 of the largest finite magnitude)):
 *   MXQ_AXS6        6 bits: sign + 5-bit magnitude m, value m/16;   emax 0, max 31/16
 *   MXQ_MXFP6_E2M3  6 bits: 1-2-3, bias 1;                           emax 2, max 7.5
 *   MXQ_MXFP6_E3M2  6 bits: 1-3-2, bias 3;                           emax 4, max 28
 *   MXQ_MXFP8_E4M3  8 bits: 1-4-3, bias 7, magnitude 0x7F is NaN;    emax 8, max 448
 *   MXQ_MXFP4_E2M1  4 bits: 1-2-1, bias 1;                           emax 2, max 6
 * Subnormals (exponent field 0) are value 2^(1-bias) * m / 2^M.
 *
 * Memory layouts (all row-major, all owned by the caller):
 *   values  [rows, cols] fp32 or bf16.
 *   codes   uint8[rows * cols/32 * P]: block b's payload occupies bytes
 *           [b*P, (b+1)*P), P = 24 (6-bit formats), 32 (E4M3), 16 (E2M1).
 *           Inside a payload, value j of the block is bits [w*j, w*j + w) of
 *           the little-endian bit string (bit k = bit k%8 of byte k/8).
 *   scales  uint8[rows * cols/32] E8M0 bytes (2^(byte-127); 0xFF = NaN block),
 *           or for AXS-6 uint16[rows * cols/32] headers: bits 0-7 the shared
 *           exponent byte, bits 8-9 the config field (written as 0, ignored on
 *           read), bits 10-15 zero.
 *
 * Special values: a block holding a NaN or an infinity gets scale 0xFF and
 * all-zero codes, and dequantizes to NaN. An all-zero block gets scale 0.
 * The code's sign bit is the input's sign bit (-0 stays -0). Any NaN that a
 * dequantize / fake-quantize writes is the canonical quiet NaN (fp32
 * 0x7FC00000, bf16 0x7FC0).
 *
 * Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 * stream) of the current device; the library never synchronizes, allocates
 * no memory and keeps no per-call state, so concurrent calls from several
 * host threads are safe. All pointers must be device (or managed) memory of
 * the current device. Argument errors are detected on the host before any
 * launch and return a status; nothing is written in that case. Launch
 * failures return MXQ_ERR_CUDA; faults during execution surface at the
 * caller's next synchronization, as with any CUDA kernel.
 */
#ifndef MXQ_H
#define MXQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MXQ_API __attribute__((visibility("default")))
#else
#define MXQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MXQ_AXS6 = 0,
    MXQ_MXFP6_E2M3 = 1,
    MXQ_MXFP6_E3M2 = 2,
    MXQ_MXFP8_E4M3 = 3,
    MXQ_MXFP4_E2M1 = 4
} mxq_format;

typedef enum { MXQ_F32 = 0, MXQ_BF16 = 1 } mxq_dtype;

typedef enum {
    MXQ_OK = 0,
    MXQ_ERR_INVALID_ARG = 1, /* bad enum, null / host / other-device pointer          */
    MXQ_ERR_SHAPE = 2,       /* rows < 0, cols <= 0, cols % 32 != 0, size overflow    */
    MXQ_ERR_ALIGN = 3,       /* a pointer misses its alignment (see each call)        */
    MXQ_ERR_UNSUPPORTED = 4, /* valid request the library does not implement         */
    MXQ_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed                  */
    MXQ_ERR_TIMEOUT = 6      /* a bounded device-side wait gave up (mxq_check_device) */
} mxq_status;

/* A cudaStream_t, passed as an opaque pointer so this header needs no CUDA headers. */
typedef void* mxq_stream;

/*
 * Quantize: values -> packed codes + scales.
 *   src     [rows, cols] values of type `dtype`, 16-byte aligned.
 *   codes   mxq_codes_bytes(fmt, rows, cols) bytes, 16-byte aligned.
 *   scales  mxq_scales_bytes(fmt, rows, cols) bytes (2-byte aligned for AXS-6).
 * rows == 0 is a valid no-op. src must not overlap codes or scales.
 * Source: the block rule above ("AXS-6" block figure; "Sonar: Online MXFP6",
 * Start a model; "EFQ-Softmax", stage table "Block scale").
 */
MXQ_API mxq_status mxq_quantize(mxq_format fmt, const void* src, mxq_dtype dtype, int64_t rows, int64_t cols,
                        void* codes, void* scales, mxq_stream stream);

/*
 * Dequantize: codes + scales -> values of type `dtype`
 *   value = decode(code) * 2^(scale byte - 127), rounded to nearest even into
 *   `dtype` (exact except for bf16 results below 2^-126 and overflow).
 *   codes   16-byte aligned; dst [rows, cols] 16-byte aligned; scales as above.
 * dst must not overlap codes or scales.
 */
MXQ_API mxq_status mxq_dequantize(mxq_format fmt, const void* codes, const void* scales, int64_t rows, int64_t cols,
                          void* dst, mxq_dtype dtype, mxq_stream stream);

/*
 * Fused fake-quantize: dst = dequantize(quantize(src)) in one pass, with no
 * codes written to memory ("AXS-6", Quick Start Example: fused fake quantize
 * with block_size=32, no intermediate allocation). dst has src's type and
 * shape; dst == src (in place) is allowed, any other overlap is not. Both
 * 16-byte aligned.
 */
MXQ_API mxq_status mxq_fake_quantize(mxq_format fmt, const void* src, mxq_dtype dtype, int64_t rows, int64_t cols,
                             void* dst, mxq_stream stream);

/*
 * Exp-then-quantize softmax probability stage ("EFQ-Softmax" explainer,
 * Jargon: shifted scores, exp-then-quantize; stage table: probability
 * generation, block scale). For every row r:
 *   m   = max_j scores[r, j]            (NaN if the row holds a NaN)
 *   p_j = expf_mxq(scores[r, j] - m)     (fp32 subtraction, then the library's
 *                                         own deterministic fp32 exponential:
 *                                         Cody-Waite reduction by ln 2 split in
 *                                         two constants, degree-7 Taylor
 *                                         polynomial in fused multiply-adds)
 *   then p is block-quantized exactly like mxq_quantize with dtype MXQ_F32.
 * p is never written to memory. Supported formats: all five (MXFP4 E2M1 is
 * the one the stage feeds). scores 16-byte aligned; any cols % 32 == 0.
 * Runs as a bulk-copy (TMA) pipeline whose waits are bounded; see
 * mxq_check_device.
 */
MXQ_API mxq_status mxq_exp_quantize(mxq_format fmt, const float* scores, int64_t rows, int64_t cols,
                            void* codes, void* scales, mxq_stream stream);

/*
 * Exp-free E2M1 probabilities ("EFQ-Softmax: exp-free E2M1 probabilities",
 * opening paragraph and the paragraph on the per-block rule): the shifted
 * scores go straight to nonnegative MXFP4 codes; no exponential is evaluated.
 * Per row r and block of 32 keys:
 *   u_j   = RN(RN(scores[r, j] - m) * L2E)   (m = row maximum as above,
 *                                             L2E = 1/ln 2 rounded to fp32:
 *                                             u_j = log2 of exp(s_j - m))
 *   Es    = clamp(floor(max_j u_j) - 2, -127, 127)   exponent-only block scale,
 *           stored as the E8M0 byte Es + 127
 *   code  = clamp(rint(RN(2 u_j - 2 Es)) + 2, 0, 7)  ties to even, sign bit 0
 * The page fixes the rule's structure (scale from the block's local maximum,
 * one affine rule per block) but not its constants; these are the straight
 * line through E2M1's grid in the log domain (codes 2, 4, 6 = 1, 2, 4 exactly).
 * A block holding a NaN stores 0xFF and codes 0. Output layout as
 * mxq_quantize(MXQ_MXFP4_E2M1): codes [rows, cols/32 * 16] bytes (key 2i in
 * the low nibble), scales [rows, cols/32] bytes; mxq_dequantize decodes them.
 * scores 16-byte aligned, cols % 32 == 0; other rules and errors as
 * mxq_exp_quantize. Runs on the bulk-copy pipeline of mxq_exp_quantize, whose
 * waits are bounded (see mxq_check_device).
 */
MXQ_API mxq_status mxq_exp_free_quantize(const float* scores, int64_t rows, int64_t cols, void* codes, void* scales,
                                         mxq_stream stream);

/*
 * Grouped quantize: n independent tensors of one format and one value type
 * converted by a single launch (a decoder layer's seven weight matrices in the
 * online layer-by-layer conversion of "Sonar: Online MXFP6", Start a model).
 * Each descriptor obeys the rules of mxq_quantize. 1 <= n <= MXQ_MAX_GROUP.
 * The descriptor array is read on the host during the call only.
 */
#define MXQ_MAX_GROUP 64
typedef struct {
    const void* src;
    void* codes;
    void* scales;
    int64_t rows;
    int64_t cols;
} mxq_tensor;

MXQ_API mxq_status mxq_quantize_grouped(mxq_format fmt, mxq_dtype dtype, const mxq_tensor* tensors, int n,
                                mxq_stream stream);

/*
 * Column-direction blocks: each block is 32 consecutive ROWS of one column of
 * src [rows, cols] (weights stored [in, out]; operands of a backward pass).
 * The output is exactly what mxq_quantize would produce for the transpose
 * src^T [cols, rows]: codes [cols, rows/32 * P] and scales [cols, rows/32],
 * so each column's blocks are contiguous. rows % 32 == 0 and cols % 32 == 0
 * (MXQ_ERR_SHAPE otherwise), rows <= 16776960. Alignment and overlap rules as
 * mxq_quantize. ("Sonar: Online MXFP6", Start a model: the blocks of 32 run
 * along the weight's input dimension.)
 */
MXQ_API mxq_status mxq_quantize_cols(mxq_format fmt, const void* src, mxq_dtype dtype, int64_t rows, int64_t cols,
                                     void* codes, void* scales, mxq_stream stream);
/* Inverse of mxq_quantize_cols: codes/scales in the transposed layout ->
 * dst [rows, cols] of type dtype (the values mxq_dequantize gives for the
 * transpose, transposed back). Same shape rules. */
MXQ_API mxq_status mxq_dequantize_cols(mxq_format fmt, const void* codes, const void* scales, int64_t rows,
                                       int64_t cols, void* dst, mxq_dtype dtype, mxq_stream stream);

/*
 * eXmY element formats ("eXmY" abstract: any bit width, any split of the bits
 * after the sign into exponent and mantissa, dense byte-addressable packing).
 * ebits E and mbits M with 0 <= E <= 5, M >= 1, 3 <= W = 1+E+M <= 9
 * (MXQ_ERR_UNSUPPORTED otherwise). Value of a code: sign, exponent field e,
 * mantissa m, bias b = 2^(E-1) - 1 (E >= 1) or 0 (E = 0):
 *   e > 0: 2^(e-b) (1 + m/2^M);  e = 0: 2^(1-b) m/2^M
 * (E = 0 is sign + fixed point m/2^(M-1)); no code is reserved for Inf/NaN.
 * Block rule as above with emax = 2^(E-1) (0 for E = 0). Layouts: codes
 * uint8[rows * cols/32 * 4W] (W-bit codes LSB-first, a block's payload is W
 * 32-bit words; the array 16-byte aligned), scales uint8[rows * cols/32] E8M0 bytes.
 * e2m1 / e2m3 / e3m2 give exactly MXFP4 / MXFP6 E2M3 / E3M2; e0m5 gives AXS-6's
 * codes (with a one-byte scale). Rounding is integer arithmetic on the fp32
 * bit patterns (no conversion instruction exists for arbitrary splits).
 */
MXQ_API mxq_status mxq_quantize_exmy(int ebits, int mbits, const void* src, mxq_dtype dtype, int64_t rows,
                                     int64_t cols, void* codes, void* scales, mxq_stream stream);
MXQ_API mxq_status mxq_dequantize_exmy(int ebits, int mbits, const void* codes, const void* scales, int64_t rows,
                                       int64_t cols, void* dst, mxq_dtype dtype, mxq_stream stream);
MXQ_API mxq_status mxq_fake_quantize_exmy(int ebits, int mbits, const void* src, mxq_dtype dtype, int64_t rows,
                                          int64_t cols, void* dst, mxq_stream stream);

/*
 * Batch: n independent conversions on one value type in a single launch, for
 * example the tensors of one layer going to the formats a per-module policy
 * chose ("Sonar: Online MXFP6", Start a model and Select the FP6 encoding), or
 * weights dequantized beside activations quantized. Results are bit-identical
 * to the single-operation entry points; the batch pays one launch instead of n.
 *   kind MXQ_OP_QUANTIZE:      src = values [rows, cols] (dtype), dst = codes,
 *                              dst_scales = scales (mxq_quantize's layouts)
 *   kind MXQ_OP_DEQUANTIZE:    src = codes, src_scales = scales, dst = values
 *   kind MXQ_OP_FAKE_QUANTIZE: src = values, dst = values (dst == src allowed)
 * Unused pointer fields are ignored. Each op obeys the shape, alignment and
 * overlap rules of its single-operation entry point. The ops run concurrently,
 * so no op may write memory that another op of the batch reads or writes
 * (MXQ_ERR_INVALID_ARG otherwise). 1 <= n <= MXQ_MAX_BATCH; ops with rows == 0
 * are skipped. The descriptor array is read on the host during the call only.
 */
typedef enum { MXQ_OP_QUANTIZE = 0, MXQ_OP_DEQUANTIZE = 1, MXQ_OP_FAKE_QUANTIZE = 2 } mxq_op_kind;
#define MXQ_MAX_BATCH 64
typedef struct {
    int kind;               /* mxq_op_kind */
    int fmt;                /* mxq_format */
    const void* src;
    const void* src_scales;
    void* dst;
    void* dst_scales;
    int64_t rows;
    int64_t cols;
} mxq_op;

MXQ_API mxq_status mxq_run_batch(mxq_dtype dtype, const mxq_op* ops, int n, mxq_stream stream);

/*
 * Scale layout of the block-scaled tensor-core MMA. Converted weights are
 * operands of block-scaled GEMMs ("Sonar: Online MXFP6", Current limits: dense
 * dimensions in multiples of 128). The pages do not spell out how those GEMMs
 * read the scales; this is the layout of the sm_100 block-scaled MMA and of
 * cuBLAS's block-scaled GEMMs ("1D block scaling factors layout"):
 *   the [rows, kb] E8M0 scale matrix of an operand [rows, K] (kb = K / 32) is
 *   padded with zero bytes to rows128 = ceil(rows/128)*128 rows and
 *   kb4 = ceil(kb/4)*4 columns and cut into 128 x 4 tiles of 512 bytes,
 *   stored tile-row by tile-row (tile (R, C) at byte (R * kb4/4 + C) * 512);
 *   inside a tile, row r and column c sit at byte (r % 32) * 16 + (r / 32) * 4 + c.
 * The codes of an MXFP8 E4M3 operand are then exactly a row-major
 * float8_e4m3fn [rows, K] matrix, those of MXFP4 a row-major packed
 * float4_e2m1 [rows, K/2] matrix (element 2i in the low nibble).
 */
/* Bytes of the tiled scale array of a [rows, cols] operand: rows128 * kb4
 * (0 on bad input: rows < 0, cols <= 0 or cols % 32 != 0). */
MXQ_API size_t mxq_mma_scales_bytes(int64_t rows, int64_t cols);
/* mxq_quantize with the scales written in the tiled layout above. Codes are
 * identical to mxq_quantize's. scales: device, mxq_mma_scales_bytes(rows, cols)
 * bytes, written in full: when rows % 128 or (cols/32) % 4 is nonzero the pad
 * bytes are zeroed by a cudaMemsetAsync on the same stream before the kernel.
 * E8M0 formats only: MXQ_AXS6 (whose header is 16 bits) -> MXQ_ERR_UNSUPPORTED.
 * Other rules, errors and overlap checks as mxq_quantize. */
MXQ_API mxq_status mxq_quantize_mma(mxq_format fmt, const void* src, mxq_dtype dtype, int64_t rows, int64_t cols,
                                    void* codes, void* scales, mxq_stream stream);
/* Rearrange a plain scale array (uint8 [rows, kblocks], as written by
 * mxq_quantize, mxq_exp_quantize or mxq_quantize_cols for its transposed
 * operand) into the tiled layout. out: device, 4-byte aligned,
 * mxq_mma_scales_bytes(rows, 32 * kblocks) bytes, all written (pad = 0); it
 * may not overlap scales. rows == 0 is a no-op; rows < 0, kblocks <= 0 or
 * kblocks > 67108860 (4 * (2^31 - 1) / 128: one tile-row's output words are
 * counted in 32 bits) -> MXQ_ERR_SHAPE. */
MXQ_API mxq_status mxq_swizzle_scales(const void* scales, int64_t rows, int64_t kblocks, void* out,
                                      mxq_stream stream);

/*
 * Device-side status. The kernels that move data with the bulk-copy (TMA)
 * engine wait on their own asynchronous copies: mxq_exp_quantize and
 * mxq_exp_free_quantize (every format and size), mxq_quantize_cols, and
 * mxq_fake_quantize on tensors of 2^19 blocks or more. Every such wait is
 * bounded (one second). A wait that runs out makes the kernel stop early,
 * leaving its outputs incomplete, and sets a device error word. The outputs of
 * any call of these entry points are therefore undefined until a later
 * mxq_check_device returns MXQ_OK: the call itself returns MXQ_OK when its
 * launch succeeded, before the kernel has run. mxq_check_device synchronizes
 * the current device and returns MXQ_ERR_TIMEOUT if a wait ran out since the
 * last call (clearing the word), MXQ_ERR_CUDA if the device reported an error,
 * MXQ_OK otherwise. It is host-blocking; call it where a synchronization is
 * acceptable (after a step, in tests). There is one word per device, shared by
 * every stream and host thread using that device: a check by one thread
 * reports (and clears) a timeout of a kernel another thread launched.
 */
MXQ_API mxq_status mxq_check_device(void);
/* Self-test of that mechanism: first runs mxq_check_device() and returns its
 * status, without testing, if it is not MXQ_OK (a pending timeout of an
 * earlier call is reported, not cleared away); then launches one warp that
 * waits on an mbarrier nothing arrives at, with a limit of limit_ms
 * milliseconds (1..1000), and returns mxq_check_device(): MXQ_ERR_TIMEOUT when
 * the wait gave up and was reported as it should. Synchronizes the device.
 * MXQ_ERR_INVALID_ARG for a limit out of range. No counterpart on the pages: a
 * diagnostic of the library. */
MXQ_API mxq_status mxq_selftest_timeout(int limit_ms);

/* Bytes of the packed code array: rows * cols/32 * payload (0 on bad input). */
MXQ_API size_t mxq_codes_bytes(mxq_format fmt, int64_t rows, int64_t cols);
/* Bytes of the scale array: rows * cols/32 (x2 for AXS-6 headers; 0 on bad input). */
MXQ_API size_t mxq_scales_bytes(mxq_format fmt, int64_t rows, int64_t cols);
/* Information bits per block: 8 scale bits + 32 * element bits, plus the
 * 2-bit config field for AXS-6 -> 202, 200, 200, 264, 136; -1 on bad input. */
MXQ_API int mxq_block_bits(mxq_format fmt);
/* Static, human-readable description of a status code. */
MXQ_API const char* mxq_status_string(mxq_status status);
/* Library version, "major.minor.patch". */
MXQ_API const char* mxq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MXQ_H */
