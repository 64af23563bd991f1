/*
 * oracle.c -- plain, slow, scalar CPU oracle for block-scaled shared-exponent
 * quantization (AXS-6, MXFP6 E2M3 / E3M2, MXFP8 E4M3, MXFP4 E2M1).
 *
 * TEST INFRASTRUCTURE. Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference leg of bench.py may load this library. The
 * product path (libmxq) never calls it and shares no code with it: no
 * header, table, constant generator or helper is common to the two.
 *
 * Every intermediate of the method is computed in IEEE double, where it is
 * exact: inputs are fp32/bf16, scales are powers of two in [2^-127, 2^127]
 * and grid quotients are below 2^10.  The one step done in fp32 on purpose is
 * the exponential of the exp-then-quantize softmax stage, because the method
 * fixes that stage's precision at fp32 and the produced codes depend on it.
 *
 * Sources (page title, then section / figure):
 *  [AXS]   "AXS-6: Adaptive eXponent Sharing" -- block figure (8-bit shared
 *          exponent + 2-bit config once per 32 values, sign + 5-bit mantissa
 *          per value), quick-start example (block_size=32, fused fake quantize).
 *  [EFQ]   "EFQ-Softmax: exp-free E2M1 probabilities" -- Jargon (E2M1 = 1 sign,
 *          2 exponent, 1 mantissa bit; MXFP4; microscaling block; shifted
 *          scores; exp-then-quantize), the stage table (block scale is
 *          exponent-only, taken from the block's local maximum).
 *  [SONAR] "Sonar: Online MXFP6" -- Start a model (packed six-bit data and an
 *          E8M0 scale for each block of 32 values, one layer at a time),
 *          Select the FP6 encoding (E2M3 more mantissa, E3M2 larger range).
 *  [EXMY]  "eXmY: A Data Type and Technique for Arbitrary Bit Precision
 *          Quantization" -- abstract (non-power-of-two widths packed densely,
 *          byte addressable).
 *
 * Readings where the pages are silent (each one is also listed in the
 * design notes of the repository):
 *  - element formats: the OCP MX closed forms. value = (-1)^s 2^(e-b)(1+m/2^M)
 *    for e>0, (-1)^s 2^(1-b) m/2^M for e=0; E4M3 has one NaN magnitude (0x7F)
 *    and no infinities; E2M1/E2M3/E3M2 have neither.
 *  - AXS-6 element: sign + 5-bit magnitude m read as the fixed-point value
 *    m/16 (so emax = 0 and the block maximum lands in [1, 2)).
 *  - shared scale: Es = clamp(floor(log2 amax) - emax, -127, 127), stored as
 *    the E8M0 byte Es + 127; an all-zero block stores byte 0; a block holding
 *    a NaN or an infinity stores 0xFF, all codes 0, and decodes to NaN.
 *  - rounding: round to nearest, ties to the even magnitude code, then
 *    saturate to the largest finite magnitude.
 *  - sign: the code's sign bit is the input's sign bit (so -0 stays -0).
 *  - packing: LSB-first bit string per block, value j at bits [w j, w j + w).
 *  - AXS-6 header: uint16, bits 0-7 exponent byte, bits 8-9 config = 0.
 *  - output rounding of dequantized values: round to nearest even into the
 *    output type (fp32 / bf16), overflow to infinity; any NaN output is the
 *    canonical quiet NaN (fp32 0x7FC00000, bf16 0x7FC0).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

/* format ids of this oracle (its own numbering; callers map by name) */
enum { ORC_AXS6 = 0, ORC_E2M3 = 1, ORC_E3M2 = 2, ORC_E4M3 = 3, ORC_E2M1 = 4, ORC_NFMT = 5 };
/* value types */
enum { ORC_F32 = 0, ORC_BF16 = 1 };

typedef struct {
    int bits;    /* code width w                                   */
    int mbits;   /* mantissa bits M (AXS-6: 5 bits of magnitude)   */
    int bias;    /* exponent bias b (unused for AXS-6)             */
    int emax;    /* floor(log2(largest finite magnitude))          */
    int fixed;   /* 1: magnitude is the fixed-point value m/16     */
    int nan_mag; /* magnitude code that means NaN, or -1          */
} fmt_t;

static const fmt_t FMT[ORC_NFMT] = {
    /* AXS6 */ {6, 5, 0, 0, 1, -1},
    /* E2M3 */ {6, 3, 1, 2, 0, -1},
    /* E3M2 */ {6, 2, 3, 4, 0, -1},
    /* E4M3 */ {8, 3, 7, 8, 0, 0x7F},
    /* E2M1 */ {4, 1, 1, 2, 0, -1},
};

static int fmt_ok(int f) { return f >= 0 && f < ORC_NFMT; }

static uint32_t sign_mask(const fmt_t* F) { return 1u << (F->bits - 1); }

/* Largest finite magnitude code: all ones below the sign, minus the NaN code. */
static uint32_t max_mag(const fmt_t* F) {
    uint32_t m = sign_mask(F) - 1u;
    if ((int)m == F->nan_mag) m -= 1u;
    return m;
}

/* Value of a code, from the closed forms above. */
static double decode_f(const fmt_t* F, uint32_t code) {
    uint32_t s = code & sign_mask(F);
    uint32_t mag = code & (sign_mask(F) - 1u);
    double v;
    if (F->fixed) {
        v = (double)mag / 16.0;
    } else if ((int)mag == F->nan_mag) {
        return NAN;
    } else {
        uint32_t e = mag >> F->mbits;
        uint32_t m = mag & ((1u << F->mbits) - 1u);
        if (e == 0)
            v = ldexp((double)m, 1 - F->bias - F->mbits);
        else
            v = ldexp((double)((1u << F->mbits) + m), (int)e - F->bias - F->mbits);
    }
    return s ? -v : v;
}

double orc_decode(int f, uint32_t code) { return fmt_ok(f) ? decode_f(&FMT[f], code) : NAN; }

int orc_bits(int f) { return fmt_ok(f) ? FMT[f].bits : -1; }
int orc_emax(int f) { return fmt_ok(f) ? FMT[f].emax : -1; }
double orc_maxval(int f) { return fmt_ok(f) ? decode_f(&FMT[f], max_mag(&FMT[f])) : NAN; }

/* Round a finite y >= 0 (already divided by the block scale) to the nearest
 * grid magnitude, ties to the even code, saturating at the largest magnitude. */
static uint32_t round_mag_f(const fmt_t* F, double y) {
    if (y >= decode_f(F, max_mag(F))) return max_mag(F);
    if (F->fixed) return (uint32_t)nearbyint(y * 16.0); /* 16y < 31 here */
    if (y == 0.0) return 0u;
    int e2;
    frexp(y, &e2);                 /* y = fr * 2^e2, fr in [0.5, 1) */
    int ey = e2 - 1;               /* floor(log2 y)                 */
    int emin = 1 - F->bias;        /* smallest normal exponent      */
    if (ey < emin) ey = emin;      /* subnormal range: fixed step   */
    double q = ldexp(1.0, ey - F->mbits);     /* grid step in y's binade */
    double n = nearbyint(y / q);              /* y/q exact; ties to even */
    uint32_t M = 1u << F->mbits;
    if (n == (double)(2u * M)) { ey += 1; n = (double)M; }   /* carried into next binade */
    if (n < (double)M) return (uint32_t)n;                   /* subnormal: e = 0, m = n  */
    return ((uint32_t)(ey + F->bias) << F->mbits) | ((uint32_t)n - M);
}

uint32_t orc_round_mag(int f, double y) { return round_mag_f(&FMT[f], y); }

/* orc_round_mag over an array (test harness convenience). */
void orc_round_mags(int f, const double* y, int64_t n, uint32_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = orc_round_mag(f, y[i]);
}

/* Shared-scale exponent Es for a block; returns 0xFF (NaN block) or Es + 127. */
static int block_scale_byte(const fmt_t* F, const double* x, int n) {
    double amax = 0.0;
    for (int i = 0; i < n; ++i) {
        if (isnan(x[i]) || isinf(x[i])) return 0xFF;
        if (fabs(x[i]) > amax) amax = fabs(x[i]);
    }
    int Es;
    if (amax == 0.0) {
        Es = -127;
    } else {
        int e2;
        frexp(amax, &e2);
        Es = (e2 - 1) - F->emax;   /* floor(log2 amax) - emax */
        if (Es < -127) Es = -127;
        if (Es > 127) Es = 127;
    }
    return Es + 127;
}

/* O1 for one block of 32 values: codes[i] (unpacked) and the scale byte. */
static int quantize_block_f(const fmt_t* F, const double* x, uint32_t* codes) {
    int byte = block_scale_byte(F, x, 32);
    if (byte == 0xFF) {
        for (int i = 0; i < 32; ++i) codes[i] = 0u;
        return byte;
    }
    int Es = byte - 127;
    for (int i = 0; i < 32; ++i) {
        double y = ldexp(fabs(x[i]), -Es);            /* exact power-of-two scaling */
        uint32_t mag = round_mag_f(F, y);
        codes[i] = (signbit(x[i]) ? sign_mask(F) : 0u) | mag;
    }
    return byte;
}

int orc_quantize_block(int f, const double* x, uint32_t* codes) { return quantize_block_f(&FMT[f], x, codes); }

/* ---- value types ------------------------------------------------------- */

static double load_value(const void* src, int dtype, int64_t i) {
    if (dtype == ORC_F32) {
        float v;
        memcpy(&v, (const char*)src + 4 * i, 4);
        return (double)v;
    }
    uint16_t h;
    memcpy(&h, (const char*)src + 2 * i, 2);
    uint32_t u = (uint32_t)h << 16;     /* bf16 is the top half of an fp32 */
    float v;
    memcpy(&v, &u, 4);
    return (double)v;
}

/* Round v to a binary float with p significant bits, smallest normal
 * exponent emin and largest exponent emax: nearest, ties to even, overflow
 * to infinity, gradual underflow. */
double orc_round_binary(double v, int p, int emin, int emax) {
    if (isnan(v) || isinf(v) || v == 0.0) return v;
    int e2;
    frexp(fabs(v), &e2);
    int ev = e2 - 1;
    if (ev < emin) ev = emin;
    double q = ldexp(1.0, ev - (p - 1));
    double r = nearbyint(v / q) * q;
    if (fabs(r) >= ldexp(1.0, emax + 1)) return copysign(INFINITY, v);
    return r;
}

static void store_value(void* dst, int dtype, int64_t i, double v) {
    if (dtype == ORC_F32) {
        uint32_t u;
        if (isnan(v)) {
            u = 0x7FC00000u;
        } else {
            float fv = (float)orc_round_binary(v, 24, -126, 127); /* exact now */
            memcpy(&u, &fv, 4);
        }
        memcpy((char*)dst + 4 * i, &u, 4);
    } else {
        uint16_t h;
        if (isnan(v)) {
            h = 0x7FC0u;
        } else {
            float fv = (float)orc_round_binary(v, 8, -126, 127); /* representable in bf16 */
            uint32_t u;
            memcpy(&u, &fv, 4);
            h = (uint16_t)(u >> 16);
        }
        memcpy((char*)dst + 2 * i, &h, 2);
    }
}

/* ---- packing ----------------------------------------------------------- */

static int payload_bytes(const fmt_t* F) { return 32 * F->bits / 8; }

/* value j of a block occupies bits [w j, w j + w) of the block's payload,
 * bit k of the payload being bit (k % 8) of byte k / 8. */
static void pack_block(const fmt_t* F, const uint32_t* codes, uint8_t* out) {
    int w = F->bits;
    memset(out, 0, (size_t)payload_bytes(F));
    for (int j = 0; j < 32; ++j)
        for (int t = 0; t < w; ++t)
            if ((codes[j] >> t) & 1u) {
                int k = w * j + t;
                out[k / 8] |= (uint8_t)(1u << (k % 8));
            }
}

static void unpack_block(const fmt_t* F, const uint8_t* in, uint32_t* codes) {
    int w = F->bits;
    for (int j = 0; j < 32; ++j) {
        uint32_t c = 0;
        for (int t = 0; t < w; ++t) {
            int k = w * j + t;
            if ((in[k / 8] >> (k % 8)) & 1u) c |= 1u << t;
        }
        codes[j] = c;
    }
}

static void store_scale(const fmt_t* F, void* scales, int64_t b, int byte) {
    if (F->fixed) {
        uint16_t h = (uint16_t)byte;  /* config field (bits 8-9) = 0 */
        memcpy((char*)scales + 2 * b, &h, 2);
    } else {
        ((uint8_t*)scales)[b] = (uint8_t)byte;
    }
}

static int load_scale(const fmt_t* F, const void* scales, int64_t b) {
    if (F->fixed) {
        uint16_t h;
        memcpy(&h, (const char*)scales + 2 * b, 2);
        return h & 0xFF;             /* config bits are not read */
    }
    return ((const uint8_t*)scales)[b];
}

/* ---- whole-tensor entry points ---------------------------------------- */
/* Tensors are [rows, cols] row-major with cols % 32 == 0, so the blocks are
 * the consecutive 32-value groups of the flat array. Return 0 on success. */

static int check(int f, int dtype, int64_t rows, int64_t cols) {
    if (!fmt_ok(f) || (dtype != ORC_F32 && dtype != ORC_BF16)) return 1;
    if (rows < 0 || cols <= 0 || cols % 32 != 0) return 2;
    return 0;
}

static void quantize_f(const fmt_t* F, const void* src, int dtype, int64_t nb, uint8_t* codes, void* scales) {
    double x[32];
    uint32_t c[32];
    for (int64_t b = 0; b < nb; ++b) {
        for (int i = 0; i < 32; ++i) x[i] = load_value(src, dtype, 32 * b + i);
        int byte = quantize_block_f(F, x, c);
        pack_block(F, c, codes + b * payload_bytes(F));
        store_scale(F, scales, b, byte);
    }
}

static void dequantize_f(const fmt_t* F, const uint8_t* codes, const void* scales, int64_t nb, void* dst, int dtype) {
    uint32_t c[32];
    for (int64_t b = 0; b < nb; ++b) {
        unpack_block(F, codes + b * payload_bytes(F), c);
        int byte = load_scale(F, scales, b);
        for (int i = 0; i < 32; ++i) {
            double v = (byte == 0xFF) ? NAN : ldexp(decode_f(F, c[i]), byte - 127);
            store_value(dst, dtype, 32 * b + i, v);
        }
    }
}

static void fake_quantize_f(const fmt_t* F, const void* src, int dtype, int64_t nb, void* dst) {
    double x[32];
    uint32_t c[32];
    for (int64_t b = 0; b < nb; ++b) {
        for (int i = 0; i < 32; ++i) x[i] = load_value(src, dtype, 32 * b + i);
        int byte = quantize_block_f(F, x, c);
        for (int i = 0; i < 32; ++i) {
            double v = (byte == 0xFF) ? NAN : ldexp(decode_f(F, c[i]), byte - 127);
            store_value(dst, dtype, 32 * b + i, v);
        }
    }
}

int orc_quantize(int f, const void* src, int dtype, int64_t rows, int64_t cols,
                 uint8_t* codes, void* scales) {
    int rc = check(f, dtype, rows, cols);
    if (rc) return rc;
    quantize_f(&FMT[f], src, dtype, rows * (cols / 32), codes, scales);
    return 0;
}

int orc_dequantize(int f, const uint8_t* codes, const void* scales, int64_t rows, int64_t cols,
                   void* dst, int dtype) {
    int rc = check(f, dtype, rows, cols);
    if (rc) return rc;
    dequantize_f(&FMT[f], codes, scales, rows * (cols / 32), dst, dtype);
    return 0;
}

int orc_fake_quantize(int f, const void* src, int dtype, int64_t rows, int64_t cols, void* dst) {
    int rc = check(f, dtype, rows, cols);
    if (rc) return rc;
    fake_quantize_f(&FMT[f], src, dtype, rows * (cols / 32), dst);
    return 0;
}

/* ---- eXmY element formats ---------------------------------------------- */
/*
 * [EXMY] abstract: a data type for any bit width (3, 5, 6, 7, 9 bits ...) and
 * every split of the bits after the sign into exponent and mantissa (e.g.
 * e0m6 ... e6m0 at 7 bits), with dense byte-addressable packing.
 * Readings (the abstract fixes none of them): value of a code with E exponent
 * bits and M mantissa bits as in the element formats above, with bias
 * b = 2^(E-1) - 1 for E >= 1 and b = 0 for E = 0 (a sign + fixed-point
 * magnitude m / 2^(M-1)); no code is reserved for Inf or NaN; the shared scale
 * and rounding rules are the block rule above with emax = 2^(E-1) (0 when
 * E = 0); codes packed LSB-first, W = 1 + E + M bits each, so a block's payload
 * is 4W bytes; the scale is one E8M0 byte. Supported: 0 <= E <= 5, M >= 1,
 * 3 <= W <= 9. (e2m1, e2m3 and e3m2 are then MXFP4 / MXFP6; e0m5 is AXS-6.)
 */
static int exmy_desc(int E, int M, fmt_t* F) {
    if (E < 0 || E > 5 || M < 1 || 1 + E + M < 3 || 1 + E + M > 9) return 1;
    F->bits = 1 + E + M;
    F->mbits = M;
    F->bias = E >= 1 ? (1 << (E - 1)) - 1 : 0;
    F->emax = E >= 1 ? (1 << (E - 1)) : 0;
    F->fixed = 0;
    F->nan_mag = -1;
    return 0;
}

double orc_exmy_decode(int E, int M, uint32_t code) {
    fmt_t F;
    return exmy_desc(E, M, &F) ? NAN : decode_f(&F, code);
}

double orc_exmy_maxval(int E, int M) {
    fmt_t F;
    return exmy_desc(E, M, &F) ? NAN : decode_f(&F, max_mag(&F));
}

int orc_exmy_emax(int E, int M) {
    fmt_t F;
    return exmy_desc(E, M, &F) ? -1 : F.emax;
}

void orc_exmy_round_mags(int E, int M, const double* y, int64_t n, uint32_t* out) {
    fmt_t F;
    if (exmy_desc(E, M, &F)) return;
    for (int64_t i = 0; i < n; ++i) out[i] = round_mag_f(&F, y[i]);
}

int orc_quantize_exmy(int E, int M, const void* src, int dtype, int64_t rows, int64_t cols,
                      uint8_t* codes, uint8_t* scales) {
    fmt_t F;
    if (exmy_desc(E, M, &F)) return 1;
    int rc = check(0, dtype, rows, cols);
    if (rc) return rc;
    quantize_f(&F, src, dtype, rows * (cols / 32), codes, scales);
    return 0;
}

int orc_dequantize_exmy(int E, int M, const uint8_t* codes, const uint8_t* scales, int64_t rows,
                        int64_t cols, void* dst, int dtype) {
    fmt_t F;
    if (exmy_desc(E, M, &F)) return 1;
    int rc = check(0, dtype, rows, cols);
    if (rc) return rc;
    dequantize_f(&F, codes, scales, rows * (cols / 32), dst, dtype);
    return 0;
}

int orc_fake_quantize_exmy(int E, int M, const void* src, int dtype, int64_t rows, int64_t cols,
                           void* dst) {
    fmt_t F;
    if (exmy_desc(E, M, &F)) return 1;
    int rc = check(0, dtype, rows, cols);
    if (rc) return rc;
    fake_quantize_f(&F, src, dtype, rows * (cols / 32), dst);
    return 0;
}

/* ---- exp-then-quantize softmax probability stage ---------------------- */
/*
 * [EFQ] Jargon / stage table: shifted scores d = s - rowmax, exponentiated in
 * higher precision (fp32 here), materialized, then quantized per 32-key block
 * to MXFP4 (E2M1 codes, exponent-only block scale).
 *
 * The exponential is the method's own deterministic fp32 function, defined
 * so that any two faithful implementations agree bit for bit:
 *   t  = RN(d * L2E)                  L2E    = 1/ln 2 rounded to fp32
 *   n  = t rounded to an integer, ties to even
 *   r  = RN(d - n*LN2_HI)  (fused)    LN2_HI = ln 2 cut to 16 significant bits
 *   r  = RN(r - n*LN2_LO)  (fused)    LN2_LO = ln 2 - LN2_HI rounded to fp32
 *   p  = Horner of sum_{k=0..7} r^k/k!, 1/k! rounded to fp32, one fused
 *        multiply-add per step from the r^7 term down
 *   e^d = p * 2^n, as RN(RN(p * 2^(n+64)) * 2^-64) when n < -126 and
 *        RN(RN(p * 2^(n-64)) * 2^64) when n > 127
 *   t < -160 gives +0, t > 160 gives +inf, NaN gives NaN.
 * (Cody & Waite's two-constant range reduction, then a Taylor polynomial.)
 */
static float pow2f(int k) { /* k in [-126, 127] */
    uint32_t u = (uint32_t)(k + 127) << 23;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

float orc_expf(float d) {
    const float L2E = 0x1.715476p+0f;
    const float LN2_HI = 0x1.62e4p-1f;
    const float LN2_LO = 0x1.7f7d1cp-20f;
    const float C[8] = {0x1p+0f, 0x1p+0f, 0x1p-1f, 0x1.555556p-3f,
                        0x1.555556p-5f, 0x1.111112p-7f, 0x1.6c16c2p-10f, 0x1.a01a02p-13f};
    if (isnan(d)) return d;
    float t = d * L2E;
    if (t < -160.0f) return 0.0f;
    if (t > 160.0f) return INFINITY;
    float n = rintf(t);
    float r = fmaf(-n, LN2_HI, d);
    r = fmaf(-n, LN2_LO, r);
    float p = C[7];
    for (int k = 6; k >= 0; --k) p = fmaf(p, r, C[k]);
    int ni = (int)n;
    if (ni < -126) return (p * pow2f(ni + 64)) * pow2f(-64);
    if (ni > 127) return (p * pow2f(ni - 64)) * pow2f(64);
    return p * pow2f(ni);
}

/* scores [rows, cols] fp32 -> E2M1 codes + E8M0 scales of exp(s - rowmax).
 * The row maximum is taken over the whole row; a NaN anywhere makes it NaN. */
int orc_exp_quantize(int f, const float* scores, int64_t rows, int64_t cols,
                     uint8_t* codes, void* scales) {
    int rc = check(f, ORC_F32, rows, cols);
    if (rc) return rc;
    const fmt_t* F = &FMT[f];
    int64_t bpr = cols / 32;
    double x[32];
    uint32_t c[32];
    for (int64_t r = 0; r < rows; ++r) {
        const float* s = scores + r * cols;
        float m = -INFINITY;
        int has_nan = 0;
        for (int64_t j = 0; j < cols; ++j) {
            if (isnan(s[j])) has_nan = 1;
            else if (s[j] > m) m = s[j];
        }
        if (has_nan) m = NAN;
        for (int64_t bj = 0; bj < bpr; ++bj) {
            for (int i = 0; i < 32; ++i) {
                float d = s[32 * bj + i] - m;     /* fp32 subtraction */
                x[i] = (double)orc_expf(d);
            }
            int64_t b = r * bpr + bj;
            int byte = orc_quantize_block(f, x, c);
            pack_block(F, c, codes + b * payload_bytes(F));
            store_scale(F, scales, b, byte);
        }
    }
    return 0;
}

/* ---- exp-free E2M1 probabilities (EFQ-Softmax) ------------------------ */
/*
 * [EFQ] opening paragraph, "What is it" and the paragraph on the per-block
 * rule: instead of exponentiating the shifted scores and quantizing the
 * result, each microscaling block takes an exponent-only scale from its own
 * local maximum, normalizes the shifted scores with it and maps them to
 * nonnegative E2M1 codes with one affine rule; no exponential is evaluated.
 * The page gives neither the slope nor the offset of that rule. Reading
 * adopted (PARITY UNPINNED against the paper's constants, which are not on
 * the page; the rule below is pinned to exp-then-quantize where the two must
 * agree):
 *   d     = RN(s - m)                  shifted score, fp32, m = row maximum
 *   u     = RN(d * L2E)                log2 of the probability exp(d), fp32
 *   u_max = max over the block's 32 u  (NaN if any is NaN)
 *   Es    = clamp(floor(u_max) - 2, -127, 127)    exponent-only block scale
 *           (2 = floor(log2 6), E2M1's emax, as for the named formats);
 *           byte Es + 127; a NaN block stores 0xFF and codes 0
 *   w     = RN(2*u - 2*Es)             one fused multiply-add, fp32
 *   code  = clamp(rint(w) + 2, 0, 7)   ties to even; sign bit 0
 * The E2M1 magnitudes 1, 2, 4 (codes 2, 4, 6) sit at log2 0, 1, 2 and the
 * odd codes 1.5, 3, 6 at log2 0.58, 1.58, 2.58, so code = 2*log2(p/2^Es) + 2
 * is the straight line through the grid in the log domain: exact at every
 * even code and within 0.17 of a code step at the odd ones. Its decoded
 * value E2M1(code) * 2^Es approximates exp(d).
 */
int orc_exp_free_quantize(const float* scores, int64_t rows, int64_t cols, uint8_t* codes, uint8_t* scales) {
    const float L2E = 0x1.715476p+0f;
    if (rows < 0 || cols <= 0 || cols % 32) return 2;
    int64_t bpr = cols / 32;
    float u[32];
    uint32_t c[32];
    for (int64_t r = 0; r < rows; ++r) {
        const float* s = scores + r * cols;
        float m = -INFINITY;
        int has_nan = 0;
        for (int64_t j = 0; j < cols; ++j) {
            if (isnan(s[j])) has_nan = 1;
            else if (s[j] > m) m = s[j];
        }
        if (has_nan) m = NAN;
        for (int64_t bj = 0; bj < bpr; ++bj) {
            float umax = -INFINITY;
            int nan_block = 0;
            for (int i = 0; i < 32; ++i) {
                float d = s[32 * bj + i] - m;   /* fp32 subtraction */
                u[i] = d * L2E;                 /* fp32 product */
                if (isnan(u[i])) nan_block = 1;
                else if (u[i] > umax) umax = u[i];
            }
            int64_t b = r * bpr + bj;
            int byte;
            if (nan_block) {
                byte = 0xFF;
                for (int i = 0; i < 32; ++i) c[i] = 0;
            } else {
                double fl = floor((double)umax);
                int es = fl < -200.0 ? -127 : (int)fl - 2;
                if (es < -127) es = -127;
                if (es > 127) es = 127;
                byte = es + 127;
                for (int i = 0; i < 32; ++i) {
                    float w = fmaf(2.0f, u[i], -2.0f * (float)es);
                    double k = isinf(w) ? (w < 0 ? -1e9 : 1e9) : (double)rintf(w);
                    k += 2.0;
                    c[i] = k < 0.0 ? 0u : (k > 7.0 ? 7u : (uint32_t)k);
                }
            }
            pack_block(&FMT[ORC_E2M1], c, codes + b * payload_bytes(&FMT[ORC_E2M1]));
            scales[b] = (uint8_t)byte;
        }
    }
    return 0;
}

/* sizes, for the test harness */
int64_t orc_codes_bytes(int f, int64_t rows, int64_t cols) {
    return fmt_ok(f) ? rows * (cols / 32) * payload_bytes(&FMT[f]) : -1;
}
int64_t orc_scales_bytes(int f, int64_t rows, int64_t cols) {
    return fmt_ok(f) ? rows * (cols / 32) * (FMT[f].fixed ? 2 : 1) : -1;
}

/*
 * Scale-factor layout read by the block-scaled tensor-core MMA.
 *
 * The pages do not define it: "Sonar: Online MXFP6" (Current limits) runs its
 * converted weights through block-scaled GEMM kernels with dense dimensions in
 * multiples of 128, and those kernels read the per-block E8M0 scales in the
 * layout of the hardware's block-scaled MMA (NVIDIA cuBLAS documentation,
 * "1D block scaling factors layout"). Reading adopted, written out from that
 * definition:
 *   - the [rows, kb] scale matrix (kb = blocks of 32 along K per row) is
 *     padded with zero bytes to rows128 = ceil(rows/128)*128 rows and
 *     kb4 = ceil(kb/4)*4 columns;
 *   - it is cut into tiles of 128 rows x 4 columns, 512 bytes each, stored
 *     tile-row by tile-row: tile (R, C) starts at byte (R * kb4/4 + C) * 512;
 *   - inside a tile, row r (0..127) and column c (0..3) sit at byte
 *     (r % 32) * 16 + (r / 32) * 4 + c.
 */
int64_t orc_mma_scales_bytes(int64_t rows, int64_t kb) {
    if (rows < 0 || kb < 0) return -1;
    return ((rows + 127) / 128) * 128 * (((kb + 3) / 4) * 4);
}

int64_t orc_mma_scale_index(int64_t r, int64_t k, int64_t kb) {
    const int64_t tiles_per_row = (kb + 3) / 4;
    const int64_t tile = (r / 128) * tiles_per_row + k / 4;
    const int64_t rr = r % 128;
    return tile * 512 + (rr % 32) * 16 + (rr / 32) * 4 + (k % 4);
}

int orc_swizzle_scales(const uint8_t* scales, int64_t rows, int64_t kb, uint8_t* out) {
    if (rows < 0 || kb <= 0) return 1;
    const int64_t n = orc_mma_scales_bytes(rows, kb);
    for (int64_t i = 0; i < n; ++i) out[i] = 0;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t k = 0; k < kb; ++k) out[orc_mma_scale_index(r, k, kb)] = scales[r * kb + k];
    return 0;
}
