// mxq_device.cuh -- device-side building blocks of libmxq (sm_100a).
//
// Element formats and the block rule (see include/mxq.h):
//   "AXS-6: Adaptive eXponent Sharing", block figure -- 8-bit shared exponent
//   per 32 values, sign + 5-bit magnitude per value (read as m/16);
//   "Sonar: Online MXFP6", Start a model -- packed six-bit E2M3/E3M2 codes with
//   an E8M0 scale per block of 32; "EFQ-Softmax", Jargon -- E2M1 (MXFP4),
//   exponent-only scale from the block's local maximum.
//
// Rounding uses the sm_100a conversion instructions
// cvt.rn.satfinite.{e2m3x2,e3m2x2,e4m3x2,e2m1x2}.f32 (round to nearest even,
// saturate to the largest finite value), two values per instruction; AXS-6
// rounds with a float add of 1.5*2^23. Decoding either places the magnitude
// bits into an fp32 bit pattern and rescales by exact powers of two, or (the
// column-direction dequantize) takes the exact values from the up-conversions
// cvt.rn.f16x2.{e2m3x2,e3m2x2,e4m3x2,e2m1x2} and multiplies by the scale.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace mxq {

enum : int { F_AXS6 = 0, F_E2M3 = 1, F_E3M2 = 2, F_E4M3 = 3, F_E2M1 = 4 };

template <int F> struct Fmt;
// W: code bits; EMAX: floor(log2 max); M: mantissa bits; BIAS: exponent bias
template <> struct Fmt<F_AXS6> { static constexpr int W = 6, EMAX = 0, M = 5, BIAS = 0; static constexpr bool FIXED = true; };
template <> struct Fmt<F_E2M3> { static constexpr int W = 6, EMAX = 2, M = 3, BIAS = 1; static constexpr bool FIXED = false; };
template <> struct Fmt<F_E3M2> { static constexpr int W = 6, EMAX = 4, M = 2, BIAS = 3; static constexpr bool FIXED = false; };
template <> struct Fmt<F_E4M3> { static constexpr int W = 8, EMAX = 8, M = 3, BIAS = 7; static constexpr bool FIXED = false; };
template <> struct Fmt<F_E2M1> { static constexpr int W = 4, EMAX = 2, M = 1, BIAS = 1; static constexpr bool FIXED = false; };

// bytes of one block's packed payload
template <int F> __host__ __device__ constexpr int payload() { return 4 * Fmt<F>::W; }

// ---------------------------------------------------------------------------
// memory primitives

__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}
__device__ __forceinline__ void st_stream_v4(void* p, uint4 v) {
    asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1,%2,%3,%4};"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
// 32 bytes = one DRAM sector per lane (sm_100 256-bit accesses); p 32-byte aligned
__device__ __forceinline__ void ld_v8(const void* p, uint32_t* r) {
    asm volatile("ld.global.nc.L1::no_allocate.L2::evict_first.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "l"(p));
}
__device__ __forceinline__ void st_v8(void* p, const uint32_t* r) {
    asm volatile("st.global.L1::no_allocate.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
                 :: "l"(p), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
// 32-byte loads with an L2 priority hint: keep (first pass over data that is
// read again soon) or drop first (last use)
__device__ __forceinline__ void ld_v8_keep(const void* p, uint32_t* r) {
    asm volatile("ld.global.nc.L1::no_allocate.L2::evict_last.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "l"(p));
}
// 16-byte halves through L1 (the second half of a sector then hits L1); p 16-byte aligned
__device__ __forceinline__ void ld_2v4(const void* p, uint32_t* r) {
    uint4 a, b;
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w) : "l"(p));
    asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(b.x), "=r"(b.y), "=r"(b.z), "=r"(b.w) : "l"(reinterpret_cast<const char*>(p) + 16));
    r[0] = a.x; r[1] = a.y; r[2] = a.z; r[3] = a.w; r[4] = b.x; r[5] = b.y; r[6] = b.z; r[7] = b.w;
}
__device__ __forceinline__ void st_2v4(void* p, const uint32_t* r) {
    st_stream_v4(p, make_uint4(r[0], r[1], r[2], r[3]));
    st_stream_v4(reinterpret_cast<char*>(p) + 16, make_uint4(r[4], r[5], r[6], r[7]));
}
// 32 bytes at p: one 256-bit access when a32, else two 128-bit ones
__device__ __forceinline__ void ld32(const void* p, uint32_t* r, bool a32) {
    if (a32) ld_v8(p, r);
    else ld_2v4(p, r);
}
__device__ __forceinline__ void st32(void* p, const uint32_t* r, bool a32) {
    if (a32) st_v8(p, r);
    else st_2v4(p, r);
}

// ---------------------------------------------------------------------------
// programmatic dependent launch: wait for the grids this one depends on (before any global
// memory access), then let the next launch in the stream be scheduled

__device__ __forceinline__ void pdl_wait_then_release() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// packed fp32 pair arithmetic (one instruction for two IEEE round-to-nearest ops)

__device__ __forceinline__ unsigned long long pk(float a, float b) {
    unsigned long long r;
    asm("mov.b64 %0, {%1,%2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk(unsigned long long r, float& a, float& b) {
    asm("mov.b64 {%0,%1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ void mul2(float& a, float& b, float s) {
    unsigned long long r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(pk(a, b)), "l"(pk(s, s)));
    upk(r, a, b);
}
// packed pair ops on 64-bit {lo, hi} values
__device__ __forceinline__ unsigned long long f2mul(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ unsigned long long f2add(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ unsigned long long f2sub(unsigned long long a, unsigned long long b) {
    unsigned long long r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ unsigned long long f2fma(unsigned long long a, unsigned long long b, unsigned long long c) {
    unsigned long long r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ unsigned long long dup2(float s) { return pk(s, s); }

// NaN-propagating maxima (a NaN operand gives NaN); |a|,|b| variants for amax
__device__ __forceinline__ float max_nan(float a, float b) {
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ float max3_nan(float a, float b, float c) {
    float r;
    asm("max.NaN.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
// three-input minimum (a NaN operand is ignored)
__device__ __forceinline__ float min3f(float a, float b, float c) {
    float r;
    asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}
// max(|a|, |b|) of two bf16 pairs, lane-wise; NaN -> NaN (sign bits of the result are not meaningful)
__device__ __forceinline__ uint32_t absmax_bf16x2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.NaN.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ float absmax_f32(float a, float b) {
    float r;
    asm("max.NaN.xorsign.abs.f32 %0, %1, %2;" : "=f"(r) : "f"(a), "f"(b));
    return r;
}

// ---------------------------------------------------------------------------
// the shared scale

// |x| bit patterns order as unsigned integers: finite < +Inf < NaN.
// byte = 0xFF for a NaN/Inf block, else clamp(floor(log2 amax) - EMAX + 127, 0, 254);
// for amax normal that is max(biased exponent - EMAX, 0), and every subnormal
// or zero amax gives 0.
template <int F>
__device__ __forceinline__ uint32_t scale_byte(uint32_t amax_bits) {
    int b = (int)(amax_bits >> 23) - Fmt<F>::EMAX;
    return amax_bits >= 0x7F800000u ? 0xFFu : (uint32_t)max(b, 0);
}

// 2^(127 - byte) as fp32 (the reciprocal of the block scale), byte in [0, 254]
__device__ __forceinline__ float inv_scale(uint32_t byte) {
    uint32_t bits = byte >= 254u ? 0x00400000u : (254u - byte) << 23;
    return __uint_as_float(bits);
}
// 2^(byte - 127) as fp32, byte in [0, 254]
__device__ __forceinline__ float fwd_scale(uint32_t byte) {
    return __uint_as_float(byte == 0u ? 0x00400000u : byte << 23);
}

// ---------------------------------------------------------------------------
// hardware rounding to the element formats, two at a time: result holds
// code(lo) in the low byte (low nibble for E2M1) and code(hi) above it.

template <int F> __device__ __forceinline__ uint32_t cvt2(float lo, float hi);
template <> __device__ __forceinline__ uint32_t cvt2<F_E2M3>(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e2m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
template <> __device__ __forceinline__ uint32_t cvt2<F_E3M2>(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e3m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
template <> __device__ __forceinline__ uint32_t cvt2<F_E4M3>(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}
template <> __device__ __forceinline__ uint32_t cvt2<F_E2M1>(float lo, float hi) {
    uint32_t r;
    asm("{ .reg .b8 t; cvt.rn.satfinite.e2m1x2.f32 t, %1, %2; cvt.u32.u8 %0, t; }"
        : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// Eight values -> one word of eight E2M1 codes (nibble k = code of value k):
// four conversions straight into byte registers, one vector move.
__device__ __forceinline__ uint32_t cvt8_e2m1(float v0, float v1, float v2, float v3, float v4, float v5, float v6,
                                              float v7) {
    uint32_t w;
    asm("{ .reg .b8 b0, b1, b2, b3;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n"
        "mov.b32 %0, {b0, b1, b2, b3}; }"
        : "=r"(w) : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
    return w;
}
// Four values -> one word of four E4M3 codes (byte k = code of value k).
__device__ __forceinline__ uint32_t cvt4_e4m3(float v0, float v1, float v2, float v3) {
    uint32_t w;
    asm("{ .reg .b16 h0, h1;\n"
        "cvt.rn.satfinite.e4m3x2.f32 h0, %2, %1;\n"
        "cvt.rn.satfinite.e4m3x2.f32 h1, %4, %3;\n"
        "mov.b32 %0, {h0, h1}; }"
        : "=r"(w) : "f"(v0), "f"(v1), "f"(v2), "f"(v3));
    return w;
}

// AXS-6 code of x (already multiplied by 2^-Es): sign | min(rne(16|x|), 31).
// rne by adding 1.5*2^23 (|16x| < 2^22): the sum's low mantissa bits are the
// rounded integer.
__device__ __forceinline__ uint32_t axs6_code(float y) {
    float t = fabsf(y) * 16.0f;
    uint32_t m = __float_as_uint(t + 12582912.0f) - 0x4B400000u;
    m = min(m, 31u);
    return m | ((__float_as_uint(y) >> 26) & 0x20u);
}

// Codes of n = 2k values, one code per byte (E2M1: one per nibble, packed).
// Returned as words with codes in ascending byte order.
//   6-bit / 8-bit formats: out[j] holds codes 4j..4j+3, one per byte.
//   E2M1: out[j] holds codes 8j..8j+7, one per nibble.
template <int F, int N>
__device__ __forceinline__ void encode(const float* y, uint32_t* out) {
    if constexpr (F == F_AXS6) {
#pragma unroll
        for (int j = 0; j < N / 4; ++j)
            out[j] = axs6_code(y[4 * j]) | axs6_code(y[4 * j + 1]) << 8 | axs6_code(y[4 * j + 2]) << 16 |
                     axs6_code(y[4 * j + 3]) << 24;
    } else if constexpr (F == F_E2M1) {
#pragma unroll
        for (int j = 0; j < (N + 7) / 8; ++j) {
            uint32_t w = 0;
#pragma unroll
            for (int k = 0; k < 4 && 8 * j + 2 * k < N; ++k) w |= cvt2<F>(y[8 * j + 2 * k], y[8 * j + 2 * k + 1]) << (8 * k);
            out[j] = w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < N / 4; ++j)
            out[j] = cvt2<F>(y[4 * j], y[4 * j + 1]) | cvt2<F>(y[4 * j + 2], y[4 * j + 3]) << 16;
    }
}

// four 6-bit codes, one per byte (b0..b3) -> 24-bit field b0 | b1<<6 | b2<<12 | b3<<18
__device__ __forceinline__ uint32_t pack6x4(uint32_t x) {
    uint32_t y = (x & 0x003F003Fu) | ((x >> 2) & 0x0FC00FC0u);
    return (y & 0x00000FFFu) | ((y >> 4) & 0x00FFF000u);
}
// inverse: 24-bit field -> four codes, one per byte
__device__ __forceinline__ uint32_t unpack6x4(uint32_t z) {
    uint32_t y = (z & 0x00000FFFu) | ((z << 4) & 0x0FFF0000u);
    return (y & 0x003F003Fu) | ((y << 2) & 0x3F003F00u);
}

// ---------------------------------------------------------------------------
// decoding: code -> exact value * 2^(byte-127)

// fp32 bit pattern whose value is decode(code) * 2^-(127-BIAS) (FP formats) or
// decode(code) * 2^-126 (AXS-6): the magnitude field lands on the fp32
// exponent/mantissa fields (subnormal patterns included), sign on bit 31.
template <int F>
__device__ __forceinline__ uint32_t code_to_bits(uint32_t c) {
    constexpr int W = Fmt<F>::W;
    constexpr int SH = Fmt<F>::FIXED ? 19 : 23 - Fmt<F>::M;
    return ((c & ((1u << (W - 1)) - 1u)) << SH) | ((c << (32 - W)) & 0x80000000u);
}
template <int F> __device__ __forceinline__ float decode_unit() {
    return __uint_as_float((uint32_t)((Fmt<F>::FIXED ? 126 : 127 - Fmt<F>::BIAS) + 127) << 23);
}

// values of two codes times the block scale s = 2^(byte-127); exact products
// except for the final rounding of results below the fp32 normal range.
template <int F>
__device__ __forceinline__ void decode2(uint32_t c0, uint32_t c1, float s, float& v0, float& v1) {
    v0 = __uint_as_float(code_to_bits<F>(c0));
    v1 = __uint_as_float(code_to_bits<F>(c1));
    mul2(v0, v1, decode_unit<F>());
    mul2(v0, v1, s);
}

// ---------------------------------------------------------------------------
// exact element values by the sm_100a up-conversions: cvt.rn.f16x2.{e2m3x2,e3m2x2,e4m3x2} turns
// two codes (one per byte of a 16-bit operand, low byte -> low half) into their f16 values,
// cvt.rn.f16x2.e2m1x2 two nibbles of a byte. Every value of these formats is an f16 normal or
// zero, so the conversion is exact (an E4M3 NaN code gives an f16 NaN); the f16 -> f32 widening
// is exact too.

// four codes, one per byte of x (6-bit codes in the low 6 bits, 8-bit codes whole) -> f32 values
template <int F>
__device__ __forceinline__ void up4(uint32_t x, float& v0, float& v1, float& v2, float& v3) {
    static_assert(F == F_E2M3 || F == F_E3M2 || F == F_E4M3, "byte-wide codes");
    if constexpr (F == F_E2M3)
        asm("{ .reg .b16 lo, hi; .reg .b32 a, b; .reg .f16 a0, a1, b0, b1;\n"
            "mov.b32 {lo, hi}, %4;\n"
            "cvt.rn.f16x2.e2m3x2 a, lo;\n cvt.rn.f16x2.e2m3x2 b, hi;\n"
            "mov.b32 {a0, a1}, a;\n mov.b32 {b0, b1}, b;\n"
            "cvt.f32.f16 %0, a0;\n cvt.f32.f16 %1, a1;\n cvt.f32.f16 %2, b0;\n cvt.f32.f16 %3, b1; }"
            : "=f"(v0), "=f"(v1), "=f"(v2), "=f"(v3) : "r"(x));
    else if constexpr (F == F_E3M2)
        asm("{ .reg .b16 lo, hi; .reg .b32 a, b; .reg .f16 a0, a1, b0, b1;\n"
            "mov.b32 {lo, hi}, %4;\n"
            "cvt.rn.f16x2.e3m2x2 a, lo;\n cvt.rn.f16x2.e3m2x2 b, hi;\n"
            "mov.b32 {a0, a1}, a;\n mov.b32 {b0, b1}, b;\n"
            "cvt.f32.f16 %0, a0;\n cvt.f32.f16 %1, a1;\n cvt.f32.f16 %2, b0;\n cvt.f32.f16 %3, b1; }"
            : "=f"(v0), "=f"(v1), "=f"(v2), "=f"(v3) : "r"(x));
    else
        asm("{ .reg .b16 lo, hi; .reg .b32 a, b; .reg .f16 a0, a1, b0, b1;\n"
            "mov.b32 {lo, hi}, %4;\n"
            "cvt.rn.f16x2.e4m3x2 a, lo;\n cvt.rn.f16x2.e4m3x2 b, hi;\n"
            "mov.b32 {a0, a1}, a;\n mov.b32 {b0, b1}, b;\n"
            "cvt.f32.f16 %0, a0;\n cvt.f32.f16 %1, a1;\n cvt.f32.f16 %2, b0;\n cvt.f32.f16 %3, b1; }"
            : "=f"(v0), "=f"(v1), "=f"(v2), "=f"(v3) : "r"(x));
}
// eight E2M1 codes, one per nibble of x (code k in nibble k) -> f32 values
__device__ __forceinline__ void up8_e2m1(uint32_t x, float* v) {
    asm("{ .reg .b8 c0, c1, c2, c3; .reg .b32 a, b, c, d; .reg .f16 a0, a1, b0, b1, e0, e1, d0, d1;\n"
        "mov.b32 {c0, c1, c2, c3}, %8;\n"
        "cvt.rn.f16x2.e2m1x2 a, c0;\n cvt.rn.f16x2.e2m1x2 b, c1;\n"
        "cvt.rn.f16x2.e2m1x2 c, c2;\n cvt.rn.f16x2.e2m1x2 d, c3;\n"
        "mov.b32 {a0, a1}, a;\n mov.b32 {b0, b1}, b;\n mov.b32 {e0, e1}, c;\n mov.b32 {d0, d1}, d;\n"
        "cvt.f32.f16 %0, a0;\n cvt.f32.f16 %1, a1;\n cvt.f32.f16 %2, b0;\n cvt.f32.f16 %3, b1;\n"
        "cvt.f32.f16 %4, e0;\n cvt.f32.f16 %5, e1;\n cvt.f32.f16 %6, d0;\n cvt.f32.f16 %7, d1; }"
        : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]), "=f"(v[6]), "=f"(v[7])
        : "r"(x));
}

// Sixteen consecutive codes of a payload, starting at a word boundary (hw: their W/2 words), as
// exact f32 values of the element format (AXS-6: m/16 with the sign; E4M3 NaN codes: NaN).
// 6-bit codes are spread to one per byte first: a 24-bit group c0 | c1 << 6 | c2 << 12 | c3 << 18
// becomes c0 | c1 << 8 | c2 << 16 | c3 << 24 in two shift-and-merge steps.
template <int F>
__device__ __forceinline__ void decode16(const uint32_t* hw, float* v) {
    if constexpr (F == F_E4M3) {
#pragma unroll
        for (int i = 0; i < 4; ++i) up4<F>(hw[i], v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else if constexpr (F == F_E2M1) {
        up8_e2m1(hw[0], v);
        up8_e2m1(hw[1], v + 8);
    } else {
        uint32_t g[4];
        g[0] = hw[0];
        g[1] = __funnelshift_r(hw[0], hw[1], 24);
        g[2] = __funnelshift_r(hw[1], hw[2], 16);
        g[3] = hw[2] >> 8;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            // bits 24.. of a group are the next group's: the masks below drop them
            const uint32_t y = (g[i] & 0x0000FFFFu) | ((g[i] << 4) & 0xFFFF0000u);
            const uint32_t z = ((y & 0x003F003Fu) | ((y << 2) & 0x3F003F00u));
            if constexpr (F == F_AXS6) {
                // sign | 5-bit magnitude m, value m / 16: the magnitude converted exactly, the sign copied
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t c = z >> (8 * k);
                    v[4 * i + k] = __uint_as_float(__float_as_uint((float)(c & 31u) * 0.0625f) | ((c & 32u) << 26));
                }
            } else {
                up4<F>(z, v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
        }
    }
}

// fp32 pair -> bf16x2, round to nearest even
__device__ __forceinline__ uint32_t bf16x2(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

}  // namespace mxq
