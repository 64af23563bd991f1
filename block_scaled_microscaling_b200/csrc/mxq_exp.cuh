// mxq_exp.cuh -- the library's own fp32 exponential for the exp-then-quantize
// softmax stage ("EFQ-Softmax: exp-free E2M1 probabilities", Jargon:
// exp-then-quantize of the row-max-shifted scores, in higher precision than the
// E2M1 result). Shared by the softmax-stage kernels.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

#include "mxq_block.cuh"
#include "mxq_device.cuh"

namespace mxq {

// The library's own fp32 exponential (the same definition the CPU oracle
// implements independently):
//   t = RN(d * L2E), n = t rounded to an integer, ties to even,
//   r = RN(d - n*LN2_HI) and r = RN(r - n*LN2_LO), both fused (Cody & Waite),
//   p = Horner over 1/k!, k = 7..0, one fused multiply-add per step,
//   e^d = p * 2^n (outside 2^[-126,127] as two exact-then-rounded products
//   through 2^(n+-64)); t < -160 -> +0, t > 160 -> +inf, NaN -> NaN.
// L2E = 1/ln2 and LN2_LO = ln2 - LN2_HI rounded to fp32, LN2_HI = ln 2 cut to
// 16 significant bits, 1/k! rounded to fp32.
constexpr float kL2E = 0x1.715476p+0f, kLn2Hi = 0x1.62e4p-1f, kLn2Lo = 0x1.7f7d1cp-20f;
constexpr float kC0 = 0x1p+0f, kC1 = 0x1p+0f, kC2 = 0x1p-1f, kC3 = 0x1.555556p-3f, kC4 = 0x1.555556p-5f,
                kC5 = 0x1.111112p-7f, kC6 = 0x1.6c16c2p-10f, kC7 = 0x1.a01a02p-13f;
constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: x + kRound rounds x to an integer (|x| < 2^22)

__device__ __forceinline__ float pow2i(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }

// general form, any input
__device__ __forceinline__ float expf_mxq(float d) {
    if (d != d) return d;
    float t = __fmul_rn(d, kL2E);
    if (t < -160.0f) return 0.0f;
    if (t > 160.0f) return __uint_as_float(0x7F800000u);
    float n = __fsub_rn(__fadd_rn(t, kRound), kRound);  // rint(t), ties to even
    float r = __fmaf_rn(-n, kLn2Hi, d);
    r = __fmaf_rn(-n, kLn2Lo, r);
    float p = kC7;
    p = __fmaf_rn(p, r, kC6);
    p = __fmaf_rn(p, r, kC5);
    p = __fmaf_rn(p, r, kC4);
    p = __fmaf_rn(p, r, kC3);
    p = __fmaf_rn(p, r, kC2);
    p = __fmaf_rn(p, r, kC1);
    p = __fmaf_rn(p, r, kC0);
    int ni = (int)n;
    if (ni < -126) return __fmul_rn(__fmul_rn(p, pow2i(ni + 64)), pow2i(-64));
    if (ni > 127) return __fmul_rn(__fmul_rn(p, pow2i(ni - 64)), pow2i(64));
    return __fmul_rn(p, pow2i(ni));
}

// Same function on a packed pair of shifted scores d = (lo, hi), valid when both
// t = d*L2E lie in [-126, 127] (then 2^n is one normal fp32 and one product
// suffices): n from the 1.5*2^23 add, 2^n's bits from that sum's bits.
__device__ __forceinline__ unsigned long long expf_mxq2(unsigned long long d) {
    const unsigned long long tm = f2add(f2mul(d, dup2(kL2E)), dup2(kRound));
    const unsigned long long nn = f2sub(dup2(kRound), tm);  // -n, exact
    unsigned long long r = f2fma(nn, dup2(kLn2Hi), d);
    r = f2fma(nn, dup2(kLn2Lo), r);
    unsigned long long p = f2fma(dup2(kC7), r, dup2(kC6));
    p = f2fma(p, r, dup2(kC5));
    p = f2fma(p, r, dup2(kC4));
    p = f2fma(p, r, dup2(kC3));
    p = f2fma(p, r, dup2(kC2));
    p = f2fma(p, r, dup2(kC1));
    p = f2fma(p, r, dup2(kC0));
    float a, b;
    upk(tm, a, b);
    // bits(tm) = 0x4B400000 + n, so (n + 127) << 23 = bits(tm) * 2^23 + 0x3F800000 (mod 2^32)
    const float sa = __uint_as_float(__float_as_uint(a) * 0x800000u + 0x3F800000u);
    const float sb = __uint_as_float(__float_as_uint(b) * 0x800000u + 0x3F800000u);
    return f2mul(p, pk(sa, sb));
}

// Shifted scores d = x - mr -> e^d, in place, for n values (n even); packed
// path unless some t = d*L2E < -126 among them.
template <int N>
__device__ __forceinline__ void exp_values(uint32_t (&w)[N], float mr) {
    float tmin = 0.0f;
#pragma unroll
    for (int i = 0; i < N / 2; ++i) {
        float a, b;
        upk(f2sub(pk(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1])), dup2(mr)), a, b);
        w[2 * i] = __float_as_uint(a);
        w[2 * i + 1] = __float_as_uint(b);
        tmin = min3f(tmin, a, b);
    }
    if (__fmul_rn(tmin, kL2E) >= -126.0f) {
#pragma unroll
        for (int i = 0; i < N / 2; ++i) {
            float a, b;
            upk(expf_mxq2(pk(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1]))), a, b);
            w[2 * i] = __float_as_uint(a);
            w[2 * i + 1] = __float_as_uint(b);
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) w[i] = __float_as_uint(expf_mxq(__uint_as_float(w[i])));
    }
}

// One block of 32 scores (fp32 bit patterns in w) with the row maximum mr:
// p = e^(s - mr), the block's scale byte from max p, the codes of p; writes
// the payload and the scale of block blk.
template <int F>
__device__ __forceinline__ void exp_quant_block(uint32_t (&w)[32], float mr, long long blk, void* codes, void* scales,
                                                bool a32) {
    exp_values<32>(w, mr);
    float q[11];
#pragma unroll
    for (int i = 0; i < 10; ++i) q[i] = max3_nan(__uint_as_float(w[3 * i]), __uint_as_float(w[3 * i + 1]), __uint_as_float(w[3 * i + 2]));
    q[10] = max_nan(__uint_as_float(w[30]), __uint_as_float(w[31]));
    float pm = max3_nan(max3_nan(q[0], q[1], q[2]), max3_nan(q[3], q[4], q[5]), max3_nan(q[6], q[7], q[8]));
    pm = max3_nan(pm, q[9], q[10]);  // p >= 0 or NaN: the block maximum (or NaN)
    const uint32_t byte = scale_byte<F>(__float_as_uint(pm) & 0x7FFFFFFFu);
    uint32_t out[8];
    if constexpr (F == F_AXS6) {
        // probabilities are never negative: m = min(rne(p * 2^(4 - Es)), 31) by one packed
        // fused multiply-add with 1.5 * 2^23 per pair (the product is exact, the add rounds it
        // to an integer, ties to even), no sign to carry; scale bytes 4 .. 254 (2^(4 - Es) a
        // normal fp32), the rest (and NaN blocks) through the general encoder
        if (byte >= 4u && byte <= 254u) {
            const unsigned long long G = dup2(__uint_as_float((258u - byte) << 23)), C = dup2(kRound);
            uint32_t z[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                uint32_t c[2];
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                    float ta, tb;
                    upk(f2fma(pk(__uint_as_float(w[4 * j + 2 * q]), __uint_as_float(w[4 * j + 2 * q + 1])), G, C), ta, tb);
                    uint32_t m2;
                    asm("min.u16x2 %0, %1, %2;" : "=r"(m2) : "r"(__byte_perm(__float_as_uint(ta), __float_as_uint(tb), 0x5410)),
                        "r"(0x001F001Fu));
                    c[q] = m2 - (m2 >> 16) * 65472u;  // code_lo | code_hi << 6
                }
                z[j] = c[0] | (c[1] << 12);
            }
            pack6x8(z, out);
            pack6x8(z + 4, out + 3);
        } else {
            encode_block<F, float>(w, byte, out);
        }
    } else {
        encode_block<F, float>(w, byte, out);
    }
    store_payload<F>(codes, blk, out, a32);
    store_scale<F>(scales, blk, byte);
}

}  // namespace mxq
