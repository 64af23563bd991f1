// mxq_exmy.cu -- generic eXmY element formats (sm_100a).
//
// "eXmY: A Data Type and Technique for Arbitrary Bit Precision Quantization",
// abstract: one data type for any width (3, 5, 6, 7, 9 bits ...) and any
// split of the bits after the sign into E exponent and M mantissa bits, with
// dense, byte-addressable packing. Readings (the abstract fixes none): the
// value of a code is the element-format closed form with bias 2^(E-1) - 1
// (E >= 1) or 0 (E = 0: sign + fixed-point m / 2^(M-1)); no code is reserved;
// the block rule is the one of the named formats with emax = 2^(E-1) (0 for
// E = 0); W = 1 + E + M bit codes are packed LSB-first, so a block's payload is
// exactly W 32-bit words; the scale is one E8M0 byte.
//
// There is no conversion instruction for arbitrary splits, so rounding is
// integer arithmetic on the fp32 bit pattern of y = |x| * 2^-Es (an exact
// power-of-two scaling):
//   normal range   add half an ulp of the target minus one plus the kept
//                  lsb (round to nearest, ties to even), shift, re-bias;
//   subnormal      y + 2^(24 - b - M) in fp32 (that binade's ulp is the
//                  subnormal step) and subtract the constant's bits;
//   then clamp to the largest magnitude and set the sign bit.
// Kernels are templated on W (static packing positions) with E, M at run time.
#include <cstdint>
#include <cstring>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mxq_block.cuh"
#include "mxq_device.cuh"
#include "mxq_internal.h"

namespace mxq {

constexpr int kExThreads = 256;

struct ExmyParams {
    int M;            // mantissa bits
    int emax;         // floor(log2 max)
    uint32_t maxmag;  // 2^(E+M) - 1
    uint32_t shift;   // 23 - M
    uint32_t rebias;  // (127 - b) << M
    uint32_t sub_lim; // fp32 bits of 2^(1-b): below it the grid step is fixed
    float sub_c;      // 2^(24 - b - M)
    float dec_unit;   // 2^(127 - b)
    uint32_t emin_b;  // 128 - b: biased fp32 exponent of the smallest normal 2^(1-b)
    uint32_t cadd;    // ((23 - M) << 23) | 0x400000: the rounding constant's bits less its exponent
    uint32_t kcode;   // (b - 128) << M (mod 2^32)
    float maxval;     // value of the largest magnitude code
    // the two-values-per-word path (bf16 values, M <= 5), every constant in both 16-bit lanes:
    uint32_t emin2;   // (128 - b) << 7: bf16 exponent field of 2^(1-b)
    uint32_t cadd2;   // ((7 - M) << 7) | 0x40: added to an exponent field, the bf16 bits of 1.5 * 2^(e + 7 - M)
    uint32_t kneg2;   // -(((128 - b) << M) in both lanes): the code's exponent offset
    uint32_t max2;    // maxmag
    uint32_t sh7;     // 7 - M
};

static ExmyParams exmy_params(int E, int M) {
    const int b = E >= 1 ? (1 << (E - 1)) - 1 : 0;
    ExmyParams p;
    p.M = M;
    p.emax = E >= 1 ? (1 << (E - 1)) : 0;
    p.maxmag = (1u << (E + M)) - 1u;
    p.shift = (uint32_t)(23 - M);
    p.rebias = (uint32_t)(127 - b) << M;
    p.sub_lim = (uint32_t)(1 - b + 127) << 23;
    const int ce = 24 - b - M;
    uint32_t cb = (uint32_t)(ce + 127) << 23;
    float cf;
    memcpy(&cf, &cb, 4);
    p.sub_c = cf;
    uint32_t db = (uint32_t)(127 - b + 127) << 23;
    float df;
    memcpy(&df, &db, 4);
    p.dec_unit = df;
    p.emin_b = (uint32_t)(128 - b);
    p.cadd = ((uint32_t)(23 - M) << 23) | 0x400000u;
    p.kcode = (uint32_t)(b - 128) << M;
    // largest magnitude: exponent field 2^E - 1, mantissa 2^M - 1 (E = 0: fixed point (2^M - 1) / 2^(M - 1))
    p.maxval = E >= 1 ? ldexpf(1.0f + (float)((1 << M) - 1) / (float)(1 << M), (1 << E) - 1 - b)
                      : (float)((1 << M) - 1) / (float)(1 << (M - 1));
    auto both = [](uint32_t v) { return v | (v << 16); };
    p.emin2 = both((uint32_t)(128 - b) << 7);
    p.cadd2 = M <= 7 ? both(((uint32_t)(7 - M) << 7) | 0x40u) : 0u;
    p.kneg2 = 0u - both((uint32_t)(128 - b) << M);
    p.max2 = both(p.maxmag);
    p.sh7 = M <= 7 ? (uint32_t)(7 - M) : 0u;
    return p;
}

// magnitude code of y >= 0 (fp32, already scaled), one formula for the normal and the subnormal
// range: with e = max(exponent of y, 1 - b), the grid step there is 2^(e - M); adding
// C = 1.5 * 2^(e + 23 - M) rounds y to that step (round to nearest, ties to even, exact for
// y / step < 2^22) and leaves q = y / step in the low bits of the sum; the code is
// (e + b - 1) * 2^M + q (a carry of q into the next binade gives the next binade's first code),
// clamped to the largest magnitude.
__device__ __forceinline__ uint32_t exmy_mag(float y, const ExmyParams& p) {
    const uint32_t eb = max(__float_as_uint(y) >> 23, p.emin_b);  // biased e
    const uint32_t cb = eb * 0x800000u + p.cadd;
    const uint32_t q = __float_as_uint(y + __uint_as_float(cb)) - cb;
    return min((eb << p.M) + q + p.kcode, p.maxmag);
}

// The grid value nearest y >= 0 (already scaled), saturated: the same sum as exmy_mag, but the
// rounded value is read back as RN(y + C) - C (exact: both lie in C's binade) instead of as a code.
__device__ __forceinline__ float exmy_round_value(float y, const ExmyParams& p) {
    const uint32_t eb = max(__float_as_uint(y) >> 23, p.emin_b);
    const float c = __uint_as_float(eb * 0x800000u + p.cadd);
    return fminf(__fsub_rn(__fadd_rn(y, c), c), p.maxval);
}

template <int W> __device__ __forceinline__ void pack_codes(const uint32_t* c, uint32_t* out) {
#pragma unroll
    for (int i = 0; i < W; ++i) out[i] = 0;
#pragma unroll
    for (int k = 0; k < 32; ++k) {
        const int bit = W * k, wd = bit >> 5, off = bit & 31;
        out[wd] |= c[k] << off;
        if (off + W > 32) out[wd + 1] |= c[k] >> (32 - off);
    }
}
template <int W> __device__ __forceinline__ uint32_t code_of(const uint32_t* pw, int k) {
    const int bit = W * k, wd = bit >> 5, off = bit & 31;
    uint32_t c = pw[wd] >> off;
    if (off + W > 32) c |= pw[wd + 1] << (32 - off);
    return c & ((1u << W) - 1u);
}

// sign bit (as an fp32 sign) of value k of a block held as words
template <typename T> __device__ __forceinline__ uint32_t w2sign(const uint32_t* w, int k);
template <> __device__ __forceinline__ uint32_t w2sign<float>(const uint32_t* w, int k) { return w[k] & 0x80000000u; }
template <> __device__ __forceinline__ uint32_t w2sign<__nv_bfloat16>(const uint32_t* w, int k) {
    return (k & 1) ? (w[k >> 1] & 0x80000000u) : ((w[k >> 1] << 16) & 0x80000000u);
}

// values of one block -> W payload words
template <int W, typename T>
__device__ __forceinline__ void exmy_encode(const uint32_t* w, uint32_t byte, const ExmyParams& p, uint32_t* out) {
    const float inv = inv_scale(byte);
    uint32_t c[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float a, b;
        upk(f2mul(pair<T>(w, i), dup2(inv)), a, b);
        c[2 * i] = exmy_mag(fabsf(a), p) | ((__float_as_uint(a) >> 31) << (W - 1));
        c[2 * i + 1] = exmy_mag(fabsf(b), p) | ((__float_as_uint(b) >> 31) << (W - 1));
    }
    pack_codes<W>(c, out);
    if (byte == 0xFFu) {
#pragma unroll
        for (int i = 0; i < W; ++i) out[i] = 0;
    }
}

// ---- bf16 values, M <= 5: two values per 32-bit word --------------------------------------
//
// The same rounding as exmy_mag, on the two bf16 values of a word at once: y = x * 2^-Es with
// mul.rn.bf16x2 (exact: a power of two times an 8-bit significand; a result below bf16's normal
// range is far below half the format's smallest step, so it still gives code 0), the binade
// constant C = 1.5 * 2^(e + 7 - M) built in each 16-bit lane from y's exponent field (clamped
// from below with max.u16x2), RN(y + C) with add.rn.bf16x2 (bf16's 8-bit significand puts
// C's ulp at the grid step 2^(e - M), and y + C stays in C's binade while M <= 5), then the step
// count q = bits(sum) - bits(C) and code = (e << M) + q - ((128 - b) << M) in 32-bit integer
// adds: every lane's partial results lie in [0, 2^16), so no carry or borrow crosses lanes.
// Saturation with min.u16x2, signs moved from bits 15/31 to bits W-1 / W+15.
__device__ __forceinline__ uint32_t bf2mul(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t bf2add(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t umax2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}
__device__ __forceinline__ uint32_t umin2(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// 16 fields of 2W bits (codes of values 2i, 2i+1) -> W payload words, LSB-first
template <int W> __device__ __forceinline__ void pack_pairs(const uint32_t* f, uint32_t* out) {
#pragma unroll
    for (int i = 0; i < W; ++i) out[i] = 0;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const int bit = 2 * W * k, wd = bit >> 5, off = bit & 31;
        out[wd] |= f[k] << off;
        if (off + 2 * W > 32) out[wd + 1] |= f[k] >> (32 - off);
    }
}

template <int W>
__device__ __forceinline__ void exmy_encode_bf16x2(const uint32_t* w, uint32_t byte, const ExmyParams& p, uint32_t* out) {
    const uint32_t s = ((254u - byte) << 7) * 0x10001u;  // 2^(127 - byte) in both lanes; byte <= 253
    constexpr uint32_t kSign = (1u << (W - 1)) | (1u << (W + 15));
    uint32_t f[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint32_t y = bf2mul(w[i], s) & 0x7FFF7FFFu;
        const uint32_t e = umax2(y & 0x7F807F80u, p.emin2);
        const uint32_t c = e + p.cadd2;
        const uint32_t q = bf2add(y, c) - c;
        uint32_t code = umin2((e >> p.sh7) + q + p.kneg2, p.max2);
        code |= (w[i] >> (16 - W)) & kSign;
        f[i] = code - (code >> 16) * (65536u - (1u << W));  // c0 | c1 << W
    }
    pack_pairs<W>(f, out);
}

// W payload words -> 32 output values (bf16 pairs or fp32 words)
template <int W, typename T>
__device__ __forceinline__ void exmy_decode(const uint32_t* pw, uint32_t byte, const ExmyParams& p, uint32_t* o) {
    const unsigned long long D = dup2(p.dec_unit), S = dup2(fwd_scale(byte));
    const uint32_t sh = p.shift;
    auto bits = [&](uint32_t c) { return ((c & ((1u << (W - 1)) - 1u)) << sh) | ((c >> (W - 1)) << 31); };
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float a, b;
        upk(f2mul(f2mul(pk(__uint_as_float(bits(code_of<W>(pw, 2 * i))), __uint_as_float(bits(code_of<W>(pw, 2 * i + 1)))), D), S),
            a, b);
        if constexpr (sizeof(T) == 4) {
            o[2 * i] = __float_as_uint(a);
            o[2 * i + 1] = __float_as_uint(b);
        } else {
            o[i] = bf16x2(a, b);
        }
    }
    if (byte == 0xFFu) {
#pragma unroll
        for (int i = 0; i < Blk<T>::NW; ++i) o[i] = sizeof(T) == 4 ? 0x7FC00000u : 0x7FC07FC0u;
    }
}

// Dequantize: a warp's 32 consecutive payloads (32 x 4W bytes) arrive through shared memory, so
// that global memory sees 16-byte coalesced loads instead of W 4-byte loads per lane at a 4W-byte
// stride. stage: 32 * W words of this warp.
template <int W>
__device__ __forceinline__ void warp_load_words(const void* codes, long long first_blk, int nvalid, uint32_t* pw,
                                                uint32_t* stage, int lane) {
    const char* g = reinterpret_cast<const char*>(codes) + first_blk * 4 * W;
    const int nbytes = 4 * W * nvalid;
    for (int i = 16 * lane; i + 16 <= nbytes; i += 512)
        *reinterpret_cast<uint4*>(reinterpret_cast<char*>(stage) + i) = ld_stream_v4(g + i);
    if (lane == 0)
        for (int i = nbytes & ~15; i < nbytes; i += 4) stage[i / 4] = __ldg(reinterpret_cast<const uint32_t*>(g + i));
    __syncwarp();
#pragma unroll
    for (int i = 0; i < W; ++i) pw[i] = stage[lane * W + i];
    __syncwarp();
}

// SW: the two-values-per-word rounding (bf16 values, M <= 5); a block whose scale byte is 254
// (2^-127, not a normal bf16) or 0xFF takes the fp32 path
template <int W, typename T, bool SW = false>
__global__ void __launch_bounds__(kExThreads) k_quantize_exmy(const void* __restrict__ src, void* __restrict__ codes,
                                                              uint8_t* __restrict__ scales, long long nblocks,
                                                              ExmyParams p, bool a32) {
    const long long stride = (long long)gridDim.x * kExThreads;
    for (long long b = (long long)blockIdx.x * kExThreads + threadIdx.x; b < nblocks; b += stride) {
        uint32_t w[Blk<T>::NW];
        load_block<T>(src, b, w, a32);
        const uint32_t am = block_amax<T>(w);
        const uint32_t byte = am >= 0x7F800000u ? 0xFFu : (uint32_t)max((int)(am >> 23) - p.emax, 0);
        uint32_t out[W];
        if constexpr (SW) {
            if (byte <= 253u) exmy_encode_bf16x2<W>(w, byte, p, out);
            else exmy_encode<W, T>(w, byte, p, out);
        } else {
            exmy_encode<W, T>(w, byte, p, out);
        }
        char* q = reinterpret_cast<char*>(codes) + b * 4 * W;
        if constexpr (W == 4 || W == 8) {  // 16 or 32 bytes per lane: whole 16-byte stores
#pragma unroll
            for (int i = 0; i < W; i += 4) st_stream_v4(q + 4 * i, make_uint4(out[i], out[i + 1], out[i + 2], out[i + 3]));
        } else {
#pragma unroll
            for (int i = 0; i < W; ++i) reinterpret_cast<uint32_t*>(q)[i] = out[i];
        }
        scales[b] = (uint8_t)byte;
    }
}

template <int W, typename T>
__global__ void __launch_bounds__(kExThreads) k_dequantize_exmy(const void* __restrict__ codes,
                                                                const uint8_t* __restrict__ scales,
                                                                void* __restrict__ dst, long long nblocks, ExmyParams p,
                                                                bool a32) {
    __shared__ __align__(16) uint32_t stage[kExThreads / 32][32 * W];
    const int lane = threadIdx.x & 31;
    const long long stride = (long long)gridDim.x * kExThreads;
    for (long long first = (long long)blockIdx.x * kExThreads + (threadIdx.x & ~31); first < nblocks;
         first += stride) {  // warp-uniform trip count
        const long long b = first + lane;
        const int nvalid = (int)min(32LL, nblocks - first);
        const uint32_t byte = lane < nvalid ? __ldg(scales + b) : 0u;  // in flight with the payloads
        uint32_t pw[W];
        warp_load_words<W>(codes, first, nvalid, pw, stage[threadIdx.x >> 5], lane);
        if (lane < nvalid) {
            uint32_t o[Blk<T>::NW];
            exmy_decode<W, T>(pw, byte, p, o);
            store_block<T>(dst, b, o, a32);
        }
    }
}

template <int W, typename T>
__global__ void __launch_bounds__(kExThreads) k_fake_quantize_exmy(const void* src, void* dst, long long nblocks,
                                                                   ExmyParams p, bool a32) {
    const long long stride = (long long)gridDim.x * kExThreads;
    for (long long b = (long long)blockIdx.x * kExThreads + threadIdx.x; b < nblocks; b += stride) {
        uint32_t w[Blk<T>::NW];
        load_block<T>(src, b, w, a32);
        const uint32_t am = block_amax<T>(w);
        const uint32_t byte = am >= 0x7F800000u ? 0xFFu : (uint32_t)max((int)(am >> 23) - p.emax, 0);
        // no codes: each value goes straight to its grid value, times the block scale, sign copied
        // (bit-identical to decoding the encoded block)
        const unsigned long long inv = dup2(inv_scale(byte == 0xFFu ? 0u : byte)), fwd = dup2(fwd_scale(byte == 0xFFu ? 0u : byte));
        uint32_t o[Blk<T>::NW];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float a, c;
            upk(f2mul(pair<T>(w, i), inv), a, c);
            const float ra = exmy_round_value(fabsf(a), p), rc = exmy_round_value(fabsf(c), p);
            upk(f2mul(pk(ra, rc), fwd), a, c);
            a = __uint_as_float(__float_as_uint(a) | (w2sign<T>(w, 2 * i)));
            c = __uint_as_float(__float_as_uint(c) | (w2sign<T>(w, 2 * i + 1)));
            if constexpr (sizeof(T) == 4) {
                o[2 * i] = __float_as_uint(a);
                o[2 * i + 1] = __float_as_uint(c);
            } else {
                o[i] = bf16x2(a, c);
            }
        }
        if (byte == 0xFFu) {
#pragma unroll
            for (int i = 0; i < Blk<T>::NW; ++i) o[i] = sizeof(T) == 4 ? 0x7FC00000u : 0x7FC07FC0u;
        }
        store_block<T>(dst, b, o, a32);
    }
}

// Grid: one CTA per 256 blocks (one pass: the hardware starts a CTA wherever one finishes) for
// dequantize, fake-quantize and the two-lane bf16 quantize; SMs x resident CTAs walking
// grid-stride for the fp32 quantize. Measured on bf16 16384x8192 over five splits (fraction of
// the copy peak): dequantize 0.85-0.94 -> 0.90-0.93 with one pass; the two-lane quantize
// 0.89-0.97 in one pass vs 0.64-0.87 persistent; the quantize on fp32 arithmetic, bound by its
// integer rounding, 0.62-0.74 persistent vs 0.62-0.68 in one pass.
static int ex_grid(const void* fn, long long nb, bool one_pass) {
    long long want = (nb + kExThreads - 1) / kExThreads;
    if (want < 1) want = 1;
    if (one_pass) return (int)(want < 0x7FFFFFFFLL ? want : 0x7FFFFFFFLL);
    int dev = 0, sms = 148, per = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, fn, kExThreads, 0);
    const long long cap = (long long)sms * (per > 0 ? per : 1);
    return (int)(want < cap ? want : cap);
}
static bool al32(const void* a, const void* b) {
    return ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 31) == 0;
}

template <int W, typename T>
static cudaError_t ex_launch(int op, const void* in, void* out, const void* aux_in, void* aux_out, long long nb,
                             const ExmyParams& p, cudaStream_t st) {
    if (op == 0) {
        auto k = k_quantize_exmy<W, T>;
        bool two_lane = false;
        if constexpr (sizeof(T) == 2) two_lane = p.M <= 5;
        if (two_lane) k = k_quantize_exmy<W, T, true>;
        k<<<ex_grid((const void*)k, nb, two_lane), kExThreads, 0, st>>>(in, out, reinterpret_cast<uint8_t*>(aux_out), nb,
                                                                      p, al32(in, in));
    } else if (op == 1) {
        auto k = k_dequantize_exmy<W, T>;
        k<<<ex_grid((const void*)k, nb, true), kExThreads, 0, st>>>(in, reinterpret_cast<const uint8_t*>(aux_in), out, nb, p,
                                                            al32(out, out));
    } else {
        auto k = k_fake_quantize_exmy<W, T>;
        k<<<ex_grid((const void*)k, nb, true), kExThreads, 0, st>>>(in, out, nb, p, al32(in, out));
    }
    return cudaGetLastError();
}

bool exmy_supported(int E, int M) { return E >= 0 && E <= 5 && M >= 1 && 1 + E + M >= 3 && 1 + E + M <= 9; }

// op: 0 quantize (in = values, out = codes, aux_out = scales), 1 dequantize
// (in = codes, aux_in = scales, out = values), 2 fake-quantize (in -> out)
cudaError_t launch_exmy(int op, int E, int M, int dtype, const void* in, void* out, const void* aux_in, void* aux_out,
                        long long nb, cudaStream_t st) {
    if (!exmy_supported(E, M)) return cudaErrorInvalidValue;
    const ExmyParams p = exmy_params(E, M);
#define MXQ_EX(WW)                                                                                 \
    case WW:                                                                                       \
        return dtype == 1 ? ex_launch<WW, __nv_bfloat16>(op, in, out, aux_in, aux_out, nb, p, st) \
                          : ex_launch<WW, float>(op, in, out, aux_in, aux_out, nb, p, st);
    switch (1 + E + M) {
        MXQ_EX(3)
        MXQ_EX(4)
        MXQ_EX(5)
        MXQ_EX(6)
        MXQ_EX(7)
        MXQ_EX(8)
        MXQ_EX(9)
    }
#undef MXQ_EX
    return cudaErrorInvalidValue;
}

}  // namespace mxq
