// mxq_block.cuh -- one block of 32 values: load, maximum, encode to a packed
// payload, decode back (sm_100a). Shared by the codec and softmax kernels.
//
// Block rule ("AXS-6: Adaptive eXponent Sharing", block figure; "Sonar: Online
// MXFP6", Start a model; "EFQ-Softmax" stage table): one E8M0 scale from the
// block's absolute maximum, values rounded to nearest even with saturation,
// codes packed LSB-first (value j at bits [W*j, W*j+W) of the payload).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mxq_device.cuh"

namespace mxq {

template <typename T> struct Blk { static constexpr int NW = 32 * (int)sizeof(T) / 4; };  // words per block

// ---- values in ----------------------------------------------------------------------

template <typename T>
__device__ __forceinline__ void load_block(const void* base, long long b, uint32_t* w, bool a32) {
    const char* p = reinterpret_cast<const char*>(base) + b * 32 * (long long)sizeof(T);
#pragma unroll
    for (int i = 0; i < Blk<T>::NW / 8; ++i) ld32(p + 32 * i, w + 8 * i, a32);
}

// fp32 bit pattern of max |x| over the block (NaN -> a pattern above 0x7F800000)
template <typename T> __device__ __forceinline__ uint32_t block_amax(const uint32_t* w);
template <> __device__ __forceinline__ uint32_t block_amax<__nv_bfloat16>(const uint32_t* w) {
    uint32_t m[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) m[i] = absmax_bf16x2(w[2 * i], w[2 * i + 1]);
#pragma unroll
    for (int s = 4; s > 0; s >>= 1)
#pragma unroll
        for (int i = 0; i < s; ++i) m[i] = absmax_bf16x2(m[i], m[i + s]);
    return max((m[0] & 0x7FFFu) << 16, m[0] & 0x7FFF0000u);
}
template <> __device__ __forceinline__ uint32_t block_amax<float>(const uint32_t* w) {
    float m[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) m[i] = absmax_f32(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1]));
#pragma unroll
    for (int s = 8; s > 0; s >>= 1)
#pragma unroll
        for (int i = 0; i < s; ++i) m[i] = absmax_f32(m[i], m[i + s]);
    return __float_as_uint(m[0]) & 0x7FFFFFFFu;
}

// values 2i, 2i+1 of the block as a packed fp32 pair
template <typename T> __device__ __forceinline__ unsigned long long pair(const uint32_t* w, int i);
template <> __device__ __forceinline__ unsigned long long pair<__nv_bfloat16>(const uint32_t* w, int i) {
    return pk(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
}
template <> __device__ __forceinline__ unsigned long long pair<float>(const uint32_t* w, int i) {
    return pk(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1]));
}
// ---- codes of one block ---------------------------------------------------------------
//
// Each format produces, for pair i (values 2i, 2i+1), a small integer h_i
// holding code(2i) in its low W bits and code(2i+1) above it, then the pairs
// are packed LSB-first into the payload words.

// 6-bit: two codes one per byte -> 12-bit field c0 | c1 << 6
__device__ __forceinline__ uint32_t squeeze6(uint32_t h) { return h - 192u * (h >> 8); }

template <int F, typename T>
__device__ __forceinline__ uint32_t code_pair(const uint32_t* w, int i, float inv) {
    float a, b;
    upk(f2mul(pair<T>(w, i), dup2(inv)), a, b);
    if constexpr (F == F_AXS6) {
        // sign | min(rne(16|y|), 31) for both values at once in 16-bit lanes: rne by a
        // 1.5*2^23 add (the x16 is exact; the sum's low 16 bits are the rounded integer),
        // the two integers gathered by one byte permute, clamped by one 16x2 minimum; the
        // signs replicated from the top bytes by a second permute
        const uint32_t ta = __float_as_uint(fabsf(a) * 16.0f + 12582912.0f);
        const uint32_t tb = __float_as_uint(fabsf(b) * 16.0f + 12582912.0f);
        uint32_t m2;
        asm("min.u16x2 %0, %1, %2;" : "=r"(m2) : "r"(__byte_perm(ta, tb, 0x5410)), "r"(0x001F001Fu));
        uint32_t sg;  // 0xFFFF / 0 per 16-bit lane: prmt selector nibbles 0xB, 0xF replicate the sign bit of
                      // byte 3 of a and of b (CUDA's __byte_perm ignores the replicate bit)
        asm("prmt.b32 %0, %1, %2, 0xFFBB;" : "=r"(sg) : "r"(__float_as_uint(a)), "r"(__float_as_uint(b)));
        const uint32_t c2 = m2 | (sg & 0x00200020u);
        return c2 - (c2 >> 16) * 65472u;  // code_a | code_b << 6
    } else if constexpr (Fmt<F>::W == 6) {
        return squeeze6(cvt2<F>(a, b));
    } else {
        return cvt2<F>(a, b);  // E4M3: 16 bits, E2M1: 8 bits
    }
}

// AXS-6 codes of the two bf16 values of word w (low half first), g2 = 2^(4 - Es) in both bf16
// lanes: |x| * 2^(4 - Es) = 16|y| is exact, and one bf16x2 fused multiply-add with 192 rounds it
// to an integer, ties to even (bf16's unit in the last place is 1 on [128, 256) and 16|y| < 32),
// so each lane holds 192 + rne(16|y|); minus 192, clamped at 31 by a 16x2 minimum, the sign
// copied from bit 15 of each lane. Returns code_lo | code_hi << 6.
__device__ __forceinline__ uint32_t axs6_pair_bf16(uint32_t w, uint32_t g2) {
    uint32_t t, m2;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(t) : "r"(w & 0x7FFF7FFFu), "r"(g2), "r"(0x43404340u));
    asm("min.u16x2 %0, %1, %2;" : "=r"(m2) : "r"(t - 0x43404340u), "r"(0x001F001Fu));
    const uint32_t c2 = m2 | ((w >> 10) & 0x00200020u);
    return c2 - (c2 >> 16) * 65472u;
}

// the four 12-bit pairs of codes q[0..3] (eight 6-bit codes) -> three payload words
__device__ __forceinline__ void pack6x8(const uint32_t* q, uint32_t* out) {
    out[0] = q[0] | (q[1] << 24);
    out[1] = (q[1] >> 8) | (q[2] << 16);
    out[2] = (q[2] >> 16) | (q[3] << 8);
}

// payload words of a block (P/4 of them: 6-bit 6, E4M3 8, E2M1 4)
template <int F, typename T>
__device__ __forceinline__ void encode_block(const uint32_t* w, uint32_t byte, uint32_t* out) {
    if constexpr (F == F_AXS6 && sizeof(T) == 2) {
        // bf16 values, scale 2^(4 - Es) a normal bf16 (scale bytes 4 .. 254): two values per word
        if (byte >= 4u && byte <= 254u) {
            const uint32_t g = (258u - byte) << 7;
            const uint32_t g2 = g | (g << 16);
            uint32_t z[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) z[j] = axs6_pair_bf16(w[2 * j], g2) | (axs6_pair_bf16(w[2 * j + 1], g2) << 12);
            pack6x8(z, out);
            pack6x8(z + 4, out + 3);
            return;
        }
    }
    const float inv = inv_scale(byte);
    const uint32_t keep = byte == 0xFFu ? 0u : 0xFFFFFFFFu;
    if constexpr (Fmt<F>::W == 6) {
        uint32_t z[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) z[j] = (code_pair<F, T>(w, 2 * j, inv) | (code_pair<F, T>(w, 2 * j + 1, inv) << 12)) & keep;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const uint32_t* q = z + 4 * k;
            out[3 * k + 0] = q[0] | (q[1] << 24);
            out[3 * k + 1] = (q[1] >> 8) | (q[2] << 16);
            out[3 * k + 2] = (q[2] >> 16) | (q[3] << 8);
        }
    } else if constexpr (Fmt<F>::W == 8) {
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float a0, a1, a2, a3;
            upk(f2mul(pair<T>(w, 2 * j), dup2(inv)), a0, a1);
            upk(f2mul(pair<T>(w, 2 * j + 1), dup2(inv)), a2, a3);
            out[j] = cvt4_e4m3(a0, a1, a2, a3) & keep;
        }
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float a[8];
#pragma unroll
            for (int q = 0; q < 4; ++q) upk(f2mul(pair<T>(w, 4 * j + q), dup2(inv)), a[2 * q], a[2 * q + 1]);
            out[j] = cvt8_e2m1(a[0], a[1], a[2], a[3], a[4], a[5], a[6], a[7]) & keep;
        }
    }
}

template <int F>
__device__ __forceinline__ void store_payload(void* codes, long long b, const uint32_t* out, bool a32) {
    char* p = reinterpret_cast<char*>(codes) + b * payload<F>();
    if constexpr (Fmt<F>::W == 6) {  // 24 bytes at a multiple of 8
        uint2* q = reinterpret_cast<uint2*>(p);
        q[0] = make_uint2(out[0], out[1]);
        q[1] = make_uint2(out[2], out[3]);
        q[2] = make_uint2(out[4], out[5]);
    } else if constexpr (Fmt<F>::W == 8) {
        st32(p, out, a32);
    } else {
        st_stream_v4(p, make_uint4(out[0], out[1], out[2], out[3]));
    }
}
// 6-bit payloads are 24 bytes: a warp's 32 consecutive blocks are assembled in
// shared memory and leave as 16-byte stores (48 of them) instead of 3 x 8 bytes
// per thread.
template <int F>
__device__ __forceinline__ void warp_store6(void* codes, long long first_blk, int nvalid, const uint32_t* out,
                                            uint8_t* stage, int lane) {
    uint2* q = reinterpret_cast<uint2*>(stage + 24 * lane);
    q[0] = make_uint2(out[0], out[1]);
    q[1] = make_uint2(out[2], out[3]);
    q[2] = make_uint2(out[4], out[5]);
    __syncwarp();
    char* g = reinterpret_cast<char*>(codes) + first_blk * 24;
    const int nbytes = 24 * nvalid;
    for (int i = 16 * lane; i + 16 <= nbytes; i += 512)
        st_stream_v4(g + i, *reinterpret_cast<const uint4*>(stage + i));
    if ((nbytes & 15) && lane == 0) *reinterpret_cast<uint2*>(g + (nbytes & ~15)) = *reinterpret_cast<const uint2*>(stage + (nbytes & ~15));
    __syncwarp();
}

// Inverse of warp_store6: the warp's nvalid 24-byte payloads (consecutive blocks from
// first_blk) arrive as 16-byte loads shared by the lanes, through shared memory; lane j gets
// block first_blk + j (lanes past nvalid get stale bytes and must not use them).
__device__ __forceinline__ void warp_load6(const void* codes, long long first_blk, int nvalid, uint32_t* pw,
                                           uint8_t* stage, int lane) {
    const char* g = reinterpret_cast<const char*>(codes) + first_blk * 24;
    const int nbytes = 24 * nvalid;
    for (int i = 16 * lane; i + 16 <= nbytes; i += 512) *reinterpret_cast<uint4*>(stage + i) = ld_stream_v4(g + i);
    if ((nbytes & 15) && lane == 0)
        *reinterpret_cast<uint2*>(stage + (nbytes & ~15)) = *reinterpret_cast<const uint2*>(g + (nbytes & ~15));
    __syncwarp();
    const uint2* q = reinterpret_cast<const uint2*>(stage + 24 * lane);
    const uint2 a = q[0], b = q[1], c = q[2];
    pw[0] = a.x;
    pw[1] = a.y;
    pw[2] = b.x;
    pw[3] = b.y;
    pw[4] = c.x;
    pw[5] = c.y;
    __syncwarp();  // the stage is rewritten by the warp's next call
}

template <int F>
__device__ __forceinline__ void load_payload(const void* codes, long long b, uint32_t* out, bool a32) {
    const char* p = reinterpret_cast<const char*>(codes) + b * payload<F>();
    if constexpr (Fmt<F>::W == 6) {  // 3 x 8 bytes, through L1 so the partial sectors are fetched once
        const uint2* q = reinterpret_cast<const uint2*>(p);
        uint2 a = __ldg(q), c = __ldg(q + 1), d = __ldg(q + 2);
        out[0] = a.x; out[1] = a.y; out[2] = c.x; out[3] = c.y; out[4] = d.x; out[5] = d.y;
    } else if constexpr (Fmt<F>::W == 8) {
        ld32(p, out, a32);
    } else {
        uint4 v = ld_stream_v4(p);
        out[0] = v.x; out[1] = v.y; out[2] = v.z; out[3] = v.w;
    }
}

template <int F>
__device__ __forceinline__ void store_scale(void* scales, long long b, uint32_t byte) {
    if constexpr (Fmt<F>::FIXED) reinterpret_cast<uint16_t*>(scales)[b] = (uint16_t)byte;  // config = 0
    else reinterpret_cast<uint8_t*>(scales)[b] = (uint8_t)byte;
}
// Byte offset of block b's scale (b = r * kb + k, kb blocks per row) in the
// scale layout of the block-scaled tensor-core MMA: [rows, kb] padded to
// multiples of 128 x 4, cut into 128 x 4 tiles of 512 bytes stored tile-row by
// tile-row, row r / column c of a tile at byte (r % 32) * 16 + (r / 32) * 4 + c.
__device__ __forceinline__ long long mma_scale_offset(long long b, long long kb) {
    long long r, k;
    if ((unsigned long long)b <= 0xFFFFFFFFull && (unsigned long long)kb <= 0xFFFFFFFFull) {
        const uint32_t r32 = (uint32_t)b / (uint32_t)kb;
        r = r32;
        k = (long long)((uint32_t)b - r32 * (uint32_t)kb);
    } else {
        r = b / kb;
        k = b - r * kb;
    }
    const long long tiles = (kb + 3) >> 2;
    return ((((r >> 7) * tiles) + (k >> 2)) << 9) + ((r & 31) << 4) + (((r >> 5) & 3) << 2) + (k & 3);
}

template <int F>
__device__ __forceinline__ uint32_t load_scale(const void* scales, long long b) {
    if constexpr (Fmt<F>::FIXED) return __ldg(reinterpret_cast<const uint16_t*>(scales) + b) & 0xFFu;
    else return __ldg(reinterpret_cast<const uint8_t*>(scales) + b);
}

// ---- decoding ---------------------------------------------------------------------------

// code k (0..31) of a payload as the fp32 pattern of decode(code) * 2^-(127-BIAS)
// (AXS-6: * 2^-126): magnitude onto the exponent/mantissa fields, sign to bit 31.
template <int F>
__device__ __forceinline__ uint32_t payload_bits(const uint32_t* pw, int k) {
    constexpr int W = Fmt<F>::W;
    constexpr int SH = Fmt<F>::FIXED ? 19 : 23 - Fmt<F>::M;
    const int bit = W * k;
    uint32_t c;
    if constexpr (W == 6) {
        const int lo = bit & 31;  // fields may straddle two words
        c = (lo <= 26) ? (pw[bit >> 5] >> lo) : ((pw[bit >> 5] >> lo) | (pw[(bit >> 5) + 1] << (32 - lo)));
    } else {
        c = pw[bit >> 5] >> (bit & 31);
    }
    return ((c & ((1u << (W - 1)) - 1u)) << SH) | ((c << (32 - W)) & 0x80000000u);
}

// output: 32 values of the block as output words (bf16 pairs or fp32). Bit placement and two
// exact products: the up-conversion decode (decode16) was no faster in the row-direction
// kernels, which are bound by memory, and raised the batch kernel's registers from 44 to 59.
template <int F, typename T>
__device__ __forceinline__ void decode_block(const uint32_t* pw, uint32_t byte, uint32_t* o) {
    const float s = fwd_scale(byte);
    const unsigned long long D = dup2(decode_unit<F>()), S = dup2(s);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float a, b;
        upk(f2mul(f2mul(pk(__uint_as_float(payload_bits<F>(pw, 2 * i)), __uint_as_float(payload_bits<F>(pw, 2 * i + 1))), D), S),
            a, b);
        if constexpr (sizeof(T) == 4) {
            o[2 * i] = __float_as_uint(a);
            o[2 * i + 1] = __float_as_uint(b);
        } else {
            o[i] = bf16x2(a, b);
        }
    }
    // E4M3's NaN magnitude (0x7F) and NaN blocks: canonical quiet NaN
    if constexpr (F == F_E4M3) {
        uint32_t nan_bytes = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) nan_bytes |= ((pw[j] & 0x7F7F7F7Fu) + 0x01010101u) & 0x80808080u;
        if (nan_bytes) {
#pragma unroll
            for (int k = 0; k < 32; ++k) {
                if (((pw[k >> 2] >> (8 * (k & 3))) & 0x7Fu) == 0x7Fu) {
                    if constexpr (sizeof(T) == 4) o[k] = 0x7FC00000u;
                    else o[k >> 1] = (k & 1) ? ((o[k >> 1] & 0x0000FFFFu) | 0x7FC00000u) : ((o[k >> 1] & 0xFFFF0000u) | 0x7FC0u);
                }
            }
        }
    }
    if (byte == 0xFFu) {
#pragma unroll
        for (int i = 0; i < Blk<T>::NW; ++i) o[i] = sizeof(T) == 4 ? 0x7FC00000u : 0x7FC07FC0u;
    }
}

template <typename T>
__device__ __forceinline__ void store_block(void* dst, long long b, const uint32_t* o, bool a32) {
    char* p = reinterpret_cast<char*>(dst) + b * 32 * (long long)sizeof(T);
#pragma unroll
    for (int i = 0; i < Blk<T>::NW / 8; ++i) st32(p + 32 * i, o + 8 * i, a32);
}

// fake-quantize of one block: codes computed and decoded in registers
template <int F, typename T>
__device__ __forceinline__ void fake_block(const uint32_t* w, uint32_t byte, uint32_t* o) {
    uint32_t pw[8];
    encode_block<F, T>(w, byte, pw);
    decode_block<F, T>(pw, byte, o);
}


}  // namespace mxq
