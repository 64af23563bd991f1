// mxq_codec.cu -- quantize / dequantize / fused fake-quantize kernels (sm_100a).
//
// Data layout: [rows, cols] row-major with cols % 32 == 0, so the blocks of 32
// values are the consecutive 32-value groups of the flat array; a kernel
// walks blocks, not rows ("AXS-6: Adaptive eXponent Sharing", block figure;
// "Sonar: Online MXFP6", Start a model: one E8M0 scale per block of 32).
//
// Work decomposition (all three kernels):
//   * a lane owns 16 bytes of values (8 bf16 or 4 fp32) -- one 128-bit,
//     fully coalesced global access per lane;
//   * the 4 (bf16) or 8 (fp32) lanes that hold one block reduce its absolute
//     maximum with an xor-shuffle butterfly on |x| bit patterns (unsigned
//     order: finite < Inf < NaN, so NaN/Inf detection comes for free);
//   * a warp tile is U = 4 such 512-byte rows (32 bf16 / 16 fp32 blocks), all
//     loads of a tile issued before any use;
//   * packed codes of a tile are assembled in the warp's slice of shared
//     memory and leave in 16-byte stores (payloads are 16/24/32 bytes per
//     block, so a lane's codes are 2..8 bytes at odd offsets otherwise);
//   * persistent grid (SMs x resident CTAs), warps stride over tiles.
// Grouped quantize runs the same kernel over a table of tensors (kernel
// parameter), tiles never straddle two tensors.
#include <cstdint>
#include <mutex>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mxq_device.cuh"
#include "mxq_internal.h"

namespace mxq {

constexpr int kWarps = 8;  // warps per CTA
constexpr int kU = 4;      // 512-byte rows per warp tile

template <typename T> struct Lay {
    static constexpr int VPL = 16 / (int)sizeof(T);  // values per lane per row
    static constexpr int LPB = 32 / VPL;             // lanes per block
    static constexpr int BPR = 32 / LPB;             // blocks per 512-byte row
    static constexpr int BPT = kU * BPR;             // blocks per warp tile
};

// 16 bytes of values -> VPL floats and the maximum |x| bit pattern
template <typename T> struct Widen;
template <> struct Widen<float> {
    static __device__ __forceinline__ uint32_t run(uint4 v, float* x) {
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[i] = __uint_as_float(w[i]);
            m = max(m, w[i] & 0x7FFFFFFFu);
        }
        return m;
    }
};
template <> struct Widen<__nv_bfloat16> {
    static __device__ __forceinline__ uint32_t run(uint4 v, float* x) {
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
        uint32_t m2 = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            x[2 * i] = __uint_as_float(w[i] << 16);
            x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
            uint32_t a = w[i] & 0x7FFF7FFFu;
            asm("max.u16x2 %0, %0, %1;" : "+r"(m2) : "r"(a));
        }
        return max(m2 << 16, m2 & 0xFFFF0000u);
    }
};

// block amax across the LPB lanes of a block, then the shared scale byte
template <int F, int LPB>
__device__ __forceinline__ uint32_t block_byte(uint32_t am) {
#pragma unroll
    for (int o = 1; o < LPB; o <<= 1) am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
    return scale_byte<F>(am);
}

// VPL values -> y = x * 2^-Es (exact: power-of-two scaling of fp32 inputs)
template <int VPL>
__device__ __forceinline__ void apply_inv(float* x, uint32_t byte) {
    float s = inv_scale(byte);
#pragma unroll
    for (int i = 0; i < VPL; i += 2) mul2(x[i], x[i + 1], s);
}

// Encode one lane's VPL values into its LB = VPL*W/8 code bytes at smem dst.
template <int F, int VPL>
__device__ __forceinline__ void encode_store(const float* y, uint32_t keep, uint8_t* dst) {
    constexpr int W = Fmt<F>::W;
    uint32_t c[VPL / 4 > 0 ? VPL / 4 : 1];
    encode<F, VPL>(y, c);
    if constexpr (W == 8) {
        if constexpr (VPL == 8) {
            *reinterpret_cast<uint2*>(dst) = make_uint2(c[0] & keep, c[1] & keep);
        } else {
            *reinterpret_cast<uint32_t*>(dst) = c[0] & keep;
        }
    } else if constexpr (W == 4) {
        if constexpr (VPL == 8) {
            *reinterpret_cast<uint32_t*>(dst) = c[0] & keep;
        } else {
            *reinterpret_cast<uint16_t*>(dst) = (uint16_t)(c[0] & keep);
        }
    } else {  // 6-bit: 4 codes -> 3 bytes
        if constexpr (VPL == 8) {
            uint32_t z0 = pack6x4(c[0]) & keep, z1 = pack6x4(c[1]) & keep;
            uint32_t lo = z0 | (z1 << 24);
            uint16_t* d = reinterpret_cast<uint16_t*>(dst);  // 6-byte slot, 2-byte aligned
            d[0] = (uint16_t)lo;
            d[1] = (uint16_t)(lo >> 16);
            d[2] = (uint16_t)(z1 >> 8);
        } else {
            uint32_t z = pack6x4(c[0]) & keep;
            dst[0] = (uint8_t)z;
            dst[1] = (uint8_t)(z >> 8);
            dst[2] = (uint8_t)(z >> 16);
        }
    }
}

// Load one lane's LB code bytes from smem src and return the VPL codes, one per byte
// (E2M1: one per nibble) in words, ascending.
template <int F, int VPL>
__device__ __forceinline__ void load_codes(const uint8_t* src, uint32_t* c) {
    constexpr int W = Fmt<F>::W;
    if constexpr (W == 8) {
        if constexpr (VPL == 8) {
            uint2 t = *reinterpret_cast<const uint2*>(src);
            c[0] = t.x;
            c[1] = t.y;
        } else {
            c[0] = *reinterpret_cast<const uint32_t*>(src);
        }
    } else if constexpr (W == 4) {
        if constexpr (VPL == 8) c[0] = *reinterpret_cast<const uint32_t*>(src);
        else c[0] = *reinterpret_cast<const uint16_t*>(src);
    } else {
        if constexpr (VPL == 8) {
            const uint16_t* s = reinterpret_cast<const uint16_t*>(src);
            uint32_t lo = (uint32_t)s[0] | ((uint32_t)s[1] << 16), hi = s[2];
            c[0] = unpack6x4(lo & 0x00FFFFFFu);
            c[1] = unpack6x4((lo >> 24) | (hi << 8));
        } else {
            c[0] = unpack6x4((uint32_t)src[0] | ((uint32_t)src[1] << 8) | ((uint32_t)src[2] << 16));
        }
    }
}

// i-th code of the per-byte / per-nibble words
template <int F> __device__ __forceinline__ uint32_t code_at(const uint32_t* c, int i) {
    if constexpr (Fmt<F>::W == 4) return (c[i >> 3] >> (4 * (i & 7))) & 0xFu;
    else return (c[i >> 2] >> (8 * (i & 3))) & 0xFFu;
}

// VPL codes + block scale -> VPL output values packed as 16 bytes of T
template <int F, typename T, int VPL>
__device__ __forceinline__ uint4 decode_out(const uint32_t* c, uint32_t byte) {
    float v[VPL];
    float s = fwd_scale(byte);
#pragma unroll
    for (int i = 0; i < VPL; i += 2) decode2<F>(code_at<F>(c, i), code_at<F>(c, i + 1), s, v[i], v[i + 1]);
    uint32_t w[4];
    if constexpr (sizeof(T) == 4) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t b = __float_as_uint(v[i]);
            if constexpr (F == F_E4M3) b = ((code_at<F>(c, i) & 0x7Fu) == 0x7Fu) ? 0x7FC00000u : b;
            w[i] = byte == 0xFFu ? 0x7FC00000u : b;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t b = bf16x2(v[2 * i], v[2 * i + 1]);
            if constexpr (F == F_E4M3) {
                if ((code_at<F>(c, 2 * i) & 0x7Fu) == 0x7Fu) b = (b & 0xFFFF0000u) | 0x7FC0u;
                if ((code_at<F>(c, 2 * i + 1) & 0x7Fu) == 0x7Fu) b = (b & 0x0000FFFFu) | 0x7FC00000u;
            }
            w[i] = byte == 0xFFu ? 0x7FC07FC0u : b;
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

template <int F>
__device__ __forceinline__ void store_scale(void* scales, long long b, uint32_t byte) {
    if constexpr (Fmt<F>::FIXED) reinterpret_cast<uint16_t*>(scales)[b] = (uint16_t)byte;  // config = 0
    else reinterpret_cast<uint8_t*>(scales)[b] = (uint8_t)byte;
}
template <int F>
__device__ __forceinline__ uint32_t load_scale(const void* scales, long long b) {
    if constexpr (Fmt<F>::FIXED) return __ldg(reinterpret_cast<const uint16_t*>(scales) + b) & 0xFFu;
    else return __ldg(reinterpret_cast<const uint8_t*>(scales) + b);
}

// copy nbytes (multiple of 8) between global and the warp's staging slice
__device__ __forceinline__ void stage_out(uint8_t* g, const uint8_t* s, int nbytes, int lane) {
    for (int i = 16 * lane; i + 16 <= nbytes; i += 512) st_stream_v4(g + i, *reinterpret_cast<const uint4*>(s + i));
    if ((nbytes & 15) && lane == 0) {
        int i = nbytes & ~15;
        *reinterpret_cast<uint2*>(g + i) = *reinterpret_cast<const uint2*>(s + i);
    }
}
__device__ __forceinline__ void stage_in(uint8_t* s, const uint8_t* g, int nbytes, int lane) {
    for (int i = 16 * lane; i + 16 <= nbytes; i += 512) *reinterpret_cast<uint4*>(s + i) = ld_stream_v4(g + i);
    if ((nbytes & 15) && lane == 0) {
        int i = nbytes & ~15;
        *reinterpret_cast<uint2*>(s + i) = *reinterpret_cast<const uint2*>(g + i);
    }
}

template <int NSEG>
__device__ __forceinline__ int find_seg(const SegTable<NSEG>& tab, long long t) {
    int s = 0;
    if constexpr (NSEG > 1) {
        while (s + 1 < tab.n && t >= tab.seg[s + 1].tile0) ++s;
    }
    return s;
}

// ---------------------------------------------------------------------------

template <int F, typename T, int NSEG>
__global__ void __launch_bounds__(kWarps * 32) k_quantize(const __grid_constant__ SegTable<NSEG> tab) {
    using L = Lay<T>;
    constexpr int LB = L::VPL * Fmt<F>::W / 8;  // code bytes per lane per row
    constexpr int PB = payload<F>();
    __shared__ __align__(16) uint8_t stage[kWarps][32 * kU * LB];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t* st = stage[warp];
    for (long long t = (long long)blockIdx.x * kWarps + warp; t < tab.ntiles; t += (long long)gridDim.x * kWarps) {
        const Seg& g = tab.seg[find_seg(tab, t)];
        const long long tb = (t - g.tile0) * L::BPT;
        const int nvalid = (int)min((long long)L::BPT, g.nblocks - tb);
        const T* src = reinterpret_cast<const T*>(g.src) + tb * 32;
        uint4 v[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u)
            v[u] = (u * L::BPR + lane / L::LPB < nvalid) ? ld_stream_v4(src + (u * 32 + lane) * L::VPL)
                                                        : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            float x[L::VPL];
            uint32_t am = Widen<T>::run(v[u], x);
            uint32_t byte = block_byte<F, L::LPB>(am);
            apply_inv<L::VPL>(x, byte);
            encode_store<F, L::VPL>(x, byte == 0xFFu ? 0u : 0xFFFFFFFFu, st + (u * 32 + lane) * LB);
            const int blk = u * L::BPR + lane / L::LPB;
            if ((lane % L::LPB) == 0 && blk < nvalid) store_scale<F>(g.scales, tb + blk, byte);
        }
        __syncwarp();
        stage_out(reinterpret_cast<uint8_t*>(g.codes) + tb * PB, st, nvalid * PB, lane);
        __syncwarp();
    }
}

template <int F, typename T>
__global__ void __launch_bounds__(kWarps * 32) k_dequantize(const uint8_t* __restrict__ codes,
                                                            const void* __restrict__ scales,
                                                            T* __restrict__ dst, long long nblocks) {
    using L = Lay<T>;
    constexpr int LB = L::VPL * Fmt<F>::W / 8;
    constexpr int PB = payload<F>();
    __shared__ __align__(16) uint8_t stage[kWarps][32 * kU * LB];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint8_t* st = stage[warp];
    const long long ntiles = (nblocks + L::BPT - 1) / L::BPT;
    for (long long t = (long long)blockIdx.x * kWarps + warp; t < ntiles; t += (long long)gridDim.x * kWarps) {
        const long long tb = t * L::BPT;
        const int nvalid = (int)min((long long)L::BPT, nblocks - tb);
        stage_in(st, codes + tb * PB, nvalid * PB, lane);
        uint32_t bytes[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int blk = u * L::BPR + lane / L::LPB;
            bytes[u] = blk < nvalid ? load_scale<F>(scales, tb + blk) : 0u;
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int blk = u * L::BPR + lane / L::LPB;
            uint32_t c[2];
            load_codes<F, L::VPL>(st + (u * 32 + lane) * LB, c);
            uint4 o = decode_out<F, T, L::VPL>(c, bytes[u]);
            if (blk < nvalid) st_stream_v4(dst + (tb + 0) * 32 + (u * 32 + lane) * L::VPL, o);
        }
        __syncwarp();
    }
}

template <int F, typename T>
__global__ void __launch_bounds__(kWarps * 32) k_fake_quantize(const T* src, T* dst, long long nblocks) {
    using L = Lay<T>;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long ntiles = (nblocks + L::BPT - 1) / L::BPT;
    for (long long t = (long long)blockIdx.x * kWarps + warp; t < ntiles; t += (long long)gridDim.x * kWarps) {
        const long long tb = t * L::BPT;
        const int nvalid = (int)min((long long)L::BPT, nblocks - tb);
        const T* s = src + tb * 32;
        uint4 v[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u)
            v[u] = (u * L::BPR + lane / L::LPB < nvalid) ? ld_stream_v4(s + (u * 32 + lane) * L::VPL)
                                                        : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            float x[L::VPL];
            uint32_t am = Widen<T>::run(v[u], x);
            uint32_t byte = block_byte<F, L::LPB>(am);
            apply_inv<L::VPL>(x, byte);
            uint32_t c[2];
            encode<F, L::VPL>(x, c);
            uint4 o = decode_out<F, T, L::VPL>(c, byte);
            if (u * L::BPR + lane / L::LPB < nvalid) st_stream_v4(dst + tb * 32 + (u * 32 + lane) * L::VPL, o);
        }
    }
}

// ---------------------------------------------------------------------------
// launchers

// Persistent grid: resident CTAs per SM (occupancy query, cached per kernel and
// device) times the SM count, capped by the number of warp tiles.
static int resident_ctas(const void* fn, int dev) {
    struct Entry { const void* fn; int dev; int ctas; };
    static Entry cache[256];
    static int used = 0;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (cache[i].fn == fn && cache[i].dev == dev) return cache[i].ctas;
    int sms = 148, per_sm = 1;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kWarps * 32, 0);
    int ctas = sms * (per_sm > 0 ? per_sm : 1);
    if (used < 256) cache[used++] = {fn, dev, ctas};
    return ctas;
}

template <typename K>
static int grid_for(K kernel, long long ntiles) {
    int dev = 0;
    cudaGetDevice(&dev);
    long long cap = resident_ctas(reinterpret_cast<const void*>(kernel), dev);
    long long want = (ntiles + kWarps - 1) / kWarps;
    return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

template <int F, typename T, int NSEG>
static cudaError_t launch_q(const SegTable<NSEG>& tab, cudaStream_t st) {
    auto k = k_quantize<F, T, NSEG>;
    k<<<grid_for(k, tab.ntiles), kWarps * 32, 0, st>>>(tab);
    return cudaGetLastError();
}

template <int NSEG>
cudaError_t launch_quantize(int fmt, int dtype, SegTable<NSEG>& tab, cudaStream_t st) {
    const int bpt = dtype == 1 ? Lay<__nv_bfloat16>::BPT : Lay<float>::BPT;
    long long tiles = 0;
    for (int i = 0; i < tab.n; ++i) {
        tab.seg[i].tile0 = tiles;
        tiles += (tab.seg[i].nblocks + bpt - 1) / bpt;
    }
    tab.ntiles = tiles;
    if (tiles == 0) return cudaSuccess;
#define MXQ_Q(FF)                                                                     \
    case FF:                                                                          \
        return dtype == 1 ? launch_q<FF, __nv_bfloat16, NSEG>(tab, st) : launch_q<FF, float, NSEG>(tab, st);
    switch (fmt) {
        MXQ_Q(F_AXS6)
        MXQ_Q(F_E2M3)
        MXQ_Q(F_E3M2)
        MXQ_Q(F_E4M3)
        MXQ_Q(F_E2M1)
    }
#undef MXQ_Q
    return cudaErrorInvalidValue;
}
template cudaError_t launch_quantize<1>(int, int, SegTable<1>&, cudaStream_t);
template cudaError_t launch_quantize<kMaxSeg>(int, int, SegTable<kMaxSeg>&, cudaStream_t);

template <int F, typename T>
static cudaError_t launch_dq_t(const void* codes, const void* scales, void* dst, long long nb, cudaStream_t st) {
    auto k = k_dequantize<F, T>;
    long long tiles = (nb + Lay<T>::BPT - 1) / Lay<T>::BPT;
    k<<<grid_for(k, tiles), kWarps * 32, 0, st>>>(reinterpret_cast<const uint8_t*>(codes), scales,
                                                   reinterpret_cast<T*>(dst), nb);
    return cudaGetLastError();
}

cudaError_t launch_dequantize(int fmt, const void* codes, const void* scales, void* dst, int dtype, long long nb,
                              cudaStream_t st) {
#define MXQ_D(FF)                                                                      \
    case FF:                                                                           \
        return dtype == 1 ? launch_dq_t<FF, __nv_bfloat16>(codes, scales, dst, nb, st) \
                          : launch_dq_t<FF, float>(codes, scales, dst, nb, st);
    switch (fmt) {
        MXQ_D(F_AXS6)
        MXQ_D(F_E2M3)
        MXQ_D(F_E3M2)
        MXQ_D(F_E4M3)
        MXQ_D(F_E2M1)
    }
#undef MXQ_D
    return cudaErrorInvalidValue;
}

template <int F, typename T>
static cudaError_t launch_fq_t(const void* src, void* dst, long long nb, cudaStream_t st) {
    auto k = k_fake_quantize<F, T>;
    long long tiles = (nb + Lay<T>::BPT - 1) / Lay<T>::BPT;
    k<<<grid_for(k, tiles), kWarps * 32, 0, st>>>(reinterpret_cast<const T*>(src), reinterpret_cast<T*>(dst), nb);
    return cudaGetLastError();
}

cudaError_t launch_fake_quantize(int fmt, const void* src, void* dst, int dtype, long long nb, cudaStream_t st) {
#define MXQ_F(FF)                                                                  \
    case FF:                                                                       \
        return dtype == 1 ? launch_fq_t<FF, __nv_bfloat16>(src, dst, nb, st)       \
                          : launch_fq_t<FF, float>(src, dst, nb, st);
    switch (fmt) {
        MXQ_F(F_AXS6)
        MXQ_F(F_E2M3)
        MXQ_F(F_E3M2)
        MXQ_F(F_E4M3)
        MXQ_F(F_E2M1)
    }
#undef MXQ_F
    return cudaErrorInvalidValue;
}

}  // namespace mxq
