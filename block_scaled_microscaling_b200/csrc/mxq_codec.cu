// mxq_codec.cu -- quantize / dequantize / fused fake-quantize kernels (sm_100a).
//
// Data layout: [rows, cols] row-major with cols % 32 == 0, so the blocks of 32
// values are the consecutive 32-value groups of the flat array; a kernel
// walks blocks, not rows ("AXS-6: Adaptive eXponent Sharing", block figure;
// "Sonar: Online MXFP6", Start a model: one E8M0 scale per block of 32).
//
// Work decomposition: one thread owns one block of 32 values at a time.
//   * values move in 32-byte (one DRAM sector) accesses: a bf16 block is 2 of
//     them, an fp32 block 4 (256-bit ld/st on sm_100; two 128-bit halves when a
//     pointer is only 16-byte aligned);
//   * the block maximum is a NaN-propagating max of |x| over packed pairs
//     (max.NaN.xorsign.abs), the scale byte integer arithmetic on its exponent;
//   * x * 2^-Es is a packed fp32x2 multiply, rounding the sm_100a conversion
//     instruction (two values per instruction), packing shifts and integer
//     multiply-adds; a block's payload (16/24/32 bytes) leaves in 8/16/32-byte
//     stores, its scale in one byte (two for AXS-6);
//   * grid-stride loop over blocks on a grid of SMs x resident CTAs.
// Grouped quantize runs the same kernel over a table of tensors (kernel
// parameter); a thread finds its tensor by a linear scan of the table.
#include <cstdint>
#include <mutex>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mxq_block.cuh"
#include "mxq_device.cuh"
#include "mxq_internal.h"

namespace mxq {

constexpr int kThreads = 256;

template <int NSEG>
__device__ __forceinline__ int find_seg(const SegTable<NSEG>& tab, long long b) {
    int s = 0;
    if constexpr (NSEG > 1) {
        while (s + 1 < tab.n && b >= tab.seg[s + 1].blk0) ++s;
    }
    return s;
}

// ---------------------------------------------------------------------------
// kernels

template <int F, typename T, int NSEG>
__global__ void __launch_bounds__(kThreads) k_quantize(const __grid_constant__ SegTable<NSEG> tab) {
    const long long stride = (long long)gridDim.x * kThreads;
    for (long long gb = (long long)blockIdx.x * kThreads + threadIdx.x; gb < tab.nblocks; gb += stride) {
        const Seg& g = tab.seg[find_seg(tab, gb)];
        const long long b = gb - g.blk0;
        const bool a32 = ((reinterpret_cast<uintptr_t>(g.src) | reinterpret_cast<uintptr_t>(g.codes)) & 31) == 0;
        uint32_t w[Blk<T>::NW];
        load_block<T>(g.src, b, w, a32);
        const uint32_t byte = scale_byte<F>(block_amax<T>(w));
        uint32_t out[8];
        encode_block<F, T>(w, byte, out);
        store_payload<F>(g.codes, b, out, a32);
        store_scale<F>(g.scales, b, byte);
    }
}

template <int F, typename T>
__global__ void __launch_bounds__(kThreads) k_dequantize(const void* __restrict__ codes, const void* __restrict__ scales,
                                                         void* __restrict__ dst, long long nblocks, bool a32) {
    const long long stride = (long long)gridDim.x * kThreads;
    for (long long b = (long long)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride) {
        uint32_t pw[8];
        load_payload<F>(codes, b, pw, a32);
        const uint32_t byte = load_scale<F>(scales, b);
        uint32_t o[Blk<T>::NW];
        decode_block<F, T>(pw, byte, o);
        store_block<T>(dst, b, o, a32);
    }
}

template <int F, typename T>
__global__ void __launch_bounds__(kThreads) k_fake_quantize(const void* src, void* dst, long long nblocks, bool a32) {
    const long long stride = (long long)gridDim.x * kThreads;
    for (long long b = (long long)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride) {
        uint32_t w[Blk<T>::NW];
        load_block<T>(src, b, w, a32);
        const uint32_t byte = scale_byte<F>(block_amax<T>(w));
        uint32_t o[Blk<T>::NW];
        fake_block<F, T>(w, byte, o);
        store_block<T>(dst, b, o, a32);
    }
}

// ---------------------------------------------------------------------------
// launchers

// Resident CTAs per SM (occupancy query) times the SM count, cached per kernel and device.
static int resident_ctas(const void* fn, int dev) {
    struct Entry { const void* fn; int dev; int ctas; };
    static Entry cache[512];
    static int used = 0;
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (cache[i].fn == fn && cache[i].dev == dev) return cache[i].ctas;
    int sms = 148, per_sm = 1;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, 0);
    int ctas = sms * (per_sm > 0 ? per_sm : 1);
    if (used < 512) cache[used++] = {fn, dev, ctas};
    return ctas;
}

template <typename K>
static int grid_for(K kernel, long long nblocks) {
    int dev = 0;
    cudaGetDevice(&dev);
    long long cap = resident_ctas(reinterpret_cast<const void*>(kernel), dev);
    long long want = (nblocks + kThreads - 1) / kThreads;
    return (int)(want < cap ? (want > 0 ? want : 1) : cap);
}

static bool aligned32(const void* a, const void* b) {
    return ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 31) == 0;
}

template <int F, typename T, int NSEG>
static cudaError_t launch_q(const SegTable<NSEG>& tab, cudaStream_t st) {
    auto k = k_quantize<F, T, NSEG>;
    k<<<grid_for(k, tab.nblocks), kThreads, 0, st>>>(tab);
    return cudaGetLastError();
}

// blk0 of each tensor = its first block in the concatenated block space; nblocks = all blocks
template <int NSEG>
cudaError_t launch_quantize(int fmt, int dtype, SegTable<NSEG>& tab, cudaStream_t st) {
    long long blocks = 0;
    for (int i = 0; i < tab.n; ++i) {
        tab.seg[i].blk0 = blocks;
        blocks += tab.seg[i].nblocks;
    }
    tab.nblocks = blocks;
    if (blocks == 0) return cudaSuccess;
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
    k<<<grid_for(k, nb), kThreads, 0, st>>>(codes, scales, dst, nb, aligned32(codes, dst));
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
    k<<<grid_for(k, nb), kThreads, 0, st>>>(src, dst, nb, aligned32(src, dst));
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
