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

// 128 threads per CTA: finer grain at the end of a one-pass grid (47 MB single-operation
// quantize, fraction of the copy peak: E2M3 0.786 -> 0.803, E3M2 0.793 -> 0.810; larger sizes and
// the grouped decoder-layer launches unchanged)
constexpr int kThreads = 128;

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

// Per-kernel shape choices, picked by measurement on B200 (median of repeated
// graph timings over the five workloads): a thread keeps two blocks in flight
// only in the grouped FP6 quantize (decoder layers, ~100M values per launch:
// 0.92 vs 0.77-0.82 of HBM peak); one block elsewhere (a 47 MB launch loses
// ~5% with two: fewer, longer threads). Shared-memory staging of 6-bit stores
// helps single-tensor quantize (MXFP6 0.91 vs 0.79; AXS-6 0.90 vs 0.83 once its
// rounding was packed into 16-bit lanes) but not the grouped kernel.
template <int F, typename T, int NSEG> __host__ __device__ constexpr int q_unroll() {
    return (NSEG > 1 && Fmt<F>::W == 6 && !Fmt<F>::FIXED && sizeof(T) == 2) ? 2 : 1;
}
template <int F, typename T, int NSEG> __host__ __device__ constexpr bool q_stage() {
    return NSEG == 1 && Fmt<F>::W == 6;
}

// MMA: scales go to the block-scaled MMA tile layout (single tensor, E8M0 formats); a separate
// instantiation, so the plain and grouped kernels carry no trace of it.
template <int F, typename T, int NSEG, bool MMA = false>
__global__ void __launch_bounds__(kThreads) k_quantize(const __grid_constant__ SegTable<NSEG> tab) {
    pdl_wait_then_release();
    static_assert(!MMA || (NSEG == 1 && !Fmt<F>::FIXED), "tile-layout scales: one tensor, E8M0 format");
    constexpr int U = q_unroll<F, T, NSEG>();
    constexpr bool STAGE = q_stage<F, T, NSEG>();
    __shared__ __align__(16) uint8_t stage[STAGE ? kThreads / 32 : 1][STAGE ? 32 * 24 : 16];
    const int lane = threadIdx.x & 31;
    const long long stride = (long long)gridDim.x * kThreads;
    const long long N = tab.nblocks;
    // warp-uniform trip count: every lane of a warp takes the same iterations
    for (long long base = (long long)blockIdx.x * kThreads + (threadIdx.x & ~31); base < N; base += U * stride) {
        uint32_t w[U][Blk<T>::NW];
        const Seg* g[U];
        long long b[U];
        bool a32[U], ok[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long gb = base + u * stride + lane;
            ok[u] = gb < N;
            g[u] = &tab.seg[find_seg(tab, ok[u] ? gb : 0)];
            b[u] = gb - g[u]->blk0;
            a32[u] = ((reinterpret_cast<uintptr_t>(g[u]->src) | reinterpret_cast<uintptr_t>(g[u]->codes)) & 31) == 0;
            if (ok[u]) load_block<T>(g[u]->src, b[u], w[u], a32[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const uint32_t byte = scale_byte<F>(block_amax<T>(w[u]));
            uint32_t out[8];
            encode_block<F, T>(w[u], byte, out);
            if constexpr (STAGE) {
                // whole warp in one tensor: staged 16-byte stores; else per thread
                const long long first = base + u * stride;  // lane 0's block, warp-uniform
                const int nvalid = (int)min(32LL, N - first);
                const Seg* g0 = &tab.seg[find_seg(tab, first < N ? first : 0)];
                const bool same = __all_sync(0xFFFFFFFFu, !ok[u] || g[u] == g0);
                if (nvalid > 0 && same) {
                    warp_store6<F>(g0->codes, first - g0->blk0, nvalid, out, stage[threadIdx.x >> 5], lane);
                } else if (ok[u]) {
                    store_payload<F>(g[u]->codes, b[u], out, a32[u]);
                }
            } else {
                if (ok[u]) store_payload<F>(g[u]->codes, b[u], out, a32[u]);
            }
            if (ok[u]) {
                if constexpr (MMA)
                    reinterpret_cast<uint8_t*>(g[u]->scales)[mma_scale_offset(b[u], g[u]->kb_mma)] = (uint8_t)byte;
                else
                    store_scale<F>(g[u]->scales, b[u], byte);
            }
        }
    }
}

// COOP (6-bit formats): a warp's 32 payloads arrive as shared 16-byte loads through shared
// memory (warp_load6) instead of three 8-byte loads per thread, the scale load issued first so
// both are in flight together. Measured on B200 (bf16 out, MXFP6 E2M3): 0.93 vs 0.82 of the HBM
// copy peak at 373 MB per launch, but slower below about 190 MB (10.2 vs 8.3 us at 47 MB), so the
// launcher picks it by size.
template <int F, typename T, bool COOP = false>
__global__ void __launch_bounds__(kThreads) k_dequantize(const void* __restrict__ codes, const void* __restrict__ scales,
                                                         void* __restrict__ dst, long long nblocks, bool a32) {
    pdl_wait_then_release();
    if constexpr (COOP) {
        static_assert(Fmt<F>::W == 6, "24-byte payloads");
        __shared__ __align__(16) uint8_t stage[kThreads / 32][32 * 24];
        const int lane = threadIdx.x & 31;
        const long long stride = (long long)gridDim.x * kThreads;
        for (long long first = (long long)blockIdx.x * kThreads + (threadIdx.x & ~31); first < nblocks;
             first += stride) {  // warp-uniform trip count
            const int nvalid = (int)min(32LL, nblocks - first);
            const long long b = first + lane;
            const uint32_t byte = lane < nvalid ? load_scale<F>(scales, b) : 0u;
            uint32_t pw[8];
            warp_load6(codes, first, nvalid, pw, stage[threadIdx.x >> 5], lane);
            if (lane < nvalid) {
                uint32_t o[Blk<T>::NW];
                decode_block<F, T>(pw, byte, o);
                store_block<T>(dst, b, o, a32);
            }
        }
        return;
    }
    constexpr int U = 1;
    const long long stride = (long long)gridDim.x * kThreads;
    for (long long base = (long long)blockIdx.x * kThreads + threadIdx.x; base < nblocks; base += U * stride) {
        uint32_t pw[U][8];
        uint32_t byte[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long b = base + u * stride;
            if (b < nblocks) {
                load_payload<F>(codes, b, pw[u], a32);
                byte[u] = load_scale<F>(scales, b);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long b = base + u * stride;
            if (b < nblocks) {
                uint32_t o[Blk<T>::NW];
                decode_block<F, T>(pw[u], byte[u], o);
                store_block<T>(dst, b, o, a32);
            }
        }
    }
}

template <int F, typename T>
__global__ void __launch_bounds__(kThreads) k_fake_quantize(const void* src, void* dst, long long nblocks, bool a32) {
    pdl_wait_then_release();
    constexpr int U = 1;
    const long long stride = (long long)gridDim.x * kThreads;
    for (long long base = (long long)blockIdx.x * kThreads + threadIdx.x; base < nblocks; base += U * stride) {
        uint32_t w[U][Blk<T>::NW];
#pragma unroll
        for (int u = 0; u < U; ++u)
            if (base + u * stride < nblocks) load_block<T>(src, base + u * stride, w[u], a32);
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const long long b = base + u * stride;
            if (b < nblocks) {
                const uint32_t byte = scale_byte<F>(block_amax<T>(w[u]));
                uint32_t o[Blk<T>::NW];
                fake_block<F, T>(w[u], byte, o);
                store_block<T>(dst, b, o, a32);
            }
        }
    }
}

// ---------------------------------------------------------------------------
// launchers

// Resident CTAs per SM (occupancy query) times the SM count, cached per kernel and device.
int resident_ctas(const void* fn, int dev) {
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

// Two grid shapes, chosen per kernel by measurement on B200 (graphs of back-to-back launches
// on HBM-resident data, fraction of the copy peak):
//  - persistent (one_pass = false): SMs x resident CTAs, each thread walks its blocks
//    grid-stride, U at a time;
//  - one pass (one_pass = true): one CTA per kThreads blocks, each thread one block; the hardware
//    starts a new CTA wherever one finishes.
// Single-tensor quantize takes one pass at every size (bf16 16384x8192: MXFP6 0.90 -> 0.97,
// MXFP8 0.93 -> 1.04; bf16 4096x4096: 0.76 -> 0.78), and so do dequantize with per-thread
// payload loads above 2^21 blocks (MXFP8 16384x8192: 0.89 -> 1.01). Persistent stays where
// it measured better: the grouped quantize with two blocks in flight (decoder layer 0.92 vs
// 0.87), the batch kernel (0.91 vs 0.88), dequantize at 47 MB (E2M3 0.90 vs 0.87) and the
// warp-shared 6-bit dequantize (0.94 vs 0.88).
template <typename K>
static int grid_for(K kernel, long long nblocks, bool one_pass = false) {
    long long want = (nblocks + kThreads - 1) / kThreads;
    if (want < 1) want = 1;
    if (one_pass) return (int)(want < 0x7FFFFFFFLL ? want : 0x7FFFFFFFLL);
    int dev = 0;
    cudaGetDevice(&dev);
    const long long cap = resident_ctas(reinterpret_cast<const void*>(kernel), dev);
    return (int)(want < cap ? want : cap);
}

static bool aligned32(const void* a, const void* b) {
    return ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 31) == 0;
}

template <int F, typename T, int NSEG>
static cudaError_t launch_q(const SegTable<NSEG>& tab, cudaStream_t st) {
    auto k = k_quantize<F, T, NSEG>;
    if constexpr (NSEG == 1 && !Fmt<F>::FIXED) {
        if (tab.seg[0].kb_mma) k = k_quantize<F, T, 1, true>;
    } else {
        if (tab.seg[0].kb_mma) return cudaErrorInvalidValue;
    }
    const cudaError_t e = launch_pdl(k, (unsigned)grid_for(k, tab.nblocks, NSEG == 1), kThreads, st, tab);
    return e != cudaSuccess ? e : cudaGetLastError();
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
    bool coop = false;
    if constexpr (Fmt<F>::W == 6) coop = nb >= (1LL << 21);  // >= 64M values
    if (coop) k = k_dequantize<F, T, Fmt<F>::W == 6>;
    // programmatic launch only for the one-pass grid: with the persistent grid it measured slower
    // (E2M3 at 47 MB: 0.84 vs 0.89); there the kernel's griddepcontrol.wait is a no-op
    const bool one_pass = !coop && nb >= (1LL << 21);
    const unsigned grid = (unsigned)grid_for(k, nb, one_pass);
    if (one_pass) {
        const cudaError_t e = launch_pdl(k, grid, kThreads, st, codes, scales, dst, nb, aligned32(codes, dst));
        if (e != cudaSuccess) return e;
    } else {
        k<<<grid, kThreads, 0, st>>>(codes, scales, dst, nb, aligned32(codes, dst));
    }
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
