// mxq_stream.cu -- bulk-copy (TMA engine) streaming form of the fused
// fake-quantize (sm_100a).
//
// "AXS-6: Adaptive eXponent Sharing", Quick Start Example: quantize then
// dequantize in one pass with no intermediate allocation. The kernel moves
// the values with the TMA engine instead of per-thread loads and stores:
// plain 256-bit loads and stores issued by every thread leave the load/store
// unit queue full (LSU throttle) short of the HBM copy rate, while bulk copies
// reach it.
//
// One persistent CTA per SM. A tile is 32·CW blocks of 32 values (one block per
// consumer thread). One producer thread streams tiles into a ring of NS
// shared-memory stages (cp.async.bulk global -> shared, "full" mbarrier per
// stage, L = NS/2 tiles ahead); CW consumer warps fake-quantize each block in
// place in shared memory and signal a "done" mbarrier; the producer then writes
// the stage back (cp.async.bulk shared -> global, bulk groups) and reuses it
// once that store has read it (cp.async.bulk.wait_group.read). Each value is
// read and written once, by the copy engine.
//
// Shared-memory reads and writes of a block (64 or 128 bytes per thread) go in
// 16-byte pieces in a lane-rotated order, so that the lanes sharing a
// wavefront hit different bank groups; fake-quantize maps each value to its own
// position, so the pieces go back where they came from.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mxq_block.cuh"
#include "mxq_device.cuh"
#include "mxq_internal.h"
#include "mxq_tma.cuh"

namespace mxq {

template <int F, typename T, int CW, int NS>
__global__ void __launch_bounds__(32 * (CW + 1)) k_fake_quantize_stream(const void* src, void* dst, long long nblocks,
                                                                      unsigned int* err) {
    constexpr int BB = 32 * (int)sizeof(T);  // bytes per block
    constexpr int P = BB / 16;               // 16-byte pieces per block
    constexpr int TB = 32 * CW;              // blocks per tile
    constexpr int TILE = TB * BB;
    constexpr int L = NS / 2;                // tiles loaded ahead; NS - L stores in flight
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) unsigned long long full[NS], done[NS];
    __shared__ int abort_flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long G = gridDim.x, ntiles = (nblocks + TB - 1) / TB;
    const long long my = ntiles > (long long)blockIdx.x ? (ntiles - 1 - blockIdx.x) / G + 1 : 0;
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&done[s]), CW);
        }
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (my == 0) return;
    volatile int* ab = &abort_flag;
    const uint32_t ring0 = smem_u32(ring);
    auto tile_blocks = [&](long long i) { return (int)min((long long)TB, nblocks - (blockIdx.x + i * G) * TB); };

    if (warp == CW) {  // producer: loads and stores
        if (lane != 0) return;
        const unsigned long long strm = l2_policy_stream();
        auto load = [&](long long i) {
            const int s = (int)(i % NS);
            const uint32_t bytes = (uint32_t)(tile_blocks(i) * BB);
            mbar_expect_tx(smem_u32(&full[s]), bytes);
            bulk_load(ring0 + s * TILE, static_cast<const char*>(src) + (blockIdx.x + i * G) * TILE, bytes,
                      smem_u32(&full[s]), strm);
        };
        long long i = 0;
        for (; i < L && i < my; ++i) load(i);
        long long issued = i;
        bool ok = true;
        for (i = 0; i < my; ++i) {
            const int s = (int)(i % NS);
            if (!(ok = mbar_wait(smem_u32(&done[s]), (uint32_t)(i / NS) & 1u, ab, err))) break;
            bulk_store(static_cast<char*>(dst) + (blockIdx.x + i * G) * TILE, ring0 + s * TILE,
                       (uint32_t)(tile_blocks(i) * BB));
            bulk_commit();
            bulk_wait_read<NS - L - 1>();  // the store of tile i + L - NS has read its stage
            if (i + L < my) {
                load(i + L);
                issued = i + L + 1;
            }
        }
        bulk_wait_all();
        if (!ok) {
            // gave up: let the loads still in flight land before the CTA's shared memory goes away
            for (long long q = i; q < issued; ++q) {
                const uint32_t bar = smem_u32(&full[q % NS]), par = (uint32_t)(q / NS) & 1u;
                const unsigned long long t0 = global_ns();
                while (!mbar_test(bar, par) && global_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        return;
    }

    // consumers: thread tid owns block tid of each tile
    const int rot = sizeof(T) == 4 ? (tid & 7) : ((tid >> 1) & 3);
    for (long long i = 0; i < my; ++i) {
        const int s = (int)(i % NS);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&full[s]), (uint32_t)(i / NS) & 1u, ab, err))) return;
        if (tid < tile_blocks(i)) {
            const uint32_t base = ring0 + s * TILE + tid * BB;
            uint32_t w[Blk<T>::NW];
#pragma unroll
            for (int c = 0; c < P; ++c) {
                const uint4 v = lds128u(base + 16 * ((c + rot) % P));
                w[4 * c] = v.x;
                w[4 * c + 1] = v.y;
                w[4 * c + 2] = v.z;
                w[4 * c + 3] = v.w;
            }
            const uint32_t byte = scale_byte<F>(block_amax<T>(w));
            uint32_t o[Blk<T>::NW];
            fake_block<F, T>(w, byte, o);
#pragma unroll
            for (int c = 0; c < P; ++c) sts128(base + 16 * ((c + rot) % P), o[4 * c], o[4 * c + 1], o[4 * c + 2], o[4 * c + 3]);
            fence_proxy_async();  // the bulk store that reads these bytes is issued by another thread
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&done[s]));
    }
}

// 8 consumer warps (tiles of 256 blocks: 32 KB fp32, 16 KB bf16), 6 stages
constexpr int kSWarps = 8, kSStages = 6;

template <int F, typename T>
static cudaError_t launch_fqs_t(const void* src, void* dst, long long nb, cudaStream_t st) {
    auto kern = k_fake_quantize_stream<F, T, kSWarps, kSStages>;
    const int smem = kSStages * 32 * kSWarps * 32 * (int)sizeof(T), threads = 32 * (kSWarps + 1);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    unsigned int* err = nullptr;
    if ((e = device_error_word(&err)) != cudaSuccess) return e;
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    const long long tiles = (nb + 32 * kSWarps - 1) / (32 * kSWarps);
    long long ctas = (long long)sms * (per_sm > 0 ? per_sm : 1);
    if (ctas > tiles) ctas = tiles;
    kern<<<(unsigned)ctas, threads, smem, st>>>(src, dst, nb, err);
    return cudaGetLastError();
}

cudaError_t launch_fake_quantize_stream(int fmt, const void* src, void* dst, int dtype, long long nb,
                                        cudaStream_t st) {
    if (nb == 0) return cudaSuccess;
#define MXQ_FS(FF)                                                                \
    case FF:                                                                      \
        return dtype == 1 ? launch_fqs_t<FF, __nv_bfloat16>(src, dst, nb, st)     \
                          : launch_fqs_t<FF, float>(src, dst, nb, st);
    switch (fmt) {
        MXQ_FS(F_AXS6)
        MXQ_FS(F_E2M3)
        MXQ_FS(F_E3M2)
        MXQ_FS(F_E4M3)
        MXQ_FS(F_E2M1)
    }
#undef MXQ_FS
    return cudaErrorInvalidValue;
}

}  // namespace mxq
