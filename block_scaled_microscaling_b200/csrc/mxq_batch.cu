// mxq_batch.cu -- several independent conversions in one launch (sm_100a).
//
// A batch is up to 64 quantize / dequantize / fake-quantize operations of any
// of the five formats on one value type: the tensors of a layer converted to
// the formats a per-module policy picked ("Sonar: Online MXFP6", Start a model
// and Select the FP6 encoding: E2M3 by default, E3M2 where range matters), or
// weights dequantized next to activations quantized. Every launch on B200 pays
// a fixed cost (launch, first DRAM round trip, drain of the last stores: about
// 1.5 us, a fifth of a 47 MB conversion); one launch for the whole batch pays
// it once and streams the operations back to back with no ramp between them.
//
// Work decomposition: the blocks of every operation are cut into warp tiles
// of 32 blocks (one block per lane, as in the single-operation kernels); the
// tiles of all operations are numbered consecutively and warps take them
// grid-stride, so at any moment the SMs work on one or two neighbouring
// operations. A warp finds its operation by a forward scan of the table (its
// tile numbers only increase) and dispatches on (kind, format) -- uniform
// across the warp, no divergence.
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mxq_block.cuh"
#include "mxq_device.cuh"
#include "mxq_internal.h"

namespace mxq {

constexpr int kBThreads = 256;
constexpr int kBWarps = kBThreads / 32;

template <int F, typename T>
__device__ __forceinline__ void tile_quantize(const BatchOp& op, long long first, int lane, uint8_t* stage) {
    const long long b = first + lane;
    const bool ok = b < op.nblocks;
    uint32_t w[Blk<T>::NW] = {};
    if (ok) load_block<T>(op.in, b, w, op.a32);
    const uint32_t byte = scale_byte<F>(block_amax<T>(w));
    uint32_t out[8];
    encode_block<F, T>(w, byte, out);
    if constexpr (Fmt<F>::W == 6) {
        warp_store6<F>(op.out, first, (int)min(32LL, op.nblocks - first), out, stage, lane);
    } else {
        if (ok) store_payload<F>(op.out, b, out, op.a32);
    }
    if (ok) store_scale<F>(op.scales_out, b, byte);
}

template <int F, typename T>
__device__ __forceinline__ void tile_dequantize(const BatchOp& op, long long first, int lane) {
    const long long b = first + lane;
    if (b >= op.nblocks) return;
    uint32_t pw[8];
    load_payload<F>(op.in, b, pw, op.a32);
    const uint32_t byte = load_scale<F>(op.scales_in, b);
    uint32_t o[Blk<T>::NW];
    decode_block<F, T>(pw, byte, o);
    store_block<T>(op.out, b, o, op.a32);
}

template <int F, typename T>
__device__ __forceinline__ void tile_fake_quantize(const BatchOp& op, long long first, int lane) {
    const long long b = first + lane;
    if (b >= op.nblocks) return;
    uint32_t w[Blk<T>::NW];
    load_block<T>(op.in, b, w, op.a32);
    const uint32_t byte = scale_byte<F>(block_amax<T>(w));
    uint32_t o[Blk<T>::NW];
    fake_block<F, T>(w, byte, o);
    store_block<T>(op.out, b, o, op.a32);
}

template <typename T>
__global__ void __launch_bounds__(kBThreads) k_batch(const __grid_constant__ BatchTable tab) {
    pdl_wait_then_release();
    __shared__ __align__(16) uint8_t stage[kBWarps][32 * 24];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const long long nwarps = (long long)gridDim.x * kBWarps;
    int o = 0;
    for (long long t = (long long)blockIdx.x * kBWarps + wid; t < tab.ntiles; t += nwarps) {
        while (o + 1 < tab.n && t >= tab.op[o + 1].tile0) ++o;
        const BatchOp& op = tab.op[o];
        const long long first = (t - op.tile0) * 32;
        switch (op.kind * 8 + op.fmt) {
#define MXQ_B(FF)                                                   \
    case FF: tile_quantize<FF, T>(op, first, lane, stage[wid]); break; \
    case 8 + FF: tile_dequantize<FF, T>(op, first, lane); break;      \
    case 16 + FF: tile_fake_quantize<FF, T>(op, first, lane); break;
            MXQ_B(F_AXS6)
            MXQ_B(F_E2M3)
            MXQ_B(F_E3M2)
            MXQ_B(F_E4M3)
            MXQ_B(F_E2M1)
#undef MXQ_B
            default: break;
        }
    }
}

cudaError_t launch_batch(int dtype, BatchTable& tab, cudaStream_t st) {
    long long tiles = 0;
    for (int i = 0; i < tab.n; ++i) {
        BatchOp& op = tab.op[i];
        if (op.kind < 0 || op.kind > 2 || op.fmt < F_AXS6 || op.fmt > F_E2M1) return cudaErrorInvalidValue;
        op.tile0 = tiles;
        tiles += (op.nblocks + 31) / 32;
    }
    tab.ntiles = tiles;
    if (tiles == 0) return cudaSuccess;
    const void* fn = dtype == 1 ? reinterpret_cast<const void*>(k_batch<__nv_bfloat16>)
                                : reinterpret_cast<const void*>(k_batch<float>);
    int dev = 0;
    cudaGetDevice(&dev);
    long long grid = resident_ctas(fn, dev);
    const long long want = (tiles + kBWarps - 1) / kBWarps;
    if (want < grid) grid = want;
    const cudaError_t e = dtype == 1 ? launch_pdl(k_batch<__nv_bfloat16>, (unsigned)grid, kBThreads, st, tab)
                                     : launch_pdl(k_batch<float>, (unsigned)grid, kBThreads, st, tab);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace mxq
