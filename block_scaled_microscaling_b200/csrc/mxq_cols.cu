// mxq_cols.cu -- column-direction blocks: 32 consecutive rows of one column
// share a scale (weights stored [in, out], backward-pass operands). The
// result is laid out as the row-direction quantization of the transpose:
// codes [cols, rows/32 * P] and scales [cols, rows/32], so a consumer reads
// each column's blocks contiguously.
//
// Tile: 256 rows x 32 columns. Loads: one thread per row, the row's 64 (bf16)
// or 128 (fp32) bytes as whole 32-byte sectors, into shared memory with 16-byte
// chunks permuted per row (conflict-free writes). Compute: warp w takes
// row-block w, lane j column j; all lanes read the same row at once (a
// permutation of one row: conflict-free). Payloads are staged per column and
// leave as contiguous runs of the column's row-blocks.
#include <cstdint>
#include <mutex>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mxq_block.cuh"
#include "mxq_device.cuh"
#include "mxq_internal.h"

namespace mxq {

constexpr int kColThreads = 256;
constexpr int kTileRows = 256;  // 8 row-blocks
constexpr int kTileCols = 32;

// byte offset of element (r, j) of the tile; rows of 32 * sizeof(T) bytes,
// chunk c of row r stored at c ^ sw(r)
template <typename T> __device__ __forceinline__ uint32_t tile_off(int r, int j) {
    if constexpr (sizeof(T) == 2) {
        const int c = j >> 3;  // 4 chunks of 8 values
        return (uint32_t)(r * 64 + 16 * (c ^ ((r >> 1) & 3)) + 2 * (j & 7));
    } else {
        const int c = j >> 2;  // 8 chunks of 4 values
        return (uint32_t)(r * 128 + 16 * (c ^ (r & 7)) + 4 * (j & 3));
    }
}

template <typename T>
__device__ __forceinline__ void tile_row_store(uint8_t* tile, int r, const uint32_t* w) {
    constexpr int NC = sizeof(T) == 2 ? 4 : 8;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int pos = sizeof(T) == 2 ? (c ^ ((r >> 1) & 3)) : (c ^ (r & 7));
        *reinterpret_cast<uint4*>(tile + r * 16 * NC + 16 * pos) = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
    }
}
template <typename T>
__device__ __forceinline__ void tile_row_load(const uint8_t* tile, int r, uint32_t* w) {
    constexpr int NC = sizeof(T) == 2 ? 4 : 8;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int pos = sizeof(T) == 2 ? (c ^ ((r >> 1) & 3)) : (c ^ (r & 7));
        const uint4 v = *reinterpret_cast<const uint4*>(tile + r * 16 * NC + 16 * pos);
        w[4 * c] = v.x;
        w[4 * c + 1] = v.y;
        w[4 * c + 2] = v.z;
        w[4 * c + 3] = v.w;
    }
}

// the 32 values of column j, rows 32*rb .. 32*rb+31, as the words of a block
// (bf16: two values per word, low half first; fp32: one per word)
template <typename T>
__device__ __forceinline__ void gather_column(const uint8_t* tile, int rb, int j, uint32_t* w) {
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const uint32_t lo = *reinterpret_cast<const uint16_t*>(tile + tile_off<T>(32 * rb + 2 * i, j));
            const uint32_t hi = *reinterpret_cast<const uint16_t*>(tile + tile_off<T>(32 * rb + 2 * i + 1, j));
            w[i] = lo | (hi << 16);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = *reinterpret_cast<const uint32_t*>(tile + tile_off<T>(32 * rb + i, j));
    }
}
template <typename T>
__device__ __forceinline__ void scatter_column(uint8_t* tile, int rb, int j, const uint32_t* o) {
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            *reinterpret_cast<uint16_t*>(tile + tile_off<T>(32 * rb + 2 * i, j)) = (uint16_t)o[i];
            *reinterpret_cast<uint16_t*>(tile + tile_off<T>(32 * rb + 2 * i + 1, j)) = (uint16_t)(o[i] >> 16);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) *reinterpret_cast<uint32_t*>(tile + tile_off<T>(32 * rb + i, j)) = o[i];
    }
}

// grid: (column strips, row chunks); rows % 32 == 0, cols % 32 == 0
template <int F, typename T>
__global__ void __launch_bounds__(kColThreads) k_quantize_cols(const void* __restrict__ src, void* __restrict__ codes,
                                                              void* __restrict__ scales, long long rows, long long cols) {
    constexpr int PB = payload<F>();
    constexpr int SB = Fmt<F>::FIXED ? 2 : 1;
    __shared__ __align__(16) uint8_t tile[kTileRows * kTileCols * sizeof(T)];
    __shared__ __align__(16) uint8_t out[kTileCols * 8 * PB];
    __shared__ __align__(16) uint8_t sc[kTileCols * 8 * SB];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const long long RB = rows / 32;
    const long long col0 = (long long)blockIdx.x * kTileCols;
    const long long row0 = (long long)blockIdx.y * kTileRows;
    const int nrows = (int)min((long long)kTileRows, rows - row0);
    const int nrb = nrows / 32;
    const bool a32 = ((reinterpret_cast<uintptr_t>(src) | (uintptr_t)(cols * sizeof(T))) & 31) == 0;
    if (t < nrows) {
        uint32_t w[8 * sizeof(T)];
        const char* p = reinterpret_cast<const char*>(src) + ((row0 + t) * cols + col0) * (long long)sizeof(T);
#pragma unroll
        for (int i = 0; i < (int)sizeof(T); ++i) ld32(p + 32 * i, w + 8 * i, a32);  // 32 * sizeof(T) bytes
        tile_row_store<T>(tile, t, w);
    }
    __syncthreads();
    if (warp < nrb) {
        uint32_t w[Blk<T>::NW];
        gather_column<T>(tile, warp, lane, w);
        const uint32_t byte = scale_byte<F>(block_amax<T>(w));
        uint32_t o[8];
        encode_block<F, T>(w, byte, o);
        uint32_t* q = reinterpret_cast<uint32_t*>(out + (lane * 8 + warp) * PB);
#pragma unroll
        for (int i = 0; i < PB / 4; ++i) q[i] = o[i];
        if constexpr (SB == 2) reinterpret_cast<uint16_t*>(sc)[lane * 8 + warp] = (uint16_t)byte;
        else sc[lane * 8 + warp] = (uint8_t)byte;
    }
    __syncthreads();
    // column j's row-blocks of this chunk are contiguous in the output: nrb * PB bytes
    const int seg = nrb * PB;
    for (int i = t; i < kTileCols * (seg / 8); i += kColThreads) {
        const int j = i / (seg / 8), k = i % (seg / 8);
        const long long g = ((col0 + j) * RB + blockIdx.y * 8) * PB + 8 * k;
        *reinterpret_cast<uint2*>(reinterpret_cast<char*>(codes) + g) = *reinterpret_cast<const uint2*>(out + j * 8 * PB + 8 * k);
    }
    for (int i = t; i < kTileCols * nrb; i += kColThreads) {
        const int j = i / nrb, k = i % nrb;
        const long long g = (col0 + j) * RB + blockIdx.y * 8 + k;
        if constexpr (SB == 2) reinterpret_cast<uint16_t*>(scales)[g] = reinterpret_cast<const uint16_t*>(sc)[j * 8 + k];
        else reinterpret_cast<uint8_t*>(scales)[g] = sc[j * 8 + k];
    }
}

template <int F, typename T>
__global__ void __launch_bounds__(kColThreads) k_dequantize_cols(const void* __restrict__ codes,
                                                                const void* __restrict__ scales, void* __restrict__ dst,
                                                                long long rows, long long cols) {
    constexpr int PB = payload<F>();
    __shared__ __align__(16) uint8_t tile[kTileRows * kTileCols * sizeof(T)];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const long long RB = rows / 32;
    const long long col0 = (long long)blockIdx.x * kTileCols;
    const long long row0 = (long long)blockIdx.y * kTileRows;
    const int nrows = (int)min((long long)kTileRows, rows - row0);
    const int nrb = nrows / 32;
    const bool a32 = ((reinterpret_cast<uintptr_t>(dst) | (uintptr_t)(cols * sizeof(T))) & 31) == 0;
    if (warp < nrb) {
        const long long b = (col0 + lane) * RB + blockIdx.y * 8 + warp;  // block of the transposed layout
        uint32_t pw[8];
        load_payload<F>(codes, b, pw, false);
        const uint32_t byte = load_scale<F>(scales, b);
        uint32_t o[Blk<T>::NW];
        decode_block<F, T>(pw, byte, o);
        scatter_column<T>(tile, warp, lane, o);
    }
    __syncthreads();
    if (t < nrows) {
        uint32_t w[8 * sizeof(T)];
        tile_row_load<T>(tile, t, w);
        char* p = reinterpret_cast<char*>(dst) + ((row0 + t) * cols + col0) * (long long)sizeof(T);
#pragma unroll
        for (int i = 0; i < (int)sizeof(T); ++i) st32(p + 32 * i, w + 8 * i, a32);
    }
}

template <int F, typename T>
static cudaError_t launch_qc_t(const void* src, void* codes, void* scales, long long rows, long long cols,
                               cudaStream_t st) {
    dim3 grid((unsigned)(cols / kTileCols), (unsigned)((rows + kTileRows - 1) / kTileRows));
    k_quantize_cols<F, T><<<grid, kColThreads, 0, st>>>(src, codes, scales, rows, cols);
    return cudaGetLastError();
}
template <int F, typename T>
static cudaError_t launch_dqc_t(const void* codes, const void* scales, void* dst, long long rows, long long cols,
                                cudaStream_t st) {
    dim3 grid((unsigned)(cols / kTileCols), (unsigned)((rows + kTileRows - 1) / kTileRows));
    k_dequantize_cols<F, T><<<grid, kColThreads, 0, st>>>(codes, scales, dst, rows, cols);
    return cudaGetLastError();
}

bool cols_grid_ok(long long rows, long long cols) {
    return cols / kTileCols <= 0x7FFFFFFFLL && (rows + kTileRows - 1) / kTileRows <= 65535;
}

cudaError_t launch_quantize_cols(int fmt, const void* src, int dtype, long long rows, long long cols, void* codes,
                                 void* scales, cudaStream_t st) {
#define MXQ_QC(FF)                                                                              \
    case FF:                                                                                    \
        return dtype == 1 ? launch_qc_t<FF, __nv_bfloat16>(src, codes, scales, rows, cols, st) \
                          : launch_qc_t<FF, float>(src, codes, scales, rows, cols, st);
    switch (fmt) {
        MXQ_QC(F_AXS6)
        MXQ_QC(F_E2M3)
        MXQ_QC(F_E3M2)
        MXQ_QC(F_E4M3)
        MXQ_QC(F_E2M1)
    }
#undef MXQ_QC
    return cudaErrorInvalidValue;
}

cudaError_t launch_dequantize_cols(int fmt, const void* codes, const void* scales, void* dst, int dtype, long long rows,
                                   long long cols, cudaStream_t st) {
#define MXQ_DQC(FF)                                                                              \
    case FF:                                                                                     \
        return dtype == 1 ? launch_dqc_t<FF, __nv_bfloat16>(codes, scales, dst, rows, cols, st) \
                          : launch_dqc_t<FF, float>(codes, scales, dst, rows, cols, st);
    switch (fmt) {
        MXQ_DQC(F_AXS6)
        MXQ_DQC(F_E2M3)
        MXQ_DQC(F_E3M2)
        MXQ_DQC(F_E4M3)
        MXQ_DQC(F_E2M1)
    }
#undef MXQ_DQC
    return cudaErrorInvalidValue;
}

}  // namespace mxq
