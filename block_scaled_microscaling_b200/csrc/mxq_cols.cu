// mxq_cols.cu -- column-direction blocks: 32 consecutive rows of one column
// share a scale (weights stored [in, out], backward-pass operands). The
// result is laid out as the row-direction quantization of the transpose:
// codes [cols, rows/32 * P] and scales [cols, rows/32], so a consumer reads
// each column's blocks contiguously.
//
// Tile: 256 rows x 128 bytes (64 bf16 or 32 fp32 columns; the last strip of a
// bf16 matrix may be 32 columns wide). Loads: one thread per row, the row's
// bytes as whole 32-byte sectors, into shared memory with the 16-byte chunk c
// of row r at chunk index c ^ (r mod 8) (conflict-free writes). Compute: warp w
// takes row-block w, lane l the CPL = 128 / (32 * sizeof(T)) columns l*CPL ..;
// for a row, the 32 lanes read one 4-byte word each (all 128 bytes of the row:
// conflict-free), and for bf16 a byte permute splits each word into the two
// columns. Payloads and scales are staged per column (in the tile's memory,
// once its values are in registers) and leave as contiguous runs of the
// column's row-blocks.
#include <cstdint>
#include <mutex>
#include <cuda.h>  // CUtensorMap and its enums (types only: the encoder is fetched through the runtime)
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "mxq_block.cuh"
#include "mxq_device.cuh"
#include "mxq_internal.h"
#include "mxq_tma.cuh"

namespace mxq {

constexpr int kColThreads = 256;
constexpr int kTileRows = 256;  // 8 row-blocks
constexpr int kRowBytes = 128;  // bytes of a tile row

template <typename T> struct ColTile {
    static constexpr int TC = kRowBytes / (int)sizeof(T);  // columns per tile
    static constexpr int CPL = TC / 32;                     // columns per lane
};

// byte offset of 4-byte word q (0..31) of tile row r
__device__ __forceinline__ uint32_t word_off(int r, int q) {
    return (uint32_t)(r * kRowBytes + 16 * ((q >> 2) ^ (r & 7)) + 4 * (q & 3));
}

// row r of the tile from / to registers, 16 bytes per chunk, the first nch chunks
__device__ __forceinline__ void tile_row_store(uint8_t* tile, int r, const uint32_t* w, int nch) {
#pragma unroll
    for (int c = 0; c < 8; ++c)
        if (c < nch)
            *reinterpret_cast<uint4*>(tile + r * kRowBytes + 16 * (c ^ (r & 7))) =
                make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
}
__device__ __forceinline__ void tile_row_load(const uint8_t* tile, int r, uint32_t* w, int nch) {
#pragma unroll
    for (int c = 0; c < 8; ++c)
        if (c < nch) {
            const uint4 v = *reinterpret_cast<const uint4*>(tile + r * kRowBytes + 16 * (c ^ (r & 7)));
            w[4 * c] = v.x;
            w[4 * c + 1] = v.y;
            w[4 * c + 2] = v.z;
            w[4 * c + 3] = v.w;
        }
}

// The CPL blocks of lane `lane`'s columns in row-block rb: block k holds column lane*CPL + k,
// as the words of a block (bf16: two values per word, low half first; fp32: one per word).
// Within a row-block the swizzle phase r mod 8 is a compile-time value in the unrolled loops.
template <typename T>
__device__ __forceinline__ void gather_columns(const uint8_t* tile, int rb, int lane, uint32_t (*w)[Blk<T>::NW]) {
    const uint8_t* base = tile + rb * 32 * kRowBytes;
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {  // rows 2i, 2i + 1: columns 2 lane, 2 lane + 1 share a word
            const uint32_t a = *reinterpret_cast<const uint32_t*>(base + word_off(2 * i, lane));
            const uint32_t b = *reinterpret_cast<const uint32_t*>(base + word_off(2 * i + 1, lane));
            w[0][i] = __byte_perm(a, b, 0x5410);
            w[1][i] = __byte_perm(a, b, 0x7632);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) w[0][i] = *reinterpret_cast<const uint32_t*>(base + word_off(i, lane));
    }
}
template <typename T>
__device__ __forceinline__ void scatter_columns(uint8_t* tile, int rb, int lane, const uint32_t (*o)[Blk<T>::NW]) {
    uint8_t* base = tile + rb * 32 * kRowBytes;
    if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            *reinterpret_cast<uint32_t*>(base + word_off(2 * i, lane)) = __byte_perm(o[0][i], o[1][i], 0x5410);
            *reinterpret_cast<uint32_t*>(base + word_off(2 * i + 1, lane)) = __byte_perm(o[0][i], o[1][i], 0x7632);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) *reinterpret_cast<uint32_t*>(base + word_off(i, lane)) = o[0][i];
    }
}

// grid: (column strips of TC, row chunks of 256); rows % 32 == 0, cols % 32 == 0
template <int F, typename T>
__global__ void __launch_bounds__(kColThreads) k_quantize_cols(const void* __restrict__ src, void* __restrict__ codes,
                                                              void* __restrict__ scales, long long rows, long long cols) {
    constexpr int TC = ColTile<T>::TC, CPL = ColTile<T>::CPL;
    constexpr int PB = payload<F>();
    constexpr int SB = Fmt<F>::FIXED ? 2 : 1;
    constexpr int CS = 8 * PB + 8;  // column stride of the staged payloads: 8 bytes of padding keep the
                                    // lanes (one column each) on different bank pairs
    static_assert(TC * CS + TC * 8 * SB <= kTileRows * kRowBytes, "staging fits in the tile");
    __shared__ __align__(16) uint8_t tile[kTileRows * kRowBytes];
    uint8_t* const out = tile;                // staged payloads and scales reuse the tile once
    uint8_t* const sc = tile + TC * CS;       // every warp has gathered its columns
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const long long RB = rows / 32;
    const long long col0 = (long long)blockIdx.x * TC;
    const long long row0 = (long long)blockIdx.y * kTileRows;
    const int nrows = (int)min((long long)kTileRows, rows - row0);
    const int nrb = nrows / 32;
    const int ncols = (int)min((long long)TC, cols - col0);
    const int rowbytes = ncols * (int)sizeof(T);  // 64 or 128
    const bool a32 = ((reinterpret_cast<uintptr_t>(src) | (uintptr_t)(cols * sizeof(T))) & 31) == 0;
    if (t < nrows) {
        uint32_t w[32];
        const char* p = reinterpret_cast<const char*>(src) + ((row0 + t) * cols + col0) * (long long)sizeof(T);
#pragma unroll
        for (int i = 0; i < 4; ++i)
            if (32 * i < rowbytes) ld32(p + 32 * i, w + 8 * i, a32);
        tile_row_store(tile, t, w, rowbytes / 16);
    }
    __syncthreads();
    uint32_t w[CPL][Blk<T>::NW];
    if (warp < nrb) gather_columns<T>(tile, warp, lane, w);
    __syncthreads();  // the tile's bytes are in registers: its memory takes the staged outputs
    if (warp < nrb) {
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
            const int j = lane * CPL + k;  // column within the strip
            if (j < ncols) {
                const uint32_t byte = scale_byte<F>(block_amax<T>(w[k]));
                uint32_t o[8];
                encode_block<F, T>(w[k], byte, o);
                uint32_t* q = reinterpret_cast<uint32_t*>(out + j * CS + warp * PB);
#pragma unroll
                for (int i = 0; i < PB / 4; ++i) q[i] = o[i];
                if constexpr (SB == 2) reinterpret_cast<uint16_t*>(sc)[j * 8 + warp] = (uint16_t)byte;
                else sc[j * 8 + warp] = (uint8_t)byte;
            }
        }
    }
    __syncthreads();
    // column j's row-blocks of this chunk are contiguous in the output: nrb * PB bytes
    if (nrb == 8 && ncols == TC) {  // full tile: compile-time strides
        constexpr int SEG8 = PB;    // 8-byte pieces per column (8 row-blocks x PB bytes / 8)
#pragma unroll
        for (int i = t; i < TC * SEG8; i += kColThreads) {
            const int j = i / SEG8, k = i % SEG8;
            const long long g = ((col0 + j) * RB + blockIdx.y * 8) * PB + 8 * k;
            *reinterpret_cast<uint2*>(reinterpret_cast<char*>(codes) + g) = *reinterpret_cast<const uint2*>(out + j * CS + 8 * k);
        }
#pragma unroll
        for (int i = t; i < TC * 8; i += kColThreads) {
            const int j = i >> 3, k = i & 7;
            const long long g = (col0 + j) * RB + blockIdx.y * 8 + k;
            if constexpr (SB == 2) reinterpret_cast<uint16_t*>(scales)[g] = reinterpret_cast<const uint16_t*>(sc)[j * 8 + k];
            else reinterpret_cast<uint8_t*>(scales)[g] = sc[j * 8 + k];
        }
        return;
    }
    const int seg8 = nrb * PB / 8;
    for (int i = t; i < ncols * seg8; i += kColThreads) {
        const int j = i / seg8, k = i % seg8;
        const long long g = ((col0 + j) * RB + blockIdx.y * 8) * PB + 8 * k;
        *reinterpret_cast<uint2*>(reinterpret_cast<char*>(codes) + g) = *reinterpret_cast<const uint2*>(out + j * CS + 8 * k);
    }
    for (int i = t; i < ncols * nrb; i += kColThreads) {
        const int j = i / nrb, k = i % nrb;
        const long long g = (col0 + j) * RB + blockIdx.y * 8 + k;
        if constexpr (SB == 2) reinterpret_cast<uint16_t*>(scales)[g] = reinterpret_cast<const uint16_t*>(sc)[j * 8 + k];
        else reinterpret_cast<uint8_t*>(scales)[g] = sc[j * 8 + k];
    }
}

// ---- quantize, persistent and fed by the tensor-copy engine ---------------------------------------
//
// The same tile and the same compute as k_quantize_cols, but each CTA walks its tiles (tile
// blockIdx.x + n * gridDim.x) with two tile buffers: a 2-D tensor copy (cp.async.bulk.tensor,
// 256 rows x 128 bytes, 128-byte swizzle) brings tile n + 2 while tile n + 1 waits and tile n is
// encoded. The 128-byte swizzle stores 16-byte chunk c of tile row r at chunk c ^ (r mod 8) of a
// 1024-byte-aligned buffer: exactly the layout gather_columns reads. No wave tail (a one-shot
// grid of 256-row tiles covered 1.38 waves at 4096 x 4096) and no per-thread load instructions.
// Waits are bounded (the library's device error word); on a timeout every thread leaves the
// loop together and thread 0 lets the copies in flight land first.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<unsigned long long>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

constexpr int kTileBytes = kTileRows * kRowBytes;  // 32 KB

template <int F, typename T> struct QColsSmem {
    static constexpr int TC = ColTile<T>::TC, PB = payload<F>(), SB = Fmt<F>::FIXED ? 2 : 1;
    static constexpr int CS = 8 * PB + 8;
    static constexpr int bytes = 2 * kTileBytes + TC * CS + TC * 8 * SB + 1024;  // + alignment slack
};

template <int F, typename T>
__global__ void __launch_bounds__(kColThreads) k_quantize_cols_tma(const __grid_constant__ CUtensorMap tmap,
                                                                  void* __restrict__ codes, void* __restrict__ scales,
                                                                  long long rows, long long cols, unsigned int* err) {
    constexpr int TC = ColTile<T>::TC, CPL = ColTile<T>::CPL;
    constexpr int PB = payload<F>();
    constexpr int SB = Fmt<F>::FIXED ? 2 : 1;
    constexpr int CS = 8 * PB + 8;
    extern __shared__ uint8_t dsm[];
    uint8_t* const tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsm) + 1023) & ~uintptr_t(1023));
    uint8_t* const out = tiles + 2 * kTileBytes;
    uint8_t* const sc = out + TC * CS;
    __shared__ __align__(8) unsigned long long full[2];
    __shared__ int abort_flag;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const long long RB = rows / 32;
    const long long nsx = (cols + TC - 1) / TC, ntiles = nsx * ((rows + kTileRows - 1) / kTileRows);
    const long long G = gridDim.x;
    if (t == 0) {
        mbar_init(smem_u32(&full[0]), 1);
        mbar_init(smem_u32(&full[1]), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    volatile int* ab = &abort_flag;
    long long issued = 0;  // thread 0: tiles whose copy has been issued
    auto issue = [&](long long n) {
        const long long tile = blockIdx.x + n * G;
        if (tile >= ntiles) return;
        const int b = (int)(n & 1);
        mbar_expect_tx(smem_u32(&full[b]), kTileBytes);
        tma_load_2d(smem_u32(tiles + b * kTileBytes), &tmap, (int)((tile % nsx) * TC), (int)((tile / nsx) * kTileRows),
                    smem_u32(&full[b]));
        issued = n + 1;
    };
    if (t == 0) {
        issue(0);
        issue(1);
    }
    long long n = 0;
    for (;; ++n) {
        const long long tile = blockIdx.x + n * G;
        if (tile >= ntiles) break;
        const int b = (int)(n & 1);
        const bool ok = mbar_wait(smem_u32(&full[b]), (uint32_t)(n >> 1) & 1u, ab, err);
        if (__syncthreads_or(!ok)) break;
        const long long sx = tile % nsx, sy = tile / nsx;
        const long long col0 = sx * TC, row0 = sy * kTileRows;
        const int nrb = (int)min((long long)kTileRows, rows - row0) / 32;
        const int ncols = (int)min((long long)TC, cols - col0);
        uint32_t w[CPL][Blk<T>::NW];
        if (warp < nrb) gather_columns<T>(tiles + b * kTileBytes, warp, lane, w);
        __syncthreads();  // buffer b read by every warp, the previous tile's staged outputs stored
        if (t == 0) issue(n + 2);
        if (warp < nrb) {
#pragma unroll
            for (int k = 0; k < CPL; ++k) {
                const int j = lane * CPL + k;  // column within the strip
                if (j < ncols) {
                    const uint32_t byte = scale_byte<F>(block_amax<T>(w[k]));
                    uint32_t o[8];
                    encode_block<F, T>(w[k], byte, o);
                    uint32_t* q = reinterpret_cast<uint32_t*>(out + j * CS + warp * PB);
#pragma unroll
                    for (int i = 0; i < PB / 4; ++i) q[i] = o[i];
                    if constexpr (SB == 2) reinterpret_cast<uint16_t*>(sc)[j * 8 + warp] = (uint16_t)byte;
                    else sc[j * 8 + warp] = (uint8_t)byte;
                }
            }
        }
        __syncthreads();
        // column j's row-blocks of this tile are contiguous in the output: nrb * PB bytes
        if (nrb == 8 && ncols == TC) {
#pragma unroll
            for (int i = t; i < TC * PB; i += kColThreads) {
                const int j = i / PB, k = i % PB;
                const long long g = ((col0 + j) * RB + sy * 8) * PB + 8 * k;
                *reinterpret_cast<uint2*>(reinterpret_cast<char*>(codes) + g) = *reinterpret_cast<const uint2*>(out + j * CS + 8 * k);
            }
#pragma unroll
            for (int i = t; i < TC * 8; i += kColThreads) {
                const int j = i >> 3, k = i & 7;
                const long long g = (col0 + j) * RB + sy * 8 + k;
                if constexpr (SB == 2) reinterpret_cast<uint16_t*>(scales)[g] = reinterpret_cast<const uint16_t*>(sc)[j * 8 + k];
                else reinterpret_cast<uint8_t*>(scales)[g] = sc[j * 8 + k];
            }
        } else {
            const int seg8 = nrb * PB / 8;
            for (int i = t; i < ncols * seg8; i += kColThreads) {
                const int j = i / seg8, k = i % seg8;
                const long long g = ((col0 + j) * RB + sy * 8) * PB + 8 * k;
                *reinterpret_cast<uint2*>(reinterpret_cast<char*>(codes) + g) = *reinterpret_cast<const uint2*>(out + j * CS + 8 * k);
            }
            for (int i = t; i < ncols * nrb; i += kColThreads) {
                const int j = i / nrb, k = i % nrb;
                const long long g = (col0 + j) * RB + sy * 8 + k;
                if constexpr (SB == 2) reinterpret_cast<uint16_t*>(scales)[g] = reinterpret_cast<const uint16_t*>(sc)[j * 8 + k];
                else reinterpret_cast<uint8_t*>(scales)[g] = sc[j * 8 + k];
            }
        }
    }
    if (t == 0) {  // after a timeout: the copies issued and not consumed land before shared memory goes away
        for (long long q = n; q < issued; ++q) {
            const uint32_t bar = smem_u32(&full[q & 1]), par = (uint32_t)(q >> 1) & 1u;
            const unsigned long long t0 = global_ns();
            while (!mbar_test(bar, par) && global_ns() - t0 < kWaitLimitNs) {
            }
        }
    }
}

// Tensor map of a [rows, cols] matrix of 2- or 4-byte values: boxes of 256 rows x 128 bytes,
// 128-byte swizzle. The encoder is the driver's, fetched once through the runtime.
static bool encode_tile_map(CUtensorMap* m, const void* base, long long rows, long long cols, int esize) {
    static PFN_cuTensorMapEncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(p);
        else
            cudaGetLastError();
    });
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * (cuuint64_t)esize};
    const cuuint32_t box[2] = {(cuuint32_t)(kRowBytes / esize), (cuuint32_t)kTileRows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, esize == 2 ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---- dequantize, one CTA per tile: 32-column tiles (64-byte bf16 rows) ---------------------------
// Taken only by matrices whose output, codes or scales reach 2^31 bytes (its offsets are 64-bit);
// the persistent kernel further below takes everything else. Tiles of 256 rows x 32 columns,
// chunk c of row r at c ^ (r/2 mod 4) for 64-byte rows and c ^ (r mod 8) for 128-byte rows.
constexpr int kNarrowCols = 32;

// byte offset of element (r, j) of the tile; rows of 32 * sizeof(T) bytes,
// chunk c of row r stored at c ^ sw(r)
template <typename T> __device__ __forceinline__ uint32_t ntile_off(int r, int j) {
    if constexpr (sizeof(T) == 2) {
        const int c = j >> 3;  // 4 chunks of 8 values
        return (uint32_t)(r * 64 + 16 * (c ^ ((r >> 1) & 3)) + 2 * (j & 7));
    } else {
        const int c = j >> 2;  // 8 chunks of 4 values
        return (uint32_t)(r * 128 + 16 * (c ^ (r & 7)) + 4 * (j & 3));
    }
}

template <typename T>
__device__ __forceinline__ void ntile_row_load(const uint8_t* tile, int r, uint32_t* w) {
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

// Lane j's byte offsets of column j in the swizzled rows, one per swizzle phase (the chunk index
// is xor-ed with (r / 2) mod 4 for 64-byte rows, r mod 8 for 128-byte rows; within a row-block
// that phase depends only on the row's index inside the block, so it is a compile-time value
// in the unrolled loops below and every shared-memory access is a base plus an immediate).
template <typename T> struct NColOffsets {
    static constexpr int NP = sizeof(T) == 2 ? 4 : 8;
    uint32_t off[NP];
    __device__ __forceinline__ explicit NColOffsets(int j) {
#pragma unroll
        for (int q = 0; q < NP; ++q)
            off[q] = sizeof(T) == 2 ? (uint32_t)(16 * ((j >> 3) ^ q) + 2 * (j & 7)) : (uint32_t)(16 * ((j >> 2) ^ q) + 4 * (j & 3));
    }
};

template <typename T>
__device__ __forceinline__ void nscatter_column(uint8_t* tile, int rb, const NColOffsets<T>& co, const uint32_t* o) {
    if constexpr (sizeof(T) == 2) {
        uint8_t* base = tile + rb * 32 * 64;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            *reinterpret_cast<uint16_t*>(base + (2 * i) * 64 + co.off[i & 3]) = (uint16_t)o[i];
            *reinterpret_cast<uint16_t*>(base + (2 * i + 1) * 64 + co.off[i & 3]) = (uint16_t)(o[i] >> 16);
        }
    } else {
        uint8_t* base = tile + rb * 32 * 128;
#pragma unroll
        for (int i = 0; i < 32; ++i) *reinterpret_cast<uint32_t*>(base + i * 128 + co.off[i & 7]) = o[i];
    }
}


template <int F, typename T>
__global__ void __launch_bounds__(kColThreads) k_dequantize_cols(const void* __restrict__ codes,
                                                                const void* __restrict__ scales, void* __restrict__ dst,
                                                                long long rows, long long cols) {
    constexpr int PB = payload<F>();
    __shared__ __align__(16) uint8_t tile[kTileRows * kNarrowCols * sizeof(T)];
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const long long RB = rows / 32;
    const long long col0 = (long long)blockIdx.x * kNarrowCols;
    const long long row0 = (long long)blockIdx.y * kTileRows;
    const int nrows = (int)min((long long)kTileRows, rows - row0);
    const int nrb = nrows / 32;
    const bool a32 = ((reinterpret_cast<uintptr_t>(dst) | (uintptr_t)(cols * sizeof(T))) & 31) == 0;
    constexpr int SB = Fmt<F>::FIXED ? 2 : 1;
    constexpr int CS = 8 * PB + 8;  // padded column stride, as in quantize_cols
    __shared__ __align__(16) uint8_t in[kNarrowCols * CS];
    __shared__ __align__(16) uint8_t sc[kNarrowCols * 8 * SB];
    // column j's nrb payloads of this chunk are contiguous in the transposed layout: read them
    // with coalesced 8-byte loads (and the scales with coalesced byte loads) into shared memory
    {
        const int seg8 = nrb * PB / 8;
        for (int i = t; i < kNarrowCols * seg8; i += kColThreads) {
            const int j = i / seg8, k = i % seg8;
            const long long g = ((col0 + j) * RB + blockIdx.y * 8) * PB + 8 * k;
            *reinterpret_cast<uint2*>(in + j * CS + 8 * k) = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const char*>(codes) + g));
        }
        for (int i = t; i < kNarrowCols * nrb; i += kColThreads) {
            const int j = i / nrb, k = i % nrb;
            const long long g = (col0 + j) * RB + blockIdx.y * 8 + k;
            if constexpr (SB == 2) reinterpret_cast<uint16_t*>(sc)[j * 8 + k] = __ldg(reinterpret_cast<const uint16_t*>(scales) + g);
            else sc[j * 8 + k] = __ldg(reinterpret_cast<const uint8_t*>(scales) + g);
        }
    }
    __syncthreads();
    if (warp < nrb) {
        uint32_t pw[8];
        const uint32_t* q = reinterpret_cast<const uint32_t*>(in + lane * CS + warp * PB);
#pragma unroll
        for (int i = 0; i < PB / 4; ++i) pw[i] = q[i];
        const uint32_t byte = SB == 2 ? (reinterpret_cast<const uint16_t*>(sc)[lane * 8 + warp] & 0xFFu) : sc[lane * 8 + warp];
        uint32_t o[Blk<T>::NW];
        decode_block<F, T>(pw, byte, o);
        nscatter_column<T>(tile, warp, NColOffsets<T>(lane), o);
    }
    __syncthreads();
    if (t < nrows) {
        uint32_t w[8 * sizeof(T)];
        ntile_row_load<T>(tile, t, w);
        char* p = reinterpret_cast<char*>(dst) + ((row0 + t) * cols + col0) * (long long)sizeof(T);
#pragma unroll
        for (int i = 0; i < (int)sizeof(T); ++i) st32(p + 32 * i, w + 8 * i, a32);
    }
}

// the 16 codes k = 16h .. 16h+15 of a payload start at word h * W / 2 (W-bit codes, 16 per
// half): hw gets that half's W/2 words
template <int F>
__device__ __forceinline__ void load_half_payload(const uint8_t* block, int h, uint32_t* hw) {
    constexpr int NH = Fmt<F>::W / 2;
    const uint32_t* q = reinterpret_cast<const uint32_t*>(block) + h * NH;
#pragma unroll
    for (int i = 0; i < NH; ++i) hw[i] = q[i];
}

// true when a half payload holds an E4M3 NaN magnitude (0x7F)
template <int F> __device__ __forceinline__ bool half_has_nan(const uint32_t* hw) {
    if constexpr (F == F_E4M3) {
        uint32_t m = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) m |= ((hw[i] & 0x7F7F7F7Fu) + 0x01010101u) & 0x80808080u;
        return m != 0;
    } else {
        return false;
    }
}

// ---- dequantize: persistent, payloads prefetched two tiles ahead ----------------------------------
//
// Tiles of 256 rows x 128 output bytes per row (64 bf16 or 32 fp32 columns: one whole line per
// row; a column's 8 row-blocks of payload are one run of 8 payloads, 192 bytes for the 6-bit
// formats, on a 64-byte boundary when the column's run is: whole DRAM accesses). Each
// CTA walks tiles blockIdx.x + n * gridDim.x in band-major order (the CTAs running at one time
// cover a few adjacent row bands, so the rows they write are close together) and keeps the loads
// of tiles n + 1 and n + 2 in flight while it decodes and stores tile n: the payloads come in by
// 8-byte cp.async copies into a ring of three stages, the scales by plain loads into a register
// that is written to its stage one iteration later. cp.async waits are the hardware's own (no
// spin on a flag), so no wait here needs a bound.
// Decode, bf16 output (64 columns): warp w takes row-blocks (w & 3) and (w & 3) + 4 of column
// group w >> 2 (32 columns); lane L columns 2p, 2p + 1 of the group (p = L & 15), rows 16h ..
// 16h + 15 of each row-block (h = L >> 4), so each decoded word is one row's pair of neighbouring
// columns. fp32 output (32 columns): warp w takes row-block w, lane j column j (a whole block),
// each decoded value one word of its row.
constexpr int kDqRbt = 8, kDqRows = 32 * kDqRbt, kDqStages = 3;
template <typename T> __host__ __device__ constexpr int dq_cols() { return 128 / (int)sizeof(T); }  // columns of a tile

template <int F, int NC> struct DqStage {
    static constexpr int PB = payload<F>(), SB = Fmt<F>::FIXED ? 2 : 1;
    static constexpr int CS = kDqRbt * PB + 8;                      // padded column stride of the payloads
    static constexpr int SC = NC * CS;                               // offset of the scales
    static constexpr int bytes = (SC + NC * kDqRbt * SB + 15) / 16 * 16;
};

__device__ __forceinline__ void cp_async8(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// chunk swizzle of output row r (16-byte chunk c stored at c ^ dq_swz(r)): bits 0 and 2 from
// r & 3 spread out, bit 2 flipped by r & 16. The decoding lanes of one row index write rows 16
// apart (bit 4 of r) into different banks; the 4 rows x 2 threads of a quarter-warp reading
// chunks {2hf + c} of their rows cover all banks.
__device__ __forceinline__ int dq_swz(int r) { return ((r & 1) | ((r & 2) << 1)) ^ (((r >> 4) & 1) << 2); }

// tile coordinates of tiles first, first + step, ... (band-major: tx fastest), by additions
struct DqWalk {
    int tx, by, ntx, nby, dx, dy;
    __device__ __forceinline__ DqWalk(int ntx_, int nby_) : ntx(ntx_), nby(nby_) {
        const int G = (int)gridDim.x, b = (int)blockIdx.x;
        tx = b % ntx;
        by = b / ntx;
        dx = G % ntx;
        dy = G / ntx;
    }
    __device__ __forceinline__ bool valid() const { return by < nby; }
    __device__ __forceinline__ void next() {
        tx += dx;
        by += dy;
        if (tx >= ntx) {
            tx -= ntx;
            ++by;
        }
    }
};

// 16 values of a column (rows 16h .. 16h + 15 of a row-block) as exact f32 values: the
// up-conversions for the floating-point formats; AXS-6 by placing its magnitude on the fp32 fields
// (cheaper there than converting m to float, by measurement)
template <int F> __device__ __forceinline__ void dq_vals16(const uint32_t* hw, float* v) {
    if constexpr (F == F_AXS6) {
        const unsigned long long D = dup2(decode_unit<F>());
#pragma unroll
        for (int k = 0; k < 16; k += 2)
            upk(f2mul(pk(__uint_as_float(payload_bits<F>(hw, k)), __uint_as_float(payload_bits<F>(hw, k + 1))), D), v[k],
                v[k + 1]);
    } else {
        decode16<F>(hw, v);
    }
}

// Sizes: every byte offset into the codes, scales and output fits in 31 bits (the launcher
// checks), so the per-tile arithmetic is 32-bit.
template <int F, typename T>
__global__ void __launch_bounds__(kColThreads, 2) k_dequantize_cols_p(const void* __restrict__ codes,
                                                                     const void* __restrict__ scales,
                                                                     void* __restrict__ dst, int rows, int cols) {
    constexpr int kDqCols = dq_cols<T>();
    using St = DqStage<F, kDqCols>;
    constexpr int PB = St::PB, SB = St::SB, CS = St::CS;
    constexpr int SEG8 = kDqRbt * PB / 8;             // 8-byte pieces of one column's payloads in a tile
    constexpr int NU = kDqCols * SEG8 / kColThreads;  // this thread's pieces of a full tile
    static_assert(kDqCols * SEG8 % kColThreads == 0, "whole pieces per thread");
    extern __shared__ __align__(16) uint8_t dsm[];
    uint8_t* const tile = dsm;                    // kDqRows x 128 bytes
    uint8_t* const stages = dsm + kDqRows * 128;  // kDqStages x St::bytes
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int RB = rows / 32;
    const int nby = (rows + kDqRows - 1) / kDqRows;
    const int ntx = (cols + kDqCols - 1) / kDqCols;
    const bool a32 = ((reinterpret_cast<uintptr_t>(dst) | (uintptr_t)(cols * sizeof(T))) & 31) == 0;
    const uint32_t st0 = smem_u32(stages);
    const int col_bytes = RB * PB;  // one column's payloads in the transposed layout
    // a column's scales of a full tile are one aligned 8-byte (AXS-6: 16-byte) load when the
    // column's scale run starts on that boundary
    const bool wide_scales = RB % kDqRbt == 0 && (reinterpret_cast<uintptr_t>(scales) & (kDqRbt * SB - 1)) == 0;
    const char* const cbase = reinterpret_cast<const char*>(codes);
    const char* const sbase = reinterpret_cast<const char*>(scales);
    char* const dbase = reinterpret_cast<char*>(dst);

    // per-thread offsets, the same for every full tile: its NU payload pieces (shared, and global
    // relative to the tile's first column run) and its column's scale run
    uint32_t so_u[NU];
    int go_u[NU];
#pragma unroll
    for (int u = 0; u < NU; ++u) {
        const int i = t + u * kColThreads, j = i / SEG8, k = i - j * SEG8;
        so_u[u] = (uint32_t)(j * CS + 8 * k);
        go_u[u] = j * col_bytes + 8 * k;
    }
    const int gs_t = t * RB * SB;  // column t's scale run (bytes), t < kDqCols

    bool swide = false;  // the pending scale registers hold a whole column's run
    uint4 sw = make_uint4(0, 0, 0, 0);
    // copies of the tile at `w` into stage `stage` (one commit group per tile, empty past the last
    // tile); this thread's scale(s) of the tile are loaded into registers, to be stored later
    auto issue = [&](const DqWalk& w, int stage, int& soff) {
        soff = -1;
        swide = false;
        if (w.valid()) {
            const int col0 = w.tx * kDqCols;
            const int ncols = min(kDqCols, cols - col0);
            const int nrb = min(kDqRbt, RB - w.by * kDqRbt);
            const int tb = col0 * RB + w.by * kDqRbt;  // first column's first row-block
            const char* src = cbase + tb * PB;
            const uint32_t sb = st0 + (uint32_t)(stage * St::bytes);
            if (ncols == kDqCols && nrb == kDqRbt) {
#pragma unroll
                for (int u = 0; u < NU; ++u) cp_async8(sb + so_u[u], src + go_u[u]);
            } else {
                const int seg8 = nrb * PB / 8;
                for (int i = t; i < ncols * seg8; i += kColThreads) {
                    const int j = i / seg8, k = i % seg8;
                    cp_async8(sb + (uint32_t)(j * CS + 8 * k), src + j * col_bytes + 8 * k);
                }
            }
            if (wide_scales && nrb == kDqRbt) {  // a column's kDqRbt scales in one aligned load
                if (t < ncols) {
                    const char* g = sbase + tb * SB + gs_t;
                    if constexpr (SB == 2) {
                        sw = __ldg(reinterpret_cast<const uint4*>(g));
                    } else {
                        const uint2 v = __ldg(reinterpret_cast<const uint2*>(g));
                        sw.x = v.x;
                        sw.y = v.y;
                    }
                    soff = stage * St::bytes + St::SC + t * kDqRbt * SB;
                    swide = true;
                }
            } else {
                for (int i = t; i < ncols * nrb; i += kColThreads) {  // byte by byte, straight to the stage
                    const int j = i / nrb, k = i - (i / nrb) * nrb;
                    const int g = tb + j * RB + k;
                    const int off = stage * St::bytes + St::SC + (j * kDqRbt + k) * SB;
                    if constexpr (SB == 2) *reinterpret_cast<uint16_t*>(stages + off) = __ldg(reinterpret_cast<const uint16_t*>(scales) + g);
                    else stages[off] = __ldg(reinterpret_cast<const uint8_t*>(scales) + g);
                }
            }
        }
        cp_async_commit();
    };
    auto put_scale = [&](int soff) {
        if (soff < 0 || !swide) return;
        if constexpr (SB == 2) *reinterpret_cast<uint4*>(stages + soff) = sw;
        else *reinterpret_cast<uint2*>(stages + soff) = make_uint2(sw.x, sw.y);
    };

    // decode role (bf16): row-blocks rb and rb + 4 of column group cg; columns ja, ja + 1, rows 16h ..
    const int rb = sizeof(T) == 2 ? (warp & 3) : warp, cg = sizeof(T) == 2 ? (warp >> 2) : 0;
    const int p = lane & 15, h = lane >> 4;
    const int ja = sizeof(T) == 2 ? cg * 32 + 2 * p : lane;
    const int pa_off = ja * CS + rb * PB, sa_off = St::SC + (ja * kDqRbt + rb) * SB;
    uint8_t* const obase = sizeof(T) == 2 ? tile + (rb * 32 + 16 * h) * 128 + 4 * (p & 3)
                                          : tile + rb * 32 * 128 + 4 * (lane & 3);
    uint32_t c16[8];  // bf16: chunk offsets by row & 3 (4 used); fp32: by row & 7
#pragma unroll
    for (int q = 0; q < 8; ++q)
        c16[q] = sizeof(T) == 2 ? (uint32_t)(16 * ((4 * cg + (p >> 2)) ^ dq_swz((q & 3) + 16 * h)))
                                : (uint32_t)(16 * ((lane >> 2) ^ q));
    // store role, bf16: thread (r, hf) stores bytes 32hf .. 32hf + 31 of output rows r and r + 128
    // and, in a full 64-column strip, bytes 64 + 32hf .. (a strip of 32 columns is 64 bytes);
    // fp32: thread t stores its row t, 128 bytes (chunk c at c ^ (t & 7))
    const int r = sizeof(T) == 2 ? (t >> 1) : t, hf = sizeof(T) == 2 ? (t & 1) : 0;
    uint32_t rd[8];  // byte offsets of its chunks in the output tile (bf16: 4 of row r; row r + 128: + 128 * 128)
#pragma unroll
    for (int c = 0; c < 8; ++c)
        rd[c] = sizeof(T) == 2 ? (uint32_t)(r * 128 + 16 * ((((c & 3) & 1) + 2 * hf + 4 * ((c & 3) >> 1)) ^ dq_swz(r)))
                               : (uint32_t)(r * 128 + 16 * (c ^ (r & 7)));
    const int rowoff = r * cols * (int)sizeof(T) + 32 * hf;

    DqWalk cur(ntx, nby), ahead(ntx, nby);
    int so = -1;
    issue(ahead, 0, so);
    put_scale(so);  // the first tile's scales: one exposed load latency per CTA
    ahead.next();
    issue(ahead, 1, so);
    ahead.next();
    for (int stage = 0; cur.valid(); cur.next(), stage = stage == kDqStages - 1 ? 0 : stage + 1) {
        const int col0 = cur.tx * kDqCols, row0 = cur.by * kDqRows;
        const int ncols = min(kDqCols, cols - col0);
        const int nrows = min(kDqRows, rows - row0);
        cp_async_wait<1>();  // this thread's copies of the tile have landed
        __syncthreads();     // everyone's have; the previous tile's rows have left the output tile
        const uint8_t* stg = stages + stage * St::bytes;
        if constexpr (sizeof(T) == 2) {
            if (cg * 32 < ncols) {
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if (rb + 4 * half >= nrows / 32) break;
                    const uint8_t* sp = stg + pa_off + half * 4 * PB;
                    uint32_t ha[Fmt<F>::W / 2], hb[Fmt<F>::W / 2];
                    load_half_payload<F>(sp, h, ha);
                    load_half_payload<F>(sp + CS, h, hb);
                    uint32_t ba, bb;
                    if constexpr (SB == 2) {
                        ba = *reinterpret_cast<const uint16_t*>(stg + sa_off + half * 4 * SB) & 0xFFu;
                        bb = *reinterpret_cast<const uint16_t*>(stg + sa_off + half * 4 * SB + kDqRbt * SB) & 0xFFu;
                    } else {
                        ba = stg[sa_off + half * 4];
                        bb = stg[sa_off + half * 4 + kDqRbt];
                    }
                    float va[16], vb[16];
                    dq_vals16<F>(ha, va);
                    dq_vals16<F>(hb, vb);
                    const unsigned long long S = pk(fwd_scale(ba), fwd_scale(bb));
                    uint32_t o[16];
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        float x, y;
                        upk(f2mul(pk(va[k], vb[k]), S), x, y);
                        o[k] = bf16x2(x, y);
                    }
                    if (ba == 0xFFu || bb == 0xFFu || half_has_nan<F>(ha) || half_has_nan<F>(hb)) {
#pragma unroll
                        for (int k = 0; k < 16; ++k) {  // canonical quiet NaN for NaN blocks and E4M3 NaN codes
                            const bool na = ba == 0xFFu || (F == F_E4M3 && ((ha[k >> 2] >> (8 * (k & 3))) & 0x7Fu) == 0x7Fu);
                            const bool nb = bb == 0xFFu || (F == F_E4M3 && ((hb[k >> 2] >> (8 * (k & 3))) & 0x7Fu) == 0x7Fu);
                            if (na) o[k] = (o[k] & 0xFFFF0000u) | 0x7FC0u;
                            if (nb) o[k] = (o[k] & 0x0000FFFFu) | 0x7FC00000u;
                        }
                    }
                    uint8_t* ob = obase + half * 128 * 128;  // row-block rb + 4: 128 rows further
#pragma unroll
                    for (int k = 0; k < 16; ++k) *reinterpret_cast<uint32_t*>(ob + k * 128 + c16[k & 3]) = o[k];
                }
            }
        } else {
            if (rb < nrows / 32) {  // one row-block per warp, lane j = column j, all 32 rows
                const uint8_t* sp = stg + pa_off;
                uint32_t ha[Fmt<F>::W / 2], hb[Fmt<F>::W / 2];
                load_half_payload<F>(sp, 0, ha);
                load_half_payload<F>(sp, 1, hb);
                const uint32_t byte =
                    SB == 2 ? (*reinterpret_cast<const uint16_t*>(stg + sa_off) & 0xFFu) : (uint32_t)stg[sa_off];
                float v[32];
                dq_vals16<F>(ha, v);
                dq_vals16<F>(hb, v + 16);
                const unsigned long long S = dup2(fwd_scale(byte));
                uint32_t o[32];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    float x, y;
                    upk(f2mul(pk(v[2 * k], v[2 * k + 1]), S), x, y);
                    o[2 * k] = __float_as_uint(x);
                    o[2 * k + 1] = __float_as_uint(y);
                }
                if (byte == 0xFFu || half_has_nan<F>(ha) || half_has_nan<F>(hb)) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) {  // canonical quiet NaN for NaN blocks and E4M3 NaN codes
                        const uint32_t* hw = k < 16 ? ha : hb;
                        const int kk = k & 15;
                        if (byte == 0xFFu || (F == F_E4M3 && ((hw[kk >> 2] >> (8 * (kk & 3))) & 0x7Fu) == 0x7Fu))
                            o[k] = 0x7FC00000u;
                    }
                }
#pragma unroll
                for (int k = 0; k < 32; ++k) *reinterpret_cast<uint32_t*>(obase + k * 128 + c16[k & 7]) = o[k];
            }
        }
        __syncthreads();  // the output tile is complete; this stage is free
        put_scale(so);    // the next tile's scales into its stage (read after the next barrier)
        issue(ahead, stage == 0 ? kDqStages - 1 : stage - 1, so);
        ahead.next();
        if constexpr (sizeof(T) == 2) {
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                if (r + 128 * half < nrows) {
                    char* q = dbase + ((row0 + 128 * half) * cols + col0) * 2 + rowoff;
                    uint32_t w[16];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 v = *reinterpret_cast<const uint4*>(tile + rd[c] + half * 128 * 128);
                        w[4 * c] = v.x;
                        w[4 * c + 1] = v.y;
                        w[4 * c + 2] = v.z;
                        w[4 * c + 3] = v.w;
                    }
                    st32(q, w, a32);
                    if (ncols == kDqCols) st32(q + 64, w + 8, a32);
                }
            }
        } else {
            if (r < nrows) {
                char* q = dbase + (row0 * cols + col0) * 4 + rowoff;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    uint32_t w[16];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const uint4 v = *reinterpret_cast<const uint4*>(tile + rd[4 * hh + c]);
                        w[4 * c] = v.x;
                        w[4 * c + 1] = v.y;
                        w[4 * c + 2] = v.z;
                        w[4 * c + 3] = v.w;
                    }
                    st32(q + 64 * hh, w, a32);
                    st32(q + 64 * hh + 32, w + 8, a32);
                }
            }
        }
    }
    cp_async_wait<0>();  // no copy may land in shared memory after the CTA has left
}

template <int F, typename T> static constexpr int dq_p_smem() {
    return kDqRows * 128 + kDqStages * DqStage<F, dq_cols<T>()>::bytes;
}

template <int F, typename T>
static cudaError_t launch_qc_t(const void* src, void* codes, void* scales, long long rows, long long cols,
                               cudaStream_t st) {
    constexpr int TC = ColTile<T>::TC;
    CUtensorMap map;
    // the tensor copy takes 32-bit coordinates: wider matrices take the one-shot kernel
    if (cols <= 0x7FFFFFFFLL && rows <= 0x7FFFFFFFLL && encode_tile_map(&map, src, rows, cols, (int)sizeof(T))) {
        auto kern = k_quantize_cols_tma<F, T>;
        constexpr int smem = QColsSmem<F, T>::bytes;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        int dev = 0, sms = 148, per_sm = 1;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kColThreads, smem);
        const long long ntiles = ((cols + TC - 1) / TC) * ((rows + kTileRows - 1) / kTileRows);
        long long grid = (long long)sms * (per_sm > 0 ? per_sm : 1);
        if (grid > ntiles) grid = ntiles;
        unsigned int* err = nullptr;
        if ((e = device_error_word(&err)) != cudaSuccess) return e;
        kern<<<(unsigned)grid, kColThreads, smem, st>>>(map, codes, scales, rows, cols, err);
        return cudaGetLastError();
    }
    dim3 grid((unsigned)((cols + TC - 1) / TC), (unsigned)((rows + kTileRows - 1) / kTileRows));
    k_quantize_cols<F, T><<<grid, kColThreads, 0, st>>>(src, codes, scales, rows, cols);
    return cudaGetLastError();
}
template <int F, typename T>
static cudaError_t launch_dqc_t(const void* codes, const void* scales, void* dst, long long rows, long long cols,
                                cudaStream_t st) {
    // 32-bit offsets: the outputs, the codes and the scales each below 2^31 bytes
    if (rows * cols * (long long)sizeof(T) < (1LL << 31) && rows * (cols / 32) * payload<F>() < (1LL << 31)) {
        auto kern = k_dequantize_cols_p<F, T>;
        constexpr int smem = dq_p_smem<F, T>();
        constexpr int NC = dq_cols<T>();
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        int dev = 0, sms = 148, per_sm = 1;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kColThreads, smem);
        // two CTAs per SM, though shared memory would hold three: the 8-byte copies are staged
        // through L1, and a third CTA's stages leave L1 too small for them (bf16 16384x8192,
        // fraction of the HBM peak, E2M3 / E4M3 / E2M1: 0.57 / 0.90 / 0.80 with three CTAs,
        // 0.81 / 0.92 / 0.84 with two)
        if (per_sm > 2) per_sm = 2;
        const long long ntiles = ((cols + NC - 1) / NC) * ((rows + kDqRows - 1) / kDqRows);
        long long grid = (long long)sms * (per_sm > 0 ? per_sm : 1);
        if (grid > ntiles) grid = ntiles;
        kern<<<(unsigned)grid, kColThreads, smem, st>>>(codes, scales, dst, (int)rows, (int)cols);
        return cudaGetLastError();
    }
    dim3 grid((unsigned)(cols / kNarrowCols), (unsigned)((rows + kTileRows - 1) / kTileRows));
    k_dequantize_cols<F, T><<<grid, kColThreads, 0, st>>>(codes, scales, dst, rows, cols);
    return cudaGetLastError();
}

bool cols_grid_ok(long long rows, long long cols) {
    return (cols + 31) / 32 <= 0x7FFFFFFFLL && (rows + kTileRows - 1) / kTileRows <= 65535;
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
