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

// ---- dequantize: 32-column tiles (64-byte bf16 rows) -------------------------------------------
// The 128-byte-row tile above was slower for dequantize (bf16 16384x8192: 0.53 vs 0.62 of the
// HBM peak), so dequantize keeps tiles of 256 rows x 32 columns, chunk c of row r at c ^ (r/2 mod 4)
// for 64-byte rows and c ^ (r mod 8) for 128-byte rows.
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
