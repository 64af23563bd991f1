// mxq_mma.cu -- E8M0 scales rearranged into the layout the block-scaled
// tensor-core MMA reads (sm_100a).
//
// Converted weights feed block-scaled GEMMs ("Sonar: Online MXFP6", Current
// limits: dense dimensions in multiples of 128), whose kernels take the
// per-block scales of an [rows, K] operand as 128 x 4 tiles: the [rows, kb]
// scale matrix (kb = K / 32) padded with zeros to multiples of 128 rows and 4
// columns, tiles of 512 bytes stored tile-row by tile-row, row r / column c of
// a tile at byte (r % 32) * 16 + (r / 32) * 4 + c. mxq_quantize_mma writes that
// layout directly (mxq_codec.cu); this kernel converts a plain scale array.
//
// One thread writes one 4-byte word of the output: the four columns of one row inside one tile.
// Output words are consecutive across a warp (coalesced 128-byte lines); the four input bytes
// come from one row of the plain array, in one 4-byte load when the rows are 4-byte aligned.
// blockIdx.y walks the tile-rows (128 rows each), so the per-word index arithmetic is 32-bit
// and division-free except for shifts.
#include <cstdint>
#include <cuda_runtime.h>

#include "mxq_internal.h"

namespace mxq {

__global__ void __launch_bounds__(256) k_swizzle_scales(const uint8_t* __restrict__ s, long long rows, int kb,
                                                         uint32_t* __restrict__ out, int tiles, long long ntr,
                                                         bool words) {
    const int per_tr = tiles * 128;  // output words of one tile-row
    for (long long tr = blockIdx.y; tr < ntr; tr += gridDim.y) {
        uint32_t* o_tr = out + tr * per_tr;
        for (int o = blockIdx.x * blockDim.x + threadIdx.x; o < per_tr; o += gridDim.x * blockDim.x) {
            const int tile = o >> 7;
            const int w = o & 127;  // word inside the tile: (r % 32) * 4 + r / 32
            const long long r = tr * 128 + (w & 3) * 32 + (w >> 2);
            const int k0 = tile * 4;
            uint32_t v = 0;
            if (r < rows) {
                const uint8_t* row = s + r * kb;
                if (words) {  // kb % 4 == 0 and an aligned array: the four bytes are one word
                    v = __ldg(reinterpret_cast<const uint32_t*>(row + k0));
                } else {
#pragma unroll
                    for (int c = 0; c < 4; ++c)
                        if (k0 + c < kb) v |= (uint32_t)__ldg(row + k0 + c) << (8 * c);
                }
            }
            o_tr[o] = v;
        }
    }
}

cudaError_t launch_swizzle_scales(const void* scales, long long rows, long long kb, void* out, cudaStream_t st) {
    const long long ntr = (rows + 127) / 128, tiles = (kb + 3) / 4;
    if (ntr == 0 || tiles == 0) return cudaSuccess;
    if (tiles * 128 > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    const bool words = kb % 4 == 0 && (reinterpret_cast<uintptr_t>(scales) & 3) == 0;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long gx = (tiles * 128 + 255) / 256;
    long long gy = ntr < 65535 ? ntr : 65535;
    if (gx * gy > 16LL * sms) gy = (16LL * sms + gx - 1) / gx;  // tile-rows grid-stride beyond 16 CTAs per SM
    if (gy < 1) gy = 1;
    dim3 grid((unsigned)gx, (unsigned)gy);
    k_swizzle_scales<<<grid, 256, 0, st>>>(static_cast<const uint8_t*>(scales), rows, (int)kb,
                                           static_cast<uint32_t*>(out), (int)tiles, ntr, words);
    return cudaGetLastError();
}

}  // namespace mxq
