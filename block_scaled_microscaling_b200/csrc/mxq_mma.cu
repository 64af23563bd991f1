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
// One thread writes one 4-byte word of the output: the four columns of one row
// inside one tile. Output words are consecutive across a warp (coalesced
// 128-byte lines); the four input bytes come from one row of the plain array.
#include <cstdint>
#include <cuda_runtime.h>

#include "mxq_internal.h"

namespace mxq {

__global__ void __launch_bounds__(256) k_swizzle_scales(const uint8_t* __restrict__ s, long long rows, long long kb,
                                                         uint32_t* __restrict__ out, long long nwords) {
    const long long tiles = (kb + 3) >> 2;  // tiles per tile-row
    for (long long o = (long long)blockIdx.x * blockDim.x + threadIdx.x; o < nwords;
         o += (long long)gridDim.x * blockDim.x) {
        const long long tile = o >> 7;
        const int w = (int)(o & 127);                       // word inside the tile: (r % 32) * 4 + r / 32
        const long long r = (tile / tiles) * 128 + (w & 3) * 32 + (w >> 2);
        const long long k0 = (tile % tiles) * 4;
        uint32_t v = 0;
        if (r < rows) {
            const uint8_t* row = s + r * kb;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (k0 + c < kb) v |= (uint32_t)__ldg(row + k0 + c) << (8 * c);
        }
        out[o] = v;
    }
}

cudaError_t launch_swizzle_scales(const void* scales, long long rows, long long kb, void* out, cudaStream_t st) {
    const long long nwords = ((rows + 127) / 128) * 128 * ((kb + 3) / 4);  // bytes / 4
    if (nwords == 0) return cudaSuccess;
    long long grid = (nwords + 255) / 256;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (grid > 16LL * sms) grid = 16LL * sms;  // grid-stride beyond 16 CTAs per SM
    k_swizzle_scales<<<(unsigned)grid, 256, 0, st>>>(static_cast<const uint8_t*>(scales), rows, kb,
                                                      static_cast<uint32_t*>(out), nwords);
    return cudaGetLastError();
}

}  // namespace mxq
