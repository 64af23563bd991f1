// mxq_expq.cu -- fused exp-then-quantize softmax probability stage (sm_100a).
//
// "EFQ-Softmax: exp-free E2M1 probabilities" explainer, Jargon (shifted scores,
// exp-then-quantize, MXFP4, microscaling block) and its stage table: the
// conventional path exponentiates the row-max-shifted scores in higher
// precision, materializes the probability block and quantizes it to E2M1 with
// an exponent-only scale from each 32-key block's maximum. Here the block is
// never materialized: scores are read once and probabilities live in registers.
//
// One CTA per row (32 to 1024 threads, two to four blocks each), two passes: the
// first streams the row from HBM for its maximum with loads marked to stay in
// L2, the second re-reads it from L2 and exponentiates and quantizes each
// 32-key block in registers. The launcher keeps the rows in flight within half
// of L2, so HBM sees each score once. Any row length (cols % 32 == 0).
// MXFP4 and MXFP8 take the bulk-copy pipeline of mxq_expq_tma.cu instead; this
// kernel serves the 6-bit formats.
#include <cstdint>
#include <cuda_runtime.h>

#include "mxq_block.cuh"
#include "mxq_device.cuh"
#include "mxq_exp.cuh"
#include "mxq_internal.h"

namespace mxq {

__device__ __forceinline__ float max32(const uint32_t (&w)[32]) {
    float m[11];
#pragma unroll
    for (int i = 0; i < 10; ++i)
        m[i] = max3_nan(__uint_as_float(w[3 * i]), __uint_as_float(w[3 * i + 1]), __uint_as_float(w[3 * i + 2]));
    m[10] = max_nan(__uint_as_float(w[30]), __uint_as_float(w[31]));
    float mx = max3_nan(max3_nan(m[0], m[1], m[2]), max3_nan(m[3], m[4], m[5]), max3_nan(m[6], m[7], m[8]));
    return max3_nan(mx, m[9], m[10]);
}

// first pass: the block, asking L2 to keep it for the second pass
__device__ __forceinline__ void load_keep(const float* s, long long b, uint32_t (&w)[32], bool a32) {
    const char* p = reinterpret_cast<const char*>(s) + b * 128;
    if (a32) {
#pragma unroll
        for (int i = 0; i < 4; ++i) ld_v8_keep(p + 32 * i, w + 8 * i);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) ld_2v4(p + 32 * i, w + 8 * i);
    }
}

// One row per CTA (TPR threads), CTAs walking
// rows with a grid stride. Pass 1 streams the row from HBM for its maximum
// (NaN if any key is NaN), the loads marked to stay in L2; one CTA barrier
// gives every thread the maximum; pass 2 reads the row again -- from L2 -- and
// exponentiates and quantizes it block by block. The launcher caps the CTAs
// in flight so that their rows fit comfortably in L2.
template <int F, int TPR>
__global__ void __launch_bounds__(TPR) k_exp_quantize(const float* __restrict__ scores, void* __restrict__ codes,
                                                     void* __restrict__ scales, long long rows, long long cols,
                                                     bool a32) {
    __shared__ float wmax[TPR / 32];
    __shared__ float rmax;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const long long bpr = cols / 32;
    const float NEG_INF = __uint_as_float(0xFF800000u);
    for (long long row = blockIdx.x; row < rows; row += gridDim.x) {
        const float* s = scores + row * cols;
        float mx = NEG_INF;
        long long b = t;
        for (; b + TPR < bpr; b += 2 * TPR) {  // two blocks in flight
            uint32_t w0[32], w1[32];
            load_keep(s, b, w0, a32);
            load_keep(s, b + TPR, w1, a32);
            mx = max3_nan(mx, max32(w0), max32(w1));
        }
        if (b < bpr) {
            uint32_t w0[32];
            load_keep(s, b, w0, a32);
            mx = max_nan(mx, max32(w0));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = max_nan(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
        if constexpr (TPR > 32) {
            if (lane == 0) wmax[warp] = mx;
            __syncthreads();
            if (warp == 0) {
                float v = lane < TPR / 32 ? wmax[lane] : NEG_INF;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v = max_nan(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
                if (lane == 0) rmax = v;
            }
            __syncthreads();
            mx = rmax;
        }
        for (long long bb = t; bb < bpr; bb += TPR) {
            uint32_t w[32];
            load_block<float>(s, bb, w, a32);
            exp_quant_block<F>(w, mx, row * bpr + bb, codes, scales, a32);
        }
        if constexpr (TPR > 32) __syncthreads();  // rmax is rewritten for the next row
    }
}

bool exp_quantize_supported(long long cols) { return cols > 0 && cols % 32 == 0; }

template <int F, int TPR>
static cudaError_t launch_xq_t(const float* scores, long long rows, long long cols, void* codes, void* scales,
                               cudaStream_t st) {
    auto kern = k_exp_quantize<F, TPR>;
    int dev = 0, sms = 148, per_sm = 1, l2 = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, TPR, 0);
    long long ctas = (long long)sms * (per_sm > 0 ? per_sm : 1);
    // rows in flight x row bytes <= 60% of L2, so pass 2 finds its row there
    const long long budget = (l2 > 0 ? (long long)l2 : (126LL << 20)) * 3 / 5;
    const long long by_l2 = budget / (cols * 4);
    if (by_l2 < ctas) ctas = by_l2 > sms ? by_l2 : sms;
    if (ctas > rows) ctas = rows;
    if (ctas < 1) ctas = 1;
    const bool a32 = ((reinterpret_cast<uintptr_t>(scores) | reinterpret_cast<uintptr_t>(codes)) & 31) == 0;
    kern<<<(unsigned)ctas, TPR, 0, st>>>(scores, codes, scales, rows, cols, a32);
    return cudaGetLastError();
}

// Threads per row: two to four blocks per thread, 32 to 1024 (more, smaller
// CTAs per SM overlap one row's load phase with another's compute phase).
template <int F>
static cudaError_t launch_xq(const float* scores, long long rows, long long cols, void* codes, void* scales,
                             cudaStream_t st) {
    const long long bpr = cols / 32;
    if (bpr <= 64) return launch_xq_t<F, 32>(scores, rows, cols, codes, scales, st);
    if (bpr <= 128) return launch_xq_t<F, 64>(scores, rows, cols, codes, scales, st);
    if (bpr <= 256) return launch_xq_t<F, 128>(scores, rows, cols, codes, scales, st);
    if (bpr <= 1024) return launch_xq_t<F, 256>(scores, rows, cols, codes, scales, st);
    if (bpr <= 2048) return launch_xq_t<F, 512>(scores, rows, cols, codes, scales, st);
    return launch_xq_t<F, 1024>(scores, rows, cols, codes, scales, st);
}

cudaError_t launch_exp_quantize(int fmt, const float* scores, long long rows, long long cols, void* codes,
                                void* scales, cudaStream_t st) {
    if (!exp_quantize_supported(cols)) return cudaErrorNotSupported;
    if (exp_quantize_tma_supported(fmt, scores))
        return launch_exp_quantize_tma(fmt, scores, rows, cols, codes, scales, st);
    switch (fmt) {
        case F_AXS6: return launch_xq<F_AXS6>(scores, rows, cols, codes, scales, st);
        case F_E2M3: return launch_xq<F_E2M3>(scores, rows, cols, codes, scales, st);
        case F_E3M2: return launch_xq<F_E3M2>(scores, rows, cols, codes, scales, st);
        case F_E4M3: return launch_xq<F_E4M3>(scores, rows, cols, codes, scales, st);
        case F_E2M1: return launch_xq<F_E2M1>(scores, rows, cols, codes, scales, st);
    }
    return cudaErrorInvalidValue;
}

}  // namespace mxq
