// mxq_expq.cu -- fused exp-then-quantize softmax probability stage (sm_100a).
//
// "EFQ-Softmax: exp-free E2M1 probabilities" explainer, Jargon (shifted scores,
// exp-then-quantize, MXFP4, microscaling block) and its stage table: the
// conventional path exponentiates the row-max-shifted scores in higher
// precision, materializes the probability block and quantizes it to E2M1 with
// an exponent-only scale from each 32-key block's maximum. Here the block is
// never materialized: scores are read once, probabilities live in registers.
//
// One thread-block cluster per row. The row is split into C <= 8 contiguous
// runs of whole 32-key blocks, one per CTA; each thread keeps up to R = 4
// 16-byte chunks (16 scores) in registers. The row maximum is reduced warp ->
// CTA (shared memory) -> cluster (distributed shared memory, two cluster
// barriers), then each chunk goes through exp, the 8-lane block amax
// butterfly, the block scale, rounding and packing, and leaves through a
// per-warp staging slice. cols <= C*1024*16 = 131072 keys per row.
#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_runtime.h>

#include "mxq_device.cuh"
#include "mxq_internal.h"

namespace cg = cooperative_groups;

namespace mxq {

constexpr int kR = 4;            // 16-byte chunks per thread
constexpr int kMaxCluster = 8;   // portable cluster size
constexpr int kMaxThreads = 1024;

// The library's own fp32 exponential (the same definition the CPU oracle
// implements independently):
//   t = RN(d * L2E), n = rint(t) (ties to even),
//   r = RN(d - n*LN2_HI) and r = RN(r - n*LN2_LO), both fused (Cody & Waite),
//   p = Horner over 1/k!, k = 7..0, one fused multiply-add per step,
//   e^d = p * 2^n (split in two exact-then-rounded products outside
//   2^[-126,127]); t < -160 -> +0, t > 160 -> +inf, NaN -> NaN.
// L2E = 1/ln2 and LN2_LO = ln2 - LN2_HI rounded to fp32, LN2_HI = ln 2 cut to
// 16 significant bits, 1/k! rounded to fp32.
__device__ __forceinline__ float pow2i(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }

__device__ __forceinline__ float expf_mxq(float d) {
    const float L2E = 0x1.715476p+0f, LN2_HI = 0x1.62e4p-1f, LN2_LO = 0x1.7f7d1cp-20f;
    if (d != d) return d;
    float t = __fmul_rn(d, L2E);
    if (t < -160.0f) return 0.0f;
    if (t > 160.0f) return __uint_as_float(0x7F800000u);
    float n = rintf(t);
    float r = __fmaf_rn(-n, LN2_HI, d);
    r = __fmaf_rn(-n, LN2_LO, r);
    float p = 0x1.a01a02p-13f;
    p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);
    p = __fmaf_rn(p, r, 0x1.111112p-7f);
    p = __fmaf_rn(p, r, 0x1.555556p-5f);
    p = __fmaf_rn(p, r, 0x1.555556p-3f);
    p = __fmaf_rn(p, r, 0x1p-1f);
    p = __fmaf_rn(p, r, 0x1p+0f);
    p = __fmaf_rn(p, r, 0x1p+0f);
    int ni = (int)n;
    if (ni < -126) return __fmul_rn(__fmul_rn(p, pow2i(ni + 64)), pow2i(-64));
    if (ni > 127) return __fmul_rn(__fmul_rn(p, pow2i(ni - 64)), pow2i(64));
    return __fmul_rn(p, pow2i(ni));
}

template <int F>
__global__ void __launch_bounds__(kMaxThreads) k_exp_quantize(const float* __restrict__ scores,
                                                             uint8_t* __restrict__ codes,
                                                             void* __restrict__ scales, long long cols) {
    constexpr int W = Fmt<F>::W;
    constexpr int LB = 4 * W / 8;  // code bytes per 16-byte chunk
    constexpr int PB = payload<F>();
    __shared__ float wmax[32];
    __shared__ int wnan[32];
    __shared__ float cta_max;
    __shared__ float row_max;
    __shared__ __align__(16) uint8_t stage[32][32 * LB];

    cg::cluster_group cl = cg::this_cluster();
    const int C = (int)cl.num_blocks();
    const int c = (int)cl.block_rank();
    const long long row = blockIdx.x / C;
    const long long bpr = cols / 32;
    const long long b0 = (long long)c * bpr / C, b1 = (long long)(c + 1) * bpr / C;
    const int nch = (int)(b1 - b0) * 8;  // chunks owned by this CTA
    const float* s = scores + row * cols + b0 * 32;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5, NT = blockDim.x;
    const float NEG_INF = __uint_as_float(0xFF800000u);

    float x[kR][4];
    float m = NEG_INF;
    int nan = 0;
#pragma unroll
    for (int j = 0; j < kR; ++j) {
        const int k = t + j * NT;
        uint4 v = k < nch ? ld_stream_v4(s + 4 * k) : make_uint4(0xFF800000u, 0xFF800000u, 0xFF800000u, 0xFF800000u);
        x[j][0] = __uint_as_float(v.x);
        x[j][1] = __uint_as_float(v.y);
        x[j][2] = __uint_as_float(v.z);
        x[j][3] = __uint_as_float(v.w);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            nan |= x[j][i] != x[j][i];
            m = fmaxf(m, x[j][i]);
        }
    }
    // row maximum: warp, CTA, cluster
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    nan = __any_sync(0xFFFFFFFFu, nan);
    if (lane == 0) {
        wmax[warp] = m;
        wnan[warp] = nan;
    }
    __syncthreads();
    if (warp == 0) {
        const int nw = NT >> 5;
        float mm = lane < nw ? wmax[lane] : NEG_INF;
        int nn = lane < nw ? wnan[lane] : 0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mm = fmaxf(mm, __shfl_xor_sync(0xFFFFFFFFu, mm, o));
        nn = __any_sync(0xFFFFFFFFu, nn);
        if (lane == 0) cta_max = nn ? __uint_as_float(0x7FC00000u) : mm;
    }
    cl.sync();
    if (t == 0) {
        float mm = NEG_INF;
        int nn = 0;
        for (int r = 0; r < C; ++r) {
            float v = *cl.map_shared_rank(&cta_max, r);
            nn |= v != v;
            mm = fmaxf(mm, v);
        }
        row_max = nn ? __uint_as_float(0x7FC00000u) : mm;
    }
    cl.sync();  // remote reads done before any CTA may exit; row_max visible
    const float mr = row_max;

    uint8_t* st = stage[warp];
    uint8_t* gcodes = codes + (row * bpr + b0) * PB;
#pragma unroll
    for (int j = 0; j < kR; ++j) {
        const int k = t + j * NT;
        float p[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) p[i] = expf_mxq(__fsub_rn(x[j][i], mr));
        uint32_t am = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) am = max(am, __float_as_uint(p[i]) & 0x7FFFFFFFu);
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
        const uint32_t byte = scale_byte<F>(am);
        const float inv = inv_scale(byte);
        mul2(p[0], p[1], inv);
        mul2(p[2], p[3], inv);
        uint32_t cw[1];
        encode<F, 4>(p, cw);
        uint32_t w = byte == 0xFFu ? 0u : cw[0];
        if constexpr (W == 6) {
            w = pack6x4(w);
            st[lane * 3] = (uint8_t)w;
            st[lane * 3 + 1] = (uint8_t)(w >> 8);
            st[lane * 3 + 2] = (uint8_t)(w >> 16);
        } else if constexpr (W == 4) {
            *reinterpret_cast<uint16_t*>(st + lane * 2) = (uint16_t)w;
        } else {
            *reinterpret_cast<uint32_t*>(st + lane * 4) = w;
        }
        if ((lane & 7) == 0 && k < nch) {
            const long long b = row * bpr + b0 + k / 8;
            if constexpr (Fmt<F>::FIXED) reinterpret_cast<uint16_t*>(scales)[b] = (uint16_t)byte;
            else reinterpret_cast<uint8_t*>(scales)[b] = (uint8_t)byte;
        }
        __syncwarp();
        const int k0 = warp * 32 + j * NT;  // first chunk of this warp's row slice
        const int nvalid = max(0, min(32, nch - k0));
        const int nbytes = nvalid * LB;      // multiple of 8 (whole blocks)
        if (8 * lane < nbytes)
            *reinterpret_cast<uint2*>(gcodes + (long long)k0 * LB + 8 * lane) =
                *reinterpret_cast<const uint2*>(st + 8 * lane);
        __syncwarp();
    }
}

bool exp_quantize_supported(long long cols) { return cols > 0 && cols % 32 == 0 && cols <= 131072; }

template <int F>
static cudaError_t launch_xq(const float* scores, long long rows, long long cols, void* codes, void* scales,
                             cudaStream_t st) {
    const long long bpr = cols / 32;
    int C = (int)((cols + 4095) / 4096);
    if (C > kMaxCluster) C = kMaxCluster;
    if (C < 1) C = 1;
    const long long max_blocks = (bpr + C - 1) / C;
    const long long chunks = max_blocks * 8;
    long long nt = (chunks + kR - 1) / kR;
    nt = (nt + 31) / 32 * 32;
    if (nt > kMaxThreads) return cudaErrorNotSupported;
    if (rows * C > 0x7FFFFFFFLL) return cudaErrorNotSupported;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(rows * C), 1, 1);
    cfg.blockDim = dim3((unsigned)nt, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_exp_quantize<F>, scores, reinterpret_cast<uint8_t*>(codes), scales, cols);
}

cudaError_t launch_exp_quantize(int fmt, const float* scores, long long rows, long long cols, void* codes,
                                void* scales, cudaStream_t st) {
    if (!exp_quantize_supported(cols)) return cudaErrorNotSupported;
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
