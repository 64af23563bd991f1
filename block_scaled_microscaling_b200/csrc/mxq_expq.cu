// mxq_expq.cu -- fused exp-then-quantize softmax probability stage (sm_100a).
//
// "EFQ-Softmax: exp-free E2M1 probabilities" explainer, Jargon (shifted scores,
// exp-then-quantize, MXFP4, microscaling block) and its stage table: the
// conventional path exponentiates the row-max-shifted scores in higher
// precision, materializes the probability block and quantizes it to E2M1 with
// an exponent-only scale from each 32-key block's maximum. Here the block is
// never materialized: scores are read once and probabilities live in registers.
//
// A thread-block cluster works on one row at a time; the row is split into
// C contiguous runs of whole 32-key blocks, one run per CTA, one block per
// thread (read as four 32-byte sectors). Clusters are persistent: each walks
// rows with a stride, prefetching its next row's blocks into a second register
// buffer while the current row is reduced and quantized. The row maximum goes
// thread -> warp -> CTA (shared memory) -> cluster (distributed shared memory,
// one cluster barrier per row); then each thread exponentiates its 32 keys with
// packed fp32x2 arithmetic and quantizes its block. C <= 8 (portable cluster)
// for rows up to 131072 keys, 16 (non-portable) up to 262144.
#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_runtime.h>

#include "mxq_block.cuh"
#include "mxq_device.cuh"
#include "mxq_internal.h"

namespace cg = cooperative_groups;

namespace mxq {

constexpr int kMaxThreads = 512;  // two 32-value register buffers per thread need <= 128 registers

// The library's own fp32 exponential (the same definition the CPU oracle
// implements independently):
//   t = RN(d * L2E), n = t rounded to an integer, ties to even,
//   r = RN(d - n*LN2_HI) and r = RN(r - n*LN2_LO), both fused (Cody & Waite),
//   p = Horner over 1/k!, k = 7..0, one fused multiply-add per step,
//   e^d = p * 2^n (outside 2^[-126,127] as two exact-then-rounded products
//   through 2^(n+-64)); t < -160 -> +0, t > 160 -> +inf, NaN -> NaN.
// L2E = 1/ln2 and LN2_LO = ln2 - LN2_HI rounded to fp32, LN2_HI = ln 2 cut to
// 16 significant bits, 1/k! rounded to fp32.
constexpr float kL2E = 0x1.715476p+0f, kLn2Hi = 0x1.62e4p-1f, kLn2Lo = 0x1.7f7d1cp-20f;
constexpr float kC0 = 0x1p+0f, kC1 = 0x1p+0f, kC2 = 0x1p-1f, kC3 = 0x1.555556p-3f, kC4 = 0x1.555556p-5f,
                kC5 = 0x1.111112p-7f, kC6 = 0x1.6c16c2p-10f, kC7 = 0x1.a01a02p-13f;
constexpr float kRound = 12582912.0f;  // 1.5 * 2^23: x + kRound rounds x to an integer (|x| < 2^22)

__device__ __forceinline__ float pow2i(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }

// general form, any input
__device__ __forceinline__ float expf_mxq(float d) {
    if (d != d) return d;
    float t = __fmul_rn(d, kL2E);
    if (t < -160.0f) return 0.0f;
    if (t > 160.0f) return __uint_as_float(0x7F800000u);
    float n = __fsub_rn(__fadd_rn(t, kRound), kRound);  // rint(t), ties to even
    float r = __fmaf_rn(-n, kLn2Hi, d);
    r = __fmaf_rn(-n, kLn2Lo, r);
    float p = kC7;
    p = __fmaf_rn(p, r, kC6);
    p = __fmaf_rn(p, r, kC5);
    p = __fmaf_rn(p, r, kC4);
    p = __fmaf_rn(p, r, kC3);
    p = __fmaf_rn(p, r, kC2);
    p = __fmaf_rn(p, r, kC1);
    p = __fmaf_rn(p, r, kC0);
    int ni = (int)n;
    if (ni < -126) return __fmul_rn(__fmul_rn(p, pow2i(ni + 64)), pow2i(-64));
    if (ni > 127) return __fmul_rn(__fmul_rn(p, pow2i(ni - 64)), pow2i(64));
    return __fmul_rn(p, pow2i(ni));
}

// Same function on a packed pair of shifted scores d = (lo, hi), valid when both
// t = d*L2E lie in [-126, 127] (then 2^n is one normal fp32 and one product
// suffices): n from the 1.5*2^23 add, 2^n's bits from that sum's bits.
__device__ __forceinline__ unsigned long long expf_mxq2(unsigned long long d) {
    const unsigned long long tm = f2add(f2mul(d, dup2(kL2E)), dup2(kRound));
    const unsigned long long nn = f2sub(dup2(kRound), tm);  // -n, exact
    unsigned long long r = f2fma(nn, dup2(kLn2Hi), d);
    r = f2fma(nn, dup2(kLn2Lo), r);
    unsigned long long p = f2fma(dup2(kC7), r, dup2(kC6));
    p = f2fma(p, r, dup2(kC5));
    p = f2fma(p, r, dup2(kC4));
    p = f2fma(p, r, dup2(kC3));
    p = f2fma(p, r, dup2(kC2));
    p = f2fma(p, r, dup2(kC1));
    p = f2fma(p, r, dup2(kC0));
    float a, b;
    upk(tm, a, b);
    // bits(tm) = 0x4B400000 + n, so (n + 127) << 23 = bits(tm) * 2^23 + 0x3F800000 (mod 2^32)
    const float sa = __uint_as_float(__float_as_uint(a) * 0x800000u + 0x3F800000u);
    const float sb = __uint_as_float(__float_as_uint(b) * 0x800000u + 0x3F800000u);
    return f2mul(p, pk(sa, sb));
}

// One row's work for one CTA once its block is in registers: row maximum
// through the cluster, then exp + quantize of the thread's block. `it` picks
// the maximum slot (double-buffered, so one cluster barrier per row suffices:
// a CTA can write slot it&1 again only after the next row's barrier, which
// every CTA reaches after its reads of this row's slots).
template <int F>
__device__ __forceinline__ void exp_row(uint32_t (&w)[32], bool valid, long long blk, int it, int C,
                                        cg::cluster_group& cl, float* wmax, float* slot, float* row_max,
                                        void* codes, void* scales, bool a32) {
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const float NEG_INF = __uint_as_float(0xFF800000u);
    float mx = NEG_INF;
    if (valid) {
        float m[11];
#pragma unroll
        for (int i = 0; i < 10; ++i)
            m[i] = max3_nan(__uint_as_float(w[3 * i]), __uint_as_float(w[3 * i + 1]), __uint_as_float(w[3 * i + 2]));
        m[10] = max_nan(__uint_as_float(w[30]), __uint_as_float(w[31]));
        mx = max3_nan(max3_nan(m[0], m[1], m[2]), max3_nan(m[3], m[4], m[5]), max3_nan(m[6], m[7], m[8]));
        mx = max3_nan(mx, m[9], m[10]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max_nan(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
    if (lane == 0) wmax[warp] = mx;
    __syncthreads();
    if (warp == 0) {
        const int nw = blockDim.x >> 5;
        float v = lane < nw ? wmax[lane] : NEG_INF;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = max_nan(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
        if (lane == 0) {
            slot[it & 1] = v;
            cluster_publish_fence();
        }
    }
    cluster_arrive_relaxed();
    cluster_wait();
    if (warp == 0) {  // the C remote maxima, read in parallel by lanes 0..C-1
        float v = lane < C ? cl.map_shared_rank(slot, lane)[it & 1] : NEG_INF;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = max_nan(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
        if (lane == 0) *row_max = v;
    }
    __syncthreads();
    if (!valid) return;
    const float mr = *row_max;

    // shifted scores, then e^d (packed path unless some t < -126 in this block)
    float tmin = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        unsigned long long d = f2sub(pk(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1])), dup2(mr));
        float a, b;
        upk(d, a, b);
        w[2 * i] = __float_as_uint(a);
        w[2 * i + 1] = __float_as_uint(b);
        tmin = fminf(tmin, fminf(a, b));
    }
    if (__fmul_rn(tmin, kL2E) >= -126.0f) {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            float a, b;
            upk(expf_mxq2(pk(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1]))), a, b);
            w[2 * i] = __float_as_uint(a);
            w[2 * i + 1] = __float_as_uint(b);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(expf_mxq(__uint_as_float(w[i])));
    }
    // p >= 0 or NaN: a NaN-propagating max gives the block maximum (or NaN)
    float q[11];
#pragma unroll
    for (int i = 0; i < 10; ++i) q[i] = max3_nan(__uint_as_float(w[3 * i]), __uint_as_float(w[3 * i + 1]), __uint_as_float(w[3 * i + 2]));
    q[10] = max_nan(__uint_as_float(w[30]), __uint_as_float(w[31]));
    float pm = max3_nan(max3_nan(q[0], q[1], q[2]), max3_nan(q[3], q[4], q[5]), max3_nan(q[6], q[7], q[8]));
    pm = max3_nan(pm, q[9], q[10]);
    const uint32_t byte = scale_byte<F>(__float_as_uint(pm) & 0x7FFFFFFFu);
    uint32_t out[8];
    encode_block<F, float>(w, byte, out);
    store_payload<F>(codes, blk, out, a32);
    store_scale<F>(scales, blk, byte);
}

// Persistent clusters: cluster k handles rows k, k + G, k + 2G, ...; each
// thread prefetches its block of the next row into a second register buffer
// while the current row is reduced and quantized.
template <int F>
__global__ void __launch_bounds__(kMaxThreads) k_exp_quantize(const float* __restrict__ scores, void* __restrict__ codes,
                                                             void* __restrict__ scales, long long rows, long long cols,
                                                             bool a32) {
    __shared__ float wmax[32];
    __shared__ float slot[2];
    __shared__ float row_max;

    cg::cluster_group cl = cg::this_cluster();
    const int C = (int)cl.num_blocks();
    const int c = (int)cl.block_rank();
    const long long G = gridDim.x / C;
    const long long bpr = cols / 32;
    const long long b0 = (long long)c * bpr / C, b1 = (long long)(c + 1) * bpr / C;
    const bool valid = (long long)threadIdx.x < b1 - b0;
    const long long col_blk = b0 + threadIdx.x;

    long long r = blockIdx.x / C;
    uint32_t A[32], B[32];
    if (valid && r < rows) load_block<float>(scores, r * bpr + col_blk, A, a32);
    int it = 0;
    while (r < rows) {
        if (valid && r + G < rows) load_block<float>(scores, (r + G) * bpr + col_blk, B, a32);
        exp_row<F>(A, valid, r * bpr + col_blk, it, C, cl, wmax, slot, &row_max, codes, scales, a32);
        r += G;
        ++it;
        if (r >= rows) break;
        if (valid && r + G < rows) load_block<float>(scores, (r + G) * bpr + col_blk, A, a32);
        exp_row<F>(B, valid, r * bpr + col_blk, it, C, cl, wmax, slot, &row_max, codes, scales, a32);
        r += G;
        ++it;
    }
    cl.sync();  // no CTA leaves while another may still read its slots
}

bool exp_quantize_supported(long long cols) { return cols > 0 && cols % 32 == 0 && cols <= 262144; }

template <int F>
static cudaError_t launch_xq(const float* scores, long long rows, long long cols, void* codes, void* scales,
                             cudaStream_t st) {
    const long long bpr = cols / 32;
    long long C = (bpr + 127) / 128;  // about 128 blocks (4096 keys) per CTA
    if (C > 8) C = 8;                 // portable cluster size
    if (C < 1) C = 1;
    if ((bpr + C - 1) / C > kMaxThreads) C = 16;  // non-portable size, long rows only
    const long long per_cta = (bpr + C - 1) / C;
    const long long nt = (per_cta + 31) / 32 * 32;
    if (nt > kMaxThreads) return cudaErrorNotSupported;
    const bool a32 = ((reinterpret_cast<uintptr_t>(scores) | reinterpret_cast<uintptr_t>(codes)) & 31) == 0;

    cudaLaunchConfig_t cfg = {};
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
    if (C > 8) {
        cudaError_t e = cudaFuncSetAttribute(k_exp_quantize<F>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (e != cudaSuccess) return e;
    }
    // as many clusters as fit on the GPU at once (each then loops over rows)
    cfg.gridDim = dim3((unsigned)(C * 1024), 1, 1);
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, k_exp_quantize<F>, &cfg) != cudaSuccess || active < 1) {
        cudaGetLastError();
        active = 148;
    }
    long long G = rows < active ? rows : active;
    cfg.gridDim = dim3((unsigned)(G * C), 1, 1);
    return cudaLaunchKernelEx(&cfg, k_exp_quantize<F>, scores, codes, scales, rows, cols, a32);
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
