// mxq_expq_tma.cu -- the exp-then-quantize softmax stage as a bulk-copy
// pipeline (sm_100a), for the 4- and 8-bit formats (MXFP4 E2M1, the format the
// stage feeds, and MXFP8 E4M3).
//
// "EFQ-Softmax: exp-free E2M1 probabilities" explainer, Jargon and stage
// table: p = exp(s - rowmax) in higher precision, then each block of 32 keys
// gets an exponent-only scale from its own maximum and E2M1 codes. The row
// maximum must be complete before the first exponential, so a row is read
// twice: pass A for its maximum, pass B for exp + quantize.
//
// One persistent CTA per SM; a producer thread streams 64 KB stages of scores
// (4 KB per consumer warp) into a ring of three shared-memory stages with
// cp.async.bulk (the TMA engine), each stage guarded by a "full" and an "empty"
// mbarrier; sixteen consumer warps read the stages. The producer's order
// interleaves pass B of row i with pass A of row i+1 stage by stage, so HBM
// streams the next row while the current one is exponentiated; pass A's copies
// ask L2 to keep the row (evict_last), pass B's copies find it there
// (evict_first), and HBM sees each score once. The row maximum is combined
// across the consumer warps through a shared-memory slot and an mbarrier
// (double-buffered by row parity). Any row length: a row is a sequence of
// stages, the last one partial.
//
// Pass A: each consumer thread takes eight 16-byte pieces of the stage
// (conflict-free: a warp reads 512 consecutive bytes). Pass B: a thread owns a
// block of 32 keys (block_exp_quant: read in a lane-rotated order so that the
// shared-memory wavefronts are conflict-free, codes rotated back before the
// store).
//
// Every wait is bounded (one second by %globaltimer, or sooner once another
// warp has given up): a wait that runs out sets the library's device error
// word, which mxq_check_device reports as MXQ_ERR_TIMEOUT, and the CTA leaves
// after the producer has waited (bounded again) for its own copies in flight.
#include <cstdint>
#include <cuda_runtime.h>

#include "mxq_block.cuh"
#include "mxq_device.cuh"
#include "mxq_exp.cuh"
#include "mxq_internal.h"
#include "mxq_tma.cuh"

namespace mxq {

__device__ unsigned int g_device_error;  // bit 0: a bounded wait ran out

// ---- consumer work on one stage ----------------------------------------------------------
//
// A stage holds 32·CW blocks of 32 scores (CW consumer warps, 4 KB per warp).

// pass A: maximum of the stage's first n16 16-byte pieces (NaN if any is NaN);
// piece g = t + 32·CW·j, so a warp reads 512 consecutive bytes per load
template <int CW>
__device__ __forceinline__ float chunk_max(uint32_t stage, int n16, int t) {
    float m = __uint_as_float(0xFF800000u);
    if (n16 == 256 * CW) {  // a full stage: no bounds checks
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 v = lds128(stage + 16 * (t + 32 * CW * j));
            m = max3_nan(m, max3_nan(v.x, v.y, v.z), v.w);
        }
        return m;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const int g = t + 32 * CW * j;
        if (g < n16) {
            const float4 v = lds128(stage + 16 * g);
            m = max3_nan(m, max3_nan(v.x, v.y, v.z), v.w);
        }
    }
    return m;
}

// pass B: thread t owns block t of the stage. Its 128 bytes are read as eight
// 16-byte pieces, piece (c xor r) into slot c with r = lane mod 8, so the eight
// lanes that share a shared-memory wavefront hit eight different bank groups;
// maximum, exponent and rounding do not depend on the order, and the packed codes
// are permuted back (slot s holds piece s xor r) before the store.
template <int F>
__device__ __forceinline__ void block_exp_quant(uint32_t stage, bool valid, float m, long long b, void* codes,
                                                void* scales, int t) {
    const uint32_t r = (uint32_t)(t & 7);
    const uint32_t base = (stage + 128u * (uint32_t)t) ^ (16u * r);  // stage + 128 t is 128-byte aligned
    uint32_t w[32];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const float4 v = lds128(base ^ (16u * c));
        w[4 * c] = __float_as_uint(v.x);
        w[4 * c + 1] = __float_as_uint(v.y);
        w[4 * c + 2] = __float_as_uint(v.z);
        w[4 * c + 3] = __float_as_uint(v.w);
    }
    exp_values<32>(w, m);
    float q[11];
#pragma unroll
    for (int i = 0; i < 10; ++i)
        q[i] = max3_nan(__uint_as_float(w[3 * i]), __uint_as_float(w[3 * i + 1]), __uint_as_float(w[3 * i + 2]));
    q[10] = max_nan(__uint_as_float(w[30]), __uint_as_float(w[31]));
    float pm = max3_nan(max3_nan(q[0], q[1], q[2]), max3_nan(q[3], q[4], q[5]), max3_nan(q[6], q[7], q[8]));
    pm = max3_nan(pm, q[9], q[10]);  // p >= 0 or NaN
    const uint32_t byte = scale_byte<F>(__float_as_uint(pm) & 0x7FFFFFFFu);
    const unsigned long long inv2 = dup2(inv_scale(byte));
    const uint32_t keep = byte == 0xFFu ? 0u : 0xFFFFFFFFu;
    float a[32];
#pragma unroll
    for (int i = 0; i < 16; ++i) upk(f2mul(pk(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1])), inv2), a[2 * i], a[2 * i + 1]);
    if (!valid) return;
    if constexpr (F == F_E2M1) {
        // word i = codes of slots 2i, 2i+1; output word j = pieces 2j, 2j+1 = word j ^ (r >> 1),
        // its two halves swapped when r is odd
        uint32_t h[4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
            h[i] = __byte_perm(cvt8_e2m1(a[8 * i], a[8 * i + 1], a[8 * i + 2], a[8 * i + 3], a[8 * i + 4], a[8 * i + 5],
                                         a[8 * i + 6], a[8 * i + 7]),
                               0, (r & 1) ? 0x1032 : 0x3210);
        const bool x1 = r & 2, x2 = r & 4;
        const uint32_t g0 = x1 ? h[1] : h[0], g1 = x1 ? h[0] : h[1], g2 = x1 ? h[3] : h[2], g3 = x1 ? h[2] : h[3];
        st_stream_v4(reinterpret_cast<char*>(codes) + b * 16,
                     make_uint4((x2 ? g2 : g0) & keep, (x2 ? g3 : g1) & keep, (x2 ? g0 : g2) & keep, (x2 ? g1 : g3) & keep));
    } else {
        // word c = codes of slot c; output word j = word j ^ r
        uint32_t h[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) h[c] = cvt4_e4m3(a[4 * c], a[4 * c + 1], a[4 * c + 2], a[4 * c + 3]);
#pragma unroll
        for (int bit = 0; bit < 3; ++bit) {
            const int sh = 1 << bit;
            const bool on = (r >> bit) & 1;
            uint32_t u[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) u[j] = on ? h[j ^ sh] : h[j];
#pragma unroll
            for (int j = 0; j < 8; ++j) h[j] = u[j];
        }
        char* p = reinterpret_cast<char*>(codes) + b * 32;
        st_stream_v4(p, make_uint4(h[0] & keep, h[1] & keep, h[2] & keep, h[3] & keep));
        st_stream_v4(p + 16, make_uint4(h[4] & keep, h[5] & keep, h[6] & keep, h[7] & keep));
    }
    reinterpret_cast<uint8_t*>(scales)[b] = (uint8_t)byte;
}

// ---- the kernel ---------------------------------------------------------------------------

template <int F, int CW, int NS>
__global__ void __launch_bounds__(32 * (CW + 1), 1) k_exp_quantize_tma(const float* __restrict__ scores, void* codes,
                                                                  void* scales, long long rows, long long cols,
                                                                  unsigned int* err) {
    constexpr int CH = CW * 4096;  // stage bytes: 32·CW blocks of 128 bytes
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) unsigned long long full[NS], empty[NS], red[2];
    __shared__ float part[2][CW];
    __shared__ int abort_flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long G = gridDim.x;
    const long long n = rows > (long long)blockIdx.x ? (rows - 1 - blockIdx.x) / G + 1 : 0;  // rows of this CTA
    const long long rowbytes = cols * 4, bpr = cols / 32;
    const int nc = (int)((rowbytes + CH - 1) / CH);
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), CW);
        }
        mbar_init(smem_u32(&red[0]), CW);
        mbar_init(smem_u32(&red[1]), CW);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (n == 0) return;
    volatile int* ab = &abort_flag;
    const uint32_t ring0 = smem_u32(ring);
    auto chunk_bytes = [&](int j) { return (int)min((long long)CH, rowbytes - (long long)j * CH); };

    if (warp == CW) {  // producer: one thread issues every copy
        if (lane != 0) return;
        const unsigned long long keep = l2_policy_keep(), strm = l2_policy_stream();
        long long k = 0;
        auto issue = [&](long long i, int j, bool pass_a) -> bool {
            const int s = (int)(k % NS);
            if (!mbar_wait(smem_u32(&empty[s]), ((uint32_t)(k / NS) & 1u) ^ 1u, ab, err)) return false;
            const long long r = blockIdx.x + i * G;
            const uint32_t bytes = (uint32_t)chunk_bytes(j);
            mbar_expect_tx(smem_u32(&full[s]), bytes);
            bulk_load(ring0 + s * CH, reinterpret_cast<const char*>(scores) + r * rowbytes + (long long)j * CH, bytes,
                      smem_u32(&full[s]), pass_a ? keep : strm);
            ++k;
            return true;
        };
        bool ok = true;
        for (int j = 0; j < nc && ok; ++j) ok = issue(0, j, true);
        for (long long i = 0; i + 1 < n && ok; ++i)
            for (int j = 0; j < nc && ok; ++j) ok = issue(i, j, false) && issue(i + 1, j, true);
        for (int j = 0; j < nc && ok; ++j) ok = issue(n - 1, j, false);
        if (!ok) {
            // gave up: let the copies still in flight land before the CTA's shared memory goes away
            for (long long q = k > NS ? k - NS : 0; q < k; ++q) {
                const uint32_t bar = smem_u32(&full[q % NS]), par = (uint32_t)(q / NS) & 1u;
                const unsigned long long t0 = global_ns();
                while (!mbar_test(bar, par) && global_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
        return;
    }

    // consumers: tid 0 .. 32·CW - 1
    long long k = 0;
    auto acquire = [&](int& s) -> bool {
        s = (int)(k % NS);
        const bool ok = mbar_wait(smem_u32(&full[s]), (uint32_t)(k / NS) & 1u, ab, err);
        return __all_sync(0xFFFFFFFFu, ok);
    };
    auto release = [&](int s) {
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
        ++k;
    };
    // row maximum over the consumer warps; q = this CTA's row counter (slot q & 1)
    auto reduce = [&](float acc, long long q, float& m) -> bool {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc = max_nan(acc, __shfl_xor_sync(0xFFFFFFFFu, acc, o));
        const int p = (int)(q & 1);
        if (lane == 0) {
            part[p][warp] = acc;
            mbar_arrive(smem_u32(&red[p]));
        }
        const bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&red[p]), (uint32_t)(q >> 1) & 1u, ab, err));
        volatile float* pp = part[p];
        m = pp[0];
#pragma unroll
        for (int w = 1; w < CW; ++w) m = max_nan(m, pp[w]);
        return ok;
    };
    const float NEG_INF = __uint_as_float(0xFF800000u);
    float acc = NEG_INF, mB = 0.0f;
    int s;
    for (int j = 0; j < nc; ++j) {  // pass A of the first row
        if (!acquire(s)) return;
        acc = max_nan(acc, chunk_max<CW>(ring0 + s * CH, chunk_bytes(j) / 16, tid));
        release(s);
    }
    if (!reduce(acc, 0, mB)) return;
    for (long long i = 0; i + 1 < n; ++i) {  // pass B of row i, pass A of row i + 1, stage by stage
        const long long blk_row = (blockIdx.x + i * G) * bpr;
        acc = NEG_INF;
        for (int j = 0; j < nc; ++j) {
            if (!acquire(s)) return;
            block_exp_quant<F>(ring0 + s * CH, tid < chunk_bytes(j) / 128, mB, blk_row + (long long)j * 32 * CW + tid,
                               codes, scales, tid);
            release(s);
            if (!acquire(s)) return;
            acc = max_nan(acc, chunk_max<CW>(ring0 + s * CH, chunk_bytes(j) / 16, tid));
            release(s);
        }
        if (!reduce(acc, i + 1, mB)) return;
    }
    const long long blk_row = (blockIdx.x + (n - 1) * G) * bpr;
    for (int j = 0; j < nc; ++j) {  // pass B of the last row
        if (!acquire(s)) return;
        block_exp_quant<F>(ring0 + s * CH, tid < chunk_bytes(j) / 128, mB, blk_row + (long long)j * 32 * CW + tid,
                           codes, scales, tid);
        release(s);
    }
}

// ---- launch -----------------------------------------------------------------------------

// Shape by measurement on B200 (fp32 4096 x 32768 scores -> MXFP4, fraction of the copy peak):
// 16 consumer warps and three 64 KB stages, one CTA per SM: 0.72; 8 warps x 3 x 32 KB, two CTAs
// per SM: 0.72; 8 warps x 6 x 32 KB, one CTA: 0.62; 4 warps x 3 x 16 KB, four CTAs: 0.70. An L2
// prefetch of the row after next did not help (0.70). Keeping the row resident in shared memory
// and freeing it in pass B, so that each score crosses L2 -> SM once, was slower (0.54): the
// next row cannot stream in while the current one fills two thirds of the ring.
constexpr int kXWarps = 16, kXStages = 3;

bool exp_quantize_tma_supported(int fmt, const void* scores) {
    return (fmt == F_E2M1 || fmt == F_E4M3) && (reinterpret_cast<uintptr_t>(scores) & 15) == 0;
}

template <int F, int CW, int NS>
static cudaError_t launch_xt(const float* scores, long long rows, long long cols, void* codes, void* scales,
                             cudaStream_t st) {
    auto kern = k_exp_quantize_tma<F, CW, NS>;
    const int smem = NS * CW * 4096, threads = 32 * (CW + 1);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148, per_sm = 1;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem);
    long long ctas = (long long)sms * (per_sm > 0 ? per_sm : 1);
    if (ctas > rows) ctas = rows;
    unsigned int* err = nullptr;
    if ((e = device_error_word(&err)) != cudaSuccess) return e;
    kern<<<(unsigned)ctas, threads, smem, st>>>(scores, codes, scales, rows, cols, err);
    return cudaGetLastError();
}

cudaError_t launch_exp_quantize_tma(int fmt, const float* scores, long long rows, long long cols, void* codes,
                                    void* scales, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (fmt == F_E2M1) return launch_xt<F_E2M1, kXWarps, kXStages>(scores, rows, cols, codes, scales, st);
    if (fmt == F_E4M3) return launch_xt<F_E4M3, kXWarps, kXStages>(scores, rows, cols, codes, scales, st);
    return cudaErrorInvalidValue;
}

// Self-test of the bounded wait: one warp waits on an mbarrier that nothing
// arrives at; the wait gives up after limit_ns and sets the device error word.
__global__ void __launch_bounds__(32) k_selftest_timeout(unsigned long long limit_ns, unsigned int* err) {
    __shared__ __align__(8) unsigned long long bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    mbar_wait(smem_u32(&bar), 0, &abort_flag, err, limit_ns);
}

cudaError_t launch_selftest_timeout(unsigned long long limit_ns, cudaStream_t st) {
    unsigned int* err = nullptr;
    cudaError_t e = device_error_word(&err);
    if (e != cudaSuccess) return e;
    k_selftest_timeout<<<1, 32, 0, st>>>(limit_ns, err);
    return cudaGetLastError();
}

// address of the device error word on the current device (cached per device)
cudaError_t device_error_word(unsigned int** p) {
    static unsigned int* addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!addr[dev]) {
        void* a = nullptr;
        if ((e = cudaGetSymbolAddress(&a, g_device_error)) != cudaSuccess) return e;
        addr[dev] = static_cast<unsigned int*>(a);
    }
    *p = addr[dev];
    return cudaSuccess;
}

cudaError_t read_device_error(unsigned int* value, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
    if (e != cudaSuccess || !clear || *value == 0) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

}  // namespace mxq
