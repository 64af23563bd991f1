// mxq_expq_tma.cu -- the exp-then-quantize softmax stage as a bulk-copy
// pipeline (sm_100a), for every format (MXFP4 E2M1 is the one the stage feeds).
//
// "EFQ-Softmax: exp-free E2M1 probabilities" explainer, Jargon and stage
// table: p = exp(s - rowmax) in higher precision, then each block of 32 keys
// gets an exponent-only scale from its own maximum and E2M1 codes. The row
// maximum must be complete before the first exponential, so a row is read
// twice: pass A for its maximum, pass B for exp + quantize.
//
// One persistent CTA per SM walks its rows (row blockIdx.x + i * gridDim.x) with
// three warp roles:
//  - a producer thread streams every row, in order, through a ring of 32 KB
//    shared-memory stages with cp.async.bulk (the TMA engine), each stage guarded
//    by a "full" and an "empty" mbarrier; the copies ask L2 to keep the row
//    (evict_last). Before the first stage of row i it waits until the consumers
//    have finished row i - LEAD, which bounds the rows a CTA holds in L2;
//  - MW maximum warps take each stage as soon as it lands, fold it into the row
//    maximum and free it, so the ring refills at once and HBM always has the
//    whole ring in flight; at the end of a row they combine their partial maxima
//    and publish the row maximum in one of four slots (mbarrier "mready");
//  - CW consumer warps (pass B): for row i they wait for its maximum, then each
//    thread reads blocks of 32 scores straight from L2 with 32-byte loads (marked
//    evict_first: last use), exponentiates and quantizes them in registers and
//    stores codes and scales; then they signal "bfree" for the row.
// HBM therefore reads each score once, and the HBM stream never waits for the
// exponentials of earlier rows except through the LEAD bound. Any row length: a
// row is a sequence of stages, the last one partial.
//
// The exp-free E2M1 rule runs in the same kernel on long rows, and on rows of up
// to 128 KB in a row-resident variant (k_exp_free_res) that keeps the row in
// shared memory between its maximum and its codes, so each score crosses L2 -> SM
// once.
//
// Every wait is bounded (one second by %globaltimer, or sooner once another
// warp has given up): a wait that runs out sets the library's device error
// word, which mxq_check_device reports as MXQ_ERR_TIMEOUT, and the CTA leaves
// after the producer has waited (bounded again) for its own copies in flight.
#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "mxq_block.cuh"
#include "mxq_device.cuh"
#include "mxq_exp.cuh"
#include "mxq_internal.h"
#include "mxq_tma.cuh"

namespace mxq {

__device__ unsigned int g_device_error;  // bit 0: a bounded wait ran out

constexpr int kXStageBytes = 32768;  // one ring stage: 256 blocks of 32 scores

// maximum of the stage's first n16 16-byte pieces (NaN if any is NaN); thread t of
// the NT maximum threads takes pieces t + NT·j, so a warp reads 512 consecutive bytes
template <int NT, int SB = kXStageBytes>
__device__ __forceinline__ float stage_max(uint32_t stage, int n16, int t) {
    constexpr int PER = SB / 16 / NT;
    float m = __uint_as_float(0xFF800000u);
    if (n16 == SB / 16) {  // a full stage: no bounds checks
#pragma unroll 8
        for (int j = 0; j < PER; ++j) {
            const float4 v = lds128(stage + 16 * (t + NT * j));
            m = max3_nan(m, max3_nan(v.x, v.y, v.z), v.w);
        }
        return m;
    }
    for (int j = 0; j < PER; ++j) {
        const int g = t + NT * j;
        if (g < n16) {
            const float4 v = lds128(stage + 16 * g);
            m = max3_nan(m, max3_nan(v.x, v.y, v.z), v.w);
        }
    }
    return m;
}

// named barrier among the maximum warps (id 1)
__device__ __forceinline__ void named_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ---- exp-free E2M1 rule ------------------------------------------------------------------
//
// "EFQ-Softmax: exp-free E2M1 probabilities", opening paragraph and the paragraph on the
// per-block rule: each microscaling block takes an exponent-only scale from its local maximum,
// normalizes the shifted scores with it and maps them to nonnegative E2M1 codes with one affine
// rule; no exponential. The page gives no constants; the library's reading (the oracle states
// the same rule independently):
//   u = RN(RN(s - m) * L2E), u_max = max over the block, Es = clamp(floor(u_max) - 2, -127, 127),
//   w = RN(2u - 2Es) (one fused multiply-add), code = clamp(rint(w) + 2, 0, 7), ties to even.
// rint(w) + 2 for w clamped to [-2, 5] is the low byte of RN(w + 1.5 * 2^23 + 2); the codes of
// eight keys leave as one word (key k in nibble k) through byte permutes.
// Codes of the 32 keys in w (any order): word j holds the codes of w[8j .. 8j+7], key 8j+k in
// nibble k. Returns the scale byte; a NaN block gives 0xFF and zero words.
__device__ __forceinline__ uint32_t exp_free_codes(const uint32_t (&w)[32], float m, uint32_t (&out)[4]) {
    unsigned long long u[16];
#pragma unroll
    for (int i = 0; i < 16; ++i)
        u[i] = f2mul(f2sub(pk(__uint_as_float(w[2 * i]), __uint_as_float(w[2 * i + 1])), dup2(m)), dup2(kL2E));
    float q[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float a, b;
        upk(u[i], a, b);
        q[i] = max_nan(a, b);
    }
    float um = max3_nan(max3_nan(q[0], q[1], q[2]), max3_nan(q[3], q[4], q[5]), max3_nan(q[6], q[7], q[8]));
    um = max3_nan(um, max3_nan(q[9], q[10], q[11]), max3_nan(q[12], q[13], max_nan(q[14], q[15])));
    int fl;
    asm("cvt.rmi.s32.f32 %0, %1;" : "=r"(fl) : "f"(um));  // floor; -inf saturates to INT_MIN
    const int es = min(max(fl, -125), 129) - 2;
    const bool nan_block = um != um;
    const unsigned long long two = dup2(2.0f), off = dup2(-2.0f * (float)es), rnd = dup2(12582914.0f);
    uint32_t c[32];  // low byte of each: the code
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        float a, b;
        upk(f2fma(two, u[i], off), a, b);
        a = fminf(fmaxf(a, -2.0f), 5.0f);
        b = fminf(fmaxf(b, -2.0f), 5.0f);
        upk(f2add(pk(a, b), rnd), a, b);
        c[2 * i] = __float_as_uint(a);
        c[2 * i + 1] = __float_as_uint(b);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t* k = c + 8 * j;
        const uint32_t ev = __byte_perm(__byte_perm(k[0], k[2], 0x0040), __byte_perm(k[4], k[6], 0x0040), 0x5410);
        const uint32_t od = __byte_perm(__byte_perm(k[1], k[3], 0x0040), __byte_perm(k[5], k[7], 0x0040), 0x5410);
        out[j] = nan_block ? 0u : (ev | (od << 4));
    }
    return nan_block ? 0xFFu : (uint32_t)(es + 127);
}

__device__ __forceinline__ void exp_free_block(const uint32_t (&w)[32], float m, long long blk, void* codes,
                                               void* scales) {
    uint32_t out[4];
    const uint32_t byte = exp_free_codes(w, m, out);
    st_stream_v4(reinterpret_cast<char*>(codes) + blk * 16, make_uint4(out[0], out[1], out[2], out[3]));
    reinterpret_cast<uint8_t*>(scales)[blk] = (uint8_t)byte;
}

// ---- a block read from shared memory ------------------------------------------------------
//
// Thread t reads the 128 bytes of its block as eight 16-byte pieces, piece (c xor r) into slot
// c with r = t mod 8, so the eight lanes that share a shared-memory wavefront hit eight
// different bank groups. Maximum, exponent and rounding do not depend on the order; the packed
// codes are permuted back (slot c holds piece c xor r) before the store.
__device__ __forceinline__ void load_block_rot(uint32_t blk_addr, uint32_t r, uint32_t (&w)[32]) {
    const uint32_t base = blk_addr ^ (16u * r);  // blk_addr is 128-byte aligned
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const float4 v = lds128(base ^ (16u * c));
        w[4 * c] = __float_as_uint(v.x);
        w[4 * c + 1] = __float_as_uint(v.y);
        w[4 * c + 2] = __float_as_uint(v.z);
        w[4 * c + 3] = __float_as_uint(v.w);
    }
}

// E2M1 codes in slot order (word i: slots 2i, 2i+1, two bytes each) -> the block's 16 bytes.
// Output word j = pieces 2j, 2j+1 = word j ^ (r >> 1), its two halves swapped when r is odd.
__device__ __forceinline__ void store_rot_e2m1(const uint32_t (&h0)[4], uint32_t r, uint32_t keep, void* codes,
                                               long long b) {
    uint32_t h[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __byte_perm(h0[i], 0, (r & 1) ? 0x1032 : 0x3210);
    const bool x1 = r & 2, x2 = r & 4;
    const uint32_t g0 = x1 ? h[1] : h[0], g1 = x1 ? h[0] : h[1], g2 = x1 ? h[3] : h[2], g3 = x1 ? h[2] : h[3];
    st_stream_v4(reinterpret_cast<char*>(codes) + b * 16,
                 make_uint4((x2 ? g2 : g0) & keep, (x2 ? g3 : g1) & keep, (x2 ? g0 : g2) & keep, (x2 ? g1 : g3) & keep));
}

__device__ __forceinline__ void exp_free_rot(const uint32_t (&w)[32], uint32_t r, float m, long long b, void* codes,
                                             void* scales) {
    uint32_t h[4];
    const uint32_t byte = exp_free_codes(w, m, h);
    store_rot_e2m1(h, r, 0xFFFFFFFFu, codes, b);
    reinterpret_cast<uint8_t*>(scales)[b] = (uint8_t)byte;
}

// ---- the kernel ---------------------------------------------------------------------------

template <int F, int CW, int MW, int NS, int LEAD, bool XF>
__global__ void __launch_bounds__(32 * (CW + MW + 1), 1)
    k_exp_quantize_tma(const float* __restrict__ scores, void* codes, void* scales, long long rows, long long cols,
                       bool a32, unsigned int* err) {
    static_assert(LEAD >= 1 && LEAD <= 4, "four row slots bound the producer's lead");
    constexpr int CH = kXStageBytes, NM = 32 * MW;
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) unsigned long long full[NS], empty[NS], mready[4], bfree[4];
    __shared__ float mval[4], mpart[2][MW];
    __shared__ int abort_flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long G = gridDim.x;
    const long long n = rows > (long long)blockIdx.x ? (rows - 1 - blockIdx.x) / G + 1 : 0;  // rows of this CTA
    const long long rowbytes = cols * 4, bpr = cols / 32;
    const int nc = (int)((rowbytes + CH - 1) / CH);
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), MW);
        }
        for (int s = 0; s < 4; ++s) {
            mbar_init(smem_u32(&mready[s]), 1);
            mbar_init(smem_u32(&bfree[s]), CW);
        }
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (n == 0) return;
    volatile int* ab = &abort_flag;
    const uint32_t ring0 = smem_u32(ring);
    auto chunk_bytes = [&](int j) { return (int)min((long long)CH, rowbytes - (long long)j * CH); };

    if (warp == CW + MW) {  // producer: one thread issues every copy
        if (lane != 0) return;
        const unsigned long long keep = l2_policy_keep();
        long long k = 0;
        bool ok = true;
        for (long long i = 0; i < n && ok; ++i) {
            if (i >= LEAD) {  // the consumers are done with row i - LEAD
                const long long q = i - LEAD;
                ok = mbar_wait(smem_u32(&bfree[q & 3]), (uint32_t)(q >> 2) & 1u, ab, err);
            }
            const char* src = reinterpret_cast<const char*>(scores) + (blockIdx.x + i * G) * rowbytes;
            for (int j = 0; j < nc && ok; ++j, ++k) {
                const int s = (int)(k % NS);
                ok = mbar_wait(smem_u32(&empty[s]), ((uint32_t)(k / NS) & 1u) ^ 1u, ab, err);
                if (!ok) break;
                const uint32_t bytes = (uint32_t)chunk_bytes(j);
                mbar_expect_tx(smem_u32(&full[s]), bytes);
                bulk_load(ring0 + s * CH, src + (long long)j * CH, bytes, smem_u32(&full[s]), keep);
            }
        }
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

    if (warp >= CW) {  // maximum warps: pass A
        // Every maximum warp executes one named barrier per row, also after one of its waits
        // has given up (then it only keeps the barrier count: no warp can be left waiting).
        const int t = tid - 32 * CW, mw = warp - CW;
        long long k = 0;
        bool alive = true;
        const float NEG_INF = __uint_as_float(0xFF800000u);
        for (long long i = 0; i < n; ++i) {
            float acc = NEG_INF;
            for (int j = 0; j < nc; ++j, ++k) {
                if (!alive) continue;
                const int s = (int)(k % NS);
                alive = __all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&full[s]), (uint32_t)(k / NS) & 1u, ab, err));
                if (!alive) continue;
                acc = max_nan(acc, stage_max<NM>(ring0 + s * CH, chunk_bytes(j) / 16, t));
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc = max_nan(acc, __shfl_xor_sync(0xFFFFFFFFu, acc, o));
            const int p = (int)(i & 1);
            if (lane == 0) mpart[p][mw] = acc;
            if constexpr (MW > 1) named_sync(1, NM);
            else __syncwarp();
            if (t == 0 && !*ab) {
                float m = mpart[p][0];
#pragma unroll
                for (int w = 1; w < MW; ++w) m = max_nan(m, mpart[p][w]);
                mval[i & 3] = m;
                mbar_arrive(smem_u32(&mready[i & 3]));  // release: mval is visible to the waiters
            }
        }
        return;
    }

    // consumers: pass B, thread tid of 32·CW
    const char* sc = reinterpret_cast<const char*>(scores);
    for (long long i = 0; i < n; ++i) {
        const int slot = (int)(i & 3);
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&mready[slot]), (uint32_t)(i >> 2) & 1u, ab, err))) return;
        const float m = *reinterpret_cast<volatile float*>(&mval[slot]);
        const long long row = blockIdx.x + i * G;
        const char* s = sc + row * rowbytes;
        for (long long b = tid; b < bpr; b += 32 * CW) {
            uint32_t w[32];
            load_block<float>(s, b, w, a32);
            if constexpr (XF) exp_free_block(w, m, row * bpr + b, codes, scales);
            else exp_quant_block<F>(w, m, row * bpr + b, codes, scales, a32);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(&bfree[slot]));
    }
}

// ---- the row-resident kernel (exp-free rule, rows of at most 128 KB) ----------------------
//
// The same three roles, but a row stays in shared memory from its copy to its last code, so each
// score crosses L2 -> SM once: the producer streams stage after stage of the CTA's rows (L2
// evict_first: read once) into a ring of NS stages; the maximum warps fold each stage into the
// row maximum as it lands, meet at a named barrier per row, and their warp 0 publishes the row
// maximum (sixteen row slots); the consumers, in groups of SB/128 threads taking the stages in
// turn, wait for the row maximum, read their blocks from shared memory (load_block_rot) and free
// each stage when done. A row of up to NS - 3 stages leaves at least three stages streaming the
// next rows while the consumers work on it.
// Measured on fp32 4096 x 32768 scores (fraction of the HBM copy peak): exp-free 0.93 here vs
// 0.86 through L2. Exp-then-quantize in this form 0.78 vs 0.81 through L2 (its exponentials hold
// the resident row longer, so less of the ring streams), so it keeps the L2 kernel. 16 KB stages
// were no better (0.93 / 0.78). Rows cut in halves across a two-CTA cluster, the halves' maxima
// exchanged through distributed shared memory every row, were slower still (0.54 / 0.60: the
// per-row coupling of the two CTAs stalls both).
template <int CW, int MW, int NS, int SB>
__global__ void __launch_bounds__(32 * (CW + MW + 1), 1)
    k_exp_free_res(const float* __restrict__ scores, void* codes, void* scales, long long rows, long long cols,
                   unsigned int* err) {
    constexpr int CH = SB, NM = 32 * MW, GT = SB / 128, NG = 32 * CW / GT;  // NG groups of GT threads
    static_assert(NG >= 1 && NG * GT == 32 * CW && GT % 32 == 0, "one consumer thread per block of a stage");
    static_assert(NS <= 15, "sixteen row slots: no role runs more than NS rows ahead of the consumers");
    extern __shared__ __align__(128) uint8_t ring[];
    __shared__ __align__(8) unsigned long long full[NS], empty[NS], mready[16];
    __shared__ float mval[16], mpart[2][MW];
    __shared__ int abort_flag;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long G = gridDim.x;
    const long long n = rows > (long long)blockIdx.x ? (rows - 1 - blockIdx.x) / G + 1 : 0;  // rows of this CTA
    const long long rowbytes = cols * 4, bpr = cols / 32;
    const int nc = (int)((rowbytes + CH - 1) / CH);  // <= NS - 3 (launcher)
    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(smem_u32(&full[s]), 1);
            mbar_init(smem_u32(&empty[s]), GT / 32);
        }
        for (int s = 0; s < 16; ++s) mbar_init(smem_u32(&mready[s]), 1);
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (n == 0) return;
    volatile int* ab = &abort_flag;
    const uint32_t ring0 = smem_u32(ring);
    auto chunk_bytes = [&](int j) { return (int)min((long long)CH, rowbytes - (long long)j * CH); };
    auto row_src = [&](long long i) { return reinterpret_cast<const char*>(scores) + (blockIdx.x + i * G) * rowbytes; };

    auto producer = [&]() {
        const unsigned long long strm = l2_policy_stream();
        long long k = 0;
        bool ok = true;
        for (long long i = 0; i < n && ok; ++i) {
            const char* src = row_src(i);
            for (int j = 0; j < nc; ++j, ++k) {
                const int s = (int)(k % NS);
                ok = mbar_wait(smem_u32(&empty[s]), ((uint32_t)(k / NS) & 1u) ^ 1u, ab, err);
                if (!ok) break;
                const uint32_t bytes = (uint32_t)chunk_bytes(j);
                mbar_expect_tx(smem_u32(&full[s]), bytes);
                bulk_load(ring0 + s * CH, src + (long long)j * CH, bytes, smem_u32(&full[s]), strm);
            }
        }
        if (!ok) {  // gave up: let the copies still in flight land before shared memory goes away
            for (long long q = k > NS ? k - NS : 0; q < k; ++q) {
                const uint32_t bar = smem_u32(&full[q % NS]), par = (uint32_t)(q / NS) & 1u;
                const unsigned long long t0 = global_ns();
                while (!mbar_test(bar, par) && global_ns() - t0 < kWaitLimitNs) {
                }
            }
        }
    };

    auto max_warps = [&]() {
        // one named barrier per row for every maximum warp, also after a wait has given up
        // (then the warp only keeps the barrier count); thread 0 then combines and publishes
        const int t = tid - 32 * CW, mw = warp - CW;
        long long k = 0;
        bool alive = true;
        const float NEG_INF = __uint_as_float(0xFF800000u);
        for (long long i = 0; i < n; ++i) {
            float acc = NEG_INF;
            for (int j = 0; j < nc; ++j, ++k) {
                if (!alive) continue;
                const int s = (int)(k % NS);
                alive = __all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&full[s]), (uint32_t)(k / NS) & 1u, ab, err));
                if (alive) acc = max_nan(acc, stage_max<NM, SB>(ring0 + s * CH, chunk_bytes(j) / 16, t));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc = max_nan(acc, __shfl_xor_sync(0xFFFFFFFFu, acc, o));
            const int q = (int)(i & 15);
            if (lane == 0) mpart[i & 1][mw] = acc;
            if constexpr (MW > 1) named_sync(1, NM);
            else __syncwarp();
            if (mw == 0 && alive && lane == 0 && !*ab) {
                float m = mpart[i & 1][0];
#pragma unroll
                for (int w = 1; w < MW; ++w) m = max_nan(m, mpart[i & 1][w]);
                mval[q] = m;
                mbar_arrive(smem_u32(&mready[q]));
            }
        }
    };

    auto consumers = [&]() {  // group g takes the stages k with k % NG == g; thread tl owns block tl
        const int g = tid / GT, tl = tid - g * GT;
        const uint32_t r = (uint32_t)(tl & 7);
        for (long long i = 0; i < n; ++i) {
            const int q = (int)(i & 15);
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&mready[q]), (uint32_t)(i >> 4) & 1u, ab, err))) return;
            const float m = *reinterpret_cast<volatile float*>(&mval[q]);
            const long long blk0 = (blockIdx.x + i * G) * bpr;
            for (int j = 0; j < nc; ++j) {
                const long long k = i * nc + j;
                if ((int)(k % NG) != g) continue;
                const int s = (int)(k % NS);
                if (!__all_sync(0xFFFFFFFFu, mbar_wait(smem_u32(&full[s]), (uint32_t)(k / NS) & 1u, ab, err))) return;
                if (tl < chunk_bytes(j) / 128) {
                    uint32_t w[32];
                    load_block_rot(ring0 + s * CH + 128u * (uint32_t)tl, r, w);
                    const long long b = blk0 + (long long)j * GT + tl;
                    exp_free_rot(w, r, m, b, codes, scales);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&empty[s]));
            }
        }
    };

    if (warp == CW + MW) {
        if (lane == 0) producer();
    } else if (warp >= CW) {
        max_warps();
    } else {
        consumers();
    }
}

// ---- launch -----------------------------------------------------------------------------

// Shape by measurement on B200 (fp32 4096 x 32768 scores -> MXFP4, fraction of the copy peak;
// consumer warps / maximum warps / stages / lead): 16/2/4/3 0.82-0.83 (kept); 16/2/6/2 0.72,
// 16/2/6/3 0.81, 16/2/6/4 0.82, 16/4/6/3 0.81, 16/4/4/3 0.82, 16/1/6/2 0.63, 12/2/6/3 0.76,
// 20/2/4/3 0.79, 24/2/4/3 0.78. A lead of two rows starves the HBM stream: the producer's
// ring runs more than a row ahead of the landed data, so it reaches the row gate while
// the consumers still wait for the row the gate names. Two blocks in flight per consumer
// thread (0.81) and an L1 prefetch of a thread's next block (0.79) did not help. The
// previous design, one ring shared by both passes with the passes interleaved stage by
// stage, reached 0.76: at most one HBM stage per SM was in flight.
constexpr int kXWarps = 16, kXMaxWarps = 2, kXStages = 4, kXLead = 3;

// every format (the block routine is generic); bulk copies need 16-byte aligned scores, which
// the C ABI requires. For the 6-bit formats and AXS-6 this kernel measured 0.75-0.77 of the copy
// peak against 0.59 for the one-CTA-per-row kernel it replaced (two passes over the row through
// L2 by plain loads).
bool exp_quantize_tma_supported(int, const void* scores) { return (reinterpret_cast<uintptr_t>(scores) & 15) == 0; }

// Row-resident shape (exp-free rule): 16 consumer warps, 2 maximum warps, a ring of kRStages
// stages of kRStageBytes; rows of up to four stages (32768 fp32 keys) stay resident, longer rows
// take the L2 kernel.
constexpr int kRWarps = 16, kRMaxWarps = 2, kRStageBytes = 32768, kRStages = 7;

static cudaError_t launch_res(const float* scores, long long rows, long long cols, void* codes, void* scales,
                              cudaStream_t st) {
    auto kern = k_exp_free_res<kRWarps, kRMaxWarps, kRStages, kRStageBytes>;
    const int smem = kRStages * kRStageBytes, threads = 32 * (kRWarps + kRMaxWarps + 1);
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

static bool resident_rows(long long cols) {
    return cols * 4 <= 131072 && cols * 4 <= (long long)(kRStages - 3) * kRStageBytes;
}

template <int F, int CW, int MW, int NS, int LEAD, bool XF = false>
static cudaError_t launch_xt(const float* scores, long long rows, long long cols, void* codes, void* scales,
                             cudaStream_t st) {
    if (XF && resident_rows(cols)) return launch_res(scores, rows, cols, codes, scales, st);
    auto kern = k_exp_quantize_tma<F, CW, MW, NS, LEAD, XF>;
    const int smem = NS * kXStageBytes, threads = 32 * (CW + MW + 1);
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
    const bool a32 = ((reinterpret_cast<uintptr_t>(scores) | reinterpret_cast<uintptr_t>(codes)) & 31) == 0;
    kern<<<(unsigned)ctas, threads, smem, st>>>(scores, codes, scales, rows, cols, a32, err);
    return cudaGetLastError();
}

cudaError_t launch_exp_quantize_tma(int fmt, const float* scores, long long rows, long long cols, void* codes,
                                    void* scales, cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if (fmt == F_E2M1) return launch_xt<F_E2M1, kXWarps, kXMaxWarps, kXStages, kXLead>(scores, rows, cols, codes, scales, st);
    if (fmt == F_E4M3) return launch_xt<F_E4M3, kXWarps, kXMaxWarps, kXStages, kXLead>(scores, rows, cols, codes, scales, st);
    if (fmt == F_E2M3) return launch_xt<F_E2M3, kXWarps, kXMaxWarps, kXStages, kXLead>(scores, rows, cols, codes, scales, st);
    if (fmt == F_E3M2) return launch_xt<F_E3M2, kXWarps, kXMaxWarps, kXStages, kXLead>(scores, rows, cols, codes, scales, st);
    if (fmt == F_AXS6) return launch_xt<F_AXS6, kXWarps, kXMaxWarps, kXStages, kXLead>(scores, rows, cols, codes, scales, st);
    return cudaErrorInvalidValue;
}

// The exp-free rule through the same pipeline (scores 16-byte aligned, cols % 32 == 0).
cudaError_t launch_exp_free_quantize(const float* scores, long long rows, long long cols, void* codes, void* scales,
                                     cudaStream_t st) {
    if (rows == 0) return cudaSuccess;
    if ((reinterpret_cast<uintptr_t>(scores) & 15) != 0 || cols <= 0 || cols % 32 != 0) return cudaErrorInvalidValue;
    return launch_xt<F_E2M1, kXWarps, kXMaxWarps, kXStages, kXLead, true>(scores, rows, cols, codes, scales, st);
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

// address of the device error word on the current device (cached per device; calls may come
// from several host threads at once, so the cache entries are atomic)
cudaError_t device_error_word(unsigned int** p) {
    static std::atomic<unsigned int*> addr[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    unsigned int* a = addr[dev].load(std::memory_order_acquire);
    if (!a) {
        void* s = nullptr;
        if ((e = cudaGetSymbolAddress(&s, g_device_error)) != cudaSuccess) return e;
        a = static_cast<unsigned int*>(s);
        addr[dev].store(a, std::memory_order_release);
    }
    *p = a;
    return cudaSuccess;
}

cudaError_t read_device_error(unsigned int* value, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(value, g_device_error, sizeof(unsigned int));
    if (e != cudaSuccess || !clear || *value == 0) return e;
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(unsigned int));
}

}  // namespace mxq
