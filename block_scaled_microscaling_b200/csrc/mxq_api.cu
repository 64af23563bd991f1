// mxq_api.cu -- the C ABI of libmxq (declared in include/mxq.h).
//
// Host side only: argument validation (before any launch), size queries,
// status strings, and dispatch to the kernel launchers. Every compute step
// runs in the kernels of mxq_codec.cu / mxq_expq.cu; there is no host
// fallback.
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "../../include/mxq.h"
#include "mxq_internal.h"

namespace {

int elem_bits(mxq_format f) {
    switch (f) {
        case MXQ_AXS6:
        case MXQ_MXFP6_E2M3:
        case MXQ_MXFP6_E3M2: return 6;
        case MXQ_MXFP8_E4M3: return 8;
        case MXQ_MXFP4_E2M1: return 4;
    }
    return -1;
}
bool fmt_ok(mxq_format f) { return elem_bits(f) > 0; }
bool dtype_ok(mxq_dtype d) { return d == MXQ_F32 || d == MXQ_BF16; }
int dtype_bytes(mxq_dtype d) { return d == MXQ_F32 ? 4 : 2; }

constexpr int64_t kMaxElems = (int64_t)1 << 50;

mxq_status check_shape(int64_t rows, int64_t cols) {
    if (rows < 0 || cols <= 0 || cols % 32 != 0) return MXQ_ERR_SHAPE;
    if (rows > 0 && cols > kMaxElems / rows) return MXQ_ERR_SHAPE;
    return MXQ_OK;
}

// device (or managed) memory of the current device, aligned to `align`
mxq_status check_ptr(const void* p, uintptr_t align) {
    if (p == nullptr) return MXQ_ERR_INVALID_ARG;
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) {
        cudaGetLastError();  // the failed query also sets the (non-sticky) last error: clear it
        return MXQ_ERR_INVALID_ARG;
    }
    if (a.type != cudaMemoryTypeDevice && a.type != cudaMemoryTypeManaged) return MXQ_ERR_INVALID_ARG;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return MXQ_ERR_CUDA;
    if (a.type == cudaMemoryTypeDevice && a.device != dev) return MXQ_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(p) % align != 0) return MXQ_ERR_ALIGN;
    return MXQ_OK;
}

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
    uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

size_t codes_bytes(mxq_format f, int64_t rows, int64_t cols) {
    return (size_t)rows * (size_t)(cols / 32) * (size_t)(4 * elem_bits(f));
}
size_t scales_bytes(mxq_format f, int64_t rows, int64_t cols) {
    return (size_t)rows * (size_t)(cols / 32) * (f == MXQ_AXS6 ? 2u : 1u);
}
uintptr_t scales_align(mxq_format f) { return f == MXQ_AXS6 ? 2 : 1; }

mxq_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return MXQ_OK;
    if (e == cudaErrorNotSupported) return MXQ_ERR_UNSUPPORTED;
    return MXQ_ERR_CUDA;
}

#define MXQ_TRY(x)                         \
    do {                                   \
        mxq_status s_ = (x);               \
        if (s_ != MXQ_OK) return s_;       \
    } while (0)

mxq_status check_quantize_args(mxq_format fmt, const void* src, mxq_dtype dtype, int64_t rows, int64_t cols,
                               void* codes, void* scales) {
    if (!fmt_ok(fmt) || !dtype_ok(dtype)) return MXQ_ERR_INVALID_ARG;
    MXQ_TRY(check_shape(rows, cols));
    if (rows == 0) return MXQ_OK;
    MXQ_TRY(check_ptr(src, 16));
    MXQ_TRY(check_ptr(codes, 16));
    MXQ_TRY(check_ptr(scales, scales_align(fmt)));
    const size_t nsrc = (size_t)rows * (size_t)cols * dtype_bytes(dtype);
    const size_t nc = codes_bytes(fmt, rows, cols), ns = scales_bytes(fmt, rows, cols);
    if (overlap(src, nsrc, codes, nc) || overlap(src, nsrc, scales, ns) || overlap(codes, nc, scales, ns))
        return MXQ_ERR_INVALID_ARG;
    return MXQ_OK;
}

mxq_status check_dequantize_args(mxq_format fmt, const void* codes, const void* scales, int64_t rows, int64_t cols,
                                 void* dst, mxq_dtype dtype) {
    if (!fmt_ok(fmt) || !dtype_ok(dtype)) return MXQ_ERR_INVALID_ARG;
    MXQ_TRY(check_shape(rows, cols));
    if (rows == 0) return MXQ_OK;
    MXQ_TRY(check_ptr(codes, 16));
    MXQ_TRY(check_ptr(scales, scales_align(fmt)));
    MXQ_TRY(check_ptr(dst, 16));
    const size_t nd = (size_t)rows * (size_t)cols * dtype_bytes(dtype);
    if (overlap(dst, nd, codes, codes_bytes(fmt, rows, cols)) || overlap(dst, nd, scales, scales_bytes(fmt, rows, cols)))
        return MXQ_ERR_INVALID_ARG;
    return MXQ_OK;
}

mxq_status check_fake_args(mxq_format fmt, const void* src, mxq_dtype dtype, int64_t rows, int64_t cols, void* dst) {
    if (!fmt_ok(fmt) || !dtype_ok(dtype)) return MXQ_ERR_INVALID_ARG;
    MXQ_TRY(check_shape(rows, cols));
    if (rows == 0) return MXQ_OK;
    MXQ_TRY(check_ptr(src, 16));
    MXQ_TRY(check_ptr(dst, 16));
    const size_t nb = (size_t)rows * (size_t)cols * dtype_bytes(dtype);
    if (src != dst && overlap(src, nb, dst, nb)) return MXQ_ERR_INVALID_ARG;
    return MXQ_OK;
}

bool aligned32(const void* a, const void* b) {
    return ((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(b)) & 31) == 0;
}

}  // namespace

extern "C" {

mxq_status mxq_quantize(mxq_format fmt, const void* src, mxq_dtype dtype, int64_t rows, int64_t cols, void* codes,
                        void* scales, mxq_stream stream) {
    MXQ_TRY(check_quantize_args(fmt, src, dtype, rows, cols, codes, scales));
    if (rows == 0) return MXQ_OK;
    mxq::SegTable<1> tab{};
    tab.seg[0] = {src, codes, scales, rows * (cols / 32), 0, 0};
    tab.n = 1;
    return from_cuda(mxq::launch_quantize<1>((int)fmt, (int)dtype, tab, (cudaStream_t)stream));
}

size_t mxq_mma_scales_bytes(int64_t rows, int64_t cols) {
    if (check_shape(rows, cols) != MXQ_OK) return 0;
    return (size_t)((rows + 127) / 128) * 128 * (size_t)(((cols / 32) + 3) / 4) * 4;
}

mxq_status mxq_quantize_mma(mxq_format fmt, const void* src, mxq_dtype dtype, int64_t rows, int64_t cols,
                            void* codes, void* scales, mxq_stream stream) {
    if (!fmt_ok(fmt) || !dtype_ok(dtype)) return MXQ_ERR_INVALID_ARG;
    if (fmt == MXQ_AXS6) return MXQ_ERR_UNSUPPORTED;
    MXQ_TRY(check_shape(rows, cols));
    if (rows == 0) return MXQ_OK;
    MXQ_TRY(check_ptr(src, 16));
    MXQ_TRY(check_ptr(codes, 16));
    MXQ_TRY(check_ptr(scales, 1));
    const size_t nsrc = (size_t)rows * (size_t)cols * dtype_bytes(dtype);
    const size_t nc = codes_bytes(fmt, rows, cols), ns = mxq_mma_scales_bytes(rows, cols);
    if (overlap(src, nsrc, codes, nc) || overlap(src, nsrc, scales, ns) || overlap(codes, nc, scales, ns))
        return MXQ_ERR_INVALID_ARG;
    const int64_t kb = cols / 32;
    if (rows % 128 != 0 || kb % 4 != 0) {
        cudaError_t e = cudaMemsetAsync(scales, 0, ns, (cudaStream_t)stream);
        if (e != cudaSuccess) return from_cuda(e);
    }
    mxq::SegTable<1> tab{};
    tab.seg[0] = {src, codes, scales, rows * kb, 0, kb};
    tab.n = 1;
    return from_cuda(mxq::launch_quantize<1>((int)fmt, (int)dtype, tab, (cudaStream_t)stream));
}

mxq_status mxq_swizzle_scales(const void* scales, int64_t rows, int64_t kblocks, void* out, mxq_stream stream) {
    // a tile-row's 4-byte output words are counted in 32 bits: kblocks up to 4 * (2^31 - 1) / 128
    if (rows < 0 || kblocks <= 0 || kblocks > kMaxElems / 32 || kblocks > 4 * (0x7FFFFFFFLL / 128)) return MXQ_ERR_SHAPE;
    MXQ_TRY(check_shape(rows, 32 * kblocks));
    if (rows == 0) return MXQ_OK;
    MXQ_TRY(check_ptr(scales, 1));
    MXQ_TRY(check_ptr(out, 4));
    if (overlap(scales, (size_t)rows * (size_t)kblocks, out, mxq_mma_scales_bytes(rows, 32 * kblocks)))
        return MXQ_ERR_INVALID_ARG;
    return from_cuda(mxq::launch_swizzle_scales(scales, rows, kblocks, out, (cudaStream_t)stream));
}

mxq_status mxq_quantize_grouped(mxq_format fmt, mxq_dtype dtype, const mxq_tensor* tensors, int n,
                                mxq_stream stream) {
    if (!fmt_ok(fmt) || !dtype_ok(dtype) || tensors == nullptr || n < 1 || n > MXQ_MAX_GROUP)
        return MXQ_ERR_INVALID_ARG;
    mxq::SegTable<mxq::kMaxSeg> tab{};
    int m = 0;
    for (int i = 0; i < n; ++i) {
        const mxq_tensor& t = tensors[i];
        MXQ_TRY(check_quantize_args(fmt, t.src, dtype, t.rows, t.cols, t.codes, t.scales));
        if (t.rows == 0) continue;
        tab.seg[m++] = {t.src, t.codes, t.scales, t.rows * (t.cols / 32), 0, 0};
    }
    if (m == 0) return MXQ_OK;
    tab.n = m;
    return from_cuda(mxq::launch_quantize<mxq::kMaxSeg>((int)fmt, (int)dtype, tab, (cudaStream_t)stream));
}

mxq_status mxq_dequantize(mxq_format fmt, const void* codes, const void* scales, int64_t rows, int64_t cols,
                          void* dst, mxq_dtype dtype, mxq_stream stream) {
    MXQ_TRY(check_dequantize_args(fmt, codes, scales, rows, cols, dst, dtype));
    if (rows == 0) return MXQ_OK;
    return from_cuda(mxq::launch_dequantize((int)fmt, codes, scales, dst, (int)dtype, rows * (cols / 32),
                                            (cudaStream_t)stream));
}

mxq_status mxq_fake_quantize(mxq_format fmt, const void* src, mxq_dtype dtype, int64_t rows, int64_t cols, void* dst,
                             mxq_stream stream) {
    MXQ_TRY(check_fake_args(fmt, src, dtype, rows, cols, dst));
    if (rows == 0) return MXQ_OK;
    // the bulk-copy stream pays a pipeline fill and drain that only large tensors amortize (AXS-6 fp32
    // on B200: 3.0 vs 2.3 us at 8K values, 13.7 vs 13.2 us at 8M, 44.8 vs 50.8 us at 33M values)
    const long long nb = rows * (cols / 32);
    if (nb < (1LL << 19))
        return from_cuda(mxq::launch_fake_quantize((int)fmt, src, dst, (int)dtype, nb, (cudaStream_t)stream));
    return from_cuda(mxq::launch_fake_quantize_stream((int)fmt, src, dst, (int)dtype, nb, (cudaStream_t)stream));
}

mxq_status mxq_run_batch(mxq_dtype dtype, const mxq_op* ops, int n, mxq_stream stream) {
    if (!dtype_ok(dtype) || ops == nullptr || n < 1 || n > MXQ_MAX_BATCH) return MXQ_ERR_INVALID_ARG;
    struct Range {
        const void* p;
        size_t n;
    };
    Range rin[MXQ_MAX_BATCH][2], rout[MXQ_MAX_BATCH][2];
    mxq::BatchTable tab{};
    int m = 0;
    for (int i = 0; i < n; ++i) {
        const mxq_op& o = ops[i];
        const mxq_format f = (mxq_format)o.fmt;
        if (!fmt_ok(f)) return MXQ_ERR_INVALID_ARG;
        // shapes are checked before any size is formed from them
        const mxq_status shape = check_shape(o.rows, o.cols);
        if (shape != MXQ_OK) return o.kind < MXQ_OP_QUANTIZE || o.kind > MXQ_OP_FAKE_QUANTIZE ? MXQ_ERR_INVALID_ARG : shape;
        const size_t nv = (size_t)o.rows * (size_t)o.cols * dtype_bytes(dtype);
        mxq::BatchOp b{};
        b.kind = o.kind;
        b.fmt = o.fmt;
        b.nblocks = o.rows * (o.cols / 32);
        if (o.kind == MXQ_OP_QUANTIZE) {
            MXQ_TRY(check_quantize_args(f, o.src, dtype, o.rows, o.cols, o.dst, o.dst_scales));
            b.in = o.src;
            b.out = o.dst;
            b.scales_out = o.dst_scales;
            rin[m][0] = {o.src, nv};
            rin[m][1] = {nullptr, 0};
            rout[m][0] = {o.dst, codes_bytes(f, o.rows, o.cols)};
            rout[m][1] = {o.dst_scales, scales_bytes(f, o.rows, o.cols)};
        } else if (o.kind == MXQ_OP_DEQUANTIZE) {
            MXQ_TRY(check_dequantize_args(f, o.src, o.src_scales, o.rows, o.cols, o.dst, dtype));
            b.in = o.src;
            b.scales_in = o.src_scales;
            b.out = o.dst;
            rin[m][0] = {o.src, codes_bytes(f, o.rows, o.cols)};
            rin[m][1] = {o.src_scales, scales_bytes(f, o.rows, o.cols)};
            rout[m][0] = {o.dst, nv};
            rout[m][1] = {nullptr, 0};
        } else if (o.kind == MXQ_OP_FAKE_QUANTIZE) {
            MXQ_TRY(check_fake_args(f, o.src, dtype, o.rows, o.cols, o.dst));
            b.in = o.src;
            b.out = o.dst;
            rin[m][0] = {o.src, nv};
            rin[m][1] = {nullptr, 0};
            rout[m][0] = {o.dst, nv};
            rout[m][1] = {nullptr, 0};
        } else {
            return MXQ_ERR_INVALID_ARG;
        }
        if (o.rows == 0) continue;
        b.a32 = aligned32(b.in, b.out) ? 1 : 0;
        tab.op[m++] = b;
    }
    // the ops run concurrently: an op's outputs may not touch another op's inputs or outputs
    for (int i = 0; i < m; ++i)
        for (int j = 0; j < m; ++j) {
            if (i == j) continue;
            for (int a = 0; a < 2; ++a)
                for (int c = 0; c < 2; ++c) {
                    const Range& w = rout[i][a];
                    if (w.n == 0) continue;
                    if ((rin[j][c].n && overlap(w.p, w.n, rin[j][c].p, rin[j][c].n)) ||
                        (rout[j][c].n && overlap(w.p, w.n, rout[j][c].p, rout[j][c].n)))
                        return MXQ_ERR_INVALID_ARG;
                }
        }
    if (m == 0) return MXQ_OK;
    tab.n = m;
    return from_cuda(mxq::launch_batch((int)dtype, tab, (cudaStream_t)stream));
}

mxq_status mxq_check_device(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return MXQ_ERR_CUDA;
    unsigned int v = 0;
    if (mxq::read_device_error(&v, true) != cudaSuccess) return MXQ_ERR_CUDA;
    return v ? MXQ_ERR_TIMEOUT : MXQ_OK;
}

mxq_status mxq_selftest_timeout(int limit_ms) {
    if (limit_ms < 1 || limit_ms > 1000) return MXQ_ERR_INVALID_ARG;
    // start from a clear word; a timeout left by an earlier call is reported, not cleared away
    const mxq_status before = mxq_check_device();
    if (before != MXQ_OK) return before;
    if (mxq::launch_selftest_timeout((unsigned long long)limit_ms * 1000000ull, 0) != cudaSuccess) return MXQ_ERR_CUDA;
    return mxq_check_device();
}

mxq_status mxq_exp_quantize(mxq_format fmt, const float* scores, int64_t rows, int64_t cols, void* codes,
                            void* scales, mxq_stream stream) {
    MXQ_TRY(check_quantize_args(fmt, scores, MXQ_F32, rows, cols, codes, scales));
    if (!mxq::exp_quantize_supported(cols)) return MXQ_ERR_UNSUPPORTED;
    if (rows == 0) return MXQ_OK;
    return from_cuda(mxq::launch_exp_quantize((int)fmt, scores, rows, cols, codes, scales, (cudaStream_t)stream));
}

mxq_status mxq_exp_free_quantize(const float* scores, int64_t rows, int64_t cols, void* codes, void* scales,
                                 mxq_stream stream) {
    MXQ_TRY(check_quantize_args(MXQ_MXFP4_E2M1, scores, MXQ_F32, rows, cols, codes, scales));
    if (rows == 0) return MXQ_OK;
    return from_cuda(mxq::launch_exp_free_quantize(scores, rows, cols, codes, scales, (cudaStream_t)stream));
}

mxq_status mxq_quantize_cols(mxq_format fmt, const void* src, mxq_dtype dtype, int64_t rows, int64_t cols,
                             void* codes, void* scales, mxq_stream stream) {
    if (!fmt_ok(fmt) || !dtype_ok(dtype)) return MXQ_ERR_INVALID_ARG;
    if (rows < 0 || rows % 32 != 0 || cols <= 0 || cols % 32 != 0) return MXQ_ERR_SHAPE;
    if (rows == 0) return MXQ_OK;
    if (!mxq::cols_grid_ok(rows, cols)) return MXQ_ERR_SHAPE;
    // same sizes/alignment/overlap rules as the row-direction call on the transpose
    MXQ_TRY(check_quantize_args(fmt, src, dtype, cols, rows, codes, scales));
    return from_cuda(mxq::launch_quantize_cols((int)fmt, src, (int)dtype, rows, cols, codes, scales,
                                               (cudaStream_t)stream));
}

mxq_status mxq_dequantize_cols(mxq_format fmt, const void* codes, const void* scales, int64_t rows, int64_t cols,
                               void* dst, mxq_dtype dtype, mxq_stream stream) {
    if (!fmt_ok(fmt) || !dtype_ok(dtype)) return MXQ_ERR_INVALID_ARG;
    if (rows < 0 || rows % 32 != 0 || cols <= 0 || cols % 32 != 0) return MXQ_ERR_SHAPE;
    if (rows == 0) return MXQ_OK;
    if (!mxq::cols_grid_ok(rows, cols)) return MXQ_ERR_SHAPE;
    MXQ_TRY(check_shape(cols, rows));
    MXQ_TRY(check_ptr(codes, 16));
    MXQ_TRY(check_ptr(scales, scales_align(fmt)));
    MXQ_TRY(check_ptr(dst, 16));
    const size_t nd = (size_t)rows * (size_t)cols * dtype_bytes(dtype);
    if (overlap(dst, nd, codes, codes_bytes(fmt, cols, rows)) || overlap(dst, nd, scales, scales_bytes(fmt, cols, rows)))
        return MXQ_ERR_INVALID_ARG;
    return from_cuda(mxq::launch_dequantize_cols((int)fmt, codes, scales, dst, (int)dtype, rows, cols,
                                                 (cudaStream_t)stream));
}

mxq_status mxq_quantize_exmy(int ebits, int mbits, const void* src, mxq_dtype dtype, int64_t rows, int64_t cols,
                             void* codes, void* scales, mxq_stream stream) {
    if (!dtype_ok(dtype)) return MXQ_ERR_INVALID_ARG;
    if (!mxq::exmy_supported(ebits, mbits)) return MXQ_ERR_UNSUPPORTED;
    MXQ_TRY(check_shape(rows, cols));
    if (rows == 0) return MXQ_OK;
    MXQ_TRY(check_ptr(src, 16));
    MXQ_TRY(check_ptr(codes, 16));
    MXQ_TRY(check_ptr(scales, 1));
    const size_t W = (size_t)(1 + ebits + mbits), nb = (size_t)rows * (size_t)(cols / 32);
    const size_t nsrc = (size_t)rows * (size_t)cols * dtype_bytes(dtype);
    if (overlap(src, nsrc, codes, nb * 4 * W) || overlap(src, nsrc, scales, nb) || overlap(codes, nb * 4 * W, scales, nb))
        return MXQ_ERR_INVALID_ARG;
    return from_cuda(mxq::launch_exmy(0, ebits, mbits, (int)dtype, src, codes, nullptr, scales, (long long)nb,
                                      (cudaStream_t)stream));
}

mxq_status mxq_dequantize_exmy(int ebits, int mbits, const void* codes, const void* scales, int64_t rows, int64_t cols,
                               void* dst, mxq_dtype dtype, mxq_stream stream) {
    if (!dtype_ok(dtype)) return MXQ_ERR_INVALID_ARG;
    if (!mxq::exmy_supported(ebits, mbits)) return MXQ_ERR_UNSUPPORTED;
    MXQ_TRY(check_shape(rows, cols));
    if (rows == 0) return MXQ_OK;
    MXQ_TRY(check_ptr(codes, 16));
    MXQ_TRY(check_ptr(scales, 1));
    MXQ_TRY(check_ptr(dst, 16));
    const size_t W = (size_t)(1 + ebits + mbits), nb = (size_t)rows * (size_t)(cols / 32);
    const size_t nd = (size_t)rows * (size_t)cols * dtype_bytes(dtype);
    if (overlap(dst, nd, codes, nb * 4 * W) || overlap(dst, nd, scales, nb)) return MXQ_ERR_INVALID_ARG;
    return from_cuda(mxq::launch_exmy(1, ebits, mbits, (int)dtype, codes, dst, scales, nullptr, (long long)nb,
                                      (cudaStream_t)stream));
}

mxq_status mxq_fake_quantize_exmy(int ebits, int mbits, const void* src, mxq_dtype dtype, int64_t rows, int64_t cols,
                                  void* dst, mxq_stream stream) {
    if (!dtype_ok(dtype)) return MXQ_ERR_INVALID_ARG;
    if (!mxq::exmy_supported(ebits, mbits)) return MXQ_ERR_UNSUPPORTED;
    MXQ_TRY(check_shape(rows, cols));
    if (rows == 0) return MXQ_OK;
    MXQ_TRY(check_ptr(src, 16));
    MXQ_TRY(check_ptr(dst, 16));
    const size_t nbytes = (size_t)rows * (size_t)cols * dtype_bytes(dtype);
    if (src != dst && overlap(src, nbytes, dst, nbytes)) return MXQ_ERR_INVALID_ARG;
    return from_cuda(mxq::launch_exmy(2, ebits, mbits, (int)dtype, src, dst, nullptr, nullptr,
                                      (long long)(rows * (cols / 32)), (cudaStream_t)stream));
}

size_t mxq_codes_bytes(mxq_format fmt, int64_t rows, int64_t cols) {
    if (!fmt_ok(fmt) || check_shape(rows, cols) != MXQ_OK) return 0;
    return codes_bytes(fmt, rows, cols);
}

size_t mxq_scales_bytes(mxq_format fmt, int64_t rows, int64_t cols) {
    if (!fmt_ok(fmt) || check_shape(rows, cols) != MXQ_OK) return 0;
    return scales_bytes(fmt, rows, cols);
}

int mxq_block_bits(mxq_format fmt) {
    if (!fmt_ok(fmt)) return -1;
    return 8 + 32 * elem_bits(fmt) + (fmt == MXQ_AXS6 ? 2 : 0);
}

const char* mxq_status_string(mxq_status s) {
    switch (s) {
        case MXQ_OK: return "ok";
        case MXQ_ERR_INVALID_ARG: return "invalid argument (format, type, or a null/host/other-device/overlapping pointer)";
        case MXQ_ERR_SHAPE: return "invalid shape (rows < 0, cols <= 0, cols not a multiple of 32, or too large)";
        case MXQ_ERR_ALIGN: return "misaligned pointer (values and codes need 16 bytes, AXS-6 headers 2)";
        case MXQ_ERR_UNSUPPORTED: return "valid request that the library does not support";
        case MXQ_ERR_CUDA: return "a CUDA runtime call or kernel launch failed";
        case MXQ_ERR_TIMEOUT: return "a bounded device-side wait gave up";
    }
    return "unknown status";
}

const char* mxq_version(void) { return "0.1.0"; }

}  // extern "C"
