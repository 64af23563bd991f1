// mxq_internal.h -- launch interface between the C ABI (mxq_api.cu) and the
// kernels (mxq_codec.cu, mxq_expq.cu). Not part of the public header.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace mxq {

constexpr int kMaxSeg = 64;  // == MXQ_MAX_GROUP

// SMs x resident CTAs of 256 threads for a kernel (occupancy query, cached per kernel and device)
int resident_ctas(const void* fn, int dev);

// one tensor of a (grouped) quantize launch
struct Seg {
    const void* src;
    void* codes;
    void* scales;
    long long nblocks;  // blocks of 32 values
    long long blk0;     // first block of this tensor in the concatenation (filled by the launcher)
    long long kb_mma;   // 0: scales [rows, cols/32] row-major; else blocks per row, scales in the MMA tile layout
};
template <int N> struct SegTable {
    Seg seg[N];
    int n;
    long long nblocks;  // all tensors' blocks
};

// one conversion of a batch launch: kind 0 quantize (in values -> out codes, scales_out),
// 1 dequantize (in codes + scales_in -> out values), 2 fake-quantize (in values -> out values)
struct BatchOp {
    int kind;
    int fmt;
    int a32;            // in and out both 32-byte aligned: 256-bit accesses
    const void* in;
    const void* scales_in;
    void* out;
    void* scales_out;
    long long nblocks;  // blocks of 32 values
    long long tile0;    // first warp tile (32 blocks) of this op in the batch (filled by the launcher)
};
struct BatchTable {
    BatchOp op[kMaxSeg];
    int n;
    long long ntiles;
};
cudaError_t launch_batch(int dtype, BatchTable& tab, cudaStream_t st);

// fmt: 0 AXS-6, 1 E2M3, 2 E3M2, 3 E4M3, 4 E2M1; dtype: 0 fp32, 1 bf16
template <int NSEG>
cudaError_t launch_quantize(int fmt, int dtype, SegTable<NSEG>& tab, cudaStream_t st);
cudaError_t launch_dequantize(int fmt, const void* codes, const void* scales, void* dst, int dtype,
                              long long nblocks, cudaStream_t st);
cudaError_t launch_fake_quantize(int fmt, const void* src, void* dst, int dtype, long long nblocks,
                                 cudaStream_t st);
// the same through the bulk-copy streaming kernel (mxq_stream.cu); 16-byte aligned pointers
cudaError_t launch_fake_quantize_stream(int fmt, const void* src, void* dst, int dtype, long long nblocks,
                                        cudaStream_t st);
// returns cudaErrorNotSupported when cols is beyond what one cluster holds
cudaError_t launch_exp_quantize(int fmt, const float* scores, long long rows, long long cols, void* codes,
                                void* scales, cudaStream_t st);
bool exp_quantize_supported(long long cols);
// bulk-copy pipeline form of the softmax stage (every format; scores 16-byte aligned)
bool exp_quantize_tma_supported(int fmt, const void* scores);
cudaError_t launch_exp_free_quantize(const float* scores, long long rows, long long cols, void* codes, void* scales,
                                     cudaStream_t st);
cudaError_t launch_exp_quantize_tma(int fmt, const float* scores, long long rows, long long cols, void* codes,
                                    void* scales, cudaStream_t st);
// Launch with programmatic stream serialization: the kernel may be scheduled while the previous
// kernel of the stream drains; it waits for it (griddepcontrol.wait) before touching memory and
// then lets the next launch be scheduled. Measured on back-to-back launches (fraction of the
// copy peak): batch step 0.91 -> 0.92, single-tensor quantize at 47 MB +2% (MXFP8 +6%), at
// 268 MB +0.5-1%. Used for the batch kernel, quantize and the one-pass dequantize.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), unsigned grid, unsigned block, cudaStream_t st, Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(block, 1, 1);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute a[1];
    a[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    a[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = a;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, args...);
}

// the device error word (bit 0: a bounded wait in a kernel ran out): its device address for
// kernel arguments, and its value (clear resets it)
cudaError_t device_error_word(unsigned int** p);
cudaError_t read_device_error(unsigned int* value, bool clear);
// one warp waits (bounded by limit_ns) on an mbarrier nothing arrives at
cudaError_t launch_selftest_timeout(unsigned long long limit_ns, cudaStream_t st);
// column-direction blocks (32 rows of a column), transposed output layout
cudaError_t launch_quantize_cols(int fmt, const void* src, int dtype, long long rows, long long cols, void* codes,
                                 void* scales, cudaStream_t st);
cudaError_t launch_dequantize_cols(int fmt, const void* codes, const void* scales, void* dst, int dtype, long long rows,
                                   long long cols, cudaStream_t st);
bool cols_grid_ok(long long rows, long long cols);
// plain [rows, kb] E8M0 scales -> block-scaled MMA tile layout (padding written as 0)
cudaError_t launch_swizzle_scales(const void* scales, long long rows, long long kb, void* out, cudaStream_t st);
// eXmY: op 0 quantize (in values -> out codes, aux_out scales), 1 dequantize
// (in codes + aux_in scales -> out values), 2 fake-quantize (in -> out)
bool exmy_supported(int E, int M);
cudaError_t launch_exmy(int op, int E, int M, int dtype, const void* in, void* out, const void* aux_in, void* aux_out,
                        long long nblocks, cudaStream_t st);

}  // namespace mxq
