// mxq_expq.cu -- entry of the fused exp-then-quantize softmax probability stage.
//
// "EFQ-Softmax: exp-free E2M1 probabilities" explainer, Jargon (shifted scores,
// exp-then-quantize, MXFP4, microscaling block) and its stage table: the
// conventional path exponentiates the row-max-shifted scores in higher
// precision, materializes the probability block and quantizes it with an
// exponent-only scale from each 32-key block's maximum. Here the block is never
// materialized: every format runs on the bulk-copy pipeline of mxq_expq_tma.cu
// (scores are 16-byte aligned, as the C ABI requires).
#include <cstdint>
#include <cuda_runtime.h>

#include "mxq_internal.h"

namespace mxq {

bool exp_quantize_supported(long long cols) { return cols > 0 && cols % 32 == 0; }

cudaError_t launch_exp_quantize(int fmt, const float* scores, long long rows, long long cols, void* codes,
                                void* scales, cudaStream_t st) {
    if (!exp_quantize_supported(cols) || !exp_quantize_tma_supported(fmt, scores)) return cudaErrorNotSupported;
    return launch_exp_quantize_tma(fmt, scores, rows, cols, codes, scales, st);
}

}  // namespace mxq
