// fp8_gemm_ch64.cu -- channel-major (D^T = B * A^T) instantiations of the
// row-wise scaled FP8 GEMM with 64 output channels per tile (the M = 64 form
// of the single-CTA tcgen05 MMA) and 16, 32 or 64 tokens per tile: twice the
// tiles of the 128-channel form, for weights too narrow to give every SM a
// 128-channel slice (see fp8_gemm.cuh).
#include "fp8_gemm.cuh"

namespace rn {

cudaError_t gemm_channel_major_64(int tokens, const GemmArgs& g, cudaStream_t stream) {
    using namespace gemm_detail;
    if (tokens == 16) return RowwiseGemm<Shape<_64, _16, _128>, true>::run(g, stream);
    if (tokens == 32) return RowwiseGemm<Shape<_64, _32, _128>, true>::run(g, stream);
    if (tokens == 64) return RowwiseGemm<Shape<_64, _64, _128>, true>::run(g, stream);
    return cudaErrorInvalidValue;
}

}  // namespace rn
