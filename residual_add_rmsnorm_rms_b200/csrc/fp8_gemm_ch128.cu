// fp8_gemm_ch128.cu -- channel-major (D^T = B * A^T) instantiations of the
// row-wise scaled FP8 GEMM with 128 output channels per tile and 16, 32 or 64
// tokens per tile (see fp8_gemm.cuh).
#include "fp8_gemm.cuh"

namespace rn {

cudaError_t gemm_channel_major_128(int tokens, const GemmArgs& g, cudaStream_t stream) {
    using namespace gemm_detail;
    if (tokens == 16) return RowwiseGemm<Shape<_128, _16, _128>, true>::run(g, stream);
    if (tokens == 32) return RowwiseGemm<Shape<_128, _32, _128>, true>::run(g, stream);
    if (tokens == 64) return RowwiseGemm<Shape<_128, _64, _128>, true>::run(g, stream);
    return cudaErrorInvalidValue;
}

}  // namespace rn
