// fp8_gemm.cu -- tile-configuration dispatch of the row-wise scaled FP8 GEMM
// and its token-major 128 x 128 and 128 x 256 instantiations (the template and the two
// orientations are described in fp8_gemm.cuh). The channel-major
// instantiations for decode-sized M live in fp8_gemm_ch128.cu and
// fp8_gemm_ch64.cu so that the three units compile in parallel.
#include "fp8_gemm.cuh"

namespace rn {

cudaError_t gemm_channel_major_128(int tokens, const GemmArgs& g, cudaStream_t stream);
cudaError_t gemm_channel_major_64(int tokens, const GemmArgs& g, cudaStream_t stream);

cudaError_t launch_fp8_rowwise_gemm(const GemmArgs& g, cudaStream_t stream) {
    using namespace gemm_detail;
    switch (g.config) {
        case kGemmTok128Ch128:
            return RowwiseGemm<Shape<_128, _128, _128>, false>::run(g, stream);
        case kGemmTok128Ch256:
            return RowwiseGemm<Shape<_128, _256, _128>, false>::run(g, stream);
        case kGemmCh128Tok16: return gemm_channel_major_128(16, g, stream);
        case kGemmCh128Tok32: return gemm_channel_major_128(32, g, stream);
        case kGemmCh128Tok64: return gemm_channel_major_128(64, g, stream);
        case kGemmCh64Tok16: return gemm_channel_major_64(16, g, stream);
        case kGemmCh64Tok32: return gemm_channel_major_64(32, g, stream);
        case kGemmCh64Tok64: return gemm_channel_major_64(64, g, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace rn
