// rn_gemm.h -- interface between the C-ABI layer (rmsnorm_api.cpp) and the
// row-wise scaled fp8 GEMM (fp8_gemm*.cu). Internal.
#pragma once

#include <cstdint>

#include <cuda_runtime_api.h>

namespace rn {

// Operands of the row-wise scaled fp8 GEMM (device pointers; see fp8_gemm.cu).
struct GemmArgs {
    const void* a;        // [M x K] e4m3
    const void* b;        // [N x K] e4m3
    const float* a_scale; // [M]
    const float* b_scale; // [N]
    void* d;              // [M x N] bf16
    int64_t M, N, K;
    int device;
    int num_sms;
    int config;           // GemmConfig: tile shape and orientation
    bool pdl;             // launch with programmatic dependent launch
    unsigned long long ctx_id = 0;  // id of the current CUDA context (0: unknown)
};

// Tile configurations of the fp8 GEMM (values of rn_gemm_config in the public
// header). Token-major tiles are (tokens x channels); channel-major tiles
// compute D^T and are (channels x tokens).
enum GemmConfig {
    kGemmTok128Ch128 = 0,
    kGemmCh128Tok16 = 1,
    kGemmCh128Tok32 = 2,
    kGemmCh128Tok64 = 3,
    kGemmCh64Tok16 = 4,
    kGemmCh64Tok32 = 5,
    kGemmCh64Tok64 = 6,
    kGemmTok128Ch256 = 7,
    kNumGemmConfigs = 8
};

// Runs the row-wise scaled fp8 GEMM on `stream` (tcgen05 tensor cores).
cudaError_t launch_fp8_rowwise_gemm(const GemmArgs& g, cudaStream_t stream);

}  // namespace rn
