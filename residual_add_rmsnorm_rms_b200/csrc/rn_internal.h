// rn_internal.h -- interface between the C-ABI layer (rmsnorm_api.cpp) and
// the sm_100a kernels (rmsnorm_kernels.cu). Not installed, not part of the ABI.
#pragma once

#include <cstdint>

#include <cuda_runtime_api.h>

namespace rn {

// Flattened operands of one call. residual is read and written in place.
struct Args {
    const void* x;
    void* residual;      // fused ops only
    const void* weight;  // nullptr = all ones
    void* out;           // 16-bit output (rms_norm, fused_add_rms_norm)
    uint8_t* q;          // e4m3 codes (fp8 op)
    float* scale;        // per-row scale (fp8 op)
    int64_t T;
    int64_t H;
    float eps;
};

// Operands of the fused SwiGLU + FP8 cast: x = [gate | up] rows of 2I.
struct SwigluArgs {
    const void* x;
    uint8_t* q;
    float* scale;
    int64_t T;
    int64_t I;
};

struct Launch {
    int kernel;  // 0 = vector, 1 = scalar, 2 = staged
    int tpr;     // threads per row
    int vpt;     // vector kernel: 16-byte vectors per thread; staged kernel: stages
    int rpc;     // rows per CTA
    int block;   // threads per CTA
    int smem;    // dynamic shared memory bytes
    int64_t grid;
    bool pdl;    // launch with programmatic stream serialization (PDL)
    bool pair = false;  // vector kernel, even VPT: 32-byte accesses (see rmsnorm_kernels.cu)
    bool prefetch = false;  // vector kernel under PDL: L2 prefetch of the first rows (ibid.)
};

// kSwigluFp8 names the SwiGLU + FP8 kernel to the launch planner only.
enum Op { kRmsNorm = 0, kFusedAdd = 1, kFusedAddFp8 = 2, kSwigluFp8 = 3 };
enum Dt { kF16 = 0, kBF16 = 1 };

// Compiled vectors-per-thread widths of the vector kernel, ascending.
constexpr int kVptList[] = {1, 2, 3, 4, 5, 6, 7, 8, 10, 12, 14, 15, 16};
constexpr int kNumVpt = sizeof(kVptList) / sizeof(kVptList[0]);

// Largest block the vector kernel of a given width is compiled for (its
// __launch_bounds__), which bounds the registers it may use per thread.
constexpr int max_block_for_vpt(int vpt) { return vpt <= 4 ? 1024 : (vpt <= 8 ? 512 : 256); }

// Dynamic shared memory the staged kernel may be configured for (B200: 227 KB
// per block) and the per-SM budget the planner spreads over resident CTAs.
constexpr int kStagedMaxSmem = 227 * 1024;
constexpr int kStagedSmemPerSm = 220 * 1024;

// Enqueues one launch; returns the CUDA error of the launch itself.
cudaError_t launch(int op, int dtype, const Args& a, const Launch& l, cudaStream_t s);

// Enqueues the fused SwiGLU + FP8 cast (vector plan: kernel 0; scalar: 1).
cudaError_t launch_swiglu_fp8(int dtype, const SwigluArgs& a, const Launch& l, cudaStream_t s);

// The compute capability (major * 10 + minor) the library's device code
// loaded on the current device was compiled for.
cudaError_t kernel_binary_version(int* version);

// Reads, and clears when set, the device-side error flags of the current
// device (bit 0: an mbarrier wait timed out). Synchronous.
cudaError_t read_and_clear_device_errors(unsigned* flags);

}  // namespace rn
