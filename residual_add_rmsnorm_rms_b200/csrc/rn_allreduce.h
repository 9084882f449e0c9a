// rn_allreduce.h -- interface between the C-ABI layer (rmsnorm_api.cpp) and
// the tensor-parallel all-reduce kernels (allreduce_kernels.cu). Internal.
#pragma once

#include <cstdint>

#include <cuda_runtime_api.h>

namespace rn {

// Tensor-parallel all-reduce fused with the residual add and RMSNorm.

constexpr int kArMaxWorld = 8;      // ranks in one group (one NVSwitch domain)
constexpr int kArMaxBlocks = 1024;  // signal-pad capacity, in blocks per rank
constexpr int kArMaxBlock = 512;    // threads per block (the kernel's launch bound)
constexpr int kArSignalBytes = 64 + 4 * kArMaxBlocks * kArMaxWorld * 4;  // per rank

struct ArArgs {
    int world;                        // ranks in the group
    int rank;                         // rank driven by blockIdx.y == 0
    void* buffers[kArMaxWorld];       // every rank's exchange buffer (this process's address)
    uint32_t* signals[kArMaxWorld];   // every rank's signal pad (kArSignalBytes)
    int64_t slot_elems;               // 16-bit elements per buffer half (call parity picks one):
                                      // >= T*H (one-shot) or 3*T*H (two-shot)
    long long timeout_ns;             // bound on each wait for a peer
    const void* x;                    // partial sums [local ranks][T][H]
    void* residual;                   // [local ranks][T][H], in place
    const void* weight;               // [H] or nullptr
    void* out;                        // 16-bit op: [local ranks][T][H]
    uint8_t* q;                       // fp8 op: codes [local ranks][T][H]
    float* scale;                     // fp8 op: [local ranks][T]
    int64_t T, H;
    float eps;
};

struct ArLaunch {
    int tpr;          // threads per row
    int vpt;          // 16-byte vectors per thread per row: 1, 2, 4 or 8
    int rpc;          // rows per block
    int block;        // threads per block
    int smem;         // dynamic shared memory bytes
    int grid_x;       // blocks per rank (the same on every rank)
    int local_ranks;  // gridDim.y
    bool two_shot;    // reduce-scatter of row slices + gather of finished rows
    bool wide = false;  // groups of 4-8 ranks: the 80-register kernel (more blocks per SM)
};

// Resident blocks per SM of the all-reduce kernel for this shape.
cudaError_t allreduce_blocks_per_sm(int dtype, bool fp8, int world, const ArLaunch& l,
                                    int* blocks);

// Launches the all-reduce kernel: cooperatively (every block resident) when
// one launch computes several ranks, whose blocks wait on one another.
cudaError_t launch_allreduce(int dtype, bool fp8, const ArArgs& a, const ArLaunch& l,
                             cudaStream_t s);

// Static exchange memory of rn_allreduce_fused_add_rms_norm_local (a whole
// group on one device): kArMaxWorld signal pads, kLocalPadStride bytes apart,
// then up to kLocalBufferBytes of exchange buffers.
constexpr int64_t kLocalPadStride = ((kArSignalBytes + 255) / 256) * 256;
constexpr int64_t kLocalBufferBytes = 32LL << 20;
constexpr int64_t kLocalScratchBytes = kLocalPadStride * kArMaxWorld + kLocalBufferBytes;

// Device address of that memory on the current device.
cudaError_t local_scratch_address(void** p);

// Reads, and clears when set, the all-reduce kernel's error flags on the
// current device (bit 1: a wait for a peer timed out). Synchronous.
cudaError_t read_and_clear_allreduce_errors(unsigned* flags);

}  // namespace rn
