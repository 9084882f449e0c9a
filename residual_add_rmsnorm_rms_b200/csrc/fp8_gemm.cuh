// fp8_gemm.cuh -- the row-wise scaled FP8 GEMM template shared by the
// translation units that instantiate its tile shapes:
//
//   D[m, n] = bf16( b_scale[n] * (a_scale[m] * sum_k A[m, k] * B[n, k]) )
//
// A [M x K] e4m3 (row-major, K contiguous) is what fused_add_rms_norm_fp8
// produces together with its per-token a_scale; B [N x K] e4m3 is a weight
// with one scale per output channel. This is the consumer of the fused
// residual + RMSNorm + FP8 pass in the decode path of "Custom CUDA kernels
// juice Llama 3.1 405B on AMD MI300X, skipping Nvidia lock-in" and the
// row-wise fp8 linear layers (RowWiseTorchFP8ScaledMMLinearKernel) in the
// table of "VLLM_ROCM_USE_AITER=1 slows Gemma 4 on an AMD MI300X".
//
// Built from CUTLASS's sm100 collectives: tcgen05 MMA issued by one thread
// with the accumulator in tensor memory, TMA loads of both operand tiles into
// a multi-stage shared-memory pipeline, warp-specialised (load / MMA /
// epilogue warps), persistent tile scheduler, cluster 1 x 1 x 1 (no
// multicast), K step 128, launched with programmatic dependent launch (the
// kernel waits for the previous kernel in the stream before its first global
// memory access, so its launch and prologue overlap that kernel's tail). The epilogue is an epilogue-visitor tree: fp32
// accumulator x a_scale[m], then x b_scale[n], rounded once to bf16, stored
// by TMA.
//
// Two orientations:
//  * token-major (kSwapAB = false): the MMA's M runs over tokens and its N over
//    output channels; tile MmaTile = (tokens, channels, 128).
//  * channel-major (kSwapAB = true): computes D^T = B * A^T, so the MMA's M
//    runs over the weight's output channels and its N over tokens; tile
//    MmaTile = (channels, tokens, 128). D^T is column-major [N x M], which is
//    D row-major. For a handful of tokens this keeps the MMA's fixed 64/128
//    rows on the weight instead of padding the tokens to 128: the tensor core
//    then does only as much work as the tokens need and the kernel streams
//    the weight.
// Both orientations apply the two scales in the same order (a_scale first),
// so they round identically.
#pragma once

#include <atomic>
#include <cstdint>
#include <type_traits>

#include "cutlass/cutlass.h"
#include "cute/tensor.hpp"
#include "cutlass/epilogue/collective/collective_builder.hpp"
#include "cutlass/epilogue/fusion/sm90_visitor_tma_warpspecialized.hpp"
#include "cutlass/gemm/collective/collective_builder.hpp"
#include "cutlass/gemm/device/gemm_universal_adapter.h"
#include "cutlass/gemm/kernel/gemm_universal.hpp"
#include "cutlass/util/packed_stride.hpp"

#include "rn_gemm.h"

namespace rn {
namespace gemm_detail {

using namespace cute;
namespace fusion = cutlass::epilogue::fusion;

using ElementAB = cutlass::float_e4m3_t;
using ElementD = cutlass::bfloat16_t;
constexpr int kAlignAB = 16;  // elements: 16 bytes of e4m3 per TMA row granule
constexpr int kAlignD = 8;    // elements: 16 bytes of bf16
constexpr int kGemmMaxDevices = 64;

template <class MmaTile, bool kSwapAB>
struct RowwiseGemm {
    using Cluster = Shape<_1, _1, _1>;
    // Both operands are stored K-contiguous: the first as RowMajor [rows x K],
    // the second as ColumnMajor K x cols (i.e. [cols x K] row-major).
    using LayoutFirst = cutlass::layout::RowMajor;
    using LayoutSecond = cutlass::layout::ColumnMajor;
    using LayoutD = std::conditional_t<kSwapAB, cutlass::layout::ColumnMajor,
                                       cutlass::layout::RowMajor>;
    // Per-row broadcast of the MMA problem = ColBroadcast, per-column =
    // RowBroadcast. a_scale follows the tokens, b_scale the channels.
    using RowVec = fusion::Sm90ColBroadcast<0, MmaTile, float, float, Stride<_1, _0, int64_t>>;
    using ColVec = fusion::Sm90RowBroadcast<0, MmaTile, float, float, Stride<_0, _1, int64_t>>;
    using ScaleA = std::conditional_t<kSwapAB, ColVec, RowVec>;
    using ScaleB = std::conditional_t<kSwapAB, RowVec, ColVec>;
    using MulA = fusion::Sm90Compute<cutlass::multiplies, float, float,
                                     cutlass::FloatRoundStyle::round_to_nearest>;
    using MulB = fusion::Sm90Compute<cutlass::multiplies, ElementD, float,
                                     cutlass::FloatRoundStyle::round_to_nearest>;
    using Evt = fusion::Sm90EVT<MulB, ScaleB, fusion::Sm90EVT<MulA, ScaleA, fusion::Sm90AccFetch>>;

    using Epilogue = typename cutlass::epilogue::collective::CollectiveBuilder<
        cutlass::arch::Sm100, cutlass::arch::OpClassTensorOp, MmaTile, Cluster,
        cutlass::epilogue::collective::EpilogueTileAuto, float, float, void, LayoutD, kAlignD,
        ElementD, LayoutD, kAlignD, cutlass::epilogue::TmaWarpSpecialized1Sm, Evt>::CollectiveOp;

    using Mainloop = typename cutlass::gemm::collective::CollectiveBuilder<
        cutlass::arch::Sm100, cutlass::arch::OpClassTensorOp, ElementAB, LayoutFirst, kAlignAB,
        ElementAB, LayoutSecond, kAlignAB, float, MmaTile, Cluster,
        cutlass::gemm::collective::StageCountAutoCarveout<
            static_cast<int>(sizeof(typename Epilogue::SharedStorage))>,
        cutlass::gemm::KernelTmaWarpSpecialized1SmSm100>::CollectiveOp;

    using Kernel =
        cutlass::gemm::kernel::GemmUniversal<Shape<int, int, int, int>, Mainloop, Epilogue, void>;
    using Gemm = cutlass::gemm::device::GemmUniversalAdapter<Kernel>;

    static cudaError_t run(const GemmArgs& g, cudaStream_t stream) {
        const int M = static_cast<int>(g.M), N = static_cast<int>(g.N), K = static_cast<int>(g.K);
        // The MMA problem: (rows, cols) = (M, N), or (N, M) when swapped.
        const int R = kSwapAB ? N : M, C = kSwapAB ? M : N;
        const void* first = kSwapAB ? g.b : g.a;
        const void* second = kSwapAB ? g.a : g.b;
        typename Gemm::Arguments args;
        args.mode = cutlass::gemm::GemmUniversalMode::kGemm;
        args.problem_shape = {R, C, K, 1};
        const auto s1 = cutlass::make_cute_packed_stride(typename Kernel::StrideA{},
                                                         make_shape(R, K, 1));
        const auto s2 = cutlass::make_cute_packed_stride(typename Kernel::StrideB{},
                                                         make_shape(C, K, 1));
        const auto sD = cutlass::make_cute_packed_stride(typename Kernel::StrideD{},
                                                         make_shape(R, C, 1));
        args.mainloop = {static_cast<const ElementAB*>(first), s1,
                         static_cast<const ElementAB*>(second), s2};
        args.epilogue.ptr_C = nullptr;
        args.epilogue.dC = sD;
        args.epilogue.ptr_D = static_cast<ElementD*>(g.d);
        args.epilogue.dD = sD;
        args.epilogue.thread = {
            {g.b_scale, 0.f, {}},            // b_scale[n] (outer multiply)
            {{g.a_scale, 0.f, {}}, {}, {}},  // a_scale[m] * accumulator
            {}};
        args.hw_info.device_id = g.device;
        args.hw_info.sm_count = g.num_sms;
        if (Gemm::can_implement(args) != cutlass::Status::kSuccess) return cudaErrorInvalidValue;
        if (Gemm::get_workspace_size(args) != 0) return cudaErrorInvalidValue;  // none by design
        if (Kernel::initialize_workspace(args, nullptr, stream) != cutlass::Status::kSuccess)
            return cudaErrorInvalidConfiguration;
        typename Gemm::Params params = Kernel::to_underlying_arguments(args, nullptr);
        // The adapter's initialize() sets the kernel's dynamic shared memory
        // limit on every call; here it is set once per device and CUDA context
        // (and on every call when the context id is unknown).
        static std::atomic<unsigned long long> ready[kGemmMaxDevices];
        const bool known = g.ctx_id != 0 && g.device >= 0 && g.device < kGemmMaxDevices;
        if (!known || ready[g.device].load(std::memory_order_relaxed) != g.ctx_id) {
            const cudaError_t e = cudaFuncSetAttribute(
                cutlass::device_kernel<Kernel>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                static_cast<int>(Kernel::SharedStorageSize));
            if (e != cudaSuccess) return e;
            if (known) ready[g.device].store(g.ctx_id, std::memory_order_relaxed);
        }
        if (Gemm::run(params, stream, nullptr, g.pdl) != cutlass::Status::kSuccess)
            return cudaErrorLaunchFailure;
        return cudaGetLastError();
    }
};

}  // namespace gemm_detail
}  // namespace rn
