// swiglu_fp8_kernels.cu -- fused SwiGLU + per-token dynamic FP8 e4m3 cast.
//
// The second of the three kernels of "Custom CUDA kernels juice Llama 3.1
// 405B on AMD MI300X, skipping Nvidia lock-in": the SwiGLU activation merged
// with an FP8 cast. Per row t of x = [gate | up] ([T x 2I], 16-bit):
//   y_i = silu(gate_i) * up_i,  silu(a) = a / (1 + e^-a)      (fp32)
//   scale_t = max_i |y_i| / 448,  q_i = e4m3(RNE, satfinite)(y_i * 448 / max|y|)
// with scale 0 and all-zero codes for a row whose max |y| is 0.
//
// HBM-bound like the norm kernels (2 x 2 bytes read and 1 byte written per
// output element), so the same register-resident mapping is used: `tpr`
// threads per row, VPT 16-byte vectors of gate and of up per thread, all
// loads issued before use, one max-reduction per row (warp butterfly, then a
// named barrier across the row's warps), one pass writing the codes. With an
// even VPT, I % 16 == 0, 32-byte aligned x rows and 16-byte aligned code rows
// (kPair), a thread's vectors come in adjacent pairs moved by sm_100's 32-byte
// loads (codes: 16-byte stores), as in the norm kernels' vector kernel. silu
// takes two multi-function-unit operations per element (a base-2 exponential
// of an argument carried in two floats, and a reciprocal) and packed
// two-lane fp32 arithmetic for the rest: at ~1.3e12 elements/s the library's
// accurate exponential and IEEE division would make the kernel issue-bound. Under programmatic dependent launch a block
// prefetches its first row into L2 before waiting for the previous kernel,
// as the norm kernels do.
#include <cstdint>

#include "rn_device.cuh"
#include "rn_internal.h"

namespace rn {
namespace {

// log2(e) split into a float and the float nearest to the remainder
// (Cody and Waite's argument reduction, "Software Manual for the Elementary
// Functions", 1980), and ln(2).
constexpr float kLog2eHi = 1.44269502162933349609375f;
constexpr float kLog2eLo = 1.925963033500e-8f;
constexpr float kLn2 = 0.693147180559945309f;

// 2^x for an fp32 x on the multi-function unit (ex2.approx: the integer
// part of x is exact, the relative error is a few ulp whatever |x|).
__device__ __forceinline__ float exp2_mufu(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// 1 / d on the multi-function unit (rcp.approx: within an ulp; with .ftz a
// divisor past 2^126 gives 0, and +inf gives 0).
__device__ __forceinline__ float rcp_mufu(float d) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(d));
    return r;
}

// silu(g) * u for a pair, in fp32, with packed two-lane arithmetic:
//   silu(g) = g * 1 / (1 + e^-g),  e^-g = 2^p,  p = -g log2(e).
// Forming p as one float would round it by up to half an ulp of |g| * 1.44,
// an error e^-g inherits multiplied by |g| * 1.44 (tens of ulp at |g| = 20).
// Here p = p_hi + p_lo to about 2^-40 relative: p_lo is the exact rounding
// error of -g * kLog2eHi (an fma) plus -g * kLog2eLo, and
// 2^p = 2^p_hi * (1 + p_lo ln 2) to within (p_lo ln 2)^2 < 2^-32. With the
// base-2 exponential and the reciprocal of the multi-function unit and four
// more roundings, y is within a few ulp of its exact value for any finite
// gate, so the row maximum, hence the per-token scale, is within 1e-6. An
// exponent past 128 gives e^-g = +inf and silu = 0; for g < -87.3 the
// divisor exceeds 2^126 and silu (then below 1e-36 in magnitude) is 0 too.
__device__ __forceinline__ float2 swiglu2(float2 g, float2 u) {
    const float2 ng = make_float2(-g.x, -g.y);
    const float2 lhi = make_float2(kLog2eHi, kLog2eHi);
    const float2 one = make_float2(1.0f, 1.0f);
    const float2 p_hi = __fmul2_rn(ng, lhi);
    float2 p_lo = __ffma2_rn(ng, lhi, make_float2(-p_hi.x, -p_hi.y));
    p_lo = __ffma2_rn(ng, make_float2(kLog2eLo, kLog2eLo), p_lo);
    const float2 e_hi = make_float2(exp2_mufu(p_hi.x), exp2_mufu(p_hi.y));
    const float2 e = __fmul2_rn(e_hi, __ffma2_rn(p_lo, make_float2(kLn2, kLn2), one));
    const float2 d = __fadd2_rn(e, one);
    const float2 silu = __fmul2_rn(g, make_float2(rcp_mufu(d.x), rcp_mufu(d.y)));
    return __fmul2_rn(silu, u);
}

// Index (in 16-byte vectors) of a thread's vector k: strided by tpr, or with
// kPair, pair k / 2 strided by tpr and its two vectors adjacent.
template <bool kPair>
__device__ __forceinline__ int swiglu_vec_index(int lr, int k, int tpr) {
    if constexpr (kPair) return 2 * (lr + (k >> 1) * tpr) + (k & 1);
    return lr + k * tpr;
}

// L2 prefetch of the block's first rows ([gate | up], 4I bytes each) in 4 KB
// pieces spread over the row group's threads. Rows are 16-byte aligned and
// 4I is a multiple of 16 on the vector path.
__device__ __forceinline__ void swiglu_prefetch_first_rows(const SwigluArgs& a, const int tpr,
                                                           const int rpc) {
    constexpr uint32_t kChunk = 4096;
    const int row_in_cta = threadIdx.x / tpr;
    const int lr = threadIdx.x - row_in_cta * tpr;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * rpc + row_in_cta;
    if (row >= a.T) return;
    const uint32_t row_bytes = static_cast<uint32_t>(a.I) * 4u;
    const char* xr = static_cast<const char*>(a.x) + row * row_bytes;
    for (uint32_t off = static_cast<uint32_t>(lr) * kChunk; off < row_bytes;
         off += static_cast<uint32_t>(tpr) * kChunk)
        prefetch_l2(xr + off, row_bytes - off < kChunk ? row_bytes - off : kChunk);
}

template <typename T, int VPT, bool kPair>
__global__ void __launch_bounds__(max_block_for_vpt(VPT))
    rn_swiglu_fp8_kernel(const SwigluArgs a, const int tpr, const int rpc, const int prefetch) {
    static_assert(!kPair || VPT % 2 == 0, "pairs need an even vector count");
    constexpr int kStep = kPair ? 2 : 1;
    using F = Fmt<T>;
    extern __shared__ float red[];  // [2][rpc][warps per row]
    pdl_allow_dependents();
    if (prefetch) swiglu_prefetch_first_rows(a, tpr, rpc);
    pdl_wait_for_prior_grid();

    const int row_in_cta = threadIdx.x / tpr;
    const int lr = threadIdx.x - row_in_cta * tpr;
    const int wpr = tpr >> 5;
    const int ivec = static_cast<int>(a.I >> 3);
    int parity = 0;

    for (int64_t base = static_cast<int64_t>(blockIdx.x) * rpc; base < a.T;
         base += static_cast<int64_t>(gridDim.x) * rpc) {
        const int64_t row = base + row_in_cta;
        const bool active = row < a.T;
        const int64_t r0 = active ? row : 0;
        const uint4* grow = static_cast<const uint4*>(a.x) + r0 * 2 * ivec;
        const uint4* urow = grow + ivec;

        uint4 g[VPT], u[VPT];
        const uint4 z4 = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int k = 0; k < VPT; k += kStep) {
            const int j = swiglu_vec_index<kPair>(lr, k, tpr);
            const bool ok = active && j < ivec;
            if constexpr (kPair) {
                if (ok) {
                    ld_stream2(grow + j, g[k], g[k + 1]);
                    ld_stream2(urow + j, u[k], u[k + 1]);
                } else {
                    g[k] = g[k + 1] = u[k] = u[k + 1] = z4;
                }
            } else {
                g[k] = ok ? ld_stream(grow + j) : z4;
                u[k] = ok ? ld_stream(urow + j) : z4;
            }
        }
        float2 y[VPT][4];
        float pm = 0.f;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const uint32_t* gs = &g[k].x;
            const uint32_t* us = &u[k].x;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                y[k][c] = swiglu2(F::unpack(gs[c]), F::unpack(us[c]));
                pm = fmaxf(pm, fmaxf(fabsf(y[k][c].x), fabsf(y[k][c].y)));
            }
        }

        const int width = tpr < 32 ? tpr : 32;
        for (int o = width >> 1; o > 0; o >>= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, o));
        if (wpr > 1) {
            float* slot = red + (parity * rpc + row_in_cta) * wpr;
            if ((lr & 31) == 0) slot[lr >> 5] = pm;
            group_barrier(1 + row_in_cta, tpr);
            float m = 0.f;
            for (int i = 0; i < wpr; ++i) m = fmaxf(m, slot[i]);
            pm = m;
            parity ^= 1;
        }

        const float qmul = pm > 0.f ? 448.0f / pm : 0.f;
        const float2 q2 = make_float2(qmul, qmul);
        if (active && lr == 0) a.scale[row] = pm > 0.f ? pm / 448.0f : 0.f;
        uint2* qrow = reinterpret_cast<uint2*>(a.q) + r0 * ivec;
        auto codes = [&](int k) {
            uint32_t e[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float2 p = __fmul2_rn(y[k][c], q2);
                e[c] = e4m3x2(p.x, p.y);
            }
            uint2 o = make_uint2(e[0] | (e[1] << 16), e[2] | (e[3] << 16));
            if (!(pm > 0.f)) o = make_uint2(0, 0);
            return o;
        };
#pragma unroll
        for (int k = 0; k < VPT; k += kStep) {
            const int j = swiglu_vec_index<kPair>(lr, k, tpr);
            if (!(active && j < ivec)) continue;
            const uint2 o = codes(k);
            if constexpr (kPair) {
                const uint2 o1 = codes(k + 1);
                st_v4(reinterpret_cast<uint4*>(qrow + j), make_uint4(o.x, o.y, o1.x, o1.y));
            } else {
                st_v2(qrow + j, o);
            }
        }
    }
}

// Any I and element-aligned pointers: one 256-thread block per row, silu
// evaluated twice (max pass, then code pass).
constexpr int kSwigluScalarBlock = 256;

template <typename T>
__global__ void __launch_bounds__(kSwigluScalarBlock) rn_swiglu_fp8_scalar_kernel(const SwigluArgs a) {
    using F = Fmt<T>;
    __shared__ float red[kSwigluScalarBlock / 32];
    pdl_allow_dependents();
    pdl_wait_for_prior_grid();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t row = blockIdx.x; row < a.T; row += gridDim.x) {
        const int64_t off = row * 2 * a.I;
        float pm = 0.f;
        for (int64_t i = threadIdx.x; i < a.I; i += kSwigluScalarBlock) {
            const float y = swiglu2(make_float2(F::load1(a.x, off + i), 0.f),
                                    make_float2(F::load1(a.x, off + a.I + i), 0.f)).x;
            pm = fmaxf(pm, fabsf(y));
        }
        for (int o = 16; o > 0; o >>= 1) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, o));
        if (lane == 0) red[warp] = pm;
        __syncthreads();
        pm = 0.f;
        for (int i = 0; i < kSwigluScalarBlock / 32; ++i) pm = fmaxf(pm, red[i]);
        const float qmul = pm > 0.f ? 448.0f / pm : 0.f;
        for (int64_t i = threadIdx.x; i < a.I; i += kSwigluScalarBlock) {
            const float y = swiglu2(make_float2(F::load1(a.x, off + i), 0.f),
                                    make_float2(F::load1(a.x, off + a.I + i), 0.f)).x;
            a.q[row * a.I + i] = pm > 0.f ? static_cast<uint8_t>(e4m3x2(y * qmul, 0.f) & 0xff)
                                          : uint8_t(0);
        }
        if (threadIdx.x == 0) a.scale[row] = pm > 0.f ? pm / 448.0f : 0.f;
        __syncthreads();
    }
}

template <typename T, int I = 0>
cudaError_t swiglu_dispatch_vpt(const SwigluArgs& a, const Launch& l, cudaStream_t s) {
    if constexpr (I < kNumVpt) {
        if (l.vpt == kVptList[I]) {
            const int pf = l.pdl && l.prefetch ? 1 : 0;
            if constexpr (kVptList[I] % 2 == 0) {
                if (l.pair)
                    return launch_kernel(rn_swiglu_fp8_kernel<T, kVptList[I], true>, l, s, a,
                                         l.tpr, l.rpc, pf);
            }
            return launch_kernel(rn_swiglu_fp8_kernel<T, kVptList[I], false>, l, s, a, l.tpr,
                                 l.rpc, pf);
        }
        return swiglu_dispatch_vpt<T, I + 1>(a, l, s);
    } else {
        return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t swiglu_launch_typed(const SwigluArgs& a, const Launch& l, cudaStream_t s) {
    if (l.kernel == 0) return swiglu_dispatch_vpt<T>(a, l, s);
    Launch ls = l;
    ls.block = kSwigluScalarBlock;
    ls.smem = 0;
    return launch_kernel(rn_swiglu_fp8_scalar_kernel<T>, ls, s, a);
}

}  // namespace

cudaError_t launch_swiglu_fp8(int dtype, const SwigluArgs& a, const Launch& l, cudaStream_t s) {
    if (dtype == kBF16) return swiglu_launch_typed<__nv_bfloat16>(a, l, s);
    if (dtype == kF16) return swiglu_launch_typed<__half>(a, l, s);
    return cudaErrorInvalidValue;
}

}  // namespace rn
