// rmsnorm_kernels.cu -- sm_100a kernels for rms_norm, fused_add_rms_norm and
// fused_add_rms_norm_fp8 over dense [T x H] fp16/bf16 rows.
//
// The operators are those wrapped in "vllm.kernels.aiter_ops"
// (rms_no_var_16bit_only, rms_add_no_var_16bit_only); the fp8 variant is the
// single-pass residual + RMSNorm + FP8 cast of "Custom CUDA kernels juice
// Llama 3.1 405B on AMD MI300X, skipping Nvidia lock-in".
//
// The work is HBM-bound (a few flops per byte), so the design is about bytes:
//  * vector kernel: a group of `tpr` threads owns one row; each thread keeps
//    VPT 16-byte vectors (8 elements each) of the row in registers between
//    the reduction and the output, so a row crosses HBM exactly once in each
//    direction (read x [+ residual], write [residual +] out or q). All of a
//    thread's loads are issued before any is consumed, for bytes in flight.
//    Loads skip L1 (each byte is used once); the weight is read through the
//    read-only path and stays cached (it is shared by every row).
//  * reductions: xor butterfly inside the warp (every lane ends with the same
//    total), then, for rows wider than a warp, one named barrier per row
//    group and a fixed-order sum over the group's warps from shared memory.
//    The order is fixed, so results are bit-reproducible run to run.
//  * scalar kernel: one CTA per row, two passes (the second re-reads the row,
//    mostly from L2); any H and any element-aligned pointers. It exists for
//    correctness on inputs the vector kernel cannot take.
//
// Numerics (identical in both kernels): residual sums in fp32 then one
// round-to-nearest-even to 16 bits (fp32 holds >= 2p+2 bits of either 16-bit
// format, so this equals the correctly rounded sum); squares accumulated in
// fp32; inv = 1 / sqrt(ss / H + eps) with IEEE sqrt and division; y = (v * w)
// * inv, where v * w is exact in fp32; fp8: P = max |v * w| (exact),
// q = e4m3(RNE, satfinite)((v * w) * (448 / P)), scale = (P * inv) / 448,
// which equals max |y| / 448 because rounding is monotonic.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "rn_internal.h"

namespace rn {
namespace {

// ---------------------------------------------------------------- formats

template <typename T>
struct Fmt;

template <>
struct Fmt<__nv_bfloat16> {
    static __device__ __forceinline__ float2 unpack(uint32_t u) {
        __nv_bfloat162 h;
        memcpy(&h, &u, 4);
        return __bfloat1622float2(h);
    }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
        uint32_t u;
        memcpy(&u, &h, 4);
        return u;
    }
    static __device__ __forceinline__ float load1(const void* p, int64_t i) {
        return __bfloat162float(static_cast<const __nv_bfloat16*>(p)[i]);
    }
    static __device__ __forceinline__ float round1(float v) {
        return __bfloat162float(__float2bfloat16_rn(v));
    }
    static __device__ __forceinline__ void store1(void* p, int64_t i, float v) {
        static_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
    }
};

template <>
struct Fmt<__half> {
    static __device__ __forceinline__ float2 unpack(uint32_t u) {
        __half2 h;
        memcpy(&h, &u, 4);
        return __half22float2(h);
    }
    static __device__ __forceinline__ uint32_t pack(float lo, float hi) {
        __half2 h = __floats2half2_rn(lo, hi);
        uint32_t u;
        memcpy(&u, &h, 4);
        return u;
    }
    static __device__ __forceinline__ float load1(const void* p, int64_t i) {
        return __half2float(static_cast<const __half*>(p)[i]);
    }
    static __device__ __forceinline__ float round1(float v) {
        return __half2float(__float2half_rn(v));
    }
    static __device__ __forceinline__ void store1(void* p, int64_t i, float v) {
        static_cast<__half*>(p)[i] = __float2half_rn(v);
    }
};

// ---------------------------------------------------------------- PTX helpers

// Streaming 16-byte load: coherent global load that does not allocate in L1
// (the residual is written back by the same kernel, so the non-coherent path
// is not used for activations).
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 v;
    asm volatile("ld.global.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

__device__ __forceinline__ void st_v4(uint4* p, const uint4& v) {
    asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_v2(uint2* p, const uint2& v) {
    asm volatile("st.global.v2.u32 [%0], {%1, %2};" ::"l"(p), "r"(v.x), "r"(v.y) : "memory");
}

// Barrier over the `nthreads` threads of one row group (ids 1..15; 0 is
// __syncthreads).
__device__ __forceinline__ void group_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Two fp32 values to two e4m3fn codes (round to nearest even, saturating to
// +-448); `lo` lands in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// ---------------------------------------------------------------- vector kernel

template <typename T, int VPT, int OP>
__global__ void __launch_bounds__(max_block_for_vpt(VPT))
    rn_vector_kernel(const Args a, const int tpr, const int rpc) {
    using F = Fmt<T>;
    constexpr bool kFused = OP != kRmsNorm;
    constexpr bool kFp8 = OP == kFusedAddFp8;
    extern __shared__ float2 red[];  // [2][rpc][warps per row]

    const int row_in_cta = threadIdx.x / tpr;
    const int lr = threadIdx.x - row_in_cta * tpr;
    const int wpr = tpr >> 5;
    const int64_t nvec = a.H >> 3;
    const float hf = static_cast<float>(a.H);
    const uint4* __restrict__ xv = static_cast<const uint4*>(a.x);
    uint4* rv = static_cast<uint4*>(a.residual);
    const uint4* __restrict__ wv = static_cast<const uint4*>(a.weight);
    const bool has_w = wv != nullptr;
    int parity = 0;

    // The loop bound depends only on the block, so every thread of a warp
    // runs the same iterations (the shuffles below use the full mask).
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * rpc; base < a.T;
         base += static_cast<int64_t>(gridDim.x) * rpc) {
        const int64_t row = base + row_in_cta;
        const bool active = row < a.T;
        const int64_t roff = row * nvec;

        uint4 v[VPT];
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int64_t j = lr + static_cast<int64_t>(k) * tpr;
            v[k] = (active && j < nvec) ? ld_stream(xv + roff + j) : make_uint4(0, 0, 0, 0);
        }
        if constexpr (kFused) {
            uint4 r[VPT];
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                const int64_t j = lr + static_cast<int64_t>(k) * tpr;
                r[k] = (active && j < nvec) ? ld_stream(rv + roff + j) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                const int64_t j = lr + static_cast<int64_t>(k) * tpr;
                uint32_t* xs = &v[k].x;
                const uint32_t* rs = &r[k].x;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float2 fx = F::unpack(xs[c]);
                    const float2 fr = F::unpack(rs[c]);
                    xs[c] = F::pack(fx.x + fr.x, fx.y + fr.y);
                }
                if (active && j < nvec) st_v4(rv + roff + j, v[k]);
            }
        }

        float ss = 0.f, pm = 0.f;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const uint32_t* xs = &v[k].x;
            uint4 wk = make_uint4(0, 0, 0, 0);
            if constexpr (kFp8) {
                const int64_t j = lr + static_cast<int64_t>(k) * tpr;
                if (has_w && j < nvec) wk = __ldg(wv + j);
            }
            const uint32_t* ws = &wk.x;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const float2 f = F::unpack(xs[c]);
                ss = fmaf(f.x, f.x, ss);
                ss = fmaf(f.y, f.y, ss);
                if constexpr (kFp8) {
                    const float2 wf = has_w ? F::unpack(ws[c]) : make_float2(1.f, 1.f);
                    pm = fmaxf(pm, fabsf(f.x * wf.x));
                    pm = fmaxf(pm, fabsf(f.y * wf.y));
                }
            }
        }

        const int width = tpr < 32 ? tpr : 32;
        for (int o = width >> 1; o > 0; o >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if constexpr (kFp8) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, o));
        }
        if (wpr > 1) {
            float2* slot = red + (static_cast<int64_t>(parity) * rpc + row_in_cta) * wpr;
            if ((lr & 31) == 0) slot[lr >> 5] = make_float2(ss, pm);
            group_barrier(1 + row_in_cta, tpr);
            float s = 0.f, m = 0.f;
            for (int i = 0; i < wpr; ++i) {
                const float2 t = slot[i];
                s += t.x;
                m = fmaxf(m, t.y);
            }
            ss = s;
            pm = m;
            parity ^= 1;  // the next row uses the other half of `red`
        }

        const float inv = 1.0f / sqrtf(ss / hf + a.eps);

        if constexpr (!kFp8) {
            uint4* ov = static_cast<uint4*>(a.out);
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                const int64_t j = lr + static_cast<int64_t>(k) * tpr;
                if (!(active && j < nvec)) continue;
                const uint4 wk = has_w ? __ldg(wv + j) : make_uint4(0, 0, 0, 0);
                const uint32_t* xs = &v[k].x;
                const uint32_t* ws = &wk.x;
                uint4 o;
                uint32_t* os = &o.x;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float2 f = F::unpack(xs[c]);
                    const float2 wf = has_w ? F::unpack(ws[c]) : make_float2(1.f, 1.f);
                    os[c] = F::pack((f.x * wf.x) * inv, (f.y * wf.y) * inv);
                }
                st_v4(ov + roff + j, o);
            }
        } else {
            const float qmul = pm > 0.f ? 448.0f / pm : 0.f;
            if (active && lr == 0) a.scale[row] = pm > 0.f ? (pm * inv) / 448.0f : 0.f;
            uint2* qv = reinterpret_cast<uint2*>(a.q);
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                const int64_t j = lr + static_cast<int64_t>(k) * tpr;
                if (!(active && j < nvec)) continue;
                const uint4 wk = has_w ? __ldg(wv + j) : make_uint4(0, 0, 0, 0);
                const uint32_t* xs = &v[k].x;
                const uint32_t* ws = &wk.x;
                uint32_t e[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float2 f = F::unpack(xs[c]);
                    const float2 wf = has_w ? F::unpack(ws[c]) : make_float2(1.f, 1.f);
                    e[c] = e4m3x2((f.x * wf.x) * qmul, (f.y * wf.y) * qmul);
                }
                uint2 o = make_uint2(e[0] | (e[1] << 16), e[2] | (e[3] << 16));
                if (!(pm > 0.f)) o = make_uint2(0, 0);
                st_v2(qv + roff + j, o);
            }
        }
    }
}

// ---------------------------------------------------------------- scalar kernel

constexpr int kScalarBlock = 256;

template <typename T, int OP>
__global__ void __launch_bounds__(kScalarBlock) rn_scalar_kernel(const Args a) {
    using F = Fmt<T>;
    constexpr bool kFused = OP != kRmsNorm;
    constexpr bool kFp8 = OP == kFusedAddFp8;
    __shared__ float2 red[kScalarBlock / 32];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const float hf = static_cast<float>(a.H);

    for (int64_t row = blockIdx.x; row < a.T; row += gridDim.x) {
        const int64_t off = row * a.H;
        float ss = 0.f, pm = 0.f;
        for (int64_t i = threadIdx.x; i < a.H; i += kScalarBlock) {
            float v = F::load1(a.x, off + i);
            if constexpr (kFused) {
                v = F::round1(v + F::load1(a.residual, off + i));
                F::store1(a.residual, off + i, v);
            }
            ss = fmaf(v, v, ss);
            if constexpr (kFp8) {
                const float w = a.weight ? F::load1(a.weight, i) : 1.f;
                pm = fmaxf(pm, fabsf(v * w));
            }
        }
        for (int o = 16; o > 0; o >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if constexpr (kFp8) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, o));
        }
        if (lane == 0) red[warp] = make_float2(ss, pm);
        __syncthreads();
        ss = 0.f;
        pm = 0.f;
        for (int i = 0; i < kScalarBlock / 32; ++i) {
            ss += red[i].x;
            pm = fmaxf(pm, red[i].y);
        }
        const float inv = 1.0f / sqrtf(ss / hf + a.eps);
        const float qmul = pm > 0.f ? 448.0f / pm : 0.f;
        for (int64_t i = threadIdx.x; i < a.H; i += kScalarBlock) {
            // The second pass re-reads what this same thread read or wrote.
            const float v = kFused ? F::load1(a.residual, off + i) : F::load1(a.x, off + i);
            const float w = a.weight ? F::load1(a.weight, i) : 1.f;
            if constexpr (kFp8) {
                a.q[off + i] = pm > 0.f ? static_cast<uint8_t>(e4m3x2((v * w) * qmul, 0.f) & 0xff)
                                        : uint8_t(0);
            } else {
                F::store1(a.out, off + i, (v * w) * inv);
            }
        }
        if (kFp8 && threadIdx.x == 0) a.scale[row] = pm > 0.f ? (pm * inv) / 448.0f : 0.f;
        __syncthreads();  // `red` is reused by the next row
    }
}

// ---------------------------------------------------------------- dispatch

template <typename T, int OP, int VPT>
cudaError_t launch_vector(const Args& a, const Launch& l, cudaStream_t s) {
    rn_vector_kernel<T, VPT, OP><<<static_cast<unsigned>(l.grid), l.block, l.smem, s>>>(a, l.tpr,
                                                                                        l.rpc);
    return cudaGetLastError();
}

template <typename T, int OP, int I = 0>
cudaError_t dispatch_vpt(const Args& a, const Launch& l, cudaStream_t s) {
    if constexpr (I < kNumVpt) {
        if (l.vpt == kVptList[I]) return launch_vector<T, OP, kVptList[I]>(a, l, s);
        return dispatch_vpt<T, OP, I + 1>(a, l, s);
    } else {
        return cudaErrorInvalidValue;
    }
}

template <typename T, int OP>
cudaError_t launch_typed(const Args& a, const Launch& l, cudaStream_t s) {
    if (l.kernel == 0) return dispatch_vpt<T, OP>(a, l, s);
    rn_scalar_kernel<T, OP><<<static_cast<unsigned>(l.grid), kScalarBlock, 0, s>>>(a);
    return cudaGetLastError();
}

template <typename T>
cudaError_t launch_op(int op, const Args& a, const Launch& l, cudaStream_t s) {
    switch (op) {
        case kRmsNorm: return launch_typed<T, kRmsNorm>(a, l, s);
        case kFusedAdd: return launch_typed<T, kFusedAdd>(a, l, s);
        case kFusedAddFp8: return launch_typed<T, kFusedAddFp8>(a, l, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch(int op, int dtype, const Args& a, const Launch& l, cudaStream_t s) {
    if (dtype == kBF16) return launch_op<__nv_bfloat16>(op, a, l, s);
    if (dtype == kF16) return launch_op<__half>(op, a, l, s);
    return cudaErrorInvalidValue;
}

}  // namespace rn
