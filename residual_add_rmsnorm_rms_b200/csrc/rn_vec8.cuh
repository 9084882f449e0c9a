// rn_vec8.cuh -- arithmetic on 8 16-bit elements held in one 16-byte vector
// (uint4: 4 packed pairs), shared by the norm kernels and the all-reduce
// fused kernels so that both round identically. Internal.
#pragma once

#include <type_traits>

#include "rn_device.cuh"

namespace rn {
namespace {

// A uint4 holds 8 16-bit elements (4 packed pairs). Weights arrive as 4 fp32
// pairs. The fp32 arithmetic uses Blackwell's paired instructions (two
// lanes of fp32 per instruction, each rounded exactly like its scalar form).

struct W8 {
    float2 w[4];
};

template <typename T>
__device__ __forceinline__ W8 w8_from_bits(const uint4& b) {
    W8 r;
    r.w[0] = Fmt<T>::unpack(b.x);
    r.w[1] = Fmt<T>::unpack(b.y);
    r.w[2] = Fmt<T>::unpack(b.z);
    r.w[3] = Fmt<T>::unpack(b.w);
    return r;
}

__device__ __forceinline__ W8 w8_from_f32(const float4* p) {
    const float4 a = p[0], b = p[1];
    W8 r;
    r.w[0] = make_float2(a.x, a.y);
    r.w[1] = make_float2(a.z, a.w);
    r.w[2] = make_float2(b.x, b.y);
    r.w[3] = make_float2(b.z, b.w);
    return r;
}

// Two lanes of a * b + c in fp32 from packed 16-bit a and b (the mixed-
// precision fma of sm_100, fma.rn.f32.{bf16,f16}: the product of two 16-bit
// values is exact, so the result equals widening both and one fp32 fma).
// The `kMixed` forms below use it in place of widening the 16-bit operands
// and a paired fp32 multiply; measured on B200 it makes rms_norm 3-14 %
// faster, and the fused ops (which hold more values per thread, and spill in
// the fp8 op) 0-6 % slower, so only bf16 rms_norm takes it.
template <typename T>
__device__ __forceinline__ float2 mfma2(uint32_t a, uint32_t b, float2 c);
template <>
__device__ __forceinline__ float2 mfma2<__nv_bfloat16>(uint32_t a, uint32_t b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %2;\n\tmov.b32 {bl, bh}, %3;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %4;\n\tfma.rn.f32.bf16 %1, ah, bh, %5;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "r"(a), "r"(b), "f"(c.x), "f"(c.y));
    return d;
}
template <>
__device__ __forceinline__ float2 mfma2<__half>(uint32_t a, uint32_t b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\tmov.b32 {al, ah}, %2;\n\tmov.b32 {bl, bh}, %3;\n\t"
        "fma.rn.f32.f16 %0, al, bl, %4;\n\tfma.rn.f32.f16 %1, ah, bh, %5;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "r"(a), "r"(b), "f"(c.x), "f"(c.y));
    return d;
}

template <typename T>
__device__ __forceinline__ uint4 add8(const uint4& x, const uint4& r) {
    return make_uint4(Fmt<T>::add2(x.x, r.x), Fmt<T>::add2(x.y, r.y), Fmt<T>::add2(x.z, r.z),
                      Fmt<T>::add2(x.w, r.w));
}

// acc += v * v, pairwise (acc.x collects even elements, acc.y odd ones).
template <typename T, bool kMixed = false>
__device__ __forceinline__ float2 ssq8(const uint4& v, float2 acc) {
    const uint32_t* u = &v.x;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        if constexpr (kMixed) {
            acc = mfma2<T>(u[c], u[c], acc);
        } else {
            const float2 f = Fmt<T>::unpack(u[c]);
            acc = __ffma2_rn(f, f, acc);
        }
    }
    return acc;
}

// Pair c (0..3) of 8 weights, as fp32: from widened fp32 weights (W8) or
// straight from the packed 16-bit weights (uint4), widened pair by pair so
// only 4 registers stay live.
template <typename T>
__device__ __forceinline__ float2 wpair(const W8& w, int c) {
    return w.w[c];
}
template <typename T>
__device__ __forceinline__ float2 wpair(const uint4& w, int c) {
    return Fmt<T>::unpack((&w.x)[c]);
}

// v * w for pair c, exact in fp32 (a product of two 16-bit values): the
// mixed-precision fma from packed 16-bit weights, else widening and a
// paired multiply.
template <typename T, bool kHasW, bool kMixed, typename WT>
__device__ __forceinline__ float2 vw2(uint32_t v, const WT& w, int c) {
    // adding -0 leaves every product as it is (+0 would turn -0 into +0)
    if constexpr (kMixed && kHasW && std::is_same_v<WT, uint4>)
        return mfma2<T>(v, (&w.x)[c], make_float2(-0.f, -0.f));
    float2 p = Fmt<T>::unpack(v);
    if constexpr (kHasW) p = __fmul2_rn(p, wpair<T>(w, c));
    return p;
}

// max(pm, max |v * w|).
template <typename T, bool kHasW, typename WT>
__device__ __forceinline__ float amax8(const uint4& v, const WT& w, float pm) {
    const uint32_t* u = &v.x;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float2 p = vw2<T, kHasW, false>(u[c], w, c);
        pm = fmaxf(pm, fmaxf(fabsf(p.x), fabsf(p.y)));
    }
    return pm;
}

// RNE16((v * w) * inv) for 8 elements.
template <typename T, bool kHasW, bool kMixed = false, typename WT>
__device__ __forceinline__ uint4 scale8(const uint4& v, const WT& w, float2 inv2) {
    const uint32_t* u = &v.x;
    uint4 o;
    uint32_t* os = &o.x;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float2 p = vw2<T, kHasW, kMixed>(u[c], w, c);
        os[c] = Fmt<T>::pack(__fmul2_rn(p, inv2));
    }
    return o;
}

// e4m3(RNE, satfinite)((v * w) * qmul) for 8 elements, 8 bytes.
template <typename T, bool kHasW, typename WT>
__device__ __forceinline__ uint2 quant8(const uint4& v, const WT& w, float2 qmul2) {
    const uint32_t* u = &v.x;
    uint32_t e[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float2 p = __fmul2_rn(vw2<T, kHasW, false>(u[c], w, c), qmul2);
        e[c] = e4m3x2(p.x, p.y);
    }
    return make_uint2(e[0] | (e[1] << 16), e[2] | (e[3] << 16));
}

}  // namespace
}  // namespace rn
