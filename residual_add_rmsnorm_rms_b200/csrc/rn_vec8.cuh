// rn_vec8.cuh -- arithmetic on 8 16-bit elements held in one 16-byte vector
// (uint4: 4 packed pairs), shared by the norm kernels and the all-reduce
// fused kernels so that both round identically. Internal.
#pragma once

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

template <typename T>
__device__ __forceinline__ uint4 add8(const uint4& x, const uint4& r) {
    return make_uint4(Fmt<T>::add2(x.x, r.x), Fmt<T>::add2(x.y, r.y), Fmt<T>::add2(x.z, r.z),
                      Fmt<T>::add2(x.w, r.w));
}

// acc += v * v, pairwise (acc.x collects even elements, acc.y odd ones).
template <typename T>
__device__ __forceinline__ float2 ssq8(const uint4& v, float2 acc) {
    const uint32_t* u = &v.x;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const float2 f = Fmt<T>::unpack(u[c]);
        acc = __ffma2_rn(f, f, acc);
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

// max(pm, max |v * w|): v * w is exact in fp32 (a product of two 16-bit values).
template <typename T, bool kHasW, typename WT>
__device__ __forceinline__ float amax8(const uint4& v, const WT& w, float pm) {
    const uint32_t* u = &v.x;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float2 p = Fmt<T>::unpack(u[c]);
        if constexpr (kHasW) p = __fmul2_rn(p, wpair<T>(w, c));
        pm = fmaxf(pm, fmaxf(fabsf(p.x), fabsf(p.y)));
    }
    return pm;
}

// RNE16((v * w) * inv) for 8 elements.
template <typename T, bool kHasW, typename WT>
__device__ __forceinline__ uint4 scale8(const uint4& v, const WT& w, float2 inv2) {
    const uint32_t* u = &v.x;
    uint4 o;
    uint32_t* os = &o.x;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        float2 p = Fmt<T>::unpack(u[c]);
        if constexpr (kHasW) p = __fmul2_rn(p, wpair<T>(w, c));
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
        float2 p = Fmt<T>::unpack(u[c]);
        if constexpr (kHasW) p = __fmul2_rn(p, wpair<T>(w, c));
        p = __fmul2_rn(p, qmul2);
        e[c] = e4m3x2(p.x, p.y);
    }
    return make_uint2(e[0] | (e[1] << 16), e[2] | (e[3] << 16));
}

}  // namespace
}  // namespace rn
