// rn_device.cuh -- device helpers shared by the library's kernel files:
// 16-bit format conversions, global-memory and barrier PTX, the e4m3 cast,
// programmatic-dependent-launch controls, and the host-side launch helper.
// Internal; not part of the C ABI.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <utility>

#include "rn_internal.h"

namespace rn {
namespace {

// ---------------------------------------------------------------- formats
//
// Per 16-bit format: packed residual add (one round-to-nearest-even of the
// exact sum of each pair: the correctly rounded sum, identical to adding in
// fp32 and rounding once), exact widening of a packed pair to fp32, and
// narrowing of an fp32 pair with one round-to-nearest-even.

template <typename T>
struct Fmt;

template <>
struct Fmt<__nv_bfloat16> {
    static __device__ __forceinline__ uint32_t add2(uint32_t a, uint32_t b) {
        uint32_t d;
        asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
        return d;
    }
    static __device__ __forceinline__ float2 unpack(uint32_t u) {
        // bf16 is the upper half of an fp32 word
        return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
    }
    static __device__ __forceinline__ uint32_t pack(float2 f) {
        __nv_bfloat162 h = __floats2bfloat162_rn(f.x, f.y);
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
    static __device__ __forceinline__ uint32_t add2(uint32_t a, uint32_t b) {
        uint32_t d;
        asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
        return d;
    }
    static __device__ __forceinline__ float2 unpack(uint32_t u) {
        __half2 h;
        memcpy(&h, &u, 4);
        return __half22float2(h);
    }
    static __device__ __forceinline__ uint32_t pack(float2 f) {
        __half2 h = __floats2half2_rn(f.x, f.y);
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

// 32-byte (256-bit) global accesses, new with sm_100: two adjacent 16-byte
// vectors in one instruction. The address must be 32-byte aligned.
__device__ __forceinline__ void ld_stream2(const uint4* p, uint4& a, uint4& b) {
    asm volatile("ld.global.L1::no_allocate.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(a.x), "=r"(a.y), "=r"(a.z), "=r"(a.w), "=r"(b.x), "=r"(b.y), "=r"(b.z),
                   "=r"(b.w)
                 : "l"(p));
}

__device__ __forceinline__ void st_v8(uint4* p, const uint4& a, const uint4& b) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(p), "r"(a.x),
                 "r"(a.y), "r"(a.z), "r"(a.w), "r"(b.x), "r"(b.y), "r"(b.z), "r"(b.w)
                 : "memory");
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

// Programmatic dependent launch. Every kernel lets the next kernel in the
// stream begin launching at once (its blocks then wait, below, for this grid
// to finish), and waits for the previous kernel in the stream to complete and
// flush its memory before touching global memory. Without the launch
// attribute both are no-ops, so the kernels are correct either way.
__device__ __forceinline__ void pdl_allow_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_for_prior_grid() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Asks the bulk-copy unit to bring `bytes` (a multiple of 16) from 16-byte
// aligned global address `p` into L2. Nothing reaches the SM and nothing
// waits for it; it is a hint without effect on what later loads return (L2
// is the device's point of coherence, so a line that another kernel writes
// after the prefetch is read back with that write).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}


// Launches `kernel` with the plan's shape, with the PDL attribute when asked.
template <typename... KArgs, typename... Args2>
cudaError_t launch_kernel(void (*kernel)(KArgs...), const Launch& l, cudaStream_t s,
                          Args2&&... args) {
    if (l.pdl) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(l.grid));
        cfg.blockDim = dim3(static_cast<unsigned>(l.block));
        cfg.dynamicSmemBytes = static_cast<size_t>(l.smem);
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args2>(args)...);
    }
    kernel<<<static_cast<unsigned>(l.grid), l.block, l.smem, s>>>(std::forward<Args2>(args)...);
    return cudaGetLastError();
}


}  // namespace
}  // namespace rn
