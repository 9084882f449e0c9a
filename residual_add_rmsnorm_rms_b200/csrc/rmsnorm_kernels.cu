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
//    read-only path and stays cached (it is shared by every row). With an
//    even VPT and 32-byte aligned rows (kPair), a thread's vectors come in
//    adjacent pairs moved by sm_100's 32-byte loads and stores: half the
//    memory instructions for the same bytes (the fp8 op on [8192 x 3840]
//    went from 36.6 to 34.6 us on B200, fused_add_rms_norm at four vectors
//    per thread from 40.2 to 39.1 us).
//  * reductions: xor butterfly inside the warp (every lane ends with the same
//    total), then, for rows wider than a warp, one named barrier per row
//    group and a fixed-order sum over the group's warps from shared memory.
//    The order is fixed, so results are bit-reproducible run to run.
//  * staged kernel: persistent; whole rows streamed into a shared-memory ring
//    by bulk asynchronous copies (see its section).
//  * scalar kernel: one CTA per row, two passes (the second re-reads the row,
//    mostly from L2); any H and any element-aligned pointers. It exists for
//    correctness on inputs the vector kernel cannot take.
//
// Numerics (all kernels): the residual sum is the correctly rounded 16-bit
// sum (packed add.rn in the fast kernels; fp32 add then one rounding in the
// scalar kernel, which is the same value because fp32 holds >= 2p+2 bits of
// either 16-bit format); squares accumulated in fp32; inv = 1 / sqrt(ss / H +
// eps) with IEEE sqrt and division; y = (v * w) * inv, where v * w is exact in
// fp32; fp8: P = max |v * w| (exact), q = e4m3(RNE, satfinite)((v * w) *
// (448 / P)), scale = (P * inv) / 448, which equals max |y| / 448 because
// rounding is monotonic.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>
#include <type_traits>
#include <utility>

#include "rn_device.cuh"
#include "rn_internal.h"
#include "rn_vec8.cuh"

namespace rn {
namespace {

// ---------------------------------------------------------------- vector kernel

// Index (in 16-byte vectors within the row) of a thread's vector k: strided
// by tpr so that a warp's accesses are contiguous, or with kPair, pair k / 2
// strided by tpr and the two vectors of a pair adjacent.
template <bool kPair>
__device__ __forceinline__ int vec_index(int lr, int k, int tpr) {
    if constexpr (kPair) return 2 * (lr + (k >> 1) * tpr) + (k & 1);
    return lr + k * tpr;
}

template <typename T, int VPT, int OP, bool kHasW, bool kPair>
__device__ __forceinline__ void vector_rows(const Args& a, const int tpr, const int rpc,
                                            float2* red) {
    static_assert(!kPair || VPT % 2 == 0, "pairs need an even vector count");
    constexpr bool kFused = OP != kRmsNorm;
    constexpr bool kFp8 = OP == kFusedAddFp8;
    // bf16 rms_norm at four or more vectors per thread widens nothing:
    // squares and products straight from the 16-bit values with the
    // mixed-precision fma (rn_vec8.cuh; 3-14 % faster on T >= 4096). fp16
    // keeps widening: with the mixed fma, rms_norm no longer reproduced the
    // fused op's output bit for bit on fp16 rows, so its exactness there is
    // not established. The one- and two-vector shapes of decode-sized rows
    // keep widening too (two vectors per thread: up to 27 % slower with it).
    constexpr bool kMixed = OP == kRmsNorm && std::is_same_v<T, __nv_bfloat16> && VPT >= 4;

    const int row_in_cta = threadIdx.x / tpr;
    const int lr = threadIdx.x - row_in_cta * tpr;
    const int wpr = tpr >> 5;
    const int nvec = static_cast<int>(a.H >> 3);
    const float hf = static_cast<float>(a.H);
    const uint4* __restrict__ wv = static_cast<const uint4*>(a.weight);
    int parity = 0;

    // The loop bound depends only on the block, so every thread of a warp
    // runs the same iterations (the shuffles below use the full mask).
    for (int64_t base = static_cast<int64_t>(blockIdx.x) * rpc; base < a.T;
         base += static_cast<int64_t>(gridDim.x) * rpc) {
        const int64_t row = base + row_in_cta;
        const bool active = row < a.T;
        const int64_t roff = (active ? row : 0) * nvec;
        const uint4* xrow = static_cast<const uint4*>(a.x) + roff;
        uint4* rrow = static_cast<uint4*>(a.residual) + roff;

        // With kPair the row has an even number of vectors (nvec), so a pair
        // is either wholly inside the row or wholly outside.
        constexpr int kStep = kPair ? 2 : 1;
        const uint4 z4 = make_uint4(0, 0, 0, 0);
        uint4 v[VPT];
#pragma unroll
        for (int k = 0; k < VPT; k += kStep) {
            const int j = vec_index<kPair>(lr, k, tpr);
            const bool ok = active && j < nvec;
            if constexpr (kPair) {
                if (ok) ld_stream2(xrow + j, v[k], v[k + 1]);
                else v[k] = v[k + 1] = z4;
            } else {
                v[k] = ok ? ld_stream(xrow + j) : z4;
            }
        }
        if constexpr (kFused) {
            uint4 r[VPT];
#pragma unroll
            for (int k = 0; k < VPT; k += kStep) {
                const int j = vec_index<kPair>(lr, k, tpr);
                const bool ok = active && j < nvec;
                if constexpr (kPair) {
                    if (ok) ld_stream2(rrow + j, r[k], r[k + 1]);
                    else r[k] = r[k + 1] = z4;
                } else {
                    r[k] = ok ? ld_stream(rrow + j) : z4;
                }
            }
#pragma unroll
            for (int k = 0; k < VPT; k += kStep) {
                const int j = vec_index<kPair>(lr, k, tpr);
                v[k] = add8<T>(v[k], r[k]);
                if constexpr (kPair) {
                    v[k + 1] = add8<T>(v[k + 1], r[k + 1]);
                    if (active && j < nvec) st_v8(rrow + j, v[k], v[k + 1]);
                } else {
                    if (active && j < nvec) st_v4(rrow + j, v[k]);
                }
            }
        }

        float2 acc = make_float2(0.f, 0.f);
        float pm = 0.f;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            acc = ssq8<T, kMixed>(v[k], acc);
            if constexpr (kFp8) {
                const int j = vec_index<kPair>(lr, k, tpr);
                uint4 w = make_uint4(0, 0, 0, 0);
                if constexpr (kHasW) {
                    if (j < nvec) w = __ldg(wv + j);
                }
                pm = amax8<T, kHasW>(v[k], w, pm);
            }
        }
        float ss = acc.x + acc.y;

        const int width = tpr < 32 ? tpr : 32;
        for (int o = width >> 1; o > 0; o >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if constexpr (kFp8) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, o));
        }
        if (wpr > 1) {
            float2* slot = red + (parity * rpc + row_in_cta) * wpr;
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
            uint4* orow = static_cast<uint4*>(a.out) + roff;
            const float2 inv2 = make_float2(inv, inv);
#pragma unroll
            for (int k = 0; k < VPT; k += kStep) {
                const int j = vec_index<kPair>(lr, k, tpr);
                if (!(active && j < nvec)) continue;
                uint4 w = make_uint4(0, 0, 0, 0);
                if constexpr (kHasW) w = __ldg(wv + j);
                if constexpr (kPair) {
                    uint4 w1 = make_uint4(0, 0, 0, 0);
                    if constexpr (kHasW) w1 = __ldg(wv + j + 1);
                    st_v8(orow + j, scale8<T, kHasW, kMixed>(v[k], w, inv2),
                          scale8<T, kHasW, kMixed>(v[k + 1], w1, inv2));
                } else {
                    st_v4(orow + j, scale8<T, kHasW, kMixed>(v[k], w, inv2));
                }
            }
        } else {
            const float qmul = pm > 0.f ? 448.0f / pm : 0.f;
            const float2 q2 = make_float2(qmul, qmul);
            if (active && lr == 0) a.scale[row] = pm > 0.f ? (pm * inv) / 448.0f : 0.f;
            uint2* qrow = reinterpret_cast<uint2*>(a.q) + roff;
#pragma unroll
            for (int k = 0; k < VPT; k += kStep) {
                const int j = vec_index<kPair>(lr, k, tpr);
                if (!(active && j < nvec)) continue;
                // (both codes computed before the zero-row test: the other
                // order put a 16-byte temporary in local memory)
                if constexpr (kPair) {
                    uint4 w0 = make_uint4(0, 0, 0, 0), w1 = w0;
                    if constexpr (kHasW) {
                        w0 = __ldg(wv + j);
                        w1 = __ldg(wv + j + 1);
                    }
                    uint2 o0 = quant8<T, kHasW>(v[k], w0, q2);
                    uint2 o1 = quant8<T, kHasW>(v[k + 1], w1, q2);
                    if (!(pm > 0.f)) o0 = o1 = make_uint2(0, 0);
                    st_v4(reinterpret_cast<uint4*>(qrow + j), make_uint4(o0.x, o0.y, o1.x, o1.y));
                } else {
                    uint4 w = make_uint4(0, 0, 0, 0);
                    if constexpr (kHasW) w = __ldg(wv + j);
                    uint2 o = quant8<T, kHasW>(v[k], w, q2);
                    if (!(pm > 0.f)) o = make_uint2(0, 0);
                    st_v2(qrow + j, o);
                }
            }
        }
    }
}

// Bytes of a row one L2 prefetch covers.
constexpr uint32_t kPrefetchChunk = 4096;

// L2 prefetch of the rows of the block's first row group (x, and the
// residual for the fused ops), spread over the row group's threads in
// 4 KB pieces. Rows are 16-byte aligned and 2H is a multiple of 16 here.
template <int OP>
__device__ __forceinline__ void prefetch_first_rows(const Args& a, const int tpr, const int rpc) {
    const int row_in_cta = threadIdx.x / tpr;
    const int lr = threadIdx.x - row_in_cta * tpr;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * rpc + row_in_cta;
    if (row >= a.T) return;
    const uint32_t row_bytes = static_cast<uint32_t>(a.H) * 2u;
    const char* xr = static_cast<const char*>(a.x) + row * row_bytes;
    const char* rr = static_cast<const char*>(a.residual) + row * row_bytes;
    for (uint32_t off = static_cast<uint32_t>(lr) * kPrefetchChunk; off < row_bytes;
         off += static_cast<uint32_t>(tpr) * kPrefetchChunk) {
        const uint32_t n = row_bytes - off < kPrefetchChunk ? row_bytes - off : kPrefetchChunk;
        prefetch_l2(xr + off, n);
        if constexpr (OP != kRmsNorm) prefetch_l2(rr + off, n);
    }
}

// `prefetch` (set only under programmatic dependent launch): before waiting
// for the previous kernel in the stream, the block asks L2 for its first
// rows. Blocks become resident while the previous kernel drains, so HBM
// keeps streaming across the kernel boundary instead of idling for one load
// latency, and the first loads after the wait hit L2.
template <typename T, int VPT, int OP, bool kPair>
__global__ void __launch_bounds__(max_block_for_vpt(VPT))
    rn_vector_kernel(const Args a, const int tpr, const int rpc, const int prefetch) {
    extern __shared__ float2 red[];  // [2][rpc][warps per row]
    pdl_allow_dependents();
    if (prefetch) prefetch_first_rows<OP>(a, tpr, rpc);
    pdl_wait_for_prior_grid();
    if (a.weight)
        vector_rows<T, VPT, OP, true, kPair>(a, tpr, rpc, red);
    else
        vector_rows<T, VPT, OP, false, kPair>(a, tpr, rpc, red);
}

// ---------------------------------------------------------------- staged kernel
//
// Persistent, row -> CTA. Thread 0 streams whole rows of x (and the residual)
// into a ring of `stages` shared-memory slots with one bulk asynchronous copy
// per row and tensor (cp.async.bulk, completion counted on an mbarrier), up
// to `stages` rows ahead, so the bytes in flight per SM are set by shared
// memory rather than by registers. The weight is widened to fp32 into shared
// memory once per CTA. All threads then make two passes over the staged row:
// (1) residual add, write-back (global, and over the x slot in shared memory),
// sum of squares [and max |v * w|]; (2) the output. CTA b owns rows
// b, b + gridDim.x, ... Every mbarrier wait is bounded; on a timeout the CTA
// records kErrWaitTimeout in g_rn_device_error, waits (bounded) for the copies
// it issued, and returns.

__device__ unsigned int g_rn_device_error = 0;

constexpr unsigned kErrWaitTimeout = 1u;
constexpr long long kWaitLimitCycles = 4000000000LL;  // ~2 s at 1.9 GHz

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for phase `parity` of an mbarrier; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitLimitCycles) return false;
    }
    return true;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both ends 16-byte
// aligned), completing on mbarrier `bar`; L2 evict-first (read once).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(dst),
        "l"(src), "r"(bytes), "r"(bar), "l"(policy)
        : "memory");
}

__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

template <typename T, int OP, bool kHasW>
__device__ __forceinline__ void staged_rows(const Args& a, const int stages,
                                            const uint32_t slot_bytes, unsigned char* smem) {
    constexpr bool kFused = OP != kRmsNorm;
    constexpr bool kFp8 = OP == kFusedAddFp8;
    constexpr int kSlots = kFused ? 2 : 1;  // x [, residual] per stage

    const int tid = threadIdx.x;
    const int nthr = blockDim.x;
    const int nwarps = nthr >> 5;
    const int nvec = static_cast<int>(a.H >> 3);
    const uint32_t row_bytes = static_cast<uint32_t>(a.H) * 2u;
    const uint32_t stage_bytes = kSlots * slot_bytes;
    const int64_t G = gridDim.x;
    const int64_t first = blockIdx.x;
    const int64_t nrows = first < a.T ? (a.T - 1 - first) / G + 1 : 0;
    // layout: [stages x stage][fp32 weight, 4H bytes][mbarriers][reduction]
    float4* wf = reinterpret_cast<float4*>(smem + static_cast<size_t>(stages) * stage_bytes);
    uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<unsigned char*>(wf) +
                                                 static_cast<size_t>(a.H) * 4);
    float2* red = reinterpret_cast<float2*>(bars + stages);
    const float hf = static_cast<float>(a.H);
    const char* xg = static_cast<const char*>(a.x);
    char* rg = static_cast<char*>(a.residual);

    uint64_t policy = 0;
    if (tid == 0) {
        policy = policy_evict_first();
        for (int s = 0; s < stages; ++s) mbar_init(smem_u32(bars + s), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    auto issue = [&](int s, int64_t row) {
        const uint32_t bar = smem_u32(bars + s);
        const uint32_t dst = smem_u32(smem + static_cast<size_t>(s) * stage_bytes);
        mbar_arrive_expect_tx(bar, kSlots * row_bytes);
        bulk_load(dst, xg + row * row_bytes, row_bytes, bar, policy);
        if constexpr (kFused) bulk_load(dst + slot_bytes, rg + row * row_bytes, row_bytes, bar, policy);
    };
    if constexpr (kHasW) {
        const uint4* wv = static_cast<const uint4*>(a.weight);
        for (int j = tid; j < nvec; j += nthr) {
            const W8 w = w8_from_bits<T>(__ldg(wv + j));
            wf[2 * j] = make_float4(w.w[0].x, w.w[0].y, w.w[1].x, w.w[1].y);
            wf[2 * j + 1] = make_float4(w.w[2].x, w.w[2].y, w.w[3].x, w.w[3].y);
        }
    }
    __syncthreads();
    if (tid == 0) {
        for (int s = 0; s < stages && s < nrows; ++s) issue(s, first + s * G);
    }

    int64_t k = 0;
    for (; k < nrows; ++k) {
        const int s = static_cast<int>(k % stages);
        const uint32_t parity = static_cast<uint32_t>((k / stages) & 1);
        const int64_t row = first + k * G;
        const bool ok = mbar_wait(smem_u32(bars + s), parity);
        uint4* sx = reinterpret_cast<uint4*>(smem + static_cast<size_t>(s) * stage_bytes);
        const uint4* sr = reinterpret_cast<const uint4*>(reinterpret_cast<unsigned char*>(sx) + slot_bytes);

        // pass 1: [residual add + write-back], sum of squares [, max |v * w|]
        float2 acc = make_float2(0.f, 0.f);
        float pm = 0.f;
        if (ok) {
            uint4* rrow = reinterpret_cast<uint4*>(rg + row * row_bytes);
            for (int j = tid; j < nvec; j += nthr) {
                uint4 v = sx[j];
                if constexpr (kFused) {
                    v = add8<T>(v, sr[j]);
                    st_v4(rrow + j, v);
                    sx[j] = v;
                }
                acc = ssq8<T>(v, acc);
                if constexpr (kFp8) {
                    W8 w{};
                    if constexpr (kHasW) w = w8_from_f32(wf + 2 * j);
                    pm = amax8<T, kHasW>(v, w, pm);
                }
            }
        }
        float ss = acc.x + acc.y;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if constexpr (kFp8) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, o));
        }
        if ((tid & 31) == 0) red[tid >> 5] = make_float2(ss, pm);
        // Barrier A: publishes `red` and makes a timeout uniform across the CTA.
        if (__syncthreads_or(!ok)) {
            if (tid == 0) atomicOr(&g_rn_device_error, kErrWaitTimeout);
            break;
        }
        ss = 0.f;
        pm = 0.f;
        for (int i = 0; i < nwarps; ++i) {
            const float2 t = red[i];
            ss += t.x;
            pm = fmaxf(pm, t.y);
        }
        const float inv = 1.0f / sqrtf(ss / hf + a.eps);

        // pass 2: outputs from the staged (written-back) row
        if constexpr (!kFp8) {
            uint4* og = reinterpret_cast<uint4*>(static_cast<char*>(a.out) + row * row_bytes);
            const float2 inv2 = make_float2(inv, inv);
            for (int j = tid; j < nvec; j += nthr) {
                W8 w{};
                if constexpr (kHasW) w = w8_from_f32(wf + 2 * j);
                st_v4(og + j, scale8<T, kHasW>(sx[j], w, inv2));
            }
        } else {
            const float qmul = pm > 0.f ? 448.0f / pm : 0.f;
            const float2 q2 = make_float2(qmul, qmul);
            if (tid == 0) a.scale[row] = pm > 0.f ? (pm * inv) / 448.0f : 0.f;
            uint2* qg = reinterpret_cast<uint2*>(a.q + row * a.H);
            for (int j = tid; j < nvec; j += nthr) {
                W8 w{};
                if constexpr (kHasW) w = w8_from_f32(wf + 2 * j);
                uint2 o = quant8<T, kHasW>(sx[j], w, q2);
                if (!(pm > 0.f)) o = make_uint2(0, 0);
                st_v2(qg + j, o);
            }
        }
        // Barrier B: every thread is done with stage s (and with `red`).
        __syncthreads();
        if (tid == 0 && k + stages < nrows) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(s, first + (k + stages) * G);
        }
    }
    if (k < nrows && tid == 0) {
        // Timed out: wait (bounded) for the copies still in flight, then leave.
        const int64_t last = (k + stages < nrows ? k + stages : nrows);
        for (int64_t kk = k; kk < last; ++kk) {
            mbar_wait(smem_u32(bars + (kk % stages)), static_cast<uint32_t>((kk / stages) & 1));
        }
    }
}

template <typename T, int OP>
__global__ void __launch_bounds__(1024)
    rn_staged_kernel(const Args a, const int stages, const uint32_t slot_bytes) {
    extern __shared__ __align__(128) unsigned char smem[];
    pdl_allow_dependents();
    pdl_wait_for_prior_grid();
    if (a.weight)
        staged_rows<T, OP, true>(a, stages, slot_bytes, smem);
    else
        staged_rows<T, OP, false>(a, stages, slot_bytes, smem);
}

// ---------------------------------------------------------------- scalar kernel

constexpr int kScalarBlock = 256;

template <typename T, int OP>
__global__ void __launch_bounds__(kScalarBlock) rn_scalar_kernel(const Args a) {
    using F = Fmt<T>;
    constexpr bool kFused = OP != kRmsNorm;
    constexpr bool kFp8 = OP == kFusedAddFp8;
    __shared__ float2 red[kScalarBlock / 32];
    pdl_allow_dependents();
    pdl_wait_for_prior_grid();
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
    const int pf = l.prefetch && l.pdl ? 1 : 0;
    if constexpr (VPT % 2 == 0) {
        if (l.pair)
            return launch_kernel(rn_vector_kernel<T, VPT, OP, true>, l, s, a, l.tpr, l.rpc, pf);
    }
    return launch_kernel(rn_vector_kernel<T, VPT, OP, false>, l, s, a, l.tpr, l.rpc, pf);
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

// Opt each staged-kernel instantiation into large dynamic shared memory once
// per device (the attribute is per function and per device context).
template <typename T, int OP>
cudaError_t prepare_staged(int smem) {
    static unsigned long long done_mask = 0;  // bit d: device d configured
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? (1ull << dev) : 0;
    if (bit && (__atomic_load_n(&done_mask, __ATOMIC_ACQUIRE) & bit)) return cudaSuccess;
    (void)smem;
    e = cudaFuncSetAttribute(rn_staged_kernel<T, OP>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kStagedMaxSmem);
    if (e == cudaSuccess && bit) __atomic_fetch_or(&done_mask, bit, __ATOMIC_ACQ_REL);
    return e;
}

template <typename T, int OP>
cudaError_t launch_typed(const Args& a, const Launch& l, cudaStream_t s) {
    if (l.kernel == 0) return dispatch_vpt<T, OP>(a, l, s);
    if (l.kernel == 2) {
        cudaError_t e = prepare_staged<T, OP>(l.smem);
        if (e != cudaSuccess) return e;
        const uint32_t slot = static_cast<uint32_t>(((a.H * 2 + 127) / 128) * 128);
        return launch_kernel(rn_staged_kernel<T, OP>, l, s, a, l.vpt, slot);
    }
    Launch ls = l;
    ls.block = kScalarBlock;
    ls.smem = 0;
    return launch_kernel(rn_scalar_kernel<T, OP>, ls, s, a);
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

cudaError_t read_and_clear_device_errors(unsigned* flags) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_rn_device_error, sizeof v);
    if (e != cudaSuccess) return e;
    *flags = v;
    if (v) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_rn_device_error, &zero, sizeof zero);
    }
    return e;
}

cudaError_t kernel_binary_version(int* version) {
    cudaFuncAttributes attr;
    const cudaError_t e = cudaFuncGetAttributes(&attr, rn_scalar_kernel<__nv_bfloat16, kRmsNorm>);
    if (e == cudaSuccess) *version = attr.binaryVersion;
    return e;
}

cudaError_t launch(int op, int dtype, const Args& a, const Launch& l, cudaStream_t s) {
    if (dtype == kBF16) return launch_op<__nv_bfloat16>(op, a, l, s);
    if (dtype == kF16) return launch_op<__half>(op, a, l, s);
    return cudaErrorInvalidValue;
}

}  // namespace rn
