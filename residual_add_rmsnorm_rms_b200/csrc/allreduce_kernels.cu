// allreduce_kernels.cu -- tensor-parallel all-reduce fused with the residual
// add and RMSNorm (+ per-token FP8 cast), one kernel per call.
//
// In a tensor-parallel decoder layer every rank ends its row-parallel linear
// layer with a partial sum of the activations; an all-reduce adds the W
// partials and the residual add + RMSNorm follows (SGLang takes all-reduce and
// RMSNorm from AITER: "AITER: AMD's operator library for ROCm", ecosystem
// section). Here each rank computes, for every row,
//   x = RNE16(sum over ranks of the partials),  residual := RNE16(x + residual),
//   out = RNE16(rms_norm(residual) * w)   or   (q, scale) as fused_add_rms_norm_fp8,
// identically on every rank (the residual is replicated across the group).
//
// One-shot exchange over peer memory (NVLink / NVSwitch loads; no collective
// library, no multicast): every rank owns an exchange buffer and a signal pad
// that all ranks can address. The pad starts with this rank's call counter
// (the epoch of its last call) and an arrival counter, then the flags. Block
// b of every rank owns the same rows; in call e (= counter + 1, 0 skipped):
//  1. it copies its rows of the local partial into its own buffer (the half
//     selected by e's parity),
//  2. publishes them: e is stored with system-scope release semantics into
//     flag [e & 1][b][rank] of every rank's pad,
//  3. waits (bounded by timeout_ns on the global timer) until flag
//     [e & 1][b][p] of its own pad equals e, for every rank p,
//  4. reads the rows from all W buffers (volatile 16-byte loads: never a stale
//     L1 line), sums them in rank order 0..W-1 and finishes the row exactly
//     as fused_add_rms_norm(_fp8) does (same 8-element arithmetic),
//  5. counts itself in the arrival counter; the last block of the rank to
//     arrive resets it and stores e as the call counter for the next launch.
// The counter lives on the device, so a captured CUDA graph replays correctly
// (each replayed launch takes the next epoch). A rank overwrites a buffer
// half, or a flag, only two calls after it last wrote it: by then every peer
// has finished reading the half and has seen the flag, because a peer
// publishes call e+1 only after its call e kernel completed (stream order)
// and each rank waits for all peers' call e+1 flags before starting call e+2.
// So the flags are compared for equality and never need resetting. Every
// call launches, even with no rows (one block then only publishes and waits),
// so all ranks' counters advance together for any sequence of row counts.
// The grid is the same on every rank and no larger than what the device
// holds resident, and blocks are dispatched in index order, so the blocks
// resident on every rank always include the lowest-numbered blocks still
// waiting, which can therefore finish: no block waits on a block that cannot
// run (the bounded wait guards the rest). Several ranks may be driven by one
// launch (blockIdx.y = rank - first rank, operands stacked by rank), which
// runs a whole group on one device; blocks of one launch then wait on one
// another, so that launch is cooperative (every block resident).
//
// With two ranks the sum is one packed 16-bit add (correctly rounded, as the
// residual add). With more, it is accumulated in binary64 in rank order,
// converted to binary32 by rounding to odd (toward zero, then the last bit
// set if anything was dropped) and rounded once to the 16-bit format. Rounding to odd with at
// least two more bits than the target makes the second rounding correct
// (Boldo and Melquiond, "When double rounding is odd", 2005), so x is the
// correctly rounded sum whenever the binary64 sum is exact: always for fp16
// partials (every fp16 value is an integer multiple of 2^-24 below 2^16), and
// for bf16 partials whose non-zero values span at most 42 binades (W <= 8
// values then fit 53 bits). Every rank computes bit-identical results.
//
// A wait that runs out sets bit 1 of the device error flags and leaves that
// block's rows unwritten (the other blocks are unaffected); the block still
// counts its arrival, so the rank's call counter advances.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <cstdint>

#include "rn_device.cuh"
#include "rn_internal.h"
#include "rn_allreduce.h"
#include "rn_vec8.cuh"

namespace rn {
namespace {

__device__ unsigned int g_rn_ar_error = 0;
constexpr unsigned kErrPeerTimeout = 2u;

// Signal pad layout, in 32-bit words: the call counter, the arrival counter,
// padding to 64 bytes, then flags [2 parities][2 stages][kArMaxBlocks][kArMaxWorld].
constexpr int kPadEpoch = 0;
constexpr int kPadArrived = 1;
constexpr int kPadFlags = 16;
static_assert((kPadFlags + 4 * kArMaxBlocks * kArMaxWorld) * 4 == kArSignalBytes,
              "signal pad size");

__device__ __forceinline__ uint4 ld_volatile_v4(const uint4* p) {
    uint4 v;
    asm volatile("ld.volatile.global.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint2 ld_volatile_v2(const uint2* p) {
    uint2 v;
    asm volatile("ld.volatile.global.v2.u32 {%0, %1}, [%2];"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p)
                 : "memory");
    return v;
}

__device__ __forceinline__ uint4 ld_copy(const uint4* p, bool exchange) {
    return exchange ? ld_volatile_v4(p) : ld_stream(p);
}
__device__ __forceinline__ uint2 ld_copy(const uint2* p, bool) { return ld_volatile_v2(p); }
__device__ __forceinline__ void st_copy(uint4* p, const uint4& v) { st_v4(p, v); }
__device__ __forceinline__ void st_copy(uint2* p, const uint2& v) { st_v2(p, v); }

// Copies the rows [s0, s1) this block owns (row groups of rpc rows,
// block-strided: the mapping of the reduce step) from src to dst, as `nvec`
// vectors per row (16 bytes for 16-bit rows, 8 for e4m3 rows). Thread
// (row, lr) moves vectors lr, lr + tpr, ... of its row, U row groups at a
// time, all loads before any store, so a thread keeps U * VPT loads (at
// least 64 bytes) in flight. `exchange` selects volatile loads (memory other ranks write).
template <int VPT, typename V>
__device__ __forceinline__ void copy_rows(V* dst, const V* src, const int64_t s0,
                                          const int64_t s1, const int tpr, const int rpc,
                                          const int nvec, const bool exchange) {
    // at least 64 bytes of loads in flight per thread, 16- or 8-byte vectors
    constexpr int U = (VPT >= 4 ? 1 : 4 / VPT) * (sizeof(V) == 8 ? 2 : 1);
    const int row_in_cta = threadIdx.x / tpr;
    const int lr = threadIdx.x - row_in_cta * tpr;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * rpc;
    for (int64_t base = s0 + static_cast<int64_t>(blockIdx.x) * rpc; base < s1;
         base += U * stride) {
        V v[U][VPT];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = base + u * stride + row_in_cta;
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                const int j = lr + k * tpr;
                if (row < s1 && j < nvec) v[u][k] = ld_copy(src + row * nvec + j, exchange);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = base + u * stride + row_in_cta;
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                const int j = lr + k * tpr;
                if (row < s1 && j < nvec) st_copy(dst + row * nvec + j, v[u][k]);
            }
        }
    }
}

__device__ __forceinline__ void st_release_sys(uint32_t* p, uint32_t v) {
    asm volatile("st.release.sys.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint32_t ld_acquire_sys(const uint32_t* p) {
    uint32_t v;
    asm volatile("ld.acquire.sys.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long global_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Rounds to odd at binary32 precision: toward zero, then the last significand
// bit set when the conversion dropped anything. NaN stays NaN; a finite value
// beyond the binary32 range becomes the largest finite binary32 with its last
// bit set, which every 16-bit format then rounds to infinity.
__device__ __forceinline__ float round_to_odd_f32(double s) {
    float f = __double2float_rz(s);
    if (static_cast<double>(f) != s) f = __uint_as_float(__float_as_uint(f) | 1u);
    return f;
}

// RNE16 of the sum over the ranks of 8 elements: kW is the group size
// rounded up to 1, 2, 4 or 8 (W of them present). One rank: the value itself.
// Two ranks: the packed 16-bit add, which rounds the exact sum once (as the
// residual add does). More: the rank-order binary64 sum, rounded to odd at
// binary32, then to nearest even at 16 bits.
template <typename T, int kW>
__device__ __forceinline__ uint4 sum8(const uint4 (&pv)[kW], int W) {
    if constexpr (kW == 1) {
        return pv[0];
    } else if constexpr (kW == 2) {
        return add8<T>(pv[0], pv[1]);
    } else {
        uint4 o;
        uint32_t* os = &o.x;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float2 f0 = Fmt<T>::unpack((&pv[0].x)[c]);
            double sx = f0.x, sy = f0.y;  // start from rank 0: keeps -0 + -0 = -0
#pragma unroll
            for (int p = 1; p < kW; ++p) {
                if (p < W) {
                    const float2 f = Fmt<T>::unpack((&pv[p].x)[c]);
                    sx += static_cast<double>(f.x);
                    sy += static_cast<double>(f.y);
                }
            }
            os[c] = Fmt<T>::pack(make_float2(round_to_odd_f32(sx), round_to_odd_f32(sy)));
        }
        return o;
    }
}

// Byte offsets inside one buffer half (T x H 16-bit values per region): the
// partial (both algorithms), then, for the two-shot algorithm, the finished
// residual rows and the finished output rows (16-bit out, or e4m3 codes
// followed by the T fp32 scales).
struct SlotLayout {
    int64_t partial, residual2, out2, scale2;
    __device__ explicit SlotLayout(const ArArgs& a) {
        const int64_t th2 = a.T * a.H * 2;
        partial = 0;
        residual2 = th2;
        out2 = 2 * th2;
        scale2 = 2 * th2 + a.T * a.H;
    }
};

__device__ __forceinline__ char* slot_base(const ArArgs& a, int p, uint32_t epoch) {
    return static_cast<char*>(a.buffers[p]) + static_cast<int64_t>(epoch & 1u) * a.slot_elems * 2;
}

// Step 4 for the rows [s0, s1) this block owns in that range (row groups of
// rpc rows, block-strided, as in the vector kernel): reduce + residual add +
// RMSNorm (+ FP8) into this rank's outputs; with kStage2 (two-shot) the
// finished rows are also written to this rank's buffer for the other ranks.
template <typename T, int VPT, int kW, bool kFp8, bool kHasW, bool kStage2>
__device__ __forceinline__ void reduce_rows(const ArArgs& a, const int tpr, const int rpc,
                                            float2* red, const int ly, const int rank,
                                            const uint32_t epoch, const int nvec,
                                            const int64_t local, const int64_t s0,
                                            const int64_t s1) {
    const int W = a.world;
    const SlotLayout lay(a);
    const int64_t slot = static_cast<int64_t>(epoch & 1u) * (a.slot_elems >> 3);
    const uint4* __restrict__ wv = static_cast<const uint4*>(a.weight);
    const float hf = static_cast<float>(a.H);
    const uint4* peer[kW];
#pragma unroll
    for (int p = 0; p < kW; ++p)
        peer[p] = static_cast<const uint4*>(a.buffers[p < W ? p : 0]) + slot;  // partials at 0
    const int row_in_cta = threadIdx.x / tpr;
    const int lr = threadIdx.x - row_in_cta * tpr;
    const int wpr = tpr >> 5;
    char* const mine = slot_base(a, rank, epoch);
    int parity = 0;
    for (int64_t base = s0 + static_cast<int64_t>(blockIdx.x) * rpc; base < s1;
         base += static_cast<int64_t>(gridDim.x) * rpc) {
        const int64_t row = base + row_in_cta;
        const bool active = row < s1;
        const int64_t roff = (active ? row : 0) * nvec;
        uint4* rrow = static_cast<uint4*>(a.residual) + local + roff;

        uint4 r[VPT];  // residual (and weight) loads first: in flight during the exchange reads
        uint4 wk[VPT];
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int j = lr + k * tpr;
            r[k] = (active && j < nvec) ? ld_stream(rrow + j) : make_uint4(0, 0, 0, 0);
            wk[k] = make_uint4(0, 0, 0, 0);
            if constexpr (kHasW) {
                if (j < nvec) wk[k] = __ldg(wv + j);
            }
        }
        uint4 v[VPT];
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int j = lr + k * tpr;
            if (active && j < nvec) {
                uint4 pv[kW];
#pragma unroll
                for (int p = 0; p < kW; ++p)
                    pv[p] = p < W ? ld_volatile_v4(peer[p] + roff + j) : make_uint4(0, 0, 0, 0);
                v[k] = sum8<T, kW>(pv, W);
            } else {
                v[k] = make_uint4(0, 0, 0, 0);
            }
        }
        float2 acc = make_float2(0.f, 0.f);
        float pm = 0.f;
#pragma unroll
        for (int k = 0; k < VPT; ++k) {
            const int j = lr + k * tpr;
            v[k] = add8<T>(v[k], r[k]);
            if (active && j < nvec) {
                st_v4(rrow + j, v[k]);
                if constexpr (kStage2)
                    st_v4(reinterpret_cast<uint4*>(mine + lay.residual2) + roff + j, v[k]);
            }
            acc = ssq8<T>(v[k], acc);
            if constexpr (kFp8) pm = amax8<T, kHasW>(v[k], wk[k], pm);
        }
        float ss = acc.x + acc.y;
        const int width = tpr < 32 ? tpr : 32;
        for (int o = width >> 1; o > 0; o >>= 1) {
            ss += __shfl_xor_sync(0xffffffffu, ss, o);
            if constexpr (kFp8) pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, o));
        }
        if (wpr > 1) {
            float2* s2 = red + (parity * rpc + row_in_cta) * wpr;
            if ((lr & 31) == 0) s2[lr >> 5] = make_float2(ss, pm);
            group_barrier(1 + row_in_cta, tpr);
            float s = 0.f, m = 0.f;
            for (int i = 0; i < wpr; ++i) {
                const float2 t = s2[i];
                s += t.x;
                m = fmaxf(m, t.y);
            }
            ss = s;
            pm = m;
            parity ^= 1;
        }
        const float inv = 1.0f / sqrtf(ss / hf + a.eps);

        if constexpr (!kFp8) {
            uint4* orow = static_cast<uint4*>(a.out) + local + roff;
            const float2 inv2 = make_float2(inv, inv);
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                const int j = lr + k * tpr;
                if (!(active && j < nvec)) continue;
                const uint4 o = scale8<T, kHasW>(v[k], wk[k], inv2);
                st_v4(orow + j, o);
                if constexpr (kStage2) st_v4(reinterpret_cast<uint4*>(mine + lay.out2) + roff + j, o);
            }
        } else {
            const float qmul = pm > 0.f ? 448.0f / pm : 0.f;
            const float2 q2 = make_float2(qmul, qmul);
            if (active && lr == 0) {
                const float sc = pm > 0.f ? (pm * inv) / 448.0f : 0.f;
                a.scale[static_cast<int64_t>(ly) * a.T + row] = sc;
                if constexpr (kStage2) reinterpret_cast<float*>(mine + lay.scale2)[row] = sc;
            }
            uint2* qrow = reinterpret_cast<uint2*>(a.q) + local + roff;
#pragma unroll
            for (int k = 0; k < VPT; ++k) {
                const int j = lr + k * tpr;
                if (!(active && j < nvec)) continue;
                uint2 o = quant8<T, kHasW>(v[k], wk[k], q2);
                if (!(pm > 0.f)) o = make_uint2(0, 0);
                st_v2(qrow + j, o);
                if constexpr (kStage2) st_v2(reinterpret_cast<uint2*>(mine + lay.out2) + roff + j, o);
            }
        }
    }
}

// Two-shot step 6: copy the finished rows [s0, s1) that rank `owner` wrote
// into its buffer (this block's share of them) into this rank's outputs.
template <int VPT, bool kFp8>
__device__ __forceinline__ void gather_rows(const ArArgs& a, const int tpr, const int rpc,
                                            const int owner, const uint32_t epoch,
                                            const int nvec, const int64_t local,
                                            const int64_t s0, const int64_t s1) {
    const SlotLayout lay(a);
    const char* src = slot_base(a, owner, epoch);
    copy_rows<VPT>(static_cast<uint4*>(a.residual) + local,
                   reinterpret_cast<const uint4*>(src + lay.residual2), s0, s1, tpr, rpc, nvec,
                   true);
    if constexpr (!kFp8) {
        copy_rows<VPT>(static_cast<uint4*>(a.out) + local,
                       reinterpret_cast<const uint4*>(src + lay.out2), s0, s1, tpr, rpc, nvec,
                       true);
    } else {
        copy_rows<VPT>(reinterpret_cast<uint2*>(a.q) + local,
                       reinterpret_cast<const uint2*>(src + lay.out2), s0, s1, tpr, rpc, nvec,
                       true);
        const volatile float* sc2 = reinterpret_cast<const volatile float*>(src + lay.scale2);
        const int64_t stride = static_cast<int64_t>(gridDim.x) * rpc;
        for (int64_t base = s0 + static_cast<int64_t>(blockIdx.x) * rpc; base < s1; base += stride)
            for (int64_t r = base + threadIdx.x; r < base + rpc && r < s1; r += blockDim.x)
                a.scale[static_cast<int64_t>(blockIdx.y) * a.T + r] = sc2[r];
    }
}

// Publishes this block's stage `stage` of call `epoch` to every rank, then
// waits (bounded) for the same block of every rank. The barrier first orders
// every thread's prior writes before the release stores, and a system-scope
// release orders everything that happens before it: no separate fence is
// needed. Thread p publishes to and waits for rank p, so the W releases and
// polls proceed in parallel. Returns true (on every thread) when a wait ran out.
__device__ __forceinline__ bool exchange_barrier(const ArArgs& a, const int rank,
                                                 const uint32_t epoch, const int stage) {
    const int W = a.world;
    const int flag0 =
        kPadFlags + (((epoch & 1u) * 2 + stage) * kArMaxBlocks + blockIdx.x) * kArMaxWorld;
    __syncthreads();
    if (threadIdx.x < W) st_release_sys(a.signals[threadIdx.x] + flag0 + rank, epoch);
    bool late = false;
    if (threadIdx.x < W) {
        const uint32_t* f = a.signals[rank] + flag0 + threadIdx.x;
        if (ld_acquire_sys(f) != epoch) {
            const unsigned long long t0 = global_ns();
            while (ld_acquire_sys(f) != epoch) {
                if (global_ns() - t0 > static_cast<unsigned long long>(a.timeout_ns)) {
                    late = true;
                    break;
                }
                __nanosleep(64);
            }
        }
    }
    return __syncthreads_or(late) != 0;
}

template <typename T, int VPT, int kW, bool kFp8, bool kHasW, bool kTwoShot>
__device__ __forceinline__ void allreduce_rows(const ArArgs& a, const int tpr, const int rpc,
                                               float2* red) {
    const int ly = blockIdx.y;
    const int rank = a.rank + ly;
    const int W = a.world;
    const int nvec = static_cast<int>(a.H >> 3);
    const int64_t local = static_cast<int64_t>(ly) * a.T * nvec;  // in 16-byte vectors
    uint32_t* const pad = a.signals[rank];
    uint32_t epoch = *reinterpret_cast<volatile uint32_t*>(pad + kPadEpoch) + 1u;
    if (epoch == 0) epoch = 1;
    // two-shot: rank q owns the rows [q * S, (q + 1) * S)
    const int64_t S = kTwoShot ? (a.T + W - 1) / W : a.T;

    // 1. this block's rows of the local partial into this rank's buffer: the
    //    block's share of every slice, so that block b of the slice's owner
    //    waits only for block b of each rank
    {
        const uint4* x = static_cast<const uint4*>(a.x) + local;
        uint4* mine = reinterpret_cast<uint4*>(slot_base(a, rank, epoch));
        for (int q = 0; q < (kTwoShot ? W : 1); ++q) {
            const int64_t s0 = q * S, s1 = s0 + S < a.T ? s0 + S : a.T;
            copy_rows<VPT>(mine, x, s0 < a.T ? s0 : a.T, s1, tpr, rpc, nvec, false);
        }
    }

    // 2.-3. publish and wait for every rank's copy of the same rows
    bool late = exchange_barrier(a, rank, epoch, 0);
    if (!late) {
        if constexpr (!kTwoShot) {
            // 4. reduce + finish every row
            reduce_rows<T, VPT, kW, kFp8, kHasW, false>(a, tpr, rpc, red, ly, rank, epoch, nvec,
                                                        local, 0, a.T);
        } else {
            // 4. reduce + finish this rank's slice, also into its buffer;
            // 5. publish and wait; 6. copy every other slice from its owner
            const int64_t s0 = rank * S, s1 = s0 + S < a.T ? s0 + S : a.T;
            reduce_rows<T, VPT, kW, kFp8, kHasW, true>(a, tpr, rpc, red, ly, rank, epoch, nvec,
                                                       local, s0 < a.T ? s0 : a.T, s1);
            late = exchange_barrier(a, rank, epoch, 1);
            if (!late) {
                for (int q = 0; q < W; ++q) {
                    if (q == rank) continue;
                    const int64_t g0 = q * S, g1 = g0 + S < a.T ? g0 + S : a.T;
                    if (g0 < a.T) gather_rows<VPT, kFp8>(a, tpr, rpc, q, epoch, nvec, local, g0, g1);
                }
            }
        }
    }
    if (late && threadIdx.x == 0) atomicOr(&g_rn_ar_error, kErrPeerTimeout);

    // 7. arrival; the last block of this rank advances the call counter. Every
    //    block read the counter before arriving, and the next launch reads it
    //    only after this grid has completed, so no fence is needed.
    __syncthreads();
    if (threadIdx.x == 0 && atomicAdd(pad + kPadArrived, 1u) == gridDim.x - 1) {
        pad[kPadArrived] = 0u;
        pad[kPadEpoch] = epoch;
    }
}

template <typename T, int VPT, int kW, bool kFp8, bool kTwoShot>
__global__ void __launch_bounds__(kArMaxBlock)
    rn_allreduce_kernel(const ArArgs a, const int tpr, const int rpc) {
    extern __shared__ float2 red[];  // [2][rpc][warps per row]
    if (a.weight)
        allreduce_rows<T, VPT, kW, kFp8, true, kTwoShot>(a, tpr, rpc, red);
    else
        allreduce_rows<T, VPT, kW, kFp8, false, kTwoShot>(a, tpr, rpc, red);
}

// Groups of four or eight ranks on many rows: the same kernel held to 80
// registers, so three 256-thread blocks fit an SM instead of two (the
// rank-order reduction otherwise keeps every rank's vectors live: ~125
// registers). Measured on one device, [8192 x 3840] bf16: 8 ranks two-shot
// 636 -> 557 us, one-shot 1672 -> 1346 us; 4 ranks two-shot 329 -> 295 us.
// Its few spilled words cost more than the occupancy gains on a handful of
// rows (8 ranks, T = 64: 17.7 -> 22.0 us), and two ranks are 6 % slower at 80
// at any size, so the host picks it only for kW >= 4 and many rows.
template <typename T, int VPT, int kW, bool kFp8, bool kTwoShot>
__global__ void __maxnreg__(80) rn_allreduce_wide_kernel(const ArArgs a, const int tpr,
                                                           const int rpc) {
    extern __shared__ float2 red[];  // [2][rpc][warps per row]
    if (a.weight)
        allreduce_rows<T, VPT, kW, kFp8, true, kTwoShot>(a, tpr, rpc, red);
    else
        allreduce_rows<T, VPT, kW, kFp8, false, kTwoShot>(a, tpr, rpc, red);
}

using ArKernel = void (*)(const ArArgs, const int, const int);

template <typename T, int VPT, int kW, bool kFp8, bool kTwoShot>
ArKernel pick_kernel(bool wide) {
    if constexpr (kW >= 4) {
        if (wide) return rn_allreduce_wide_kernel<T, VPT, kW, kFp8, kTwoShot>;
    }
    return rn_allreduce_kernel<T, VPT, kW, kFp8, kTwoShot>;
}

template <typename T, int kW, bool kFp8, bool kTwoShot>
ArKernel pick_vpt(int vpt, bool wide) {
    switch (vpt) {
        case 1: return pick_kernel<T, 1, kW, kFp8, kTwoShot>(wide);
        case 2: return pick_kernel<T, 2, kW, kFp8, kTwoShot>(wide);
        case 4: return pick_kernel<T, 4, kW, kFp8, kTwoShot>(wide);
        case 8: return pick_kernel<T, 8, kW, kFp8, kTwoShot>(wide);
        default: return nullptr;
    }
}

// Two-shot kernels exist for groups of 3 to 8 ranks (it moves more data than
// one-shot with two ranks).
template <typename T, bool kFp8>
ArKernel pick_w(int world, int vpt, bool two_shot, bool wide) {
    if (two_shot) {
        if (world < 3) return nullptr;
        if (world <= 4) return pick_vpt<T, 4, kFp8, true>(vpt, wide);
        return pick_vpt<T, 8, kFp8, true>(vpt, wide);
    }
    if (world == 1) return pick_vpt<T, 1, kFp8, false>(vpt, wide);
    if (world == 2) return pick_vpt<T, 2, kFp8, false>(vpt, wide);
    if (world <= 4) return pick_vpt<T, 4, kFp8, false>(vpt, wide);
    return pick_vpt<T, 8, kFp8, false>(vpt, wide);
}

ArKernel pick(int dtype, bool fp8, int world, const ArLaunch& l) {
    if (world < 1 || world > kArMaxWorld) return nullptr;
    if (dtype == kBF16)
        return fp8 ? pick_w<__nv_bfloat16, true>(world, l.vpt, l.two_shot, l.wide)
                   : pick_w<__nv_bfloat16, false>(world, l.vpt, l.two_shot, l.wide);
    if (dtype == kF16)
        return fp8 ? pick_w<__half, true>(world, l.vpt, l.two_shot, l.wide)
                   : pick_w<__half, false>(world, l.vpt, l.two_shot, l.wide);
    return nullptr;
}

}  // namespace

cudaError_t allreduce_blocks_per_sm(int dtype, bool fp8, int world, const ArLaunch& l,
                                    int* blocks) {
    const ArKernel k = pick(dtype, fp8, world, l);
    if (!k) return cudaErrorInvalidValue;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(blocks, k, l.block,
                                                         static_cast<size_t>(l.smem));
}

cudaError_t launch_allreduce(int dtype, bool fp8, const ArArgs& a, const ArLaunch& l,
                             cudaStream_t s) {
    const ArKernel k = pick(dtype, fp8, a.world, l);
    if (!k) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(l.grid_x), static_cast<unsigned>(l.local_ranks));
    cfg.blockDim = dim3(static_cast<unsigned>(l.block));
    cfg.dynamicSmemBytes = static_cast<size_t>(l.smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = l.local_ranks > 1 ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k, a, l.tpr, l.rpc);
}

// Exchange memory of rn_allreduce_fused_add_rms_norm_local: signal pads, then
// buffers (rn_allreduce.h). Zero at module load; the pads are cleared again by
// the host whenever the group size on a device changes.
static __device__ __align__(256) unsigned char g_rn_local_scratch[kLocalScratchBytes];

cudaError_t local_scratch_address(void** p) {
    return cudaGetSymbolAddress(p, g_rn_local_scratch);
}

cudaError_t read_and_clear_allreduce_errors(unsigned* flags) {
    unsigned v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_rn_ar_error, sizeof v);
    if (e != cudaSuccess) return e;
    *flags = v;
    if (v) {
        const unsigned zero = 0;
        e = cudaMemcpyToSymbol(g_rn_ar_error, &zero, sizeof zero);
    }
    return e;
}

}  // namespace rn
