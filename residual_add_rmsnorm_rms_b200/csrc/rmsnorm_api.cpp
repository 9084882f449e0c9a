// rmsnorm_api.cpp -- the C ABI of include/rmsnorm_b200.h: argument
// validation (the eligibility rules of the AITER wrappers in
// "vllm.kernels.aiter_ops": 16-bit activations, matching weight dtype or
// None, no variance-size override, free flattening to dense 2-D), aliasing
// rules, launch planning and the launch itself. Pure host code.
#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include <atomic>
#include <initializer_list>

#include <cuda.h>
#include <cuda_runtime_api.h>

#include "../../include/rmsnorm_b200.h"
#include "rn_internal.h"
#include "rn_allreduce.h"
#include "rn_gemm.h"

// The header's sizes restate internal constants; a mismatch must not build.
static_assert(RN_LOCAL_EXCHANGE_BYTES == rn::kLocalBufferBytes,
              "RN_LOCAL_EXCHANGE_BYTES differs from the static exchange memory");
static_assert(RN_ALLREDUCE_SIGNAL_BYTES == rn::kArSignalBytes,
              "RN_ALLREDUCE_SIGNAL_BYTES differs from the signal pad layout");
static_assert(RN_ALLREDUCE_MAX_WORLD == rn::kArMaxWorld,
              "RN_ALLREDUCE_MAX_WORLD differs from the kernels' group limit");
// (unary + compares the two enums as integers)
static_assert(+RN_GEMM_TOK128_CH128 == +rn::kGemmTok128Ch128 &&
                  +RN_GEMM_CH128_TOK16 == +rn::kGemmCh128Tok16 &&
                  +RN_GEMM_CH128_TOK32 == +rn::kGemmCh128Tok32 &&
                  +RN_GEMM_CH128_TOK64 == +rn::kGemmCh128Tok64 &&
                  +RN_GEMM_CH64_TOK16 == +rn::kGemmCh64Tok16 &&
                  +RN_GEMM_CH64_TOK32 == +rn::kGemmCh64Tok32 &&
                  +RN_GEMM_CH64_TOK64 == +rn::kGemmCh64Tok64 &&
                  +RN_GEMM_TOK128_CH256 == +rn::kGemmTok128Ch256 && rn::kNumGemmConfigs == 8,
              "rn_gemm_config must match the GEMM dispatch");

namespace {

thread_local char g_cuda_error[256] = "";
std::atomic<int> g_force_tpr{0};
std::atomic<int> g_force_vpt{0};
std::atomic<int> g_force_rpc{0};
std::atomic<int> g_force_staged_c{0};
std::atomic<int> g_force_staged_s{0};
std::atomic<int> g_force_staged_t{0};
std::atomic<int> g_pdl{-1};              // -1 default, 0 off, 1 on
std::atomic<long long> g_max_grid{0};    // 0: no cap
std::atomic<int> g_prefetch{-1};         // -1 default, 0 off, 1 on
std::atomic<int> g_force_gemm{-1};       // fp8 GEMM tile configuration; -1: automatic
// Launch defaults, measured on B200 (prefill [8192 x 3840], two ops
// alternating in one stream): programmatic dependent launch lets the next
// kernel's blocks start as this one drains (+4-5 %); rms_norm and the fused
// ops on fewer rows cap the vector kernel's grid at 16 blocks per SM (blocks
// then stride over rows; see default_grid_cap).
// The L2 prefetch of each block's first rows before it waits for the
// previous kernel keeps HBM busy across the kernel boundary: the prefill
// step 73.84 -> 71.33 us, [4096 x H] cells of the sweep 2-10 % faster,
// identical results.
constexpr bool kPdlDefault = true;
constexpr bool kPrefetchDefault = true;
constexpr int kVectorBlocksPerSmCap = 16;
constexpr int kDefaultSms = 148;  // B200; dry runs (no device) plan for it

int elem_size(int32_t dt) {
    switch (dt) {
        case RN_F16:
        case RN_BF16: return 2;
        case RN_E4M3: return 1;
        case RN_F32: return 4;
        default: return 0;
    }
}

struct Flat {
    char* ptr = nullptr;
    int64_t T = 0, H = 0, numel = 0;
    int esize = 0;
    int64_t bytes() const { return numel * esize; }
};

// flatten_to_2d_is_free ("vllm.kernels.aiter_ops"), applied to every rank:
// unit last stride; each leading dim of size != 1 has the dense stride.
rn_status flatten(const rn_tensor* t, Flat* f) {
    if (t->ndim < 1 || t->ndim > RN_MAX_DIMS) return RN_ERR_SHAPE;
    if (!t->sizes || !t->strides) return RN_ERR_NULL;
    const int n = t->ndim;
    int64_t numel = 1;
    for (int i = 0; i < n; ++i) {
        if (t->sizes[i] < 0) return RN_ERR_SHAPE;
        if (t->sizes[i] != 0 && numel > INT64_MAX / t->sizes[i]) return RN_ERR_SHAPE;
        numel *= t->sizes[i];
    }
    const int64_t H = t->sizes[n - 1];
    if (H == 0) return RN_ERR_SHAPE;
    if (numel > 0) {
        if (t->strides[n - 1] != 1) return RN_ERR_LAYOUT;
        int64_t expected = H;
        for (int i = n - 2; i >= 0; --i) {
            if (t->sizes[i] != 1 && t->strides[i] != expected) return RN_ERR_LAYOUT;
            expected *= t->sizes[i];
        }
    }
    f->ptr = static_cast<char*>(t->data);
    f->H = H;
    f->numel = numel;
    f->T = numel / H;
    f->esize = elem_size(t->dtype);
    return RN_OK;
}

bool overlap(const Flat& a, const Flat& b) {
    if (a.bytes() == 0 || b.bytes() == 0) return false;
    const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.ptr), a1 = a0 + a.bytes();
    const uintptr_t b0 = reinterpret_cast<uintptr_t>(b.ptr), b1 = b0 + b.bytes();
    return a0 < b1 && b0 < a1;
}

bool same_extent(const Flat& a, const Flat& b) { return a.ptr == b.ptr && a.bytes() == b.bytes(); }

bool aligned(const void* p, uintptr_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

int clamp_rpc(int rpc, int tpr, int64_t T) {
    if (rpc < 1) rpc = 1;
    if (tpr > 32 && rpc > 15) rpc = 15;  // named barriers 1..15, one per row group
    if (T > 0 && rpc > T) {
        // Keep sub-warp groups whole-warp: a warp never straddles two CTAs.
        const int64_t min_rpc = tpr < 32 ? 32 / tpr : 1;
        rpc = static_cast<int>(T < min_rpc ? min_rpc : T);
        if (tpr < 32) rpc = static_cast<int>(((rpc + min_rpc - 1) / min_rpc) * min_rpc);
    }
    return rpc;
}

bool vpt_compiled(int vpt) {
    for (int i = 0; i < rn::kNumVpt; ++i)
        if (rn::kVptList[i] == vpt) return true;
    return false;
}

bool tpr_valid(int tpr) {
    if (tpr >= 1 && tpr <= 32) return (tpr & (tpr - 1)) == 0;
    return tpr > 32 && tpr <= 1024 && tpr % 32 == 0;
}

// Smallest legal threads-per-row that covers nvec vectors at width vpt.
int tpr_for(int64_t nvec, int vpt) {
    const int64_t need = (nvec + vpt - 1) / vpt;
    if (need <= 32) {
        int t = 1;
        while (t < need) t <<= 1;
        return t;
    }
    return static_cast<int>(((need + 31) / 32) * 32);
}

void fill_vector_plan(int tpr, int vpt, int64_t T, rn_plan* p, int want_rpc = 0) {
    // Aim for ~256-thread blocks: several rows per block for narrow rows.
    int rpc = want_rpc > 0 ? want_rpc : (tpr >= 256 ? 1 : 256 / tpr);
    while (rpc > 1 && tpr * rpc > rn::max_block_for_vpt(vpt)) --rpc;
    if (tpr < 32) rpc = ((rpc + 32 / tpr - 1) / (32 / tpr)) * (32 / tpr);  // whole warps
    rpc = clamp_rpc(rpc, tpr, T);
    p->kernel = RN_KERNEL_VECTOR;
    p->threads_per_row = tpr;
    p->vectors_per_thread = vpt;
    p->rows_per_cta = rpc;
    p->block_threads = tpr * rpc;
    const int wpr = tpr / 32;
    p->smem_bytes = wpr > 1 ? static_cast<int32_t>(2 * rpc * wpr * sizeof(float) * 2) : 0;
    p->grid = T > 0 ? (T + rpc - 1) / rpc : 0;
}

int64_t round_up(int64_t v, int64_t m) { return (v + m - 1) / m * m; }

int64_t staged_smem(int op, int64_t H, int stages) {
    const int nin = op == rn::kRmsNorm ? 1 : 2;
    // ring + fp32 copy of the weight + one mbarrier per stage + reduction slots
    return stages * nin * round_up(2 * H, 128) + 4 * H + stages * 8 + 32 * 8;
}

// Fills a STAGED plan for (c CTAs per SM, S stages, threads); false if it
// does not fit the per-block shared memory.
bool fill_staged_plan(int op, int64_t T, int64_t H, int c, int S, int threads, int num_sms,
                      rn_plan* p) {
    const int64_t smem = staged_smem(op, H, S);
    if (S < 2 || smem > rn::kStagedMaxSmem || threads < 32 || threads > 1024 || threads % 32)
        return false;
    p->kernel = RN_KERNEL_STAGED;
    p->threads_per_row = threads;
    p->vectors_per_thread = 0;
    p->rows_per_cta = 1;
    p->block_threads = threads;
    p->smem_bytes = static_cast<int32_t>(smem);
    p->stages = S;
    p->ctas_per_sm = c;
    const int64_t g = static_cast<int64_t>(c) * num_sms;
    p->grid = T < g ? T : g;
    return true;
}

void fill_scalar_plan(int64_t T, rn_plan* p) {
    p->kernel = RN_KERNEL_SCALAR;
    p->threads_per_row = 256;
    p->vectors_per_thread = 0;
    p->rows_per_cta = 1;
    p->block_threads = 256;
    p->smem_bytes = 0;
    p->grid = T;
}

// Automatic choice of (threads per row, vectors per thread, rows per block)
// for the vector kernel, from a sweep of forced shapes on B200 (H 2048..16384,
// T 1..32768, all three ops):
//  * many rows (T x threads-per-row at 4 vectors/thread >= one full wave of
//    1024 threads per SM): 4 vectors per thread (<= 64 registers, so 32 warps
//    per SM stay resident with 64 bytes of loads in flight per thread and
//    tensor), tolerating up to 1/8 idle vector slots; rows per block such
//    that a block holds ~256 threads (~512 when T >= 16384, where coarser
//    blocks cost less at the tail), two rows for 129..256 threads per row,
//    one above;
//  * few rows (decode): about 256 threads per row (512 for H > 4096; 1024 for
//    H >= 16384 with T <= 64) with
//    the fewest vectors per thread that cover the row (more threads per row
//    buy latency, not bandwidth, past that point); rows per block as above
//    but never fewer blocks than SMs.
// Rows per block. rms_norm, which moves half the bytes of the fused ops per
// row: about 256 threads per block (the nearest whole number of rows). The
// fused ops: 256 threads, 512 on many rows. From forced-shape sweeps on B200
// (rms_norm at T = 4096-65536 was up to 13 % faster with ~256-thread blocks
// than with the fused ops' rule, except that 160-thread rows still want two
// per block).
int rows_per_block(int op, int tpr, int64_t T) {
    if (op == rn::kRmsNorm) {
        const int r = (256 + tpr / 2) / tpr;
        return r < 1 ? 1 : r;
    }
    if (tpr <= 128) return (T >= 16384 ? 512 : 256) / tpr;
    if (tpr <= 256) return 2;
    return 1;
}

// Row count from which the fused ops run an uncapped grid (one row group per
// block), and the one from which the fp8 op's blocks grow to ~512 threads.
constexpr int64_t kFusedManyRows = 8192;
constexpr int64_t kFp8WideBlockRows = 16384;

// Rows per block of the fused ops when the rows fill at least a wave, from a
// grid of forced shapes on B200 with the first-row prefetch (T = 4096-65536,
// H = 2048-16384; each rule within 1 % of the best shape on average):
// fused_add_rms_norm, about 512 threads; fused_add_rms_norm_fp8 and the
// SwiGLU kernel, about 256 threads below kFp8WideBlockRows rows (two rows of
// 129-256 threads), about 512 from there on.
int many_rows_per_block(int op, int tpr, int64_t T) {
    if (op == rn::kRmsNorm) return rows_per_block(op, tpr, T);
    if (op != rn::kFusedAdd && T < kFp8WideBlockRows) {
        if (tpr <= 128) return 256 / tpr;
        return tpr <= 256 ? 2 : 1;
    }
    const int r = (512 + tpr / 2) / tpr;
    return r < 1 ? 1 : r;
}

// Cap on the vector kernel's grid, in blocks (0: none). With the first-row
// prefetch, the fused ops on kFusedManyRows rows or more run fastest with one
// row group per block (2-7 % faster than 16 blocks per SM striding over the
// rows at T = 16384-65536), and so does the SwiGLU kernel from 4096 rows
// ([8192 x 15360] 6 % faster, [4096 x 15360] 3 %; [32768 x 15360] 1.8 %
// slower); otherwise 16 blocks per SM.
long long default_grid_cap(int op, int64_t T, int num_sms) {
    if ((op == rn::kFusedAdd || op == rn::kFusedAddFp8) && T >= kFusedManyRows) return 0;
    if (op == rn::kSwigluFp8 && T >= 4096) return 0;
    return static_cast<long long>(kVectorBlocksPerSmCap) * num_sms;
}

bool auto_vector_plan(int op, int dt, int64_t T, int64_t H, int num_sms, rn_plan* p) {
    const int64_t nvec = H / 8;
    auto idle_of = [&](int tpr, int vpt) {
        const int64_t slots = static_cast<int64_t>(tpr) * vpt;
        return static_cast<double>(slots - nvec) / static_cast<double>(slots);
    };
    const int tpr4 = tpr_for(nvec, 4);
    const bool many_rows = tpr4 <= rn::max_block_for_vpt(4) &&
                           static_cast<double>(T) * tpr4 >= 1.0 * num_sms * 1024;
    if (many_rows) {
        // Eight vectors per thread, one row per block of 128-256 threads:
        // half the warps per row of the four-vector plan, so half the
        // cross-warp reduction. Taken by rms_norm on rows that would need 512
        // threads at four vectors (H = 16384: 2-5 % faster at T =
        // 4096-65536, both formats), and by the bf16 fp8 op on such rows and,
        // below kFusedManyRows rows, on rows of 128 or more threads at eight
        // vectors (T = 4096: H = 7168 4.4 % faster, 8192 2 %; from T = 8192
        // on, 5-10 % slower). The fp16 fp8 op, whose fp16 -> fp32 widening
        // costs more issue slots than bf16's shifts, keeps four vectors (4-7 %
        // faster at T = 4096, H = 7168-16384).
        const int tpr8 = tpr_for(nvec, 8);
        const bool fp8_bf16 = op == rn::kFusedAddFp8 && dt == rn::kBF16;
        const bool wide = tpr4 >= 512 && (op == rn::kRmsNorm || fp8_bf16);
        const bool fp8_few = fp8_bf16 && T < kFusedManyRows && tpr8 >= 128;
        if ((wide || fp8_few) && tpr8 <= rn::max_block_for_vpt(8) && idle_of(tpr8, 8) <= 1.0 / 8) {
            fill_vector_plan(tpr8, 8, T, p, 1);
            return true;
        }
        // Four vectors per thread first. (Three that tile the row exactly beat
        // four with idle lanes, H = 3840, by 1.9 % for fused_add_rms_norm
        // with 16-byte accesses; with 32-byte pairs four win by 0.6 %.)
        for (int vpt : {4, 5, 3, 6, 8, 2}) {
            const int tpr = tpr_for(nvec, vpt);
            if (tpr > rn::max_block_for_vpt(vpt) || idle_of(tpr, vpt) > 1.0 / 8) continue;
            fill_vector_plan(tpr, vpt, T, p, many_rows_per_block(op, tpr, T));
            return true;
        }
    }
    // very few very wide rows: every extra thread per row shortens the row
    const int target = (nvec >= 2048 && T <= 64) ? 1024 : (nvec <= 512 ? 256 : 512);
    for (int i = 0; i < rn::kNumVpt; ++i) {
        const int vpt = rn::kVptList[i];
        const int tpr = tpr_for(nvec, vpt);
        if (tpr > target || tpr > rn::max_block_for_vpt(vpt) || idle_of(tpr, vpt) > 1.0 / 8)
            continue;
        // narrow rows share a block, but keep at least one block per SM
        int rpc = rows_per_block(op, tpr, T);
        const int64_t per_sm = T / num_sms > 0 ? T / num_sms : 1;
        if (rpc > per_sm) rpc = static_cast<int>(per_sm);
        fill_vector_plan(tpr, vpt, T, p, rpc);
        return true;
    }
    // Rows too wide for the preferred targets: any width that fits.
    for (int i = 0; i < rn::kNumVpt; ++i) {
        const int vpt = rn::kVptList[i];
        const int tpr = tpr_for(nvec, vpt);
        if (tpr > rn::max_block_for_vpt(vpt)) continue;
        fill_vector_plan(tpr, vpt, T, p, 1);
        return true;
    }
    return false;
}

rn_status plan_shape(int op, int dt, int64_t T, int64_t H, bool vector_ok, int num_sms,
                     rn_plan* p, bool allow_staged);

// The launch plan: the kernel and its shape, then the grid cap (the kernels
// stride over the rows a capped grid does not cover). `allow_staged` is false
// for kernels that have no staged form.
rn_status plan_impl(int op, int dt, int64_t T, int64_t H, bool vector_ok, int num_sms, rn_plan* p,
                    bool allow_staged = true) {
    const rn_status st = plan_shape(op, dt, T, H, vector_ok, num_sms, p, allow_staged);
    if (st != RN_OK) return st;
    long long cap = g_max_grid.load();
    if (cap == 0 && p->kernel == RN_KERNEL_VECTOR) cap = default_grid_cap(op, T, num_sms);
    if (cap > 0 && p->grid > cap) p->grid = cap;
    if (p->grid > 0x7fffffffLL) p->grid = 0x7fffffffLL;
    return RN_OK;
}

rn_status plan_shape(int op, int dt, int64_t T, int64_t H, bool vector_ok, int num_sms,
                     rn_plan* p, bool allow_staged) {
    if (H < 1 || T < 0) return RN_ERR_SHAPE;
    std::memset(p, 0, sizeof *p);
    if (!vector_ok || H % 8 != 0) {
        fill_scalar_plan(T, p);
        return RN_OK;
    }
    const int fc = g_force_staged_c.load(), fs = g_force_staged_s.load(),
              ft = g_force_staged_t.load();
    if (allow_staged && fc && fs && ft && fill_staged_plan(op, T, H, fc, fs, ft, num_sms, p))
        return RN_OK;
    std::memset(p, 0, sizeof *p);
    const int ftpr = g_force_tpr.load(), fvpt = g_force_vpt.load();
    if (ftpr && fvpt) {
        const int64_t nvec = H / 8;
        if (static_cast<int64_t>(ftpr) * fvpt >= nvec && ftpr <= rn::max_block_for_vpt(fvpt)) {
            fill_vector_plan(ftpr, fvpt, T, p, g_force_rpc.load());
        } else {
            fill_scalar_plan(T, p);
        }
        return RN_OK;
    }
    // The STAGED kernel is chosen only when forced: measured on B200 it trails
    // the VECTOR kernel at every shape tried (T up to 65536, H 2048..16384).
    if (!auto_vector_plan(op, dt, T, H, num_sms, p)) fill_scalar_plan(T, p);
    return RN_OK;
}

int device_sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return kDefaultSms;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
        return kDefaultSms;
    return n;
}

// Tile configuration of the fp8 GEMM for an [M x K] x [N x K]^T problem.
// A decode-sized GEMM is bound by streaming the weight, and a CTA streams
// only its own tiles, so the choice maximises the tiles in flight: among the
// channel-major shapes (channels x tokens: 64 or 128 x 16, 32 or 64), the one
// with the most tiles that still fit in one wave (ties: fewer channels, then
// fewer tokens per tile). When none fits, up to 64 tokens take the 128-channel
// tile of the smallest token width >= M (fewest tiles), larger M a token-major
// tile. Measured on B200 over the Gemma 4 12B weight
// shapes, this picks the fastest configuration or one within 5 % of it.
int gemm_auto_config(int64_t M, int64_t N, int num_sms) {
    struct Shape { int config, ch, tok; };
    static constexpr Shape kChannelMajor[] = {
        {rn::kGemmCh64Tok16, 64, 16},   {rn::kGemmCh64Tok32, 64, 32},
        {rn::kGemmCh64Tok64, 64, 64},   {rn::kGemmCh128Tok16, 128, 16},
        {rn::kGemmCh128Tok32, 128, 32}, {rn::kGemmCh128Tok64, 128, 64}};
    int best = -1;
    int64_t best_tiles = 0;
    for (const Shape& c : kChannelMajor) {
        const int64_t tiles = ((N + c.ch - 1) / c.ch) * ((M + c.tok - 1) / c.tok);
        if (tiles <= num_sms && tiles > best_tiles) {
            best = c.config;
            best_tiles = tiles;
        }
    }
    if (best >= 0) return best;
    if (M <= 16) return rn::kGemmCh128Tok16;
    if (M <= 32) return rn::kGemmCh128Tok32;
    if (M <= 64) return rn::kGemmCh128Tok64;
    // token-major: 128 x 256 tiles once they fill a wave (12-16 % faster than
    // 128 x 128 at M = 8192 on B200), else 128 x 128 for twice the tiles
    const int64_t tiles256 = ((M + 127) / 128) * ((N + 255) / 256);
    return tiles256 >= num_sms ? rn::kGemmTok128Ch256 : rn::kGemmTok128Ch128;
}

int gemm_config(int64_t M, int64_t N, int num_sms) {
    const int f = g_force_gemm.load();
    return f >= 0 ? f : gemm_auto_config(M, N, num_sms);
}

struct Common {
    Flat x, out, res, q, scale, w;
    bool has_w = false;
    int dt = 0;
};

rn_status check_weight(const rn_tensor* weight, int32_t xdt, int64_t H, Common* c) {
    if (!weight) return RN_OK;
    if (weight->dtype != xdt) return RN_ERR_WEIGHT_DTYPE;
    if (weight->ndim != 1) return RN_ERR_SHAPE;
    Flat f;
    rn_status st = flatten(weight, &f);
    if (st != RN_OK) return st;
    if (f.numel != H) return RN_ERR_SHAPE;
    c->w = f;
    c->has_w = true;
    return RN_OK;
}

rn_status check_scalars(float eps, int64_t variance_size) {
    if (variance_size != -1) return RN_ERR_VARIANCE_SIZE;
    if (!std::isfinite(eps) || eps < 0.f) return RN_ERR_EPS;
    return RN_OK;
}

bool is16(int32_t dt) { return dt == RN_F16 || dt == RN_BF16; }

// Descriptor-level checks of one call, in the documented order: NULL
// descriptors, variance_size and eps, dtypes, weight dtype, shapes and
// layouts. Fills `c`.
rn_status check_descriptors(int op, const rn_tensor* o, const rn_tensor* sc, const rn_tensor* x,
                            const rn_tensor* r, const rn_tensor* w, float eps,
                            int64_t variance_size, Common* c) {
    if (!o || !x || (op != rn::kRmsNorm && !r) || (op == rn::kFusedAddFp8 && !sc))
        return RN_ERR_NULL;
    rn_status st = check_scalars(eps, variance_size);
    if (st != RN_OK) return st;
    if (!is16(x->dtype)) return RN_ERR_DTYPE;
    if (op != rn::kRmsNorm && r->dtype != x->dtype) return RN_ERR_DTYPE;
    if (op == rn::kFusedAddFp8) {
        if (o->dtype != RN_E4M3 || sc->dtype != RN_F32) return RN_ERR_DTYPE;
    } else if (o->dtype != x->dtype) {
        return RN_ERR_DTYPE;
    }
    if (w && w->dtype != x->dtype) return RN_ERR_WEIGHT_DTYPE;
    c->dt = x->dtype == RN_BF16 ? rn::kBF16 : rn::kF16;
    if ((st = flatten(x, &c->x)) != RN_OK) return st;
    Flat* of = op == rn::kFusedAddFp8 ? &c->q : &c->out;
    if ((st = flatten(o, of)) != RN_OK) return st;
    if (of->T != c->x.T || of->H != c->x.H) return RN_ERR_SHAPE;
    if (op != rn::kRmsNorm) {
        if ((st = flatten(r, &c->res)) != RN_OK) return st;
        if (c->res.T != c->x.T || c->res.H != c->x.H) return RN_ERR_SHAPE;
    }
    if (op == rn::kFusedAddFp8) {
        // scale: T fp32 values, dense (e.g. [T] or [T x 1]); unused when T == 0.
        if (c->x.T > 0) {
            if ((st = flatten(sc, &c->scale)) != RN_OK) return st;
            if (c->scale.numel != c->x.T) return RN_ERR_SHAPE;
        } else if (sc->ndim < 1 || sc->ndim > RN_MAX_DIMS) {
            return RN_ERR_SHAPE;
        }
    }
    return check_weight(w, x->dtype, c->x.H, c);
}

// Pointer-level checks (NULL data, element alignment, aliasing) and the plan.
// Only called for T > 0.
rn_status check_pointers_and_plan(int op, const Common& c, int num_sms, rn_plan* plan) {
    const int64_t T = c.x.T, H = c.x.H;
    if (!c.x.ptr || (op != rn::kFusedAddFp8 && !c.out.ptr)) return RN_ERR_NULL;
    if (op != rn::kRmsNorm && !c.res.ptr) return RN_ERR_NULL;
    if (op == rn::kFusedAddFp8 && (!c.q.ptr || !c.scale.ptr)) return RN_ERR_NULL;
    if (c.has_w && !c.w.ptr) return RN_ERR_NULL;
    if (!aligned(c.x.ptr, 2) || (c.out.ptr && !aligned(c.out.ptr, 2)) ||
        (c.res.ptr && !aligned(c.res.ptr, 2)) || (c.has_w && !aligned(c.w.ptr, 2)) ||
        (c.scale.ptr && !aligned(c.scale.ptr, 4)))
        return RN_ERR_LAYOUT;
    // Aliasing: written buffers must not overlap each other or any input,
    // except out == x exactly (in place) for the 16-bit-output ops.
    Flat written[3];
    int nw = 0;
    if (op == rn::kFusedAddFp8) {
        written[nw++] = c.res;
        written[nw++] = c.q;
        written[nw++] = c.scale;
    } else {
        written[nw++] = c.out;
        if (op == rn::kFusedAdd) written[nw++] = c.res;
    }
    for (int i = 0; i < nw; ++i) {
        for (int j = i + 1; j < nw; ++j)
            if (overlap(written[i], written[j])) return RN_ERR_ALIAS;
        const bool is_out = (op != rn::kFusedAddFp8 && i == 0);
        if (overlap(written[i], c.x) && !(is_out && same_extent(written[i], c.x)))
            return RN_ERR_ALIAS;
        if (c.has_w && overlap(written[i], c.w)) return RN_ERR_ALIAS;
    }
    if (op != rn::kRmsNorm && overlap(c.res, c.x)) return RN_ERR_ALIAS;

    bool vector_ok = (H % 8 == 0) && aligned(c.x.ptr, 16) && (!c.has_w || aligned(c.w.ptr, 16));
    if (op != rn::kFusedAddFp8) vector_ok = vector_ok && aligned(c.out.ptr, 16);
    if (op != rn::kRmsNorm) vector_ok = vector_ok && aligned(c.res.ptr, 16);
    if (op == rn::kFusedAddFp8) vector_ok = vector_ok && aligned(c.q.ptr, 8);
    rn_status st = plan_impl(op, c.dt, T, H, vector_ok, num_sms, plan);
    if (st != RN_OK) return st;

    return RN_OK;
}

// All checks of one call; *launch_needed is false for the T == 0 no-op.
rn_status prepare(int op, const rn_tensor* o, const rn_tensor* sc, const rn_tensor* x,
                  const rn_tensor* r, const rn_tensor* w, float eps, int64_t variance_size,
                  int num_sms, Common* c, rn_plan* plan, bool* launch_needed) {
    *launch_needed = false;
    std::memset(plan, 0, sizeof *plan);
    rn_status st = check_descriptors(op, o, sc, x, r, w, eps, variance_size, c);
    if (st != RN_OK) return st;
    if (c->x.T == 0) return RN_OK;
    st = check_pointers_and_plan(op, *c, num_sms, plan);
    if (st != RN_OK) return st;
    *launch_needed = true;
    return RN_OK;
}

// Whether the vector kernel may move its vectors in adjacent pairs with
// 32-byte accesses: an even vector count per row (H % 16 == 0) and 32-byte
// aligned 16-bit rows (x, and out or residual where written; the weight is
// read 16 bytes at a time), 16-byte aligned code rows for the fp8 op.
bool pair_ok(int op, int64_t H, const void* x, const void* res, const void* out,
             const void* q) {
    if (H % 16 != 0 || !aligned(x, 32)) return false;
    if (op != rn::kRmsNorm && !aligned(res, 32)) return false;
    if (op != rn::kFusedAddFp8) return aligned(out, 32);
    return aligned(q, 16);
}

// Enqueues the norm kernel `plan` describes; `pair` as pair_ok (used by the
// vector kernel when its vector count per thread is even).
rn_status launch_plan(int op, int dt, const rn::Args& a, const rn_plan& plan, bool pdl,
                      bool pair, void* stream) {
    rn::Launch l{plan.kernel,
                 plan.threads_per_row,
                 plan.kernel == RN_KERNEL_STAGED ? plan.stages : plan.vectors_per_thread,
                 plan.rows_per_cta,
                 plan.block_threads,
                 plan.smem_bytes,
                 plan.grid,
                 pdl};
    l.pair = pair && plan.kernel == RN_KERNEL_VECTOR && plan.vectors_per_thread % 2 == 0;
    l.prefetch = g_prefetch.load() < 0 ? kPrefetchDefault : g_prefetch.load() == 1;
    const cudaError_t e = rn::launch(op, dt, a, l, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        std::snprintf(g_cuda_error, sizeof g_cuda_error, "%s: %s", cudaGetErrorName(e),
                      cudaGetErrorString(e));
        return RN_ERR_CUDA;
    }
    return RN_OK;
}

rn_status run(int op, const rn_tensor* o, const rn_tensor* sc, const rn_tensor* x,
              const rn_tensor* r, const rn_tensor* w, float eps, int64_t variance_size,
              void* stream) {
    Common c;
    rn_plan plan;
    bool launch_needed;
    rn_status st = check_descriptors(op, o, sc, x, r, w, eps, variance_size, &c);
    if (st != RN_OK || c.x.T == 0) return st;
    st = prepare(op, o, sc, x, r, w, eps, variance_size, device_sms(), &c, &plan,
                 &launch_needed);
    if (st != RN_OK || !launch_needed) return st;
    rn::Args a;
    a.x = c.x.ptr;
    a.residual = c.res.ptr;
    a.weight = c.has_w ? c.w.ptr : nullptr;
    a.out = c.out.ptr;
    a.q = reinterpret_cast<uint8_t*>(c.q.ptr);
    a.scale = reinterpret_cast<float*>(c.scale.ptr);
    a.T = c.x.T;
    a.H = c.x.H;
    a.eps = eps;
    return launch_plan(op, c.dt, a, plan, g_pdl.load() < 0 ? kPdlDefault : g_pdl.load() == 1,
                       pair_ok(op, a.H, a.x, a.residual, a.out, a.q), stream);
}

// The current CUDA context's unique id (defined with the local all-reduce state).
bool current_context_id(unsigned long long* id);

}  // namespace

extern "C" {

rn_status rn_rms_norm(const rn_tensor* out, const rn_tensor* x, const rn_tensor* weight,
                      float eps, int64_t variance_size, void* stream) {
    return run(rn::kRmsNorm, out, nullptr, x, nullptr, weight, eps, variance_size, stream);
}

rn_status rn_fused_add_rms_norm(const rn_tensor* out, const rn_tensor* x,
                                const rn_tensor* residual, const rn_tensor* weight, float eps,
                                int64_t variance_size, void* stream) {
    return run(rn::kFusedAdd, out, nullptr, x, residual, weight, eps, variance_size, stream);
}

rn_status rn_fused_add_rms_norm_fp8(const rn_tensor* q, const rn_tensor* scale,
                                    const rn_tensor* x, const rn_tensor* residual,
                                    const rn_tensor* weight, float eps, int64_t variance_size,
                                    void* stream) {
    return run(rn::kFusedAddFp8, q, scale, x, residual, weight, eps, variance_size, stream);
}

rn_status rn_silu_and_mul_fp8(const rn_tensor* q, const rn_tensor* scale, const rn_tensor* x,
                              void* stream) {
    if (!q || !scale || !x) return RN_ERR_NULL;
    if (!is16(x->dtype) || q->dtype != RN_E4M3 || scale->dtype != RN_F32) return RN_ERR_DTYPE;
    Flat fx, fq, fs;
    rn_status st = flatten(x, &fx);
    if (st != RN_OK) return st;
    if (fx.H % 2 != 0) return RN_ERR_SHAPE;
    const int64_t I = fx.H / 2;
    if ((st = flatten(q, &fq)) != RN_OK) return st;
    if (fq.H != I || fq.T != fx.T) return RN_ERR_SHAPE;
    if (fx.T == 0) return RN_OK;
    if ((st = flatten(scale, &fs)) != RN_OK) return st;
    if (fs.numel != fx.T) return RN_ERR_SHAPE;
    fs.esize = 4;
    if (!fx.ptr || !fq.ptr || !fs.ptr) return RN_ERR_NULL;
    if (!aligned(fx.ptr, 2) || !aligned(fs.ptr, 4)) return RN_ERR_LAYOUT;
    if (overlap(fq, fx) || overlap(fs, fx) || overlap(fq, fs)) return RN_ERR_ALIAS;
    const bool vector_ok = I % 8 == 0 && aligned(fx.ptr, 16) && aligned(fq.ptr, 8);
    rn_plan plan;
    // The row mapping of the fused norm ops on I-wide rows (rows per block as
    // for the fp8 op): per output element it moves 2 x 2 bytes in and 1 byte
    // out, within a few bytes of that op.
    const int sdt = x->dtype == RN_BF16 ? rn::kBF16 : rn::kF16;
    if ((st = plan_impl(rn::kSwigluFp8, sdt, fx.T, I, vector_ok, device_sms(), &plan, false)) !=
        RN_OK)
        return st;
    rn::SwigluArgs a{fx.ptr, reinterpret_cast<uint8_t*>(fq.ptr), reinterpret_cast<float*>(fs.ptr),
                     fx.T, I};
    rn::Launch l{plan.kernel == RN_KERNEL_VECTOR ? 0 : 1,
                 plan.threads_per_row,
                 plan.vectors_per_thread,
                 plan.rows_per_cta,
                 plan.block_threads,
                 plan.smem_bytes,
                 plan.grid,
                 g_pdl.load() < 0 ? kPdlDefault : g_pdl.load() == 1};
    // 32-byte pairs: an even vector count per thread, I % 16 == 0 (gate and up
    // rows then start 32-byte aligned), 32-byte aligned x and 16-byte aligned q
    l.pair = plan.kernel == RN_KERNEL_VECTOR && plan.vectors_per_thread % 2 == 0 && I % 16 == 0 &&
             aligned(fx.ptr, 32) && aligned(fq.ptr, 16);
    l.prefetch = g_prefetch.load() < 0 ? kPrefetchDefault : g_prefetch.load() == 1;
    const cudaError_t e = rn::launch_swiglu_fp8(x->dtype == RN_BF16 ? rn::kBF16 : rn::kF16, a, l,
                                                static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
        std::snprintf(g_cuda_error, sizeof g_cuda_error, "%s: %s", cudaGetErrorName(e),
                      cudaGetErrorString(e));
        return RN_ERR_CUDA;
    }
    return RN_OK;
}

rn_status rn_fp8_rowwise_gemm(const rn_tensor* d, const rn_tensor* a, const rn_tensor* b,
                              const rn_tensor* a_scale, const rn_tensor* b_scale, void* stream) {
    if (!d || !a || !b || !a_scale || !b_scale) return RN_ERR_NULL;
    if (a->dtype != RN_E4M3 || b->dtype != RN_E4M3 || d->dtype != RN_BF16 ||
        a_scale->dtype != RN_F32 || b_scale->dtype != RN_F32)
        return RN_ERR_DTYPE;
    Flat fa, fb, fd, fsa, fsb;
    rn_status st;
    if ((st = flatten(a, &fa)) != RN_OK) return st;
    if ((st = flatten(b, &fb)) != RN_OK) return st;
    if ((st = flatten(d, &fd)) != RN_OK) return st;
    const int64_t M = fa.T, K = fa.H, N = fb.T;
    if (fb.H != K || fd.T != M || fd.H != N || N == 0) return RN_ERR_SHAPE;
    if (K % 16 != 0 || N % 8 != 0) return RN_ERR_SHAPE;
    const int64_t kMax = 0x7fffffffLL;
    if (M > kMax || N > kMax || K > kMax) return RN_ERR_SHAPE;
    if ((st = flatten(b_scale, &fsb)) != RN_OK) return st;
    if (fsb.numel != N) return RN_ERR_SHAPE;
    if (M == 0) return RN_OK;
    if ((st = flatten(a_scale, &fsa)) != RN_OK) return st;
    if (fsa.numel != M) return RN_ERR_SHAPE;
    if (!fa.ptr || !fb.ptr || !fd.ptr || !fsa.ptr || !fsb.ptr) return RN_ERR_NULL;
    if (!aligned(fa.ptr, 16) || !aligned(fb.ptr, 16) || !aligned(fd.ptr, 16) ||
        !aligned(fsa.ptr, 4) || !aligned(fsb.ptr, 4))
        return RN_ERR_LAYOUT;
    if (overlap(fd, fa) || overlap(fd, fb) || overlap(fd, fsa) || overlap(fd, fsb))
        return RN_ERR_ALIAS;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) {
        rn::GemmArgs g{fa.ptr, fb.ptr, reinterpret_cast<const float*>(fsa.ptr),
                       reinterpret_cast<const float*>(fsb.ptr), fd.ptr, M, N, K, dev,
                       device_sms(), 0, false};
        g.config = gemm_config(M, N, g.num_sms);
        g.pdl = g_pdl.load() < 0 ? kPdlDefault : g_pdl.load() == 1;
        if (!current_context_id(&g.ctx_id)) g.ctx_id = 0;
        e = rn::launch_fp8_rowwise_gemm(g, static_cast<cudaStream_t>(stream));
    }
    if (e != cudaSuccess) {
        std::snprintf(g_cuda_error, sizeof g_cuda_error, "%s: %s", cudaGetErrorName(e),
                      cudaGetErrorString(e));
        return RN_ERR_CUDA;
    }
    return RN_OK;
}

// ---- tensor-parallel all-reduce fused ops

}  // extern "C"

namespace {

constexpr long long kArDefaultTimeoutNs = 1000000000LL;  // 1 s
constexpr int64_t kArMaxH = static_cast<int64_t>(rn::kArMaxBlock) * 8 * 8;

bool overlaps_bytes(const Flat& f, const void* p, int64_t bytes) {
    if (!f.ptr || f.numel == 0 || !p || bytes <= 0) return false;
    const auto a0 = reinterpret_cast<uintptr_t>(f.ptr);
    const auto a1 = a0 + static_cast<uintptr_t>(f.bytes());
    const auto b0 = reinterpret_cast<uintptr_t>(p);
    const auto b1 = b0 + static_cast<uintptr_t>(bytes);
    return a0 < b1 && b0 < a1;
}

// Row mapping of the all-reduce kernel: a power-of-two group of threads per
// row holding two 16-byte vectors each (up to the 512-thread block, then 4 or
// 8), 256-thread blocks of several rows for narrow rows. Measured on B200 for
// H = 3840 and 2, 4 and 8 ranks at T = 8192, two vectors per thread is the
// fastest of 1, 2, 4 and 8 for both algorithms (by 3 to 35 %): fewer leave too
// few loads in flight, more cost resident warps.
rn_status ar_shape(int64_t H, rn::ArLaunch* l) {
    const int64_t nvec = H / 8;
    int tpr = 1, vpt = 1;
    const int ftpr = g_force_tpr.load(), fvpt = g_force_vpt.load();
    if (ftpr > 0 && (ftpr & (ftpr - 1)) == 0 && ftpr <= rn::kArMaxBlock &&
        (fvpt == 1 || fvpt == 2 || fvpt == 4 || fvpt == 8) &&
        static_cast<int64_t>(ftpr) * fvpt >= nvec) {
        tpr = ftpr;  // a forced vector-kernel shape that suits this kernel too
        vpt = fvpt;
    } else {
        const int target = 2;
        while (static_cast<int64_t>(tpr) * target < nvec && tpr < rn::kArMaxBlock) tpr *= 2;
        const int64_t need = (nvec + tpr - 1) / tpr;
        while (vpt < need) vpt *= 2;
        if (vpt > 8) return RN_ERR_SHAPE;
    }
    l->tpr = tpr;
    l->vpt = vpt;
    l->rpc = tpr >= 256 ? 1 : 256 / tpr;
    l->block = tpr * l->rpc;
    l->smem = static_cast<int>(2 * l->rpc * (tpr >= 64 ? tpr / 32 : 1) * sizeof(float) * 2);
    return RN_OK;
}

// Automatic choice of the two-shot algorithm: each rank reads (W - 1) * 2TH
// bytes from its peers in one-shot and (W - 1) / W * 6TH in two-shot (its
// slice's partials, then the other slices' finished residual and output rows),
// at the cost of a second exchange barrier (a few microseconds). Two-shot is
// taken from four ranks on, once it saves at least 2.3 MB of peer reads per
// rank: about 3 us at the 770 GB/s a B200 peer copy reaches over NVLink.
// Rows from which groups of three to eight ranks run the all-reduce kernel
// held to 80 registers (allreduce_kernels.cu, rn_allreduce_wide_kernel), by
// algorithm. Measured on one device (H = 3840, 4 and 8 ranks, both outputs):
// one-shot gains 2-31 % from 256 rows on and loses up to 10 % at 64; two-shot
// loses 2-12 % up to 512 rows, breaks even at 1024 and gains 7-15 % from 2048.
constexpr int64_t kArWideRowsOneShot = 256;
constexpr int64_t kArWideRowsTwoShot = 2048;

bool ar_two_shot_pays(int W, int64_t T, int64_t H) {
    if (W < 4) return false;
    const double th = static_cast<double>(T) * static_cast<double>(H);
    const double saved = (W - 1) * 2.0 * th - (W - 1) * 6.0 * th / W;
    return saved >= 2.3e6;
}

rn_status check_comm(const rn_allreduce_comm* comm) {
    if (comm->world < 1 || comm->world > RN_ALLREDUCE_MAX_WORLD) return RN_ERR_COMM;
    if (comm->rank < 0 || comm->rank >= comm->world) return RN_ERR_COMM;
    if (!(comm->local_ranks == 1 || (comm->local_ranks == comm->world && comm->rank == 0)))
        return RN_ERR_COMM;
    for (int p = 0; p < comm->world; ++p) {
        if (!comm->buffers[p] || !comm->signals[p]) return RN_ERR_COMM;
        if (!aligned(comm->buffers[p], 16) || !aligned(comm->signals[p], 16)) return RN_ERR_COMM;
    }
    return RN_OK;
}

rn_status run_allreduce(bool fp8, const rn_tensor* o, const rn_tensor* sc, const rn_tensor* x,
                        const rn_tensor* r, const rn_tensor* w, float eps,
                        const rn_allreduce_comm* comm, void* stream) {
    const int op = fp8 ? rn::kFusedAddFp8 : rn::kFusedAdd;
    if (!comm) return RN_ERR_NULL;
    Common c;
    rn_status st = check_descriptors(op, o, sc, x, r, w, eps, -1, &c);
    if (st != RN_OK) return st;
    if ((st = check_comm(comm)) != RN_OK) return st;
    const int L = comm->local_ranks;
    if (c.x.T % L != 0) return RN_ERR_SHAPE;
    const int64_t T = c.x.T / L, H = c.x.H;
    if (H % 8 != 0) return RN_ERR_LAYOUT;
    if (H > kArMaxH) return RN_ERR_SHAPE;
    const int64_t slot_bytes = (comm->buffer_bytes / 2) & ~static_cast<int64_t>(15);
    if (comm->buffer_bytes < 0 || slot_bytes < 2 * T * H) return RN_ERR_COMM;
    if (comm->algorithm < RN_ALLREDUCE_AUTO || comm->algorithm > RN_ALLREDUCE_TWO_SHOT)
        return RN_ERR_COMM;
    const bool two_shot_fits = comm->world >= 3 && slot_bytes >= 6 * T * H;
    if (comm->algorithm == RN_ALLREDUCE_TWO_SHOT && !two_shot_fits) return RN_ERR_COMM;
    rn::ArLaunch l;
    if ((st = ar_shape(H, &l)) != RN_OK) return st;
    l.two_shot = comm->algorithm == RN_ALLREDUCE_TWO_SHOT ||
                 (comm->algorithm == RN_ALLREDUCE_AUTO && two_shot_fits &&
                  ar_two_shot_pays(comm->world, T, H));
    if (T > 0) {
        rn_plan unused;
        if ((st = check_pointers_and_plan(op, c, device_sms(), &unused)) != RN_OK) return st;
        if (!aligned(c.x.ptr, 16) || !aligned(c.res.ptr, 16) ||
            (c.has_w && !aligned(c.w.ptr, 16)) || (!fp8 && !aligned(c.out.ptr, 16)) ||
            (fp8 && !aligned(c.q.ptr, 8)))
            return RN_ERR_LAYOUT;
        for (int i = 0; i < L; ++i) {
            const void* buf = comm->buffers[comm->rank + i];
            const void* pad = comm->signals[comm->rank + i];
            for (const Flat* f : {&c.x, &c.res, &c.out, &c.q, &c.scale, &c.w})
                if (overlaps_bytes(*f, buf, comm->buffer_bytes) ||
                    overlaps_bytes(*f, pad, rn::kArSignalBytes))
                    return RN_ERR_ALIAS;
        }
    }
    rn::ArArgs a = {};
    a.world = comm->world;
    a.rank = comm->rank;
    for (int p = 0; p < comm->world; ++p) {
        a.buffers[p] = comm->buffers[p];
        a.signals[p] = static_cast<uint32_t*>(comm->signals[p]);
    }
    a.slot_elems = slot_bytes / 2;
    a.timeout_ns = comm->timeout_ns > 0 ? comm->timeout_ns : kArDefaultTimeoutNs;
    a.x = c.x.ptr;
    a.residual = c.res.ptr;
    a.weight = c.has_w ? c.w.ptr : nullptr;
    a.out = c.out.ptr;
    a.q = reinterpret_cast<uint8_t*>(c.q.ptr);
    a.scale = reinterpret_cast<float*>(c.scale.ptr);
    a.T = T;
    a.H = H;
    a.eps = eps;
    l.local_ranks = L;
    l.wide = comm->world >= 3 && T >= (l.two_shot ? kArWideRowsTwoShot : kArWideRowsOneShot);
    int per_sm = 0;
    cudaError_t e = rn::allreduce_blocks_per_sm(c.dt, fp8, comm->world, l, &per_sm);
    if (e == cudaSuccess) {
        const int64_t resident = static_cast<int64_t>(per_sm) * device_sms() / L;
        const int64_t groups = T > 0 ? (T + l.rpc - 1) / l.rpc : 1;
        int64_t g = groups < resident ? groups : resident;
        if (g > rn::kArMaxBlocks) g = rn::kArMaxBlocks;
        if (g < 1) return RN_ERR_CONFIG;
        l.grid_x = static_cast<int>(g);
        e = rn::launch_allreduce(c.dt, fp8, a, l, static_cast<cudaStream_t>(stream));
    }
    if (e != cudaSuccess) {
        std::snprintf(g_cuda_error, sizeof g_cuda_error, "%s: %s", cudaGetErrorName(e),
                      cudaGetErrorString(e));
        return RN_ERR_CUDA;
    }
    return RN_OK;
}

// Per device: the address of the library's static exchange memory and the
// group size its signal pads were last prepared for.
struct LocalGroup {
    void* base = nullptr;
    int world = 0;
    unsigned long long ctx_id = 0;  // the context `base` belongs to
};
constexpr int kMaxDevices = 64;
LocalGroup g_local[kMaxDevices];
std::mutex g_local_mu;

// The unique id of the calling thread's current CUDA context, through the
// driver entry points the runtime hands out (the library does not link the
// driver library itself, so it still loads on machines without a GPU).
bool current_context_id(unsigned long long* id) {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(f);
        f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(f);
    });
    CUcontext ctx = nullptr;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

rn_status local_cuda_error(cudaError_t e) {
    std::snprintf(g_cuda_error, sizeof g_cuda_error, "%s: %s", cudaGetErrorName(e),
                  cudaGetErrorString(e));
    return RN_ERR_CUDA;
}

// ---- activations in host memory (rn_host_*) ------------------------------
//
// Chunk c of the rows goes to stream c % n and to slot c % n of the scratch:
// copy in, one launch of the device kernel on the slot, copy out, all on
// that stream. A slot is reused only by a later chunk of the same stream, so
// stream order alone keeps a slot's copy out before the next chunk's copy in.

constexpr int64_t kHostAlign = 256;
// x bytes per chunk copy, at least: on B200 over PCIe 5, 5 MB chunks ran the
// prefill step 7 % slower than 8-10 MB chunks, 2 MB chunks 16 % slower
constexpr int64_t kHostMinCopyBytes = int64_t{8} << 20;

// Byte offsets of the regions of one slot of `rows` rows.
struct HostSlot {
    int64_t x = 0, r = 0, q = 0, s = 0, bytes = 0;
};

HostSlot host_slot(int op, int64_t rows, int64_t H) {
    HostSlot l;
    int64_t off = round_up(rows * H * 2, kHostAlign);  // x, and the 16-bit out in place
    if (op != rn::kRmsNorm) {
        l.r = off;
        off += round_up(rows * H * 2, kHostAlign);
    }
    if (op == rn::kFusedAddFp8) {
        l.q = off;
        off += round_up(rows * H, kHostAlign);
        l.s = off;
        off += round_up(rows * 4, kHostAlign);
    }
    l.bytes = off;
    return l;
}

// The most rows of which `slots` slots fit in `bytes` (0 if not one).
int64_t host_rows_fitting(int op, int64_t H, int64_t bytes, int64_t slots) {
    // capped so that the byte counts below cannot overflow
    const int64_t per_slot = std::min<int64_t>(bytes / slots, int64_t{1} << 60);
    const int64_t per_row = 2 * H + (op != rn::kRmsNorm ? 2 * H : 0) +
                            (op == rn::kFusedAddFp8 ? H + 4 : 0);
    int64_t rows = per_slot / per_row;
    while (rows > 0 && host_slot(op, rows, H).bytes > per_slot) --rows;
    return rows;
}

rn_status host_plan(int op, int64_t T, int64_t H, int64_t scratch_bytes, int n_streams,
                    int64_t want_rows, rn_host_plan* p) {
    std::memset(p, 0, sizeof *p);
    if (op < rn::kRmsNorm || op > rn::kFusedAddFp8) return RN_ERR_CONFIG;
    if (n_streams < 1 || n_streams > RN_HOST_MAX_STREAMS) return RN_ERR_CONFIG;
    if (T < 0 || H < 1) return RN_ERR_SHAPE;
    // keeps every byte count below 2^62
    if (H > (int64_t{1} << 40) || static_cast<double>(T) * static_cast<double>(H) > 1e17)
        return RN_ERR_SHAPE;
    if (T == 0) return RN_OK;
    if (scratch_bytes < 0) scratch_bytes = 0;
    int64_t rows;
    if (want_rows > 0) {
        rows = want_rows < T ? want_rows : T;
    } else {
        const int64_t n = n_streams;
        rows = (T + 4 * n - 1) / (4 * n);
        const int64_t min_rows = (kHostMinCopyBytes + 2 * H - 1) / (2 * H);
        if (rows < min_rows) rows = min_rows;
        if (rows > T) rows = T;
        const int64_t fit = host_rows_fitting(op, H, scratch_bytes, n);
        if (fit < 1) return RN_ERR_CAPACITY;
        if (rows > fit) rows = fit;
    }
    const int64_t chunks = (T + rows - 1) / rows;
    const int64_t slots = chunks < n_streams ? chunks : n_streams;
    const int64_t slot_bytes = host_slot(op, rows, H).bytes;
    if (slot_bytes > scratch_bytes / slots) return RN_ERR_CAPACITY;
    p->chunk_rows = rows;
    p->chunks = chunks;
    p->slot_bytes = slot_bytes;
    p->slots = static_cast<int32_t>(slots);
    return RN_OK;
}

rn_status run_host(int op, const rn_tensor* o, const rn_tensor* sc, const rn_tensor* x,
                   const rn_tensor* r, const rn_tensor* w, float eps, int64_t variance_size,
                   const rn_host_pipeline* hp) {
    Common c;
    rn_status st = check_descriptors(op, o, sc, x, r, w, eps, variance_size, &c);
    if (st != RN_OK) return st;
    if (!hp) return RN_ERR_NULL;
    if (hp->n_streams < 1 || hp->n_streams > RN_HOST_MAX_STREAMS || hp->reserved != 0)
        return RN_ERR_CONFIG;
    if (!hp->streams) return RN_ERR_NULL;
    if (c.x.T == 0) return RN_OK;
    rn_plan whole;  // the whole-problem plan is not used: each chunk is planned
    st = check_pointers_and_plan(op, c, kDefaultSms, &whole);
    if (st != RN_OK) return st;
    if (!hp->scratch) return RN_ERR_NULL;
    if (!aligned(hp->scratch, kHostAlign)) return RN_ERR_LAYOUT;
    rn_host_plan hpl;
    st = host_plan(op, c.x.T, c.x.H, hp->scratch_bytes, hp->n_streams, hp->chunk_rows, &hpl);
    if (st != RN_OK) return st;
    Flat used;
    used.ptr = static_cast<char*>(hp->scratch);
    used.numel = hpl.slots * hpl.slot_bytes;
    used.esize = 1;
    for (const Flat* f : {&c.x, &c.out, &c.res, &c.q, &c.scale, &c.w})
        if (f->ptr && overlap(used, *f)) return RN_ERR_ALIAS;
    // The kernels dereference the scratch and the weight: both must be device
    // memory (a host weight is the likely mistake with these entry points).
    for (const void* d : {static_cast<const void*>(hp->scratch),
                          static_cast<const void*>(c.has_w ? c.w.ptr : nullptr)}) {
        if (!d) continue;
        cudaPointerAttributes attr;
        const cudaError_t e = cudaPointerGetAttributes(&attr, d);
        if (e != cudaSuccess) return local_cuda_error(e);
        if (attr.type != cudaMemoryTypeDevice && attr.type != cudaMemoryTypeManaged)
            return RN_ERR_LAYOUT;
    }

    const int64_t T = c.x.T, H = c.x.H;
    const bool fused = op != rn::kRmsNorm, fp8 = op == rn::kFusedAddFp8;
    const bool vector_ok = H % 8 == 0 && (!c.has_w || aligned(c.w.ptr, 16));
    const int num_sms = device_sms();
    const HostSlot L = host_slot(op, hpl.chunk_rows, H);
    for (int64_t k = 0; k < hpl.chunks; ++k) {
        const int64_t t0 = k * hpl.chunk_rows;
        const int64_t rows = T - t0 < hpl.chunk_rows ? T - t0 : hpl.chunk_rows;
        const int slot = static_cast<int>(k % hpl.slots);
        char* base = static_cast<char*>(hp->scratch) + slot * hpl.slot_bytes;
        cudaStream_t s = static_cast<cudaStream_t>(hp->streams[slot]);
        const int64_t b16 = rows * H * 2, off16 = t0 * H * 2;
        cudaError_t e = cudaMemcpyAsync(base + L.x, c.x.ptr + off16, b16, cudaMemcpyDefault, s);
        if (e == cudaSuccess && fused)
            e = cudaMemcpyAsync(base + L.r, c.res.ptr + off16, b16, cudaMemcpyDefault, s);
        if (e != cudaSuccess) return local_cuda_error(e);

        rn::Args a;
        a.x = base + L.x;
        a.residual = fused ? base + L.r : nullptr;
        a.weight = c.has_w ? c.w.ptr : nullptr;
        a.out = fp8 ? nullptr : base + L.x;  // in place over the slot's x
        a.q = fp8 ? reinterpret_cast<uint8_t*>(base + L.q) : nullptr;
        a.scale = fp8 ? reinterpret_cast<float*>(base + L.s) : nullptr;
        a.T = rows;
        a.H = H;
        a.eps = eps;
        rn_plan plan;
        st = plan_impl(op, c.dt, rows, H, vector_ok, num_sms, &plan);
        if (st != RN_OK) return st;
        // no programmatic dependent launch: the kernel follows copies
        st = launch_plan(op, c.dt, a, plan, false, pair_ok(op, H, a.x, a.residual, a.out, a.q),
                         s);
        if (st != RN_OK) return st;

        if (fused) e = cudaMemcpyAsync(c.res.ptr + off16, base + L.r, b16, cudaMemcpyDefault, s);
        if (e == cudaSuccess && !fp8)
            e = cudaMemcpyAsync(c.out.ptr + off16, base + L.x, b16, cudaMemcpyDefault, s);
        if (e == cudaSuccess && fp8)
            e = cudaMemcpyAsync(c.q.ptr + t0 * H, base + L.q, rows * H, cudaMemcpyDefault, s);
        if (e == cudaSuccess && fp8)
            e = cudaMemcpyAsync(c.scale.ptr + t0 * 4, base + L.s, rows * 4, cudaMemcpyDefault, s);
        if (e != cudaSuccess) return local_cuda_error(e);
    }
    return RN_OK;
}

}  // namespace

extern "C" {

rn_status rn_allreduce_fused_add_rms_norm_local(const rn_tensor* out, const rn_tensor* x,
                                                const rn_tensor* residual,
                                                const rn_tensor* weight, float eps,
                                                int32_t world, void* stream) {
    if (world < 1 || world > rn::kArMaxWorld) return RN_ERR_COMM;
    Common c;
    rn_status st = check_descriptors(rn::kFusedAdd, out, nullptr, x, residual, weight, eps, -1, &c);
    if (st != RN_OK) return st;
    if (c.x.T % world != 0) return RN_ERR_SHAPE;
    const int64_t T = c.x.T / world, H = c.x.H;
    // Two buffer halves of T*H 16-bit values each (one-shot); from three
    // ranks on, halves of 3*T*H values (room for two-shot) when the static
    // memory holds them.
    const int64_t one_shot_bytes = ((4 * T * H + 32 + 255) / 256) * 256;
    int64_t buffer_bytes = one_shot_bytes;
    if (world >= 3) {
        const int64_t two_shot_bytes = ((12 * T * H + 32 + 255) / 256) * 256;
        if (two_shot_bytes * world <= rn::kLocalBufferBytes) buffer_bytes = two_shot_bytes;
    }
    if (buffer_bytes * world > rn::kLocalBufferBytes) return RN_ERR_CAPACITY;

    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return local_cuda_error(e);
    if (dev < 0 || dev >= kMaxDevices) return RN_ERR_CONFIG;
    const auto s = static_cast<cudaStream_t>(stream);
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    e = cudaStreamIsCapturing(s, &cs);
    if (e != cudaSuccess) return local_cuda_error(e);
    // The static array's address is valid for the context it was looked up
    // in; a context created after a device reset reloads the library's
    // device code, so the lookup and the pad clearing are redone.
    unsigned long long ctx_id = 0;
    if (!current_context_id(&ctx_id)) return local_cuda_error(cudaErrorDeviceUninitialized);
    rn_allreduce_comm comm = {};
    {
        std::lock_guard<std::mutex> lock(g_local_mu);
        LocalGroup& g = g_local[dev];
        if (g.base && g.ctx_id != ctx_id) {
            g.base = nullptr;
            g.world = 0;
        }
        if (!g.base || g.world != world) {
            // first use in this context or a new group size: the setup
            // (symbol lookup, clearing the pads on `stream`) must not be
            // captured
            if (cs != cudaStreamCaptureStatusNone) return RN_ERR_CONFIG;
        }
        if (!g.base) {
            void* p = nullptr;
            e = rn::local_scratch_address(&p);  // the current device is `dev`
            if (e != cudaSuccess) return local_cuda_error(e);
            g.base = p;
            g.ctx_id = ctx_id;
        }
        if (g.world != world) {
            e = cudaMemsetAsync(g.base, 0, rn::kLocalPadStride * rn::kArMaxWorld, s);
            if (e != cudaSuccess) return local_cuda_error(e);
            g.world = world;
        }
        char* base = static_cast<char*>(g.base);
        comm.world = world;
        comm.rank = 0;
        comm.local_ranks = world;
        for (int p = 0; p < world; ++p) {
            comm.signals[p] = base + p * rn::kLocalPadStride;
            comm.buffers[p] = base + rn::kLocalPadStride * rn::kArMaxWorld + p * buffer_bytes;
        }
        comm.buffer_bytes = buffer_bytes;
        comm.timeout_ns = 0;
        comm.algorithm = RN_ALLREDUCE_AUTO;
    }
    return run_allreduce(false, out, nullptr, x, residual, weight, eps, &comm, stream);
}

rn_status rn_allreduce_fused_add_rms_norm(const rn_tensor* out, const rn_tensor* x,
                                          const rn_tensor* residual, const rn_tensor* weight,
                                          float eps, const rn_allreduce_comm* comm,
                                          void* stream) {
    return run_allreduce(false, out, nullptr, x, residual, weight, eps, comm, stream);
}

rn_status rn_allreduce_fused_add_rms_norm_fp8(const rn_tensor* q, const rn_tensor* scale,
                                              const rn_tensor* x, const rn_tensor* residual,
                                              const rn_tensor* weight, float eps,
                                              const rn_allreduce_comm* comm, void* stream) {
    return run_allreduce(true, q, scale, x, residual, weight, eps, comm, stream);
}

rn_status rn_validate(int32_t op, const rn_tensor* out_or_q, const rn_tensor* scale,
                      const rn_tensor* x, const rn_tensor* residual, const rn_tensor* weight,
                      float eps, int64_t variance_size, rn_plan* plan) {
    if (op < 0 || op > 2) return RN_ERR_CONFIG;
    Common c;
    rn_plan local;
    bool launch_needed;
    rn_status st = prepare(op, out_or_q, scale, x, residual, weight, eps, variance_size,
                           kDefaultSms, &c, plan ? plan : &local, &launch_needed);
    return st;
}

const char* rn_status_string(rn_status s) {
    switch (s) {
        case RN_OK: return "ok";
        case RN_ERR_NULL: return "a required pointer is NULL";
        case RN_ERR_DTYPE: return "unsupported or mismatched dtype";
        case RN_ERR_WEIGHT_DTYPE: return "weight dtype differs from the activation dtype";
        case RN_ERR_SHAPE: return "bad shape (ndim, H == 0, mismatched [T x H], weight or scale size)";
        case RN_ERR_LAYOUT: return "not a dense unit-stride 2-D view, or misaligned pointer";
        case RN_ERR_ALIAS: return "forbidden overlap between operands";
        case RN_ERR_VARIANCE_SIZE: return "variance_size override is not supported";
        case RN_ERR_EPS: return "eps must be finite and >= 0";
        case RN_ERR_CUDA: return "CUDA error (see rn_last_cuda_error)";
        case RN_ERR_CONFIG: return "unsupported configuration (tuning request, op or stream count)";
        case RN_ERR_COMM: return "bad all-reduce group description or exchange buffers too small";
        case RN_ERR_CAPACITY: return "problem larger than the static exchange memory or the scratch";
    }
    return "unknown status";
}

const char* rn_last_cuda_error(void) { return g_cuda_error; }

rn_status rn_plan_launch(int32_t op, int32_t dtype, int64_t T, int64_t H, int32_t vector_ok,
                         rn_plan* plan) {
    if (!plan) return RN_ERR_NULL;
    if (op < 0 || op > 3) return RN_ERR_CONFIG;
    if (!is16(dtype)) return RN_ERR_DTYPE;
    const int dt = dtype == RN_BF16 ? rn::kBF16 : rn::kF16;
    if (op == RN_OP_SILU_AND_MUL_FP8)
        return plan_impl(rn::kSwigluFp8, dt, T, H, vector_ok != 0, kDefaultSms, plan, false);
    return plan_impl(op, dt, T, H, vector_ok != 0, kDefaultSms, plan);
}

rn_status rn_force_staged(int32_t ctas_per_sm, int32_t stages, int32_t threads) {
    if (ctas_per_sm == 0 && stages == 0 && threads == 0) {
        g_force_staged_c.store(0);
        g_force_staged_s.store(0);
        g_force_staged_t.store(0);
        return RN_OK;
    }
    if (!(ctas_per_sm == 1 || ctas_per_sm == 2 || ctas_per_sm == 4) || stages < 2 ||
        stages > 64 || threads < 32 || threads > 1024 || threads % 32)
        return RN_ERR_CONFIG;
    g_force_staged_s.store(stages);
    g_force_staged_t.store(threads);
    g_force_staged_c.store(ctas_per_sm);
    return RN_OK;
}

rn_status rn_set_launch_options(int32_t pdl, int64_t max_grid) {
    if (pdl < -1 || pdl > 1 || max_grid < 0) return RN_ERR_CONFIG;
    g_pdl.store(pdl);
    g_max_grid.store(max_grid);
    return RN_OK;
}

rn_status rn_kernel_binary_version(int32_t* version) {
    if (!version) return RN_ERR_NULL;
    int v = 0;
    const cudaError_t e = rn::kernel_binary_version(&v);
    if (e != cudaSuccess) {
        std::snprintf(g_cuda_error, sizeof g_cuda_error, "%s: %s", cudaGetErrorName(e),
                      cudaGetErrorString(e));
        return RN_ERR_CUDA;
    }
    *version = v;
    return RN_OK;
}

rn_status rn_set_prefetch(int32_t mode) {
    if (mode < -1 || mode > 1) return RN_ERR_CONFIG;
    g_prefetch.store(mode);
    return RN_OK;
}

rn_status rn_device_errors(uint32_t* flags) {
    if (!flags) return RN_ERR_NULL;
    unsigned v = 0, v_ar = 0;
    cudaError_t e = rn::read_and_clear_device_errors(&v);
    if (e == cudaSuccess) e = rn::read_and_clear_allreduce_errors(&v_ar);
    v |= v_ar;
    if (e != cudaSuccess) {
        std::snprintf(g_cuda_error, sizeof g_cuda_error, "%s: %s", cudaGetErrorName(e),
                      cudaGetErrorString(e));
        return RN_ERR_CUDA;
    }
    *flags = v;
    return RN_OK;
}

rn_status rn_force_plan(int32_t threads_per_row, int32_t vectors_per_thread,
                        int32_t rows_per_cta) {
    if (threads_per_row == 0 && vectors_per_thread == 0) {
        g_force_tpr.store(0);
        g_force_vpt.store(0);
        g_force_rpc.store(0);
        return RN_OK;
    }
    if (!tpr_valid(threads_per_row) || !vpt_compiled(vectors_per_thread) || rows_per_cta < 0 ||
        rows_per_cta > 1024)
        return RN_ERR_CONFIG;
    g_force_rpc.store(rows_per_cta);
    g_force_vpt.store(vectors_per_thread);
    g_force_tpr.store(threads_per_row);
    return RN_OK;
}

int32_t rn_supported_vectors_per_thread(int32_t* out, int32_t cap) {
    for (int i = 0; i < rn::kNumVpt && i < cap; ++i) out[i] = rn::kVptList[i];
    return rn::kNumVpt;
}

rn_status rn_fp8_gemm_config(int64_t M, int64_t N, int64_t K, int32_t num_sms,
                             int32_t* config) {
    if (!config) return RN_ERR_NULL;
    if (M < 0 || N < 1 || K < 1) return RN_ERR_SHAPE;
    *config = gemm_config(M, N, num_sms > 0 ? num_sms : kDefaultSms);
    return RN_OK;
}

rn_status rn_fp8_gemm_force_config(int32_t config) {
    if (config < -1 || config >= rn::kNumGemmConfigs) return RN_ERR_CONFIG;
    g_force_gemm.store(config);
    return RN_OK;
}

rn_status rn_host_plan_chunks(int32_t op, int64_t T, int64_t H, int64_t scratch_bytes,
                              int32_t n_streams, int64_t chunk_rows, rn_host_plan* plan) {
    if (!plan) return RN_ERR_NULL;
    return host_plan(op, T, H, scratch_bytes, n_streams, chunk_rows, plan);
}

rn_status rn_host_rms_norm(const rn_tensor* out, const rn_tensor* x, const rn_tensor* weight,
                           float eps, int64_t variance_size, const rn_host_pipeline* pipeline) {
    return run_host(rn::kRmsNorm, out, nullptr, x, nullptr, weight, eps, variance_size,
                    pipeline);
}

rn_status rn_host_fused_add_rms_norm(const rn_tensor* out, const rn_tensor* x,
                                     const rn_tensor* residual, const rn_tensor* weight,
                                     float eps, int64_t variance_size,
                                     const rn_host_pipeline* pipeline) {
    return run_host(rn::kFusedAdd, out, nullptr, x, residual, weight, eps, variance_size,
                    pipeline);
}

rn_status rn_host_fused_add_rms_norm_fp8(const rn_tensor* q, const rn_tensor* scale,
                                         const rn_tensor* x, const rn_tensor* residual,
                                         const rn_tensor* weight, float eps,
                                         int64_t variance_size,
                                         const rn_host_pipeline* pipeline) {
    return run_host(rn::kFusedAddFp8, q, scale, x, residual, weight, eps, variance_size,
                    pipeline);
}

const char* rn_version(void) { return "0.4.0"; }

}  // extern "C"
