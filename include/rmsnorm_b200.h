/*
 * rmsnorm_b200.h -- C ABI of the B200 (sm_100a) RMSNorm library.
 *
 * Three operators over a dense [T x H] matrix of 16-bit activations (fp16 or
 * bf16), each accumulating in fp32:
 *
 *   rn_rms_norm               out = x / sqrt(mean(x^2) + eps) * weight
 *   rn_fused_add_rms_norm     residual := x + residual (rounded to the 16-bit
 *                             dtype and written back), out = rms_norm(residual)
 *   rn_fused_add_rms_norm_fp8 the fused pass with a per-token dynamic cast to
 *                             OCP FP8 e4m3fn instead of a 16-bit output
 *
 * Sources. The operators and their eligibility rules are those of the AITER
 * wrappers in "vllm.kernels.aiter_ops": rms_no_var_16bit_only and
 * rms_add_no_var_16bit_only accept only fp16/bf16 activations, a weight of the
 * same dtype or None, no variance-size override, and inputs whose flattening
 * to 2-D is free (flatten_to_2d_is_free). The single-pass residual + RMSNorm
 * + FP8 fusion is the first kernel of "Custom CUDA kernels juice Llama 3.1
 * 405B on AMD MI300X, skipping Nvidia lock-in". The pages name the operators
 * without writing the formula; the library computes textbook RMSNorm (eps
 * inside the square root, weight applied after normalising).
 *
 * Common conventions for every entry point:
 *
 *  - Memory. Every data pointer is a DEVICE pointer on the current CUDA
 *    device, except the activations of the rn_host_* entry points, which
 *    live in host memory. The caller owns and allocates all memory; the
 *    library allocates nothing and keeps no pointer after returning. Its
 *    only global state:
 *    the test and tuning overrides (rn_force_plan, rn_force_staged,
 *    rn_set_launch_options, rn_set_prefetch, rn_fp8_gemm_force_config), the
 *    thread-local error text, the device error flags (rn_device_errors), the
 *    static exchange memory of rn_allreduce_fused_add_rms_norm_local, and,
 *    per device, the id of the CUDA context in which each GEMM kernel's
 *    shared-memory limit was last set.
 *  - Views. A tensor is described by rn_tensor (pointer, dtype, sizes and
 *    strides in ELEMENTS). It must flatten to a dense [T x H] matrix for free:
 *    the last stride is 1 and each leading dimension of size != 1 has the
 *    stride equal to the product of the sizes after it. This is the
 *    flatten_to_2d_is_free rule of "vllm.kernels.aiter_ops", applied to 1-D
 *    and 2-D views as well (so padded 2-D rows are rejected too, matching the
 *    docstring's "dense 2D inputs" and its rejection of a strided last dim).
 *    H = sizes[ndim-1], T = numel / H. 1 <= ndim <= RN_MAX_DIMS.
 *  - weight. NULL (the descriptor pointer) means "no weight" (all ones);
 *    otherwise a 1-D view of H elements, stride 1, same dtype as x.
 *  - variance_size must be -1 (None); any other value is rejected with
 *    RN_ERR_VARIANCE_SIZE, as the AITER predicates reject an override.
 *  - eps must be finite and >= 0. The kernels use it as the given float.
 *  - Streams. Work is enqueued on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and the call returns without waiting. Validation errors
 *    return synchronously and launch nothing; a failed launch returns
 *    RN_ERR_CUDA (text in rn_last_cuda_error()).
 *  - T == 0 (with a valid H >= 1) is a no-op returning RN_OK; H == 0 is
 *    RN_ERR_SHAPE.
 *  - Aliasing. out may be exactly x (same pointer and extent: in place).
 *    Every other overlap between a written buffer (out, residual, q, scale)
 *    and any other operand is RN_ERR_ALIAS.
 *  - Alignment. Data pointers must be aligned to their element size
 *    (RN_ERR_LAYOUT otherwise). The fast vectorised kernels additionally need
 *    16-byte aligned 16-bit rows (H % 8 == 0 and 16-byte aligned bases) and an
 *    8-byte aligned q; other inputs run a correct scalar kernel. With
 *    H % 16 == 0, 32-byte aligned 16-bit bases and a 16-byte aligned q they
 *    move data with 32-byte accesses (faster; same results up to the order of
 *    the fp32 sum of squares).
 *  - Numerics (on the GPU): sum of squares in fp32, inv = 1 / sqrt(ss/H + eps)
 *    with IEEE sqrt and division, y = (v * w) * inv (the 16-bit product v * w
 *    is exact in fp32), one rounding to nearest-even to the output type.
 *    Squares or products beyond the fp32 range (|v| > ~1.8e19, bf16 only)
 *    are outside the supported input range.
 */
#ifndef RMSNORM_B200_H
#define RMSNORM_B200_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RN_MAX_DIMS 8

/* Exported symbols (the library is built with hidden default visibility). */
#if defined(__GNUC__)
#define RN_API __attribute__((visibility("default")))
#else
#define RN_API
#endif

typedef enum {
    RN_OK = 0,
    RN_ERR_NULL = 1,          /* a required descriptor, data, sizes or strides pointer is NULL */
    RN_ERR_DTYPE = 2,         /* x not fp16/bf16; out/residual dtype != x; q not E4M3; scale not F32 */
    RN_ERR_WEIGHT_DTYPE = 3,  /* weight dtype != x dtype */
    RN_ERR_SHAPE = 4,         /* bad ndim, negative size, H == 0, [T x H] mismatch, weight not [H], scale not [T] */
    RN_ERR_LAYOUT = 5,        /* flattening to dense 2-D is not free, or a pointer misaligned for its dtype */
    RN_ERR_ALIAS = 6,         /* forbidden overlap between operands */
    RN_ERR_VARIANCE_SIZE = 7, /* variance_size != -1 */
    RN_ERR_EPS = 8,           /* eps negative, NaN or infinite */
    RN_ERR_CUDA = 9,          /* a CUDA runtime call failed */
    RN_ERR_CONFIG = 10,       /* unsupported tuning request, op, or host-pipeline stream count */
    RN_ERR_COMM = 11,         /* all-reduce: bad group description or exchange buffers too small */
    RN_ERR_CAPACITY = 12      /* beyond the static exchange memory, or host-pipeline scratch too small */
} rn_status;

typedef enum {
    RN_F16 = 0,   /* IEEE binary16 */
    RN_BF16 = 1,  /* bfloat16 */
    RN_E4M3 = 2,  /* OCP FP8 e4m3fn (1 byte; largest finite 448; NaN = S.1111.111) */
    RN_F32 = 3    /* IEEE binary32 */
} rn_dtype;

/* A strided view of caller-owned device memory. Strides are in elements. */
typedef struct {
    void* data;
    int32_t dtype;          /* rn_dtype */
    int32_t ndim;           /* 1 .. RN_MAX_DIMS */
    const int64_t* sizes;   /* ndim entries, >= 0 */
    const int64_t* strides; /* ndim entries, in elements */
} rn_tensor;

/* rms_norm: out = RNE16(x / sqrt(mean(x^2) + eps) * weight), per row.
 * out, x: [T x H] fp16/bf16 (same dtype). weight: [H] or NULL.
 * "vllm.kernels.aiter_ops", rms_no_var_16bit_only. */
RN_API rn_status rn_rms_norm(const rn_tensor* out, const rn_tensor* x,
                      const rn_tensor* weight, float eps, int64_t variance_size,
                      void* stream);

/* fused_add_rms_norm: residual := RNE16(x + residual) (in place), then
 * out = RNE16(residual / sqrt(mean(residual^2) + eps) * weight), normalising
 * the rounded values that were written back.
 * out, x, residual: [T x H], same 16-bit dtype; residual is read and written.
 * "vllm.kernels.aiter_ops", rms_add_no_var_16bit_only. */
RN_API rn_status rn_fused_add_rms_norm(const rn_tensor* out, const rn_tensor* x,
                                const rn_tensor* residual, const rn_tensor* weight,
                                float eps, int64_t variance_size, void* stream);

/* fused_add_rms_norm_fp8: residual := RNE16(x + residual) (in place); per row
 * y = residual / sqrt(mean(residual^2) + eps) * weight (fp32, not rounded),
 * scale[t] = max|y| / 448 (fp32) and q = e4m3fn(round-to-nearest-even,
 * saturating to +-448)(y / scale). A row whose max|y| is 0 gets scale 0 and
 * all-zero codes. Dequantise with q * scale[t].
 * q: [T x H] RN_E4M3 (row-major, 1 byte per element). scale: T elements of
 * RN_F32 (any shape with numel T, dense). x, residual: as above.
 * The residual + RMSNorm + FP8 single pass of "Custom CUDA kernels juice
 * Llama 3.1 405B on AMD MI300X, skipping Nvidia lock-in". */
RN_API rn_status rn_fused_add_rms_norm_fp8(const rn_tensor* q, const rn_tensor* scale,
                                    const rn_tensor* x, const rn_tensor* residual,
                                    const rn_tensor* weight, float eps,
                                    int64_t variance_size, void* stream);

/* silu_and_mul_fp8: the fused SwiGLU + per-token dynamic FP8 cast, the
 * second kernel of "Custom CUDA kernels juice Llama 3.1 405B on AMD MI300X,
 * skipping Nvidia lock-in" ("the SwiGLU activation function, again merging
 * it with an FP8 cast"). Per row of x = [gate | up] ([T x 2I], fp16/bf16,
 * gate in the first half): y_i = silu(gate_i) * up_i with silu(a) =
 * a / (1 + e^-a) in fp32 (a base-2 exponential of an argument carried in two
 * floats and a reciprocal: relative error of y a few ulp, below 1e-6, for
 * any finite gate; silu(a) = 0 for a < -87.3, where its true magnitude is
 * below 1e-36), scale[t] = max|y| / 448, q = e4m3fn(RNE, satfinite)
 * (y / scale); a row with max|y| = 0 gets scale 0 and zero codes.
 * q: [T x I] RN_E4M3 dense; scale: T RN_F32 dense; x: any view whose flattening
 * to [T x 2I] is free (the rules of the norm ops). 2I must be even.
 * Validation, streams, aliasing (q and scale overlap nothing) and T == 0 as
 * for the norm ops. */
RN_API rn_status rn_silu_and_mul_fp8(const rn_tensor* q, const rn_tensor* scale,
                                     const rn_tensor* x, void* stream);

/* fp8_rowwise_gemm: D[m, n] = bf16(b_scale[n] * (a_scale[m] * sum_k A[m, k] *
 * B[n, k])), with fp32 accumulation on the tensor cores (tcgen05) and one
 * rounding to bf16. The consumer of fused_add_rms_norm_fp8's codes and
 * per-token scales: A is [M x K] e4m3 (row-major, as q), a_scale has M fp32
 * values (as scale), B is an [N x K] e4m3 weight (row-major: K contiguous)
 * with one fp32 scale per output channel in b_scale, and D is [M x N] bf16
 * row-major. Row-wise fp8 linear layers appear in the table of
 * "VLLM_ROCM_USE_AITER=1 slows Gemma 4 on an AMD MI300X"
 * (RowWiseTorchFP8ScaledMMLinearKernel).
 * Requirements: dense views (flattening rule of the norm ops), K % 16 == 0,
 * N % 8 == 0, 16-byte-aligned A, B and D, K, N and M below 2^31; D must not
 * overlap any input. M == 0 is a no-op. Needs no workspace. Asynchronous on
 * `stream`, with programmatic dependent launch as the other kernels
 * (rn_set_launch_options); validation errors return before any CUDA call.
 * The tile shape is chosen per call (rn_fp8_gemm_config). */
RN_API rn_status rn_fp8_rowwise_gemm(const rn_tensor* d, const rn_tensor* a,
                                     const rn_tensor* b, const rn_tensor* a_scale,
                                     const rn_tensor* b_scale, void* stream);

/* Tile configurations of rn_fp8_rowwise_gemm. TOK tiles put the tensor core's
 * MMA rows on tokens: (tokens x channels) = 128 x 128. CH tiles compute D^T =
 * B * A^T, putting the MMA rows on the weight's output channels: (channels x
 * tokens), for decode-sized M where 128 token rows would be mostly padding;
 * TOK128_CH256 is the token-major tile with 256 channels.
 * Every configuration computes the same values: the scales are applied in the
 * same order and the fp32 accumulation over K differs only in its order. */
typedef enum {
    RN_GEMM_TOK128_CH128 = 0,
    RN_GEMM_CH128_TOK16 = 1,
    RN_GEMM_CH128_TOK32 = 2,
    RN_GEMM_CH128_TOK64 = 3,
    RN_GEMM_CH64_TOK16 = 4,
    RN_GEMM_CH64_TOK32 = 5,
    RN_GEMM_CH64_TOK64 = 6,
    RN_GEMM_TOK128_CH256 = 7
} rn_gemm_config;

/* The configuration rn_fp8_rowwise_gemm uses for an M x N x K problem on a
 * device with `num_sms` SMs (<= 0: 148). Among the CH configurations, the one
 * with the most tiles (ceil(N / channels) * ceil(M / tokens)) not above
 * num_sms, ties going to fewer channels, then fewer tokens per tile; if none
 * fits, CH128 with the smallest token width >= M for M <= 64; above,
 * TOK128_CH256 when ceil(M / 128) * ceil(N / 256) >= num_sms, else
 * TOK128_CH128. Honours rn_fp8_gemm_force_config. Pure host logic. RN_ERR_SHAPE for
 * M < 0, N < 1 or K < 1. */
RN_API rn_status rn_fp8_gemm_config(int64_t M, int64_t N, int64_t K, int32_t num_sms,
                                    int32_t* config);

/* Test hook: force rn_gemm_config `config` for every later GEMM in the
 * process; -1 restores the automatic choice; other values RN_ERR_CONFIG. Not
 * thread-safe with concurrent launches; meant for tests and tuning. */
RN_API rn_status rn_fp8_gemm_force_config(int32_t config);

/* ---- tensor-parallel all-reduce fused with the residual add and RMSNorm --
 *
 * In a tensor-parallel decoder layer each rank's row-parallel linear layer
 * leaves a partial sum of the activations; an all-reduce adds the partials
 * before the residual add and RMSNorm (SGLang takes all-reduce and RMSNorm
 * from AITER: "AITER: AMD's operator library for ROCm", ecosystem section).
 * These entry points do all three in one kernel per call, on every rank:
 *   x = RNE16(sum over the ranks' partials), residual := RNE16(x + residual),
 *   then out = RNE16(rms_norm(residual) * w)   (rn_allreduce_fused_add_rms_norm)
 *   or q, scale as rn_fused_add_rms_norm_fp8   (rn_allreduce_fused_add_rms_norm_fp8).
 * Every rank obtains bit-identical results (the residual is replicated).
 * x is the correctly rounded sum of the partials whenever their binary64 sum
 * is exact: always for fp16, and for bf16 whenever an element's non-zero
 * partials span at most 42 binades; otherwise it can differ from it by one
 * unit in the last place.
 *
 * Exchange: one-shot over peer memory (NVLink/NVSwitch loads and stores, no
 * collective library). Every rank owns an exchange buffer and a signal pad
 * that every rank's device can address (CUDA IPC or any peer mapping); each
 * call copies the local partial into the rank's own buffer, publishes it
 * through the peers' signal pads, waits for all peers, then reads the W
 * partials. Every rank of the group must make the same sequence of calls,
 * with the same T, H, dtype and op, on the same device model, each call
 * enqueued after the previous one on one stream per rank.
 *
 * Operands are those of rn_fused_add_rms_norm(_fp8), with `x` the local
 * partial; when one call computes several ranks (local_ranks > 1), x,
 * residual, out and q carry a leading rank dimension ([local_ranks, T, H] or
 * any dense view flattening to [local_ranks * T, H]) and scale holds
 * local_ranks * T values. Requirements beyond those of the fused ops: H a
 * multiple of 8 and at most 32768, x, residual, out, weight, buffers and
 * signal pads 16-byte aligned, q 8-byte aligned. out == x (in place) is
 * allowed. T == 0 still performs the exchange handshake (so that the ranks'
 * call counters stay equal) and writes nothing. */
#define RN_ALLREDUCE_MAX_WORLD 8
/* Signal pad bytes per rank: a 64-byte header (the rank's call counter and an
 * arrival counter, kept by the kernel) and 2 parities x 2 stages x 1024
 * blocks x 8 ranks 32-bit flags. */
#define RN_ALLREDUCE_SIGNAL_BYTES 131136

/* Exchange algorithms. ONE_SHOT: every rank reads every row of every peer's
 * partial ((W - 1) * 2 * T * H bytes of peer reads per rank). TWO_SHOT (3 to 8
 * ranks): rank q reduces and finishes the rows [q * S, (q + 1) * S), S =
 * ceil(T / W), writes them to its buffer, and every rank copies the other
 * slices' finished rows ((W - 1) / W * 6 * T * H bytes per rank, a second
 * exchange barrier, buffers of 12 * T * H + 32 bytes). AUTO takes two-shot
 * when the buffers hold it, W >= 4 and it saves at least 2.3 MB of peer reads
 * per rank; both give bit-identical results. */
typedef enum {
    RN_ALLREDUCE_AUTO = 0,
    RN_ALLREDUCE_ONE_SHOT = 1,
    RN_ALLREDUCE_TWO_SHOT = 2
} rn_allreduce_algorithm;

typedef struct {
    int32_t world;       /* ranks in the group, 1..RN_ALLREDUCE_MAX_WORLD */
    int32_t rank;        /* group rank of the first (or only) rank this call computes */
    int32_t local_ranks; /* ranks this call computes on this device: 1, or `world`
                          * with rank == 0 (the whole group on one device) */
    int32_t algorithm;   /* rn_allreduce_algorithm; the same on every rank */
    void* buffers[RN_ALLREDUCE_MAX_WORLD]; /* [world] each rank's exchange buffer, as
                          * addressed from this device; the caller owns them */
    void* signals[RN_ALLREDUCE_MAX_WORLD]; /* [world] each rank's signal pad of
                          * RN_ALLREDUCE_SIGNAL_BYTES: zero-filled before the first
                          * call, then written only by these kernels; one group's */
    int64_t buffer_bytes; /* size of each exchange buffer: two halves, each holding
                          * T * H 16-bit values (one-shot: buffer_bytes >= 4 * T * H + 32)
                          * or 3 * T * H (two-shot: >= 12 * T * H + 32) */
    int64_t timeout_ns;  /* bound on each wait for a peer; <= 0 selects 1 second */
} rn_allreduce_comm;

/* Calls are numbered on the device: each launch reads its rank's call
 * counter from the signal pad and advances it when its last block finishes,
 * so calls captured in a CUDA graph stay numbered correctly on replay. */

/* Errors: the fused ops' validation, then RN_ERR_COMM for an invalid `comm`
 * (world, rank, local_ranks, algorithm, a NULL or misaligned buffer or pad,
 * buffers too small for T, H and the algorithm, TWO_SHOT with fewer than 3
 * ranks), RN_ERR_LAYOUT for the alignment rules
 * above, RN_ERR_SHAPE for H > 32768 or a row count not divisible by
 * local_ranks, RN_ERR_ALIAS when an operand overlaps a local exchange buffer
 * or signal pad, RN_ERR_CUDA when the launch fails. A peer that does not
 * publish within timeout_ns is not an error of the call (it is asynchronous):
 * the waiting block leaves its rows unwritten and sets bit 1 of
 * rn_device_errors. Asynchronous on `stream`. */
RN_API rn_status rn_allreduce_fused_add_rms_norm(const rn_tensor* out, const rn_tensor* x,
                                                 const rn_tensor* residual,
                                                 const rn_tensor* weight, float eps,
                                                 const rn_allreduce_comm* comm, void* stream);
RN_API rn_status rn_allreduce_fused_add_rms_norm_fp8(const rn_tensor* q, const rn_tensor* scale,
                                                     const rn_tensor* x,
                                                     const rn_tensor* residual,
                                                     const rn_tensor* weight, float eps,
                                                     const rn_allreduce_comm* comm,
                                                     void* stream);

/* ---- the whole group on one device, with the library's own exchange memory
 *
 * No counterpart on the pages: they describe no such entry point. It is for
 * callers that cannot allocate device memory: a plugin or kernel library
 * running inside a host framework that owns every allocation (its caching
 * allocator, or a fixed arena handed out at start-up) and gives the plugin
 * no way to ask for more, or code that may run while a stream is being
 * captured, where an allocation would be recorded into the graph or refused.
 * This is rn_allreduce_fused_add_rms_norm for a group of `world` ranks all held on
 * the current device (operands stacked [world, T, H], as with local_ranks ==
 * world; one launch computes every rank), whose exchange buffers and signal
 * pads live in a static device array of the library instead of caller
 * memory: it allocates nothing and takes no rn_allreduce_comm.
 * Capacity: world * round_up(4 * T * H + 32, 256) <= RN_LOCAL_EXCHANGE_BYTES
 * (32 MiB of buffers, plus 8 signal pads), else RN_ERR_CAPACITY before any
 * CUDA call; world outside 1..8 is RN_ERR_COMM; otherwise the checks and
 * errors of rn_allreduce_fused_add_rms_norm, with the AUTO algorithm (from
 * three ranks on, buffers sized for two-shot when
 * world * round_up(12 * T * H + 32, 256) fits; successive calls may then
 * alternate between one-shot and two-shot on the same signal pads, which is
 * safe because a flag is compared with the call number for equality). The
 * first call in a device's context looks the array up (the device must be
 * current, as for every call; a context re-created after a device reset
 * counts as new), and that call and the first call with a given `world`
 * after another clear the signal pads with cudaMemsetAsync on `stream`: make
 * those calls outside stream capture (RN_ERR_CONFIG inside). The memory is
 * shared by every call on a device and keeps what the last call left in it:
 * calls that overlap in time (other streams, other threads) race and give
 * undefined results. */
#define RN_LOCAL_EXCHANGE_BYTES 33554432
RN_API rn_status rn_allreduce_fused_add_rms_norm_local(const rn_tensor* out, const rn_tensor* x,
                                                       const rn_tensor* residual,
                                                       const rn_tensor* weight, float eps,
                                                       int32_t world, void* stream);

/* ---- operands in host memory: chunked copy-in / compute / copy-out ------
 *
 * No counterpart on the pages, which time device-resident tensors only. These
 * entry points run rn_rms_norm, rn_fused_add_rms_norm and
 * rn_fused_add_rms_norm_fp8 on activations that live in HOST memory: out, x,
 * residual, q and scale are host pointers (any memory a cudaMemcpyDefault
 * copy reaches; only page-locked host memory lets the copies run
 * asynchronously and overlap), while the weight is a device pointer as for
 * the device entry points. The T rows are cut into chunks of chunk_rows rows.
 * Chunk c runs on streams[c % n_streams] in slot (c % n_streams) of the
 * scratch: its rows of x (and residual) are copied in, the kernel of the
 * device entry point runs on the slot (16-bit output in place over the
 * slot's x), and residual and out (or residual, q and scale) are copied back
 * over the host rows. Chunks on different streams overlap, so the copy in of
 * one chunk, the kernel of another and the copy out of a third proceed at
 * once over the full-duplex host link. The results are those of the device
 * entry point bit for bit: rows are independent and each chunk is one
 * launch of the same kernels.
 *
 * Everything is enqueued and the call returns; the host buffers must stay
 * untouched until every stream has finished. Work of earlier calls on the
 * same streams orders before a chunk as usual; the scratch must not be used
 * by anything else until then. Validation follows the device entry point
 * (aliasing rules applied to the host buffers, out == x allowed), then the
 * pipeline: NULL pipeline, streams or scratch -> RN_ERR_NULL; n_streams
 * outside 1..RN_HOST_MAX_STREAMS or reserved != 0 -> RN_ERR_CONFIG; scratch
 * not 256-byte aligned -> RN_ERR_LAYOUT; the slots (see rn_host_plan_chunks)
 * not fitting in scratch_bytes -> RN_ERR_CAPACITY; scratch overlapping the
 * weight or a host operand -> RN_ERR_ALIAS; all of these before any CUDA
 * call. Last, the scratch and the weight must be device (or managed)
 * memory: cudaPointerGetAttributes is asked, RN_ERR_LAYOUT otherwise. A
 * failed copy or launch returns RN_ERR_CUDA; chunks enqueued before it
 * still run. T == 0 is a no-op. */
#define RN_HOST_MAX_STREAMS 8

typedef struct {
    void* scratch;          /* caller-owned device memory, 256-byte aligned */
    int64_t scratch_bytes;
    void* const* streams;   /* n_streams caller-owned cudaStream_t of the current device */
    int32_t n_streams;      /* 1 .. RN_HOST_MAX_STREAMS */
    int32_t reserved;       /* must be 0 */
    int64_t chunk_rows;     /* rows per chunk; <= 0: the library's choice */
} rn_host_pipeline;

typedef struct {
    int64_t chunk_rows;  /* rows per chunk (the last chunk may hold fewer) */
    int64_t chunks;      /* ceil(T / chunk_rows); 0 when T == 0 */
    int64_t slot_bytes;  /* scratch bytes of one slot */
    int32_t slots;       /* slots in use: min(n_streams, chunks) */
    int32_t reserved;
} rn_host_plan;

/* The chunking of a host-memory call: op (rn_op, not SILU_AND_MUL_FP8), a
 * [T x H] 16-bit problem, scratch_bytes of scratch, n_streams streams and the
 * requested chunk_rows (<= 0: automatic). A slot holds, for chunk_rows rows,
 * the x rows (2 * H bytes each), the residual rows (fused ops, 2 * H), the
 * codes (fp8 op, H) and the scales (fp8 op, 4), each region rounded up to 256
 * bytes. Automatic: chunks of ceil(T / (4 * n_streams)) rows, but at least
 * enough rows for 8 MiB of x per copy, at most T, and no more than
 * n_streams slots can hold in scratch_bytes. RN_ERR_CAPACITY when the slots
 * in use do not fit, RN_ERR_SHAPE for T < 0 or H < 1, RN_ERR_CONFIG for a bad
 * op or n_streams. Pure host logic. */
RN_API rn_status rn_host_plan_chunks(int32_t op, int64_t T, int64_t H, int64_t scratch_bytes,
                                     int32_t n_streams, int64_t chunk_rows, rn_host_plan* plan);

RN_API rn_status rn_host_rms_norm(const rn_tensor* out, const rn_tensor* x,
                                  const rn_tensor* weight, float eps, int64_t variance_size,
                                  const rn_host_pipeline* pipeline);
RN_API rn_status rn_host_fused_add_rms_norm(const rn_tensor* out, const rn_tensor* x,
                                            const rn_tensor* residual, const rn_tensor* weight,
                                            float eps, int64_t variance_size,
                                            const rn_host_pipeline* pipeline);
RN_API rn_status rn_host_fused_add_rms_norm_fp8(const rn_tensor* q, const rn_tensor* scale,
                                                const rn_tensor* x, const rn_tensor* residual,
                                                const rn_tensor* weight, float eps,
                                                int64_t variance_size,
                                                const rn_host_pipeline* pipeline);

/* Static text for a status code (never NULL). */
RN_API const char* rn_status_string(rn_status status);

/* Text of the last RN_ERR_CUDA returned on the calling thread ("" if none). */
RN_API const char* rn_last_cuda_error(void);

/* ---- launch planning (introspection; no memory is touched) ------------- */

typedef enum {
    RN_OP_RMS_NORM = 0,
    RN_OP_FUSED_ADD = 1,
    RN_OP_FUSED_ADD_FP8 = 2,
    RN_OP_SILU_AND_MUL_FP8 = 3 /* rn_plan_launch only: H is I, the output width */
} rn_op;
/* Kernels: VECTOR keeps each row in registers (a group of threads per row);
 * STAGED is persistent and streams whole rows into a shared-memory ring with
 * bulk asynchronous copies (one block per row at a time); SCALAR handles
 * unaligned or ragged rows. */
typedef enum { RN_KERNEL_VECTOR = 0, RN_KERNEL_SCALAR = 1, RN_KERNEL_STAGED = 2 } rn_kernel;

typedef struct {
    int32_t kernel;             /* rn_kernel */
    int32_t threads_per_row;    /* threads cooperating on one row */
    int32_t vectors_per_thread; /* VECTOR: 16-byte vectors each thread holds per row; else 0 */
    int32_t rows_per_cta;       /* rows a block works on at once */
    int32_t block_threads;      /* threads per block */
    int32_t smem_bytes;         /* dynamic shared memory per block */
    int32_t stages;             /* STAGED: depth of the shared-memory row ring; else 0 */
    int32_t ctas_per_sm;        /* STAGED: resident blocks per SM the grid is sized for; else 0 */
    int64_t grid;               /* blocks launched */
} rn_plan;

/* The launch shape the library would use for `op` on a [T x H] problem of
 * `dtype` (RN_F16/RN_BF16); `vector_ok` says whether the operands meet the
 * vector kernel's alignment (see Alignment above). Pure host logic: needs no
 * GPU. Honours rn_force_plan. Returns RN_ERR_SHAPE for H < 1 or T < 0. */
RN_API rn_status rn_plan_launch(int32_t op, int32_t dtype, int64_t T, int64_t H,
                         int32_t vector_ok, rn_plan* plan);

/* Dry run: performs every check of the entry point named by `op` (for
 * RN_OP_RMS_NORM and RN_OP_FUSED_ADD `out_or_q` is `out`; for
 * RN_OP_FUSED_ADD_FP8 it is `q`; `scale` and `residual` are ignored by the
 * ops that take none) and returns the status that call would return, without
 * touching memory, calling CUDA or launching. When it returns RN_OK and the
 * problem is not empty, `plan` (nullable) receives the launch shape. Pure host
 * logic: usable without a GPU. */
RN_API rn_status rn_validate(int32_t op, const rn_tensor* out_or_q, const rn_tensor* scale,
                      const rn_tensor* x, const rn_tensor* residual, const rn_tensor* weight,
                      float eps, int64_t variance_size, rn_plan* plan);

/* Test hook: force the vector kernel's (threads_per_row, vectors_per_thread,
 * rows_per_cta; rows_per_cta 0 = automatic) for every later call in the
 * process; (0, 0, 0) restores automatic choice. rows_per_cta is clamped to
 * what the block limit and the named barriers allow.
 * threads_per_row must be a power of two <= 32 or a multiple of 32 <= 1024,
 * and vectors_per_thread one of the compiled widths (see
 * rn_supported_vectors_per_thread); otherwise RN_ERR_CONFIG. A forced shape
 * that cannot cover a row (threads_per_row * vectors_per_thread * 8 < H) or
 * exceeds the kernel's block limit falls back to the scalar kernel. The
 * all-reduce kernels take a forced (threads_per_row, vectors_per_thread)
 * too when threads_per_row is a power of two <= 512, vectors_per_thread is
 * 1, 2, 4 or 8 and together they cover a row. Not thread-safe with
 * concurrent launches; meant for tests and tuning. */
RN_API rn_status rn_force_plan(int32_t threads_per_row, int32_t vectors_per_thread,
                                int32_t rows_per_cta);

/* Test hook: force the STAGED kernel with `ctas_per_sm` resident blocks per SM
 * (1, 2 or 4), `stages` ring slots (>= 2) and `threads` per block (a multiple
 * of 32, 32..1024) for every later call with 16-byte-aligned operands; a
 * shape whose shared memory exceeds the per-block limit falls back to the
 * automatic choice. (0, 0, 0) restores automatic choice; a forced STAGED shape
 * takes precedence over rn_force_plan. Not thread-safe with concurrent
 * launches; meant for tests and tuning. */
RN_API rn_status rn_force_staged(int32_t ctas_per_sm, int32_t stages, int32_t threads);

/* Launch options for every later call in the process (tuning hook):
 * pdl = 1 launches with programmatic dependent launch (the kernel may begin
 * launching while the previous kernel in the stream drains; it waits for that
 * kernel to complete before touching memory), 0 launches plainly, -1 restores
 * the library default; max_grid > 0 caps the blocks launched (the kernels
 * stride over the remaining rows), 0 restores the library's default cap (16
 * blocks per SM; none for the fused ops on 8192 rows or more and the SwiGLU
 * kernel on 4096 or more, whose blocks then take one row group each).
 * RN_ERR_CONFIG for other values. Not thread-safe with concurrent launches. */
RN_API rn_status rn_set_launch_options(int32_t pdl, int64_t max_grid);

/* L2 prefetch across the kernel boundary for every later call in the
 * process (tuning hook): with mode = 1, a vector-kernel launch of the norm ops
 * or of silu_and_mul_fp8 made with programmatic dependent launch asks L2 for
 * its blocks' first rows of x (and the residual) before it waits for the
 * previous kernel in the stream, so
 * HBM keeps streaming while that kernel drains. A prefetch is a hint: the
 * values every load returns are unchanged. 0 turns it off, -1 restores the
 * library default (on); RN_ERR_CONFIG for other values. Not thread-safe with
 * concurrent launches. */
RN_API rn_status rn_set_prefetch(int32_t mode);

/* Reads and clears the device-side error flags of the current device:
 * bit 0 = a bounded wait inside the STAGED kernel timed out (some rows of
 * that call were not written); bit 1 = an all-reduce call waited longer than
 * its timeout for a peer (some rows of that call were not written).
 * Synchronises with the device. */
RN_API rn_status rn_device_errors(uint32_t* flags);

/* The compute capability (major * 10 + minor: 100 for sm_100a) that the
 * library's device code loaded on the current device was compiled for.
 * Loads the code if needed; RN_ERR_CUDA without a usable device. */
RN_API rn_status rn_kernel_binary_version(int32_t* version);

/* Writes up to `cap` compiled vectors_per_thread values into `out` and
 * returns how many exist. */
RN_API int32_t rn_supported_vectors_per_thread(int32_t* out, int32_t cap);

/* Library version, "major.minor.patch". */
RN_API const char* rn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* RMSNORM_B200_H */
