/*
 * The C ABI used from plain C, through include/rmsnorm_b200.h only: test
 * infrastructure (built and run by tests/test_capi_c.py).
 *
 *   capi_from_c host   validation, status strings, planning and the GEMM
 *                      configuration choice: pure host logic, no GPU needed.
 *                      Every call here is refused before any CUDA call (the
 *                      stand-in pointers are host memory).
 *   capi_from_c gpu    fused_add_rms_norm on a [5 x 1000] bf16 problem (the
 *                      scalar kernel: H % 8 != 0) and on [37 x 3840] (the
 *                      vector kernel) in device memory from cudaMalloc, and
 *                      on [300 x 3840] in plain malloc'd host memory through
 *                      rn_host_fused_add_rms_norm (64-row chunks, two
 *                      streams), checked against the CPU oracle linked from
 *                      oracle/: the written back residual bit for bit, the
 *                      output within one unit in the last place.
 * Exit status 0 on success; the first failed check is printed.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "rmsnorm_b200.h"

/* CUDA runtime entry points used by the gpu mode (from libcudart). */
typedef int cudaError_t;
extern cudaError_t cudaMalloc(void** p, size_t n);
extern cudaError_t cudaFree(void* p);
extern cudaError_t cudaMemcpy(void* dst, const void* src, size_t n, int kind);
extern cudaError_t cudaDeviceSynchronize(void);
typedef void* cudaStream_t;
extern cudaError_t cudaStreamCreate(cudaStream_t* s);
extern cudaError_t cudaStreamDestroy(cudaStream_t s);
enum { kH2D = 1, kD2H = 2 };

/* The oracle (oracle/rmsnorm_oracle.c). */
extern int oracle_fused_add_rms_norm(const uint16_t* x, const uint16_t* r_in, const uint16_t* w,
                                     int dtype, int64_t T, int64_t H, float eps,
                                     uint16_t* r_out, uint16_t* out, double* y_out,
                                     double* row, double* yrow);
extern uint16_t oracle_f64_to_bf16(double v);

static int failures = 0;
#define CHECK(cond, ...)                                  \
    do {                                                  \
        if (!(cond)) {                                    \
            fprintf(stderr, "FAIL %s:%d: ", __FILE__, __LINE__); \
            fprintf(stderr, __VA_ARGS__);                 \
            fprintf(stderr, "\n");                        \
            ++failures;                                   \
        }                                                 \
    } while (0)

static rn_tensor view2(void* data, int32_t dtype, const int64_t* sizes, const int64_t* strides) {
    rn_tensor t;
    t.data = data;
    t.dtype = dtype;
    t.ndim = 2;
    t.sizes = sizes;
    t.strides = strides;
    return t;
}

static int host_mode(void) {
    static uint16_t hx[4 * 64], hr[4 * 64], ho[4 * 64], hw[64];
    const int64_t sz[2] = {4, 64}, st[2] = {64, 1}, wsz[1] = {64}, wst[1] = {1};
    rn_tensor x = view2(hx, RN_BF16, sz, st), r = view2(hr, RN_BF16, sz, st);
    rn_tensor o = view2(ho, RN_BF16, sz, st);
    rn_tensor w = {hw, RN_BF16, 1, wsz, wst};
    rn_tensor wf16 = {hw, RN_F16, 1, wsz, wst};
    const int64_t bad_st[2] = {128, 1};  /* padded rows: flattening not free */
    rn_tensor xpad = view2(hx, RN_BF16, sz, bad_st);
    const int64_t zsz[2] = {4, 0};
    rn_tensor xz = view2(hx, RN_BF16, zsz, st);

    CHECK(rn_fused_add_rms_norm(NULL, &x, &r, &w, 1e-6f, -1, NULL) == RN_ERR_NULL, "null out");
    CHECK(rn_fused_add_rms_norm(&o, &x, &r, &w, 1e-6f, 64, NULL) == RN_ERR_VARIANCE_SIZE,
          "variance_size");
    CHECK(rn_fused_add_rms_norm(&o, &x, &r, &w, -1.f, -1, NULL) == RN_ERR_EPS, "eps < 0");
    CHECK(rn_fused_add_rms_norm(&o, &x, &r, &wf16, 1e-6f, -1, NULL) == RN_ERR_WEIGHT_DTYPE,
          "weight dtype");
    CHECK(rn_fused_add_rms_norm(&o, &xpad, &r, &w, 1e-6f, -1, NULL) == RN_ERR_LAYOUT, "padded");
    CHECK(rn_fused_add_rms_norm(&o, &xz, &r, &w, 1e-6f, -1, NULL) == RN_ERR_SHAPE, "H == 0");
    CHECK(rn_fused_add_rms_norm(&o, &x, &x, &w, 1e-6f, -1, NULL) == RN_ERR_ALIAS,
          "residual aliasing x");
    CHECK(strlen(rn_status_string(RN_ERR_ALIAS)) > 0, "status text");
    CHECK(strncmp(rn_version(), "0.", 2) == 0, "version");

    rn_plan p;
    CHECK(rn_plan_launch(1 /* RN_OP_FUSED_ADD */, RN_BF16, 8192, 3840, 1, &p) == RN_OK, "plan");
    CHECK(p.kernel == RN_KERNEL_VECTOR && p.threads_per_row * p.vectors_per_thread * 8 >= 3840,
          "plan covers a row");
    CHECK(rn_plan_launch(1, RN_BF16, 8192, 1000, 0, &p) == RN_OK && p.kernel == RN_KERNEL_SCALAR,
          "unaligned rows take the scalar kernel");
    int32_t cfg = -1;
    CHECK(rn_fp8_gemm_config(1, 8192, 3840, 148, &cfg) == RN_OK && cfg == RN_GEMM_CH64_TOK16,
          "decode GEMM configuration");
    CHECK(rn_fp8_gemm_config(8192, 8192, 3840, 148, &cfg) == RN_OK && cfg == RN_GEMM_TOK128_CH256,
          "prefill GEMM configuration");
    rn_allreduce_comm comm;
    memset(&comm, 0, sizeof comm);
    comm.world = 9;
    CHECK(rn_allreduce_fused_add_rms_norm(&o, &x, &r, &w, 1e-6f, &comm, NULL) == RN_ERR_COMM,
          "all-reduce group of 9");
    rn_host_plan hp;
    CHECK(rn_host_plan_chunks(1, 8192, 3840, (int64_t)1 << 40, 2, 0, &hp) == RN_OK &&
              hp.chunk_rows == 1093 && hp.chunks == 8 && hp.slots == 2,
          "host chunking of the prefill batch");
    CHECK(rn_host_plan_chunks(1, 8192, 3840, 1000, 2, 0, &hp) == RN_ERR_CAPACITY,
          "host scratch too small");
    CHECK(rn_host_fused_add_rms_norm(&o, &x, &r, &w, 1e-6f, -1, NULL) == RN_ERR_NULL,
          "host call without a pipeline");
    return failures;
}

static uint16_t bf16_of(double v) { return oracle_f64_to_bf16(v); }

static int ulp_distance_bf16(uint16_t a, uint16_t b) {
    int32_t ia = (a & 0x8000) ? -(int32_t)(a & 0x7fff) : (int32_t)a;
    int32_t ib = (b & 0x8000) ? -(int32_t)(b & 0x7fff) : (int32_t)b;
    return abs(ia - ib);
}

static int gpu_case(int64_t T, int64_t H, unsigned seed) {
    const size_t n = (size_t)(T * H), bytes = n * 2;
    uint16_t *hx = malloc(bytes), *hr = malloc(bytes), *hw = malloc((size_t)H * 2);
    uint16_t *g_out = malloc(bytes), *g_res = malloc(bytes), *o_out = malloc(bytes),
             *o_res = malloc(bytes);
    double *row = malloc((size_t)H * sizeof(double)), *yrow = malloc((size_t)H * sizeof(double));
    srand(seed);
    for (size_t i = 0; i < n; ++i) {
        hx[i] = bf16_of((rand() / (double)RAND_MAX - 0.5) * 4.0);
        hr[i] = bf16_of((rand() / (double)RAND_MAX - 0.5) * 8.0);
    }
    for (int64_t i = 0; i < H; ++i) hw[i] = bf16_of(1.0 + (rand() / (double)RAND_MAX - 0.5) * 0.5);

    void *dx = NULL, *dr = NULL, *dw = NULL, *dout = NULL;
    CHECK(cudaMalloc(&dx, bytes) == 0 && cudaMalloc(&dr, bytes) == 0 &&
              cudaMalloc(&dw, (size_t)H * 2) == 0 && cudaMalloc(&dout, bytes) == 0,
          "cudaMalloc");
    if (failures) return failures;
    cudaMemcpy(dx, hx, bytes, kH2D);
    cudaMemcpy(dr, hr, bytes, kH2D);
    cudaMemcpy(dw, hw, (size_t)H * 2, kH2D);
    const int64_t sz[2] = {T, H}, st[2] = {H, 1}, wsz[1] = {H}, wst[1] = {1};
    rn_tensor x = view2(dx, RN_BF16, sz, st), r = view2(dr, RN_BF16, sz, st);
    rn_tensor o = view2(dout, RN_BF16, sz, st);
    rn_tensor w = {dw, RN_BF16, 1, wsz, wst};
    rn_status s = rn_fused_add_rms_norm(&o, &x, &r, &w, 1e-6f, -1, NULL);
    CHECK(s == RN_OK, "launch: %s %s", rn_status_string(s), rn_last_cuda_error());
    CHECK(cudaDeviceSynchronize() == 0, "synchronize");
    cudaMemcpy(g_out, dout, bytes, kD2H);
    cudaMemcpy(g_res, dr, bytes, kD2H);
    uint32_t flags = 1;
    CHECK(rn_device_errors(&flags) == RN_OK && flags == 0, "device error flags");

    CHECK(oracle_fused_add_rms_norm(hx, hr, hw, 1 /* bf16 */, T, H, 1e-6f, o_res, o_out, NULL,
                                    row, yrow) == 0,
          "oracle");
    int res_bad = 0, out_max = 0;
    for (size_t i = 0; i < n; ++i) {
        res_bad += g_res[i] != o_res[i];
        const int d = ulp_distance_bf16(g_out[i], o_out[i]);
        if (d > out_max) out_max = d;
    }
    CHECK(res_bad == 0, "[%ld x %ld] residual differs in %d elements", (long)T, (long)H, res_bad);
    CHECK(out_max <= 1, "[%ld x %ld] output off by %d ulp", (long)T, (long)H, out_max);
    cudaFree(dx);
    cudaFree(dr);
    cudaFree(dw);
    cudaFree(dout);
    free(hx); free(hr); free(hw); free(g_out); free(g_res); free(o_out); free(o_res);
    free(row); free(yrow);
    return failures;
}

/* The same problem from host memory through the chunked host entry point. */
static int gpu_host_case(int64_t T, int64_t H, unsigned seed) {
    const size_t n = (size_t)(T * H), bytes = n * 2;
    uint16_t *hx = malloc(bytes), *hr = malloc(bytes), *hr0 = malloc(bytes),
             *hw = malloc((size_t)H * 2), *g_out = malloc(bytes), *o_out = malloc(bytes),
             *o_res = malloc(bytes);
    double *row = malloc((size_t)H * sizeof(double)), *yrow = malloc((size_t)H * sizeof(double));
    srand(seed);
    for (size_t i = 0; i < n; ++i) {
        hx[i] = bf16_of((rand() / (double)RAND_MAX - 0.5) * 4.0);
        hr0[i] = hr[i] = bf16_of((rand() / (double)RAND_MAX - 0.5) * 8.0);
    }
    for (int64_t i = 0; i < H; ++i) hw[i] = bf16_of(1.0 + (rand() / (double)RAND_MAX - 0.5) * 0.5);

    rn_host_plan plan;
    CHECK(rn_host_plan_chunks(1, T, H, (int64_t)1 << 40, 2, 64, &plan) == RN_OK, "host plan");
    void *dw = NULL, *scratch = NULL;
    cudaStream_t streams[2] = {NULL, NULL};
    CHECK(cudaMalloc(&dw, (size_t)H * 2) == 0 &&
              cudaMalloc(&scratch, (size_t)(plan.slots * plan.slot_bytes)) == 0,
          "cudaMalloc");
    CHECK(cudaStreamCreate(&streams[0]) == 0 && cudaStreamCreate(&streams[1]) == 0,
          "cudaStreamCreate");
    if (failures) return failures;
    cudaMemcpy(dw, hw, (size_t)H * 2, kH2D);
    const int64_t sz[2] = {T, H}, st[2] = {H, 1}, wsz[1] = {H}, wst[1] = {1};
    rn_tensor x = view2(hx, RN_BF16, sz, st), r = view2(hr, RN_BF16, sz, st);
    rn_tensor o = view2(g_out, RN_BF16, sz, st);
    rn_tensor w = {dw, RN_BF16, 1, wsz, wst};
    rn_host_pipeline pipe;
    memset(&pipe, 0, sizeof pipe);
    pipe.scratch = scratch;
    pipe.scratch_bytes = plan.slots * plan.slot_bytes;
    pipe.streams = streams;
    pipe.n_streams = 2;
    pipe.chunk_rows = 64;
    rn_status s = rn_host_fused_add_rms_norm(&o, &x, &r, &w, 1e-6f, -1, &pipe);
    CHECK(s == RN_OK, "host call: %s %s", rn_status_string(s), rn_last_cuda_error());
    CHECK(cudaDeviceSynchronize() == 0, "synchronize");

    CHECK(oracle_fused_add_rms_norm(hx, hr0, hw, 1 /* bf16 */, T, H, 1e-6f, o_res, o_out, NULL,
                                    row, yrow) == 0,
          "oracle");
    int res_bad = 0, out_max = 0;
    for (size_t i = 0; i < n; ++i) {
        res_bad += hr[i] != o_res[i];
        const int d = ulp_distance_bf16(g_out[i], o_out[i]);
        if (d > out_max) out_max = d;
    }
    CHECK(res_bad == 0, "host [%ld x %ld] residual differs in %d elements", (long)T, (long)H,
          res_bad);
    CHECK(out_max <= 1, "host [%ld x %ld] output off by %d ulp", (long)T, (long)H, out_max);
    cudaStreamDestroy(streams[0]);
    cudaStreamDestroy(streams[1]);
    cudaFree(dw);
    cudaFree(scratch);
    free(hx); free(hr); free(hr0); free(hw); free(g_out); free(o_out); free(o_res);
    free(row); free(yrow);
    return failures;
}

int main(int argc, char** argv) {
    if (argc != 2 || (strcmp(argv[1], "host") != 0 && strcmp(argv[1], "gpu") != 0)) {
        fprintf(stderr, "usage: %s host|gpu\n", argv[0]);
        return 2;
    }
    int f = host_mode();
    if (strcmp(argv[1], "gpu") == 0) {
        f += gpu_case(5, 1000, 1);
        f += gpu_case(37, 3840, 2);
        f += gpu_host_case(300, 3840, 3);
    }
    if (f == 0) printf("ok (%s)\n", argv[1]);
    return f == 0 ? 0 : 1;
}
