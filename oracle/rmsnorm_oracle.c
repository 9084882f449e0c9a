/*
 * rmsnorm_oracle.c -- plain, slow, fp64 CPU reference for the three RMSNorm
 * operators. TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and
 * the benchmark's CPU-baseline leg use it; the CUDA library never links,
 * includes or calls anything in this directory, and this file shares no code
 * with it.
 *
 * What is computed (one row at a time, all arithmetic in IEEE binary64):
 *
 *   rms_norm            y_i = v_i / sqrt(mean_j(v_j^2) + eps) * w_i,
 *                       out_i = RNE16(y_i)
 *     The operator is named, but not written out, in "vllm.kernels.aiter_ops"
 *     (attribute rms_no_var_16bit_only: 16-bit activations, weight of the same
 *     dtype or None, no variance-size override). The formula is the textbook
 *     RMSNorm: normalise by the root mean square over the hidden dimension,
 *     with eps inside the square root, then scale by the weight.
 *
 *   fused_add_rms_norm  r'_i = RNE16(x_i + r_i) is written back over the
 *                       residual, then rms_norm is applied to r' (the rounded,
 *                       stored values). Named in "vllm.kernels.aiter_ops"
 *                       (attribute rms_add_no_var_16bit_only).
 *
 *   fused_add_rms_norm_fp8
 *                       the fused pass above, then a per-token dynamic cast to
 *                       OCP FP8 e4m3fn: amax = max_i |y_i| over the unrounded
 *                       y, s = amax / 448, q_i = E4M3(y_i / s) with
 *                       round-to-nearest-even and saturation to +-448, and the
 *                       stored scale is (float)s. q_i is the rounding of the
 *                       exact real quotient y_i / s (evaluated as 448 p_i / P,
 *                       see the loop), so rounding ties are decided exactly.
 *                       A row with amax == 0 gets s = 0 and all-zero codes. The single-pass
 *                       residual + RMSNorm + FP8 fusion is the first of the
 *                       three kernels in "Custom CUDA kernels juice Llama 3.1
 *                       405B on AMD MI300X, skipping Nvidia lock-in".
 *
 * eps arrives as a float and is widened to double, so the oracle and the GPU
 * use the same eps value. w_i = 1 when no weight is given.
 *
 * RNE16 (binary64 -> bf16 or fp16, round to nearest, ties to even, IEEE
 * overflow to infinity, gradual underflow) and the e4m3fn encoder/decoder are
 * written here from the format definitions: bf16 = sign, 8 exponent bits
 * (bias 127), 7 fraction bits; fp16 = sign, 5 exponent bits (bias 15), 10
 * fraction bits; e4m3fn = sign, 4 exponent bits (bias 7), 3 fraction bits,
 * no infinities, NaN only at S.1111.111, largest finite 448.
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared (no fast-math, no FMA
 * contraction, so every operation rounds exactly once as written).
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>
#include <string.h>

#define OR_F16 0
#define OR_BF16 1

/* ------------------------------------------------------------------------ */
/* Format decoding (exact).                                                  */

double oracle_bf16_to_f64(uint16_t h) {
    /* bf16 is the upper half of an IEEE binary32 word. */
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

double oracle_f16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)m, -24); /* subnormal: m * 2^-24 */
    } else if (e == 31) {
        v = m ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + m), e - 25); /* (1 + m/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

double oracle_e4m3_to_f64(uint8_t c) {
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 0xf;
    int m = c & 0x7;
    double v;
    if (e == 15 && m == 7) {
        v = NAN;
    } else if (e == 0) {
        v = ldexp((double)m, -9); /* subnormal: m * 2^-9 */
    } else {
        v = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    }
    return sign ? -v : v;
}

/* ------------------------------------------------------------------------ */
/* Rounding a binary64 value to a narrower binary format.                    */

/* Rounds |a| (finite, > 0) to the nearest multiple of the format's quantum
 * at a's binade; p = significand bits including the hidden bit, emin = the
 * exponent of the smallest normal. Ties go to the even multiple. The result
 * may be 2^(E+1) when rounding carries into the next binade. */
static double round_magnitude(double a, int p, int emin) {
    int k;
    frexp(a, &k);          /* a = f * 2^k, f in [0.5, 1) */
    int E = k - 1;         /* a in [2^E, 2^(E+1)) */
    if (E < emin) E = emin; /* subnormal range: fixed quantum */
    double quantum = ldexp(1.0, E - (p - 1));
    double n = a / quantum; /* exact: division by a power of two */
    double fl = floor(n);
    double frac = n - fl;   /* exact */
    double r;
    if (frac > 0.5) {
        r = fl + 1.0;
    } else if (frac < 0.5) {
        r = fl;
    } else {
        r = (fmod(fl, 2.0) == 0.0) ? fl : fl + 1.0; /* tie: to even */
    }
    return r * quantum;
}

/* Encodes an exactly representable magnitude a (>= 0) into exponent and
 * fraction fields of a format with p significand bits and the given bias. */
static uint32_t encode_fields(double a, int p, int emin, int bias) {
    if (a == 0.0) return 0;
    int k;
    frexp(a, &k);
    int E = k - 1;
    if (E < emin) { /* subnormal: exponent field 0 */
        double m = a / ldexp(1.0, emin - (p - 1));
        return (uint32_t)m;
    }
    double m = a / ldexp(1.0, E - (p - 1)) - ldexp(1.0, p - 1);
    return ((uint32_t)(E + bias) << (p - 1)) | (uint32_t)m;
}

uint16_t oracle_f64_to_bf16(double v) {
    if (isnan(v)) return 0x7fc0;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    const double maxf = ldexp(255.0, 120); /* (2 - 2^-7) * 2^127 */
    if (isinf(a)) return sign | 0x7f80;
    if (a == 0.0) return sign;
    double r = round_magnitude(a, 8, -126);
    if (r > maxf) return sign | 0x7f80; /* overflow to infinity */
    return sign | (uint16_t)encode_fields(r, 8, -126, 127);
}

uint16_t oracle_f64_to_f16(double v) {
    if (isnan(v)) return 0x7e00;
    uint16_t sign = signbit(v) ? 0x8000 : 0;
    double a = fabs(v);
    const double maxf = 65504.0;
    if (isinf(a)) return sign | 0x7c00;
    if (a == 0.0) return sign;
    double r = round_magnitude(a, 11, -14);
    if (r > maxf) return sign | 0x7c00;
    return sign | (uint16_t)encode_fields(r, 11, -14, 15);
}

/* Round to nearest even onto e4m3fn values, saturating to +-448 (never
 * producing the NaN codes); NaN maps to 0x7f. */
uint8_t oracle_f64_to_e4m3_satfinite(double v) {
    if (isnan(v)) return 0x7f;
    uint8_t sign = signbit(v) ? 0x80 : 0;
    double a = fabs(v);
    if (a == 0.0) return sign;
    double r = isinf(a) ? 448.0 : round_magnitude(a, 4, -6);
    if (r > 448.0) r = 448.0;
    return sign | (uint8_t)encode_fields(r, 4, -6, 7);
}

static double load16(const uint16_t* p, int64_t i, int dtype) {
    return dtype == OR_BF16 ? oracle_bf16_to_f64(p[i]) : oracle_f16_to_f64(p[i]);
}

static uint16_t store16(double v, int dtype) {
    return dtype == OR_BF16 ? oracle_f64_to_bf16(v) : oracle_f64_to_f16(v);
}

/* ------------------------------------------------------------------------ */
/* The operators. Row-major [T x H]; weight [H] or NULL (all ones).          */

/* y (unrounded, binary64) of RMSNorm over one row v[0..H). */
static void rms_row(const double* v, const uint16_t* w, int dtype, int64_t H,
                    double e, double* y) {
    double ss = 0.0;
    for (int64_t i = 0; i < H; ++i) ss += v[i] * v[i];
    double ms = ss / (double)H;
    double rms = sqrt(ms + e);
    for (int64_t i = 0; i < H; ++i) {
        double wi = w ? load16(w, i, dtype) : 1.0;
        y[i] = v[i] / rms * wi;
    }
}

/* Returns 0 on success, -1 on a bad argument. `row` is caller scratch of H
 * doubles; `y_out` receives the unrounded y when non-NULL ([T x H]). */
int oracle_rms_norm(const uint16_t* x, const uint16_t* w, int dtype, int64_t T,
                    int64_t H, float eps, uint16_t* out, double* y_out,
                    double* row, double* yrow) {
    if ((dtype != OR_F16 && dtype != OR_BF16) || H <= 0 || T < 0) return -1;
    double e = (double)eps;
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t* xr = x + t * H;
        for (int64_t i = 0; i < H; ++i) row[i] = load16(xr, i, dtype);
        rms_row(row, w, dtype, H, e, yrow);
        for (int64_t i = 0; i < H; ++i) {
            if (out) out[t * H + i] = store16(yrow[i], dtype);
            if (y_out) y_out[t * H + i] = yrow[i];
        }
    }
    return 0;
}

int oracle_fused_add_rms_norm(const uint16_t* x, const uint16_t* r_in,
                              const uint16_t* w, int dtype, int64_t T, int64_t H,
                              float eps, uint16_t* r_out, uint16_t* out,
                              double* y_out, double* row, double* yrow) {
    if ((dtype != OR_F16 && dtype != OR_BF16) || H <= 0 || T < 0) return -1;
    double e = (double)eps;
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t i = 0; i < H; ++i) {
            double s = load16(x, t * H + i, dtype) + load16(r_in, t * H + i, dtype);
            uint16_t rb = store16(s, dtype);
            r_out[t * H + i] = rb;
            row[i] = load16(&rb, 0, dtype); /* normalise the stored residual */
        }
        rms_row(row, w, dtype, H, e, yrow);
        for (int64_t i = 0; i < H; ++i) {
            if (out) out[t * H + i] = store16(yrow[i], dtype);
            if (y_out) y_out[t * H + i] = yrow[i];
        }
    }
    return 0;
}

int oracle_fused_add_rms_norm_fp8(const uint16_t* x, const uint16_t* r_in,
                                  const uint16_t* w, int dtype, int64_t T,
                                  int64_t H, float eps, uint16_t* r_out,
                                  uint8_t* q, float* scale, double* y_out,
                                  double* row, double* yrow) {
    if ((dtype != OR_F16 && dtype != OR_BF16) || H <= 0 || T < 0) return -1;
    double e = (double)eps;
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t i = 0; i < H; ++i) {
            double s = load16(x, t * H + i, dtype) + load16(r_in, t * H + i, dtype);
            uint16_t rb = store16(s, dtype);
            r_out[t * H + i] = rb;
            row[i] = load16(&rb, 0, dtype);
        }
        rms_row(row, w, dtype, H, e, yrow);
        double amax = 0.0, pmax = 0.0;
        for (int64_t i = 0; i < H; ++i) {
            double a = fabs(yrow[i]);
            if (a > amax) amax = a;
            double p = fabs(row[i] * (w ? load16(w, i, dtype) : 1.0));
            if (p > pmax) pmax = p;
        }
        double s = amax / 448.0;
        scale[t] = (float)s;
        for (int64_t i = 0; i < H; ++i) {
            /* q_i = E4M3(y_i / s). In real arithmetic y_i / s = 448 * p_i / P
             * with p_i = r'_i * w_i and P = max_j |p_j|: the rms cancels. p_i
             * (a product of two 16-bit values) and 448 * p_i are exact in
             * binary64, so the one correctly rounded division below returns
             * the real quotient exactly whenever that quotient is an e4m3
             * rounding tie, and the encoder rounds it as the real value. */
            double p = row[i] * (w ? load16(w, i, dtype) : 1.0);
            q[t * H + i] = pmax > 0.0 ? oracle_f64_to_e4m3_satfinite(448.0 * p / pmax) : 0;
            if (y_out) y_out[t * H + i] = yrow[i];
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Element-wise array forms of the codecs, for the tests.                    */

void oracle_decode16_array(const uint16_t* in, int dtype, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = load16(in, i, dtype);
}

void oracle_encode16_array(const double* in, int dtype, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = store16(in[i], dtype);
}

void oracle_decode_e4m3_array(const uint8_t* in, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_e4m3_to_f64(in[i]);
}

void oracle_encode_e4m3_array(const double* in, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_f64_to_e4m3_satfinite(in[i]);
}

/* ------------------------------------------------------------------------ */
/* Fused SwiGLU + per-token FP8 cast, the second kernel of "Custom CUDA      */
/* kernels juice Llama 3.1 405B on AMD MI300X, skipping Nvidia lock-in".    */
/* Row t of x holds [gate | up] (2I values). y_i = silu(gate_i) * up_i with */
/* silu(a) = a / (1 + e^-a) (libm exp, binary64); amax = max |y_i|;        */
/* s = amax / 448; q_i = E4M3(y_i / s); the stored scale is (float)s; a row */
/* with amax == 0 gets s = 0 and zero codes.                                */
int oracle_silu_and_mul_fp8(const uint16_t* x, int dtype, int64_t T, int64_t I, uint8_t* q,
                            float* scale, double* y_out, double* yrow) {
    if ((dtype != OR_F16 && dtype != OR_BF16) || I <= 0 || T < 0) return -1;
    for (int64_t t = 0; t < T; ++t) {
        const uint16_t* xr = x + t * 2 * I;
        double amax = 0.0;
        for (int64_t i = 0; i < I; ++i) {
            double a = load16(xr, i, dtype);
            double b = load16(xr, I + i, dtype);
            double y = a / (1.0 + exp(-a)) * b;
            yrow[i] = y;
            if (fabs(y) > amax) amax = fabs(y);
        }
        double s = amax / 448.0;
        scale[t] = (float)s;
        for (int64_t i = 0; i < I; ++i) {
            q[t * I + i] = amax > 0.0 ? oracle_f64_to_e4m3_satfinite(yrow[i] / s) : 0;
            if (y_out) y_out[t * I + i] = yrow[i];
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Row-wise scaled fp8 GEMM, the consumer of the per-token codes (the fp8   */
/* linear layers of "VLLM_ROCM_USE_AITER=1 slows Gemma 4 on an AMD MI300X"):*/
/*   D[m, n] = RNE_bf16( (sum_k A[m, k] * B[n, k]) * a_scale[m] * b_scale[n] ) */
/* A [M x K] and B [N x K] are e4m3fn codes. Every product of two e4m3      */
/* values is an integer multiple of 2^-18 below 2^18, so the binary64 sum of */
/* up to 2^17 products is exact: the only roundings are the two scale       */
/* products and the final cast. Rows m in [m0, m1) only (the caller may     */
/* sample rows); d_out (nullable) receives the unrounded values.            */
int oracle_fp8_rowwise_gemm(const uint8_t* A, const uint8_t* B, const float* a_scale,
                            const float* b_scale, int64_t M, int64_t N, int64_t K, int64_t m0,
                            int64_t m1, uint16_t* D, double* d_out) {
    if (M < 0 || N <= 0 || K <= 0 || K > (1 << 17) || m0 < 0 || m1 > M || m0 > m1) return -1;
    double dec[256];
    for (int c = 0; c < 256; ++c) dec[c] = oracle_e4m3_to_f64((uint8_t)c);
    for (int64_t m = m0; m < m1; ++m) {
        const uint8_t* a = A + m * K;
        for (int64_t n = 0; n < N; ++n) {
            const uint8_t* b = B + n * K;
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k) acc += dec[a[k]] * dec[b[k]];
            double y = acc * (double)a_scale[m] * (double)b_scale[n];
            D[m * N + n] = oracle_f64_to_bf16(y);
            if (d_out) d_out[m * N + n] = y;
        }
    }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* All-reduce sum of tensor-parallel partials (the all-reduce that precedes  */
/* the residual add and RMSNorm in a tensor-parallel decoder layer; AITER    */
/* provides all-reduce and RMSNorm to SGLang, "AITER: AMD's operator library */
/* for ROCm", ecosystem section). Element i of the result is the exact real  */
/* sum of the W partial values parts[r][i], rounded once to the 16-bit       */
/* format (RNE16 as above). Non-finite inputs follow IEEE addition: any NaN, */
/* or +inf with -inf, gives NaN; otherwise an infinity gives that infinity.  */
/* An exact zero sum is -0 only when every term is -0 (round-to-nearest).   */
/*                                                                          */
/* The exact sum is kept as a two's-complement integer multiple of          */
/* 2^ACC_LSB in ACC_LIMBS 64-bit limbs: every finite bf16 or fp16 value is an */
/* integer below 2^24 times a power of two >= 2^-160, and the largest sum of */
/* up to 64 terms stays below 2^300, so no bit is ever lost. The integer is */
/* then rounded to odd at 53 bits (its top 53 bits, with the lowest of them  */
/* set when anything below is non-zero), an exact binary64 value; rounding   */
/* that to nearest at 8 or 11 bits gives the correctly rounded sum (rounding */
/* to odd with at least two extra bits makes the second rounding innocuous:  */
/* Boldo and Melquiond, "When double rounding is odd", 2005).               */

#define ACC_LIMBS 6
#define ACC_LSB (-160)

typedef struct { uint64_t w[ACC_LIMBS]; } exact_acc;

/* acc += sign * m * 2^(ACC_LSB + sh), 0 <= m < 2^24, 0 <= sh <= 300. */
static void acc_add(exact_acc* acc, int negative, uint64_t m, int sh) {
    uint64_t t[ACC_LIMBS] = {0};
    int li = sh / 64, bi = sh % 64;
    t[li] = m << bi;
    if (bi != 0 && li + 1 < ACC_LIMBS) t[li + 1] = m >> (64 - bi);
    if (negative) { /* two's complement: invert, add one */
        unsigned carry = 1;
        for (int k = 0; k < ACC_LIMBS; ++k) {
            uint64_t inv = ~t[k];
            t[k] = inv + carry;
            carry = carry && t[k] == 0;
        }
    }
    unsigned carry = 0;
    for (int k = 0; k < ACC_LIMBS; ++k) {
        uint64_t s = acc->w[k] + t[k];
        unsigned c1 = s < acc->w[k];
        uint64_t s2 = s + carry;
        unsigned c2 = s2 < s;
        acc->w[k] = s2;
        carry = c1 | c2;
    }
}

/* The accumulated exact value, rounded to odd at 53 significant bits. */
static double acc_to_f64_odd(const exact_acc* acc) {
    uint64_t a[ACC_LIMBS];
    memcpy(a, acc->w, sizeof a);
    int negative = (int)(a[ACC_LIMBS - 1] >> 63);
    if (negative) {
        unsigned carry = 1;
        for (int k = 0; k < ACC_LIMBS; ++k) {
            uint64_t inv = ~a[k];
            a[k] = inv + carry;
            carry = carry && a[k] == 0;
        }
    }
    int h = -1; /* highest set bit */
    for (int k = ACC_LIMBS - 1; k >= 0 && h < 0; --k)
        for (int b = 63; b >= 0; --b)
            if ((a[k] >> b) & 1) { h = 64 * k + b; break; }
    if (h < 0) return 0.0;
    double mag;
    if (h < 53) {
        mag = ldexp((double)a[0], ACC_LSB); /* below 2^53: exact */
    } else {
        int lo = h - 52; /* keep bits [lo, h] */
        uint64_t top = 0;
        for (int b = h; b >= lo; --b) top = (top << 1) | ((a[b / 64] >> (b % 64)) & 1);
        int sticky = 0;
        for (int b = lo - 1; b >= 0 && !sticky; --b) sticky = (int)((a[b / 64] >> (b % 64)) & 1);
        if (sticky) top |= 1;
        mag = ldexp((double)top, lo + ACC_LSB);
    }
    return negative ? -mag : mag;
}

/* parts: W arrays of n 16-bit values, rank r's at parts + r * n. */
int oracle_allreduce_sum16(const uint16_t* parts, int W, int64_t n, int dtype, uint16_t* x) {
    if ((dtype != OR_F16 && dtype != OR_BF16) || W < 1 || W > 64 || n < 0) return -1;
    for (int64_t i = 0; i < n; ++i) {
        exact_acc acc;
        memset(&acc, 0, sizeof acc);
        int nan = 0, pinf = 0, ninf = 0, all_neg_zero = 1;
        for (int r = 0; r < W; ++r) {
            double v = load16(parts + (int64_t)r * n, i, dtype);
            if (isnan(v)) { nan = 1; continue; }
            if (isinf(v)) { if (v > 0) pinf = 1; else ninf = 1; continue; }
            if (!(v == 0.0 && signbit(v))) all_neg_zero = 0;
            if (v == 0.0) continue;
            int k;
            double f = frexp(fabs(v), &k);         /* |v| = f * 2^k, f in [0.5, 1) */
            uint64_t m = (uint64_t)ldexp(f, 24);  /* exact: <= 11 significant bits */
            acc_add(&acc, v < 0, m, (k - 24) - ACC_LSB);
        }
        double s;
        if (nan || (pinf && ninf)) s = NAN;
        else if (pinf) s = INFINITY;
        else if (ninf) s = -INFINITY;
        else {
            s = acc_to_f64_odd(&acc);
            if (s == 0.0) s = all_neg_zero ? -0.0 : 0.0;
        }
        x[i] = store16(s, dtype);
    }
    return 0;
}
