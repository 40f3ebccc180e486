/*
 * qlin_oracle.c -- plain, slow, obviously-correct CPU oracle for the quantized
 * linear layer (dynamic activation quantisation followed by a scaled GEMM).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package smoke check and
 * the CPU-baseline leg of the benchmark may load this library.  It shares no
 * code, header, table or constant generator with the CUDA library; neither
 * side includes or links the other.
 *
 * What it follows.  The page "Helion in vLLM: A Unified Route to Tunable Linear
 * Kernels", section "What the integration changes", names the three formats
 * (FP8 dynamic quantisation, W8A8 INT8, Block-FP8) and the three GEMM
 * strategies (plain, Split-K, Swap-AB).  The page prints no formula, so each
 * function below states the arithmetic it implements, in the plainest reading:
 *
 *   per-token (INT8 / FP8):   s[m] = amax_k |x[m,k]| / Qmax, Qmax = 127 / 448
 *                             q[m,k] = Q(x[m,k] / s[m])
 *   Block-FP8:                one scale per 1x128 (activations) or 128x128
 *                             (weights) block, s = amax_block / 448
 *   scaled GEMM:              C[m,n] = bf16( (acc[m,n] * s_a[m]) * s_w[n] + bias[n] )
 *   Block-FP8 GEMM:           C[m,n] = bf16( sum_kb P_kb[m,n] * s_a[m,kb] * s_w[n/128,kb] )
 *   bf16 GEMM:                C[m,n] = bf16( fp32(sum_k a[m,k] w[n,k]) + bias[n] ), the
 *                             matmul of the page "[Kernel][Perf] Add Hopper (SM90)
 *                             tuned config for batch-invariant persistent matmul"
 *   MXFP8 / NVFP4:            block-scaled codecs and GEMM, at the end of this
 *                             file with their readings
 *
 * Every fp32 operation is a separately rounded IEEE binary32 operation
 * (compile with -O2 -fno-fast-math -ffp-contract=off; x86-64 SSE arithmetic),
 * round-to-nearest-even.  Sums of products are formed EXACTLY in 64-bit
 * integers and rounded once, so the oracle is at least as accurate as any
 * fp32 accumulation order.
 *
 * Readings taken where the pages are silent:
 *   - amax == 0: the scale is 0 and every quantised value is +0.
 *   - x / s is a true IEEE division, not a multiply by 1/s.
 *   - INT8 rounds half-to-even and clamps to [-127, 127] (-128 never occurs).
 *   - FP8 clamps x/s to [-448, 448] ("saturation"), then rounds to the nearest
 *     OCP E4M3 (e4m3fn) code, ties to the even code, keeping the sign of zero.
 *
 * Parity pins for every function here live in tests/test_oracle_*.py.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

#define QO_FMT_INT8 0
#define QO_FMT_FP8 1
#define QO_FMT_FP8_BLOCK 2

/* ---------------------------------------------------------------- bf16 ---- */

/* bfloat16 is the upper half of a binary32: widening is a 16-bit shift. */
float qo_bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* binary32 -> bfloat16, round to nearest, ties to even (on the dropped 16 bits). */
uint16_t qo_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if (isnan(f)) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t upper = u >> 16;
    uint32_t lower = u & 0xFFFFu;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
    return (uint16_t)upper;
}

/* ---------------------------------------------------------------- e4m3 ---- */
/*
 * OCP FP8 E4M3 ("e4m3fn"): 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
 * bits, no infinities; S.1111.111 is NaN, so the largest finite magnitude is
 * S.1111.110 = 1.75 * 2^8 = 448.  Exponent field 0 holds subnormals m * 2^-9.
 */

/* Value of a code as an integer count of 2^-9 (exact for every finite code). */
int64_t qo_e4m3_units(uint8_t code) {
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    int64_t mag;
    if (e == 0)
        mag = m;                              /* m * 2^-9                   */
    else
        mag = (int64_t)(8 + m) << (e - 1);    /* (1 + m/8) * 2^(e-7) / 2^-9 */
    return (code & 0x80) ? -mag : mag;
}

float qo_e4m3_decode(uint8_t code) {
    if ((code & 0x7F) == 0x7F) return NAN;
    double v = (double)qo_e4m3_units(code) * ldexp(1.0, -9);
    if (v == 0.0 && (code & 0x80)) return -0.0f;
    return (float)v;
}

/* floor(v + 1/2) with exact ties going to the even integer; v >= 0. */
static double round_half_even_nonneg(double v) {
    double f = floor(v);
    double frac = v - f;                      /* exact: v has few bits here */
    if (frac > 0.5) return f + 1.0;
    if (frac < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* Nearest e4m3fn code to v (ties to even code), saturating at +-448. */
uint8_t qo_e4m3_encode(float v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: grid step 2^-9; rounding up to 8 steps lands on
         * 2^-6, which is code 0x08, the smallest normal -- the same integer. */
        double r = round_half_even_nonneg(a * 512.0);
        return (uint8_t)(sign | (uint8_t)r);
    }
    int e = (int)floor(log2(a));              /* unbiased exponent, -6..8 */
    /* guard log2 rounding at exact powers of two */
    if (ldexp(1.0, e) > a) e -= 1;
    if (ldexp(1.0, e + 1) <= a) e += 1;
    double steps = a / ldexp(1.0, e - 3);     /* in [8, 16), exact */
    double r = round_half_even_nonneg(steps); /* 8..16; 16 carries into e+1 */
    int code = ((e + 7) << 3) + ((int)r - 8);
    if (code > 0x7E) code = 0x7E;             /* cannot happen below 448 */
    return (uint8_t)(sign | (uint8_t)code);
}

/* ----------------------------------------------------------- quantisers ---- */

/* Round half to even to an integer, then clamp to [-127, 127]. */
static int8_t int8_rne_clamp(float v) {
    double a = round_half_even_nonneg(fabs((double)v));
    double r = signbit(v) ? -a : a;
    if (r > 127.0) r = 127.0;
    if (r < -127.0) r = -127.0;
    return (int8_t)r;
}

static uint8_t quantize_one(int fmt, float x, float s) {
    if (s == 0.0f) return 0;                  /* amax == 0 reading: q = +0 */
    float v = x / s;                          /* IEEE binary32 division */
    if (fmt == QO_FMT_INT8) return (uint8_t)int8_rne_clamp(v);
    if (v > 448.0f) v = 448.0f;               /* saturation */
    if (v < -448.0f) v = -448.0f;
    return qo_e4m3_encode(v);
}

/*
 * Per-token dynamic quantisation (INT8 or FP8): one scale per row.
 * x: bf16 bits [rows][ld], q: [rows][cols] row-major, s: [rows].
 */
void qo_quantize_per_token(int fmt, const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                           uint8_t* q, float* s) {
    const float qmax = (fmt == QO_FMT_INT8) ? 127.0f : 448.0f;
    for (int64_t r = 0; r < rows; ++r) {
        float amax = 0.0f;
        for (int64_t c = 0; c < cols; ++c) {
            float a = fabsf(qo_bf16_to_f32(x[r * ld + c]));
            if (a > amax) amax = a;
        }
        float sr = amax / qmax;               /* IEEE binary32 division */
        s[r] = sr;
        for (int64_t c = 0; c < cols; ++c)
            q[r * cols + c] = quantize_one(fmt, qo_bf16_to_f32(x[r * ld + c]), sr);
    }
}

/*
 * Block-FP8 quantisation: one e4m3 scale per block of block_rows x block_cols
 * elements (1 x 128 for activations, 128 x 128 for weights).  A block at the
 * bottom edge holds the rows that exist.  cols must be a multiple of
 * block_cols.  s: [ceil(rows/block_rows)][cols/block_cols] row-major.
 */
void qo_quantize_block(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld,
                       int64_t block_rows, int64_t block_cols, uint8_t* q, float* s) {
    int64_t nbr = (rows + block_rows - 1) / block_rows;
    int64_t nbc = cols / block_cols;
    for (int64_t br = 0; br < nbr; ++br) {
        int64_t r0 = br * block_rows;
        int64_t r1 = r0 + block_rows < rows ? r0 + block_rows : rows;
        for (int64_t bc = 0; bc < nbc; ++bc) {
            int64_t c0 = bc * block_cols, c1 = c0 + block_cols;
            float amax = 0.0f;
            for (int64_t r = r0; r < r1; ++r)
                for (int64_t c = c0; c < c1; ++c) {
                    float a = fabsf(qo_bf16_to_f32(x[r * ld + c]));
                    if (a > amax) amax = a;
                }
            float sb = amax / 448.0f;
            s[br * nbc + bc] = sb;
            for (int64_t r = r0; r < r1; ++r)
                for (int64_t c = c0; c < c1; ++c)
                    q[r * cols + c] = quantize_one(QO_FMT_FP8, qo_bf16_to_f32(x[r * ld + c]), sb);
        }
    }
}

/* ---------------------------------------------------------- scaled GEMM ---- */

/* Exact integer value of a quantised element: int8 as is, e4m3 in 2^-9 units. */
static int64_t element_units(int fmt, uint8_t code) {
    if (fmt == QO_FMT_INT8) return (int64_t)(int8_t)code;
    return qo_e4m3_units(code);
}

/*
 * Scaled GEMM, C = A_q * W_q^T with scales, both operands K-major:
 *   a_q [M][K], w_q [N][K], c [M][N] bf16 bits.
 * Per-token formats: s_a [M], s_w [N]; bias bf16 [N] or NULL.
 *   INT8: acc = sum_k a*w exactly (int32 range), y = fp32(acc)
 *   FP8 : acc = sum_k a*w exactly in 2^-18 units, y = fp32(acc) (one rounding)
 *   y = y * s_a[m]; y = y * s_w[n]; y = y + bias[n]; C = bf16(y)
 * Block-FP8: s_a [M][K/128], s_w [ceil(N/128)][K/128]; bias must be NULL.
 *   P_kb exact per 128-wide K block, acc = sum_kb P_kb*2^-18*s_a*s_w in fp64,
 *   C = bf16(fp32(acc)).
 * Only the rows m_idx[0..m_cnt) and columns n_idx[0..n_cnt) are computed
 * (NULL index = all); outputs are dense [m_cnt][n_cnt].
 * acc_out (INT8 only, may be NULL): the int32 accumulators, [m_cnt][n_cnt].
 * Returns 0, or -1 if an INT8 accumulator leaves the int32 range.
 */
int qo_scaled_mm(int fmt, int64_t M, int64_t N, int64_t K,
                 const uint8_t* a_q, const float* s_a, const uint8_t* w_q, const float* s_w,
                 const uint16_t* bias, const int64_t* m_idx, int64_t m_cnt,
                 const int64_t* n_idx, int64_t n_cnt, uint16_t* c, int32_t* acc_out) {
    if (!m_idx) m_cnt = M;
    if (!n_idx) n_cnt = N;
    const int64_t kblocks = K / 128;
    /* decode the selected rows once into exact integers */
    int64_t* ua = (int64_t*)malloc(sizeof(int64_t) * (size_t)(m_cnt * K));
    int64_t* uw = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_cnt * K));
    if (!ua || !uw) { free(ua); free(uw); return -2; }
    for (int64_t i = 0; i < m_cnt; ++i) {
        int64_t m = m_idx ? m_idx[i] : i;
        for (int64_t k = 0; k < K; ++k) ua[i * K + k] = element_units(fmt, a_q[m * K + k]);
    }
    for (int64_t j = 0; j < n_cnt; ++j) {
        int64_t n = n_idx ? n_idx[j] : j;
        for (int64_t k = 0; k < K; ++k) uw[j * K + k] = element_units(fmt, w_q[n * K + k]);
    }
    int rc = 0;
    for (int64_t i = 0; i < m_cnt; ++i) {
        int64_t m = m_idx ? m_idx[i] : i;
        const int64_t* ra = ua + i * K;
        for (int64_t j = 0; j < n_cnt; ++j) {
            int64_t n = n_idx ? n_idx[j] : j;
            const int64_t* rw = uw + j * K;
            float y;
            if (fmt == QO_FMT_FP8_BLOCK) {
                double acc = 0.0;
                for (int64_t kb = 0; kb < kblocks; ++kb) {
                    int64_t p = 0;
                    for (int64_t k = kb * 128; k < kb * 128 + 128; ++k) p += ra[k] * rw[k];
                    acc += (double)p * ldexp(1.0, -18) * (double)s_a[m * kblocks + kb]
                           * (double)s_w[(n / 128) * kblocks + kb];
                }
                y = (float)acc;
            } else {
                int64_t p = 0;
                for (int64_t k = 0; k < K; ++k) p += ra[k] * rw[k];
                if (fmt == QO_FMT_INT8) {
                    if (p > INT32_MAX || p < INT32_MIN) rc = -1;
                    if (acc_out) acc_out[i * n_cnt + j] = (int32_t)p;
                    y = (float)(int32_t)p;            /* int32 -> fp32, RNE */
                } else {
                    y = (float)p;                     /* exact sum, one rounding */
                    y = y * 0x1p-18f;                 /* exact power-of-two scaling */
                }
                y = y * s_a[m];
                y = y * s_w[n];
                if (bias) y = y + qo_bf16_to_f32(bias[n]);
            }
            c[i * n_cnt + j] = qo_f32_to_bf16(y);
        }
    }
    free(ua);
    free(uw);
    return rc;
}

/* ------------------------------------------------------------- bf16 GEMM ---- */
/*
 * bf16 matmul with fp32 accumulation and bf16 output, the workload of the
 * page "[Kernel][Perf] Add Hopper (SM90) tuned config for batch-invariant
 * persistent matmul" (sections "Summary" and "H100 NVL Sweep Results": a
 * bfloat16 matmul of activations [M,K] with weights [N,K]):
 *
 *   C[m,n] = bf16( fp32( sum_k a[m,k] * w[n,k] ) + bias[n] )
 *
 * The product of two bf16 values (8-bit significands) is exact in binary64;
 * the products are summed in binary64 in k order, the sum is rounded once to
 * binary32, the bias (if any) is added as a binary32 addition and the result
 * is rounded to bf16.  The binary64 sum differs from the exact one by at most
 * K * 2^-53 * sum_k |a w|, far below the bf16 output rounding, so comparing a
 * GPU result (fp32 accumulation in any fixed order) with this one measures the
 * GPU's accumulation error.  Row and column selection as qo_scaled_mm.
 */
int qo_gemm_bf16(int64_t M, int64_t N, int64_t K, const uint16_t* a, const uint16_t* w, const uint16_t* bias,
                 const int64_t* m_idx, int64_t m_cnt, const int64_t* n_idx, int64_t n_cnt, uint16_t* c) {
    if (!m_idx) m_cnt = M;
    if (!n_idx) n_cnt = N;
    double* da = (double*)malloc(sizeof(double) * (size_t)(m_cnt * K));
    double* dw = (double*)malloc(sizeof(double) * (size_t)(n_cnt * K));
    if (!da || !dw) { free(da); free(dw); return -2; }
    for (int64_t i = 0; i < m_cnt; ++i) {
        int64_t m = m_idx ? m_idx[i] : i;
        for (int64_t k = 0; k < K; ++k) da[i * K + k] = (double)qo_bf16_to_f32(a[m * K + k]);
    }
    for (int64_t j = 0; j < n_cnt; ++j) {
        int64_t n = n_idx ? n_idx[j] : j;
        for (int64_t k = 0; k < K; ++k) dw[j * K + k] = (double)qo_bf16_to_f32(w[n * K + k]);
    }
    for (int64_t i = 0; i < m_cnt; ++i) {
        for (int64_t j = 0; j < n_cnt; ++j) {
            int64_t n = n_idx ? n_idx[j] : j;
            double s = 0.0;
            for (int64_t k = 0; k < K; ++k) s += da[i * K + k] * dw[j * K + k];
            float y = (float)s;                         /* one rounding to binary32 */
            if (bias) y = y + qo_bf16_to_f32(bias[n]);  /* binary32 addition */
            c[i * n_cnt + j] = qo_f32_to_bf16(y);
        }
    }
    free(da);
    free(dw);
    return 0;
}

/* ------------------------------------------------------------- FP8 MoE ---- */
/*
 * The FP8 MoE layer the page "vLLM and Tencent Hunyuan upstream two HPC
 * backends for NVIDIA Hopper GPUs" describes as one execution path (section
 * "FP8 MoE pipeline as a single execution path": routing, Gate-Up GEMM,
 * activation, quantisation, Down GEMM, top-k reduction), written out step by
 * step.  The page gives the order of the steps, not their arithmetic; the
 * plainest readings, stated here:
 *
 *   routing   for each token t, the k experts with the largest fp32 router
 *             logits (ties: the lower expert index first), in descending
 *             order; weights = softmax over those k logits:
 *               m = l_0 (the largest); e_j = fp32(exp_binary64(l_j - m));
 *               s = e_0 + e_1 + ... (fp32, in j order); w_j = e_j / s (fp32)
 *   rows      token t's j-th expert e gets one row of that expert's group;
 *             within an expert the rows are ordered by token index
 *   gate-up   x is quantised per token to FP8 (qo_quantize_per_token); the
 *             row of expert e computes G = scaled_mm(x_q[t], W1_q[e], s_x[t],
 *             s_w1[e]) (the per-token FP8 GEMM of qo_scaled_mm, bf16 out, no
 *             bias); G has 2I columns, gate = G[:, :I], up = G[:, I:]
 *   act       h = silu(gate) * up in fp32 with silu(g) = g / (1 + q),
 *             q = fp32(exp_binary64(-g)); the row of h is quantised per
 *             token to FP8 (H_q, s_h)
 *   down      Y = scaled_mm(H_q, W2_q[e], s_h, s_w2[e]) (bf16, no bias)
 *   combine   out[t, n] = bf16( sum_j w_j * Y[row(t, j), n] ), the sum in fp32
 *             from +0, j in routing order, each product and add separately
 *             rounded
 *
 * Shapes: x bf16 [T, H]; logits fp32 [T, E]; W1_q [E, 2I, H] with s_w1 [E, 2I];
 * W2_q [E, H, I] with s_w2 [E, H]; out bf16 [T, H].  Also returned for checks:
 * topk ids/weights [T, k], the row of each (t, j) and the expert offsets
 * [E + 1].
 */
static float silu_f32(float g) {
    float q = (float)exp(-(double)g);      /* binary64 exponential, rounded once */
    return g / (1.0f + q);
}

/* act: h = silu(gate) * up in fp32 for each row of g (bf16 [R, 2I]), then
 * the row's per-token FP8 quantisation (amax, scale = amax / 448, codes as
 * quantize_one) into hq [R, I] and sh [R]. */
void qo_moe_act_quantize(int64_t R, int64_t I, const uint16_t* g, uint8_t* hq, float* sh) {
    for (int64_t r = 0; r < R; ++r) {
        float amax = 0.0f;
        for (int64_t i = 0; i < I; ++i) {
            const float h = silu_f32(qo_bf16_to_f32(g[r * 2 * I + i])) * qo_bf16_to_f32(g[r * 2 * I + I + i]);
            if (fabsf(h) > amax) amax = fabsf(h);
        }
        const float sc = amax / 448.0f;
        sh[r] = sc;
        for (int64_t i = 0; i < I; ++i) {
            const float h = silu_f32(qo_bf16_to_f32(g[r * 2 * I + i])) * qo_bf16_to_f32(g[r * 2 * I + I + i]);
            hq[r * I + i] = quantize_one(QO_FMT_FP8, h, sc);
        }
    }
}

/* combine: out[t, n] = bf16( sum_j w[t, j] * y[rows[t, j], n] ), fp32 from +0
 * in routing order, each product and add separately rounded. */
void qo_moe_combine(int64_t T, int64_t H, int64_t topk, const uint16_t* y, const float* w, const int32_t* rows,
                    uint16_t* out) {
    for (int64_t t = 0; t < T; ++t)
        for (int64_t n = 0; n < H; ++n) {
            float acc = 0.0f;
            for (int64_t j = 0; j < topk; ++j) {
                const float p = w[t * topk + j] * qo_bf16_to_f32(y[(int64_t)rows[t * topk + j] * H + n]);
                acc = acc + p;
            }
            out[t * H + n] = qo_f32_to_bf16(acc);
        }
}

/* Intermediates returned for checks (caller-allocated): g bf16 [R, 2I],
 * hq [R, I], sh [R], y bf16 [R, H], R = T * topk.  topk <= 64. */
int qo_moe_forward(int64_t T, int64_t H, int64_t I, int64_t E, int64_t topk, const uint16_t* x,
                   const float* logits, const uint8_t* w1_q, const float* s_w1, const uint8_t* w2_q,
                   const float* s_w2, int32_t* topk_ids, float* topk_w, int32_t* rows, int32_t* offsets,
                   uint16_t* g, uint8_t* hq, float* sh, uint16_t* y, uint16_t* out) {
    const int64_t R = T * topk;
    int rc = 0;
    if (topk < 1 || topk > 64 || topk > E) return -3;
    /* routing */
    for (int64_t t = 0; t < T; ++t) {
        const float* l = logits + t * E;
        for (int64_t j = 0; j < topk; ++j) {
            int64_t best = -1;
            for (int64_t e = 0; e < E; ++e) {
                int taken = 0;
                for (int64_t i = 0; i < j; ++i) taken |= topk_ids[t * topk + i] == (int32_t)e;
                if (taken) continue;
                if (best < 0 || l[e] > l[best]) best = e;   /* ties keep the lower index */
            }
            topk_ids[t * topk + j] = (int32_t)best;
        }
        const float m = l[topk_ids[t * topk]];
        float ev[64];
        float s = 0.0f;
        for (int64_t j = 0; j < topk; ++j) {
            ev[j] = (float)exp((double)(l[topk_ids[t * topk + j]] - m));
            s = s + ev[j];
        }
        for (int64_t j = 0; j < topk; ++j) topk_w[t * topk + j] = ev[j] / s;
    }
    /* rows: expert groups in expert order, tokens in order inside a group */
    offsets[0] = 0;
    for (int64_t e = 0; e < E; ++e) {
        int32_t n = 0;
        for (int64_t t = 0; t < T; ++t)
            for (int64_t j = 0; j < topk; ++j) n += topk_ids[t * topk + j] == (int32_t)e;
        offsets[e + 1] = offsets[e] + n;
    }
    int32_t* fill = (int32_t*)calloc((size_t)E, sizeof(int32_t));
    uint8_t* xq = (uint8_t*)malloc((size_t)(T * H));
    float* sx = (float*)malloc(sizeof(float) * (size_t)T);
    uint8_t* a1 = (uint8_t*)malloc((size_t)(R * H));
    float* sa1 = (float*)malloc(sizeof(float) * (size_t)R);
    if (!fill || !xq || !sx || !a1 || !sa1) { rc = -2; goto out; }
    for (int64_t t = 0; t < T; ++t)
        for (int64_t j = 0; j < topk; ++j) {
            const int32_t e = topk_ids[t * topk + j];
            rows[t * topk + j] = offsets[e] + fill[e]++;
        }
    /* gate-up: per-token FP8 codes of x, gathered into the expert rows */
    qo_quantize_per_token(QO_FMT_FP8, x, T, H, H, xq, sx);
    for (int64_t t = 0; t < T; ++t)
        for (int64_t j = 0; j < topk; ++j) {
            const int64_t r = rows[t * topk + j];
            memcpy(a1 + r * H, xq + t * H, (size_t)H);
            sa1[r] = sx[t];
        }
    for (int64_t e = 0; e < E; ++e) {
        const int64_t r0 = offsets[e], n = offsets[e + 1] - offsets[e];
        if (n == 0) continue;
        rc |= qo_scaled_mm(QO_FMT_FP8, n, 2 * I, H, a1 + r0 * H, sa1 + r0, w1_q + e * 2 * I * H, s_w1 + e * 2 * I,
                           NULL, NULL, n, NULL, 2 * I, g + r0 * 2 * I, NULL);
    }
    /* act */
    qo_moe_act_quantize(R, I, g, hq, sh);
    /* down */
    for (int64_t e = 0; e < E; ++e) {
        const int64_t r0 = offsets[e], n = offsets[e + 1] - offsets[e];
        if (n == 0) continue;
        rc |= qo_scaled_mm(QO_FMT_FP8, n, H, I, hq + r0 * I, sh + r0, w2_q + e * H * I, s_w2 + e * H, NULL, NULL,
                           n, NULL, H, y + r0 * H, NULL);
    }
    /* combine */
    qo_moe_combine(T, H, topk, y, topk_w, rows, out);
out:
    free(fill); free(xq); free(sx); free(a1); free(sa1);
    return rc;
}

/* ------------------------------------------------- block-scaled formats ---- */
/*
 * The page "Helion in vLLM: A Unified Route to Tunable Linear Kernels"
 * (introduction) lists NVFP4 among the formats vLLM's quantized linear layers
 * serve; the pages define neither it nor MXFP8.  The readings below follow
 * the formats' public definitions and take the plainest arithmetic where
 * those leave a step open:
 *
 * MXFP8 (OCP Microscaling Formats v1.0: E4M3 elements, blocks of 32 along K,
 * one E8M0 scale X = 2^(code - 127) per block):
 *   amax == 0:  scale code 0, every element +0 (as the FP8 reading above);
 *   otherwise:  e = floor(log2(amax)) - 8 (8 = the largest E4M3 exponent),
 *               clamped to [-127, 127]; scale code e + 127;
 *               q = E4M3(x * 2^-e), nearest code, ties to even, saturating
 *               at +-448 (amax * 2^-e lies in [256, 512), so the block's
 *               largest elements may saturate: the format's own rule).
 *   x * 2^-e is exact, so the element rounding is the only rounding.
 *
 * NVFP4 (E2M1 elements {0, 0.5, 1, 1.5, 2, 3, 4, 6} with sign, blocks of 16
 * along K, one E4M3 scale per block, one fp32 decode scale g per tensor,
 * x ~ q * s * g):
 *   t = amax / 6 (binary32 division), t = t / g (binary32 division),
 *   s = E4M3(t) (nearest, ties to even, saturating at 448);
 *   d = dec(s) * g (binary32 multiply); d == 0: every element +0;
 *   otherwise q = E2M1(x / d) (binary32 division, then the nearest E2M1
 *   value, ties to the even code, saturating at +-6, keeping the sign of
 *   zero).  Two elements per byte, element 2i in the low nibble.
 *   g is an input: per-tensor amax / (6 * 448) for weights, a calibrated
 *   constant for activations.
 *
 * Block-scaled GEMM, both operands K-major, bias bf16 [N] or NULL:
 *   MXFP8: acc = sum over 32-blocks b of 2^(ea_b + eb_b) * sum_{k in b} a_k w_k,
 *          each block sum exact (2^-18 units), the blocks added in binary64
 *          in K order (error <= K/32 * 2^-53 * sum |terms|, far below the
 *          binary32 rounding that follows);  C = bf16(fp32(acc) + bias).
 *   NVFP4: acc = sum over 16-blocks b of dec(sa_b) dec(sw_b) sum_{k in b} a_k w_k,
 *          exact in 64-bit integers (2^-20 units), rounded once to binary32;
 *          C = bf16(((acc * g_a) * g_w) + bias), each step binary32.
 */
#define QO_FMT_MXFP8 4
#define QO_FMT_NVFP4 5

/* floor(log2(a)) for a finite a > 0, exact (frexp is exact). */
static int floor_log2(double a) {
    int e;
    (void)frexp(a, &e);                       /* a = f * 2^e, f in [0.5, 1) */
    return e - 1;
}

/* E8M0 scale code -> 2^(code - 127); code 0xFF is NaN. */
double qo_e8m0_decode(uint8_t code) {
    if (code == 0xFF) return NAN;
    return ldexp(1.0, (int)code - 127);
}

/* E2M1 magnitudes by code (bits e1 e0 m): 0, 0.5, 1, 1.5, 2, 3, 4, 6. */
static const double kE2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

float qo_e2m1_decode(uint8_t code) {
    double v = kE2M1[code & 7];
    return (float)((code & 8) ? -v : v);
}

/* Nearest E2M1 code to v: the magnitude closest to |v| (values above 6 go to
 * 6), ties to the even code; the sign bit is v's sign, zero included. */
uint8_t qo_e2m1_encode(float v) {
    double a = fabs((double)v);
    if (a > 6.0) a = 6.0;                     /* saturation (keeps the distances exact) */
    int best = 0;
    double bd = a;
    for (int i = 1; i < 8; ++i) {
        double d = fabs(a - kE2M1[i]);
        if (d < bd || (d == bd && (i & 1) == 0)) {
            best = i;
            bd = d;
        }
    }
    return (uint8_t)((signbit(v) ? 8 : 0) | best);
}

/*
 * MXFP8 quantisation.  x: bf16 bits [rows][ld]; cols a multiple of 32.
 * q: [rows][cols] E4M3 codes; sf: [rows][cols/32] E8M0 codes.
 */
void qo_quantize_mxfp8(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* q, uint8_t* sf) {
    const int64_t nb = cols / 32;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b) {
            const uint16_t* xb = x + r * ld + b * 32;
            uint8_t* qb = q + r * cols + b * 32;
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float a = fabsf(qo_bf16_to_f32(xb[i]));
                if (a > amax) amax = a;
            }
            if (amax == 0.0f) {
                sf[r * nb + b] = 0;
                memset(qb, 0, 32);
                continue;
            }
            int e = floor_log2((double)amax) - 8;
            if (e < -127) e = -127;
            if (e > 127) e = 127;
            sf[r * nb + b] = (uint8_t)(e + 127);
            for (int i = 0; i < 32; ++i) {
                double v = ldexp((double)qo_bf16_to_f32(xb[i]), -e);  /* exact */
                qb[i] = qo_e4m3_encode((float)v);                      /* saturates at 448 */
            }
        }
}

/*
 * NVFP4 quantisation with the per-tensor decode scale g > 0.  x: bf16 bits
 * [rows][ld]; cols a multiple of 16.  q: [rows][cols/2] packed E2M1 (element
 * 2i in the low nibble of byte i); sf: [rows][cols/16] E4M3 codes.
 */
void qo_quantize_nvfp4(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, float g, uint8_t* q,
                       uint8_t* sf) {
    const int64_t nb = cols / 16;
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t b = 0; b < nb; ++b) {
            const uint16_t* xb = x + r * ld + b * 16;
            uint8_t* qb = q + r * (cols / 2) + b * 8;
            float amax = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float a = fabsf(qo_bf16_to_f32(xb[i]));
                if (a > amax) amax = a;
            }
            float t = amax / 6.0f;            /* binary32 division */
            t = t / g;                        /* binary32 division */
            const uint8_t s = qo_e4m3_encode(t);
            sf[r * nb + b] = s;
            const float d = qo_e4m3_decode(s) * g;   /* binary32 multiply */
            for (int i = 0; i < 8; ++i) {
                uint8_t lo = 0, hi = 0;
                if (d != 0.0f) {
                    lo = qo_e2m1_encode(qo_bf16_to_f32(xb[2 * i]) / d);
                    hi = qo_e2m1_encode(qo_bf16_to_f32(xb[2 * i + 1]) / d);
                }
                qb[i] = (uint8_t)(lo | (hi << 4));
            }
        }
}

/* E2M1 element of a packed row as an integer count of 1/2. */
static int64_t e2m1_halves(const uint8_t* row, int64_t k) {
    const uint8_t code = (uint8_t)((row[k >> 1] >> ((k & 1) * 4)) & 0xF);
    const int64_t h = (int64_t)(kE2M1[code & 7] * 2.0);
    return (code & 8) ? -h : h;
}

/*
 * Block-scaled GEMM (fmt QO_FMT_MXFP8 or QO_FMT_NVFP4), C = A W^T:
 *   MXFP8: a_q [M][K], a_sf [M][K/32], w_q [N][K], w_sf [N][K/32]; g_a, g_w unused.
 *   NVFP4: a_q [M][K/2] packed, a_sf [M][K/16], w_q [N][K/2], w_sf [N][K/16].
 * K a multiple of 32 (MXFP8) or 16 (NVFP4).  Row/column selection as
 * qo_scaled_mm.  Returns 0, or -2 if an allocation failed.
 */
int qo_gemm_block_scaled(int fmt, int64_t M, int64_t N, int64_t K, const uint8_t* a_q, const uint8_t* a_sf,
                         const uint8_t* w_q, const uint8_t* w_sf, float g_a, float g_w, const uint16_t* bias,
                         const int64_t* m_idx, int64_t m_cnt, const int64_t* n_idx, int64_t n_cnt, uint16_t* c) {
    (void)M;
    (void)N;
    if (!m_idx) m_cnt = M;
    if (!n_idx) n_cnt = N;
    const int mx = (fmt == QO_FMT_MXFP8);
    const int64_t bs = mx ? 32 : 16, nb = K / bs;
    int64_t* ua = (int64_t*)malloc(sizeof(int64_t) * (size_t)(m_cnt * K));
    int64_t* uw = (int64_t*)malloc(sizeof(int64_t) * (size_t)(n_cnt * K));
    if (!ua || !uw) { free(ua); free(uw); return -2; }
    /* elements as exact integers: E4M3 in 2^-9 units, E2M1 in 2^-1 units */
    for (int64_t i = 0; i < m_cnt; ++i) {
        const int64_t m = m_idx ? m_idx[i] : i;
        for (int64_t k = 0; k < K; ++k)
            ua[i * K + k] = mx ? qo_e4m3_units(a_q[m * K + k]) : e2m1_halves(a_q + m * (K / 2), k);
    }
    for (int64_t j = 0; j < n_cnt; ++j) {
        const int64_t n = n_idx ? n_idx[j] : j;
        for (int64_t k = 0; k < K; ++k)
            uw[j * K + k] = mx ? qo_e4m3_units(w_q[n * K + k]) : e2m1_halves(w_q + n * (K / 2), k);
    }
    for (int64_t i = 0; i < m_cnt; ++i) {
        const int64_t m = m_idx ? m_idx[i] : i;
        for (int64_t j = 0; j < n_cnt; ++j) {
            const int64_t n = n_idx ? n_idx[j] : j;
            const int64_t* ra = ua + i * K;
            const int64_t* rw = uw + j * K;
            float y;
            if (mx) {
                double acc = 0.0;
                for (int64_t b = 0; b < nb; ++b) {
                    int64_t p = 0;
                    for (int64_t k = b * 32; k < b * 32 + 32; ++k) p += ra[k] * rw[k];
                    acc += ldexp((double)p, -18) * qo_e8m0_decode(a_sf[m * nb + b])
                           * qo_e8m0_decode(w_sf[n * nb + b]);
                }
                y = (float)acc;               /* one rounding to binary32 */
                if (bias) y = y + qo_bf16_to_f32(bias[n]);
            } else {
                int64_t acc = 0;              /* 2^-20 units: 2^-2 elements x 2^-18 scales */
                for (int64_t b = 0; b < nb; ++b) {
                    int64_t p = 0;
                    for (int64_t k = b * 16; k < b * 16 + 16; ++k) p += ra[k] * rw[k];
                    acc += p * qo_e4m3_units(a_sf[m * nb + b]) * qo_e4m3_units(w_sf[n * nb + b]);
                }
                y = (float)acc;               /* int64 -> binary32, one rounding */
                y = y * 0x1p-20f;             /* exact power-of-two scaling */
                y = y * g_a;
                y = y * g_w;
                if (bias) y = y + qo_bf16_to_f32(bias[n]);
            }
            c[i * n_cnt + j] = qo_f32_to_bf16(y);
        }
    }
    free(ua);
    free(uw);
    return 0;
}
