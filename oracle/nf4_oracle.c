/*
 * nf4_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct CPU statement of the QLoRA frozen-NF4 linear
 * layer: the NF4 codebook, blockwise absmax quantization with 8-bit double
 * quantization of the absmax constants, dequantization to bf16, and the layer
 * Y = X deq(W)^T + s (X A^T) B^T with its backward (dX, dA, dB; W is frozen).
 *
 * Only the tests, the package's smoke check and the benchmark's CPU-baseline
 * leg may load this library.  It shares no code, header, table or constant
 * generator with the CUDA library; the two are meant to be compared.
 *
 * Arithmetic rules:
 *  - Everything that the method defines in fp32 (x/a, the midpoints, the
 *    double-quant scale, the dequant products) is computed in fp64 and rounded
 *    to fp32 after every single operation.  For + - * / this equals the IEEE
 *    fp32 result exactly, because 53 >= 2*24 + 2.
 *  - The layer sums are exact fp64 sums of products of bf16 values (each
 *    product of two bf16 numbers is exact in fp64); no intermediate rounding.
 *
 * Sources (web pages on QLoRA, cited by title and section):
 *  - "What does QLoRA change compared with plain LoRA when fine-tuning Llama?"
 *    (katajob), sections "NF4: 4-bit NormalFloat" and "Double quantization":
 *    16 levels placed for a zero-centred normal, blockwise scaling with blocks
 *    of (commonly) 64 contiguous weights, scales re-quantized to 8 bits with a
 *    second-level scale over groups of them, per-block dequantization to bf16
 *    inside the matmul.
 *  - "QLoRA and Quantized Fine-Tuning" (quantmemo), "The two mechanisms
 *    combined": W' = W_4bit + BA, only A and B are trained.
 *  - "QLoRA: fine-tuning a large model on one GPU" (pranaymahendrakar),
 *    "LoRA, stated once": h = W0 x + (alpha/r) B A x, B in R^{d x r},
 *    A in R^{r x k}; gradients flow through the dequantized weights to the
 *    adapters and the quantized weights receive no update.
 * Readings where the pages are silent (the quantile construction with an exact
 * zero, the top probability delta, midpoint ties, nibble order, the unsigned
 * 8-bit absmax code with a per-group max/255 scale) are stated next to the code
 * that implements them.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_OK 0
#define OR_ERR_ARG (-1)
#define OR_ERR_SHAPE (-2)
#define OR_ERR_NONFINITE (-3)

/* ---------------------------------------------------------------- helpers */

/* Round an fp64 value to the nearest fp32 (ties to even: the C conversion). */
static float r32(double v) { return (float)v; }

/* bf16 bits -> exact value. */
static double bf16_to_f64(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* fp32 -> bf16 bits, round to nearest, ties to even (the IEEE default mode
 * applied to the 8-bit significand of bfloat16).  NaN maps to a quiet NaN. */
static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return 0x7fc0;
    uint32_t lower = u & 0xffffu;      /* the 16 bits that are dropped */
    uint32_t upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1u;
    return (uint16_t)upper;
}

/* Round half to even to an integer value (used for the 8-bit absmax code). */
static double round_half_even(double v) {
    double f = floor(v);
    double d = v - f;
    if (d > 0.5) return f + 1.0;
    if (d < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* ------------------------------------------------------- NF4 codebook (a1) */

/* Standard normal CDF from its definition through the complementary error
 * function: Phi(x) = erfc(-x / sqrt 2) / 2. */
static double phi_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* Inverse of Phi by plain bisection: Phi is strictly increasing, so halving a
 * bracket that always keeps Phi(lo) < p <= Phi(hi) converges to the quantile.
 * Stops when the bracket no longer shrinks (adjacent doubles). */
static double phi_inv(double p) {
    double lo = -40.0, hi = 40.0;
    for (int it = 0; it < 2000; ++it) {
        double mid = 0.5 * (lo + hi);
        if (mid <= lo || mid >= hi) break;
        if (phi_cdf(mid) < p) lo = mid; else hi = mid;
    }
    return 0.5 * (lo + hi);
}

/* The top probability used for the outermost levels.  Reading: the pages say
 * only that the 16 levels suit zero-centred normal weights (and the layer needs
 * an exact zero); the plainest construction uses equal-probability
 * quantiles on each side of zero, and delta is taken as the mean of the centres
 * of the top equal-mass bins of a 16-bin and a 15-bin split of the line:
 * delta = 1 - (1/32 + 1/30) / 2. */
double or_nf4_delta(void) { return 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0); }

/* levels64[16]: exact (fp64) levels; levels32[16]: rounded to fp32;
 * mids32[15]: decision thresholds fl32(L_i + L_{i+1}) / 2.
 * Construction (reading, see or_nf4_delta): 8 positive levels at the
 * quantiles p_j = 1/2 + j (delta - 1/2)/8, j = 1..8; 7 negative levels at
 * -Phi^-1(q_j), q_j = 1/2 + j (delta - 1/2)/7, j = 1..7; one exact zero;
 * all divided by Phi^-1(delta) so that the range is exactly [-1, 1]. */
int or_nf4_codebook(double* levels64, float* levels32, float* mids32) {
    if (!levels64 && !levels32 && !mids32) return OR_ERR_ARG;
    const double delta = or_nf4_delta();
    const double z = phi_inv(delta);
    double lv[16];
    lv[7] = 0.0;
    for (int j = 1; j <= 8; ++j) {
        double p = 0.5 + (double)j * (delta - 0.5) / 8.0;
        lv[7 + j] = phi_inv(p) / z;
    }
    for (int j = 1; j <= 7; ++j) {
        double q = 0.5 + (double)j * (delta - 0.5) / 7.0;
        lv[7 - j] = -phi_inv(q) / z;
    }
    float l32[16];
    for (int i = 0; i < 16; ++i) l32[i] = r32(lv[i]);
    if (levels64) for (int i = 0; i < 16; ++i) levels64[i] = lv[i];
    if (levels32) for (int i = 0; i < 16; ++i) levels32[i] = l32[i];
    if (mids32)
        for (int i = 0; i < 15; ++i)
            mids32[i] = r32((double)r32((double)l32[i] + (double)l32[i + 1]) * 0.5);
    return OR_OK;
}

/* ------------------------------------------------- sizes of the NF4 format */

/* codes: two 4-bit codes per byte; absmax_q: one byte per block; dq_scale:
 * one fp32 per group of dq_block consecutive blocks (last group may be short). */
/* dq_block == 0 means no double quantization: the exact fp32 absmax of every
 * block is stored (dq_count = number of blocks, in the fp32 array) and the
 * 8-bit array is empty. */
int or_nf4_sizes(int64_t N, int64_t K, int block, int dq_block,
                 int64_t* codes_bytes, int64_t* absmax_bytes, int64_t* dq_count) {
    if (N < 0 || K < 0 || block <= 0 || dq_block < 0) return OR_ERR_ARG;
    if (block % 2 || K % block) return OR_ERR_SHAPE;
    int64_t numel = N * K, nblocks = numel / block;
    if (codes_bytes) *codes_bytes = numel / 2;
    if (absmax_bytes) *absmax_bytes = dq_block ? nblocks : 0;
    if (dq_count) *dq_count = dq_block ? (nblocks + dq_block - 1) / dq_block : nblocks;
    return OR_OK;
}

/* ------------------------------------------- quantize: a2, a3, a4 (fp32) */

/* W is [N, K] row-major fp32, flattened; block b covers elements
 * [b*block, (b+1)*block) and never straddles a row because K % block == 0.
 *  a2: a_b = max |x| over the block (exact in fp32).
 *  a3: t = fl32(x / a_b); code = number of midpoints strictly below t
 *      (a tie t == M_i takes the lower code); a zero block gives code 7 (the
 *      exact zero level) for every element.  Packing: byte j holds element 2j
 *      in its low nibble and element 2j+1 in its high nibble.
 *  a4: groups of dq_block consecutive blocks; c2 = max a_b over the group;
 *      s2 = fl32(c2 / 255) (0 when c2 == 0); q_b = min(255, rne(fl32(a_b/s2)))
 *      (0 when s2 == 0): an unsigned linear 8-bit code of the non-negative
 *      absmax values.  With dq_block == 0 (no double quantization) dq_scale
 *      receives a_b itself and absmax_q is not used.
 * absmax_out (nullable) receives the exact a_b. */
int or_nf4_quantize(const float* W, int64_t N, int64_t K, int block, int dq_block,
                    uint8_t* codes, uint8_t* absmax_q, float* dq_scale, float* absmax_out) {
    if (!W || !codes || (dq_block && !absmax_q) || !dq_scale) return OR_ERR_ARG;
    int64_t cb, ab, dc;
    int st = or_nf4_sizes(N, K, block, dq_block, &cb, &ab, &dc);
    if (st) return st;
    const int64_t numel = N * K, nblocks = numel / block;
    (void)ab;
    for (int64_t i = 0; i < numel; ++i)
        if (!isfinite(W[i])) return OR_ERR_NONFINITE;

    float mids[15];
    or_nf4_codebook(NULL, NULL, mids);

    float* a = (float*)malloc(sizeof(float) * (size_t)(nblocks ? nblocks : 1));
    if (!a) return OR_ERR_ARG;

#pragma omp parallel for schedule(static)
    for (int64_t b = 0; b < nblocks; ++b) {
        const float* x = W + b * block;
        float m = 0.0f;
        for (int e = 0; e < block; ++e) {
            float v = fabsf(x[e]);
            if (v > m) m = v;
        }
        a[b] = m;
        for (int e = 0; e < block; e += 2) {
            int c[2];
            for (int h = 0; h < 2; ++h) {
                if (m == 0.0f) { c[h] = 7; continue; }
                float t = r32((double)x[e + h] / (double)m);
                int code = 0;
                for (int i = 0; i < 15; ++i) if (t > mids[i]) ++code;
                c[h] = code;
            }
            codes[(b * block + e) / 2] = (uint8_t)(c[0] | (c[1] << 4));
        }
    }

    if (dq_block == 0) {
        for (int64_t b = 0; b < nblocks; ++b) dq_scale[b] = a[b];
        dc = 0;  /* no groups */
    }
    for (int64_t g = 0; g < dc; ++g) {
        int64_t b0 = g * dq_block, b1 = b0 + dq_block;
        if (b1 > nblocks) b1 = nblocks;
        float c2 = 0.0f;
        for (int64_t b = b0; b < b1; ++b) if (a[b] > c2) c2 = a[b];
        float s2 = (c2 > 0.0f) ? r32((double)c2 / 255.0) : 0.0f;
        dq_scale[g] = s2;
        for (int64_t b = b0; b < b1; ++b) {
            if (s2 == 0.0f) { absmax_q[b] = 0; continue; }
            double q = round_half_even((double)r32((double)a[b] / (double)s2));
            if (q > 255.0) q = 255.0;
            absmax_q[b] = (uint8_t)q;
        }
    }
    if (absmax_out) memcpy(absmax_out, a, sizeof(float) * (size_t)nblocks);
    free(a);
    return OR_OK;
}

/* ------------------------------------------------------------ dequant: a5 */

/* a'_b = fl32(q_b * s2_g);  w' = bf16_rne(fl32(L[code] * a'_b)).
 * Writes bf16 bits (out_bf16, nullable) and/or the same values as fp32
 * (out_f32, nullable; exact, since every bf16 value is an fp32 value). */
int or_nf4_dequantize(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                      int64_t N, int64_t K, int block, int dq_block,
                      uint16_t* out_bf16, float* out_f32) {
    if (!codes || (dq_block && !absmax_q) || !dq_scale || (!out_bf16 && !out_f32)) return OR_ERR_ARG;
    int64_t cb, ab, dc;
    int st = or_nf4_sizes(N, K, block, dq_block, &cb, &ab, &dc);
    if (st) return st;
    float L[16];
    or_nf4_codebook(NULL, L, NULL);
    const int64_t numel = N * K;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < numel; ++i) {
        int64_t b = i / block;
        uint8_t byte = codes[i / 2];
        int code = (i % 2 == 0) ? (byte & 0xf) : (byte >> 4);
        /* the block scale: q_b * s2 of its group, or the stored fp32 absmax */
        float ap = dq_block ? r32((double)absmax_q[b] * (double)dq_scale[b / dq_block]) : dq_scale[b];
        float w = r32((double)L[code] * (double)ap);
        uint16_t h = f32_to_bf16_rne(w);
        if (out_bf16) out_bf16[i] = h;
        if (out_f32) out_f32[i] = (float)bf16_to_f64(h);
    }
    return OR_OK;
}

/* ------------------------------------------- merge and re-quantize (f2) */

/* After training the adapter is folded into the frozen weight ("QLoRA and
 * Quantized Fine-Tuning", "The two mechanisms combined": the model computes
 * with W' + BA) and the sum is stored as NF4 again:
 *   w'[n,k]    = the dequantized weight the layer uses (bf16 value, in fp32)
 *   delta[n,k] = sum_j B[n,j] A[j,k], accumulated in fp32 in the order
 *                j = 0 .. r-1 (each product of two bf16 values is exact in fp32)
 *   merged     = fl32(w' + fl32(s * delta))
 * then quantized with or_nf4_quantize in the output format.  The sum order is
 * fixed so that the fp32 value, and hence every code, is reproducible. */
int or_nf4_merge_lora(const uint8_t* codes, const uint8_t* absmax_q, const float* dq_scale,
                      int block, int dq_block, int64_t N, int64_t K,
                      const uint16_t* A, const uint16_t* B, int r, float s,
                      int out_block, int out_dq_block, uint8_t* out_codes, uint8_t* out_absmax_q,
                      float* out_dq_scale, float* merged_out) {
    if (!A || !B || r <= 0 || !out_codes || !out_dq_scale) return OR_ERR_ARG;
    const int64_t numel = N * K;
    float* wp = (float*)malloc(sizeof(float) * (size_t)(numel ? numel : 1));
    if (!wp) return OR_ERR_ARG;
    int st = or_nf4_dequantize(codes, absmax_q, dq_scale, N, K, block, dq_block, NULL, wp);
    if (st) { free(wp); return st; }
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            float acc = 0.0f;
            for (int j = 0; j < r; ++j)
                acc = r32((double)acc + bf16_to_f64(B[n * r + j]) * bf16_to_f64(A[(int64_t)j * K + k]));
            wp[n * K + k] = r32((double)wp[n * K + k] + (double)r32((double)s * (double)acc));
        }
    if (merged_out) memcpy(merged_out, wp, sizeof(float) * (size_t)numel);
    st = or_nf4_quantize(wp, N, K, out_block, out_dq_block, out_codes, out_absmax_q, out_dq_scale, NULL);
    free(wp);
    return st;
}

/* ------------------------------------------------ LoRA dropout input (f4) */

/* The adapter branch sees dropout(X) ("QLoRA: fine-tuning a large model on
 * one GPU": lora_dropout in the LoraConfig): Xd = X * keep where the mask
 * keeps the element, else 0, rounded to bf16 like any bf16 product:
 *   Xd[i] = mask[i] ? bf16_rne(fl32(X[i] * keep)) : 0.
 * The random draw is an input (mask, 1 = keep); keep = 1 / (1 - p). */
int or_dropout_input(const uint16_t* X, const uint8_t* mask, float keep, int64_t n, uint16_t* Xd) {
    if (!X || !mask || !Xd || n < 0) return OR_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        Xd[i] = mask[i] ? f32_to_bf16_rne(r32(bf16_to_f64(X[i]) * (double)keep)) : (uint16_t)0;
    return OR_OK;
}

/* bf16 rounding exposed for the tests that pin it against textbook values. */
uint16_t or_f32_to_bf16(float f) { return f32_to_bf16_rne(f); }

/* ------------------------------------------------------ the layer: a6..a9 */

/* H = X A^T, [M, r], exact.  X bf16 [M,K]; A bf16 [r,K]. */
int or_lora_h(const uint16_t* X, int64_t M, int64_t K, const uint16_t* A, int r, double* H) {
    if (!X || !A || !H || M < 0 || K < 0 || r <= 0) return OR_ERR_ARG;
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += bf16_to_f64(X[m * K + k]) * bf16_to_f64(A[(int64_t)j * K + k]);
            H[m * r + j] = acc;
        }
    return OR_OK;
}

/* Forward (a6 + a7) for the rows listed in `rows` (all rows when rows is
 * NULL, then nrows must equal M):
 *   Y[m, n] = sum_k X[m,k] Wp[n,k] + s * sum_j H[m,j] B[n,j],  H = X A^T.
 * Wp is the dequantized weight [N,K] (bf16 values held in fp32).
 * Y is [nrows, N] fp64. */
int or_linear_fwd(const uint16_t* X, int64_t M, int64_t K, const float* Wp, int64_t N,
                  const uint16_t* A, const uint16_t* B, int r, double s,
                  const int64_t* rows, int64_t nrows, double* Y) {
    if (!X || !Wp || !A || !B || !Y || r <= 0) return OR_ERR_ARG;
    if (!rows && nrows != M) return OR_ERR_ARG;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        if (m < 0 || m >= M) { bad = 1; continue; }
        const uint16_t* xr = X + m * K;
        double* h = (double*)malloc(sizeof(double) * (size_t)r);
        for (int j = 0; j < r; ++j) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; ++k)
                acc += bf16_to_f64(xr[k]) * bf16_to_f64(A[(int64_t)j * K + k]);
            h[j] = acc;
        }
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0;
            const float* wr = Wp + n * K;
            for (int64_t k = 0; k < K; ++k) acc += bf16_to_f64(xr[k]) * (double)wr[k];
            double lora = 0.0;
            for (int j = 0; j < r; ++j) lora += h[j] * bf16_to_f64(B[n * r + j]);
            Y[i * N + n] = acc + s * lora;
        }
        free(h);
    }
    return bad ? OR_ERR_ARG : OR_OK;
}

/* Multi-adapter forward (f3; "QLoRA and Quantized Fine-Tuning": one frozen
 * base, many small adapters): token m uses adapter a = idx[m] of a stack,
 *   Y[m, n] = sum_k X[m,k] Wp[n,k] + s_a * sum_j H[m,j] B_a[n,j],  H = X A_a^T,
 * A_all bf16 [na, r, K], B_all bf16 [na, N, r], scales fp64 [na], idx [M].
 * Y is [M, N] fp64.  An index outside [0, na) is an argument error. */
int or_linear_fwd_multi(const uint16_t* X, int64_t M, int64_t K, const float* Wp, int64_t N,
                        const uint16_t* A_all, const uint16_t* B_all, int na, int r, const double* scales,
                        const int32_t* idx, double* Y) {
    if (!X || !Wp || !A_all || !B_all || !scales || !idx || !Y || r <= 0 || na <= 0) return OR_ERR_ARG;
    for (int64_t m = 0; m < M; ++m)
        if (idx[m] < 0 || idx[m] >= na) return OR_ERR_ARG;
    for (int64_t m = 0; m < M; ++m) {
        const int a = idx[m];
        int st = or_linear_fwd(X, M, K, Wp, N, A_all + (int64_t)a * r * K, B_all + (int64_t)a * N * r, r,
                               scales[a], &m, 1, Y + m * N);
        if (st) return st;
    }
    return OR_OK;
}

/* Backward (a8 + a9).  With upstream gradient dY [M,N]:
 *   dH[m,j] = s * sum_n dY[m,n] B[n,j]                       [M, r]
 *   dX[m,k] = sum_n dY[m,n] Wp[n,k] + sum_j dH[m,j] A[j,k]   rows listed
 *   dA[j,k] = sum_m dH[m,j] X[m,k]                           [r, K]
 *   dB[n,j] = s * sum_m dY[m,n] H[m,j],  H = X A^T           [N, r]
 * No gradient is produced for W (the frozen base).
 * dX is [nrows, K]; dA, dB full; dH (nullable) receives [M, r]. */
int or_linear_bwd(const uint16_t* X, const uint16_t* dY, int64_t M, int64_t K,
                  const float* Wp, int64_t N, const uint16_t* A, const uint16_t* B, int r, double s,
                  const int64_t* rows, int64_t nrows,
                  double* dX, double* dA, double* dB, double* dH_out) {
    if (!X || !dY || !Wp || !A || !B || r <= 0) return OR_ERR_ARG;
    if (nrows > 0 && !dX) return OR_ERR_ARG;
    if (!rows && nrows != M && nrows != 0) return OR_ERR_ARG;
    double* H = (double*)malloc(sizeof(double) * (size_t)(M * r + 1));
    double* dH = (double*)malloc(sizeof(double) * (size_t)(M * r + 1));
    if (!H || !dH) { free(H); free(dH); return OR_ERR_ARG; }
    or_lora_h(X, M, K, A, r, H);
    /* dH: for each row m the sum over n runs in ascending n. */
#pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; ++m) {
        double* acc = dH + m * r;
        for (int j = 0; j < r; ++j) acc[j] = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            double g = bf16_to_f64(dY[m * N + n]);
            for (int j = 0; j < r; ++j) acc[j] += g * bf16_to_f64(B[n * r + j]);
        }
        for (int j = 0; j < r; ++j) acc[j] *= s;
    }
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t m = rows ? rows[i] : i;
        if (m < 0 || m >= M) { bad = 1; continue; }
        double* out = dX + i * K;
        for (int64_t k = 0; k < K; ++k) out[k] = 0.0;
        for (int64_t n = 0; n < N; ++n) {
            double g = bf16_to_f64(dY[m * N + n]);
            const float* wr = Wp + n * K;
            for (int64_t k = 0; k < K; ++k) out[k] += g * (double)wr[k];
        }
        for (int j = 0; j < r; ++j) {
            double g = dH[m * r + j];
            for (int64_t k = 0; k < K; ++k) out[k] += g * bf16_to_f64(A[(int64_t)j * K + k]);
        }
    }
    /* dA and dB: each output element is a sum over m in ascending m; the loops
     * are nested m-outer only so that X and dY are read row by row. */
    const int64_t CH = 256;
    if (dA) {
        int64_t nch = (K + CH - 1) / CH;
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t c = 0; c < nch; ++c) {
            int64_t k0 = c * CH, k1 = k0 + CH < K ? k0 + CH : K;
            double* acc = (double*)calloc((size_t)(r * CH), sizeof(double));
            for (int64_t m = 0; m < M; ++m)
                for (int j = 0; j < r; ++j) {
                    double g = dH[m * r + j];
                    for (int64_t k = k0; k < k1; ++k)
                        acc[j * CH + (k - k0)] += g * bf16_to_f64(X[m * K + k]);
                }
            for (int j = 0; j < r; ++j)
                for (int64_t k = k0; k < k1; ++k) dA[(int64_t)j * K + k] = acc[j * CH + (k - k0)];
            free(acc);
        }
    }
    if (dB) {
        int64_t nch = (N + CH - 1) / CH;
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t c = 0; c < nch; ++c) {
            int64_t n0 = c * CH, n1 = n0 + CH < N ? n0 + CH : N;
            double* acc = (double*)calloc((size_t)(r * CH), sizeof(double));
            for (int64_t m = 0; m < M; ++m)
                for (int64_t n = n0; n < n1; ++n) {
                    double g = bf16_to_f64(dY[m * N + n]);
                    for (int j = 0; j < r; ++j) acc[(n - n0) * r + j] += g * H[m * r + j];
                }
            for (int64_t n = n0; n < n1; ++n)
                for (int j = 0; j < r; ++j) dB[n * r + j] = s * acc[(n - n0) * r + j];
            free(acc);
        }
    }
    if (dH_out) memcpy(dH_out, dH, sizeof(double) * (size_t)(M * r));
    free(H);
    free(dH);
    return bad ? OR_ERR_ARG : OR_OK;
}

/* Number of OpenMP threads the oracle will use (reported with CPU timings). */
#ifdef _OPENMP
#include <omp.h>
int or_num_threads(void) { return omp_get_max_threads(); }
#else
int or_num_threads(void) { return 1; }
#endif
