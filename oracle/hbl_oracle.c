/*
 * hbl_oracle.c -- plain, slow, scalar CPU oracle for the H-BitLinear forward
 * pass (BitNet v2).  TEST INFRASTRUCTURE ONLY: the library never links,
 * loads or calls this file.  It exists so that tests, the smoke check and the
 * CPU baseline of the benchmark have an independent statement of what the
 * GPU path must compute.  It shares no code, header, table or constant
 * generator with the CUDA library.
 *
 * Sources (web pages on BitNet v2; formulas on them were images and did not
 * survive extraction, so each formula below is the plain reading stated next
 * to it):
 *   [P2] 0755model.com write-up of BitNet v2, sections "BitNet v2：原生4位激活"
 *        and "H-BitLinear": LLaMA-like blocks with RMS normalisation and no
 *        bias; per-tensor absmean ternary weights {-1,0,1}; an online Hadamard
 *        transform before activation quantisation, computed with the fast
 *        Hadamard transform in O(n log n); Hadamard matrices have +-1 entries
 *        and mutually orthogonal rows; INT8 and INT4 activation quantisers;
 *        the layer is LN -> Hadamard -> quantise -> ternary matmul.
 *   [P4] shengxinai.com explainer, section 2.2 "原生4位激活量化的突破":
 *        a 4-bit activation takes one of 16 values.
 *   [P3] CSDN post "[论文品鉴] 1-bit LLM", section "掩码存储": ternary weights
 *        are stored by packing several values into one integer.
 *   [P2-QKV] the same 0755model.com write-up, section "实验结果" (low-bit
 *        attention, tables 2 and 3): Q, K and V states are quantised after RoPE,
 *        per head, with absmax, directly to unsigned integers, no calibration;
 *        a 3-bit KV cache is reported.
 *   [P2-ABL] the same write-up, table 5 (Hadamard ablation): the rotation is
 *        applied to weights and activations, or to activations only; section
 *        on post-training baselines: QuaRot uses a randomised Hadamard transform.
 *
 * Arithmetic: IEEE binary32, round-to-nearest-even, no contraction (build with
 * -ffp-contract=off).  Where fp32 results depend on evaluation order the order
 * is fixed here and is part of the definition:
 *   - sums (sum of squares, sum of |v|, sum of |W|) use the left-complete
 *     pairwise tree over index order (tree_sum below);
 *   - the Walsh-Hadamard butterflies run stage h = 1, 2, 4, ..., n/2 in that
 *     order, each stage mapping (a, b) -> (a + b, a - b) with a the lower index;
 *   - the 1/sqrt(n) normalisation is one multiply after the last stage.
 * The fp64 variants exist only to bound the fp32 results in tests.
 *
 * Parity status of each function is recorded in oracle/__init__.py.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

/* ---------------------------------------------------------------- helpers */

static int is_pow2_i64(int64_t n) { return n > 0 && (n & (n - 1)) == 0; }

/* Left-complete pairwise tree over index order:
 *   sum(v[0..m)) = sum(v[0..h)) + sum(v[h..m)),  h = largest power of two < m.
 * For m a power of two this is the perfect tree (h = m/2). */
static float tree_sum_f32(const float* v, int64_t m) {
    if (m <= 0) return 0.0f;
    if (m == 1) return v[0];
    int64_t h = 1;
    while (h * 2 < m) h *= 2;
    float a = tree_sum_f32(v, h);
    float b = tree_sum_f32(v + h, m - h);
    return a + b;
}

static double tree_sum_f64(const double* v, int64_t m) {
    if (m <= 0) return 0.0;
    if (m == 1) return v[0];
    int64_t h = 1;
    while (h * 2 < m) h *= 2;
    return tree_sum_f64(v, h) + tree_sum_f64(v + h, m - h);
}

ORACLE_API float oracle_tree_sum(const float* v, int64_t m) { return tree_sum_f32(v, m); }

/* bf16 is the top half of a binary32; widening is exact. */
ORACLE_API float oracle_bf16_to_f32(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* binary32 -> bf16, round to nearest, ties to even; NaN stays NaN (quiet). */
ORACLE_API uint16_t oracle_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------ Hadamard [P2] */

/* Sylvester construction: H_1 = [1], H_2m = [[H_m, H_m], [H_m, -H_m]].
 * Row-major n x n, entries +-1.  n must be a power of two. */
ORACLE_API int oracle_sylvester(int n, int8_t* H) {
    if (!is_pow2_i64(n)) return -1;
    H[0] = 1;
    for (int m = 1; m < n; m *= 2) {
        for (int i = 0; i < m; ++i)
            for (int j = 0; j < m; ++j) {
                int8_t h = H[(int64_t)i * n + j];
                H[(int64_t)i * n + (j + m)] = h;
                H[(int64_t)(i + m) * n + j] = h;
                H[(int64_t)(i + m) * n + (j + m)] = (int8_t)(-h);
            }
    }
    return 0;
}

/* Fast Walsh-Hadamard transform, unnormalised, in place: u <- u . H_n.
 * Stages h = 1, 2, ..., n/2 ascending; butterfly (a, b) -> (a + b, a - b). */
ORACLE_API int oracle_fwht_f32(float* u, int n) {
    if (!is_pow2_i64(n)) return -1;
    for (int h = 1; h < n; h *= 2)
        for (int i = 0; i < n; ++i)
            if ((i & h) == 0) {
                float a = u[i], b = u[i + h];
                u[i] = a + b;
                u[i + h] = a - b;
            }
    return 0;
}

ORACLE_API int oracle_fwht_f64(double* u, int n) {
    if (!is_pow2_i64(n)) return -1;
    for (int h = 1; h < n; h *= 2)
        for (int i = 0; i < n; ++i)
            if ((i & h) == 0) {
                double a = u[i], b = u[i + h];
                u[i] = a + b;
                u[i + h] = a - b;
            }
    return 0;
}

/* 1/sqrt(n) rounded to binary32 (computed in binary64, rounded once). */
ORACLE_API float oracle_inv_sqrt_n(int n) { return (float)(1.0 / sqrt((double)n)); }

/* sqrt(7) rounded to binary32: the INT4 absmean quantiser's scale constant. */
ORACLE_API float oracle_sqrt7(void) { return (float)sqrt(7.0); }

/* -------------------------------------------------------- RMSNorm [P2] */

/* One row: r = 1 / sqrt(tree_sum(x*x) * (1/K) + eps);  u = (x * r) * g.
 * The page glosses the layer's "LN" as layer normalisation while the model
 * description uses RMS normalisation without bias; the RMS reading is taken. */
static void rmsnorm_row_f32(const uint16_t* xb, const float* gain, int K, float norm_eps,
                            float* u, float* scratch) {
    /* The plain reading of "sum of x^2": every square x*x is one binary32
     * multiply (rounded), and the K squares are summed by the pairwise tree. */
    for (int k = 0; k < K; ++k) {
        float x = oracle_bf16_to_f32(xb[k]);
        scratch[k] = x * x;
    }
    float ss = tree_sum_f32(scratch, K);
    float ms = ss * (1.0f / (float)K);
    float r = 1.0f / sqrtf(ms + norm_eps);
    for (int k = 0; k < K; ++k) {
        float x = oracle_bf16_to_f32(xb[k]);
        float v = x * r;
        if (gain) v = v * gain[k];
        u[k] = v;
    }
}

ORACLE_API int oracle_rmsnorm(const uint16_t* X, const float* gain, int M, int K,
                              float norm_eps, float* U) {
    if (M < 0 || !is_pow2_i64(K)) return -1;
    float* scratch = (float*)malloc(sizeof(float) * (size_t)K);
    if (!scratch) return -2;
    for (int m = 0; m < M; ++m)
        rmsnorm_row_f32(X + (int64_t)m * K, gain, K, norm_eps, U + (int64_t)m * K, scratch);
    free(scratch);
    return 0;
}

/* -------------------------------------------- norm + online Hadamard [P2] */

/* V = FWHT(RMSNorm(X)) * (1/sqrt(K)), fp32, one row at a time. */
ORACLE_API int oracle_norm_fwht(const uint16_t* X, const float* gain, int M, int K,
                                float norm_eps, float* V) {
    if (M < 0 || !is_pow2_i64(K)) return -1;
    float* scratch = (float*)malloc(sizeof(float) * (size_t)K);
    if (!scratch) return -2;
    const float c = oracle_inv_sqrt_n(K);
    for (int m = 0; m < M; ++m) {
        float* v = V + (int64_t)m * K;
        rmsnorm_row_f32(X + (int64_t)m * K, gain, K, norm_eps, v, scratch);
        oracle_fwht_f32(v, K);
        for (int k = 0; k < K; ++k) v[k] = v[k] * c;
    }
    free(scratch);
    return 0;
}

/* The same map in binary64 throughout (used only to bound the fp32 result). */
ORACLE_API int oracle_norm_fwht_f64(const uint16_t* X, const float* gain, int M, int K,
                                    double norm_eps, double* V) {
    if (M < 0 || !is_pow2_i64(K)) return -1;
    double* sq = (double*)malloc(sizeof(double) * (size_t)K);
    if (!sq) return -2;
    const double c = 1.0 / sqrt((double)K);
    for (int m = 0; m < M; ++m) {
        const uint16_t* xb = X + (int64_t)m * K;
        double* v = V + (int64_t)m * K;
        for (int k = 0; k < K; ++k) {
            double x = (double)oracle_bf16_to_f32(xb[k]);
            sq[k] = x * x;
        }
        double r = 1.0 / sqrt(tree_sum_f64(sq, K) / (double)K + norm_eps);
        for (int k = 0; k < K; ++k) {
            double x = (double)oracle_bf16_to_f32(xb[k]);
            v[k] = x * r * (gain ? (double)gain[k] : 1.0);
        }
        oracle_fwht_f64(v, K);
        for (int k = 0; k < K; ++k) v[k] *= c;
    }
    free(sq);
    return 0;
}

/* ------------------------------------- variants: LayerNorm, no Hadamard [P2] */

/* LayerNorm without bias, one row:
 *   mu  = tree_sum(x) * (1/K);  d = x - mu;
 *   var = tree_sum(d*d) * (1/K)   (every square d*d rounded to binary32, as
 *                                  in the RMS sum of squares);
 *   u   = (d * (1 / sqrt(var + eps))) * g.
 * [P2] writes the layer as LN(.) and glosses it as layer normalisation. */
static void layernorm_row_f32(const uint16_t* xb, const float* gain, int K, float norm_eps,
                              float* u, float* scratch) {
    for (int k = 0; k < K; ++k) u[k] = oracle_bf16_to_f32(xb[k]);
    float mu = tree_sum_f32(u, K) * (1.0f / (float)K);
    for (int k = 0; k < K; ++k) u[k] = u[k] - mu;
    for (int k = 0; k < K; ++k) scratch[k] = u[k] * u[k];
    float var = tree_sum_f32(scratch, K) * (1.0f / (float)K);
    float r = 1.0f / sqrtf(var + norm_eps);
    for (int k = 0; k < K; ++k) {
        float v = u[k] * r;
        if (gain) v = v * gain[k];
        u[k] = v;
    }
}

/* V = T(N(X)): N = RMSNorm (layernorm == 0) or LayerNorm (layernorm != 0);
 * T = the normalised Walsh-Hadamard transform (hadamard != 0) or the identity
 * (the plain BitLinear of the layers without H).  norm_fwht is the case
 * (layernorm, hadamard) = (0, 1). */
ORACLE_API int oracle_norm_transform(const uint16_t* X, const float* gain, int M, int K,
                                     float norm_eps, int layernorm, int hadamard, float* V) {
    if (M < 0 || !is_pow2_i64(K)) return -1;
    float* scratch = (float*)malloc(sizeof(float) * (size_t)K);
    if (!scratch) return -2;
    const float c = oracle_inv_sqrt_n(K);
    for (int m = 0; m < M; ++m) {
        float* v = V + (int64_t)m * K;
        if (layernorm)
            layernorm_row_f32(X + (int64_t)m * K, gain, K, norm_eps, v, scratch);
        else
            rmsnorm_row_f32(X + (int64_t)m * K, gain, K, norm_eps, v, scratch);
        if (hadamard) {
            oracle_fwht_f32(v, K);
            for (int k = 0; k < K; ++k) v[k] = v[k] * c;
        }
    }
    free(scratch);
    return 0;
}

/* ------------------------------------------- activation quantisers [P2][P4] */

/* Quantise fp32 rows V [M x K] per token.  A zero row with eps = 0 would divide
 * by zero; inv is then taken as 0, so the row quantises to zeros (scale 0), as
 * it does for any eps > 0.
 *   act_bits = 8 (absmax):  gamma = max|v|;  q = clip(round(v * (127/(gamma+eps))), -128, 127);
 *                           scale = gamma / 127.
 *   act_bits = 4 (absmean): beta = tree_sum(|v|) * (1/K);
 *                           q = clip(round(v * (sqrt7/(beta+eps))), -8, 7);  scale = beta / sqrt7.
 * round = nearest, ties to even.  The reciprocal constant inv = C/(x+eps) is one
 * IEEE division per row; each code rounds the exact product v * inv (the
 * product of two binary32 numbers is exact in binary64) once to an integer.
 * Codes: act_bits 8 -> one int8 per element, row-major [M x K];
 *        act_bits 4 -> two's-complement nibbles, element 2j in the low nibble of
 *        byte j of the row, [M x K/2].
 * rowsum (nullable) = sum of the row's integer codes. */
static int8_t clip_round(double y, int lo, int hi) {
    double r = rint(y);
    if (r < (double)lo) r = (double)lo;
    if (r > (double)hi) r = (double)hi;
    return (int8_t)r;
}

ORACLE_API int oracle_quantize_rows(const float* V, int M, int K, float quant_eps, int act_bits,
                                    uint8_t* codes, float* scales, int32_t* rowsum) {
    if (M < 0 || !is_pow2_i64(K) || K < 2) return -1;
    if (act_bits != 4 && act_bits != 8) return -1;
    float* absv = (float*)malloc(sizeof(float) * (size_t)K);
    int8_t* q = (int8_t*)malloc((size_t)K);
    if (!absv || !q) { free(absv); free(q); return -2; }
    const float s7 = oracle_sqrt7();
    for (int m = 0; m < M; ++m) {
        const float* v = V + (int64_t)m * K;
        float inv, scale;
        int lo, hi;
        if (act_bits == 8) {
            float g = 0.0f;
            for (int k = 0; k < K; ++k) { float a = fabsf(v[k]); if (a > g) g = a; }
            inv = (g + quant_eps) > 0.0f ? 127.0f / (g + quant_eps) : 0.0f;
            scale = g / 127.0f;
            lo = -128; hi = 127;
        } else {
            for (int k = 0; k < K; ++k) absv[k] = fabsf(v[k]);
            float beta = tree_sum_f32(absv, K) * (1.0f / (float)K);
            inv = (beta + quant_eps) > 0.0f ? s7 / (beta + quant_eps) : 0.0f;
            scale = beta / s7;
            lo = -8; hi = 7;
        }
        int32_t sum = 0;
        for (int k = 0; k < K; ++k) {
            double y = (double)v[k] * (double)inv; /* exact */
            q[k] = clip_round(y, lo, hi);
            sum += q[k];
        }
        if (act_bits == 8) {
            memcpy(codes + (int64_t)m * K, q, (size_t)K);
        } else {
            uint8_t* row = codes + (int64_t)m * (K / 2);
            for (int j = 0; j < K / 2; ++j)
                row[j] = (uint8_t)(((uint8_t)q[2 * j] & 0x0f) | (((uint8_t)q[2 * j + 1] & 0x0f) << 4));
        }
        scales[m] = scale;
        if (rowsum) rowsum[m] = sum;
    }
    free(absv);
    free(q);
    return 0;
}

/* Decode codes back to integers (int8 per element). */
ORACLE_API int oracle_decode_codes(const uint8_t* codes, int M, int K, int act_bits, int8_t* q) {
    if (act_bits == 8) {
        memcpy(q, codes, (size_t)M * (size_t)K);
        return 0;
    }
    if (act_bits != 4) return -1;
    for (int64_t m = 0; m < M; ++m)
        for (int j = 0; j < K / 2; ++j) {
            uint8_t b = codes[m * (K / 2) + j];
            int lo = b & 0x0f, hi = b >> 4;
            q[m * K + 2 * j] = (int8_t)(lo >= 8 ? lo - 16 : lo);
            q[m * K + 2 * j + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
        }
    return 0;
}

/* norm -> Hadamard -> quantise, the activation half of the layer [P2]. */
ORACLE_API int oracle_norm_fwht_quant(const uint16_t* X, const float* gain, int M, int K,
                                      float norm_eps, float quant_eps, int act_bits,
                                      uint8_t* codes, float* scales, int32_t* rowsum) {
    if (M < 0 || !is_pow2_i64(K)) return -1;
    float* v = (float*)malloc(sizeof(float) * (size_t)K);
    if (!v) return -2;
    int64_t cstride = act_bits == 8 ? K : K / 2;
    int rc = 0;
    for (int m = 0; m < M && rc == 0; ++m) {
        rc = oracle_norm_fwht(X + (int64_t)m * K, gain, 1, K, norm_eps, v);
        if (rc == 0)
            rc = oracle_quantize_rows(v, 1, K, quant_eps, act_bits, codes + m * cstride,
                                      scales + m, rowsum ? rowsum + m : NULL);
    }
    free(v);
    return rc;
}

/* The activation half of a BitLinear layer with the variant choices above. */
ORACLE_API int oracle_norm_quant(const uint16_t* X, const float* gain, int M, int K,
                                 float norm_eps, float quant_eps, int act_bits, int layernorm,
                                 int hadamard, uint8_t* codes, float* scales, int32_t* rowsum) {
    if (M < 0 || !is_pow2_i64(K)) return -1;
    float* v = (float*)malloc(sizeof(float) * (size_t)K);
    if (!v) return -2;
    int64_t cstride = act_bits == 8 ? K : K / 2;
    int rc = 0;
    for (int m = 0; m < M && rc == 0; ++m) {
        rc = oracle_norm_transform(X + (int64_t)m * K, gain, 1, K, norm_eps, layernorm, hadamard,
                                   v);
        if (rc == 0)
            rc = oracle_quantize_rows(v, 1, K, quant_eps, act_bits, codes + m * cstride,
                                      scales + m, rowsum ? rowsum + m : NULL);
    }
    free(v);
    return rc;
}

/* --------------------------------------- weight rotation [P2-ABL], offline */

/* W_rot[n] = FWHT(W[n] * s) * (1/sqrt(K)) for every row n of W [N x K] fp32:
 * the weights expressed in the rotated basis, so that for activations rotated
 * by the same map, (x D H/sqrt(K)) . (w D H/sqrt(K)) = x . w (D = diag(s),
 * H H^T = K I).  s (nullable, entries +-1) is the random sign vector of the
 * randomised Hadamard transform; NULL means all ones.  Butterfly order and
 * the final multiply are those of the activation transform. */
ORACLE_API int oracle_rotate_weights(const float* W, const float* signs, int N, int K,
                                     float* W_rot) {
    if (N < 0 || !is_pow2_i64(K)) return -1;
    const float c = oracle_inv_sqrt_n(K);
    for (int64_t n = 0; n < N; ++n) {
        float* w = W_rot + n * K;
        for (int k = 0; k < K; ++k) w[k] = signs ? W[n * K + k] * signs[k] : W[n * K + k];
        oracle_fwht_f32(w, K);
        for (int k = 0; k < K; ++k) w[k] = w[k] * c;
    }
    return 0;
}

/* ------------------------------------------ QKV / KV-cache quantiser [P2-QKV] */

/* Per-head absmax quantisation to unsigned b-bit integers (b in 2..8)
 * (inv = 0 when gamma + eps == 0, as in quantize_rows) for Q,
 * K and V states after RoPE.  Each row of X [rows x D] bf16 is one head of one
 * token.  The symmetric absmax quantiser of the INT8 activations, taken to b
 * bits and offset into the unsigned range:
 *   Qp = 2^(b-1) - 1;  gamma = max|x|;  inv = Qp / (gamma + eps)   (one division)
 *   q = clip(round(x * inv), -Qp - 1, Qp)   (the exact product rounded once,
 *                                            to nearest, ties to even)
 *   u = q + 2^(b-1)  in [0, 2^b - 1];  scale = gamma / Qp;
 *   dequantised x ~ (u - 2^(b-1)) * scale.
 * Packing: groups of 32 consecutive codes of a row, each group 4*b bytes; code j
 * of a group occupies bits [b*j, b*j + b) of the group read as one
 * little-endian integer.  D must be a multiple of 32. */
ORACLE_API int oracle_kv_quant(const uint16_t* X, int64_t rows, int D, int bits, float eps,
                               uint8_t* codes, float* scales) {
    if (rows < 0 || D <= 0 || D % 32 != 0 || bits < 2 || bits > 8) return -1;
    const int qp = (1 << (bits - 1)) - 1;
    const int64_t row_bytes = (int64_t)D / 32 * 4 * bits;
    for (int64_t r = 0; r < rows; ++r) {
        const uint16_t* x = X + r * D;
        float g = 0.0f;
        for (int k = 0; k < D; ++k) {
            float a = fabsf(oracle_bf16_to_f32(x[k]));
            if (a > g) g = a;
        }
        const float inv = (g + eps) > 0.0f ? (float)qp / (g + eps) : 0.0f;
        uint8_t* out = codes + r * row_bytes;
        memset(out, 0, (size_t)row_bytes);
        for (int k = 0; k < D; ++k) {
            double y = (double)oracle_bf16_to_f32(x[k]) * (double)inv; /* exact */
            int q = clip_round(y, -qp - 1, qp);
            uint32_t u = (uint32_t)(q + (1 << (bits - 1)));
            int64_t bit = (int64_t)(k / 32) * 32 * bits + (int64_t)(k % 32) * bits;
            for (int i = 0; i < bits; ++i)
                if ((u >> i) & 1u) out[(bit + i) / 8] |= (uint8_t)(1u << ((bit + i) % 8));
        }
        scales[r] = g / (float)qp;
    }
    return 0;
}

/* Unpacks kv_quant codes to their unsigned values u [rows x D]. */
ORACLE_API int oracle_kv_unpack(const uint8_t* codes, int64_t rows, int D, int bits, uint8_t* u) {
    if (rows < 0 || D <= 0 || D % 32 != 0 || bits < 2 || bits > 8) return -1;
    const int64_t row_bytes = (int64_t)D / 32 * 4 * bits;
    for (int64_t r = 0; r < rows; ++r)
        for (int k = 0; k < D; ++k) {
            int64_t bit = (int64_t)(k / 32) * 32 * bits + (int64_t)(k % 32) * bits;
            uint32_t v = 0;
            for (int i = 0; i < bits; ++i)
                v |= (uint32_t)((codes[r * row_bytes + (bit + i) / 8] >> ((bit + i) % 8)) & 1u) << i;
            u[r * D + k] = (uint8_t)v;
        }
    return 0;
}

/* ------------------------------------------------ ternary weights [P2][P3] */

/* Per-tensor absmean ternarisation:
 *   alpha = tree_sum(|W| over the row-major flat index) / (float)(N*K);
 *   t = clip(round(W / (alpha + eps)), -1, 1)   (one IEEE division per weight).
 * t_out (nullable) receives the int8 ternary values [N x K]. */
ORACLE_API int oracle_ternarize(const float* W, int N, int K, float eps, int8_t* t_out,
                                float* alpha_out) {
    if (N <= 0 || K <= 0) return -1;
    int64_t nk = (int64_t)N * K;
    float* a = (float*)malloc(sizeof(float) * (size_t)nk);
    if (!a) return -2;
    for (int64_t i = 0; i < nk; ++i) a[i] = fabsf(W[i]);
    float alpha = tree_sum_f32(a, nk) / (float)nk;
    free(a);
    float d = alpha + eps;
    if (t_out)
        for (int64_t i = 0; i < nk; ++i) t_out[i] = clip_round((double)(W[i] / d), -1, 1);
    *alpha_out = alpha;
    return 0;
}

/* 2-bit packing [P3 "pack several values into an integer"]: 16 weights per
 * uint32 along K; word (n, k/16); weight k (local index j = k % 16) sits at
 * bits [8*(j % 4) + 2*(j / 4), +2) as the code t + 1 (0 -> -1, 1 -> 0, 2 -> +1;
 * 3 never written).  Requires K % 16 == 0. */
ORACLE_API int oracle_pack_codes(const int8_t* t, int N, int K, uint32_t* packed) {
    if (K % 16 != 0) return -1;
    int64_t wpr = K / 16;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t w = 0; w < wpr; ++w) {
            uint32_t word = 0;
            for (int j = 0; j < 16; ++j) {
                int8_t v = t[n * K + w * 16 + j];
                uint32_t code = (uint32_t)(v + 1);
                word |= code << (8 * (j % 4) + 2 * (j / 4));
            }
            packed[n * wpr + w] = word;
        }
    return 0;
}

ORACLE_API int oracle_unpack_codes(const uint32_t* packed, int N, int K, int8_t* t) {
    if (K % 16 != 0) return -1;
    int64_t wpr = K / 16;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t w = 0; w < wpr; ++w) {
            uint32_t word = packed[n * wpr + w];
            for (int j = 0; j < 16; ++j) {
                uint32_t code = (word >> (8 * (j % 4) + 2 * (j / 4))) & 3u;
                if (code == 3u) return -3;
                t[n * K + w * 16 + j] = (int8_t)((int)code - 1);
            }
        }
    return 0;
}

ORACLE_API int oracle_pack_ternary(const float* W, int N, int K, float eps, uint32_t* packed,
                                   float* alpha_out) {
    if (N <= 0 || K <= 0 || K % 16 != 0) return -1;
    int8_t* t = (int8_t*)malloc((size_t)N * (size_t)K);
    if (!t) return -2;
    int rc = oracle_ternarize(W, N, K, eps, t, alpha_out);
    if (rc == 0) rc = oracle_pack_codes(t, N, K, packed);
    free(t);
    return rc;
}

/* ------------------------------------ ternary matmul + dequantisation [P2] */

/* acc[m][n] = sum_k q[m][k] * t[n][k]   (exact, int64, must fit int32);
 * y[m][n]   = bf16_rne( (float)acc * (alpha * scale[m]) ).
 * t: the ternary values int8 [N x K] (unpacked once by the caller).
 * Rows m in [m0, m1) only (callers split rows across threads). */
ORACLE_API int oracle_ternary_gemm_rows_t(const uint8_t* codes, const float* scales,
                                          int act_bits, int M, int K, const int8_t* t,
                                          float alpha, int N, int m0, int m1, uint16_t* Y,
                                          int32_t* acc_out) {
    if (M < 0 || K <= 0 || N <= 0) return -1;
    if (m0 < 0 || m1 > M || m0 > m1) return -1;
    int8_t* q = (int8_t*)malloc((size_t)K);
    if (!q) return -2;
    int rc = 0;
    int64_t cstride = act_bits == 8 ? K : K / 2;
    for (int64_t m = m0; m < m1 && rc == 0; ++m) {
        rc = oracle_decode_codes(codes + m * cstride, 1, K, act_bits, q);
        if (rc) break;
        float sc = alpha * scales[m];
        for (int64_t n = 0; n < N; ++n) {
            const int8_t* tr = t + n * K;
            int64_t s = 0;
            for (int64_t k = 0; k < K; ++k) s += (int64_t)q[k] * (int64_t)tr[k];
            if (s > INT32_MAX || s < INT32_MIN) { rc = -4; break; }
            if (acc_out) acc_out[m * N + n] = (int32_t)s;
            if (Y) Y[m * N + n] = oracle_f32_to_bf16((float)s * sc);
        }
    }
    free(q);
    return rc;
}

/* The same from the packed weights (unpacked here). */
ORACLE_API int oracle_ternary_gemm_rows(const uint8_t* codes, const float* scales, int act_bits,
                                        int M, int K, const uint32_t* packed, float alpha, int N,
                                        int m0, int m1, uint16_t* Y, int32_t* acc_out) {
    if (M < 0 || K <= 0 || K % 16 != 0 || N <= 0) return -1;
    if (m0 < 0 || m1 > M || m0 > m1) return -1;
    int8_t* t = (int8_t*)malloc((size_t)N * (size_t)K);
    if (!t) return -2;
    int rc = oracle_unpack_codes(packed, N, K, t);
    if (rc == 0)
        rc = oracle_ternary_gemm_rows_t(codes, scales, act_bits, M, K, t, alpha, N, m0, m1, Y,
                                        acc_out);
    free(t);
    return rc;
}

ORACLE_API int oracle_ternary_gemm(const uint8_t* codes, const float* scales, int act_bits, int M,
                                   int K, const uint32_t* packed, float alpha, int N, uint16_t* Y,
                                   int32_t* acc_out) {
    return oracle_ternary_gemm_rows(codes, scales, act_bits, M, K, packed, alpha, N, 0, M, Y,
                                    acc_out);
}

/* Whole layer for rows [m0, m1) with the variant choices of norm_transform:
 * norm -> (Hadamard) -> quantise -> ternary matmul -> dequantise. */
ORACLE_API int oracle_bitlinear_forward_rows(const uint16_t* X, const float* gain, int M, int K,
                                             int N, const uint32_t* packed, float alpha,
                                             int act_bits, float norm_eps, float quant_eps,
                                             int layernorm, int hadamard, int m0, int m1,
                                             uint16_t* Y) {
    if (m0 < 0 || m1 > M || m0 > m1) return -1;
    int rows = m1 - m0;
    if (rows == 0) return 0;
    int64_t cstride = act_bits == 8 ? K : K / 2;
    uint8_t* codes = (uint8_t*)malloc((size_t)rows * (size_t)cstride);
    float* scales = (float*)malloc(sizeof(float) * (size_t)rows);
    if (!codes || !scales) { free(codes); free(scales); return -2; }
    int rc = oracle_norm_quant(X + (int64_t)m0 * K, gain, rows, K, norm_eps, quant_eps, act_bits,
                               layernorm, hadamard, codes, scales, NULL);
    if (rc == 0)
        rc = oracle_ternary_gemm(codes, scales, act_bits, rows, K, packed, alpha, N,
                                 Y + (int64_t)m0 * N, NULL);
    free(codes);
    free(scales);
    return rc;
}

/* Whole layer for rows [m0, m1): norm -> Hadamard -> quantise -> ternary matmul
 * -> dequantise.  Y is [M x N] bf16 bits; only rows [m0, m1) are written.
 * t: the ternary values int8 [N x K] (unpacked once by the caller). */
ORACLE_API int oracle_hbitlinear_forward_rows_t(const uint16_t* X, const float* gain, int M,
                                                int K, int N, const int8_t* t, float alpha,
                                                int act_bits, float norm_eps, float quant_eps,
                                                int m0, int m1, uint16_t* Y) {
    if (m0 < 0 || m1 > M || m0 > m1) return -1;
    int rows = m1 - m0;
    if (rows == 0) return 0;
    int64_t cstride = act_bits == 8 ? K : K / 2;
    uint8_t* codes = (uint8_t*)malloc((size_t)rows * (size_t)cstride);
    float* scales = (float*)malloc(sizeof(float) * (size_t)rows);
    if (!codes || !scales) { free(codes); free(scales); return -2; }
    int rc = oracle_norm_fwht_quant(X + (int64_t)m0 * K, gain, rows, K, norm_eps, quant_eps,
                                    act_bits, codes, scales, NULL);
    if (rc == 0)
        rc = oracle_ternary_gemm_rows_t(codes, scales, act_bits, rows, K, t, alpha, N, 0, rows,
                                        Y + (int64_t)m0 * N, NULL);
    free(codes);
    free(scales);
    return rc;
}

/* The same from the packed weights (unpacked here). */
ORACLE_API int oracle_hbitlinear_forward_rows(const uint16_t* X, const float* gain, int M, int K,
                                              int N, const uint32_t* packed, float alpha,
                                              int act_bits, float norm_eps, float quant_eps,
                                              int m0, int m1, uint16_t* Y) {
    if (m0 < 0 || m1 > M || m0 > m1) return -1;
    if (K <= 0 || K % 16 != 0 || N <= 0) return -1;
    if (m1 == m0) return 0;
    int8_t* t = (int8_t*)malloc((size_t)N * (size_t)K);
    if (!t) return -2;
    int rc = oracle_unpack_codes(packed, N, K, t);
    if (rc == 0)
        rc = oracle_hbitlinear_forward_rows_t(X, gain, M, K, N, t, alpha, act_bits, norm_eps,
                                              quant_eps, m0, m1, Y);
    free(t);
    return rc;
}
