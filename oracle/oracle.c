/*
 * oracle.c -- plain CPU oracle for the W4A16 AWQ g128 quantized linear layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this
 * file: only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
 * It shares no code, header, table or constant with the CUDA library; the packed
 * format it writes is the interface both sides agree on, restated here on its own.
 *
 * Build: gcc -O2 -ffp-contract=off -fopenmp -shared -fPIC (no FMA contraction, so
 * every float operation below is one IEEE-754 operation rounded to nearest-even).
 *
 * What it computes, and where the method comes from:
 *   - per-input-channel activation-aware scale s_k = max(float(pow(a_k, alpha)), 1e-4)
 *     [AWQ (MLSys 2024) translation, section 3.2 "protect salient weights by
 *     activation-aware scaling"; the closed form s = mean|x|^alpha is the plain reading
 *     of that section, whose translation breaks off before the formula];
 *   - group-wise asymmetric uint4 round-to-nearest on W*s, groups of 128 along K
 *     [DeepCompressor README, perplexity table row "W4A16 g128"; AWQ translation,
 *     section 2 "round-to-nearest (RTN)" and group-wise INT4], and the same with other
 *     group sizes, up to one group per row [SqueezeLLM article, section 4.1: the group
 *     size option, per-row by default];
 *   - 4-bit weight packing, 8 codes per 32-bit word [AWQ translation, section 1:
 *     TinyChat's 4-bit weight packing];
 *   - a 3-bit variant: the same RTN with eight levels, 32 codes per three 32-bit words
 *     [SqueezeLLM article, sections 2.1-2.2: the dense part quantized as coarse as 3 bits];
 *   - NVFP4 weights: FP4 E2M1 codes with an FP8 E4M3 scale per 16 weights and an fp32
 *     scale per tensor [DeepCompressor README: FP4_E2M1 among its data types, NVFP4 rows in
 *     its result tables; the format's layout is the published one, see its section];
 *   - the dense-and-sparse product  W x = W_dense x + W_sparse x  with an fp16 CSR
 *     W_sparse [SqueezeLLM article, sections 2.2 and 2.3; the page lost the "=" and
 *     "+" signs, read here as written above];
 *   - the outlier split: the largest |w| * act_absmean entries go to W_sparse
 *     [SqueezeLLM article, section 2.2 (sensitive weights kept in fp16) and
 *     section 5.3 (sparsity ratio 0.0045)].
 *
 * Every function here has at least one independent pin in tests/ (brute force, closed
 * forms, invariants, library routines); see the test files for which.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_NULL 1
#define ORACLE_ERR_SHAPE 2
#define ORACLE_ERR_VALUE 4

#define GROUP 128

/* ------------------------------------------------------------------------------------
 * IEEE-754 binary16 / bfloat16 conversions written from the format definitions:
 * round the exact value to the nearest point of the target grid, ties to the even
 * significand, overflow to infinity.  All arithmetic is in double, where every step
 * below is exact (scaling by powers of two, rint of a value with <= 25 significant
 * bits).
 * ---------------------------------------------------------------------------------- */

/* binary16: 11 significant bits, normal exponents -14..15, subnormal step 2^-24. */
uint16_t oracle_f32_to_f16(float f) {
    uint16_t sign = signbit(f) ? 0x8000u : 0u;
    if (isnan(f)) return (uint16_t)(sign | 0x7E00u);
    double a = fabs((double)f);
    /* The largest finite value is 65504 (significand 2047, odd); a tie at 65520 rounds
     * to the even neighbour 65536, which overflows. */
    if (isinf(f) || a >= 65520.0) return (uint16_t)(sign | 0x7C00u);
    if (a < ldexp(1.0, -14)) {
        double r = rint(a / ldexp(1.0, -24)); /* 0..1024; 1024 is the smallest normal */
        return (uint16_t)(sign | (uint16_t)r);
    }
    int e;
    frexp(a, &e);                   /* a = m * 2^e, m in [0.5, 1): leading bit 2^(e-1) */
    double quantum = ldexp(1.0, e - 1 - 10);
    double r = rint(a / quantum);   /* 1024..2048 */
    int biased = e - 1 + 15;
    if (r == 2048.0) { r = 1024.0; biased += 1; }
    if (biased >= 31) return (uint16_t)(sign | 0x7C00u);
    return (uint16_t)(sign | (uint16_t)(biased << 10) | (uint16_t)((int)r - 1024));
}

float oracle_f16_to_f32(uint16_t h) {
    int s = (h >> 15) & 1, E = (h >> 10) & 31, m = h & 1023;
    double v;
    if (E == 31) v = m ? NAN : INFINITY;
    else if (E == 0) v = ldexp((double)m, -24);
    else v = ldexp((double)(1024 + m), E - 15 - 10);
    return (float)(s ? -v : v);
}

/* bfloat16: 8 significant bits, the exponent range of binary32 (normal from 2^-126,
 * subnormal step 2^-133). */
uint16_t oracle_f32_to_bf16(float f) {
    uint16_t sign = signbit(f) ? 0x8000u : 0u;
    if (isnan(f)) return (uint16_t)(sign | 0x7FC0u);
    double a = fabs((double)f);
    /* largest finite: (2 - 2^-7) * 2^127, significand 255 (odd): the tie above it rounds
     * up to 2^128 and overflows */
    if (isinf(f) || a >= ldexp(2.0 - ldexp(1.0, -8), 127)) return (uint16_t)(sign | 0x7F80u);
    if (a < ldexp(1.0, -126)) {
        double r = rint(a / ldexp(1.0, -133)); /* 0..128; 128 is the smallest normal */
        return (uint16_t)(sign | (uint16_t)r);
    }
    int e;
    frexp(a, &e);
    double quantum = ldexp(1.0, e - 1 - 7);
    double r = rint(a / quantum);   /* 128..256 */
    int biased = e - 1 + 127;
    if (r == 256.0) { r = 128.0; biased += 1; }
    if (biased >= 255) return (uint16_t)(sign | 0x7F80u);
    return (uint16_t)(sign | (uint16_t)(biased << 7) | (uint16_t)((int)r - 128));
}

float oracle_bf16_to_f32(uint16_t h) {
    int s = (h >> 15) & 1, E = (h >> 7) & 255, m = h & 127;
    double v;
    if (E == 255) v = m ? NAN : INFINITY;
    else if (E == 0) v = ldexp((double)m, -133);
    else v = ldexp((double)(128 + m), E - 127 - 7);
    return (float)(s ? -v : v);
}

/* ------------------------------------------------------------------------------------
 * Packed format (the interface shared with the CUDA library, restated here):
 *   qweight[n][k/8]  uint32; nibble j (bits 4j..4j+3) holds element k = 8*(k/8) + ORDER[j]
 *                    with ORDER = {0,2,4,6,1,3,5,7};
 *   scales[g][n]     fp16 bits, g = k/GS (group-major), GS the group size (128 for g128);
 *   zeros[g][n/8]    uint32; nibble j holds the zero point of row 8*(n/8) + j in group g.
 * ---------------------------------------------------------------------------------- */
static const int ORACLE_ORDER[8] = {0, 2, 4, 6, 1, 3, 5, 7};

static int nibble_of_element(int e) { /* inverse of ORACLE_ORDER */
    for (int j = 0; j < 8; ++j)
        if (ORACLE_ORDER[j] == e) return j;
    return -1;
}

int oracle_pack8(const uint8_t* q /* 8 codes, element order */, uint32_t* word) {
    uint32_t w = 0;
    for (int j = 0; j < 8; ++j) {
        if (q[ORACLE_ORDER[j]] > 15) return ORACLE_ERR_VALUE;
        w |= (uint32_t)q[ORACLE_ORDER[j]] << (4 * j);
    }
    *word = w;
    return ORACLE_OK;
}

void oracle_unpack8(uint32_t word, uint8_t* q /* 8 codes, element order */) {
    for (int e = 0; e < 8; ++e) q[e] = (uint8_t)((word >> (4 * nibble_of_element(e))) & 15u);
}

/* ------------------------------------------------------------------------------------
 * Activation-aware scale [AWQ translation, section 3.2]:
 *   s_k = max( float(pow(double(a_k), double(alpha))), 1e-4 ).
 * a_k must be finite and >= 0, alpha finite; a non-finite s is a value error.
 * ---------------------------------------------------------------------------------- */
int oracle_awq_scales(const float* act_absmean, int64_t K, float alpha, float* s) {
    if (!act_absmean || !s) return ORACLE_ERR_NULL;
    if (K <= 0) return ORACLE_ERR_SHAPE;
    if (!isfinite(alpha)) return ORACLE_ERR_VALUE;
    for (int64_t k = 0; k < K; ++k) {
        float a = act_absmean[k];
        if (!isfinite(a) || a < 0.0f) return ORACLE_ERR_VALUE;
        float p = (float)pow((double)a, (double)alpha);
        if (!isfinite(p)) return ORACLE_ERR_VALUE;
        s[k] = p > 1e-4f ? p : 1e-4f;
    }
    return ORACLE_OK;
}

/* One group of gs scaled weights -> fp16 scale bits, zero point, gs codes, with qmax + 1
 * levels (qmax = 15 for 4-bit codes, 7 for 3-bit):
 *   scale32 = max((max - min) / qmax, 1e-5)        (plain asymmetric min/max range)
 *   sf      = float(fp16_rne(scale32))             (the stored scale is the one used)
 *   z       = clamp(rint(-min / sf), 0, qmax)
 *   q_i     = clamp(rint(w_i / sf) + z, 0, qmax)   (round first, then add the zero)
 * rint is round-half-to-even; every operation is one IEEE float operation. */
static int quantize_group(const float* wp, int64_t gs, float qmax, uint16_t* s16_out, uint8_t* z_out,
                          uint8_t* q_out) {
    float mx = wp[0], mn = wp[0];
    for (int64_t i = 0; i < gs; ++i) {
        if (!isfinite(wp[i])) return ORACLE_ERR_VALUE;
        if (wp[i] > mx) mx = wp[i];
        if (wp[i] < mn) mn = wp[i];
    }
    float scale32 = (mx - mn) / qmax;
    if (scale32 < 1e-5f) scale32 = 1e-5f;
    if (isinf(scale32)) return ORACLE_ERR_VALUE; /* max - min overflowed */
    uint16_t s16 = oracle_f32_to_f16(scale32);
    if ((s16 & 0x7FFFu) == 0x7C00u) return ORACLE_ERR_VALUE; /* fp16 overflow */
    float sf = oracle_f16_to_f32(s16);
    float zf = rintf(-mn / sf);
    if (zf < 0.0f) zf = 0.0f;
    if (zf > qmax) zf = qmax;
    for (int64_t i = 0; i < gs; ++i) {
        float qf = rintf(wp[i] / sf) + zf;
        if (qf < 0.0f) qf = 0.0f;
        if (qf > qmax) qf = qmax;
        q_out[i] = (uint8_t)qf;
    }
    *s16_out = s16;
    *z_out = (uint8_t)zf;
    return ORACLE_OK;
}

static int check_qshape(int64_t N, int64_t K) {
    if (N <= 0 || N % 8 != 0 || K <= 0 || K % 1024 != 0) return ORACLE_ERR_SHAPE;
    return ORACLE_OK;
}

/* group size: a multiple of 8 (whole packed words) that divides K */
static int check_gs(int64_t K, int64_t gs) {
    if (gs <= 0 || gs % 8 != 0 || K % gs != 0) return ORACLE_ERR_SHAPE;
    return ORACLE_OK;
}

static int zero_of(const uint32_t* zeros, int64_t N, int64_t n, int64_t g) {
    return (int)((zeros[g * (N / 8) + n / 8] >> (4 * (n % 8))) & 15u);
}

int oracle_pack32x3(const uint8_t* q, uint32_t* words);

/* Quantize W (fp32 [N][K]) with a given per-channel scale s ([K]) in groups of gs along K:
 * w' = float(w * s_k), then quantize_group on each run of gs along K, then pack: 4-bit
 * codes 8 per word, or 3-bit codes 32 per 3 words (gs a multiple of 32). */
static int quantize_with_scales_bits(const float* W, const float* s, int64_t N, int64_t K, int64_t gs, int bits,
                                     uint32_t* qweight, uint16_t* scales, uint32_t* zeros) {
    if (!W || !s || !qweight || !scales || !zeros) return ORACLE_ERR_NULL;
    int st = check_qshape(N, K);
    if (!st) st = check_gs(K, gs);
    if (!st && bits == 3 && gs % 32 != 0) st = ORACLE_ERR_SHAPE;
    if (!st && bits != 3 && bits != 4) st = ORACLE_ERR_SHAPE;
    if (st) return st;
    const float qmax = bits == 4 ? 15.0f : 7.0f;
    const int64_t G = K / gs;
    int err = ORACLE_OK;
    uint8_t* zcode = (uint8_t*)malloc((size_t)(N * G));
    if (!zcode) return ORACLE_ERR_VALUE;
#pragma omp parallel
    {
        float* wp = (float*)malloc(sizeof(float) * (size_t)gs);
        uint8_t* q = (uint8_t*)malloc((size_t)gs);
#pragma omp for schedule(dynamic, 4)
        for (int64_t n = 0; n < N; ++n) {
            if (!wp || !q) {
#pragma omp atomic write
                err = ORACLE_ERR_VALUE;
                continue;
            }
            for (int64_t g = 0; g < G; ++g) {
                for (int64_t i = 0; i < gs; ++i) wp[i] = W[n * K + g * gs + i] * s[g * gs + i];
                uint16_t s16;
                uint8_t z;
                int e = quantize_group(wp, gs, qmax, &s16, &z, q);
                if (e) {
#pragma omp atomic write
                    err = e;
                    continue;
                }
                scales[g * N + n] = s16;
                zcode[n * G + g] = z;
                if (bits == 4) {
                    for (int64_t w = 0; w < gs / 8; ++w) {
                        uint32_t word;
                        oracle_pack8(&q[8 * w], &word);
                        qweight[n * (K / 8) + g * (gs / 8) + w] = word;
                    }
                } else {
                    for (int64_t b = 0; b < gs / 32; ++b)
                        oracle_pack32x3(&q[32 * b], &qweight[n * (K / 32) * 3 + (g * (gs / 32) + b) * 3]);
                }
            }
        }
        free(wp);
        free(q);
    }
    /* zero points packed along n: nibble j of zeros[g][n/8] is row 8*(n/8) + j */
    for (int64_t g = 0; g < G; ++g)
        for (int64_t n8 = 0; n8 < N / 8; ++n8) {
            uint32_t word = 0;
            for (int j = 0; j < 8; ++j) word |= (uint32_t)(zcode[(n8 * 8 + j) * G + g] & 15u) << (4 * j);
            zeros[g * (N / 8) + n8] = word;
        }
    free(zcode);
    return err;
}

int oracle_quantize_with_scales_gs(const float* W, const float* s, int64_t N, int64_t K, int64_t gs,
                                   uint32_t* qweight, uint16_t* scales, uint32_t* zeros) {
    return quantize_with_scales_bits(W, s, N, K, gs, 4, qweight, scales, zeros);
}

int oracle_quantize_with_scales(const float* W, const float* s, int64_t N, int64_t K,
                                uint32_t* qweight, uint16_t* scales, uint32_t* zeros) {
    return oracle_quantize_with_scales_gs(W, s, N, K, GROUP, qweight, scales, zeros);
}

/* awq_quantize with group size gs: the scale from act_absmean and alpha, then quantize W*s. */
int oracle_awq_quantize_gs(const float* W, const float* act_absmean, float alpha, int64_t N, int64_t K,
                           int64_t gs, uint32_t* qweight, uint16_t* scales, uint32_t* zeros, float* s_out) {
    if (!W || !act_absmean || !qweight || !scales || !zeros) return ORACLE_ERR_NULL;
    int st = check_qshape(N, K);
    if (!st) st = check_gs(K, gs);
    if (st) return st;
    float* s = (float*)malloc(sizeof(float) * (size_t)K);
    if (!s) return ORACLE_ERR_VALUE;
    st = oracle_awq_scales(act_absmean, K, alpha, s);
    if (!st) st = oracle_quantize_with_scales_gs(W, s, N, K, gs, qweight, scales, zeros);
    if (!st && s_out) memcpy(s_out, s, sizeof(float) * (size_t)K);
    free(s);
    return st;
}

/* awq_quantize_g128: the scale from act_absmean and alpha, then quantize W*s. */
int oracle_awq_quantize_g128(const float* W, const float* act_absmean, float alpha, int64_t N,
                             int64_t K, uint32_t* qweight, uint16_t* scales, uint32_t* zeros,
                             float* s_out) {
    return oracle_awq_quantize_gs(W, act_absmean, alpha, N, K, GROUP, qweight, scales, zeros, s_out);
}

/* deq[n][k] = (q - z) * sf, exact in fp32 (a 5-bit integer times an 11-bit scale). */
int oracle_dequant_gs(const uint32_t* qweight, const uint16_t* scales, const uint32_t* zeros,
                      int64_t N, int64_t K, int64_t gs, float* deq) {
    if (!qweight || !scales || !zeros || !deq) return ORACLE_ERR_NULL;
    int st = check_qshape(N, K);
    if (!st) st = check_gs(K, gs);
    if (st) return st;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t k = 0; k < K; ++k) {
            int64_t g = k / gs;
            uint8_t codes[8];
            oracle_unpack8(qweight[n * (K / 8) + k / 8], codes);
            int q = codes[k % 8];
            int z = zero_of(zeros, N, n, g);
            float sf = oracle_f16_to_f32(scales[g * N + n]);
            deq[n * K + k] = (float)(q - z) * sf;
        }
    }
    return ORACLE_OK;
}

int oracle_dequant(const uint32_t* qweight, const uint16_t* scales, const uint32_t* zeros,
                   int64_t N, int64_t K, float* deq) {
    return oracle_dequant_gs(qweight, scales, zeros, N, K, GROUP, deq);
}

static int check_csr(const int32_t* row_ptr, const int32_t* col_idx, const uint16_t* values,
                     int64_t nnz, int64_t N, int64_t K) {
    if (nnz < 0) return ORACLE_ERR_SHAPE;
    if (nnz == 0 && !row_ptr) return ORACLE_OK;
    if (!row_ptr || (nnz > 0 && (!col_idx || !values))) return ORACLE_ERR_NULL;
    if (row_ptr[0] != 0 || row_ptr[N] != nnz) return ORACLE_ERR_SHAPE;
    for (int64_t n = 0; n < N; ++n) {
        if (row_ptr[n + 1] < row_ptr[n]) return ORACLE_ERR_SHAPE;
        for (int64_t j = row_ptr[n]; j < row_ptr[n + 1]; ++j) {
            if (col_idx[j] < 0 || col_idx[j] >= K) return ORACLE_ERR_SHAPE;
            if (j > row_ptr[n] && col_idx[j] <= col_idx[j - 1]) return ORACLE_ERR_SHAPE;
        }
    }
    return ORACLE_OK;
}

void oracle_unpack32x3(const uint32_t* words, uint8_t* q);

/* The code of element k of row n: 4-bit layout (8 per word) or 3-bit layout (32 per 3 words). */
static int code_at(const uint32_t* qweight, int bits, int64_t K, int64_t n, int64_t k) {
    if (bits == 4) {
        uint8_t codes[8];
        oracle_unpack8(qweight[n * (K / 8) + k / 8], codes);
        return codes[k % 8];
    }
    uint8_t codes[32];
    oracle_unpack32x3(&qweight[n * (K / 32) * 3 + (k / 32) * 3], codes);
    return codes[k % 32];
}

/* One output y[m][n] = sum_k x[m][k] deq[n][k] + sum_{j in row n} x[m][col_j] val_j, summed
 * in double (each product of a bf16 and a dequantized weight or fp16 value is exact in
 * double), plus the sum of the absolute products, which bounds any rounding error. */
static void one_output(const uint16_t* x, int64_t K, int64_t N, int64_t gs, int bits, const uint32_t* qweight,
                       const uint16_t* scales, const uint32_t* zeros, const int32_t* row_ptr,
                       const int32_t* col_idx, const uint16_t* values, int64_t m, int64_t n,
                       double* y, double* yabs) {
    double acc = 0.0, aacc = 0.0;
    for (int64_t k = 0; k < K; ++k) {
        int64_t g = k / gs;
        int q = code_at(qweight, bits, K, n, k);
        int z = zero_of(zeros, N, n, g);
        double w = (double)((float)(q - z) * oracle_f16_to_f32(scales[g * N + n]));
        double p = (double)oracle_bf16_to_f32(x[m * K + k]) * w;
        acc += p;
        aacc += fabs(p);
    }
    if (row_ptr) {
        for (int64_t j = row_ptr[n]; j < row_ptr[n + 1]; ++j) {
            double p = (double)oracle_bf16_to_f32(x[m * K + col_idx[j]]) *
                       (double)oracle_f16_to_f32(values[j]);
            acc += p;
            aacc += fabs(p);
        }
    }
    *y = acc;
    if (yabs) *yabs = aacc;
}

/* y = x deq(Q)^T + x W_sparse^T for all (m, n): x bf16 [M][K]; y, yabs double [M][N].
 * The CSR (row_ptr [N+1], col_idx/values [nnz], ascending columns per row) may be absent
 * (row_ptr == NULL and nnz == 0). */
static int linear_bits(const uint16_t* x, int64_t M, int64_t K, int64_t gs, int bits, const uint32_t* qweight,
                       const uint16_t* scales, const uint32_t* zeros, int64_t N,
                       const int32_t* row_ptr, const int32_t* col_idx, const uint16_t* values,
                       int64_t nnz, double* y, double* yabs) {
    if (!x || !qweight || !scales || !zeros || !y) return ORACLE_ERR_NULL;
    if (M <= 0) return ORACLE_ERR_SHAPE;
    int st = check_qshape(N, K);
    if (!st) st = check_gs(K, gs);
    if (st) return st;
    st = check_csr(row_ptr, col_idx, values, nnz, N, K);
    if (st) return st;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n)
            one_output(x, K, N, gs, bits, qweight, scales, zeros, row_ptr, col_idx, values, m, n,
                       &y[m * N + n], yabs ? &yabs[m * N + n] : NULL);
    return ORACLE_OK;
}

int oracle_linear_gs(const uint16_t* x, int64_t M, int64_t K, int64_t gs, const uint32_t* qweight,
                     const uint16_t* scales, const uint32_t* zeros, int64_t N,
                     const int32_t* row_ptr, const int32_t* col_idx, const uint16_t* values,
                     int64_t nnz, double* y, double* yabs) {
    return linear_bits(x, M, K, gs, 4, qweight, scales, zeros, N, row_ptr, col_idx, values, nnz, y, yabs);
}

int oracle_linear(const uint16_t* x, int64_t M, int64_t K, const uint32_t* qweight,
                  const uint16_t* scales, const uint32_t* zeros, int64_t N,
                  const int32_t* row_ptr, const int32_t* col_idx, const uint16_t* values,
                  int64_t nnz, double* y, double* yabs) {
    return oracle_linear_gs(x, M, K, GROUP, qweight, scales, zeros, N, row_ptr, col_idx, values, nnz, y, yabs);
}

/* The same outputs at P sampled positions (m_idx[p], n_idx[p]) only. */
static int linear_at_bits(const uint16_t* x, int64_t M, int64_t K, int64_t gs, int bits,
                          const uint32_t* qweight, const uint16_t* scales, const uint32_t* zeros, int64_t N,
                          const int32_t* row_ptr, const int32_t* col_idx, const uint16_t* values,
                          int64_t nnz, const int64_t* m_idx, const int64_t* n_idx, int64_t P,
                          double* y, double* yabs) {
    if (!x || !qweight || !scales || !zeros || !y || !m_idx || !n_idx) return ORACLE_ERR_NULL;
    if (M <= 0 || P < 0) return ORACLE_ERR_SHAPE;
    int st = check_qshape(N, K);
    if (!st) st = check_gs(K, gs);
    if (st) return st;
    st = check_csr(row_ptr, col_idx, values, nnz, N, K);
    if (st) return st;
    for (int64_t p = 0; p < P; ++p)
        if (m_idx[p] < 0 || m_idx[p] >= M || n_idx[p] < 0 || n_idx[p] >= N) return ORACLE_ERR_SHAPE;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t p = 0; p < P; ++p)
        one_output(x, K, N, gs, bits, qweight, scales, zeros, row_ptr, col_idx, values, m_idx[p], n_idx[p],
                   &y[p], yabs ? &yabs[p] : NULL);
    return ORACLE_OK;
}

int oracle_linear_at_gs(const uint16_t* x, int64_t M, int64_t K, int64_t gs, const uint32_t* qweight,
                        const uint16_t* scales, const uint32_t* zeros, int64_t N,
                        const int32_t* row_ptr, const int32_t* col_idx, const uint16_t* values,
                        int64_t nnz, const int64_t* m_idx, const int64_t* n_idx, int64_t P,
                        double* y, double* yabs) {
    return linear_at_bits(x, M, K, gs, 4, qweight, scales, zeros, N, row_ptr, col_idx, values, nnz, m_idx, n_idx,
                          P, y, yabs);
}

int oracle_linear_at(const uint16_t* x, int64_t M, int64_t K, const uint32_t* qweight,
                     const uint16_t* scales, const uint32_t* zeros, int64_t N,
                     const int32_t* row_ptr, const int32_t* col_idx, const uint16_t* values,
                     int64_t nnz, const int64_t* m_idx, const int64_t* n_idx, int64_t P,
                     double* y, double* yabs) {
    return oracle_linear_at_gs(x, M, K, GROUP, qweight, scales, zeros, N, row_ptr, col_idx, values, nnz, m_idx,
                               n_idx, P, y, yabs);
}

/* ------------------------------------------------------------------------------------
 * 3-bit codes [SqueezeLLM article, sections 2.1 and 2.2: once its few outliers are split
 * off, the dense part takes uniform quantization as coarse as 3 bits, eight levels].  Read
 * as the same asymmetric min/max RTN with 2^3 - 1 steps (quantize_group with qmax = 7),
 * the same groups, scales [K/gs][N] fp16 and zeros [K/gs][N/8] (nibbles, values 0..7).
 * Packed layout, 3 bits per weight: the 32 codes of k = 32 b .. 32 b + 31 of row n sit in
 * the three words qweight3[n][3 b + w], w = 0, 1, 2:
 *   - bits 4j .. 4j+2 of word w: the code of element 8 w + ORDER[j]     (elements 0..23);
 *   - bit 4j + 3 of word w: bit w of the code of element 24 + ORDER[j]  (elements 24..31).
 * Then (word >> 4i) & 0x00070007 holds elements (8 w + 2i, 8 w + 2i + 1) in its two 16-bit
 * halves, as 0x000F000F does for the 4-bit layout, and the bit-3 planes of the three words,
 * shifted by 4i + 3, 4i + 2 and 4i + 1 and masked with 0x00010001, 0x00020002 and
 * 0x00040004, hold elements (24 + 2i, 24 + 2i + 1) the same way.
 * ---------------------------------------------------------------------------------- */
int oracle_pack32x3(const uint8_t* q /* 32 codes, element order */, uint32_t* words /* 3 */) {
    uint32_t w[3] = {0u, 0u, 0u};
    for (int e = 0; e < 32; ++e)
        if (q[e] > 7) return ORACLE_ERR_VALUE;
    for (int wi = 0; wi < 3; ++wi)
        for (int j = 0; j < 8; ++j) {
            w[wi] |= (uint32_t)q[8 * wi + ORACLE_ORDER[j]] << (4 * j);
            w[wi] |= (uint32_t)((q[24 + ORACLE_ORDER[j]] >> wi) & 1u) << (4 * j + 3);
        }
    memcpy(words, w, sizeof w);
    return ORACLE_OK;
}

void oracle_unpack32x3(const uint32_t* words /* 3 */, uint8_t* q /* 32 codes, element order */) {
    for (int e = 0; e < 24; ++e) q[e] = (uint8_t)((words[e / 8] >> (4 * nibble_of_element(e % 8))) & 7u);
    for (int e = 24; e < 32; ++e) {
        const int j = nibble_of_element(e - 24);
        uint8_t c = 0;
        for (int wi = 0; wi < 3; ++wi) c |= (uint8_t)(((words[wi] >> (4 * j + 3)) & 1u) << wi);
        q[e] = c;
    }
}

/* awq_quantize with 3-bit codes: s from act_absmean and alpha, then W*s in groups of gs
 * (a multiple of 32 dividing K); qweight3 is [N][3K/32]. */
int oracle_awq_quantize3_gs(const float* W, const float* act_absmean, float alpha, int64_t N, int64_t K,
                            int64_t gs, uint32_t* qweight3, uint16_t* scales, uint32_t* zeros, float* s_out) {
    if (!W || !act_absmean || !qweight3 || !scales || !zeros) return ORACLE_ERR_NULL;
    int st = check_qshape(N, K);
    if (!st) st = check_gs(K, gs);
    if (!st && gs % 32 != 0) st = ORACLE_ERR_SHAPE;
    if (st) return st;
    float* s = (float*)malloc(sizeof(float) * (size_t)K);
    if (!s) return ORACLE_ERR_VALUE;
    st = oracle_awq_scales(act_absmean, K, alpha, s);
    if (!st) st = quantize_with_scales_bits(W, s, N, K, gs, 3, qweight3, scales, zeros);
    if (!st && s_out) memcpy(s_out, s, sizeof(float) * (size_t)K);
    free(s);
    return st;
}

/* deq[n][k] = (q - z) * sf for the 3-bit layout, exact in fp32. */
int oracle_dequant3_gs(const uint32_t* qweight3, const uint16_t* scales, const uint32_t* zeros, int64_t N,
                       int64_t K, int64_t gs, float* deq) {
    if (!qweight3 || !scales || !zeros || !deq) return ORACLE_ERR_NULL;
    int st = check_qshape(N, K);
    if (!st) st = check_gs(K, gs);
    if (st) return st;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            const int64_t g = k / gs;
            deq[n * K + k] = (float)(code_at(qweight3, 3, K, n, k) - zero_of(zeros, N, n, g)) *
                             oracle_f16_to_f32(scales[g * N + n]);
        }
    return ORACLE_OK;
}

/* The linear (all outputs, or P sampled ones) on 3-bit weights; otherwise as oracle_linear_gs. */
int oracle_linear3_gs(const uint16_t* x, int64_t M, int64_t K, int64_t gs, const uint32_t* qweight3,
                      const uint16_t* scales, const uint32_t* zeros, int64_t N, const int32_t* row_ptr,
                      const int32_t* col_idx, const uint16_t* values, int64_t nnz, double* y, double* yabs) {
    return linear_bits(x, M, K, gs, 3, qweight3, scales, zeros, N, row_ptr, col_idx, values, nnz, y, yabs);
}

int oracle_linear3_at_gs(const uint16_t* x, int64_t M, int64_t K, int64_t gs, const uint32_t* qweight3,
                         const uint16_t* scales, const uint32_t* zeros, int64_t N, const int32_t* row_ptr,
                         const int32_t* col_idx, const uint16_t* values, int64_t nnz, const int64_t* m_idx,
                         const int64_t* n_idx, int64_t P, double* y, double* yabs) {
    return linear_at_bits(x, M, K, gs, 3, qweight3, scales, zeros, N, row_ptr, col_idx, values, nnz, m_idx, n_idx,
                          P, y, yabs);
}

/* ------------------------------------------------------------------------------------
 * AWQ scale search [AWQ (MLSys 2024) translation, section 3.2: the per-channel scaling
 * factor is searched so that the quantized layer's output on calibration activations
 * stays closest to the full-precision output; with the closed form s = a^alpha the search
 * is over the exponent alpha].  For every alpha of the grid:
 *   s_k    = max(float(pow(a_k, alpha)), 1e-4)
 *   Q      = awq_quantize_g128(W, a, alpha)            (W * s, g128 RTN, packed)
 *   x'_mk  = bf16(float(x_mk) / s_k)                   (the runtime activation, 1/s folded in)
 *   yq_mn  = bf16(float(sum_k x'_mk deq_nk))           (the quantized layer, output in bf16)
 *   err    = sum_mn (yq_mn - yr_mn)^2 / sum_mn yr_mn^2,  yr_mn = sum_k x_mk W_nk  (double)
 * ---------------------------------------------------------------------------------- */
int oracle_awq_search_alpha(const float* W, const float* act_absmean, const uint16_t* x, int64_t M,
                            int64_t N, int64_t K, const float* alphas, int64_t n_alpha,
                            double* errors) {
    if (!W || !act_absmean || !x || !alphas || !errors) return ORACLE_ERR_NULL;
    if (M <= 0 || n_alpha <= 0) return ORACLE_ERR_SHAPE;
    int st = check_qshape(N, K);
    if (st) return st;
    double* yr = (double*)malloc(sizeof(double) * (size_t)(M * N));
    double* y = (double*)malloc(sizeof(double) * (size_t)(M * N));
    uint16_t* xs = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(M * K));
    uint32_t* qw = (uint32_t*)malloc(sizeof(uint32_t) * (size_t)(N * K / 8));
    uint16_t* sc = (uint16_t*)malloc(sizeof(uint16_t) * (size_t)(N * K / 128));
    uint32_t* z = (uint32_t*)malloc(sizeof(uint32_t) * (size_t)(N * K / 1024));
    float* s = (float*)malloc(sizeof(float) * (size_t)K);
    if (!yr || !y || !xs || !qw || !sc || !z || !s) st = ORACLE_ERR_VALUE;
    /* the full-precision output */
    double ref2 = 0.0;
    if (!st) {
#pragma omp parallel for collapse(2) schedule(static)
        for (int64_t m = 0; m < M; ++m)
            for (int64_t n = 0; n < N; ++n) {
                double acc = 0.0;
                for (int64_t k = 0; k < K; ++k)
                    acc += (double)oracle_bf16_to_f32(x[m * K + k]) * (double)W[n * K + k];
                yr[m * N + n] = acc;
            }
        for (int64_t i = 0; i < M * N; ++i) ref2 += yr[i] * yr[i];
    }
    for (int64_t a = 0; a < n_alpha && !st; ++a) {
        st = oracle_awq_quantize_g128(W, act_absmean, alphas[a], N, K, qw, sc, z, s);
        if (st) break;
        for (int64_t m = 0; m < M; ++m)
            for (int64_t k = 0; k < K; ++k)
                xs[m * K + k] = oracle_f32_to_bf16(oracle_bf16_to_f32(x[m * K + k]) / s[k]);
        st = oracle_linear(xs, M, K, qw, sc, z, N, NULL, NULL, NULL, 0, y, NULL);
        if (st) break;
        double e2 = 0.0;
        for (int64_t i = 0; i < M * N; ++i) {
            const double yq = (double)oracle_bf16_to_f32(oracle_f32_to_bf16((float)y[i]));
            e2 += (yq - yr[i]) * (yq - yr[i]);
        }
        errors[a] = ref2 > 0.0 ? e2 / ref2 : e2;
    }
    free(yr); free(y); free(xs); free(qw); free(sc); free(z); free(s);
    return st;
}

/* ------------------------------------------------------------------------------------
 * Outlier split [SqueezeLLM article, 2.2; the selection rule |w| * act_absmean replaces
 * the Hessian sensitivity, which needs a trained model and data]:
 *   score(n,k) = float(|w[n][k]| * a_k) on the original W;
 *   the nnz largest scores are selected; equal scores are taken in increasing linear
 *   index n*K + k;
 *   W_dense = W with the selected entries set to 0;
 *   CSR of the selected entries, rows in order, columns ascending,
 *   value = fp16_rne(float(w * s_k)) (the same scaled space as the quantized weights).
 * ---------------------------------------------------------------------------------- */
static int cmp_desc_u64(const void* a, const void* b) {
    uint64_t x = *(const uint64_t*)a, y = *(const uint64_t*)b;
    return x < y ? 1 : (x > y ? -1 : 0);
}

int oracle_split_outliers(const float* W, const float* act_absmean, float alpha, int64_t N,
                          int64_t K, int64_t nnz, float* W_dense, int32_t* row_ptr,
                          int32_t* col_idx, uint16_t* values) {
    if (!W || !act_absmean || !W_dense || !row_ptr) return ORACLE_ERR_NULL;
    if (N <= 0 || K <= 0 || nnz < 0 || nnz > N * K) return ORACLE_ERR_SHAPE;
    if (nnz > 0 && (!col_idx || !values)) return ORACLE_ERR_NULL;
    if ((uint64_t)N * (uint64_t)K > 0xFFFFFFFFull || nnz > 0x7FFFFFFF) return ORACLE_ERR_SHAPE;
    const int64_t NK = N * K;
    float* s = (float*)malloc(sizeof(float) * (size_t)K);
    uint64_t* key = (uint64_t*)malloc(sizeof(uint64_t) * (size_t)NK);
    uint8_t* chosen = (uint8_t*)calloc((size_t)NK, 1);
    int st = (s && key && chosen) ? ORACLE_OK : ORACLE_ERR_VALUE;
    if (!st) st = oracle_awq_scales(act_absmean, K, alpha, s);
    for (int64_t i = 0; !st && i < NK; ++i)
        if (!isfinite(W[i])) st = ORACLE_ERR_VALUE;
    if (!st) {
        for (int64_t i = 0; i < NK; ++i) {
            float score = fabsf(W[i]) * act_absmean[i % K];
            uint32_t bits;
            memcpy(&bits, &score, 4); /* non-negative floats order like their bit patterns */
            /* larger score first; among equal scores the lower index first */
            key[i] = ((uint64_t)bits << 32) | (uint64_t)(0xFFFFFFFFu - (uint32_t)i);
        }
        qsort(key, (size_t)NK, sizeof(uint64_t), cmp_desc_u64);
        for (int64_t t = 0; t < nnz; ++t) chosen[0xFFFFFFFFu - (uint32_t)(key[t] & 0xFFFFFFFFu)] = 1;
        int64_t j = 0;
        row_ptr[0] = 0;
        for (int64_t n = 0; n < N && !st; ++n) {
            for (int64_t k = 0; k < K; ++k) {
                int64_t i = n * K + k;
                if (chosen[i]) {
                    uint16_t h = oracle_f32_to_f16(W[i] * s[k]);
                    if ((h & 0x7FFFu) == 0x7C00u) { st = ORACLE_ERR_VALUE; break; }
                    col_idx[j] = (int32_t)k;
                    values[j] = h;
                    ++j;
                    W_dense[i] = 0.0f;
                } else {
                    W_dense[i] = W[i];
                }
            }
            row_ptr[n + 1] = (int32_t)j;
        }
    }
    free(s);
    free(key);
    free(chosen);
    return st;
}

/* ------------------------------------------------------------------------------------
 * NVFP4 weights [DeepCompressor README: the toolbox fake-quantizes to FP4_E2M1, and its
 * result tables list NVFP4 models].  The pages name the format but do not define it; it is
 * read here as the published layout:
 *   - elements: FP4 E2M1, bit 3 the sign, bits 2..1 the exponent (bias 1), bit 0 the
 *     mantissa: magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6;
 *   - one FP8 E4M3 scale per 16 consecutive weights along K of a row (bit 7 the sign, 4
 *     exponent bits with bias 7, 3 mantissa bits; largest finite 448, no infinities);
 *   - one fp32 scale per tensor.
 * On W' = W * s (the same activation-aware scaling as the 4-bit path), with one IEEE float
 * operation per step:
 *   g   = amax|W'| / 2688                (2688 = 6 * 448; g = 1 when W' is all zero)
 *   sb  = amax|block| / fp32(6 * g)
 *   s8  = e4m3(sb): round to nearest, ties to the even mantissa, saturating at 448
 *   S   = fp32(float(s8) * g)
 *   q   = e2m1(fp32(w' / S)): nearest, ties to the even mantissa, saturating at 6, the sign
 *         bit that of the quotient (also for a zero); q = 0 in a block whose S is 0
 * Dequantization: w~ = e2m1(q) * float(s8) * g, exact in double.  Codes are packed 8 per
 * 32-bit word with the 4-bit ORDER interleave (qweight [N][K/8]); the scales are bytes,
 * group-major like the fp16 scales (scales8 [K/16][N]).
 * ---------------------------------------------------------------------------------- */

/* E4M3 from the format definition: normal values (1 + m/8) 2^(e-7), e = 1..15 (not
 * e = 15 with m = 7, the NaN), subnormals m 2^-9.  Arithmetic in double is exact. */
uint8_t oracle_f32_to_e4m3(float f) {
    uint8_t sign = signbit(f) ? 0x80u : 0u;
    if (isnan(f)) return (uint8_t)(sign | 0x7Fu);
    double a = fabs((double)f);
    if (a > 448.0) return (uint8_t)(sign | 0x7Eu); /* saturate */
    if (a < ldexp(1.0, -6)) {                      /* subnormal range: step 2^-9 */
        double m = rint(a * 512.0);                /* ties to even */
        return (uint8_t)(sign | (uint8_t)m);       /* m = 8 is the smallest normal, 0x08 */
    }
    int ex;
    frexp(a, &ex); /* a = fr 2^ex, fr in [0.5, 1) */
    int e = ex - 1;
    double m = rint((ldexp(a, -e) - 1.0) * 8.0);
    if (m == 8.0) {
        m = 0.0;
        e += 1;
    }
    if (e > 8 || (e == 8 && m > 6.0)) return (uint8_t)(sign | 0x7Eu);
    return (uint8_t)(sign | (uint8_t)((e + 7) << 3) | (uint8_t)m);
}

float oracle_e4m3_to_f32(uint8_t b) {
    double s = (b & 0x80u) ? -1.0 : 1.0;
    int e = (b >> 3) & 15, m = b & 7;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) return (float)(s * ldexp((double)m, -9));
    return (float)(s * ldexp(1.0 + m / 8.0, e - 7));
}

/* E2M1 magnitudes by code (bits 2..0). */
static const double E2M1[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

float oracle_e2m1_to_f32(uint8_t c) {
    return (float)(((c & 8u) ? -1.0 : 1.0) * E2M1[c & 7u]);
}

/* Nearest E2M1 value, ties to the even mantissa (the code with bit 0 clear), saturating at
 * 6; the sign bit is the argument's.  Returns 0xFF for NaN. */
uint8_t oracle_f32_to_e2m1(float r) {
    if (isnan(r)) return 0xFFu;
    uint8_t sign = signbit(r) ? 8u : 0u;
    double a = fabs((double)r);
    int best = 0;
    for (int c = 1; c < 8; ++c) {
        double d = fabs(a - E2M1[c]), db = fabs(a - E2M1[best]);
        if (d < db || (d == db && (c & 1) == 0)) best = c;
    }
    return (uint8_t)(sign | (uint8_t)best);
}

/* NVFP4 quantization of W' = W * s (see the section comment): qweight [N][K/8], scales8
 * [K/16][N], *gscale = g.  K a multiple of 16, N of 8. */
int oracle_quantize_nvfp4_with_scales(const float* W, const float* s, int64_t N, int64_t K, uint32_t* qweight,
                                      uint8_t* scales8, float* gscale) {
    if (!W || !s || !qweight || !scales8 || !gscale) return ORACLE_ERR_NULL;
    if (N <= 0 || N % 8 != 0 || K <= 0 || K % 16 != 0) return ORACLE_ERR_SHAPE;
    float amax = 0.0f;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            float w = W[n * K + k] * s[k];
            if (!isfinite(w)) return ORACLE_ERR_VALUE;
            if (fabsf(w) > amax) amax = fabsf(w);
        }
    float g = amax > 0.0f ? amax / 2688.0f : 1.0f;
    float six_g = 6.0f * g;
    int err = ORACLE_OK;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < N; ++n) {
        for (int64_t b = 0; b < K / 16; ++b) {
            float wp[16];
            float bmax = 0.0f;
            for (int i = 0; i < 16; ++i) {
                wp[i] = W[n * K + 16 * b + i] * s[16 * b + i];
                if (fabsf(wp[i]) > bmax) bmax = fabsf(wp[i]);
            }
            float sb = bmax / six_g;
            uint8_t s8 = oracle_f32_to_e4m3(sb);
            float S = oracle_e4m3_to_f32(s8) * g;
            uint8_t q[16];
            for (int i = 0; i < 16; ++i) {
                if (S == 0.0f) {
                    q[i] = 0;
                    continue;
                }
                uint8_t c = oracle_f32_to_e2m1(wp[i] / S);
                if (c == 0xFFu) {
#pragma omp atomic write
                    err = ORACLE_ERR_VALUE;
                    c = 0;
                }
                q[i] = c;
            }
            scales8[b * N + n] = s8;
            oracle_pack8(&q[0], &qweight[n * (K / 8) + 2 * b]);
            oracle_pack8(&q[8], &qweight[n * (K / 8) + 2 * b + 1]);
        }
    }
    *gscale = g;
    return err;
}

/* awq_quantize with NVFP4 weights: s from act_absmean and alpha, then the NVFP4 steps on W*s. */
int oracle_awq_quantize_nvfp4(const float* W, const float* act_absmean, float alpha, int64_t N, int64_t K,
                              uint32_t* qweight, uint8_t* scales8, float* gscale, float* s_out) {
    if (!W || !act_absmean || !qweight || !scales8 || !gscale) return ORACLE_ERR_NULL;
    if (N <= 0 || N % 8 != 0 || K <= 0 || K % 16 != 0) return ORACLE_ERR_SHAPE;
    float* s = (float*)malloc(sizeof(float) * (size_t)K);
    if (!s) return ORACLE_ERR_VALUE;
    int st = oracle_awq_scales(act_absmean, K, alpha, s);
    if (!st) st = oracle_quantize_nvfp4_with_scales(W, s, N, K, qweight, scales8, gscale);
    if (!st && s_out) memcpy(s_out, s, sizeof(float) * (size_t)K);
    free(s);
    return st;
}

/* w~[n][k] = e2m1(q) * float(s8) * g, in double (exact). */
int oracle_dequant_nvfp4(const uint32_t* qweight, const uint8_t* scales8, float g, int64_t N, int64_t K,
                         double* out) {
    if (!qweight || !scales8 || !out) return ORACLE_ERR_NULL;
    if (N <= 0 || N % 8 != 0 || K <= 0 || K % 16 != 0) return ORACLE_ERR_SHAPE;
    for (int64_t n = 0; n < N; ++n)
        for (int64_t k = 0; k < K; ++k) {
            uint8_t codes[8];
            oracle_unpack8(qweight[n * (K / 8) + k / 8], codes);
            out[n * K + k] = (double)oracle_e2m1_to_f32(codes[k % 8]) *
                             (double)oracle_e4m3_to_f32(scales8[(k / 16) * N + n]) * (double)g;
        }
    return ORACLE_OK;
}

/* y = x w~^T (+ x W_sparse^T) in double for all (m, n), as oracle_linear. */
int oracle_linear_nvfp4(const uint16_t* x, int64_t M, int64_t K, const uint32_t* qweight, const uint8_t* scales8,
                        float g, int64_t N, const int32_t* row_ptr, const int32_t* col_idx, const uint16_t* values,
                        int64_t nnz, double* y, double* yabs) {
    if (!x || !qweight || !scales8 || !y) return ORACLE_ERR_NULL;
    if (M <= 0 || N <= 0 || N % 8 != 0 || K <= 0 || K % 16 != 0) return ORACLE_ERR_SHAPE;
    int st = check_csr(row_ptr, col_idx, values, nnz, N, K);
    if (st) return st;
    double* w = (double*)malloc(sizeof(double) * (size_t)(N * K));
    if (!w) return ORACLE_ERR_VALUE;
    st = oracle_dequant_nvfp4(qweight, scales8, g, N, K, w);
    if (st) {
        free(w);
        return st;
    }
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t m = 0; m < M; ++m)
        for (int64_t n = 0; n < N; ++n) {
            double acc = 0.0, aacc = 0.0;
            for (int64_t k = 0; k < K; ++k) {
                double p = (double)oracle_bf16_to_f32(x[m * K + k]) * w[n * K + k];
                acc += p;
                aacc += fabs(p);
            }
            if (row_ptr)
                for (int64_t j = row_ptr[n]; j < row_ptr[n + 1]; ++j) {
                    double p = (double)oracle_bf16_to_f32(x[m * K + col_idx[j]]) *
                               (double)oracle_f16_to_f32(values[j]);
                    acc += p;
                    aacc += fabs(p);
                }
            y[m * N + n] = acc;
            if (yabs) yabs[m * N + n] = aacc;
        }
    free(w);
    return ORACLE_OK;
}
