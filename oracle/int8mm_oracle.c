/*
 * Plain CPU oracle for the LLM.int8() matrix multiplication  Y = X * W.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
 * statement of what the GPU library computes.  Only the test suite, the
 * package smoke check and the benchmark's CPU-baseline leg may load it.  It
 * shares no code, header, table or constant generator with the CUDA path.
 *
 * Source of the method: "LLM.int8(): 8-bit Matrix Multiplication for
 * Transformers at Scale" (Dettmers, Lewis, Belkada, Zettlemoyer, 2022),
 * abstract: a two-part procedure for the feed-forward and attention
 * projection matmuls -- vector-wise quantisation with one normalisation
 * constant per inner-product vector, plus a mixed-precision decomposition
 * that moves the outlier feature dimensions into a 16-bit matmul.  The axolotl
 * "llama3-model-quantization" summary of the same talk adds: outliers sit in
 * specific feature columns of the input ("Understanding Outliers in
 * Transformer Models"), they are processed in 16 bit and the rest in 8 bit
 * ("Key Points"), and quantisation normalises by the maximum value
 * ("Key Points", block-wise paragraph).  The scite report for nuQmm quotes
 * that LLM.int8() rounds to the nearest quantisation level (RTN).
 *
 * Numerics (the plainest reading where the pages leave a step open):
 *   - fp16 inputs are converted to fp32 exactly;
 *   - a feature column k is an outlier when |X[m,k]| >= threshold for ANY
 *     row m of this call; the outlier list is ascending;
 *   - row absmax ra[m] is taken over the non-outlier columns only;
 *   - scale = 127.0f / absmax (IEEE fp32 division, round to nearest even),
 *     q = round-half-even(x * scale) in fp32, clamped to [-127, 127];
 *     absmax == 0 gives q = 0 and a stored absmax of 0;
 *   - weight absmax ca[n] is taken per output channel over ALL K;
 *   - int8 products are summed exactly (int64, then checked to fit int32);
 *   - the 16-bit outlier product sums fp32(xo)*fp32(wo) in fp32 in
 *     ascending outlier order;
 *   - outlier weight rows come from the fp16 rows kept at preparation time,
 *     else from the dequantised int8 row fp16(q * ca / 127);
 *   - y = fp16( (float)acc * ra[m] * ca[n] / 16129 + o ), left to right.
 *
 * Three variants follow the vector-wise matmul at the end of the file, with
 * the same per-value rule: a block-wise linear 8-bit codec of an fp32 vector,
 * the group-wise matmul (one constant per group of G consecutive inner
 * indices) and a 4-bit weight-only product.  The GPU library does not
 * implement them yet.
 *
 * Build: gcc -O2 -ffp-contract=off (no fast-math), -pthread.
 */
#include <fenv.h>
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* IEEE binary16 <-> binary32, written from the format definition.          */
/* ------------------------------------------------------------------------ */

float orc_half_to_float(uint16_t h) {
    int sign = (h >> 15) & 1;
    int exp = (h >> 10) & 0x1f;
    int mant = h & 0x3ff;
    float v;
    if (exp == 0) {
        v = ldexpf((float)mant, -24); /* zero or subnormal: mant * 2^-24 */
    } else if (exp == 31) {
        v = mant ? NAN : INFINITY;
    } else {
        v = ldexpf((float)(1024 + mant), exp - 25); /* (1.mant) * 2^(exp-15) */
    }
    return sign ? -v : v;
}

/* Round-to-nearest-even conversion of a binary32 value to binary16 bits. */
uint16_t orc_float_to_half(float f) {
    uint16_t sign = signbit(f) ? 0x8000u : 0u;
    if (isnan(f)) return (uint16_t)(sign | 0x7e00u);
    float a = fabsf(f);
    /* 65520 is the midpoint between 65504 (odd mantissa) and 2^16: ties go
       to the even neighbour, which overflows to infinity. */
    if (a >= 65520.0f) return (uint16_t)(sign | 0x7c00u);
    if (a < ldexpf(1.0f, -14)) {
        /* subnormal range: value = n * 2^-24, n rounded half-even; n == 1024
           lands exactly on the smallest normal, whose bits are 0x0400. */
        float n = nearbyintf(ldexpf(a, 24));
        return (uint16_t)(sign | (uint16_t)n);
    }
    int e;
    frexpf(a, &e);          /* a = fr * 2^e, fr in [0.5, 1) */
    e -= 1;                 /* a = 1.x * 2^e */
    float m = nearbyintf(ldexpf(a, 10 - e)); /* in [1024, 2048] */
    if (m == 2048.0f) {
        m = 1024.0f;
        e += 1;
    }
    if (e + 15 >= 31) return (uint16_t)(sign | 0x7c00u);
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)((int)m - 1024));
}

/* ------------------------------------------------------------------------ */
/* Shared quantisation rule: one vector, its absmax, scale and codes.        */
/* ------------------------------------------------------------------------ */

static int8_t quantize_one(float x, float scale) {
    float r = nearbyintf(x * scale); /* fp32 product, then half-even */
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/* ------------------------------------------------------------------------ */
/* (a) Outlier feature detection.                                            */
/* A column is an outlier when any row reaches the threshold in magnitude.   */
/* Writes the ascending outlier column list to idx (capacity K) and returns  */
/* its length.                                                               */
/* ------------------------------------------------------------------------ */

int orc_detect_outliers(const uint16_t* X, int M, int K, float thr, int32_t* idx) {
    fesetround(FE_TONEAREST);
    int n = 0;
    for (int k = 0; k < K; ++k) {
        int flag = 0;
        for (int m = 0; m < M; ++m) {
            float x = orc_half_to_float(X[(size_t)m * K + k]);
            if (fabsf(x) >= thr) {
                flag = 1;
                break;
            }
        }
        if (flag) idx[n++] = k;
    }
    return n;
}

/* ------------------------------------------------------------------------ */
/* (b) Row-wise (vector-wise) int8 quantisation of X with the outlier        */
/* columns removed, plus the fp16 outlier sub-matrix Xo (M x n_o).           */
/* ------------------------------------------------------------------------ */

void orc_quantize_rows(const uint16_t* X, int M, int K, const int32_t* idx, int n_o,
                       int8_t* Xq, float* ra, uint16_t* Xo) {
    fesetround(FE_TONEAREST);
    unsigned char* is_out = (unsigned char*)calloc((size_t)K > 0 ? (size_t)K : 1, 1);
    for (int j = 0; j < n_o; ++j) is_out[idx[j]] = 1;
    for (int m = 0; m < M; ++m) {
        const uint16_t* row = X + (size_t)m * K;
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            if (is_out[k]) continue;
            float a = fabsf(orc_half_to_float(row[k]));
            if (a > amax) amax = a;
        }
        ra[m] = amax;
        float scale = amax > 0.0f ? 127.0f / amax : 0.0f;
        for (int k = 0; k < K; ++k) {
            int8_t q = 0;
            if (!is_out[k] && amax > 0.0f) q = quantize_one(orc_half_to_float(row[k]), scale);
            Xq[(size_t)m * K + k] = q;
        }
        for (int j = 0; j < n_o; ++j) Xo[(size_t)m * n_o + j] = row[idx[j]];
    }
    free(is_out);
}

/* ------------------------------------------------------------------------ */
/* (c) One-time per-output-channel int8 quantisation of W (K x N, row-major) */
/* into Wq (N x K: row n holds output channel n) and ca (N).                 */
/* ------------------------------------------------------------------------ */

void orc_quantize_weight(const uint16_t* W, int K, int N, int8_t* Wq, float* ca) {
    fesetround(FE_TONEAREST);
    for (int n = 0; n < N; ++n) {
        float amax = 0.0f;
        for (int k = 0; k < K; ++k) {
            float a = fabsf(orc_half_to_float(W[(size_t)k * N + n]));
            if (a > amax) amax = a;
        }
        ca[n] = amax;
        float scale = amax > 0.0f ? 127.0f / amax : 0.0f;
        for (int k = 0; k < K; ++k) {
            int8_t q = 0;
            if (amax > 0.0f) q = quantize_one(orc_half_to_float(W[(size_t)k * N + n]), scale);
            Wq[(size_t)n * K + k] = q;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* (d1) Exact int8 product acc[m,n] = sum_k Xq[m,k] * Wq[n,k].               */
/* Rows are split across threads; each sum is an exact int64 checked to fit */
/* int32.  Returns 0, or -1 if some sum does not fit.                        */
/* ------------------------------------------------------------------------ */

typedef struct {
    const int8_t* Xq;
    const int8_t* Wq;
    int M, N, K, m0, m1;
    int32_t* acc;
    int overflow;
} gemm_job;

static void* gemm_rows(void* p) {
    gemm_job* j = (gemm_job*)p;
    for (int m = j->m0; m < j->m1; ++m) {
        const int8_t* a = j->Xq + (size_t)m * j->K;
        for (int n = 0; n < j->N; ++n) {
            const int8_t* b = j->Wq + (size_t)n * j->K;
            int64_t s = 0;
            for (int k = 0; k < j->K; ++k) s += (int64_t)a[k] * (int64_t)b[k];
            if (s > INT32_MAX || s < INT32_MIN) j->overflow = 1;
            j->acc[(size_t)m * j->N + n] = (int32_t)s;
        }
    }
    return NULL;
}

int orc_int8_gemm(const int8_t* Xq, const int8_t* Wq, int M, int N, int K, int32_t* acc,
                  int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > M) nthreads = M > 0 ? M : 1;
    gemm_job* jobs = (gemm_job*)calloc((size_t)nthreads, sizeof(gemm_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int t = 0; t < nthreads; ++t) {
        jobs[t].Xq = Xq;
        jobs[t].Wq = Wq;
        jobs[t].M = M;
        jobs[t].N = N;
        jobs[t].K = K;
        jobs[t].m0 = (int)((int64_t)M * t / nthreads);
        jobs[t].m1 = (int)((int64_t)M * (t + 1) / nthreads);
        jobs[t].acc = acc;
        jobs[t].overflow = 0;
        if (t > 0) pthread_create(&th[t], NULL, gemm_rows, &jobs[t]);
    }
    if (nthreads > 0) gemm_rows(&jobs[0]);
    int overflow = jobs[0].overflow;
    for (int t = 1; t < nthreads; ++t) {
        pthread_join(th[t], NULL);
        overflow |= jobs[t].overflow;
    }
    free(jobs);
    free(th);
    return overflow ? -1 : 0;
}

/* The same exact sum at a list of (m, n) points only. */
int orc_int8_gemm_points(const int8_t* Xq, const int8_t* Wq, int K, const int32_t* pm,
                         const int32_t* pn, int npts, int32_t* acc) {
    int overflow = 0;
    for (int p = 0; p < npts; ++p) {
        const int8_t* a = Xq + (size_t)pm[p] * K;
        const int8_t* b = Wq + (size_t)pn[p] * K;
        int64_t s = 0;
        for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)b[k];
        if (s > INT32_MAX || s < INT32_MIN) overflow = 1;
        acc[p] = (int32_t)s;
    }
    return overflow ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* The fp16 weight rows of the outlier dimensions.                           */
/* Wo (n_o x N): row j is W[idx[j], :] -- the fp16 row kept at preparation   */
/* time when idx[j] is among keep_idx, else the dequantised row              */
/* fp16((float)Wq[n, idx[j]] * ca[n] / 127).                                 */
/* W_keep is n_keep x N, row i holding W[keep_idx[i], :].                    */
/* ------------------------------------------------------------------------ */

void orc_gather_w_outlier(const uint16_t* W_keep, const int32_t* keep_idx, int n_keep,
                          const int8_t* Wq, const float* ca, int K, int N, const int32_t* idx,
                          int n_o, uint16_t* Wo) {
    fesetround(FE_TONEAREST);
    for (int j = 0; j < n_o; ++j) {
        int k = idx[j];
        int slot = -1;
        for (int i = 0; i < n_keep; ++i)
            if (keep_idx[i] == k) {
                slot = i;
                break;
            }
        for (int n = 0; n < N; ++n) {
            uint16_t w;
            if (slot >= 0) {
                w = W_keep[(size_t)slot * N + n];
            } else {
                float t = (float)Wq[(size_t)n * K + k] * ca[n];
                w = orc_float_to_half(t / 127.0f);
            }
            Wo[(size_t)j * N + n] = w;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* (d2) 16-bit outlier product o[m,n] = sum_j Xo[m,j] * Wo[j,n] in fp32,     */
/* ascending j.                                                              */
/* ------------------------------------------------------------------------ */

static float outlier_dot(const uint16_t* Xo, const uint16_t* Wo, int N, int n_o, int m, int n) {
    float s = 0.0f;
    for (int j = 0; j < n_o; ++j)
        s += orc_half_to_float(Xo[(size_t)m * n_o + j]) * orc_half_to_float(Wo[(size_t)j * N + n]);
    return s;
}

void orc_outlier_gemm(const uint16_t* Xo, const uint16_t* Wo, int M, int N, int n_o, float* o) {
    fesetround(FE_TONEAREST);
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) o[(size_t)m * N + n] = outlier_dot(Xo, Wo, N, n_o, m, n);
}

/* ------------------------------------------------------------------------ */
/* (d3) Dequantise and combine: y = fp16(acc * ra * ca / 16129 + o).         */
/* ------------------------------------------------------------------------ */

static uint16_t combine(int32_t acc, float ra, float ca, float o) {
    float v = (float)acc;
    v = v * ra;
    v = v * ca;
    v = v / 16129.0f;
    v = v + o;
    return orc_float_to_half(v);
}

void orc_epilogue(const int32_t* acc, const float* ra, const float* ca, const float* o, int M,
                  int N, uint16_t* Y) {
    fesetround(FE_TONEAREST);
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            size_t i = (size_t)m * N + n;
            Y[i] = combine(acc[i], ra[m], ca[n], o ? o[i] : 0.0f);
        }
}

/* y at a list of points, from the quantised operands (acc computed here). */
int orc_forward_points(const int8_t* Xq, const float* ra, const int8_t* Wq, const float* ca,
                       const uint16_t* Xo, const uint16_t* Wo, int K, int N, int n_o,
                       const int32_t* pm, const int32_t* pn, int npts, int32_t* acc_out,
                       uint16_t* y_out) {
    fesetround(FE_TONEAREST);
    int rc = orc_int8_gemm_points(Xq, Wq, K, pm, pn, npts, acc_out);
    for (int p = 0; p < npts; ++p) {
        float o = outlier_dot(Xo, Wo, N, n_o, pm[p], pn[p]);
        y_out[p] = combine(acc_out[p], ra[pm[p]], ca[pn[p]], o);
    }
    return rc;
}

/* ======================================================================== */
/* Variants beyond the vector-wise matmul                                   */
/* ======================================================================== */

/* ------------------------------------------------------------------------ */
/* Block-wise linear 8-bit codec of an fp32 vector.  The axolotl             */
/* "llama3-model-quantization" summary ("8-Bit Optimizers") describes it for */
/* optimizer state: cut the vector into blocks, normalise each block by its  */
/* own maximum and store an 8-bit index per value, so an outlier coarsens    */
/* only its own block.  Levels are linear (equal bins, "Key Points"); the    */
/* rule per value is the matmul's: scale = 127/absmax, half-even rounding of */
/* the fp32 product, clamp to [-127, 127]; absmax 0 gives codes 0.           */
/* Block b covers [b*B, min(n, (b+1)*B)): the last block may be short.       */
/* Inputs are finite.                                                        */
/* ------------------------------------------------------------------------ */

void orc_block_quantize(const float* x, long n, int B, int8_t* q, float* absmax) {
    fesetround(FE_TONEAREST);
    long nb = (n + B - 1) / B;
    for (long b = 0; b < nb; ++b) {
        long lo = b * (long)B;
        long hi = lo + B < n ? lo + B : n;
        float amax = 0.0f;
        for (long i = lo; i < hi; ++i) {
            float a = fabsf(x[i]);
            if (a > amax) amax = a;
        }
        absmax[b] = amax;
        float scale = amax > 0.0f ? 127.0f / amax : 0.0f;
        for (long i = lo; i < hi; ++i) q[i] = amax > 0.0f ? quantize_one(x[i], scale) : 0;
    }
}

/* x'[i] = (q[i] * absmax[block of i]) / 127 in fp32, left to right. */
void orc_block_dequantize(const int8_t* q, const float* absmax, long n, int B, float* out) {
    fesetround(FE_TONEAREST);
    for (long i = 0; i < n; ++i) {
        float t = (float)q[i] * absmax[i / B];
        out[i] = t / 127.0f;
    }
}

/* ------------------------------------------------------------------------ */
/* Group-wise int8 matmul: the vector-wise method with one normalisation    */
/* constant per group of G consecutive inner-product indices instead of one */
/* per whole vector (the granularity of nuQmm and ZeroQuant, which the      */
/* scite report for nuQmm cites as finer than vector-wise; its GPTQ snippet */
/* puts runs of consecutive weights under one constant).  G divides K.  The */
/* outlier decomposition is unchanged: outlier columns are zero in the int8 */
/* operand and go through the 16-bit product; a group whose every column is */
/* an outlier has absmax 0.                                                  */
/*   ra[m*ng + g] = max |X[m,k]| over k in group g, k not an outlier        */
/*   ca[n*ng + g] = max |W[k,n]| over k in group g                          */
/*   acc_g[m,n]   = sum over k in group g of Xq[m,k] * Wq[n,k] (exact)      */
/*   y = fp16( sum_g acc_g * ra * ca / 16129 (fp32, ascending g) + o )      */
/* With G = K every step is the vector-wise one, bit for bit.               */
/* ------------------------------------------------------------------------ */

void orc_quantize_rows_grouped(const uint16_t* X, int M, int K, int G, const int32_t* idx, int n_o,
                               int8_t* Xq, float* ra, uint16_t* Xo) {
    fesetround(FE_TONEAREST);
    int ng = K / G;
    unsigned char* is_out = (unsigned char*)calloc((size_t)K > 0 ? (size_t)K : 1, 1);
    for (int j = 0; j < n_o; ++j) is_out[idx[j]] = 1;
    for (int m = 0; m < M; ++m) {
        const uint16_t* row = X + (size_t)m * K;
        for (int g = 0; g < ng; ++g) {
            float amax = 0.0f;
            for (int k = g * G; k < (g + 1) * G; ++k) {
                if (is_out[k]) continue;
                float a = fabsf(orc_half_to_float(row[k]));
                if (a > amax) amax = a;
            }
            ra[(size_t)m * ng + g] = amax;
            float scale = amax > 0.0f ? 127.0f / amax : 0.0f;
            for (int k = g * G; k < (g + 1) * G; ++k) {
                int8_t q = 0;
                if (!is_out[k] && amax > 0.0f) q = quantize_one(orc_half_to_float(row[k]), scale);
                Xq[(size_t)m * K + k] = q;
            }
        }
        for (int j = 0; j < n_o; ++j) Xo[(size_t)m * n_o + j] = row[idx[j]];
    }
    free(is_out);
}

void orc_quantize_weight_grouped(const uint16_t* W, int K, int N, int G, int8_t* Wq, float* ca) {
    fesetround(FE_TONEAREST);
    int ng = K / G;
    for (int n = 0; n < N; ++n) {
        for (int g = 0; g < ng; ++g) {
            float amax = 0.0f;
            for (int k = g * G; k < (g + 1) * G; ++k) {
                float a = fabsf(orc_half_to_float(W[(size_t)k * N + n]));
                if (a > amax) amax = a;
            }
            ca[(size_t)n * ng + g] = amax;
            float scale = amax > 0.0f ? 127.0f / amax : 0.0f;
            for (int k = g * G; k < (g + 1) * G; ++k) {
                int8_t q = 0;
                if (amax > 0.0f) q = quantize_one(orc_half_to_float(W[(size_t)k * N + n]), scale);
                Wq[(size_t)n * K + k] = q;
            }
        }
    }
}

/* Wo (n_o x N) for the group-wise weight: the kept fp16 row, else the row  */
/* dequantised with its own group's constant, fp16((q * ca[n, k/G]) / 127). */
void orc_gather_w_outlier_grouped(const uint16_t* W_keep, const int32_t* keep_idx, int n_keep,
                                  const int8_t* Wq, const float* ca, int K, int N, int G,
                                  const int32_t* idx, int n_o, uint16_t* Wo) {
    fesetround(FE_TONEAREST);
    int ng = K / G;
    for (int j = 0; j < n_o; ++j) {
        int k = idx[j];
        int slot = -1;
        for (int i = 0; i < n_keep; ++i)
            if (keep_idx[i] == k) {
                slot = i;
                break;
            }
        for (int n = 0; n < N; ++n) {
            uint16_t w;
            if (slot >= 0) {
                w = W_keep[(size_t)slot * N + n];
            } else {
                float t = (float)Wq[(size_t)n * K + k] * ca[(size_t)n * ng + k / G];
                w = orc_float_to_half(t / 127.0f);
            }
            Wo[(size_t)j * N + n] = w;
        }
    }
}

/* acc_g (optional, M x N x ng) and Y (M x N) of the group-wise product;    */
/* o (M x N fp32, may be NULL) is the 16-bit outlier product.  Returns 0,   */
/* or -1 if a group sum does not fit int32.                                 */
int orc_grouped_forward(const int8_t* Xq, const float* ra, const int8_t* Wq, const float* ca,
                        const float* o, int M, int N, int K, int G, int32_t* acc_out, uint16_t* Y) {
    fesetround(FE_TONEAREST);
    int ng = K / G;
    int overflow = 0;
    for (int m = 0; m < M; ++m) {
        const int8_t* a = Xq + (size_t)m * K;
        for (int n = 0; n < N; ++n) {
            const int8_t* b = Wq + (size_t)n * K;
            float v = 0.0f;
            for (int g = 0; g < ng; ++g) {
                int64_t s = 0;
                for (int k = g * G; k < (g + 1) * G; ++k) s += (int64_t)a[k] * (int64_t)b[k];
                if (s > INT32_MAX || s < INT32_MIN) overflow = 1;
                if (acc_out) acc_out[((size_t)m * N + n) * ng + g] = (int32_t)s;
                float t = (float)(int32_t)s;
                t = t * ra[(size_t)m * ng + g];
                t = t * ca[(size_t)n * ng + g];
                t = t / 16129.0f;
                v = v + t;
            }
            v = v + (o ? o[(size_t)m * N + n] : 0.0f);
            Y[(size_t)m * N + n] = orc_float_to_half(v);
        }
    }
    return overflow ? -1 : 0;
}

/* ------------------------------------------------------------------------ */
/* 4-bit weight-only product for decode-sized X.  Inference is bound by     */
/* loading the weights, so fewer bits per weight cut its time at the same   */
/* parameter count (video of the talk, "4-Bit Inference"; axolotl page,     */
/* "Impact of Precision and Parameter Count").  Weights get linear 4-bit    */
/* codes in [-7, 7] with one constant per output column and group of G      */
/* consecutive k (G divides K), by the same rule as the 8-bit codes with 7  */
/* in place of 127; X stays fp16.                                           */
/*   ca[n*ng + g] = max |W[k,n]| over k in group g                          */
/*   q[n*K + k]   = clamp(round-half-even(RN32(W[k,n] * RN32(7/ca))), +-7)  */
/*   w'           = RN32(RN32(q * ca) / 7)                                  */
/*   Y[m,n]       = fp16( sum_k x[m,k] * w'[k,n] ), summed in double        */
/* ------------------------------------------------------------------------ */

/* Round-to-nearest-even conversion of a binary64 value to binary16 bits. */
uint16_t orc_double_to_half(double f) {
    uint16_t sign = signbit(f) ? 0x8000u : 0u;
    if (isnan(f)) return (uint16_t)(sign | 0x7e00u);
    double a = fabs(f);
    if (a >= 65520.0) return (uint16_t)(sign | 0x7c00u);
    if (a < ldexp(1.0, -14)) return (uint16_t)(sign | (uint16_t)nearbyint(ldexp(a, 24)));
    int e;
    frexp(a, &e);
    e -= 1;
    double m = nearbyint(ldexp(a, 10 - e));
    if (m == 2048.0) {
        m = 1024.0;
        e += 1;
    }
    if (e + 15 >= 31) return (uint16_t)(sign | 0x7c00u);
    return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)((int)m - 1024));
}

void orc_quantize_weight_int4(const uint16_t* W, int K, int N, int G, int8_t* q, float* ca) {
    fesetround(FE_TONEAREST);
    int ng = K / G;
    for (int n = 0; n < N; ++n) {
        for (int g = 0; g < ng; ++g) {
            float amax = 0.0f;
            for (int k = g * G; k < (g + 1) * G; ++k) {
                float a = fabsf(orc_half_to_float(W[(size_t)k * N + n]));
                if (a > amax) amax = a;
            }
            ca[(size_t)n * ng + g] = amax;
            float scale = amax > 0.0f ? 7.0f / amax : 0.0f;
            for (int k = g * G; k < (g + 1) * G; ++k) {
                int8_t c = 0;
                if (amax > 0.0f) {
                    float r = nearbyintf(orc_half_to_float(W[(size_t)k * N + n]) * scale);
                    if (r > 7.0f) r = 7.0f;
                    if (r < -7.0f) r = -7.0f;
                    c = (int8_t)r;
                }
                q[(size_t)n * K + k] = c;
            }
        }
    }
}

void orc_int4_product(const uint16_t* X, const int8_t* q, const float* ca, int M, int N, int K, int G,
                      uint16_t* Y) {
    fesetround(FE_TONEAREST);
    int ng = K / G;
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            double s = 0.0;
            for (int k = 0; k < K; ++k) {
                float t = (float)q[(size_t)n * K + k] * ca[(size_t)n * ng + k / G];
                float w = t / 7.0f;
                s += (double)orc_half_to_float(X[(size_t)m * K + k]) * (double)w;
            }
            Y[(size_t)m * N + n] = orc_double_to_half(s);
        }
}

/* The group-wise product at a list of (m, n) points: acc_g (npts x ng) and */
/* Y, the same arithmetic as orc_grouped_forward.  Returns 0, or -1 if a    */
/* group sum does not fit int32.                                            */
int orc_grouped_points(const int8_t* Xq, const float* ra, const int8_t* Wq, const float* ca,
                       const uint16_t* Xo, const uint16_t* Wo, int K, int N, int G, int n_o,
                       const int32_t* pm, const int32_t* pn, int npts, int32_t* acc_out,
                       uint16_t* y_out) {
    fesetround(FE_TONEAREST);
    int ng = K / G;
    int overflow = 0;
    for (int p = 0; p < npts; ++p) {
        const int8_t* a = Xq + (size_t)pm[p] * K;
        const int8_t* b = Wq + (size_t)pn[p] * K;
        float v = 0.0f;
        for (int g = 0; g < ng; ++g) {
            int64_t s = 0;
            for (int k = g * G; k < (g + 1) * G; ++k) s += (int64_t)a[k] * (int64_t)b[k];
            if (s > INT32_MAX || s < INT32_MIN) overflow = 1;
            acc_out[(size_t)p * ng + g] = (int32_t)s;
            float t = (float)(int32_t)s;
            t = t * ra[(size_t)pm[p] * ng + g];
            t = t * ca[(size_t)pn[p] * ng + g];
            t = t / 16129.0f;
            v = v + t;
        }
        v = v + outlier_dot(Xo, Wo, N, n_o, pm[p], pn[p]);
        y_out[p] = orc_float_to_half(v);
    }
    return overflow ? -1 : 0;
}

/* The 4-bit weight-only product at a list of (m, n) points. */
void orc_int4_points(const uint16_t* X, const int8_t* q, const float* ca, int K, int G, const int32_t* pm,
                     const int32_t* pn, int npts, uint16_t* y_out) {
    fesetround(FE_TONEAREST);
    int ng = K / G;
    for (int p = 0; p < npts; ++p) {
        double s = 0.0;
        for (int k = 0; k < K; ++k) {
            float t = (float)q[(size_t)pn[p] * K + k] * ca[(size_t)pn[p] * ng + k / G];
            float w = t / 7.0f;
            s += (double)orc_half_to_float(X[(size_t)pm[p] * K + k]) * (double)w;
        }
        y_out[p] = orc_double_to_half(s);
    }
}
