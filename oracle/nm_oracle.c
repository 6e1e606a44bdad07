/*
 * nm_oracle.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, obviously-correct CPU statement of what the N:M sparse GEMM
 * path computes.  Only the test-suite, the smoke check and the CPU-baseline leg
 * of the benchmark may load it.  It shares no source with the CUDA library.
 *
 * Source: "Realizable N:M Sparse Transformer Inference via Search-Kernel
 * Co-Design" (arXiv 2607.12505).
 *   - section 2.1: N:M sparsity keeps N non-zeros in every group of M weights.
 *   - section 4.2: the micro-dense kernel materialises exactly those N values
 *     per window and runs regular dense MMA fragments on them, so its result is
 *     the dense GEMM over the masked weight.  The packed format carries the
 *     values and their positions inside each window.
 * Readings where the paper is silent (all listed in the design notes):
 *   - groups run along K (the reduction axis), contiguous, aligned at k = 0;
 *   - selection is by magnitude, ties go to the lower in-group position;
 *   - exactly N slots are stored per group (zeros are chosen by the same rule);
 *   - kept values are stored in ascending in-group position.
 *
 * Arithmetic:
 *   - INT8 GEMM: exact int64 accumulation, then checked to fit int32;
 *   - INT8 scaled: (float)acc rounded to nearest, then one fp32 multiply
 *     (build with -ffp-contract=off);
 *   - FP16/BF16 GEMM: inputs decoded exactly to double, fp64 accumulation,
 *     result returned in fp64.
 *   - fused output stage (per-channel scale, per-channel bias, GELU, int8
 *     requantisation): the library's own definition, see oracle_epilogue_i8;
 *     the paper does not discuss the output stage.
 *
 * Tile-shared compress (oracle_compress_tile): the same top-N rule with the
 * column mass of a tile of V rows as the magnitude, so a tile's rows share one
 * pattern (the vector-wise reading; the paper does not fix the granularity).
 *
 * Parity pins (tests/test_oracle.py): hand-worked 4x8 examples, brute-force
 * subset enumeration, invariants, and exact integer matmul cross-checks; for
 * the output stage, hand-worked rounding/saturation cases
 * (tests/golden/epilogue_hand.json), the standard normal CDF table for GELU
 * and the identity GELU(x) - GELU(-x) = x; for the tile-shared compress,
 * hand-worked 4x8 examples (tests/golden/tile_hand.json), brute-force
 * enumeration of the subsets of largest tile mass, the V = 1 reduction to the
 * per-row rule, and an fp16 case that single-precision sums would decide wrongly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_INT8 = 0, OR_FP16 = 1, OR_BF16 = 2 };

/* ---- exact decoders for the 16-bit float formats (IEEE binary16, bfloat16) */

static double fp16_to_double(uint16_t h) {
    int sign = h >> 15;
    int e = (h >> 10) & 0x1f;
    int m = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)m, -24);                 /* subnormal: m * 2^-24 */
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(m | 0x400), e - 25);    /* (1.m) * 2^(e-15) */
    return sign ? -v : v;
}

static double bf16_to_double(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static size_t elem_size(int dtype) { return dtype == OR_INT8 ? 1 : 2; }

/* |w| of element i as a double (exact for all three formats). */
static double magnitude(const void *w, int dtype, int64_t i) {
    if (dtype == OR_INT8) return fabs((double)((const int8_t *)w)[i]);
    uint16_t h = ((const uint16_t *)w)[i];
    return fabs(dtype == OR_FP16 ? fp16_to_double(h) : bf16_to_double(h));
}

int oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* Bytes of the 4-bit index stream of one row: one nibble per kept element,
 * two per byte, low nibble first; a row with an odd count ends in a zero
 * high nibble so that rows never share a byte. */
int64_t oracle_idx_pitch(int64_t k, int N, int M) {
    int64_t kept = (k / M) * N;
    return (kept + 1) / 2;
}

/*
 * Compress: for every row r and every group g of M consecutive K positions,
 * position p is kept iff fewer than N positions q of the same group precede it
 * in the order (|w| descending, position ascending).  That is the top-N rule
 * with ties to the lower index, written as a rank test.  Kept positions come
 * out in ascending order because p is scanned upward.
 *
 * values: [n_out][k/M][N] elements of the weight dtype.
 * idx:    [n_out][idx_pitch] bytes; element e of a row sits in byte e/2,
 *         low nibble when e is even.
 * Returns 0, or -1 for an invalid argument.
 */
int oracle_compress(const void *W, int64_t n_out, int64_t k, int dtype, int N, int M,
                    void *values, uint8_t *idx) {
    if (!W || !values || !idx || n_out <= 0 || k <= 0 || M <= 0 || M > 16 || N <= 0 ||
        N > M || k % M != 0 || dtype < 0 || dtype > 2)
        return -1;
    const size_t es = elem_size(dtype);
    const int64_t groups = k / M;
    const int64_t pitch = oracle_idx_pitch(k, N, M);
    memset(idx, 0, (size_t)(n_out * pitch));
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < n_out; ++r) {
        int64_t e = 0; /* kept-element counter within the row */
        for (int64_t g = 0; g < groups; ++g) {
            const int64_t base = r * k + g * M;
            for (int p = 0; p < M; ++p) {
                double ap = magnitude(W, dtype, base + p);
                int ahead = 0;
                for (int q = 0; q < M; ++q) {
                    double aq = magnitude(W, dtype, base + q);
                    if (aq > ap || (aq == ap && q < p)) ++ahead;
                }
                if (ahead < N) {
                    memcpy((char *)values + (size_t)(r * groups * N + e) * es,
                           (const char *)W + (size_t)(base + p) * es, es);
                    uint8_t *byte = idx + r * pitch + e / 2;
                    *byte |= (uint8_t)((p & 0xF) << ((e & 1) ? 4 : 0));
                    ++e;
                }
            }
        }
    }
    return 0;
}

/*
 * Tile-shared compress, the vector-wise reading of the micro-dense format
 * (section 4.2: the kept values of a window become a dense tile that regular
 * MMA fragments consume, the activations being gathered to match).  For a
 * gather to serve a whole tile of output channels, those channels must keep
 * the same positions, so rows are taken in tiles of V consecutive rows (the
 * last tile may be shorter) and, in every tile and group of M positions:
 *   score(p) = sum over the tile's rows of |w[r][gM + p]|,
 *   p is kept iff fewer than N positions q of the group precede it in the
 *   order (score descending, position ascending).
 * This is the top-N rule of oracle_compress with the tile's column mass as the
 * magnitude; V = 1 is exactly oracle_compress.  Output uses the same canonical
 * layout as oracle_compress (every row of a tile carries the same positions).
 *
 * Scores are exact.  int8 magnitudes are integers.  fp16 magnitudes are whole
 * multiples of 2^-24 below 2^16, so a sum of V <= 4096 of them is a multiple of
 * 2^-24 below 2^28, i.e. an integer below 2^52 in units of 2^-24: exact in
 * double.  bfloat16 sums can round, so bfloat16 is refused (-3).
 * Returns 0, -1 for an invalid argument, -3 for an unsupported dtype.
 */
int oracle_compress_tile(const void *W, int64_t n_out, int64_t k, int dtype, int N, int M,
                         int64_t V, void *values, uint8_t *idx) {
    if (!W || !values || !idx || n_out <= 0 || k <= 0 || M <= 0 || M > 16 || N <= 0 ||
        N > M || k % M != 0 || dtype < 0 || dtype > 2 || V <= 0 || V > 4096)
        return -1;
    if (dtype == OR_BF16) return -3;
    const size_t es = elem_size(dtype);
    const int64_t groups = k / M;
    const int64_t pitch = oracle_idx_pitch(k, N, M);
    const int64_t tiles = (n_out + V - 1) / V;
    memset(idx, 0, (size_t)(n_out * pitch));
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < tiles; ++t) {
        const int64_t r0 = t * V;
        const int64_t r1 = r0 + V < n_out ? r0 + V : n_out;
        for (int64_t g = 0; g < groups; ++g) {
            double score[16];
            for (int p = 0; p < M; ++p) {
                score[p] = 0.0;
                for (int64_t r = r0; r < r1; ++r) score[p] += magnitude(W, dtype, r * k + g * M + p);
            }
            int e = 0; /* kept-element counter within the group */
            for (int p = 0; p < M; ++p) {
                int ahead = 0;
                for (int q = 0; q < M; ++q)
                    if (score[q] > score[p] || (score[q] == score[p] && q < p)) ++ahead;
                if (ahead >= N) continue;
                for (int64_t r = r0; r < r1; ++r) {
                    const int64_t el = g * N + e; /* element index within the row */
                    memcpy((char *)values + (size_t)(r * groups * N + el) * es,
                           (const char *)W + (size_t)(r * k + g * M + p) * es, es);
                    idx[r * pitch + el / 2] |= (uint8_t)((p & 0xF) << ((el & 1) ? 4 : 0));
                }
                ++e;
            }
        }
    }
    return 0;
}

/* Decompress: scatter every kept value to its position; all else is zero. */
int oracle_decompress(const void *values, const uint8_t *idx, int64_t n_out, int64_t k,
                      int dtype, int N, int M, void *Wm) {
    if (!values || !idx || !Wm || n_out <= 0 || k <= 0 || M <= 0 || N <= 0 || N > M ||
        k % M != 0 || dtype < 0 || dtype > 2)
        return -1;
    const size_t es = elem_size(dtype);
    const int64_t groups = k / M;
    const int64_t pitch = oracle_idx_pitch(k, N, M);
    memset(Wm, 0, (size_t)(n_out * k) * es);
    for (int64_t r = 0; r < n_out; ++r) {
        for (int64_t e = 0; e < groups * N; ++e) {
            uint8_t byte = idx[r * pitch + e / 2];
            int p = (e & 1) ? (byte >> 4) : (byte & 0xF);
            int64_t g = e / N;
            memcpy((char *)Wm + (size_t)(r * k + g * M + p) * es,
                   (const char *)values + (size_t)(r * groups * N + e) * es, es);
        }
    }
    return 0;
}

/*
 * INT8 GEMM over the masked weight: Y[t][n] = sum_k X[t][k] * Wm[n][k].
 * Exact int64 accumulation; returns -2 if any result leaves the int32 range
 * (it cannot for |x| <= 128, |w| <= 128, k <= 131072).
 * When scale is non-NULL the result is written to Yf as
 * (float)acc * scale[n] (round-to-nearest conversion, one fp32 multiply);
 * otherwise to Yi as int32.
 */
int oracle_gemm_i8(const int8_t *X, int64_t T, int64_t K, const int8_t *Wm, int64_t n_out,
                   const float *scale, int32_t *Yi, float *Yf) {
    if (!X || !Wm || T < 0 || K <= 0 || n_out <= 0 || (!scale && !Yi) || (scale && !Yf))
        return -1;
    int bad = 0;
#pragma omp parallel for schedule(static) reduction(| : bad)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t n = 0; n < n_out; ++n) {
            int64_t acc = 0;
            for (int64_t kk = 0; kk < K; ++kk)
                acc += (int64_t)X[t * K + kk] * (int64_t)Wm[n * K + kk];
            if (acc > INT32_MAX || acc < INT32_MIN) bad = 1;
            if (scale) {
                float f = (float)(int32_t)acc;
                float s = scale[n];
                volatile float prod = f * s; /* a single rounded fp32 multiply */
                Yf[t * n_out + n] = prod;
            } else {
                Yi[t * n_out + n] = (int32_t)acc;
            }
        }
    }
    return bad ? -2 : 0;
}

/*
 * FP16/BF16 GEMM over the masked weight, in fp64:
 * Y[t][n] = (sum_k x(t,k) * w(n,k)) * (scale ? scale[n] : 1), every input
 * decoded exactly; the result stays in double for the tolerance check.
 */
int oracle_gemm_f16(const uint16_t *X, int64_t T, int64_t K, const uint16_t *Wm, int64_t n_out,
                    int dtype, const float *scale, double *Y) {
    if (!X || !Wm || !Y || T < 0 || K <= 0 || n_out <= 0 || (dtype != OR_FP16 && dtype != OR_BF16))
        return -1;
    double (*dec)(uint16_t) = dtype == OR_FP16 ? fp16_to_double : bf16_to_double;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t n = 0; n < n_out; ++n) {
            double acc = 0.0;
            for (int64_t kk = 0; kk < K; ++kk)
                acc += dec(X[t * K + kk]) * dec(Wm[n * K + kk]);
            Y[t * n_out + n] = scale ? acc * (double)scale[n] : acc;
        }
    }
    return 0;
}

/*
 * Fused output stage applied to the GEMM accumulator.  The paper does not
 * discuss the output stage (its kernel description ends at the MMA), so this
 * is the library's own definition, written out step by step:
 *
 *   v = a                              a = (float)acc, rounded to nearest
 *   v = v * scale[n]   (if scale)      one rounded fp32 multiply
 *   v = v + bias[n]    (if bias)       one rounded fp32 add
 *   g = v / 2 * (1 + erf(v / sqrt 2))  (if act == 1: the erf form of GELU, in fp64)
 *   int8 output: q = clamp(round-half-even(g * out_scale), -128, 127)
 *
 * For act == 0 every step is one IEEE fp32 operation, so the result is exact
 * and fixed: v32 holds v, q is decided in fp32 (one rounded multiply, then
 * rintf).  For act == 1 the GELU is evaluated in fp64 from the fp32 v; pre
 * holds g (fp64) and q is decided from g * out_scale in fp64.  Any of pre,
 * v32, q may be NULL.
 */
static double gelu_erf(double x) { return 0.5 * x * (1.0 + erf(x / sqrt(2.0))); }

static int8_t sat_s8(double r) { return (int8_t)(r > 127.0 ? 127 : (r < -128.0 ? -128 : r)); }

int oracle_epilogue_i8(const int32_t *acc, int64_t T, int64_t n_out, const float *scale,
                       const float *bias, int act, float out_scale, double *pre, float *v32,
                       int8_t *q) {
    if (!acc || T < 0 || n_out <= 0 || (act != 0 && act != 1)) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t n = 0; n < n_out; ++n) {
            const int64_t i = t * n_out + n;
            volatile float v = (float)acc[i];
            if (scale) v = v * scale[n];
            if (bias) v = v + bias[n];
            if (v32) v32[i] = v;
            if (act == 1) {
                const double g = gelu_erf((double)v);
                if (pre) pre[i] = g;
                if (q) q[i] = sat_s8(rint(g * (double)out_scale));
            } else {
                if (pre) pre[i] = (double)v;
                if (q) {
                    volatile float p = v * out_scale;
                    q[i] = sat_s8((double)rintf(p));
                }
            }
        }
    }
    return 0;
}

/*
 * The same output stage for the FP16/BF16 path, all in fp64 on the fp64
 * accumulator (the kernel's fp32 result is compared against it within the
 * tolerance):  g = act(acc * scale[n] + bias[n]).
 */
int oracle_epilogue_f(const double *acc, int64_t T, int64_t n_out, const float *scale,
                      const float *bias, int act, double *pre) {
    if (!acc || !pre || T < 0 || n_out <= 0 || (act != 0 && act != 1)) return -1;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t n = 0; n < n_out; ++n) {
            const int64_t i = t * n_out + n;
            double v = acc[i];
            if (scale) v *= (double)scale[n];
            if (bias) v += (double)bias[n];
            pre[i] = act == 1 ? gelu_erf(v) : v;
        }
    }
    return 0;
}

/* GELU alone, for the pins (closed forms of the normal CDF). */
double oracle_gelu(double x) { return gelu_erf(x); }
