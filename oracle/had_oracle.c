/*
 * had_oracle.c -- plain, slow CPU oracle for the Hamming Attention
 * Distillation (HAD) inference forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA library and must never be used as
 * a fallback for it.
 *
 * What it computes follows "Hamming Attention Distillation: Binarizing Keys
 * and Queries for Efficient Long-Context Transformers" (arXiv 2502.01770) as
 * described on the pith.science review page, section "What carries the
 * argument" and the circularity audit (Eqs. 4-7, Eq. 12):
 *
 *   1. standardize Q and K by the data-estimated coefficients sigma_Q,
 *      sigma_K (Eq. 12), then sign-quantize to {-1,+1} (Eqs. 4-5);
 *   2. the logit of query i and key j is the +/-1 dot product, which the
 *      pages compute as a Hamming distance (XNOR + popcount) (Eq. 5);
 *   3. a top-N mask keeps only the N largest logits of each row (Eq. 6);
 *   4. softmax over the kept logits only (Eq. 7), then the sparse product
 *      with the full-precision value matrix (the referee report notes that
 *      values and the attention map stay in full precision).
 *
 * Readings where the pages are silent:
 *   - sigma is one positive fp32 number per head; z = x / sigma is an IEEE
 *     fp32 round-to-nearest division with subnormals kept;
 *   - sign(z) = -1 iff z < 0; +0, -0 and NaN give +1;
 *   - the logit is the dot product s = d - 2*Hamming; a softmax temperature
 *     tau multiplies it (the caller passes tau; 1/sqrt(d) in the workloads);
 *   - ties at the N-th largest logit go to the lower key index, so exactly N
 *     keys are kept; the kept indices are reported in ascending order;
 *   - softmax and the value product are evaluated in fp64, stored as fp32.
 *
 * Nothing here is blocked, fused or reordered beyond those definitions: the
 * logit is a +/-1 dot-product loop (not a popcount, so the popcount identity
 * is something the tests check rather than assume), the top-N is a full
 * sort of the row, and the softmax/value product is a plain double loop.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static float bf16_to_float(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

static float load_elem(const void *x, int is_bf16, long i)
{
    return is_bf16 ? bf16_to_float(((const uint16_t *)x)[i])
                   : ((const float *)x)[i];
}

/*
 * Step 1 (Eqs. 4-5, Eq. 12): sign of x / sigma[h] for every element of a
 * [B,H,n,d] tensor.  Writes +1 or -1 into sign_out (same layout).
 */
void had_oracle_binarize(const void *x, int x_is_bf16, const float *sigma,
                         long B, long H, long n, long d, int8_t *sign_out)
{
    for (long b = 0; b < B; ++b)
        for (long h = 0; h < H; ++h) {
            float sg = sigma[h];
            long base = (b * H + h) * n * d;
            for (long e = 0; e < n * d; ++e) {
                float z = load_elem(x, x_is_bf16, base + e) / sg;
                sign_out[base + e] = (z < 0.0f) ? (int8_t)-1 : (int8_t)1;
            }
        }
}

/*
 * Bit-packed form of the signs (the "binary" Q/K the pages store as bits):
 * bit k of word w of a row is 1 iff the sign of element 32*w + k is -1.
 */
void had_oracle_pack(const int8_t *sign, long rows, long d, uint32_t *bits)
{
    long words = d / 32;
    for (long r = 0; r < rows; ++r)
        for (long w = 0; w < words; ++w) {
            uint32_t word = 0;
            for (int k = 0; k < 32; ++k)
                if (sign[r * d + 32 * w + k] < 0)
                    word |= (uint32_t)1 << k;
            bits[r * words + w] = word;
        }
}

/* Step 2 (Eq. 5): logits of one query row against every key of its head. */
static void row_logits(const int8_t *sq_row, const int8_t *sk_head, long n,
                       long d, int32_t *s)
{
    for (long j = 0; j < n; ++j) {
        int32_t acc = 0;
        const int8_t *kr = sk_head + j * d;
        for (long k = 0; k < d; ++k)
            acc += (int32_t)sq_row[k] * (int32_t)kr[k];
        s[j] = acc;
    }
}

typedef struct {
    int32_t s;
    int32_t j;
} keyed_t;

/* Larger logit first; equal logits: lower key index first. */
static int by_logit_then_index(const void *a, const void *b)
{
    const keyed_t *x = (const keyed_t *)a, *y = (const keyed_t *)b;
    if (x->s != y->s)
        return (x->s > y->s) ? -1 : 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int by_index(const void *a, const void *b)
{
    const keyed_t *x = (const keyed_t *)a, *y = (const keyed_t *)b;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

/*
 * Logits of a list of query rows.  rows[] holds flat row ids
 * r = (b*H + h)*n + i; s_out is [nrows, n].
 */
void had_oracle_logits_rows(const int8_t *sq, const int8_t *sk, long B,
                            long H, long n, long d, const int64_t *rows,
                            long nrows, int32_t *s_out, int nthreads)
{
    (void)B;
    (void)H;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 4)
#endif
    for (long t = 0; t < nrows; ++t) {
        long r = (long)rows[t];
        long head = r / n;
        row_logits(sq + r * d, sk + head * n * d, n, d, s_out + t * n);
    }
}

/*
 * Steps 2-4 for a list of query rows.  Outputs (all [nrows, ...]):
 *   idx_out  [nrows, N]  kept key indices, ascending;
 *   s_out    [nrows, N]  their logits;
 *   p_out    [nrows, N]  softmax probabilities (fp64), or NULL;
 *   o_out    [nrows, d]  attention output (fp64 sums stored as fp32).
 * V is [B,H,n,d] fp32 or bf16 bits.  Returns 0, or -1 on a bad argument or
 * allocation failure.
 */
int had_oracle_attention_rows(const int8_t *sq, const int8_t *sk,
                              const void *v, int v_is_bf16, long B, long H,
                              long n, long d, long N, float tau,
                              const int64_t *rows, long nrows,
                              int32_t *idx_out, int16_t *s_out, double *p_out,
                              float *o_out, int nthreads)
{
    (void)B;
    (void)H;
    if (N < 1 || N > n || d < 1 || n < 1)
        return -1;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        int32_t *s = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
        keyed_t *order = (keyed_t *)malloc(sizeof(keyed_t) * (size_t)n);
        double *e = (double *)malloc(sizeof(double) * (size_t)N);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
        for (long t = 0; t < nrows; ++t) {
            if (!s || !order || !e) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                failed = 1;
                continue;
            }
            {
                long r = (long)rows[t];
                long head = r / n;
                row_logits(sq + r * d, sk + head * n * d, n, d, s);

                /* Eq. 6: the N largest logits, ties to the lower index. */
                for (long j = 0; j < n; ++j) {
                    order[j].s = s[j];
                    order[j].j = (int32_t)j;
                }
                qsort(order, (size_t)n, sizeof(keyed_t), by_logit_then_index);
                qsort(order, (size_t)N, sizeof(keyed_t), by_index);

                /* Eq. 7: softmax over the kept logits only (fp64). */
                int32_t m = order[0].s;
                for (long k = 1; k < N; ++k)
                    if (order[k].s > m)
                        m = order[k].s;
                double Z = 0.0;
                for (long k = 0; k < N; ++k) {
                    e[k] = exp((double)tau * (double)(order[k].s - m));
                    Z += e[k];
                }
                for (long k = 0; k < N; ++k) {
                    idx_out[t * N + k] = order[k].j;
                    s_out[t * N + k] = (int16_t)order[k].s;
                    if (p_out)
                        p_out[t * N + k] = e[k] / Z;
                }

                /* Sparse product with the full-precision values. */
                const long vbase = head * n * d;
                for (long c = 0; c < d; ++c) {
                    double acc = 0.0;
                    for (long k = 0; k < N; ++k)
                        acc += (e[k] / Z) *
                               (double)load_elem(v, v_is_bf16,
                                                 vbase + (long)order[k].j * d + c);
                    o_out[t * d + c] = (float)acc;
                }
            }
        }
        free(s);
        free(order);
        free(e);
    }
    return failed ? -1 : 0;
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
/*
 * Causal variant (the review's note that decoder LLMs are the target of the
 * long-context claims; the pages print no causal rule, so this is the plain
 * reading): query i of a head sees keys 0 .. i only and keeps the
 * N_i = min(N, i + 1) largest visible logits, ties to the lower index, in
 * ascending key order; softmax over the kept logits and the value product
 * as in the non-causal case.  Slots N_i .. N-1 of a row are empty: idx -1,
 * logit 0, p 0.
 */
int had_oracle_attention_causal_rows(const int8_t *sq, const int8_t *sk,
                                     const void *v, int v_is_bf16, long B,
                                     long H, long n, long d, long N,
                                     float tau, const int64_t *rows,
                                     long nrows, int32_t *idx_out,
                                     int16_t *s_out, double *p_out,
                                     float *o_out, int nthreads)
{
    (void)B;
    (void)H;
    if (N < 1 || N > n || d < 1 || n < 1)
        return -1;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        int32_t *s = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
        keyed_t *order = (keyed_t *)malloc(sizeof(keyed_t) * (size_t)n);
        double *e = (double *)malloc(sizeof(double) * (size_t)N);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
        for (long t = 0; t < nrows; ++t) {
            if (!s || !order || !e) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                failed = 1;
                continue;
            }
            long r = (long)rows[t];
            long head = r / n;
            long i = r % n;                  /* position of the query */
            long vis = i + 1;                /* keys 0 .. i are visible */
            long Ni = N < vis ? N : vis;
            row_logits(sq + r * d, sk + head * n * d, vis, d, s);
            for (long j = 0; j < vis; ++j) {
                order[j].s = s[j];
                order[j].j = (int32_t)j;
            }
            qsort(order, (size_t)vis, sizeof(keyed_t), by_logit_then_index);
            qsort(order, (size_t)Ni, sizeof(keyed_t), by_index);
            int32_t m = order[0].s;
            for (long k = 1; k < Ni; ++k)
                if (order[k].s > m)
                    m = order[k].s;
            double Z = 0.0;
            for (long k = 0; k < Ni; ++k) {
                e[k] = exp((double)tau * (double)(order[k].s - m));
                Z += e[k];
            }
            for (long k = 0; k < N; ++k) {
                const int kept = k < Ni;
                idx_out[t * N + k] = kept ? order[k].j : -1;
                s_out[t * N + k] = kept ? (int16_t)order[k].s : 0;
                if (p_out)
                    p_out[t * N + k] = kept ? e[k] / Z : 0.0;
            }
            const long vbase = head * n * d;
            for (long c = 0; c < d; ++c) {
                double acc = 0.0;
                for (long k = 0; k < Ni; ++k)
                    acc += (e[k] / Z) *
                           (double)load_elem(v, v_is_bf16,
                                             vbase + (long)order[k].j * d + c);
                o_out[t * d + c] = (float)acc;
            }
        }
        free(s);
        free(order);
        free(e);
    }
    return failed ? -1 : 0;
}

/* Larger weight first. */
static int by_weight_desc(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x < y) - (x > y);
}

/*
 * Top-N mass retention: the pages' premise that a small N keeps most of the
 * softmax mass of a row (pith.science review, the "concrete test" and the
 * free-parameter notes on N).  For each listed row and each threshold p_k
 * in (0, 1]: the smallest N such that the N largest weights of the full
 * softmax over all n keys (temperature tau, binarized logits) hold at least
 * p_k of the row's total.  Plain definition in fp64: weights
 * exp(tau (s_j - max s)), sorted in descending order, summed one by one;
 * the total Z is the same running sum at N = n, and N is the first count
 * whose running sum reaches p_k * Z.  Returns 0, or -1 on bad arguments or
 * an allocation failure.
 */
int had_oracle_topn_mass_rows(const int8_t *sq, const int8_t *sk, long B,
                              long H, long n, long d, double tau,
                              const double *p, int np, const int64_t *rows,
                              long nrows, int32_t *nmin_out, int nthreads)
{
    (void)B;
    (void)H;
    if (n < 1 || d < 1 || np < 1)
        return -1;
    for (int k = 0; k < np; ++k)
        if (!(p[k] > 0.0) || p[k] > 1.0)
            return -1;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        int32_t *s = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
        double *w = (double *)malloc(sizeof(double) * (size_t)n);
        double *cum = (double *)malloc(sizeof(double) * (size_t)n);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
        for (long t = 0; t < nrows; ++t) {
            if (!s || !w || !cum) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                failed = 1;
                continue;
            }
            long r = (long)rows[t];
            long head = r / n;
            row_logits(sq + r * d, sk + head * n * d, n, d, s);
            int32_t m = s[0];
            for (long j = 1; j < n; ++j)
                if (s[j] > m)
                    m = s[j];
            for (long j = 0; j < n; ++j)
                w[j] = exp(tau * (double)(s[j] - m));
            qsort(w, (size_t)n, sizeof(double), by_weight_desc);
            double acc = 0.0;
            for (long j = 0; j < n; ++j) {
                acc += w[j];
                cum[j] = acc;
            }
            const double Z = cum[n - 1];
            for (int k = 0; k < np; ++k) {
                const double target = p[k] * Z;
                long N = n;
                for (long j = 0; j < n; ++j)
                    if (cum[j] >= target) {
                        N = j + 1;
                        break;
                    }
                nmin_out[t * np + k] = (int32_t)N;
            }
        }
        free(s);
        free(w);
        free(cum);
    }
    return failed ? -1 : 0;
}

/*
 * Soft binarization, the forward pass of training stages 1-2 (pith.science
 * review of arXiv 2502.01770: the annealing schedule starts from a scaled
 * tanh whose scale c moves it toward the sign function, Eq. 13, before the
 * straight-through stage).  Reading taken: the code of an element is
 * t = tanh(c * z) with z = x / sigma[h] as in step 1 (fp32 division), the
 * product c * z rounded to fp32, tanh evaluated in fp64 and rounded to fp32.
 * The codes are fp32 numbers in (-1, 1), approaching +/-1 as c grows.
 */
void had_oracle_soft_binarize(const void *x, int x_is_bf16, const float *sigma,
                              float c, long B, long H, long n, long d,
                              float *t_out)
{
    for (long b = 0; b < B; ++b)
        for (long h = 0; h < H; ++h) {
            float sg = sigma[h];
            long base = (b * H + h) * n * d;
            for (long e = 0; e < n * d; ++e) {
                float z = load_elem(x, x_is_bf16, base + e) / sg;
                float u = c * z;
                t_out[base + e] = (float)tanh((double)u);
            }
        }
}

/* Soft logits of one query row: the dot product of the fp32 codes, in fp64. */
static void row_soft_logits(const float *tq_row, const float *tk_head, long n,
                            long d, double *s)
{
    for (long j = 0; j < n; ++j) {
        double acc = 0.0;
        const float *kr = tk_head + j * d;
        for (long k = 0; k < d; ++k)
            acc += (double)tq_row[k] * (double)kr[k];
        s[j] = acc;
    }
}

/* Soft logits [nrows, n] (fp64) of a list of flat query rows. */
void had_oracle_soft_logits_rows(const float *tq, const float *tk, long B,
                                 long H, long n, long d, const int64_t *rows,
                                 long nrows, double *s_out, int nthreads)
{
    (void)B;
    (void)H;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 4)
#endif
    for (long t = 0; t < nrows; ++t) {
        long r = (long)rows[t];
        long head = r / n;
        row_soft_logits(tq + r * d, tk + head * n * d, n, d, s_out + t * n);
    }
}

typedef struct {
    double s;
    int32_t j;
} keyed_soft_t;

/* Larger logit first; equal logits: lower key index first. */
static int by_soft_logit_then_index(const void *a, const void *b)
{
    const keyed_soft_t *x = (const keyed_soft_t *)a, *y = (const keyed_soft_t *)b;
    if (x->s != y->s)
        return (x->s > y->s) ? -1 : 1;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

static int by_soft_index(const void *a, const void *b)
{
    const keyed_soft_t *x = (const keyed_soft_t *)a, *y = (const keyed_soft_t *)b;
    return (x->j < y->j) ? -1 : (x->j > y->j);
}

/*
 * Soft attention rows: the logits of the soft codes (fp64 dot products),
 * then Eqs. 6-7 exactly as for the binarized codes: the N largest logits
 * (ties to the lower key index) in ascending key order, softmax over them
 * with temperature tau and the value product, both in fp64.  s_out holds
 * the kept logits in fp64.  Returns 0, or -1 on a bad argument or an
 * allocation failure.
 */
int had_oracle_soft_attention_rows(const float *tq, const float *tk,
                                   const void *v, int v_is_bf16, long B,
                                   long H, long n, long d, long N, float tau,
                                   const int64_t *rows, long nrows,
                                   int32_t *idx_out, double *s_out,
                                   double *p_out, float *o_out, int nthreads)
{
    (void)B;
    (void)H;
    if (N < 1 || N > n || d < 1 || n < 1)
        return -1;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)n);
        keyed_soft_t *order = (keyed_soft_t *)malloc(sizeof(keyed_soft_t) * (size_t)n);
        double *e = (double *)malloc(sizeof(double) * (size_t)N);
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 4)
#endif
        for (long t = 0; t < nrows; ++t) {
            if (!s || !order || !e) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                failed = 1;
                continue;
            }
            long r = (long)rows[t];
            long head = r / n;
            row_soft_logits(tq + r * d, tk + head * n * d, n, d, s);
            for (long j = 0; j < n; ++j) {
                order[j].s = s[j];
                order[j].j = (int32_t)j;
            }
            qsort(order, (size_t)n, sizeof(keyed_soft_t), by_soft_logit_then_index);
            qsort(order, (size_t)N, sizeof(keyed_soft_t), by_soft_index);
            double m = order[0].s;
            for (long k = 1; k < N; ++k)
                if (order[k].s > m)
                    m = order[k].s;
            double Z = 0.0;
            for (long k = 0; k < N; ++k) {
                e[k] = exp((double)tau * (order[k].s - m));
                Z += e[k];
            }
            for (long k = 0; k < N; ++k) {
                idx_out[t * N + k] = order[k].j;
                s_out[t * N + k] = order[k].s;
                if (p_out)
                    p_out[t * N + k] = e[k] / Z;
            }
            const long vbase = head * n * d;
            for (long c = 0; c < d; ++c) {
                double acc = 0.0;
                for (long k = 0; k < N; ++k)
                    acc += (e[k] / Z) *
                           (double)load_elem(v, v_is_bf16,
                                             vbase + (long)order[k].j * d + c);
                o_out[t * d + c] = (float)acc;
            }
        }
        free(s);
        free(order);
        free(e);
    }
    return failed ? -1 : 0;
}

/*
 * Eq. 7 on the soft codes for a GIVEN kept set: for each listed row, the
 * fp64 logits of its kept keys idx[t, 0..N-1] (any order, each in [0, n)),
 * then the softmax over exactly those keys (temperature tau, reference the
 * largest of them) and the value product, in fp64.  Lets a kept set chosen
 * elsewhere be scored without the oracle's own selection.  p_out [R, N]
 * (same order as idx) and o_out [R, d].  Returns 0, or -1 on a bad argument
 * or an allocation failure.
 */
int had_oracle_soft_attention_given(const float *tq, const float *tk,
                                    const void *v, int v_is_bf16, long B,
                                    long H, long n, long d, long N, float tau,
                                    const int64_t *rows, long nrows,
                                    const int32_t *idx, double *p_out,
                                    double *o_out)
{
    (void)B;
    (void)H;
    if (N < 1 || d < 1 || n < 1)
        return -1;
    for (long t = 0; t < nrows * N; ++t)
        if (idx[t] < 0 || idx[t] >= n)
            return -1;
    double *s = (double *)malloc(sizeof(double) * (size_t)N);
    double *e = (double *)malloc(sizeof(double) * (size_t)N);
    if (!s || !e) {
        free(s);
        free(e);
        return -1;
    }
    for (long t = 0; t < nrows; ++t) {
        long r = (long)rows[t];
        long head = r / n;
        const float *qr = tq + r * d;
        for (long k = 0; k < N; ++k) {
            const float *kr = tk + (head * n + idx[t * N + k]) * d;
            double acc = 0.0;
            for (long c = 0; c < d; ++c)
                acc += (double)qr[c] * (double)kr[c];
            s[k] = acc;
        }
        double m = s[0];
        for (long k = 1; k < N; ++k)
            if (s[k] > m)
                m = s[k];
        double Z = 0.0;
        for (long k = 0; k < N; ++k) {
            e[k] = exp((double)tau * (s[k] - m));
            Z += e[k];
        }
        for (long k = 0; k < N; ++k)
            p_out[t * N + k] = e[k] / Z;
        const long vbase = head * n * d;
        for (long c = 0; c < d; ++c) {
            double acc = 0.0;
            for (long k = 0; k < N; ++k)
                acc += (e[k] / Z) *
                       (double)load_elem(v, v_is_bf16, vbase + (long)idx[t * N + k] * d + c);
            o_out[t * d + c] = acc;
        }
    }
    free(s);
    free(e);
    return 0;
}

/*
 * Backward pass of the binarized forward for the straight-through training
 * stage (pith.science review of arXiv 2502.01770: after the tanh stages a
 * straight-through estimator finishes the binarization).  Readings taken:
 *   - the forward is steps 1-4 above; the top-N mask is a fixed selection
 *     (no gradient), softmax and value product are differentiated exactly;
 *   - the sign passes the gradient straight through where |z| <= clip and
 *     blocks it elsewhere (z = x / sigma in fp32; clip = 1 is the usual
 *     choice, clip = +inf passes it everywhere); z = x / sigma contributes
 *     1 / sigma; sigma itself is a data statistic and gets no gradient.
 * With dO the gradient of the loss with respect to O, per head and query i
 * over its kept set K_i (p_ij the kept softmax weights):
 *   dV_j  = sum_{i: j in K_i} p_ij dO_i
 *   dp_ij = dO_i . V_j,   D_i = sum_j p_ij dp_ij,   ds_ij = tau p_ij (dp_ij - D_i)
 *   dQb_i = sum_{j in K_i} ds_ij Kb_j,   dKb_j = sum_{i: j in K_i} ds_ij Qb_i
 *   dQ = dQb * [|zq| <= clip] / sigma_q,  dK likewise.
 * All in fp64; every head is processed by one thread in a fixed order.
 * dO is fp32 [B,H,n,d]; dq, dk, dv are fp64 [B,H,n,d].  Returns 0, or -1 on
 * a bad argument or an allocation failure.
 */
int had_oracle_attention_bwd(const void *q, const void *k, const void *v,
                             int is_bf16, const float *sigma_q,
                             const float *sigma_k, const float *dout, long B,
                             long H, long n, long d, long N, float tau,
                             float clip, double *dq, double *dk, double *dv,
                             int nthreads)
{
    if (N < 1 || N > n || d < 1 || n < 1)
        return -1;
    int failed = 0;
#ifdef _OPENMP
    if (nthreads > 0)
        omp_set_num_threads(nthreads);
#pragma omp parallel
#endif
    {
        int8_t *sq = (int8_t *)malloc((size_t)(n * d));
        int8_t *sk = (int8_t *)malloc((size_t)(n * d));
        int32_t *s = (int32_t *)malloc(sizeof(int32_t) * (size_t)n);
        keyed_t *order = (keyed_t *)malloc(sizeof(keyed_t) * (size_t)n);
        double *p = (double *)malloc(sizeof(double) * (size_t)N);
        double *ds = (double *)malloc(sizeof(double) * (size_t)N);
        double *dqb = (double *)malloc(sizeof(double) * (size_t)(n * d));
        double *dkb = (double *)malloc(sizeof(double) * (size_t)(n * d));
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (long head = 0; head < B * H; ++head) {
            if (!sq || !sk || !s || !order || !p || !ds || !dqb || !dkb) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
                failed = 1;
                continue;
            }
            const long h = head % H;
            const long base = head * n * d;
            for (long e = 0; e < n * d; ++e) {
                float zq = load_elem(q, is_bf16, base + e) / sigma_q[h];
                float zk = load_elem(k, is_bf16, base + e) / sigma_k[h];
                sq[e] = (zq < 0.0f) ? (int8_t)-1 : (int8_t)1;
                sk[e] = (zk < 0.0f) ? (int8_t)-1 : (int8_t)1;
                dqb[e] = 0.0;
                dkb[e] = 0.0;
                dv[base + e] = 0.0;
            }
            for (long i = 0; i < n; ++i) {
                /* the forward's kept set and weights */
                row_logits(sq + i * d, sk, n, d, s);
                for (long j = 0; j < n; ++j) {
                    order[j].s = s[j];
                    order[j].j = (int32_t)j;
                }
                qsort(order, (size_t)n, sizeof(keyed_t), by_logit_then_index);
                qsort(order, (size_t)N, sizeof(keyed_t), by_index);
                int32_t m = order[0].s;
                for (long t = 1; t < N; ++t)
                    if (order[t].s > m)
                        m = order[t].s;
                double Z = 0.0;
                for (long t = 0; t < N; ++t) {
                    p[t] = exp((double)tau * (double)(order[t].s - m));
                    Z += p[t];
                }
                for (long t = 0; t < N; ++t)
                    p[t] /= Z;
                /* dp, D and ds */
                const float *go = dout + base + i * d;
                double D = 0.0;
                for (long t = 0; t < N; ++t) {
                    const long vj = base + (long)order[t].j * d;
                    double dp = 0.0;
                    for (long c = 0; c < d; ++c)
                        dp += (double)go[c] * (double)load_elem(v, is_bf16, vj + c);
                    ds[t] = dp;              /* dp for now */
                    D += p[t] * dp;
                }
                for (long t = 0; t < N; ++t)
                    ds[t] = (double)tau * p[t] * (ds[t] - D);
                /* scatter to dV, dKb and gather dQb */
                for (long t = 0; t < N; ++t) {
                    const long j = order[t].j;
                    for (long c = 0; c < d; ++c) {
                        dv[base + j * d + c] += p[t] * (double)go[c];
                        dkb[j * d + c] += ds[t] * (double)sq[i * d + c];
                        dqb[i * d + c] += ds[t] * (double)sk[j * d + c];
                    }
                }
            }
            /* straight-through sign and the 1 / sigma of the standardization */
            for (long e = 0; e < n * d; ++e) {
                float zq = load_elem(q, is_bf16, base + e) / sigma_q[h];
                float zk = load_elem(k, is_bf16, base + e) / sigma_k[h];
                dq[base + e] = (fabsf(zq) <= clip) ? dqb[e] / (double)sigma_q[h] : 0.0;
                dk[base + e] = (fabsf(zk) <= clip) ? dkb[e] / (double)sigma_k[h] : 0.0;
            }
        }
        free(sq);
        free(sk);
        free(s);
        free(order);
        free(p);
        free(ds);
        free(dqb);
        free(dkb);
    }
    return failed ? -1 : 0;
}

int had_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
