/*
 * sla_oracle.c -- plain, slow, fp64 CPU oracle of the SageSLA attention
 * forward (Sparse-Linear Attention with a SageAttention-style INT8 sparse
 * part).  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the CPU
 * baseline leg of the benchmark call it; the product library never does, and
 * it shares no code with the CUDA path.
 *
 * What it computes, per (b, h), in the order the method defines it:
 *
 *  1. Pooled block means of Q and K over the valid tokens of each block
 *     (query blocks of blk_q tokens, key blocks of blk_k tokens; the last block
 *     of a sequence may be partial and uses its own token count).
 *  2. Block importance s_IJ = qbar_I . kbar_J.  The pages keep "the top k% most
 *     important key-value pairs" ("TurboDiffusion技术架构解析", §2.1, SLA
 *     formula) without naming the criterion; the pooled dot product is the
 *     reading taken here.  The dot product is accumulated in channel order
 *     with one fused multiply-add per channel (one rounding per step).
 *  3. Selection: per query block, the first k_sel key blocks in the order
 *     (score descending, block index ascending); k_sel = floor(topk * n_kb +
 *     1e-4) clamped to [0, n_kb]; the selected list is reported ascending.
 *  4. INT8 quantisation (SageAttention style, "清华开源TurboDiffusion加速框架"
 *     section "SageAttention与稀疏计算": FP16 -> INT8 on the tensor cores).
 *     K is smoothed by its per-channel mean over all N tokens; per block
 *     scale = amax / 127 in fp32; code = clamp(rint_even(x / scale), -127,
 *     127), every step in IEEE fp32 so that a GPU can reproduce it exactly.
 *     FP8 variant (quant = 2): no page names FP8 -- that section speaks of
 *     INT8/INT4 only -- so this mode is an addition on the same per-block
 *     scaling, for the e4m3 tensor-core path: scale = amax / 448 and code = the fp8 e4m3 value nearest to x / scale (ties to
 *     even, saturating at +-448; e4m3: 4 exponent bits with bias 7, 3
 *     mantissa bits, subnormals down to 2^-9, no infinities).
 *  5. Sparse branch: for every query row, exact softmax attention
 *     softmax(q k^T / sqrt(d)) v ("TurboDiffusion技术架构解析", §2.1, standard
 *     attention formula) restricted to the tokens of the selected key blocks;
 *     with quantisation on, the logits are (qhat . khat) * s_q * s_k / sqrt(d)
 *     (for FP8 the dot product of the decoded e4m3 values, exact in fp64).
 *  6. Linear branch over the remaining (unselected) key blocks: kernelised
 *     linear attention phi(Q)(phi(K)^T V) ("TurboDiffusion技术架构解析", §2.1,
 *     linear attention formula, phi = elu+1 or ReLU), normalised by
 *     phi(q) . sum phi(k); computed in state form: h_J = phi(K_J)^T V_J,
 *     z_J = sum of phi(K_J) rows, H_I = sum over unselected J of h_J.  A zero
 *     denominator gives a zero output.  phi acts on the raw bf16 Q and K.
 *  7. O = O_sparse + O_linear.
 *
 * Precision: fp64 everywhere except the quantisation step, which is specified
 * in fp32.  Build with -ffp-contract=off and without -ffast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static double bf(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

static float bf32(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void orc_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* k_sel = floor(topk * n_kb + 1e-4), clamped to [0, n_kb]. */
int orc_topk_count(int n_kb, double topk)
{
    double x = floor(topk * (double)n_kb + 1e-4);
    if (x < 0.0) x = 0.0;
    if (x > (double)n_kb) x = (double)n_kb;
    return (int)x;
}

/* mean[J][c] = (sum of x[t][c] over the valid tokens t of block J) / count */
static void pool_head(const uint16_t *x, int N, int d, int blk, double *mean)
{
    int nb = (N + blk - 1) / blk;
    for (int J = 0; J < nb; ++J) {
        int t0 = J * blk, t1 = t0 + blk < N ? t0 + blk : N;
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            for (int t = t0; t < t1; ++t) s += bf(x[(size_t)t * d + c]);
            mean[(size_t)J * d + c] = s / (double)(t1 - t0);
        }
    }
}

void orc_pool(const uint16_t *x, int BH, int N, int d, int blk, double *mean)
{
    int nb = (N + blk - 1) / blk;
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < BH; ++bh)
        pool_head(x + (size_t)bh * N * d, N, d, blk, mean + (size_t)bh * nb * d);
}

typedef struct { double s; int j; } scored;

/* order: score descending, then block index ascending */
static int cmp_scored(const void *a, const void *b)
{
    const scored *x = (const scored *)a, *y = (const scored *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

static int cmp_int(const void *a, const void *b)
{
    int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/* Scores and selection for one head.  idx: [n_qb][k_sel] ascending.
 * scores (nullable): [n_qb][n_kb]. */
static void mask_head(const uint16_t *q, const uint16_t *k, int N, int d, int blk_q, int blk_k,
                      int k_sel, int32_t *idx, uint32_t *bitmap, double *scores)
{
    int n_qb = (N + blk_q - 1) / blk_q, n_kb = (N + blk_k - 1) / blk_k;
    int words = (n_kb + 31) / 32;
    double *qm = (double *)malloc(sizeof(double) * (size_t)n_qb * d);
    double *km = (double *)malloc(sizeof(double) * (size_t)n_kb * d);
    scored *row = (scored *)malloc(sizeof(scored) * (size_t)n_kb);
    int *pick = (int *)malloc(sizeof(int) * (size_t)(n_kb + 1));
    pool_head(q, N, d, blk_q, qm);
    pool_head(k, N, d, blk_k, km);
    for (int I = 0; I < n_qb; ++I) {
        for (int J = 0; J < n_kb; ++J) {
            double s = 0.0;
            for (int c = 0; c < d; ++c) s = fma(qm[(size_t)I * d + c], km[(size_t)J * d + c], s);
            row[J].s = s;
            row[J].j = J;
            if (scores) scores[(size_t)I * n_kb + J] = s;
        }
        qsort(row, (size_t)n_kb, sizeof(scored), cmp_scored);
        for (int r = 0; r < k_sel; ++r) pick[r] = row[r].j;
        qsort(pick, (size_t)k_sel, sizeof(int), cmp_int);
        for (int r = 0; r < k_sel; ++r) idx[(size_t)I * k_sel + r] = pick[r];
        if (bitmap) {
            uint32_t *w = bitmap + (size_t)I * words;
            memset(w, 0, sizeof(uint32_t) * (size_t)words);
            for (int r = 0; r < k_sel; ++r) w[pick[r] >> 5] |= 1u << (pick[r] & 31);
        }
    }
    free(qm); free(km); free(row); free(pick);
}

void orc_block_mask(const uint16_t *q, const uint16_t *k, int BH, int N, int d, int blk_q,
                    int blk_k, double topk, int32_t *idx, uint32_t *bitmap, double *scores)
{
    int n_qb = (N + blk_q - 1) / blk_q, n_kb = (N + blk_k - 1) / blk_k;
    int k_sel = orc_topk_count(n_kb, topk);
    int words = (n_kb + 31) / 32;
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < BH; ++bh)
        mask_head(q + (size_t)bh * N * d, k + (size_t)bh * N * d, N, d, blk_q, blk_k, k_sel,
                  idx + (size_t)bh * n_qb * k_sel, bitmap ? bitmap + (size_t)bh * n_qb * words : NULL,
                  scores ? scores + (size_t)bh * n_qb * n_kb : NULL);
}

/* Symmetric per-block INT8 code of x with scale s (both fp32). */
static int8_t code8(float x, float s)
{
    if (s == 0.0f) return 0;
    float r = rintf(x / s);
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/* The fp8 e4m3 value nearest to x (ties to even, sign kept), saturated to +-448.  The
 * quantum is 2^(e-3) for |x| in [2^e, 2^(e+1)), e >= -6, and 2^-9 below 2^-6. */
float orc_e4m3(float x)
{
    if (isnan(x)) return x;
    double a = fabs((double)x);
    if (a > 448.0) return (float)copysign(448.0, (double)x);
    int E;
    frexp(a, &E);                      /* a = f * 2^E, f in [0.5, 1): floor(log2 a) = E - 1 */
    int qexp = a < ldexp(1.0, -6) ? -9 : (E - 1) - 3;
    double r = nearbyint(ldexp(a, -qexp)); /* a / quantum, rounded half to even */
    double v = ldexp(r, qexp);
    if (v > 448.0) v = 448.0;
    return (float)copysign(v, (double)x); /* the sign survives rounding to zero */
}

/* The e4m3 bit pattern of a value that e4m3 represents exactly (orc_e4m3's output). */
uint8_t orc_e4m3_bits(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a == 0.0) return sign;
    if (a < ldexp(1.0, -6)) return (uint8_t)(sign | (int)ldexp(a, 9)); /* subnormal: m * 2^-9 */
    int E;
    double f = frexp(a, &E);           /* a = (2f) * 2^(E-1), 2f in [1, 2) */
    int e = E - 1 + 7;                 /* biased exponent, 1..15 */
    int m = (int)((2.0 * f - 1.0) * 8.0);
    return (uint8_t)(sign | (e << 3) | m);
}

static double e4m3_value(uint8_t b)
{
    int e = (b >> 3) & 15, m = b & 7;
    double a = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (b & 0x80) ? -a : a;
}

/* orc_e4m3 and orc_e4m3_bits over an array (for the pins). */
void orc_e4m3_array(const float *x, float *value, uint8_t *bits, int64_t n)
{
    for (int64_t i = 0; i < n; ++i) {
        value[i] = orc_e4m3(x[i]);
        bits[i] = orc_e4m3_bits(value[i]);
    }
}

/* Symmetric per-block FP8 code of x with scale s (both fp32): e4m3 bits. */
static uint8_t code_fp8(float x, float s)
{
    if (s == 0.0f) return 0;
    return orc_e4m3_bits(orc_e4m3(x / s));
}

/* Quantise one head.  K is smoothed by its fp32-rounded per-channel mean. */
static void quant_head(const uint16_t *q, const uint16_t *k, int N, int d, int blk_q, int blk_k, int fp8,
                       int8_t *q8, int8_t *k8, float *sq, float *sk, float *kmean)
{
    int n_qb = (N + blk_q - 1) / blk_q, n_kb = (N + blk_k - 1) / blk_k;
    const float qmax = fp8 ? 448.0f : 127.0f;
    float *mu = (float *)malloc(sizeof(float) * (size_t)d);
    for (int c = 0; c < d; ++c) {
        double s = 0.0;
        for (int t = 0; t < N; ++t) s += bf(k[(size_t)t * d + c]);
        mu[c] = (float)(s / (double)N);
        if (kmean) kmean[c] = mu[c];
    }
    for (int I = 0; I < n_qb; ++I) {
        int t0 = I * blk_q, t1 = t0 + blk_q < N ? t0 + blk_q : N;
        float amax = 0.0f;
        for (size_t e = (size_t)t0 * d; e < (size_t)t1 * d; ++e) amax = fmaxf(amax, fabsf(bf32(q[e])));
        float s = amax / qmax;
        sq[I] = s;
        for (size_t e = (size_t)t0 * d; e < (size_t)t1 * d; ++e)
            q8[e] = fp8 ? (int8_t)code_fp8(bf32(q[e]), s) : code8(bf32(q[e]), s);
    }
    for (int J = 0; J < n_kb; ++J) {
        int t0 = J * blk_k, t1 = t0 + blk_k < N ? t0 + blk_k : N;
        float amax = 0.0f;
        for (int t = t0; t < t1; ++t)
            for (int c = 0; c < d; ++c) amax = fmaxf(amax, fabsf(bf32(k[(size_t)t * d + c]) - mu[c]));
        float s = amax / qmax;
        sk[J] = s;
        for (int t = t0; t < t1; ++t)
            for (int c = 0; c < d; ++c) {
                float x = bf32(k[(size_t)t * d + c]) - mu[c];
                k8[(size_t)t * d + c] = fp8 ? (int8_t)code_fp8(x, s) : code8(x, s);
            }
    }
    free(mu);
}

/* fp8 = 0: INT8 codes; fp8 = 1: FP8 e4m3 codes (bit patterns in the int8 arrays). */
void orc_quantize(const uint16_t *q, const uint16_t *k, int BH, int N, int d, int blk_q, int blk_k, int fp8,
                  int8_t *q8, int8_t *k8, float *sq, float *sk, float *kmean)
{
    int n_qb = (N + blk_q - 1) / blk_q, n_kb = (N + blk_k - 1) / blk_k;
#pragma omp parallel for schedule(dynamic)
    for (int bh = 0; bh < BH; ++bh)
        quant_head(q + (size_t)bh * N * d, k + (size_t)bh * N * d, N, d, blk_q, blk_k, fp8,
                   q8 + (size_t)bh * N * d, k8 + (size_t)bh * N * d, sq + (size_t)bh * n_qb,
                   sk + (size_t)bh * n_kb, kmean ? kmean + (size_t)bh * d : NULL);
}

/* phi = elu+1 (0) or ReLU (1) */
static double phi_f(double x, int phi)
{
    if (phi == 1) return x > 0.0 ? x : 0.0;
    return x > 0.0 ? x + 1.0 : exp(x);
}

/* Linear-attention states of one head: h[J][c][e] = sum_t phi(k_tc) v_te,
 * z[J][c] = sum_t phi(k_tc), over the valid tokens t of key block J. */
static void states_head(const uint16_t *k, const uint16_t *v, int N, int d, int blk_k, int phi,
                        double *h, double *z)
{
    int n_kb = (N + blk_k - 1) / blk_k;
    double *pk = (double *)malloc(sizeof(double) * (size_t)d);
    double *vv = (double *)malloc(sizeof(double) * (size_t)d);
    for (int J = 0; J < n_kb; ++J) {
        double *hJ = h + (size_t)J * d * d, *zJ = z + (size_t)J * d;
        memset(hJ, 0, sizeof(double) * (size_t)d * d);
        memset(zJ, 0, sizeof(double) * (size_t)d);
        int t0 = J * blk_k, t1 = t0 + blk_k < N ? t0 + blk_k : N;
        for (int t = t0; t < t1; ++t) {
            for (int c = 0; c < d; ++c) pk[c] = phi_f(bf(k[(size_t)t * d + c]), phi);
            for (int e = 0; e < d; ++e) vv[e] = bf(v[(size_t)t * d + e]);
            for (int c = 0; c < d; ++c) {
                zJ[c] += pk[c];
                for (int e = 0; e < d; ++e) hJ[(size_t)c * d + e] += pk[c] * vv[e];
            }
        }
    }
    free(pk); free(vv);
}

void orc_states(const uint16_t *k, const uint16_t *v, int N, int d, int blk_k, int phi,
                double *h, double *z)
{
    states_head(k, v, N, d, blk_k, phi, h, z);
}

/* H_I = sum of h_J and Z_I = sum of z_J over the key blocks J not selected by
 * query block I (sel: ascending list of k_sel block indices). */
static void unselected_state(const int32_t *sel, int k_sel, int n_kb, int d, const double *h,
                             const double *z, double *HI, double *ZI)
{
    memset(HI, 0, sizeof(double) * (size_t)d * d);
    memset(ZI, 0, sizeof(double) * (size_t)d);
    int r = 0;
    for (int J = 0; J < n_kb; ++J) {
        if (r < k_sel && sel[r] == J) { ++r; continue; }
        const double *hJ = h + (size_t)J * d * d, *zJ = z + (size_t)J * d;
        for (size_t e = 0; e < (size_t)d * d; ++e) HI[e] += hJ[e];
        for (int c = 0; c < d; ++c) ZI[c] += zJ[c];
    }
}

/* One output row i of one head: sparse part os[d], linear part ol[d].
 * sel: the k_sel selected key blocks of i's query block; HI/ZI: its
 * unselected state; work: scratch of k_sel*blk_k + d doubles. */
static void row_out(int i, const uint16_t *q, const uint16_t *k, const uint16_t *v, int N, int d,
                    int blk_q, int blk_k, int k_sel, const int32_t *sel, int phi, int quant,
                    const int8_t *q8, const int8_t *k8, const float *sq, const float *sk,
                    const double *HI, const double *ZI, double *os, double *ol, double *work)
{
    int I = i / blk_q;
    double inv_sqrt_d = 1.0 / sqrt((double)d);
    /* ---- sparse branch: exact softmax over the selected blocks' tokens ---- */
    int nk = 0;
    double mx = -INFINITY;
    for (int r = 0; r < k_sel; ++r) {
        int J = sel[r];
        int t0 = J * blk_k, t1 = t0 + blk_k < N ? t0 + blk_k : N;
        for (int j = t0; j < t1; ++j) {
            double l;
            if (quant == 1) {
                int64_t acc = 0;
                for (int c = 0; c < d; ++c)
                    acc += (int64_t)q8[(size_t)i * d + c] * (int64_t)k8[(size_t)j * d + c];
                l = (double)acc * (double)sq[I] * (double)sk[J] * inv_sqrt_d;
            } else if (quant == 2) {
                double acc = 0.0;
                for (int c = 0; c < d; ++c)
                    acc += e4m3_value((uint8_t)q8[(size_t)i * d + c]) * e4m3_value((uint8_t)k8[(size_t)j * d + c]);
                l = acc * (double)sq[I] * (double)sk[J] * inv_sqrt_d;
            } else {
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += bf(q[(size_t)i * d + c]) * bf(k[(size_t)j * d + c]);
                l = acc * inv_sqrt_d;
            }
            work[nk++] = l;
            if (l > mx) mx = l;
        }
    }
    for (int e = 0; e < d; ++e) os[e] = 0.0;
    if (nk > 0) {
        double den = 0.0;
        int n = 0;
        for (int r = 0; r < k_sel; ++r) {
            int J = sel[r];
            int t0 = J * blk_k, t1 = t0 + blk_k < N ? t0 + blk_k : N;
            for (int j = t0; j < t1; ++j) {
                double p = exp(work[n++] - mx);
                den += p;
                for (int e = 0; e < d; ++e) os[e] += p * bf(v[(size_t)j * d + e]);
            }
        }
        for (int e = 0; e < d; ++e) os[e] /= den;
    }
    /* ---- linear branch: phi(q)^T H_I / (phi(q) . Z_I) ---- */
    double *pq = work + nk;
    for (int c = 0; c < d; ++c) pq[c] = phi_f(bf(q[(size_t)i * d + c]), phi);
    double den = 0.0;
    for (int c = 0; c < d; ++c) den += pq[c] * ZI[c];
    for (int e = 0; e < d; ++e) {
        double num = 0.0;
        for (int c = 0; c < d; ++c) num += pq[c] * HI[(size_t)c * d + e];
        ol[e] = den != 0.0 ? num / den : 0.0;
    }
}

static int cmp_i64(const void *a, const void *b)
{
    int64_t x = *(const int64_t *)a, y = *(const int64_t *)b;
    return (x > y) - (x < y);
}

/*
 * Forward for a list of rows (quant: 0 = none, 1 = INT8, 2 = FP8 e4m3).
 * rows: [nrows][2] pairs (bh, i); when rows is
 * NULL every row of every head is produced in [BH][N] order (nrows ignored).
 * idx_in (nullable, [BH][n_qb][k_sel]) replaces the oracle's own selection.
 * out, out_s, out_l: [nrows][d] (out_s / out_l nullable).  Returns 0, or -1
 * when memory runs out or a row is out of range.
 */
int orc_forward(const uint16_t *q, const uint16_t *k, const uint16_t *v, int BH, int N, int d,
                int blk_q, int blk_k, double topk, int phi, int quant, const int32_t *idx_in,
                const int64_t *rows, int64_t nrows, double *out, double *out_s, double *out_l)
{
    int n_qb = (N + blk_q - 1) / blk_q, n_kb = (N + blk_k - 1) / blk_k;
    int k_sel = orc_topk_count(n_kb, topk);
    if (!rows) nrows = (int64_t)BH * N;
    /* order[] = row numbers sorted by (bh, i); key = bh * N + i */
    int64_t *key = (int64_t *)malloc(sizeof(int64_t) * 2 * (size_t)(nrows + 1));
    if (!key) return -1;
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t bh = rows ? rows[2 * r] : r / N, i = rows ? rows[2 * r + 1] : r % N;
        if (bh < 0 || bh >= BH || i < 0 || i >= N) { free(key); return -1; }
        key[2 * r] = bh * (int64_t)N + i;
        key[2 * r + 1] = r;
    }
    qsort(key, (size_t)nrows, 2 * sizeof(int64_t), cmp_i64);

    size_t hd = (size_t)N * d;
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * ((size_t)n_qb * k_sel + 1));
    int8_t *q8 = quant ? (int8_t *)malloc(hd) : NULL;
    int8_t *k8 = quant ? (int8_t *)malloc(hd) : NULL;
    float *sq = (float *)malloc(sizeof(float) * (size_t)n_qb);
    float *sk = (float *)malloc(sizeof(float) * (size_t)n_kb);
    double *h = (double *)malloc(sizeof(double) * (size_t)n_kb * d * d);
    double *z = (double *)malloc(sizeof(double) * (size_t)n_kb * d);
    int64_t *gstart = (int64_t *)malloc(sizeof(int64_t) * (size_t)(nrows + 1));
    if (!idx || (quant && (!q8 || !k8)) || !sq || !sk || !h || !z || !gstart) return -1;

    int64_t pos = 0;
    while (pos < nrows) {
        int bh = (int)(key[2 * pos] / N);
        int64_t end = pos;
        while (end < nrows && key[2 * end] / N == bh) ++end;
        const uint16_t *qh = q + bh * hd, *kh = k + bh * hd, *vh = v + bh * hd;
        if (idx_in)
            memcpy(idx, idx_in + (size_t)bh * n_qb * k_sel, sizeof(int32_t) * (size_t)n_qb * k_sel);
        else
            mask_head(qh, kh, N, d, blk_q, blk_k, k_sel, idx, NULL, NULL);
        if (quant) quant_head(qh, kh, N, d, blk_q, blk_k, quant == 2, q8, k8, sq, sk, NULL);
#pragma omp parallel for schedule(dynamic)
        for (int J = 0; J < n_kb; ++J) {
            int t0 = J * blk_k;
            int len = t0 + blk_k < N ? blk_k : N - t0;
            states_head(kh + (size_t)t0 * d, vh + (size_t)t0 * d, len, d, blk_k, phi,
                        h + (size_t)J * d * d, z + (size_t)J * d);
        }
        /* groups of rows that share a query block */
        int64_t ng = 0;
        for (int64_t r = pos; r < end; ++r)
            if (r == pos || (key[2 * r] % N) / blk_q != (key[2 * r - 2] % N) / blk_q) gstart[ng++] = r;
        gstart[ng] = end;
#pragma omp parallel
        {
            size_t wn = (size_t)k_sel * blk_k + (size_t)d + 16;
            double *work = (double *)malloc(sizeof(double) * wn);
            double *HI = (double *)malloc(sizeof(double) * (size_t)d * d);
            double *ZI = (double *)malloc(sizeof(double) * (size_t)d);
            double *os = (double *)malloc(sizeof(double) * (size_t)d);
            double *ol = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic)
            for (int64_t g = 0; g < ng; ++g) {
                int I = (int)((key[2 * gstart[g]] % N) / blk_q);
                const int32_t *sel = idx + (size_t)I * k_sel;
                unselected_state(sel, k_sel, n_kb, d, h, z, HI, ZI);
                for (int64_t r = gstart[g]; r < gstart[g + 1]; ++r) {
                    int i = (int)(key[2 * r] % N);
                    int64_t o = key[2 * r + 1];
                    row_out(i, qh, kh, vh, N, d, blk_q, blk_k, k_sel, sel, phi, quant, q8, k8, sq,
                            sk, HI, ZI, os, ol, work);
                    for (int e = 0; e < d; ++e) {
                        out[(size_t)o * d + e] = os[e] + ol[e];
                        if (out_s) out_s[(size_t)o * d + e] = os[e];
                        if (out_l) out_l[(size_t)o * d + e] = ol[e];
                    }
                }
            }
            free(work); free(HI); free(ZI); free(os); free(ol);
        }
        pos = end;
    }
    free(key); free(gstart); free(idx); free(q8); free(k8); free(sq); free(sk); free(h); free(z);
    return 0;
}

/* ------------------------------------------------------------------------
 * Backward: gradients of the unquantised forward (steps 1-3, 5-7 with
 * quant = 0) with respect to q, k and v, for SLA fine-tuning
 * (the jiqiren.org.cn TurboDiffusion article, 方法论: full attention is
 * replaced by SLA and the pretrained model is fine-tuned for the sparsity; the
 * "TurboDiffusion" summary page, 主要能力: SLA white-box training).  The block selection is a
 * piecewise-constant function of (q, k), so it is held fixed; everything else
 * is differentiated exactly (chain rule, fp64).  With do = dL/dO:
 *
 *  sparse branch, row i, selected tokens j, s_ij = q_i.k_j / sqrt(d),
 *  p_ij = softmax_j(s_ij), os_i = sum_j p_ij v_j:
 *    dv_j += p_ij do_i;  dp_ij = do_i.v_j;  D_i = do_i.os_i;
 *    ds_ij = p_ij (dp_ij - D_i);
 *    dq_i += ds_ij k_j / sqrt(d);  dk_j += ds_ij q_i / sqrt(d).
 *  linear branch, row i of query block I, f = phi(q_i), a = f H_I, b = f.Z_I,
 *  ol_i = a / b (a zero b gives a zero output and no gradient):
 *    da = do_i / b;  db = -(do_i.ol_i) / b;
 *    dq_i += (H_I da + Z_I db) * phi'(q_i);
 *    dH_I += f (outer) da;  dZ_I += f db.
 *  key side, per key block J: G_J = sum of dH_I and g_J = sum of dZ_I over the
 *  query blocks I that did not select J; for each token j of J:
 *    dk_j += (G_J v_j + g_J) * phi'(k_j);  dv_j += G_J^T phi(k_j).
 * phi'(x) = 1 for x > 0, else exp(x) (elu+1) or 0 (ReLU).
 * ------------------------------------------------------------------------ */
static double dphi_f(double x, int phi)
{
    if (phi == 1) return x > 0.0 ? 1.0 : 0.0;
    return x > 0.0 ? 1.0 : exp(x);
}

static int backward_head(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout, int N,
                         int d, int blk_q, int blk_k, int k_sel, const int32_t *idx, int phi, double *dq,
                         double *dk, double *dv)
{
    int n_qb = (N + blk_q - 1) / blk_q, n_kb = (N + blk_k - 1) / blk_k;
    const double rsd = 1.0 / sqrt((double)d); /* softmax scale 1/sqrt(d) */
    size_t dd = (size_t)d * d;
    double *h = (double *)malloc(sizeof(double) * (size_t)n_kb * dd);
    double *z = (double *)malloc(sizeof(double) * (size_t)n_kb * d);
    double *dH = (double *)calloc((size_t)n_qb * dd, sizeof(double));
    double *dZ = (double *)calloc((size_t)n_qb * d, sizeof(double));
    double *HI = (double *)malloc(sizeof(double) * dd);
    double *ZI = (double *)malloc(sizeof(double) * (size_t)d);
    double *G = (double *)malloc(sizeof(double) * dd);
    double *gz = (double *)malloc(sizeof(double) * (size_t)d);
    double *p = (double *)malloc(sizeof(double) * ((size_t)k_sel * blk_k + 1));
    double *vec = (double *)malloc(sizeof(double) * 8 * (size_t)d);
    unsigned char *selected = (unsigned char *)calloc((size_t)n_qb * n_kb + 1, 1);
    if (!h || !z || !dH || !dZ || !HI || !ZI || !G || !gz || !p || !vec || !selected) {
        free(h); free(z); free(dH); free(dZ); free(HI); free(ZI); free(G); free(gz); free(p); free(vec);
        free(selected);
        return -1;
    }
    double *qi = vec, *doi = vec + d, *os = vec + 2 * d, *f = vec + 3 * d, *a = vec + 4 * d, *ol = vec + 5 * d,
           *da = vec + 6 * d, *w = vec + 7 * d;
    states_head(k, v, N, d, blk_k, phi, h, z);
    for (int I = 0; I < n_qb; ++I)
        for (int r = 0; r < k_sel; ++r) selected[(size_t)I * n_kb + idx[(size_t)I * k_sel + r]] = 1;
    memset(dq, 0, sizeof(double) * (size_t)N * d);
    memset(dk, 0, sizeof(double) * (size_t)N * d);
    memset(dv, 0, sizeof(double) * (size_t)N * d);

    for (int I = 0; I < n_qb; ++I) {
        const int32_t *sel = idx + (size_t)I * k_sel;
        unselected_state(sel, k_sel, n_kb, d, h, z, HI, ZI);
        double *dHI = dH + (size_t)I * dd, *dZI = dZ + (size_t)I * d;
        int i1 = (I + 1) * blk_q < N ? (I + 1) * blk_q : N;
        for (int i = I * blk_q; i < i1; ++i) {
            for (int c = 0; c < d; ++c) {
                qi[c] = bf(q[(size_t)i * d + c]);
                doi[c] = bf(dout[(size_t)i * d + c]);
            }
            /* ---- sparse branch: recompute p and os, then the softmax gradient ---- */
            int nk = 0;
            double mx = -INFINITY;
            for (int r = 0; r < k_sel; ++r) {
                int J = sel[r], t0 = J * blk_k, t1 = t0 + blk_k < N ? t0 + blk_k : N;
                for (int j = t0; j < t1; ++j) {
                    double s = 0.0;
                    for (int c = 0; c < d; ++c) s += qi[c] * bf(k[(size_t)j * d + c]);
                    p[nk] = s * rsd;
                    if (p[nk] > mx) mx = p[nk];
                    ++nk;
                }
            }
            if (nk > 0) {
                double den = 0.0;
                for (int n = 0; n < nk; ++n) {
                    p[n] = exp(p[n] - mx);
                    den += p[n];
                }
                for (int n = 0; n < nk; ++n) p[n] /= den;
                for (int e = 0; e < d; ++e) os[e] = 0.0;
                int n = 0;
                for (int r = 0; r < k_sel; ++r) {
                    int J = sel[r], t0 = J * blk_k, t1 = t0 + blk_k < N ? t0 + blk_k : N;
                    for (int j = t0; j < t1; ++j, ++n)
                        for (int e = 0; e < d; ++e) os[e] += p[n] * bf(v[(size_t)j * d + e]);
                }
                double D = 0.0;
                for (int e = 0; e < d; ++e) D += doi[e] * os[e];
                n = 0;
                for (int r = 0; r < k_sel; ++r) {
                    int J = sel[r], t0 = J * blk_k, t1 = t0 + blk_k < N ? t0 + blk_k : N;
                    for (int j = t0; j < t1; ++j, ++n) {
                        double dp = 0.0;
                        for (int e = 0; e < d; ++e) dp += doi[e] * bf(v[(size_t)j * d + e]);
                        double ds = p[n] * (dp - D);
                        for (int c = 0; c < d; ++c) {
                            dq[(size_t)i * d + c] += ds * bf(k[(size_t)j * d + c]) * rsd;
                            dk[(size_t)j * d + c] += ds * qi[c] * rsd;
                            dv[(size_t)j * d + c] += p[n] * doi[c];
                        }
                    }
                }
            }
            /* ---- linear branch ---- */
            double b = 0.0;
            for (int c = 0; c < d; ++c) {
                f[c] = phi_f(qi[c], phi);
                b += f[c] * ZI[c];
            }
            if (b == 0.0) continue;
            for (int e = 0; e < d; ++e) {
                a[e] = 0.0;
                for (int c = 0; c < d; ++c) a[e] += f[c] * HI[(size_t)c * d + e];
                ol[e] = a[e] / b;
            }
            double dol = 0.0;
            for (int e = 0; e < d; ++e) dol += doi[e] * ol[e];
            double db = -dol / b;
            for (int e = 0; e < d; ++e) da[e] = doi[e] / b;
            for (int c = 0; c < d; ++c) {
                double df = ZI[c] * db;
                for (int e = 0; e < d; ++e) df += HI[(size_t)c * d + e] * da[e];
                dq[(size_t)i * d + c] += df * dphi_f(qi[c], phi);
                for (int e = 0; e < d; ++e) dHI[(size_t)c * d + e] += f[c] * da[e];
                dZI[c] += f[c] * db;
            }
        }
    }
    /* ---- key side of the linear branch ---- */
    for (int J = 0; J < n_kb; ++J) {
        memset(G, 0, sizeof(double) * dd);
        memset(gz, 0, sizeof(double) * (size_t)d);
        for (int I = 0; I < n_qb; ++I) {
            if (selected[(size_t)I * n_kb + J]) continue;
            for (size_t e = 0; e < dd; ++e) G[e] += dH[(size_t)I * dd + e];
            for (int c = 0; c < d; ++c) gz[c] += dZ[(size_t)I * d + c];
        }
        int t0 = J * blk_k, t1 = t0 + blk_k < N ? t0 + blk_k : N;
        for (int j = t0; j < t1; ++j) {
            for (int e = 0; e < d; ++e) w[e] = bf(v[(size_t)j * d + e]);
            for (int c = 0; c < d; ++c) {
                double kc = bf(k[(size_t)j * d + c]), fk = phi_f(kc, phi);
                double dfk = gz[c];
                for (int e = 0; e < d; ++e) {
                    dfk += G[(size_t)c * d + e] * w[e];
                    dv[(size_t)j * d + e] += G[(size_t)c * d + e] * fk;
                }
                dk[(size_t)j * d + c] += dfk * dphi_f(kc, phi);
            }
        }
    }
    free(h); free(z); free(dH); free(dZ); free(HI); free(ZI); free(G); free(gz); free(p); free(vec); free(selected);
    return 0;
}

/* Gradients of every head ([BH][N][d] bf16 q, k, v, dout -> fp64 dq, dk, dv).
 * idx_in (nullable, [BH][n_qb][k_sel]) replaces the oracle's own selection.
 * Returns 0, or -1 when memory runs out. */
int orc_backward(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout, int BH, int N,
                 int d, int blk_q, int blk_k, double topk, int phi, const int32_t *idx_in, double *dq, double *dk,
                 double *dv)
{
    int n_qb = (N + blk_q - 1) / blk_q, n_kb = (N + blk_k - 1) / blk_k;
    int k_sel = orc_topk_count(n_kb, topk);
    int fail = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : fail)
    for (int bh = 0; bh < BH; ++bh) {
        size_t hd = (size_t)N * d;
        int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * ((size_t)n_qb * k_sel + 1));
        if (!idx) { fail |= 1; continue; }
        if (idx_in)
            memcpy(idx, idx_in + (size_t)bh * n_qb * k_sel, sizeof(int32_t) * (size_t)n_qb * k_sel);
        else
            mask_head(q + bh * hd, k + bh * hd, N, d, blk_q, blk_k, k_sel, idx, NULL, NULL);
        if (backward_head(q + bh * hd, k + bh * hd, v + bh * hd, dout + bh * hd, N, d, blk_q, blk_k, k_sel, idx,
                          phi, dq + bh * hd, dk + bh * hd, dv + bh * hd))
            fail |= 1;
        free(idx);
    }
    return fail ? -1 : 0;
}

/* dq of a list of rows only (rows: [nrows][2] pairs (bh, i); dq_out [nrows][d]):
 * the same steps as the backward's dq, which needs only row i, its selected
 * blocks and its query block's unselected state, so that it can be evaluated
 * at sizes where the full backward is too slow.  idx_in as in orc_backward.
 * Returns 0, or -1 when memory runs out or a row is out of range. */
int orc_backward_dq_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout, int BH,
                         int N, int d, int blk_q, int blk_k, double topk, int phi, const int32_t *idx_in,
                         const int64_t *rows, int64_t nrows, double *dq_out)
{
    int n_qb = (N + blk_q - 1) / blk_q, n_kb = (N + blk_k - 1) / blk_k;
    int k_sel = orc_topk_count(n_kb, topk);
    const double rsd_ = 1.0 / sqrt((double)d);
    size_t hd = (size_t)N * d, dd = (size_t)d * d;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[2 * r] < 0 || rows[2 * r] >= BH || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= N) return -1;
    int fail = 0;
#pragma omp parallel for schedule(dynamic) reduction(| : fail)
    for (int bh = 0; bh < BH; ++bh) {
        int any = 0;
        for (int64_t r = 0; r < nrows; ++r) any |= rows[2 * r] == bh;
        if (!any) continue;
        const uint16_t *qh = q + bh * hd, *kh = k + bh * hd, *vh = v + bh * hd, *dh = dout + bh * hd;
        int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * ((size_t)n_qb * k_sel + 1));
        double *h = (double *)malloc(sizeof(double) * (size_t)n_kb * dd);
        double *z = (double *)malloc(sizeof(double) * (size_t)n_kb * d);
        double *HI = (double *)malloc(sizeof(double) * dd);
        double *ZI = (double *)malloc(sizeof(double) * (size_t)d);
        double *p = (double *)malloc(sizeof(double) * ((size_t)k_sel * blk_k + 1));
        double *vec = (double *)malloc(sizeof(double) * 8 * (size_t)d);
        if (!idx || !h || !z || !HI || !ZI || !p || !vec) {
            free(idx); free(h); free(z); free(HI); free(ZI); free(p); free(vec);
            fail |= 1;
            continue;
        }
        if (idx_in)
            memcpy(idx, idx_in + (size_t)bh * n_qb * k_sel, sizeof(int32_t) * (size_t)n_qb * k_sel);
        else
            mask_head(qh, kh, N, d, blk_q, blk_k, k_sel, idx, NULL, NULL);
        states_head(kh, vh, N, d, blk_k, phi, h, z);
        double *qi = vec, *doi = vec + d, *os = vec + 2 * d, *f = vec + 3 * d, *a = vec + 4 * d, *da = vec + 6 * d;
        for (int64_t r = 0; r < nrows; ++r) {
            if (rows[2 * r] != bh) continue;
            int i = (int)rows[2 * r + 1], I = i / blk_q;
            const int32_t *sel = idx + (size_t)I * k_sel;
            double *out = dq_out + (size_t)r * d;
            for (int c = 0; c < d; ++c) {
                qi[c] = bf(qh[(size_t)i * d + c]);
                doi[c] = bf(dh[(size_t)i * d + c]);
                out[c] = 0.0;
            }
            /* sparse branch */
            int nk = 0;
            double mx = -INFINITY;
            for (int s_ = 0; s_ < k_sel; ++s_) {
                int J = sel[s_], t0 = J * blk_k, t1 = t0 + blk_k < N ? t0 + blk_k : N;
                for (int j = t0; j < t1; ++j) {
                    double s = 0.0;
                    for (int c = 0; c < d; ++c) s += qi[c] * bf(kh[(size_t)j * d + c]);
                    p[nk] = s * rsd_;
                    if (p[nk] > mx) mx = p[nk];
                    ++nk;
                }
            }
            if (nk > 0) {
                double den = 0.0;
                for (int n = 0; n < nk; ++n) {
                    p[n] = exp(p[n] - mx);
                    den += p[n];
                }
                for (int n = 0; n < nk; ++n) p[n] /= den;
                for (int e = 0; e < d; ++e) os[e] = 0.0;
                int n = 0;
                for (int s_ = 0; s_ < k_sel; ++s_) {
                    int J = sel[s_], t0 = J * blk_k, t1 = t0 + blk_k < N ? t0 + blk_k : N;
                    for (int j = t0; j < t1; ++j, ++n)
                        for (int e = 0; e < d; ++e) os[e] += p[n] * bf(vh[(size_t)j * d + e]);
                }
                double D = 0.0;
                for (int e = 0; e < d; ++e) D += doi[e] * os[e];
                n = 0;
                for (int s_ = 0; s_ < k_sel; ++s_) {
                    int J = sel[s_], t0 = J * blk_k, t1 = t0 + blk_k < N ? t0 + blk_k : N;
                    for (int j = t0; j < t1; ++j, ++n) {
                        double dp = 0.0;
                        for (int e = 0; e < d; ++e) dp += doi[e] * bf(vh[(size_t)j * d + e]);
                        double ds = (dp - D) * p[n]; /* same product as the full backward */
                        for (int c = 0; c < d; ++c) out[c] += ds * bf(kh[(size_t)j * d + c]) * rsd_;
                    }
                }
            }
            /* linear branch */
            unselected_state(sel, k_sel, n_kb, d, h, z, HI, ZI);
            double b = 0.0;
            for (int c = 0; c < d; ++c) {
                f[c] = phi_f(qi[c], phi);
                b += f[c] * ZI[c];
            }
            if (b == 0.0) continue;
            double dol = 0.0;
            for (int e = 0; e < d; ++e) {
                a[e] = 0.0;
                for (int c = 0; c < d; ++c) a[e] += f[c] * HI[(size_t)c * d + e];
                dol += doi[e] * (a[e] / b);
                da[e] = doi[e] / b;
            }
            double db = -(dol / b);
            for (int c = 0; c < d; ++c) {
                double df = ZI[c] * db;
                for (int e = 0; e < d; ++e) df += HI[(size_t)c * d + e] * da[e];
                out[c] += df * dphi_f(qi[c], phi);
            }
        }
        free(idx); free(h); free(z); free(HI); free(ZI); free(p); free(vec);
    }
    return fail ? -1 : 0;
}

/* dk and dv of a list of key blocks only (blocks: [nblk][2] pairs (bh, J);
 * dk_out, dv_out: [nblk][blk_k][d], rows past N left zero): the same steps,
 * in the same order, as the full backward restricted to those key blocks, so
 * that they can be evaluated at sizes where the full backward is too slow.
 * A key block's gradient needs (a) the linear branch's state gradients dH_I,
 * dZ_I of every query block that did not select it, and (b) for every row of
 * every query block that did select it, the row's softmax over all its
 * selected tokens and D = do.os.  Each contribution is added to dk, dv in the
 * order the full backward adds it (query blocks ascending, rows ascending,
 * then the linear key side), so the results equal orc_backward's rows bit for
 * bit.  idx_in as in orc_backward.  Returns 0, or -1 when memory runs out or a
 * block is out of range. */
int orc_backward_dkdv_blocks(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                             int BH, int N, int d, int blk_q, int blk_k, double topk, int phi,
                             const int32_t *idx_in, const int64_t *blocks, int64_t nblk, double *dk_out,
                             double *dv_out)
{
    int n_qb = (N + blk_q - 1) / blk_q, n_kb = (N + blk_k - 1) / blk_k;
    int k_sel = orc_topk_count(n_kb, topk);
    const double rsd = 1.0 / sqrt((double)d);
    size_t hd = (size_t)N * d, dd = (size_t)d * d;
    for (int64_t b = 0; b < nblk; ++b)
        if (blocks[2 * b] < 0 || blocks[2 * b] >= BH || blocks[2 * b + 1] < 0 || blocks[2 * b + 1] >= n_kb) return -1;
    memset(dk_out, 0, sizeof(double) * (size_t)nblk * blk_k * d);
    memset(dv_out, 0, sizeof(double) * (size_t)nblk * blk_k * d);
    int fail = 0;
    for (int bh = 0; bh < BH && !fail; ++bh) {
        int any = 0;
        for (int64_t b = 0; b < nblk; ++b) any |= blocks[2 * b] == bh;
        if (!any) continue;
        const uint16_t *qh = q + bh * hd, *kh = k + bh * hd, *vh = v + bh * hd, *dh = dout + bh * hd;
        int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * ((size_t)n_qb * k_sel + 1));
        double *h = (double *)malloc(sizeof(double) * (size_t)n_kb * dd);
        double *z = (double *)malloc(sizeof(double) * (size_t)n_kb * d);
        double *dH = (double *)calloc((size_t)n_qb * dd, sizeof(double));
        double *dZ = (double *)calloc((size_t)n_qb * d, sizeof(double));
        double *G = (double *)malloc(sizeof(double) * dd);
        double *gz = (double *)malloc(sizeof(double) * (size_t)d);
        unsigned char *selected = (unsigned char *)calloc((size_t)n_qb * n_kb + 1, 1);
        /* per selecting row: p_ij and ds_ij of the block's keys (blk_k each) */
        double *pr = (double *)malloc(sizeof(double) * ((size_t)n_qb * blk_q * blk_k + 1));
        double *dsr = (double *)malloc(sizeof(double) * ((size_t)n_qb * blk_q * blk_k + 1));
        if (!idx || !h || !z || !dH || !dZ || !G || !gz || !selected || !pr || !dsr) {
            free(idx); free(h); free(z); free(dH); free(dZ); free(G); free(gz); free(selected); free(pr); free(dsr);
            fail = 1;
            break;
        }
        if (idx_in)
            memcpy(idx, idx_in + (size_t)bh * n_qb * k_sel, sizeof(int32_t) * (size_t)n_qb * k_sel);
        else
            mask_head(qh, kh, N, d, blk_q, blk_k, k_sel, idx, NULL, NULL);
        states_head(kh, vh, N, d, blk_k, phi, h, z);
        for (int I = 0; I < n_qb; ++I)
            for (int r = 0; r < k_sel; ++r) selected[(size_t)I * n_kb + idx[(size_t)I * k_sel + r]] = 1;
        /* (a) the linear branch's state gradients of every query block, as in the full backward */
#pragma omp parallel
        {
            double *HI = (double *)malloc(sizeof(double) * dd);
            double *ZI = (double *)malloc(sizeof(double) * (size_t)d);
            double *vec = (double *)malloc(sizeof(double) * 8 * (size_t)d);
#pragma omp for schedule(dynamic)
            for (int I = 0; I < n_qb; ++I) {
                if (!HI || !ZI || !vec) continue;
                unselected_state(idx + (size_t)I * k_sel, k_sel, n_kb, d, h, z, HI, ZI);
                double *dH_I = dH + (size_t)I * dd, *dZ_I = dZ + (size_t)I * d;
                double *qi = vec, *doi = vec + d, *f = vec + 3 * d, *a = vec + 4 * d, *ol = vec + 5 * d,
                       *da = vec + 6 * d;
                int i1 = (I + 1) * blk_q < N ? (I + 1) * blk_q : N;
                for (int i = I * blk_q; i < i1; ++i) {
                    for (int c = 0; c < d; ++c) {
                        qi[c] = bf(qh[(size_t)i * d + c]);
                        doi[c] = bf(dh[(size_t)i * d + c]);
                    }
                    double b = 0.0;
                    for (int c = 0; c < d; ++c) {
                        f[c] = phi_f(qi[c], phi);
                        b += f[c] * ZI[c];
                    }
                    if (b == 0.0) continue;
                    for (int e = 0; e < d; ++e) {
                        a[e] = 0.0;
                        for (int c = 0; c < d; ++c) a[e] += f[c] * HI[(size_t)c * d + e];
                        ol[e] = a[e] / b;
                    }
                    double dol = 0.0;
                    for (int e = 0; e < d; ++e) dol += doi[e] * ol[e];
                    double g_b = -dol / b;
                    for (int e = 0; e < d; ++e) da[e] = doi[e] / b;
                    for (int c = 0; c < d; ++c) {
                        for (int e = 0; e < d; ++e) dH_I[(size_t)c * d + e] += f[c] * da[e];
                        dZ_I[c] += f[c] * g_b;
                    }
                }
            }
            free(HI); free(ZI); free(vec);
        }
        for (int64_t bb = 0; bb < nblk; ++bb) {
            if (blocks[2 * bb] != bh) continue;
            int J = (int)blocks[2 * bb + 1], t0 = J * blk_k, t1 = t0 + blk_k < N ? t0 + blk_k : N;
            double *dkb = dk_out + (size_t)bb * blk_k * d, *dvb = dv_out + (size_t)bb * blk_k * d;
            /* (b) the softmax branch: every row of every query block that selected J, p and ds of
             * J's keys (rows evaluated in parallel, added in order below) */
#pragma omp parallel
            {
                double *p = (double *)malloc(sizeof(double) * ((size_t)k_sel * blk_k + 1));
                double *vec = (double *)malloc(sizeof(double) * 3 * (size_t)d);
#pragma omp for schedule(dynamic)
                for (int I = 0; I < n_qb; ++I) {
                    if (!p || !vec || !selected[(size_t)I * n_kb + J]) continue;
                    const int32_t *sel = idx + (size_t)I * k_sel;
                    double *qi = vec, *doi = vec + d, *os = vec + 2 * d;
                    int i1 = (I + 1) * blk_q < N ? (I + 1) * blk_q : N;
                    for (int i = I * blk_q; i < i1; ++i) {
                        for (int c = 0; c < d; ++c) {
                            qi[c] = bf(qh[(size_t)i * d + c]);
                            doi[c] = bf(dh[(size_t)i * d + c]);
                        }
                        int nk = 0, at = -1;
                        double mx = -INFINITY;
                        for (int r = 0; r < k_sel; ++r) {
                            int Jr = sel[r], u0 = Jr * blk_k, u1 = u0 + blk_k < N ? u0 + blk_k : N;
                            if (Jr == J) at = nk;
                            for (int j = u0; j < u1; ++j) {
                                double sc = 0.0;
                                for (int c = 0; c < d; ++c) sc += qi[c] * bf(kh[(size_t)j * d + c]);
                                p[nk] = sc * rsd;
                                if (p[nk] > mx) mx = p[nk];
                                ++nk;
                            }
                        }
                        double den = 0.0;
                        for (int n = 0; n < nk; ++n) {
                            p[n] = exp(p[n] - mx);
                            den += p[n];
                        }
                        for (int n = 0; n < nk; ++n) p[n] /= den;
                        for (int e = 0; e < d; ++e) os[e] = 0.0;
                        int n = 0;
                        for (int r = 0; r < k_sel; ++r) {
                            int Jr = sel[r], u0 = Jr * blk_k, u1 = u0 + blk_k < N ? u0 + blk_k : N;
                            for (int j = u0; j < u1; ++j, ++n)
                                for (int e = 0; e < d; ++e) os[e] += p[n] * bf(vh[(size_t)j * d + e]);
                        }
                        double D = 0.0;
                        for (int e = 0; e < d; ++e) D += doi[e] * os[e];
                        double *prow = pr + ((size_t)I * blk_q + (i - I * blk_q)) * blk_k;
                        double *dsrow = dsr + ((size_t)I * blk_q + (i - I * blk_q)) * blk_k;
                        for (int j = t0; j < t1; ++j) {
                            double dp = 0.0;
                            for (int e = 0; e < d; ++e) dp += doi[e] * bf(vh[(size_t)j * d + e]);
                            prow[j - t0] = p[at + (j - t0)];
                            dsrow[j - t0] = p[at + (j - t0)] * (dp - D);
                        }
                    }
                }
                free(p); free(vec);
            }
            for (int I = 0; I < n_qb; ++I) {
                if (!selected[(size_t)I * n_kb + J]) continue;
                int i1 = (I + 1) * blk_q < N ? (I + 1) * blk_q : N;
                for (int i = I * blk_q; i < i1; ++i) {
                    const double *prow = pr + ((size_t)I * blk_q + (i - I * blk_q)) * blk_k;
                    const double *dsrow = dsr + ((size_t)I * blk_q + (i - I * blk_q)) * blk_k;
                    for (int j = t0; j < t1; ++j)
                        for (int c = 0; c < d; ++c) {
                            dkb[(size_t)(j - t0) * d + c] += dsrow[j - t0] * bf(qh[(size_t)i * d + c]) * rsd;
                            dvb[(size_t)(j - t0) * d + c] += prow[j - t0] * bf(dh[(size_t)i * d + c]);
                        }
                }
            }
            /* the linear key side */
            memset(G, 0, sizeof(double) * dd);
            memset(gz, 0, sizeof(double) * (size_t)d);
            for (int I = 0; I < n_qb; ++I) {
                if (selected[(size_t)I * n_kb + J] != 0) continue;
                for (size_t e = 0; e < dd; ++e) G[e] += dH[(size_t)I * dd + e];
                for (int c = 0; c < d; ++c) gz[c] += dZ[(size_t)I * d + c];
            }
            for (int j = t0; j < t1; ++j) {
                for (int c = 0; c < d; ++c) {
                    double kc = bf(kh[(size_t)j * d + c]), fk = phi_f(kc, phi);
                    double dkf = gz[c];
                    for (int e = 0; e < d; ++e) {
                        dkf += G[(size_t)c * d + e] * bf(vh[(size_t)j * d + e]);
                        dvb[(size_t)(j - t0) * d + e] += G[(size_t)c * d + e] * fk;
                    }
                    dkb[(size_t)(j - t0) * d + c] += dkf * dphi_f(kc, phi);
                }
            }
        }
        free(idx); free(h); free(z); free(dH); free(dZ); free(G); free(gz); free(selected); free(pr); free(dsr);
    }
    return fail ? -1 : 0;
}

/* ------------------------------------------------------------------------
 * W8A8 INT8 linear layer with FusedNorm ("清华开源TurboDiffusion加速框架",
 * W8A8 INT8量化: the weights and activations of the linear layers quantised
 * to 8-bit integers for the INT8 units; the jiqiren.org.cn TurboDiffusion
 * article, 方法论 item 4: W8A8 accelerates the linear layers; "TurboDiffusion：
 * 让可视化视频生成效率提升200倍的加速引擎" §1: W8A8 together with a FusedNorm
 * operator).  Granularity, rounding and the norm are not stated; the readings:
 *   - activations: one symmetric scale per token (row), weights: one per
 *     output channel (row of W [N, K]); scale = amax / 127 and code =
 *     clamp(rint_even(y / scale), +-127) in IEEE fp32, the SageSLA rule;
 *   - FusedNorm: the row's RMS normalisation fused into its quantisation:
 *     ms = (fp64 sum of x^2) / cols rounded to fp32, r = 1 / sqrt(ms + eps)
 *     (IEEE fp32 add, sqrt and divide), y = fp32(x * r) * gamma[c] (two fp32
 *     products; gamma nullable = 1);
 *   - out[m][n] = (sum_k qx[m][k] qw[n][k]) * sx[m] * sw[n] (+ bias[n]),
 *     exact integer sum, the rest in fp64.
 * ------------------------------------------------------------------------ */
void orc_rowquant(const uint16_t *x, int rows, int cols, int norm, const float *gamma, float eps, int8_t *q,
                  float *s)
{
#pragma omp parallel for schedule(static)
    for (int m = 0; m < rows; ++m) {
        const uint16_t *xr = x + (size_t)m * cols;
        float *y = (float *)malloc(sizeof(float) * (size_t)cols);
        float r = 1.0f;
        if (norm) {
            double ss = 0.0;
            for (int c = 0; c < cols; ++c) ss += bf(xr[c]) * bf(xr[c]);
            float ms = (float)(ss / (double)cols);
            float den = sqrtf(ms + eps);
            r = 1.0f / den;
        }
        float amax = 0.0f;
        for (int c = 0; c < cols; ++c) {
            float v = bf32(xr[c]);
            if (norm) {
                v = v * r;
                if (gamma) v = v * gamma[c];
            }
            y[c] = v;
            amax = fmaxf(amax, fabsf(v));
        }
        float sc = amax / 127.0f;
        s[m] = sc;
        for (int c = 0; c < cols; ++c) q[(size_t)m * cols + c] = code8(y[c], sc);
        free(y);
    }
}

void orc_w8a8_linear(const int8_t *qx, const float *sx, const int8_t *qw, const float *sw, const float *bias, int M,
                     int N, int K, double *out)
{
#pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m)
        for (int n = 0; n < N; ++n) {
            int64_t acc = 0;
            for (int k = 0; k < K; ++k) acc += (int64_t)qx[(size_t)m * K + k] * (int64_t)qw[(size_t)n * K + k];
            double v = (double)acc * (double)sx[m] * (double)sw[n];
            if (bias) v += (double)bias[n];
            out[(size_t)m * N + n] = v;
        }
}
