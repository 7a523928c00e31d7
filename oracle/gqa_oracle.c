/*
 * gqa_oracle.c -- plain, slow, fp64 CPU oracle for grouped-query attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path (the
 * CUDA library and its Python binding) never calls it and shares no code,
 * header, table or helper with it.
 *
 * What it computes, and where the pages define it:
 *
 *  - Consecutive group mapping, kv_head = q_head / (Hq / Hkv), Hq divisible
 *    by Hkv: "Share keys and values without confusing query-head identity"
 *    (study.greatitself.com, grouped-query and multi-query attention), and the
 *    eight-to-two mapping check in "Shared KV can still produce different
 *    outputs" (lihaoran.work/?p=2890).
 *  - Raw KV-cache bytes = 2 x layers x tokens x kv_heads x head_dim x bytes:
 *    "KV-head count determines the raw cache ratio" (lihaoran.work/?p=2890),
 *    "Three numbers that people expect to move together"
 *    (deepconcepts.dev, Grouped-Query Attention).
 *  - Per query head, softmax(q K^T * scale) V with the head's own
 *    distribution: "Shared KV can still produce different outputs"
 *    (lihaoran.work/?p=2890).
 *  - The expanded formulation: each query head gets its own explicit copy of
 *    the K and V rows of its KV head (the repeat_interleave form), then plain
 *    per-head attention: "Kernels do not need to copy the KV heads"
 *    (anrans.github.io attention-variants, version 1 of its example).
 *  - Causal prefill: row r attends to tokens t <= r (lower triangle including
 *    the diagonal), masked scores excluded from the softmax: same section,
 *    the tril mask of its example.
 *  - Causal prefill backward: dq, and dk / dv summed over the group's query
 *    heads (study.greatitself.com, grouped-query and multi-query attention,
 *    training paragraph: the shared tensors receive every head's gradient,
 *    as differentiation of the explicitly repeated form gives).
 *  - FP8 KV cache: the cache stored in FP8 instead of bf16 ("Other ways to
 *    shrink the KV cache", anrans.github.io attention-variants: K and V in
 *    FP8, as serving engines support); every element is the E4M3 value of its
 *    byte times a per-tensor scale, and the attention is the same as above.
 *  - MLA decode with absorbed weights ("MLA: multi-head latent attention",
 *    anrans.github.io attention-variants, the weight-absorption and
 *    decoupled-RoPE paragraphs): the cache holds one row per token, the
 *    d_c-dim latent c followed by the d_r-dim RoPE key shared by all heads;
 *    every query head (its absorbed latent query, then its RoPE query) scores
 *    the whole row, and its output is the softmax-weighted sum of the latent
 *    part alone -- an MQA whose value is the key's first d_c entries.  The
 *    up-projection W_UV applied afterwards belongs to the output projection
 *    and is not part of it.
 *
 * Everything is done in double precision.  Inputs are the bf16 bit patterns
 * the GPU sees; bf16 is the upper 16 bits of an IEEE-754 binary32, so the
 * conversion below is exact.  The softmax is the two-pass form: maximum, then
 * exp(s - max) weights, then the weighted sum divided by the sum of weights.
 *
 * Readings taken where the pages are silent (each is listed in the design
 * notes of the repository):
 *  - decode: the query sees every cached token t < seqlens[b] (no other mask);
 *  - an empty history (seqlens[b] == 0) gives an all-zero output row;
 *  - outputs are fp64; callers compare rounded GPU outputs against them.
 *
 * Threads (pthreads) split the work over (batch, query head) pairs; each
 * pair is computed by exactly the same sequential code.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEMORY 2

/* ---- definitions the pages fix ------------------------------------------ */

/* kv head used by query head h under the consecutive grouping; -1 when the
 * grouping is not regular (Hq not divisible by Hkv) or h is out of range. */
int gqa_oracle_kv_head(int h, int Hq, int Hkv)
{
    if (Hq <= 0 || Hkv <= 0 || h < 0 || h >= Hq) return -1;
    if (Hq % Hkv != 0) return -1;
    int group = Hq / Hkv;
    return h / group;
}

/* raw KV-cache payload in bytes: K and V, for every layer, token, kv head and
 * head coordinate. */
long long gqa_oracle_kv_bytes(long long layers, long long tokens, long long kv_heads,
                              long long head_dim, long long bytes_per_elem)
{
    return 2LL * layers * tokens * kv_heads * head_dim * bytes_per_elem;
}

/* bf16 bit pattern -> double: the pattern is the top half of a binary32. */
static double bf16_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

void gqa_oracle_bf16_to_f64(const uint16_t *x, double *y, long long n)
{
    for (long long i = 0; i < n; ++i) y[i] = bf16_to_double(x[i]);
}

/* FP8 E4M3 (the "fn" variant: no infinities) byte -> double, from the format's
 * definition: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
 * exponent 0 encodes subnormals m * 2^-9; exponent 15 with mantissa 7 is NaN. */
static double e4m3_to_double(uint8_t x)
{
    const int sign = (x >> 7) & 1, e = (x >> 3) & 0xF, m = x & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);
    else v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

void gqa_oracle_e4m3_to_f64(const uint8_t *x, double *y, long long n)
{
    for (long long i = 0; i < n; ++i) y[i] = e4m3_to_double(x[i]);
}

/* ---- one query row against an explicit per-head copy of K and V --------- */

/* out[0:d] = sum_t softmax_t(scale * q.K[t]) V[t] over t < n, two-pass.
 * K, V are the head's own (already repeated) rows, row-major [n][d]. */
static void attend_row(const double *q, const double *K, const double *V, long long n, int d,
                       double scale, double *scores, double *out)
{
    for (int j = 0; j < d; ++j) out[j] = 0.0;
    if (n <= 0) return;
    double m = -INFINITY;
    for (long long t = 0; t < n; ++t) {
        double s = 0.0;
        for (int j = 0; j < d; ++j) s += q[j] * K[t * d + j];
        s *= scale;
        scores[t] = s;
        if (s > m) m = s;
    }
    double denom = 0.0;
    for (long long t = 0; t < n; ++t) {
        double w = exp(scores[t] - m);
        scores[t] = w;
        denom += w;
    }
    for (long long t = 0; t < n; ++t) {
        double w = scores[t];
        for (int j = 0; j < d; ++j) out[j] += w * V[t * d + j];
    }
    for (int j = 0; j < d; ++j) out[j] /= denom;
}

/* ---- decode -------------------------------------------------------------- */

typedef struct {
    const uint16_t *q, *k, *v;
    const int32_t *seqlens;
    int B, Hq, Hkv, d, Tmax;
    double scale;
    double *out;
    int tid, nthreads;
    int status;
    /* FP8 caches (k8, v8 non-NULL): element value = e4m3(byte) * k_scale (or v_scale) */
    const uint8_t *k8, *v8;
    double k_scale, v_scale;
} decode_job;

static void *decode_worker(void *arg)
{
    decode_job *J = (decode_job *)arg;
    const int d = J->d;
    double *qrow = (double *)malloc(sizeof(double) * (size_t)d);
    double *Kh = (double *)malloc(sizeof(double) * (size_t)J->Tmax * (size_t)d);
    double *Vh = (double *)malloc(sizeof(double) * (size_t)J->Tmax * (size_t)d);
    double *sc = (double *)malloc(sizeof(double) * (size_t)(J->Tmax > 0 ? J->Tmax : 1));
    if (!qrow || !Kh || !Vh || !sc) {
        J->status = ORACLE_NO_MEMORY;
        free(qrow); free(Kh); free(Vh); free(sc);
        return NULL;
    }
    long long pairs = (long long)J->B * J->Hq;
    for (long long p = J->tid; p < pairs; p += J->nthreads) {
        int b = (int)(p / J->Hq), h = (int)(p % J->Hq);
        int kvh = gqa_oracle_kv_head(h, J->Hq, J->Hkv);
        long long T = J->seqlens[b];
        /* explicit repeat: this query head's own copy of its KV head's rows */
        for (long long t = 0; t < T; ++t) {
            size_t src = (((size_t)b * J->Tmax + (size_t)t) * J->Hkv + (size_t)kvh) * (size_t)d;
            for (int j = 0; j < d; ++j) {
                if (J->k8) {
                    Kh[t * d + j] = e4m3_to_double(J->k8[src + j]) * J->k_scale;
                    Vh[t * d + j] = e4m3_to_double(J->v8[src + j]) * J->v_scale;
                } else {
                    Kh[t * d + j] = bf16_to_double(J->k[src + j]);
                    Vh[t * d + j] = bf16_to_double(J->v[src + j]);
                }
            }
        }
        size_t qo = ((size_t)b * J->Hq + (size_t)h) * (size_t)d;
        for (int j = 0; j < d; ++j) qrow[j] = bf16_to_double(J->q[qo + j]);
        attend_row(qrow, Kh, Vh, T, d, J->scale, sc, J->out + qo);
    }
    free(qrow); free(Kh); free(Vh); free(sc);
    return NULL;
}

static int run_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint8_t *k8,
                      const uint8_t *v8, double k_scale, double v_scale, const int32_t *seqlens, int B,
                      int Hq, int Hkv, int d, int Tmax, double scale, double *out, int nthreads);

/* q [B,Hq,d], k/v [B,Tmax,Hkv,d] bf16 bits, seqlens [B] (0 <= seqlens <= Tmax),
 * out [B,Hq,d] fp64.  Returns 0 on success. */
int gqa_oracle_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                      const int32_t *seqlens, int B, int Hq, int Hkv, int d, int Tmax,
                      double scale, double *out, int nthreads)
{
    if (!k || !v) return ORACLE_BAD_ARG;
    return run_decode(q, k, v, NULL, NULL, 1.0, 1.0, seqlens, B, Hq, Hkv, d, Tmax, scale, out, nthreads);
}

/* The same decode over an FP8 (E4M3) cache with per-tensor scales: every cached
 * element is e4m3(byte) * k_scale (keys) or e4m3(byte) * v_scale (values). */
int gqa_oracle_decode_fp8(const uint16_t *q, const uint8_t *k8, const uint8_t *v8, double k_scale,
                          double v_scale, const int32_t *seqlens, int B, int Hq, int Hkv, int d, int Tmax,
                          double scale, double *out, int nthreads)
{
    if (!k8 || !v8) return ORACLE_BAD_ARG;
    return run_decode(q, NULL, NULL, k8, v8, k_scale, v_scale, seqlens, B, Hq, Hkv, d, Tmax, scale, out,
                      nthreads);
}

static int run_decode(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint8_t *k8,
                      const uint8_t *v8, double k_scale, double v_scale, const int32_t *seqlens, int B,
                      int Hq, int Hkv, int d, int Tmax, double scale, double *out, int nthreads)
{
    if (!q || !seqlens || !out) return ORACLE_BAD_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0 || Tmax < 0) return ORACLE_BAD_ARG;
    if (Hq % Hkv != 0) return ORACLE_BAD_ARG;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Tmax) return ORACLE_BAD_ARG;
    if (nthreads < 1) nthreads = 1;
    if ((long long)nthreads > (long long)B * Hq) nthreads = B * Hq;
    decode_job *jobs = (decode_job *)calloc((size_t)nthreads, sizeof(decode_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return ORACLE_NO_MEMORY; }
    for (int i = 0; i < nthreads; ++i) {
        decode_job J = {q, k, v, seqlens, B, Hq, Hkv, d, Tmax, scale, out, i, nthreads, ORACLE_OK,
                        k8, v8, k_scale, v_scale};
        jobs[i] = J;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, decode_worker, &jobs[i]);
    decode_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    int st = ORACLE_OK;
    for (int i = 0; i < nthreads; ++i) if (jobs[i].status != ORACLE_OK) st = jobs[i].status;
    free(jobs); free(th);
    return st;
}

/* ---- causal prefill ------------------------------------------------------ */

typedef struct {
    const uint16_t *q, *k, *v;
    int B, S, Hq, Hkv, d;
    double scale;
    const int32_t *rows; /* NULL: every row; else nrows (b, h, r) triples */
    long long nrows;
    double *out;
    int tid, nthreads;
    int status;
} prefill_job;

/* every row of one (b, h): row r sees tokens 0..r inclusive */
static void prefill_head(const prefill_job *J, int b, int h, double *Kh, double *Vh,
                         double *qrow, double *sc)
{
    const int d = J->d, S = J->S;
    int kvh = gqa_oracle_kv_head(h, J->Hq, J->Hkv);
    /* explicit repeat of the whole KV head for this query head */
    for (long long t = 0; t < S; ++t) {
        size_t src = (((size_t)b * S + (size_t)t) * J->Hkv + (size_t)kvh) * (size_t)d;
        for (int j = 0; j < d; ++j) {
            Kh[t * d + j] = bf16_to_double(J->k[src + j]);
            Vh[t * d + j] = bf16_to_double(J->v[src + j]);
        }
    }
    for (long long r = 0; r < S; ++r) {
        size_t qo = (((size_t)b * S + (size_t)r) * J->Hq + (size_t)h) * (size_t)d;
        for (int j = 0; j < d; ++j) qrow[j] = bf16_to_double(J->q[qo + j]);
        attend_row(qrow, Kh, Vh, r + 1, d, J->scale, sc, J->out + qo);
    }
}

static void *prefill_worker(void *arg)
{
    prefill_job *J = (prefill_job *)arg;
    const int d = J->d, S = J->S;
    double *Kh = (double *)malloc(sizeof(double) * (size_t)S * (size_t)d);
    double *Vh = (double *)malloc(sizeof(double) * (size_t)S * (size_t)d);
    double *qrow = (double *)malloc(sizeof(double) * (size_t)d);
    double *sc = (double *)malloc(sizeof(double) * (size_t)S);
    if (!Kh || !Vh || !qrow || !sc) {
        J->status = ORACLE_NO_MEMORY;
        free(Kh); free(Vh); free(qrow); free(sc);
        return NULL;
    }
    long long pairs = (long long)J->B * J->Hq;
    for (long long p = J->tid; p < pairs; p += J->nthreads) {
        int b = (int)(p / J->Hq), h = (int)(p % J->Hq);
        if (!J->rows) {
            prefill_head(J, b, h, Kh, Vh, qrow, sc);
            continue;
        }
        /* subset mode: compute every listed row that belongs to (b, h) */
        int have_kv = 0;
        for (long long i = 0; i < J->nrows; ++i) {
            const int32_t *e = J->rows + 3 * i;
            if (e[0] != b || e[1] != h) continue;
            int kvh = gqa_oracle_kv_head(h, J->Hq, J->Hkv);
            if (!have_kv) {
                long long rmax = 0;
                for (long long u = i; u < J->nrows; ++u) {
                    const int32_t *f = J->rows + 3 * u;
                    if (f[0] == b && f[1] == h && f[2] > rmax) rmax = f[2];
                }
                for (long long t = 0; t <= rmax; ++t) {
                    size_t src = (((size_t)b * S + (size_t)t) * J->Hkv + (size_t)kvh) * (size_t)d;
                    for (int j = 0; j < d; ++j) {
                        Kh[t * d + j] = bf16_to_double(J->k[src + j]);
                        Vh[t * d + j] = bf16_to_double(J->v[src + j]);
                    }
                }
                have_kv = 1;
            }
            long long r = e[2];
            size_t qo = (((size_t)b * S + (size_t)r) * J->Hq + (size_t)h) * (size_t)d;
            for (int j = 0; j < d; ++j) qrow[j] = bf16_to_double(J->q[qo + j]);
            attend_row(qrow, Kh, Vh, r + 1, d, J->scale, sc, J->out + (size_t)i * (size_t)d);
        }
    }
    free(Kh); free(Vh); free(qrow); free(sc);
    return NULL;
}

/* q [B,S,Hq,d], k/v [B,S,Hkv,d] bf16 bits.  rows == NULL: out [B,S,Hq,d] fp64
 * for every row.  rows != NULL: nrows (b, h, r) int32 triples; out [nrows,d]
 * holds those rows in the order given.  Returns 0 on success. */
int gqa_oracle_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v, int B, int S,
                       int Hq, int Hkv, int d, double scale, const int32_t *rows,
                       long long nrows, double *out, int nthreads)
{
    if (!q || !k || !v || !out) return ORACLE_BAD_ARG;
    if (B <= 0 || S <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return ORACLE_BAD_ARG;
    if (Hq % Hkv != 0) return ORACLE_BAD_ARG;
    if (rows) {
        if (nrows < 0) return ORACLE_BAD_ARG;
        for (long long i = 0; i < nrows; ++i) {
            const int32_t *e = rows + 3 * i;
            if (e[0] < 0 || e[0] >= B || e[1] < 0 || e[1] >= Hq || e[2] < 0 || e[2] >= S)
                return ORACLE_BAD_ARG;
        }
    }
    if (nthreads < 1) nthreads = 1;
    if ((long long)nthreads > (long long)B * Hq) nthreads = B * Hq;
    prefill_job *jobs = (prefill_job *)calloc((size_t)nthreads, sizeof(prefill_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return ORACLE_NO_MEMORY; }
    for (int i = 0; i < nthreads; ++i) {
        prefill_job J = {q, k, v, B, S, Hq, Hkv, d, scale, rows, nrows, out, i, nthreads, ORACLE_OK};
        jobs[i] = J;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, prefill_worker, &jobs[i]);
    prefill_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    int st = ORACLE_OK;
    for (int i = 0; i < nthreads; ++i) if (jobs[i].status != ORACLE_OK) st = jobs[i].status;
    free(jobs); free(th);
    return st;
}

/* ---- causal prefill backward ----------------------------------------------
 *
 * Gradients of a scalar loss through the causal prefill, given dO = dL/dout:
 * "During training, a shared key or value tensor receives gradient
 * contributions from every query head in its group" (study.greatitself.com,
 * grouped-query and multi-query attention, training paragraph).  Written out
 * per query head h of KV head kvh, with s_rt = scale q_r.k_t for t <= r,
 * P_rt = exp(s_rt - lse_r), lse_r = log sum_{t<=r} exp(s_rt):
 *
 *   dP_rt = dO_r . v_t
 *   D_r   = sum_t P_rt dP_rt
 *   dS_rt = P_rt (dP_rt - D_r)
 *   dq_r  = scale sum_{t<=r} dS_rt k_t
 *   dk_t += scale sum_{r>=t} dS_rt q_r      (summed over the group's heads)
 *   dv_t += sum_{r>=t} P_rt dO_r            (summed over the group's heads)
 *
 * Each (b, kvh) is one job (so the group sums have a single writer); within
 * it every head of the group works on its own explicit copy of K and V.
 * row_sel / key_sel (S flags, or NULL for all): which query rows get dq and
 * which keys get dk / dv; the others are left zero.  The row statistics
 * (lse_r, D_r) are computed for the selected rows and for every row at or
 * after the first selected key, since dk and dv of a key need them for every
 * later row. */

typedef struct {
    const uint16_t *q, *k, *v, *dout;
    int B, S, Hq, Hkv, d;
    double scale;
    const int32_t *row_sel, *key_sel;
    int first_key;        /* first selected key (key_sel given) */
    double *dq, *dk, *dv;
    int tid, nthreads;
    int status;
} backward_job;

static void *backward_worker(void *arg)
{
    backward_job *J = (backward_job *)arg;
    const int S = J->S, d = J->d, g = J->Hq / J->Hkv;
    double *Kh = (double *)malloc(sizeof(double) * (size_t)S * (size_t)d);
    double *Vh = (double *)malloc(sizeof(double) * (size_t)S * (size_t)d);
    double *Qh = (double *)malloc(sizeof(double) * (size_t)S * (size_t)d);
    double *dOh = (double *)malloc(sizeof(double) * (size_t)S * (size_t)d);
    double *lse = (double *)malloc(sizeof(double) * (size_t)S);
    double *Dr = (double *)malloc(sizeof(double) * (size_t)S);
    double *sc = (double *)malloc(sizeof(double) * (size_t)S);
    if (!Kh || !Vh || !Qh || !dOh || !lse || !Dr || !sc) {
        J->status = ORACLE_NO_MEMORY;
        free(Kh); free(Vh); free(Qh); free(dOh); free(lse); free(Dr); free(sc);
        return NULL;
    }
    const long long jobs = (long long)J->B * J->Hkv;
    for (long long jb = J->tid; jb < jobs; jb += J->nthreads) {
        const int b = (int)(jb / J->Hkv), kvh = (int)(jb % J->Hkv);
        for (int hh = 0; hh < g; ++hh) {
            const int h = kvh * g + hh;
            if (gqa_oracle_kv_head(h, J->Hq, J->Hkv) != kvh) { J->status = ORACLE_BAD_ARG; break; }
            /* this head's own copies: q, dO rows of head h; K, V rows of its KV head */
            for (int t = 0; t < S; ++t) {
                const size_t kv = (((size_t)b * S + (size_t)t) * J->Hkv + (size_t)kvh) * (size_t)d;
                const size_t qo = (((size_t)b * S + (size_t)t) * J->Hq + (size_t)h) * (size_t)d;
                for (int j = 0; j < d; ++j) {
                    Kh[(size_t)t * d + j] = bf16_to_double(J->k[kv + j]);
                    Vh[(size_t)t * d + j] = bf16_to_double(J->v[kv + j]);
                    Qh[(size_t)t * d + j] = bf16_to_double(J->q[qo + j]);
                    dOh[(size_t)t * d + j] = bf16_to_double(J->dout[qo + j]);
                }
            }
            /* row statistics lse_r and D_r: for the selected rows and every row at or after the first
             * selected key (the rows whose weights reach a selected key) */
            for (int r = 0; r < S; ++r) {
                if (J->row_sel && J->key_sel && !J->row_sel[r] && r < J->first_key) continue;
                double m = -INFINITY;
                for (int t = 0; t <= r; ++t) {
                    double s = 0.0;
                    for (int j = 0; j < d; ++j) s += Qh[(size_t)r * d + j] * Kh[(size_t)t * d + j];
                    s *= J->scale;
                    sc[t] = s;
                    if (s > m) m = s;
                }
                double z = 0.0;
                for (int t = 0; t <= r; ++t) z += exp(sc[t] - m);
                lse[r] = m + log(z);
                double Dsum = 0.0;
                for (int t = 0; t <= r; ++t) {
                    double dP = 0.0;
                    for (int j = 0; j < d; ++j) dP += dOh[(size_t)r * d + j] * Vh[(size_t)t * d + j];
                    Dsum += exp(sc[t] - lse[r]) * dP;
                }
                Dr[r] = Dsum;
            }
            /* dq for the selected rows */
            for (int r = 0; r < S; ++r) {
                if (J->row_sel && !J->row_sel[r]) continue;
                double *dq = J->dq + (((size_t)b * S + (size_t)r) * J->Hq + (size_t)h) * (size_t)d;
                for (int t = 0; t <= r; ++t) {
                    double s = 0.0, dP = 0.0;
                    for (int j = 0; j < d; ++j) {
                        s += Qh[(size_t)r * d + j] * Kh[(size_t)t * d + j];
                        dP += dOh[(size_t)r * d + j] * Vh[(size_t)t * d + j];
                    }
                    const double P = exp(s * J->scale - lse[r]);
                    const double dS = P * (dP - Dr[r]);
                    for (int j = 0; j < d; ++j) dq[j] += J->scale * dS * Kh[(size_t)t * d + j];
                }
            }
            /* dk, dv for the selected keys, accumulated over the group's heads */
            for (int t = 0; t < S; ++t) {
                if (J->key_sel && !J->key_sel[t]) continue;
                const size_t kv = (((size_t)b * S + (size_t)t) * J->Hkv + (size_t)kvh) * (size_t)d;
                double *dk = J->dk + kv, *dv = J->dv + kv;
                for (int r = t; r < S; ++r) {
                    double s = 0.0, dP = 0.0;
                    for (int j = 0; j < d; ++j) {
                        s += Qh[(size_t)r * d + j] * Kh[(size_t)t * d + j];
                        dP += dOh[(size_t)r * d + j] * Vh[(size_t)t * d + j];
                    }
                    const double P = exp(s * J->scale - lse[r]);
                    const double dS = P * (dP - Dr[r]);
                    for (int j = 0; j < d; ++j) {
                        dv[j] += P * dOh[(size_t)r * d + j];
                        dk[j] += J->scale * dS * Qh[(size_t)r * d + j];
                    }
                }
            }
        }
    }
    free(Kh); free(Vh); free(Qh); free(dOh); free(lse); free(Dr); free(sc);
    return NULL;
}

/* q, dout [B,S,Hq,d], k, v [B,S,Hkv,d] bf16 bits; dq [B,S,Hq,d], dk, dv [B,S,Hkv,d] fp64, zeroed
 * here.  row_sel / key_sel: NULL or S int32 flags.  Returns 0 on success. */
int gqa_oracle_prefill_backward(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                                int B, int S, int Hq, int Hkv, int d, double scale, const int32_t *row_sel,
                                const int32_t *key_sel, double *dq, double *dk, double *dv, int nthreads)
{
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return ORACLE_BAD_ARG;
    if (B <= 0 || S <= 0 || Hq <= 0 || Hkv <= 0 || d <= 0) return ORACLE_BAD_ARG;
    if (Hq % Hkv != 0) return ORACLE_BAD_ARG;
    memset(dq, 0, sizeof(double) * (size_t)B * S * Hq * d);
    memset(dk, 0, sizeof(double) * (size_t)B * S * Hkv * d);
    memset(dv, 0, sizeof(double) * (size_t)B * S * Hkv * d);
    if (nthreads < 1) nthreads = 1;
    if ((long long)nthreads > (long long)B * Hkv) nthreads = B * Hkv;
    backward_job *jobs = (backward_job *)calloc((size_t)nthreads, sizeof(backward_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return ORACLE_NO_MEMORY; }
    int first_key = S;
    if (key_sel)
        for (int t = S - 1; t >= 0; --t)
            if (key_sel[t]) first_key = t;
    for (int i = 0; i < nthreads; ++i) {
        backward_job J = {q, k, v, dout, B, S, Hq, Hkv, d, scale, row_sel, key_sel, first_key, dq, dk, dv, i,
                          nthreads, ORACLE_OK};
        jobs[i] = J;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, backward_worker, &jobs[i]);
    backward_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    int st = ORACLE_OK;
    for (int i = 0; i < nthreads; ++i) if (jobs[i].status != ORACLE_OK) st = jobs[i].status;
    free(jobs); free(th);
    return st;
}

/* ---- MLA decode (absorbed weights) ---------------------------------------- */

typedef struct {
    const uint16_t *q, *kv;
    const int32_t *seqlens;
    int B, Hq, dc, dr, Tmax;
    double scale;
    double *out;
    int tid, nthreads;
    int status;
} mla_job;

static void *mla_worker(void *arg)
{
    mla_job *J = (mla_job *)arg;
    const int dk = J->dc + J->dr, dv = J->dc;
    double *qrow = (double *)malloc(sizeof(double) * (size_t)dk);
    double *Kh = (double *)malloc(sizeof(double) * (size_t)(J->Tmax > 0 ? J->Tmax : 1) * (size_t)dk);
    double *Vh = (double *)malloc(sizeof(double) * (size_t)(J->Tmax > 0 ? J->Tmax : 1) * (size_t)dv);
    double *w = (double *)malloc(sizeof(double) * (size_t)(J->Tmax > 0 ? J->Tmax : 1));
    if (!qrow || !Kh || !Vh || !w) {
        J->status = ORACLE_NO_MEMORY;
        free(qrow); free(Kh); free(Vh); free(w);
        return NULL;
    }
    long long pairs = (long long)J->B * J->Hq;
    for (long long p = J->tid; p < pairs; p += J->nthreads) {
        int b = (int)(p / J->Hq), h = (int)(p % J->Hq);
        long long T = J->seqlens[b];
        /* this head's own copies: the key is the whole cached row, the value its latent part */
        for (long long t = 0; t < T; ++t) {
            const uint16_t *row = J->kv + ((size_t)b * J->Tmax + (size_t)t) * (size_t)dk;
            for (int i = 0; i < dk; ++i) Kh[t * dk + i] = bf16_to_double(row[i]);
            for (int j = 0; j < dv; ++j) Vh[t * dv + j] = bf16_to_double(row[j]);
        }
        const uint16_t *qs = J->q + ((size_t)b * J->Hq + (size_t)h) * (size_t)dk;
        for (int i = 0; i < dk; ++i) qrow[i] = bf16_to_double(qs[i]);
        double *o = J->out + ((size_t)b * J->Hq + (size_t)h) * (size_t)dv;
        for (int j = 0; j < dv; ++j) o[j] = 0.0;
        if (T <= 0) continue;
        /* scores over latent and RoPE parts together, then the two-pass softmax */
        double m = -INFINITY;
        for (long long t = 0; t < T; ++t) {
            double s = 0.0;
            for (int i = 0; i < dk; ++i) s += qrow[i] * Kh[t * dk + i];
            w[t] = s * J->scale;
            if (w[t] > m) m = w[t];
        }
        double denom = 0.0;
        for (long long t = 0; t < T; ++t) {
            w[t] = exp(w[t] - m);
            denom += w[t];
        }
        for (long long t = 0; t < T; ++t)
            for (int j = 0; j < dv; ++j) o[j] += w[t] * Vh[t * dv + j];
        for (int j = 0; j < dv; ++j) o[j] /= denom;
    }
    free(qrow); free(Kh); free(Vh); free(w);
    return NULL;
}

/* q [B,Hq,dc+dr] (absorbed latent query, then RoPE query), kv [B,Tmax,dc+dr] (latent, then the
 * shared RoPE key) bf16 bits, seqlens [B] (0 <= seqlens <= Tmax), out [B,Hq,dc] fp64:
 * out[b,h] = sum_{t < seqlens[b]} softmax_t(scale * q[b,h] . kv[b,t]) kv[b,t,0:dc].  Returns 0 on success. */
int gqa_oracle_mla_decode(const uint16_t *q, const uint16_t *kv, const int32_t *seqlens, int B, int Hq, int dc,
                          int dr, int Tmax, double scale, double *out, int nthreads)
{
    if (!q || !kv || !seqlens || !out) return ORACLE_BAD_ARG;
    if (B <= 0 || Hq <= 0 || dc <= 0 || dr < 0 || Tmax < 0) return ORACLE_BAD_ARG;
    for (int b = 0; b < B; ++b)
        if (seqlens[b] < 0 || seqlens[b] > Tmax) return ORACLE_BAD_ARG;
    if (nthreads < 1) nthreads = 1;
    if ((long long)nthreads > (long long)B * Hq) nthreads = B * Hq;
    mla_job *jobs = (mla_job *)calloc((size_t)nthreads, sizeof(mla_job));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return ORACLE_NO_MEMORY; }
    for (int i = 0; i < nthreads; ++i) {
        mla_job J = {q, kv, seqlens, B, Hq, dc, dr, Tmax, scale, out, i, nthreads, ORACLE_OK};
        jobs[i] = J;
    }
    for (int i = 1; i < nthreads; ++i) pthread_create(&th[i], NULL, mla_worker, &jobs[i]);
    mla_worker(&jobs[0]);
    for (int i = 1; i < nthreads; ++i) pthread_join(th[i], NULL);
    int st = ORACLE_OK;
    for (int i = 0; i < nthreads; ++i) if (jobs[i].status != ORACLE_OK) st = jobs[i].status;
    free(jobs); free(th);
    return st;
}

