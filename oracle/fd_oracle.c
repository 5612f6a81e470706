/*
 * fd_oracle.c -- CPU oracle for single-query decode attention.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library. The CUDA product path
 * never calls it, and the two share no code, header, table or helper.
 *
 * Source: "Flash-Decoding for long-context inference" (Tri Dao, Daniel
 * Haziza, Francisco Massa, Grigory Sizov; Stanford CRFM blog).
 *
 *  - Section "Multi-head attention for decoding": while decoding, the query
 *    of the new token (query length 1) attends to every previous token of
 *    its sequence. Written out, for one (sequence b, query head i) row with
 *    L cached tokens and key/value head j:
 *        z_t = scale * sum_d q[d] * k_t[d]            for t < L
 *        lse = log( sum_t exp(z_t) )                  (natural log)
 *        out = sum_t exp(z_t - lse) * v_t
 *    fdo_attention() is this definition, nothing more. Subtracting the row
 *    maximum before exp() is exact in real arithmetic; it only keeps exp()
 *    from overflowing in double for large logits.
 *
 *  - Several queries per sequence ("flash decoding论文" page: with multi-turn
 *    dialogue or speculative decoding several query vectors are computed in
 *    parallel). Reading taken: sequence b holds L = seqlens[b] cached tokens
 *    of which the last q_len are the new ones, in order; query j (0-based)
 *    is the token at position L - q_len + j and attends causally to tokens
 *    t < L - (q_len - 1 - j). fdo_attention_multi() is the same definition
 *    with that length per query; q_len = 1 is fdo_attention().
 *
 *  - Section "A faster attention for decoding: Flash-Decoding": the keys and
 *    values are cut into chunks along the sequence, the attention of the
 *    query with each chunk is computed on its own together with one extra
 *    scalar per row and split (the log-sum-exp of that chunk's logits), and
 *    a final reduction rescales each split's output by its log-sum-exp and
 *    sums them. fdo_split_attention() performs these steps in that order;
 *    fdo_combine() is the final reduction alone. They exist to pin the
 *    identity that makes splitting exact, not for GPU parity.
 *
 * Readings where the page is silent (stated once here, used throughout):
 *  - grouped-query heads: query head i reads key/value head i / (Hq/Hkv);
 *  - a split's partial output is stored normalised (divided by its own
 *    softmax denominator); its weight in the reduction is exp(lse_s - LSE);
 *  - a row or split with no tokens has output 0 and log-sum-exp -inf, and an
 *    empty split gets weight 0 in the reduction;
 *  - seqlens[b] is clamped to [0, Lmax]; positions t >= seqlens[b] are never
 *    read, so whatever fills them (NaN in the ragged workload) cannot matter.
 *
 *  - Quantised key/value cache (the "flash decoding论文" page lists INT8/INT4
 *    quantisation among PaddleNLP's inference techniques). Reading taken:
 *    each cached byte is a code, dequantised with one scale per key/value
 *    head, k = k_scale[j] * decode(code), v = v_scale[j] * decode(code);
 *    the attention is then the definition above over those values.
 *    decode() is either 8-bit two's complement (int8) or the OCP 8-bit
 *    floating-point format E4M3 (1 sign bit, 4 exponent bits with bias 7,
 *    3 mantissa bits; exponent field 0 is subnormal, (m/8) * 2^-6; the one
 *    code S.1111.111 is NaN; no infinities), written out from its fields.
 *    fdo_attention_quant() is that, with any number of queries per sequence.
 *
 * Precision: inputs are bf16 bit patterns decoded exactly to double; all
 * arithmetic is IEEE double with the C library's exp() and log(). Rows are
 * independent, so they are spread over POSIX threads; each row is computed
 * by one thread, in token order.
 *
 * FDO_MUTANT (compile-time, default 0) plants one known mistake; it exists
 * only so the test suite can show that its pins catch each such mistake.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#ifndef FDO_MUTANT
#define FDO_MUTANT 0
#endif

/* bf16 is the top half of an IEEE binary32; the conversion is exact. */
static double bf16_to_double(uint16_t h) {
    uint32_t bits = (uint32_t)h << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* OCP E4M3 code -> value, from its bit fields. */
static double e4m3_to_double(uint8_t c) {
    const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
#if FDO_MUTANT == 9
    mag = ldexp(1.0 + m / 8.0, e - 7);             /* planted: subnormals read as normals */
#else
    if (e == 0)
        mag = ldexp(m / 8.0, -6);
    else
#if FDO_MUTANT == 13
        mag = ldexp(1.0 + m / 8.0, e - 8);         /* planted: exponent bias 8 */
#else
        mag = ldexp(1.0 + m / 8.0, e - 7);
#endif
#endif
    return s ? -mag : mag;
}

/* int8 code -> value (two's complement). */
static double int8_to_double(uint8_t c) {
#if FDO_MUTANT == 11
    return (double)c;                              /* planted: read as unsigned */
#else
    return c < 128 ? (double)c : (double)c - 256.0;
#endif
}

enum { FDO_KV_BF16 = 0, FDO_KV_E4M3 = 1, FDO_KV_INT8 = 2 };

typedef struct {
    int B, Hq, Hkv, D, Lmax;
    const uint16_t *q, *k, *v;
    /* quantised cache (kv_type != FDO_KV_BF16): codes and per-kv-head scales */
    int kv_type;
    const uint8_t *k8, *v8;
    const float *k_scale, *v_scale;
    const int32_t *seqlens;
    double scale;
    double *out, *lse;
    /* split form only */
    int nsplit;
    const int32_t *bounds;   /* nsplit + 1 token boundaries, ascending */
    double *part_o;          /* [B, Hq, nsplit, D] or NULL */
    double *part_lse;        /* [B, Hq, nsplit]    or NULL */
    /* several queries per sequence (fdo_attention_multi) */
    int q_len;
    /* thread partition */
    int nthreads, tid;
} job_t;

static double code_value(int kv_type, uint8_t c) {
    return kv_type == FDO_KV_E4M3 ? e4m3_to_double(c) : int8_to_double(c);
}

/* Element idx of the key cache [B,Hkv,Lmax,D], whose kv head is j. */
static double key_at(const job_t *J, size_t idx, int j) {
    if (J->kv_type == FDO_KV_BF16) return bf16_to_double(J->k[idx]);
    return (double)J->k_scale[j] * code_value(J->kv_type, J->k8[idx]);
}

/* Element idx of the value cache, whose kv head is j. */
static double value_at(const job_t *J, size_t idx, int j) {
#if FDO_MUTANT == 5
    return key_at(J, idx, j);                      /* planted: keys as values */
#else
    if (J->kv_type == FDO_KV_BF16) return bf16_to_double(J->v[idx]);
#if FDO_MUTANT == 10
    return (double)J->k_scale[j] * code_value(J->kv_type, J->v8[idx]);   /* planted: key scale on values */
#else
    return (double)J->v_scale[j] * code_value(J->kv_type, J->v8[idx]);
#endif
#endif
}

static int clamp_len(int L, int Lmax) {
    if (L < 0) return 0;
    if (L > Lmax) return Lmax;
    return L;
}

/* Logits z_t = scale * <qrow, k_t> for t in [t0, t1), query head i of sequence b. */
static void row_logits(const job_t *J, int b, int i, const uint16_t *qrow, int t0, int t1, double *z) {
    const int g = J->Hq / J->Hkv;
#if FDO_MUTANT == 2
    const int j = i % J->Hkv;                     /* planted: wrong group map */
#else
    const int j = i / g;
#endif
    for (int t = t0; t < t1; ++t) {
        const size_t krow = (((size_t)b * J->Hkv + j) * J->Lmax + t) * J->D;
        double dot = 0.0;
#if FDO_MUTANT == 12
        for (int d = 0; d < J->D - 1; ++d) dot += bf16_to_double(qrow[d]) * key_at(J, krow + d, j);   /* planted */
#else
        for (int d = 0; d < J->D; ++d) dot += bf16_to_double(qrow[d]) * key_at(J, krow + d, j);
#endif
#if FDO_MUTANT == 1
        z[t - t0] = dot;                           /* planted: scale dropped */
#else
        z[t - t0] = J->scale * dot;
#endif
    }
}

/* Softmax-weighted sum of v_t over tokens [t0, t1) given their logits.
 * Writes the normalised output o[D] and returns the log-sum-exp. */
static double row_softmax_sum(const job_t *J, int b, int i, int t0, int t1,
                              const double *z, double *o) {
    const int g = J->Hq / J->Hkv;
#if FDO_MUTANT == 2
    const int j = i % J->Hkv;
#else
    const int j = i / g;
#endif
    for (int d = 0; d < J->D; ++d) o[d] = 0.0;
    if (t1 <= t0) return -INFINITY;
    double M = z[0];
    for (int t = 1; t < t1 - t0; ++t) if (z[t] > M) M = z[t];
    double Z = 0.0;
    for (int t = 0; t < t1 - t0; ++t) Z += exp(z[t] - M);
    for (int t = t0; t < t1; ++t) {
        const double w = exp(z[t - t0] - M);
        const size_t vrow = (((size_t)b * J->Hkv + j) * J->Lmax + t) * J->D;
#if FDO_MUTANT == 14
        for (int d = 0; d < J->D; ++d) o[d] += w * value_at(J, vrow + (J->D - 1 - d), j);   /* planted */
#else
        for (int d = 0; d < J->D; ++d) o[d] += w * value_at(J, vrow + d, j);
#endif
    }
#if FDO_MUTANT != 6
    for (int d = 0; d < J->D; ++d) o[d] /= Z;       /* mutant 6 plants: no normalisation */
#endif
#if FDO_MUTANT == 4
    return (M + log(Z)) / log(2.0);                  /* planted: base-2 log-sum-exp */
#else
    return M + log(Z);
#endif
}

static int row_length(const job_t *J, int b) {
    int L = clamp_len(J->seqlens[b], J->Lmax);
#if FDO_MUTANT == 3
    if (L > 0) L -= 1;                               /* planted: last token dropped */
#endif
    return L;
}

/* --- plain definition ---------------------------------------------------- */

static void *attention_worker(void *arg) {
    const job_t *J = (const job_t *)arg;
    double *z = (double *)malloc(sizeof(double) * (size_t)(J->Lmax > 0 ? J->Lmax : 1));
    if (!z) return (void *)1;
    const int rows = J->B * J->Hq;
    for (int r = J->tid; r < rows; r += J->nthreads) {
        const int b = r / J->Hq, i = r % J->Hq;
        const int L = row_length(J, b);
        row_logits(J, b, i, J->q + (size_t)r * J->D, 0, L, z);
        J->lse[r] = row_softmax_sum(J, b, i, 0, L, z, J->out + (size_t)r * J->D);
    }
    free(z);
    return NULL;
}

/* --- split form: per-split attention + log-sum-exp, then reduction ------- */

/* Final reduction over n splits of one row (the "small final reduction
 * step"): LSE = log sum_s exp(lse_s); out = sum_s exp(lse_s - LSE) * O_s.
 * Empty splits (lse_s = -inf) carry weight 0. */
static double combine_row(int n, int D, const double *po, const double *pl, double *out) {
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    double M = -INFINITY;
    for (int s = 0; s < n; ++s) if (pl[s] > M) M = pl[s];
    if (M == -INFINITY) return -INFINITY;
    double S = 0.0;
    for (int s = 0; s < n; ++s) if (pl[s] != -INFINITY) S += exp(pl[s] - M);
    const double LSE = M + log(S);
    for (int s = 0; s < n; ++s) {
        if (pl[s] == -INFINITY) continue;
#if FDO_MUTANT == 7
        const double w = exp(pl[s]);                 /* planted: weight not rescaled by LSE */
#else
        const double w = exp(pl[s] - LSE);
#endif
        for (int d = 0; d < D; ++d) out[d] += w * po[(size_t)s * D + d];
    }
    return LSE;
}

static void *split_worker(void *arg) {
    const job_t *J = (const job_t *)arg;
    const int n = J->nsplit;
    double *z = (double *)malloc(sizeof(double) * (size_t)(J->Lmax > 0 ? J->Lmax : 1));
    double *po = (double *)malloc(sizeof(double) * (size_t)n * J->D);
    double *pl = (double *)malloc(sizeof(double) * (size_t)n);
    if (!z || !po || !pl) { free(z); free(po); free(pl); return (void *)1; }
    const int rows = J->B * J->Hq;
    for (int r = J->tid; r < rows; r += J->nthreads) {
        const int b = r / J->Hq, i = r % J->Hq;
        const int L = row_length(J, b);
        /* 1. each split: attention of the query with its chunk, plus its lse */
        for (int s = 0; s < n; ++s) {
            int t0 = J->bounds[s], t1 = J->bounds[s + 1];
            if (t0 > L) t0 = L;
            if (t1 > L) t1 = L;
            row_logits(J, b, i, J->q + ((size_t)b * J->Hq + i) * J->D, t0, t1, z);
            pl[s] = row_softmax_sum(J, b, i, t0, t1, z, po + (size_t)s * J->D);
        }
        if (J->part_o) memcpy(J->part_o + (size_t)r * n * J->D, po, sizeof(double) * (size_t)n * J->D);
        if (J->part_lse) memcpy(J->part_lse + (size_t)r * n, pl, sizeof(double) * (size_t)n);
        /* 2. reduce over the splits, each scaled through its lse */
        J->lse[r] = combine_row(n, J->D, po, pl, J->out + (size_t)r * J->D);
    }
    free(z); free(po); free(pl);
    return NULL;
}

static int run_threads_rows(job_t *proto, void *(*fn)(void *), int nthreads, int rows) {
    if (nthreads <= 0) {
        long c = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = c > 0 ? (int)c : 1;
    }
    if (nthreads > rows) nthreads = rows > 0 ? rows : 1;
    job_t *jobs = (job_t *)malloc(sizeof(job_t) * (size_t)nthreads);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!jobs || !th) { free(jobs); free(th); return -1; }
    int rc = 0;
    for (int k = 0; k < nthreads; ++k) {
        jobs[k] = *proto;
        jobs[k].nthreads = nthreads;
        jobs[k].tid = k;
    }
    for (int k = 1; k < nthreads; ++k)
        if (pthread_create(&th[k], NULL, fn, &jobs[k]) != 0) { rc = -1; jobs[k].tid = -1; }
    if (fn(&jobs[0]) != NULL) rc = -1;
    for (int k = 1; k < nthreads; ++k) {
        if (jobs[k].tid < 0) continue;
        void *ret = NULL;
        pthread_join(th[k], &ret);
        if (ret != NULL) rc = -1;
    }
    free(jobs); free(th);
    return rc == 0 ? nthreads : rc;
}

static int run_threads(job_t *proto, void *(*fn)(void *), int nthreads) {
    return run_threads_rows(proto, fn, nthreads, proto->B * proto->Hq);
}

static int check_shape(int B, int Hq, int Hkv, int D, int Lmax) {
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Lmax < 0) return -1;
    if (Hq % Hkv != 0) return -1;
    return 0;
}

/* Plain attention for every (b, i) row. Returns the number of threads used
 * (> 0) or a negative value on bad arguments / allocation failure.
 * q: [B,Hq,D]; k, v: [B,Hkv,Lmax,D] (bf16 bits); seqlens: [B];
 * out: [B,Hq,D]; lse: [B,Hq]. nthreads <= 0 means one per online core. */
int fdo_attention(int B, int Hq, int Hkv, int D, int Lmax,
                  const uint16_t *q, const uint16_t *k, const uint16_t *v,
                  const int32_t *seqlens, double scale,
                  double *out, double *lse, int nthreads) {
    if (check_shape(B, Hq, Hkv, D, Lmax)) return -1;
    if (B == 0) return 1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.Lmax = Lmax;
    J.q = q; J.k = k; J.v = v; J.seqlens = seqlens; J.scale = scale;
    J.out = out; J.lse = lse;
    return run_threads(&J, attention_worker, nthreads);
}

/* --- several queries per sequence, causal among the new tokens --------- */

static void *multi_worker(void *arg) {
    const job_t *J = (const job_t *)arg;
    double *z = (double *)malloc(sizeof(double) * (size_t)(J->Lmax > 0 ? J->Lmax : 1));
    if (!z) return (void *)1;
    /* q, out: [B, q_len, Hq, D]; lse: [B, q_len, Hq]. Row r = (b*q_len + j)*Hq + i. */
    const int rows = J->B * J->q_len * J->Hq;
    for (int r = J->tid; r < rows; r += J->nthreads) {
        const int i = r % J->Hq, bj = r / J->Hq;
        const int j = bj % J->q_len, b = bj / J->q_len;
        int L = row_length(J, b);
#if FDO_MUTANT == 8
        L -= J->q_len - j;                           /* planted: query sees one token too few */
#else
        L -= J->q_len - 1 - j;                       /* query j sees t < L - (q_len - 1 - j) */
#endif
        if (L < 0) L = 0;
        row_logits(J, b, i, J->q + (size_t)r * J->D, 0, L, z);
        J->lse[r] = row_softmax_sum(J, b, i, 0, L, z, J->out + (size_t)r * J->D);
    }
    free(z);
    return NULL;
}

/* Several queries per sequence: q [B,q_len,Hq,D], k/v [B,Hkv,Lmax,D], seqlens [B];
 * out [B,q_len,Hq,D], lse [B,q_len,Hq]. Returns threads used or a negative value. */
int fdo_attention_multi(int B, int q_len, int Hq, int Hkv, int D, int Lmax,
                        const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const int32_t *seqlens, double scale,
                        double *out, double *lse, int nthreads) {
    if (check_shape(B, Hq, Hkv, D, Lmax) || q_len < 1) return -1;
    if (B == 0) return 1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.Lmax = Lmax;
    J.q = q; J.k = k; J.v = v; J.seqlens = seqlens; J.scale = scale;
    J.out = out; J.lse = lse; J.q_len = q_len;
    return run_threads_rows(&J, multi_worker, nthreads, B * q_len * Hq);
}

/* Quantised cache: k8/v8 [B,Hkv,Lmax,D] codes (kv_type 1 = E4M3, 2 = int8),
 * k_scale/v_scale [Hkv]; q [B,q_len,Hq,D] bf16 bits; out [B,q_len,Hq,D],
 * lse [B,q_len,Hq]. Query j sees t < seqlens[b] - (q_len - 1 - j), as in
 * fdo_attention_multi. Returns threads used or a negative value. */
int fdo_attention_quant(int B, int q_len, int Hq, int Hkv, int D, int Lmax, int kv_type,
                        const uint16_t *q, const uint8_t *k8, const uint8_t *v8,
                        const float *k_scale, const float *v_scale,
                        const int32_t *seqlens, double scale,
                        double *out, double *lse, int nthreads) {
    if (check_shape(B, Hq, Hkv, D, Lmax) || q_len < 1) return -1;
    if (kv_type != FDO_KV_E4M3 && kv_type != FDO_KV_INT8) return -1;
    if (B == 0) return 1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.Lmax = Lmax;
    J.q = q; J.kv_type = kv_type; J.k8 = k8; J.v8 = v8; J.k_scale = k_scale; J.v_scale = v_scale;
    J.seqlens = seqlens; J.scale = scale;
    J.out = out; J.lse = lse; J.q_len = q_len;
    return run_threads_rows(&J, multi_worker, nthreads, B * q_len * Hq);
}

/* Split-then-reduce form. bounds holds nsplit+1 ascending token positions;
 * split s covers [bounds[s], bounds[s+1]) cut to the row's length. part_o
 * ([B,Hq,nsplit,D]) and part_lse ([B,Hq,nsplit]) receive the per-split
 * results when non-NULL. Returns threads used or a negative value. */
int fdo_split_attention(int B, int Hq, int Hkv, int D, int Lmax,
                        const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const int32_t *seqlens, double scale,
                        int nsplit, const int32_t *bounds,
                        double *out, double *lse,
                        double *part_o, double *part_lse, int nthreads) {
    if (check_shape(B, Hq, Hkv, D, Lmax) || nsplit <= 0) return -1;
    for (int s = 0; s < nsplit; ++s) if (bounds[s] > bounds[s + 1] || bounds[s] < 0) return -1;
    if (B == 0) return 1;
    job_t J;
    memset(&J, 0, sizeof J);
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.Lmax = Lmax;
    J.q = q; J.k = k; J.v = v; J.seqlens = seqlens; J.scale = scale;
    J.out = out; J.lse = lse;
    J.nsplit = nsplit; J.bounds = bounds; J.part_o = part_o; J.part_lse = part_lse;
    return run_threads(&J, split_worker, nthreads);
}

/* The final reduction alone, for rows given as partials:
 * part_o [rows, nsplit, D], part_lse [rows, nsplit] -> out [rows, D], lse [rows]. */
int fdo_combine(int rows, int nsplit, int D, const double *part_o, const double *part_lse,
                double *out, double *lse) {
    if (rows < 0 || nsplit <= 0 || D <= 0) return -1;
    for (int r = 0; r < rows; ++r)
        lse[r] = combine_row(nsplit, D, part_o + (size_t)r * nsplit * D,
                             part_lse + (size_t)r * nsplit, out + (size_t)r * D);
    return 0;
}

int fdo_mutant(void) { return FDO_MUTANT; }
