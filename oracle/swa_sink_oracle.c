/*
 * swa_sink_oracle.c -- plain, slow fp64 CPU oracle for causal GQA attention
 * over a sliding window (or the full prefix) with a per-head attention-sink
 * logit in the softmax denominator.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the benchmark's
 * CPU-baseline / reference leg load this file's library. The product path
 * (the CUDA library) never links, loads or calls it, and this file includes
 * nothing from the CUDA side.
 *
 * What is computed, and where it comes from
 * -----------------------------------------
 * "MiMo-V2-Flash Technical Report" summary (mlpod.com), section 2.2.2
 * "Learnable Attention Sink Bias": a learnable scalar sink is added to the
 * softmax denominator so a row can put weight on a virtual sink instead of the
 * tokens in its window; a max term keeps the exponentials stable. The page's
 * equations are stripped, so this file takes the plainest reading of the
 * prose (per query row i of head h, with kv head g = h / (Hq/Hkv)):
 *
 *     a_j   = scale * (q_i . k_j)                 for every visible key j
 *     m     = max(s_h, max_j a_j)                 (the sink joins the max)
 *     den   = exp(s_h - m) + sum_j exp(a_j - m)
 *     o_i   = sum_j exp(a_j - m) / den * v_j      (the sink has no value)
 *     lse_i = m + ln(den)                         (natural log, sink included)
 *     w_sink = exp(s_h - m) / den
 *
 * No sink (NULL) means s_h = -inf: exp(-inf) = 0, the textbook softmax.
 *
 * Visible keys. Section 2.2.1 of the same page and the TL;DR give the window
 * as 128 tokens; the pages do not say whether the query itself counts. The
 * reading taken: key j is visible to query i (same sequence) iff
 * i - W + 1 <= j <= i, i.e. W keys including the query itself. W <= 0 means
 * the full causal prefix (the global-attention layers of section 2.2).
 *
 * Decode / draft verification (section 2.3 "Lightweight MTP" of the same page:
 * drafts are verified in parallel by the main model): query t (0 <= t < n_q)
 * of sequence b sits at absolute position P + t, P = pos[b]. Its keys, in
 * position order, are the committed tokens at positions
 * max(0, P+t-W+1) .. P-1, read from ring slot (p mod W), followed by the new
 * tokens 0..t (drafts are causal among themselves).
 *
 * Arithmetic: inputs are bf16 bit patterns widened exactly to double; every
 * sum is a plain left-to-right loop in double. No tiling, no online softmax,
 * no reordering. The only parallelism is an outer split of independent
 * (row, head) units over POSIX threads, which does not change any sum.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 -> double, exact: a bf16 is the top 16 bits of an IEEE binary32. */
static double bf16_to_double(uint16_t b)
{
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * One query row against an explicit key list (pointers to key/value rows in
 * position order). logit: scratch of n doubles.
 */
static void attend_row(const uint16_t *q, const uint16_t *const *krow,
                       const uint16_t *const *vrow, int n, int D, double s,
                       double scale, double *logit, double *o, double *lse,
                       double *wsink)
{
    /* logits and the max (seeded with the sink) */
    double m = s;
    for (int j = 0; j < n; ++j) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += bf16_to_double(q[d]) * bf16_to_double(krow[j][d]);
        logit[j] = scale * dot;
        if (logit[j] > m)
            m = logit[j];
    }
    if (n == 0 && isinf(m) && m < 0) { /* no keys and no sink: empty row */
        for (int d = 0; d < D; ++d)
            o[d] = 0.0;
        *lse = -INFINITY;
        if (wsink)
            *wsink = 0.0;
        return;
    }
    /* denominator: the sink term plus every key term */
    double sink_term = exp(s - m); /* exp(-inf) == 0 when there is no sink */
    double den = sink_term;
    for (int j = 0; j < n; ++j) {
        logit[j] = exp(logit[j] - m);
        den += logit[j];
    }
    /* output: weighted sum of the values; the sink contributes no value */
    for (int d = 0; d < D; ++d) {
        double acc = 0.0;
        for (int j = 0; j < n; ++j)
            acc += logit[j] * bf16_to_double(vrow[j][d]);
        o[d] = acc / den;
    }
    *lse = m + log(den);
    if (wsink)
        *wsink = sink_term / den;
}

/* ------------------------------------------------------------------------ */
/* prefill                                                                   */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *q, *k, *v;
    const int32_t *cu_seqlens;
    int num_seqs, Hq, Hkv, D, window;
    const double *sink;
    double scale;
    /* unit list: (token, head) pairs; either all of them or a sample */
    const int64_t *row_tok;  /* NULL => all rows, unit u = tok*Hq + head */
    const int32_t *row_head;
    int64_t nunits;
    /* outputs: full layout (o [total,Hq,D], lse/wsink [Hq,total]) when
       row_tok is NULL, else per-unit (o [n,D], lse/wsink [n]) */
    double *o, *lse, *wsink;
    int64_t total;
    int nthreads, tid;
} prefill_job;

static int seq_of_token(const int32_t *cu, int num_seqs, int64_t t)
{
    for (int s = 0; s < num_seqs; ++s)
        if (t >= cu[s] && t < cu[s + 1])
            return s;
    return -1;
}

static void *prefill_worker(void *arg)
{
    prefill_job *J = (prefill_job *)arg;
    int64_t maxkeys = 0;
    for (int s = 0; s < J->num_seqs; ++s) {
        int64_t L = J->cu_seqlens[s + 1] - J->cu_seqlens[s];
        if (L > maxkeys)
            maxkeys = L;
    }
    if (maxkeys < 1)
        maxkeys = 1;
    const uint16_t **kr = (const uint16_t **)malloc(sizeof(*kr) * maxkeys);
    const uint16_t **vr = (const uint16_t **)malloc(sizeof(*vr) * maxkeys);
    double *logit = (double *)malloc(sizeof(double) * maxkeys);
    const int G = J->Hq / J->Hkv;

    for (int64_t u = J->tid; u < J->nunits; u += J->nthreads) {
        int64_t i;
        int h;
        if (J->row_tok) {
            i = J->row_tok[u];
            h = J->row_head[u];
        } else {
            i = u / J->Hq;
            h = (int)(u % J->Hq);
        }
        int s = seq_of_token(J->cu_seqlens, J->num_seqs, i);
        int64_t start = J->cu_seqlens[s];
        int64_t lo = start;
        if (J->window > 0 && i - J->window + 1 > lo)
            lo = i - J->window + 1;
        int g = h / G;
        int n = 0;
        for (int64_t j = lo; j <= i; ++j, ++n) {
            kr[n] = J->k + (j * J->Hkv + g) * (int64_t)J->D;
            vr[n] = J->v + (j * J->Hkv + g) * (int64_t)J->D;
        }
        double sh = J->sink ? J->sink[h] : -INFINITY;
        const uint16_t *qrow = J->q + (i * J->Hq + h) * (int64_t)J->D;
        double *o, *lse, *ws;
        if (J->row_tok) {
            o = J->o + u * J->D;
            lse = J->lse + u;
            ws = J->wsink ? J->wsink + u : NULL;
        } else {
            o = J->o + (i * J->Hq + h) * (int64_t)J->D;
            lse = J->lse + (int64_t)h * J->total + i;
            ws = J->wsink ? J->wsink + (int64_t)h * J->total + i : NULL;
        }
        attend_row(qrow, kr, vr, n, J->D, sh, J->scale, logit, o, lse, ws);
    }
    free(kr);
    free(vr);
    free(logit);
    return NULL;
}

static int run_prefill(prefill_job *base)
{
    int nt = base->nthreads < 1 ? 1 : base->nthreads;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nt);
    prefill_job *jobs = (prefill_job *)malloc(sizeof(prefill_job) * nt);
    for (int t = 0; t < nt; ++t) {
        jobs[t] = *base;
        jobs[t].nthreads = nt;
        jobs[t].tid = t;
        pthread_create(&th[t], NULL, prefill_worker, &jobs[t]);
    }
    for (int t = 0; t < nt; ++t)
        pthread_join(th[t], NULL);
    free(th);
    free(jobs);
    return 0;
}

static int check_common(const int32_t *cu, int num_seqs, int Hq, int Hkv, int D)
{
    if (!cu || num_seqs < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv)
        return -2;
    if (cu[0] != 0)
        return -2;
    for (int s = 0; s < num_seqs; ++s)
        if (cu[s + 1] < cu[s])
            return -2;
    return 0;
}

/*
 * Every row of a packed varlen batch.
 * q [total,Hq,D], k/v [total,Hkv,D] bf16 bits; o [total,Hq,D] double;
 * lse, wsink [Hq,total] double (wsink may be NULL); sink [Hq] or NULL.
 */
int oracle_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                   const int32_t *cu_seqlens, int num_seqs, int Hq, int Hkv,
                   int D, int window, const double *sink, double scale,
                   double *o, double *lse, double *wsink, int nthreads)
{
    if (check_common(cu_seqlens, num_seqs, Hq, Hkv, D))
        return -2;
    prefill_job J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v;
    J.cu_seqlens = cu_seqlens; J.num_seqs = num_seqs;
    J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.window = window;
    J.sink = sink; J.scale = scale;
    J.total = cu_seqlens[num_seqs];
    J.nunits = J.total * Hq;
    J.o = o; J.lse = lse; J.wsink = wsink;
    J.nthreads = nthreads;
    return run_prefill(&J);
}

/*
 * A sample of rows: unit u is (token row_tok[u], head row_head[u]).
 * o [n,D], lse [n], wsink [n] (may be NULL).
 */
int oracle_prefill_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const int32_t *cu_seqlens, int num_seqs, int Hq,
                        int Hkv, int D, int window, const double *sink,
                        double scale, const int64_t *row_tok,
                        const int32_t *row_head, int64_t nrows, double *o,
                        double *lse, double *wsink, int nthreads)
{
    if (check_common(cu_seqlens, num_seqs, Hq, Hkv, D))
        return -2;
    int64_t total = cu_seqlens[num_seqs];
    for (int64_t u = 0; u < nrows; ++u)
        if (row_tok[u] < 0 || row_tok[u] >= total || row_head[u] < 0 ||
            row_head[u] >= Hq)
            return -2;
    prefill_job J;
    memset(&J, 0, sizeof J);
    J.q = q; J.k = k; J.v = v;
    J.cu_seqlens = cu_seqlens; J.num_seqs = num_seqs;
    J.Hq = Hq; J.Hkv = Hkv; J.D = D; J.window = window;
    J.sink = sink; J.scale = scale;
    J.total = total;
    J.row_tok = row_tok; J.row_head = row_head; J.nunits = nrows;
    J.o = o; J.lse = lse; J.wsink = wsink;
    J.nthreads = nthreads;
    return run_prefill(&J);
}

/* ------------------------------------------------------------------------ */
/* decode / draft verification over a W-slot ring                            */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint16_t *q, *k_new, *v_new, *k_ring, *v_ring;
    const int32_t *pos;
    int B, n_q, Hq, Hkv, D, W;
    const double *sink;
    double scale;
    double *o, *lse, *wsink;
    int nthreads, tid;
} decode_job;

static void *decode_worker(void *arg)
{
    decode_job *J = (decode_job *)arg;
    int maxkeys = J->W + J->n_q;
    const uint16_t **kr = (const uint16_t **)malloc(sizeof(*kr) * maxkeys);
    const uint16_t **vr = (const uint16_t **)malloc(sizeof(*vr) * maxkeys);
    double *logit = (double *)malloc(sizeof(double) * maxkeys);
    const int G = J->Hq / J->Hkv;
    int64_t nunits = (int64_t)J->B * J->n_q * J->Hq;

    for (int64_t u = J->tid; u < nunits; u += J->nthreads) {
        int h = (int)(u % J->Hq);
        int t = (int)((u / J->Hq) % J->n_q);
        int b = (int)(u / ((int64_t)J->Hq * J->n_q));
        int g = h / G;
        int64_t P = J->pos[b];
        int64_t first = P + t - J->W + 1;
        if (first < 0)
            first = 0;
        int n = 0;
        /* committed tokens, in position order, from their ring slots */
        for (int64_t p = first; p <= P - 1; ++p, ++n) {
            int64_t slot = p % J->W;
            int64_t off = (((int64_t)b * J->W + slot) * J->Hkv + g) * J->D;
            kr[n] = J->k_ring + off;
            vr[n] = J->v_ring + off;
        }
        /* the new tokens 0..t */
        for (int uu = 0; uu <= t; ++uu, ++n) {
            int64_t off = (((int64_t)b * J->n_q + uu) * J->Hkv + g) * J->D;
            kr[n] = J->k_new + off;
            vr[n] = J->v_new + off;
        }
        double sh = J->sink ? J->sink[h] : -INFINITY;
        int64_t row = ((int64_t)b * J->n_q + t) * J->Hq + h;
        attend_row(J->q + row * J->D, kr, vr, n, J->D, sh, J->scale, logit,
                   J->o + row * J->D, J->lse + row,
                   J->wsink ? J->wsink + row : NULL);
    }
    free(kr);
    free(vr);
    free(logit);
    return NULL;
}

/*
 * q [B,n_q,Hq,D]; k_new/v_new [B,n_q,Hkv,D]; k_ring/v_ring [B,W,Hkv,D];
 * pos [B] (>= 0); o [B,n_q,Hq,D]; lse, wsink [B,n_q,Hq] (wsink may be NULL).
 */
int oracle_decode(const uint16_t *q, const uint16_t *k_new,
                  const uint16_t *v_new, const uint16_t *k_ring,
                  const uint16_t *v_ring, const int32_t *pos, int B, int n_q,
                  int Hq, int Hkv, int D, int W, const double *sink,
                  double scale, double *o, double *lse, double *wsink,
                  int nthreads)
{
    if (B < 0 || n_q <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || W <= 0 ||
        Hq % Hkv)
        return -2;
    for (int b = 0; b < B; ++b)
        if (pos[b] < 0)
            return -2;
    int nt = nthreads < 1 ? 1 : nthreads;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nt);
    decode_job *jobs = (decode_job *)malloc(sizeof(decode_job) * nt);
    for (int t = 0; t < nt; ++t) {
        decode_job J = {q, k_new, v_new, k_ring, v_ring, pos, B, n_q, Hq, Hkv,
                        D, W, sink, scale, o, lse, wsink, nt, t};
        jobs[t] = J;
        pthread_create(&th[t], NULL, decode_worker, &jobs[t]);
    }
    for (int t = 0; t < nt; ++t)
        pthread_join(th[t], NULL);
    free(th);
    free(jobs);
    return 0;
}

/*
 * Commit accepted tokens into the ring: for u < n_accept[b], the new token at
 * absolute position pos[b]+u goes to slot (pos[b]+u) mod W. Rows are copied
 * bit for bit. Returns -2 if some n_accept[b] is outside [0, n_q].
 */
int oracle_kv_commit(uint16_t *k_ring, uint16_t *v_ring, const uint16_t *k_new,
                     const uint16_t *v_new, const int32_t *pos,
                     const int32_t *n_accept, int B, int n_q, int Hkv, int D,
                     int W)
{
    for (int b = 0; b < B; ++b)
        if (n_accept[b] < 0 || n_accept[b] > n_q || pos[b] < 0)
            return -2;
    for (int b = 0; b < B; ++b) {
        for (int u = 0; u < n_accept[b]; ++u) {
            int64_t slot = ((int64_t)pos[b] + u) % W;
            for (int g = 0; g < Hkv; ++g) {
                int64_t dst = (((int64_t)b * W + slot) * Hkv + g) * D;
                int64_t src = (((int64_t)b * n_q + u) * Hkv + g) * D;
                memcpy(k_ring + dst, k_new + src, sizeof(uint16_t) * D);
                memcpy(v_ring + dst, v_new + src, sizeof(uint16_t) * D);
            }
        }
    }
    return 0;
}
