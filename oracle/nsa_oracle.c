/*
 * nsa_oracle.c -- TEST INFRASTRUCTURE, not part of the product path.
 *
 * Plain, slow fp64 CPU reference for Native Sparse Attention's selected-block
 * attention.  Only the tests, the smoke check and the benchmark's CPU-baseline leg
 * may call it.  It shares no code, header or table with the CUDA library.
 *
 * What it computes (one definition per function, written out with no blocking or
 * reordering beyond the loops that the definition itself states):
 *
 *   For a packed batch of sequences (cu_seqlens, "Flash-Sparse-Attention" project
 *   page, quick-start section), token t of sequence s (offset c_s, length L_s,
 *   local position i, query block qb = floor(i / bs)) and query head h of KV head
 *   group g = floor(h / G), G = hq / hkv (GQA sharing, same page, introduction):
 *
 *     Sel(t, g) = { b = block_idx[t, g, j] : 0 <= b < NB_s }  (a set; -1 pads)
 *     J(t, g)   = { j : floor(j / bs) in Sel(t, g), 0 <= j <= i }  (causal)
 *                 and, with a sliding window W > 0, also j > i - W (the module's
 *                 window_size of the project page's quick start: a query sees the W
 *                 most recent positions, itself included)
 *     s_j       = scale * <q[t, h], k[c_s + j, g]>
 *     LSE       = log sum_{j in J} exp(s_j)   (computed as m + log sum exp(s_j - m))
 *     p_j       = exp(s_j - LSE)
 *     O[t, h]   = sum_{j in J} p_j v[c_s + j, g]
 *   An empty J gives O = 0 and LSE = -inf.
 *
 *   Backward of the loss sum(dO * O), with the oracle's own fp64 O:
 *     dP_j = <dO[t,h], v_j>,  D = <dO[t,h], O[t,h]>,  dS_j = p_j (dP_j - D)
 *     dQ[t,h] = scale sum_j dS_j k_j
 *     dK[key j, g] += scale dS_j q[t,h],   dV[key j, g] += p_j dO[t,h]
 *
 *   Block-index inversion: for KV head g and global block B = (sum of NB over
 *   earlier sequences) + b, the list of entries t * 64 + j (global token t,
 *   slot j) with block_idx[t, g, j] = b and 0 <= b <= qb(t), ascending in t
 *   (then j).  Offsets are the exclusive prefix sum over (g major, B minor).
 *   This is the "swap the outer and inner loops" view of selected attention
 *   that the FSA pages describe (FSA blog page, second paragraph; project page,
 *   "Why it matters" section): a per-KV-block list of the query rows that use it.
 *
 * Inputs q, k, v, dout are float32 arrays holding bfloat16 values; they are
 * widened to double on use.  Layouts: q, dout [T, hq, d]; k, v [T, hkv, d];
 * block_idx int32 [T, hkv, topk]; cu_seqlens int32 [nseq + 1].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2
#define ORACLE_ERR_CAP 3

typedef struct {
    const float *q, *k, *v;
    const int32_t *cu;
    int nseq, hq, hkv, d, topk, bs;
    const int32_t *bidx;
    double scale;
    int64_t window;     /* 0: none; else keys j > i - window only */
} problem_t;

static int seq_of(const problem_t *P, int64_t t) {
    int lo = 0, hi = P->nseq - 1;
    while (lo < hi) {               /* last s with cu[s] <= t */
        int mid = (lo + hi + 1) / 2;
        if (P->cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

/* Marks the keys of J(t, g) in allowed[0..i]; returns i (local position). */
static int64_t selected_keys(const problem_t *P, int64_t t, int g, unsigned char *allowed,
                             unsigned char *blocksel, int64_t *c_out) {
    int s = seq_of(P, t);
    int64_t c = P->cu[s];
    int64_t L = (int64_t)P->cu[s + 1] - c;
    int64_t i = t - c;
    int64_t NB = (L + P->bs - 1) / P->bs;
    memset(blocksel, 0, (size_t)NB);
    for (int j = 0; j < P->topk; ++j) {
        int32_t b = P->bidx[(t * P->hkv + g) * P->topk + j];
        if (b >= 0 && b < NB) blocksel[b] = 1;
    }
    for (int64_t j = 0; j <= i; ++j)
        allowed[j] = blocksel[j / P->bs] && (P->window <= 0 || j > i - P->window);
    *c_out = c;
    return i;
}

static int64_t max_len(const problem_t *P) {
    int64_t m = 0;
    for (int s = 0; s < P->nseq; ++s) {
        int64_t L = (int64_t)P->cu[s + 1] - P->cu[s];
        if (L > m) m = L;
    }
    return m;
}

/* Softmax row of (t, h): fills p[0..i] (0 where not attended); returns LSE. */
static double softmax_row(const problem_t *P, int64_t t, int h, const unsigned char *allowed,
                          int64_t i, int64_t c, double *p) {
    int G = P->hq / P->hkv, g = h / G, d = P->d;
    const float *qr = P->q + (t * P->hq + h) * (int64_t)d;
    double m = -INFINITY;
    for (int64_t j = 0; j <= i; ++j) {
        if (!allowed[j]) { p[j] = 0.0; continue; }
        const float *kr = P->k + ((c + j) * P->hkv + g) * (int64_t)d;
        double acc = 0.0;
        for (int x = 0; x < d; ++x) acc += (double)qr[x] * (double)kr[x];
        p[j] = P->scale * acc;                  /* score for now */
        if (p[j] > m) m = p[j];
    }
    if (m == -INFINITY) return -INFINITY;       /* empty J */
    double l = 0.0;
    for (int64_t j = 0; j <= i; ++j)
        if (allowed[j]) l += exp(p[j] - m);
    double lse = m + log(l);
    for (int64_t j = 0; j <= i; ++j)
        p[j] = allowed[j] ? exp(p[j] - lse) : 0.0;
    return lse;
}

static int check_problem(const problem_t *P) {
    if (!P->q || !P->k || !P->v || !P->cu || !P->bidx) return ORACLE_ERR_ARG;
    if (P->nseq < 1 || P->hq < 1 || P->hkv < 1 || P->hq % P->hkv || P->d < 1 ||
        P->topk < 1 || P->bs < 1) return ORACLE_ERR_ARG;
    return ORACLE_OK;
}

#define MAKE_PROBLEM                                                                   \
    problem_t P = {q, k, v, cu_seqlens, nseq, hq, hkv, d, topk, block_size, block_idx, \
                   scale, window};                                                     \
    if (check_problem(&P)) return ORACLE_ERR_ARG;

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* Forward for the listed tokens (all tokens when tokens == NULL; then ntok must
 * equal T).  out [ntok, hq, d], lse [ntok, hq]. */
int nsa_oracle_fwd(const float *q, const float *k, const float *v, const int32_t *cu_seqlens,
                   int nseq, int hq, int hkv, int d, const int32_t *block_idx, int topk,
                   int block_size, double scale, const int64_t *tokens, int64_t ntok,
                   double *out, double *lse, int64_t window, int nthreads) {
    MAKE_PROBLEM
    int64_t Lmax = max_len(&P);
    int64_t NBmax = (Lmax + block_size - 1) / block_size;
    int err = ORACLE_OK;
    set_threads(nthreads);
#pragma omp parallel
    {
        unsigned char *allowed = (unsigned char *)malloc((size_t)Lmax + 1);
        unsigned char *blocksel = (unsigned char *)malloc((size_t)NBmax + 1);
        double *p = (double *)malloc(sizeof(double) * ((size_t)Lmax + 1));
        if (!allowed || !blocksel || !p) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
            int G = hq / hkv;
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < ntok * hkv; ++r) {
                int64_t n = r / hkv;
                int g = (int)(r % hkv);
                int64_t t = tokens ? tokens[n] : n;
                int64_t c;
                int64_t i = selected_keys(&P, t, g, allowed, blocksel, &c);
                for (int h = g * G; h < (g + 1) * G; ++h) {
                    double *o = out + (n * hq + h) * (int64_t)d;
                    double L = softmax_row(&P, t, h, allowed, i, c, p);
                    lse[n * hq + h] = L;
                    for (int x = 0; x < d; ++x) o[x] = 0.0;
                    if (L == -INFINITY) continue;
                    for (int64_t j = 0; j <= i; ++j) {
                        if (!allowed[j]) continue;
                        const float *vr = v + ((c + j) * hkv + g) * (int64_t)d;
                        for (int x = 0; x < d; ++x) o[x] += p[j] * (double)vr[x];
                    }
                }
            }
        }
        free(allowed);
        free(blocksel);
        free(p);
    }
    return err;
}

/* Per-row backward pieces shared by the backward entry points: for (t, h) with its
 * softmax row p[0..i], computes dP into dp[0..i] and returns D = <dO, O>. */
static double row_dp_and_D(const problem_t *P, const float *dout, int64_t t, int h,
                           const unsigned char *allowed, int64_t i, int64_t c,
                           const double *p, double *dp) {
    int G = P->hq / P->hkv, g = h / G, d = P->d;
    const float *dor = dout + (t * P->hq + h) * (int64_t)d;
    double D = 0.0;
    /* O in fp64, then D = <dO, O> */
    double *o = (double *)calloc((size_t)d, sizeof(double));
    for (int64_t j = 0; j <= i; ++j) {
        if (!allowed[j]) { dp[j] = 0.0; continue; }
        const float *vr = P->v + ((c + j) * P->hkv + g) * (int64_t)d;
        double acc = 0.0;
        for (int x = 0; x < d; ++x) {
            acc += (double)dor[x] * (double)vr[x];
            o[x] += p[j] * (double)vr[x];
        }
        dp[j] = acc;
    }
    for (int x = 0; x < d; ++x) D += (double)dor[x] * o[x];
    free(o);
    return D;
}

/* Full backward.  dq [T, hq, d], dk/dv [T, hkv, d] (all written). */
int nsa_oracle_bwd(const float *q, const float *k, const float *v, const float *dout,
                   const int32_t *cu_seqlens, int nseq, int hq, int hkv, int d,
                   const int32_t *block_idx, int topk, int block_size, double scale,
                   double *dq, double *dk, double *dv, int64_t window, int nthreads) {
    MAKE_PROBLEM
    if (!dout) return ORACLE_ERR_ARG;
    int64_t T = cu_seqlens[nseq];
    int64_t Lmax = max_len(&P);
    int64_t NBmax = (Lmax + block_size - 1) / block_size;
    int G = hq / hkv;
    int err = ORACLE_OK;
    size_t kvn = (size_t)T * hkv * d;
    memset(dk, 0, kvn * sizeof(double));
    memset(dv, 0, kvn * sizeof(double));
    set_threads(nthreads);
    int nth = 1;
#ifdef _OPENMP
    nth = omp_get_max_threads();
#endif
    double *pdk = (double *)calloc(kvn * (size_t)nth, sizeof(double));
    double *pdv = (double *)calloc(kvn * (size_t)nth, sizeof(double));
    if (!pdk || !pdv) { free(pdk); free(pdv); return ORACLE_ERR_NOMEM; }
#pragma omp parallel num_threads(nth)
    {
        int tid = 0;
#ifdef _OPENMP
        tid = omp_get_thread_num();
#endif
        double *mdk = pdk + kvn * (size_t)tid, *mdv = pdv + kvn * (size_t)tid;
        unsigned char *allowed = (unsigned char *)malloc((size_t)Lmax + 1);
        unsigned char *blocksel = (unsigned char *)malloc((size_t)NBmax + 1);
        double *p = (double *)malloc(sizeof(double) * ((size_t)Lmax + 1));
        double *dp = (double *)malloc(sizeof(double) * ((size_t)Lmax + 1));
        if (!allowed || !blocksel || !p || !dp) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t r = 0; r < T * hkv; ++r) {
                int64_t t = r / hkv;
                int g = (int)(r % hkv);
                int64_t c;
                int64_t i = selected_keys(&P, t, g, allowed, blocksel, &c);
                for (int h = g * G; h < (g + 1) * G; ++h) {
                    double *dqr = dq + (t * hq + h) * (int64_t)d;
                    for (int x = 0; x < d; ++x) dqr[x] = 0.0;
                    double L = softmax_row(&P, t, h, allowed, i, c, p);
                    if (L == -INFINITY) continue;
                    double D = row_dp_and_D(&P, dout, t, h, allowed, i, c, p, dp);
                    const float *qr = q + (t * hq + h) * (int64_t)d;
                    const float *dor = dout + (t * hq + h) * (int64_t)d;
                    for (int64_t j = 0; j <= i; ++j) {
                        if (!allowed[j]) continue;
                        double ds = p[j] * (dp[j] - D);
                        int64_t kr = ((c + j) * hkv + g) * (int64_t)d;
                        for (int x = 0; x < d; ++x) {
                            dqr[x] += scale * ds * (double)k[kr + x];
                            mdk[kr + x] += scale * ds * (double)qr[x];
                            mdv[kr + x] += p[j] * (double)dor[x];
                        }
                    }
                }
            }
        }
        free(allowed);
        free(blocksel);
        free(p);
        free(dp);
    }
    /* reduce the per-thread accumulators in thread order */
    for (int th = 0; th < nth; ++th)
        for (size_t e = 0; e < kvn; ++e) {
            dk[e] += pdk[kvn * (size_t)th + e];
            dv[e] += pdv[kvn * (size_t)th + e];
        }
    free(pdk);
    free(pdv);
    return err;
}

/* dQ for the listed tokens: dq [ntok, hq, d]. */
int nsa_oracle_bwd_dq(const float *q, const float *k, const float *v, const float *dout,
                      const int32_t *cu_seqlens, int nseq, int hq, int hkv, int d,
                      const int32_t *block_idx, int topk, int block_size, double scale,
                      const int64_t *tokens, int64_t ntok, double *dq, int64_t window,
                      int nthreads) {
    MAKE_PROBLEM
    if (!dout || !tokens) return ORACLE_ERR_ARG;
    int64_t Lmax = max_len(&P);
    int64_t NBmax = (Lmax + block_size - 1) / block_size;
    int G = hq / hkv;
    int err = ORACLE_OK;
    set_threads(nthreads);
#pragma omp parallel
    {
        unsigned char *allowed = (unsigned char *)malloc((size_t)Lmax + 1);
        unsigned char *blocksel = (unsigned char *)malloc((size_t)NBmax + 1);
        double *p = (double *)malloc(sizeof(double) * ((size_t)Lmax + 1));
        double *dp = (double *)malloc(sizeof(double) * ((size_t)Lmax + 1));
        if (!allowed || !blocksel || !p || !dp) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 4)
            for (int64_t r = 0; r < ntok * hkv; ++r) {
                int64_t n = r / hkv;
                int g = (int)(r % hkv);
                int64_t t = tokens[n];
                int64_t c;
                int64_t i = selected_keys(&P, t, g, allowed, blocksel, &c);
                for (int h = g * G; h < (g + 1) * G; ++h) {
                    double *dqr = dq + (n * hq + h) * (int64_t)d;
                    for (int x = 0; x < d; ++x) dqr[x] = 0.0;
                    double L = softmax_row(&P, t, h, allowed, i, c, p);
                    if (L == -INFINITY) continue;
                    double D = row_dp_and_D(&P, dout, t, h, allowed, i, c, p, dp);
                    for (int64_t j = 0; j <= i; ++j) {
                        if (!allowed[j]) continue;
                        double ds = p[j] * (dp[j] - D);
                        const float *kr = k + ((c + j) * hkv + g) * (int64_t)d;
                        for (int x = 0; x < d; ++x) dqr[x] += scale * ds * (double)kr[x];
                    }
                }
            }
        }
        free(allowed);
        free(blocksel);
        free(p);
        free(dp);
    }
    return err;
}

/* dK and dV of KV head g for keys [key0, key0 + nkeys), which must lie in one
 * sequence.  Every query row (t, h in group g) that attends one of those keys
 * contributes.  dk/dv [nkeys, d]. */
int nsa_oracle_bwd_dkdv_keys(const float *q, const float *k, const float *v, const float *dout,
                             const int32_t *cu_seqlens, int nseq, int hq, int hkv, int d,
                             const int32_t *block_idx, int topk, int block_size, double scale,
                             int g, int64_t key0, int nkeys, double *dk, double *dv,
                             int64_t window, int nthreads) {
    MAKE_PROBLEM
    if (!dout || g < 0 || g >= hkv || nkeys < 1) return ORACLE_ERR_ARG;
    int s = seq_of(&P, key0);
    int64_t c = cu_seqlens[s], cend = cu_seqlens[s + 1];
    if (key0 < c || key0 + nkeys > cend) return ORACLE_ERR_ARG;
    int64_t Lmax = max_len(&P);
    int64_t NBmax = (Lmax + block_size - 1) / block_size;
    int G = hq / hkv;
    int err = ORACLE_OK;
    set_threads(nthreads);
    int nth = 1;
#ifdef _OPENMP
    nth = omp_get_max_threads();
#endif
    size_t n = (size_t)nkeys * d;
    double *pdk = (double *)calloc(n * (size_t)nth, sizeof(double));
    double *pdv = (double *)calloc(n * (size_t)nth, sizeof(double));
    if (!pdk || !pdv) { free(pdk); free(pdv); return ORACLE_ERR_NOMEM; }
#pragma omp parallel num_threads(nth)
    {
        int tid = 0;
#ifdef _OPENMP
        tid = omp_get_thread_num();
#endif
        double *mdk = pdk + n * (size_t)tid, *mdv = pdv + n * (size_t)tid;
        unsigned char *allowed = (unsigned char *)malloc((size_t)Lmax + 1);
        unsigned char *blocksel = (unsigned char *)malloc((size_t)NBmax + 1);
        double *p = (double *)malloc(sizeof(double) * ((size_t)Lmax + 1));
        double *dp = (double *)malloc(sizeof(double) * ((size_t)Lmax + 1));
        if (!allowed || !blocksel || !p || !dp) {
#pragma omp atomic write
            err = ORACLE_ERR_NOMEM;
        } else {
#pragma omp for schedule(dynamic, 16)
            for (int64_t t = key0; t < cend; ++t) {
                int64_t cc;
                int64_t i = selected_keys(&P, t, g, allowed, blocksel, &cc);
                int any = 0;
                for (int64_t j = key0 - c; j < key0 - c + nkeys && j <= i; ++j) any |= allowed[j];
                if (!any) continue;
                for (int h = g * G; h < (g + 1) * G; ++h) {
                    double L = softmax_row(&P, t, h, allowed, i, c, p);
                    if (L == -INFINITY) continue;
                    double D = row_dp_and_D(&P, dout, t, h, allowed, i, c, p, dp);
                    const float *qr = q + (t * hq + h) * (int64_t)d;
                    const float *dor = dout + (t * hq + h) * (int64_t)d;
                    for (int64_t j = key0 - c; j < key0 - c + nkeys && j <= i; ++j) {
                        if (!allowed[j]) continue;
                        double ds = p[j] * (dp[j] - D);
                        int64_t o = (j - (key0 - c)) * d;
                        for (int x = 0; x < d; ++x) {
                            mdk[o + x] += scale * ds * (double)qr[x];
                            mdv[o + x] += p[j] * (double)dor[x];
                        }
                    }
                }
            }
        }
        free(allowed);
        free(blocksel);
        free(p);
        free(dp);
    }
    for (size_t e = 0; e < n; ++e) { dk[e] = 0.0; dv[e] = 0.0; }
    for (int th = 0; th < nth; ++th)
        for (size_t e = 0; e < n; ++e) {
            dk[e] += pdk[n * (size_t)th + e];
            dv[e] += pdv[n * (size_t)th + e];
        }
    free(pdk);
    free(pdv);
    return err;
}

/* Total number of blocks over all sequences. */
int64_t nsa_oracle_num_blocks(const int32_t *cu_seqlens, int nseq, int block_size) {
    int64_t nb = 0;
    for (int s = 0; s < nseq; ++s) {
        int64_t L = (int64_t)cu_seqlens[s + 1] - cu_seqlens[s];
        nb += (L + block_size - 1) / block_size;
    }
    return nb;
}

/* Block-index inversion (definition in the file header).  offsets has
 * hkv * NBtot + 1 entries; entries has room for cap values.  Returns the entry
 * count, or -1 on bad arguments, or -2 if cap is too small. */
int64_t nsa_oracle_invert(const int32_t *cu_seqlens, int nseq, int hkv, const int32_t *block_idx,
                          int topk, int block_size, int32_t *offsets, int32_t *entries,
                          int64_t cap) {
    if (!cu_seqlens || !block_idx || !offsets || nseq < 1 || hkv < 1 || topk < 1 ||
        topk > 64 || block_size < 1)
        return -1;
    int64_t NBtot = nsa_oracle_num_blocks(cu_seqlens, nseq, block_size);
    int64_t nbk = (int64_t)hkv * NBtot;
    int64_t *count = (int64_t *)calloc((size_t)nbk + 1, sizeof(int64_t));
    if (!count) return -1;
    /* blkoff[s]: global number of the first block of sequence s */
    int64_t *blkoff = (int64_t *)calloc((size_t)nseq + 1, sizeof(int64_t));
    for (int s = 0; s < nseq; ++s) {
        int64_t L = (int64_t)cu_seqlens[s + 1] - cu_seqlens[s];
        blkoff[s + 1] = blkoff[s] + (L + block_size - 1) / block_size;
    }
    /* pass 1: list lengths */
    for (int s = 0; s < nseq; ++s)
        for (int64_t t = cu_seqlens[s]; t < cu_seqlens[s + 1]; ++t) {
            int64_t qb = (t - cu_seqlens[s]) / block_size;
            for (int g = 0; g < hkv; ++g)
                for (int j = 0; j < topk; ++j) {
                    int32_t b = block_idx[(t * hkv + g) * topk + j];
                    if (b >= 0 && b <= qb) count[g * NBtot + blkoff[s] + b]++;
                }
        }
    /* offsets: exclusive prefix sum, g major, global block minor */
    int64_t run = 0;
    for (int64_t e = 0; e < nbk; ++e) {
        offsets[e] = (int32_t)run;
        run += count[e];
    }
    offsets[nbk] = (int32_t)run;
    if (!entries || run > cap) {    /* count-only query, or no room */
        free(count);
        free(blkoff);
        return entries ? -2 : run;
    }
    /* pass 2: append in ascending (t, j) order, so each list is sorted by t */
    for (int64_t e = 0; e < nbk; ++e) count[e] = offsets[e];
    for (int s = 0; s < nseq; ++s)
        for (int64_t t = cu_seqlens[s]; t < cu_seqlens[s + 1]; ++t) {
            int64_t qb = (t - cu_seqlens[s]) / block_size;
            for (int g = 0; g < hkv; ++g)
                for (int j = 0; j < topk; ++j) {
                    int32_t b = block_idx[(t * hkv + g) * topk + j];
                    if (b >= 0 && b <= qb)
                        entries[count[g * NBtot + blkoff[s] + b]++] = (int32_t)(t * 64 + j);
                }
        }
    free(count);
    free(blkoff);
    return run;
}
