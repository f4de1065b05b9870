/*
 * CPU oracle for the ROSA retrieval step -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the smoke check and the benchmark's CPU-baseline leg
 * may load this file's library.  It shares no code, header, table or helper
 * with the CUDA path and is deliberately plain and slow.
 *
 * Source: "ROSA-Tuning: Enhancing Windowed Attention with Global Recall"
 * (arXiv 2602.02499), the pages cited below by section / equation:
 *
 *   section 3.2, Eqs. (10)-(15)   binary discretisation q_bit = I[q_vec > 0]
 *                                  and multi-route packing a = sum_j bit_(r,j) 2^j
 *   section 4.1                    routes of M consecutive channels, R = C / M
 *   section 3.3, Eq. (16)          retrieval destination tau in {-1, 0, .., t-1}
 *                                  from k_{1:t} and q_{1:t}, read strictly from
 *                                  the past
 *   section 2.2                    suffix automaton: <= 2n-1 states, amortised
 *                                  O(1) transitions and suffix-link jumps
 *   appendix B.3                   tau_t = endpos(s_t) + 1 when it exists, else -1
 *   appendix C.4, Eq. (17)         read-out of the value at tau, mask I[tau >= 0]
 *   section 3.5                    counterfactual branches: each query bit forced
 *                                  to 0 and to 1, one retrieval step each from
 *                                  the same historical state
 *   section 3.3 (folding)          adjacent folding of repeated symbols into
 *                                  runs; the hit maps to the start of the next
 *                                  run (oracle_match_rle_*)
 *   appendix C.3, Eqs. (21)-(22)   read-out embedding y = m((1-b)e0 + b e1) and
 *                                  injection inj = W_out y (oracle_inject)
 *   section 3.2 (before Eq. 10)    U = LN(H), Q = U W_q, K = U W_k before the
 *                                  threshold (oracle_ln_project)
 *
 * Readings taken where the pages are garbled or silent (Eq. 16 itself is lost
 * in the page text):
 *   - causal lag g >= 1: a key end i is admissible at query time t iff
 *     i <= t - g; the default g = 2 gives tau = i + 1 <= t - 1, the range the
 *     section 3.3 text keeps; the restriction applies before maximising.
 *   - among admissible ends with the maximal match length, the most recent
 *     (largest) i is taken.
 *   - a match of length 0 never counts: tau = -1, len = 0, sym = -1.
 *   - the recalled symbol is v[i + 1] (v defaults to the key stream k).
 *
 * Two matchers are given.  oracle_match_brute is the definition written out
 * (O(T^2) per stream).  oracle_match_sam is the method the pages name: an
 * online suffix automaton over the key stream, advanced in lockstep with the
 * query stream.  The two share nothing but the output convention.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <pthread.h>

#define ORACLE_OK 0
#define ORACLE_ERR_ARG 1
#define ORACLE_ERR_NOMEM 2

/* ------------------------------------------------------------------------ */
/* Discretisation: section 3.2, Eqs. (10)-(15); section 4.1 route layout.    */
/* ------------------------------------------------------------------------ */

static float bf16_bits_to_float(uint16_t h)
{
    uint32_t w = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return f;
}

/*
 * x: bf16 bit patterns, shape [B, T, C] row-major.
 * sym: uint8 output, shape [B, R, T] with R = C / M.
 * Channel c = r * M + j carries bit j (weight 2^j) of route r's symbol.
 */
int oracle_discretize(const uint16_t *x, int B, int T, int C, int M, uint8_t *sym)
{
    if (B < 0 || T < 0 || C < 1 || M < 1 || M > 8 || C % M != 0)
        return ORACLE_ERR_ARG;
    int R = C / M;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int r = 0; r < R; ++r) {
                unsigned a = 0;
                for (int j = 0; j < M; ++j) {
                    float xv = bf16_bits_to_float(x[((size_t)b * T + t) * C + (size_t)r * M + j]);
                    unsigned bit = (xv > 0.0f) ? 1u : 0u;   /* I[x > 0] */
                    a += bit << j;                            /* bit * 2^j */
                }
                sym[((size_t)b * R + r) * T + t] = (uint8_t)a;
            }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Matching by the definition (brute force).                                 */
/*                                                                           */
/* D(t, i) = q[t] == k[i] ? 1 + D(t-1, i-1) : 0   (D = 0 off the grid) is    */
/* the length of the longest common suffix of q[0..t] and k[0..i].           */
/* L_t = max over 0 <= i <= t-g of D(t, i); i*_t = largest such i with       */
/* D(t, i) = L_t when L_t > 0.                                               */
/* ------------------------------------------------------------------------ */

static int brute_stream(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                        int T, int g, int32_t *end_idx, int32_t *len, int32_t *sym)
{
    int32_t *prev = (int32_t *)calloc((size_t)T + 1, sizeof(int32_t));
    int32_t *cur = (int32_t *)calloc((size_t)T + 1, sizeof(int32_t));
    if (!prev || !cur) { free(prev); free(cur); return ORACLE_ERR_NOMEM; }
    for (int t = 0; t < T; ++t) {
        for (int i = 0; i < T; ++i) {
            if (q[t] == k[i])
                cur[i] = 1 + ((t > 0 && i > 0) ? prev[i - 1] : 0);
            else
                cur[i] = 0;
        }
        int best = 0, best_i = -1;
        for (int i = 0; i <= t - g; ++i) {
            if (cur[i] > 0 && cur[i] >= best) {   /* ">=": later i wins ties */
                best = cur[i];
                best_i = i;
            }
        }
        end_idx[t] = best_i;
        len[t] = best;
        sym[t] = (best_i >= 0) ? (int32_t)v[best_i + 1] : -1;
        int32_t *tmp = prev; prev = cur; cur = tmp;
    }
    free(prev);
    free(cur);
    return ORACLE_OK;
}

int oracle_match_brute(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                       int S, int T, int g,
                       int32_t *end_idx, int32_t *len, int32_t *sym)
{
    if (S < 0 || T < 0 || g < 1 || !q || !k) return ORACLE_ERR_ARG;
    if (!v) v = k;
    for (int s = 0; s < S; ++s) {
        size_t o = (size_t)s * T;
        int rc = brute_stream(q + o, k + o, v + o, T, g, end_idx + o, len + o, sym + o);
        if (rc) return rc;
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Matching with an online suffix automaton (section 2.2; appendix B.3).      */
/*                                                                           */
/* State fields: len (longest string of the state), link (suffix link),      */
/* last_end (largest end position, among the keys inserted so far, of the     */
/* strings of the state), and a singly linked list of outgoing transitions.  */
/* ------------------------------------------------------------------------ */

typedef struct {
    int32_t *len, *link, *last_end, *edge_head;   /* per state */
    int32_t *edge_next, *edge_to;                 /* per edge */
    uint8_t *edge_sym;
    int n_states, n_edges, cap_states, cap_edges;
    int last;                                     /* state of the whole key prefix */
} sam_t;

static int sam_init(sam_t *a, int T)
{
    a->cap_states = 2 * T + 2;      /* <= 2n - 1 states, plus the root */
    a->cap_edges = 3 * T + 4;       /* <= 3n - 4 transitions for n >= 3 */
    a->len = (int32_t *)malloc(sizeof(int32_t) * a->cap_states);
    a->link = (int32_t *)malloc(sizeof(int32_t) * a->cap_states);
    a->last_end = (int32_t *)malloc(sizeof(int32_t) * a->cap_states);
    a->edge_head = (int32_t *)malloc(sizeof(int32_t) * a->cap_states);
    a->edge_next = (int32_t *)malloc(sizeof(int32_t) * a->cap_edges);
    a->edge_to = (int32_t *)malloc(sizeof(int32_t) * a->cap_edges);
    a->edge_sym = (uint8_t *)malloc(a->cap_edges);
    if (!a->len || !a->link || !a->last_end || !a->edge_head ||
        !a->edge_next || !a->edge_to || !a->edge_sym)
        return ORACLE_ERR_NOMEM;
    a->n_states = 1;
    a->n_edges = 0;
    a->len[0] = 0;
    a->link[0] = -1;
    a->last_end[0] = -1;
    a->edge_head[0] = -1;
    a->last = 0;
    return ORACLE_OK;
}

static void sam_free(sam_t *a)
{
    free(a->len); free(a->link); free(a->last_end); free(a->edge_head);
    free(a->edge_next); free(a->edge_to); free(a->edge_sym);
}

/* Target of the transition (s, c), or -1. */
static int sam_get(const sam_t *a, int s, uint8_t c)
{
    for (int e = a->edge_head[s]; e >= 0; e = a->edge_next[e])
        if (a->edge_sym[e] == c) return a->edge_to[e];
    return -1;
}

/* Set (s, c) -> to, adding the edge if missing. */
static int sam_set(sam_t *a, int s, uint8_t c, int to)
{
    for (int e = a->edge_head[s]; e >= 0; e = a->edge_next[e])
        if (a->edge_sym[e] == c) { a->edge_to[e] = to; return ORACLE_OK; }
    if (a->n_edges >= a->cap_edges) return ORACLE_ERR_NOMEM;
    int e = a->n_edges++;
    a->edge_sym[e] = c;
    a->edge_to[e] = to;
    a->edge_next[e] = a->edge_head[s];
    a->edge_head[s] = e;
    return ORACLE_OK;
}

/*
 * Append key symbol c, which sits at key position p (Blumer et al.'s online
 * construction), then record p as the most recent end of every state whose
 * strings are suffixes of k[0..p]: those are the states on the suffix-link
 * path from the new state up to (not including) the root.
 */
static int sam_extend(sam_t *a, uint8_t c, int p)
{
    if (a->n_states + 2 > a->cap_states) return ORACLE_ERR_NOMEM;
    int cur = a->n_states++;
    a->len[cur] = a->len[a->last] + 1;
    a->link[cur] = 0;
    a->last_end[cur] = p;
    a->edge_head[cur] = -1;
    int x = a->last;
    while (x != -1 && sam_get(a, x, c) < 0) {
        if (sam_set(a, x, c, cur)) return ORACLE_ERR_NOMEM;
        x = a->link[x];
    }
    if (x != -1) {
        int y = sam_get(a, x, c);
        if (a->len[x] + 1 == a->len[y]) {
            a->link[cur] = y;
        } else {
            int cl = a->n_states++;
            a->len[cl] = a->len[x] + 1;
            a->link[cl] = a->link[y];
            a->last_end[cl] = a->last_end[y];
            a->edge_head[cl] = -1;
            for (int e = a->edge_head[y]; e >= 0; e = a->edge_next[e])
                if (sam_set(a, cl, a->edge_sym[e], a->edge_to[e])) return ORACLE_ERR_NOMEM;
            while (x != -1 && sam_get(a, x, c) == y) {
                if (sam_set(a, x, c, cl)) return ORACLE_ERR_NOMEM;
                x = a->link[x];
            }
            a->link[y] = cl;
            a->link[cur] = cl;
        }
    }
    a->last = cur;
    for (int s = cur; s > 0; s = a->link[s])
        a->last_end[s] = p;
    return ORACLE_OK;
}

/*
 * One stream, in lockstep over t = 0..T-1:
 *   1. if t - g >= 0, insert key symbol k[t-g] (the automaton then holds
 *      exactly the admissible keys k[0..t-g]);
 *   2. advance the matching state (state, L) with query symbol q[t]: follow
 *      suffix links until a transition on q[t] exists (or the root is left
 *      without one), then take it;
 *   3. emit (last_end(state), L) when L > 0.
 *
 * A clone made by step 1 may take over the shorter strings of the state the
 * matcher stands in.  Until the next insertion the clone has exactly the
 * transitions of that state and is its suffix link, so step 2 reaches the
 * same result from either: a missing transition leads through the clone to
 * the same suffix-link chain, a present one to the same target.
 */
static int sam_stream(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                      int T, int g, int32_t *end_idx, int32_t *len, int32_t *sym)
{
    sam_t a;
    int rc = sam_init(&a, T);
    if (rc) { sam_free(&a); return rc; }
    int st = 0, L = 0;
    for (int t = 0; t < T; ++t) {
        int p = t - g;
        if (p >= 0) {
            rc = sam_extend(&a, k[p], p);
            if (rc) { sam_free(&a); return rc; }
        }
        uint8_t c = q[t];
        while (st != 0 && sam_get(&a, st, c) < 0) {
            st = a.link[st];
            L = a.len[st];
        }
        int nx = sam_get(&a, st, c);
        if (nx >= 0) {
            st = nx;
            L += 1;
        } else {
            st = 0;
            L = 0;
        }
        if (L > 0) {
            int i = a.last_end[st];
            end_idx[t] = i;
            len[t] = L;
            sym[t] = (int32_t)v[i + 1];
        } else {
            end_idx[t] = -1;
            len[t] = 0;
            sym[t] = -1;
        }
    }
    sam_free(&a);
    return ORACLE_OK;
}

typedef struct {
    const uint8_t *q, *k, *v;
    int S, T, g, nthreads, tid;
    int32_t *end_idx, *len, *sym;
    int rc;
} sam_job_t;

static void *sam_worker(void *arg)
{
    sam_job_t *j = (sam_job_t *)arg;
    j->rc = ORACLE_OK;
    for (int s = j->tid; s < j->S; s += j->nthreads) {
        size_t o = (size_t)s * j->T;
        int rc = sam_stream(j->q + o, j->k + o, j->v + o, j->T, j->g,
                            j->end_idx + o, j->len + o, j->sym + o);
        if (rc) { j->rc = rc; break; }
    }
    return NULL;
}

/* All S streams ([S, T] row-major), streams spread over nthreads threads. */
int oracle_match_sam(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                     int S, int T, int g,
                     int32_t *end_idx, int32_t *len, int32_t *sym, int nthreads)
{
    if (S < 0 || T < 0 || g < 1 || !q || !k) return ORACLE_ERR_ARG;
    if (!v) v = k;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > S) nthreads = S > 0 ? S : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    sam_job_t *jobs = (sam_job_t *)malloc(sizeof(sam_job_t) * nthreads);
    if (!th || !jobs) { free(th); free(jobs); return ORACLE_ERR_NOMEM; }
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        sam_job_t jb = {q, k, v, S, T, g, nthreads, i, end_idx, len, sym, 0};
        jobs[i] = jb;
        if (i == 0) continue;
        if (pthread_create(&th[i], NULL, sam_worker, &jobs[i]) != 0) break;
        started = i;
    }
    sam_worker(&jobs[0]);
    int rc = jobs[0].rc;
    for (int i = 1; i <= started; ++i) {
        pthread_join(th[i], NULL);
        if (jobs[i].rc) rc = jobs[i].rc;
    }
    /* streams of threads that failed to start are done here */
    for (int i = started + 1; i < nthreads; ++i) {
        sam_worker(&jobs[i]);
        if (jobs[i].rc) rc = jobs[i].rc;
    }
    free(th);
    free(jobs);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Per-bit counterfactual destinations (section 3.5: each query bit is a     */
/* decision switch; the branches "force the bit to 0" and "force it to 1"    */
/* each take one retrieval step from the same historical state).             */
/*                                                                           */
/* For position t, bit j < M and beta in {0, 1}, the branch symbol is        */
/* c = (q[t] with bit j set to beta).  The history q[0..t-1] and the keys    */
/* are unchanged, so the branch's longest admissible match and most recent   */
/* end follow from D(t-1, .) alone:                                          */
/*   D'(t, i) = k[i] == c ? 1 + D(t-1, i-1) : 0,  L' = max_{i <= t-g} D',     */
/*   i*' = largest such i with D'(t, i) = L' when L' > 0, else -1.           */
/* Outputs end_cf, len_cf: [S, T, M, 2] int32, index beta last.              */
/* ------------------------------------------------------------------------ */

static int cf_brute_stream(const uint8_t *q, const uint8_t *k, int T, int M, int g,
                           int32_t *end_cf, int32_t *len_cf)
{
    int32_t *prev = (int32_t *)calloc((size_t)T + 1, sizeof(int32_t));   /* D(t-1, .) */
    int32_t *cur = (int32_t *)calloc((size_t)T + 1, sizeof(int32_t));
    if (!prev || !cur) { free(prev); free(cur); return ORACLE_ERR_NOMEM; }
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < M; ++j)
            for (int beta = 0; beta < 2; ++beta) {
                unsigned c = ((unsigned)q[t] & ~(1u << j)) | ((unsigned)beta << j);
                int best = 0, best_i = -1;
                for (int i = 0; i <= t - g; ++i) {
                    if (k[i] != c) continue;
                    int d = 1 + ((t > 0 && i > 0) ? prev[i - 1] : 0);
                    if (d >= best) { best = d; best_i = i; }   /* later i wins ties */
                }
                size_t o = (((size_t)t * M) + j) * 2 + beta;
                end_cf[o] = best_i;
                len_cf[o] = best;
            }
        /* advance D with the actual query symbol */
        for (int i = 0; i < T; ++i)
            cur[i] = (q[t] == k[i]) ? 1 + ((t > 0 && i > 0) ? prev[i - 1] : 0) : 0;
        int32_t *tmp = prev; prev = cur; cur = tmp;
    }
    free(prev);
    free(cur);
    return ORACLE_OK;
}

int oracle_match_cf_brute(const uint8_t *q, const uint8_t *k, int S, int T, int M, int g,
                          int32_t *end_cf, int32_t *len_cf)
{
    if (S < 0 || T < 0 || M < 1 || M > 8 || g < 1 || !q || !k) return ORACLE_ERR_ARG;
    for (int s = 0; s < S; ++s) {
        size_t o = (size_t)s * T;
        size_t oc = o * (size_t)M * 2;
        int rc = cf_brute_stream(q + o, k + o, T, M, g, end_cf + oc, len_cf + oc);
        if (rc) return rc;
    }
    return ORACLE_OK;
}

/*
 * The same with the suffix automaton: at each t, after inserting k[t-g],
 * every branch symbol is tried from the matching state (state, L) that the
 * actual step starts from, by the same transition rule, without moving it;
 * then the actual symbol q[t] advances the state as in sam_stream.
 */
static int cf_sam_stream(const uint8_t *q, const uint8_t *k, int T, int M, int g,
                         int32_t *end_cf, int32_t *len_cf)
{
    sam_t a;
    int rc = sam_init(&a, T);
    if (rc) { sam_free(&a); return rc; }
    int st = 0, L = 0;
    for (int t = 0; t < T; ++t) {
        int p = t - g;
        if (p >= 0) {
            rc = sam_extend(&a, k[p], p);
            if (rc) { sam_free(&a); return rc; }
        }
        for (int j = 0; j < M; ++j)
            for (int beta = 0; beta < 2; ++beta) {
                uint8_t c = (uint8_t)(((unsigned)q[t] & ~(1u << j)) | ((unsigned)beta << j));
                int s2 = st, L2 = L;
                while (s2 != 0 && sam_get(&a, s2, c) < 0) {
                    s2 = a.link[s2];
                    L2 = a.len[s2];
                }
                int nx = sam_get(&a, s2, c);
                if (nx >= 0) { s2 = nx; L2 += 1; } else { s2 = 0; L2 = 0; }
                size_t o = (((size_t)t * M) + j) * 2 + beta;
                end_cf[o] = L2 > 0 ? a.last_end[s2] : -1;
                len_cf[o] = L2;
            }
        uint8_t c = q[t];
        while (st != 0 && sam_get(&a, st, c) < 0) {
            st = a.link[st];
            L = a.len[st];
        }
        int nx = sam_get(&a, st, c);
        if (nx >= 0) { st = nx; L += 1; } else { st = 0; L = 0; }
    }
    sam_free(&a);
    return ORACLE_OK;
}

typedef struct {
    const uint8_t *q, *k;
    int S, T, M, g, nthreads, tid;
    int32_t *end_cf, *len_cf;
    int rc;
} cf_job_t;

static void *cf_worker(void *arg)
{
    cf_job_t *j = (cf_job_t *)arg;
    j->rc = ORACLE_OK;
    for (int s = j->tid; s < j->S; s += j->nthreads) {
        size_t o = (size_t)s * j->T;
        size_t oc = o * (size_t)j->M * 2;
        int rc = cf_sam_stream(j->q + o, j->k + o, j->T, j->M, j->g, j->end_cf + oc, j->len_cf + oc);
        if (rc) { j->rc = rc; break; }
    }
    return NULL;
}

int oracle_match_cf_sam(const uint8_t *q, const uint8_t *k, int S, int T, int M, int g,
                        int32_t *end_cf, int32_t *len_cf, int nthreads)
{
    if (S < 0 || T < 0 || M < 1 || M > 8 || g < 1 || !q || !k) return ORACLE_ERR_ARG;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > S) nthreads = S > 0 ? S : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    cf_job_t *jobs = (cf_job_t *)malloc(sizeof(cf_job_t) * nthreads);
    if (!th || !jobs) { free(th); free(jobs); return ORACLE_ERR_NOMEM; }
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        cf_job_t jb = {q, k, S, T, M, g, nthreads, i, end_cf, len_cf, 0};
        jobs[i] = jb;
        if (i == 0) continue;
        if (pthread_create(&th[i], NULL, cf_worker, &jobs[i]) != 0) break;
        started = i;
    }
    cf_worker(&jobs[0]);
    int rc = jobs[0].rc;
    for (int i = 1; i <= started; ++i) {
        pthread_join(th[i], NULL);
        if (jobs[i].rc) rc = jobs[i].rc;
    }
    for (int i = started + 1; i < nthreads; ++i) {
        cf_worker(&jobs[i]);
        if (jobs[i].rc) rc = jobs[i].rc;
    }
    free(th);
    free(jobs);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Run-level retrieval with adjacent folding (section 3.3, the run-length    */
/* encoding paragraph; appendix C.5-C.6 for the per-run bookkeeping).        */
/*                                                                           */
/* Consecutive equal symbols form one run.  Key runs: symbols c[l], start    */
/* times s[l]; query runs: symbols d[m], start times u[m].  The retrieval    */
/* state changes only at run boundaries, so the answer is taken once per     */
/* query run, at its start time u[m], and held for every t of the run.       */
/* A hit on key run l maps back to the time axis as the start of the next    */
/* key run, tau = s[l+1]; it must exist and satisfy tau <= u[m] - g + 1       */
/* (g = 2: tau <= t - 1, read strictly from the past), and this restriction  */
/* applies before maximising, as for the plain operator.  With              */
/*   D(m, l) = d[m] == c[l] ? 1 + D(m-1, l-1) : 0   (run-level common suffix) */
/* the run-level length is L_m = max over admissible l of D(m, l) and l* the */
/* largest admissible l reaching it (L_m > 0).  Outputs for t in run m:      */
/*   end_idx[t] = s[l*+1] - 1  (the last time index of run l*, so that       */
/*                              tau = end_idx + 1 as for the plain operator) */
/*   len[t]     = L_m          (in runs)                                     */
/*   sym[t]     = v[s[l*+1]]                                                 */
/* or (-1, 0, -1) when L_m = 0.  Without adjacent repeats every run is one   */
/* symbol long and this is the plain operator above.                        */
/* ------------------------------------------------------------------------ */

/* Runs of x[0..T): symbol and start time of each; returns their number. */
static int fold_runs(const uint8_t *x, int T, uint8_t *rsym, int32_t *rstart)
{
    int n = 0;
    for (int t = 0; t < T; ++t)
        if (t == 0 || x[t] != x[t - 1]) {
            rsym[n] = x[t];
            rstart[n] = t;
            ++n;
        }
    return n;
}

/* Writes run m's answer (key run lstar, run length L) to every t of the run. */
static void rle_emit(const int32_t *u, int nq, int T, const int32_t *s, const uint8_t *v,
                     int m, int lstar, int L, int32_t *end_idx, int32_t *len, int32_t *sym)
{
    int t1 = (m + 1 < nq) ? u[m + 1] : T;
    for (int t = u[m]; t < t1; ++t) {
        if (L > 0) {
            int tau = s[lstar + 1];
            end_idx[t] = tau - 1;
            len[t] = L;
            sym[t] = (int32_t)v[tau];
        } else {
            end_idx[t] = -1;
            len[t] = 0;
            sym[t] = -1;
        }
    }
}

typedef struct {
    uint8_t *d, *c;
    int32_t *u, *s;
    int nq, nk;
} runs_t;

static int runs_make(runs_t *r, const uint8_t *q, const uint8_t *k, int T)
{
    r->d = (uint8_t *)malloc((size_t)T + 1);
    r->c = (uint8_t *)malloc((size_t)T + 1);
    r->u = (int32_t *)malloc(sizeof(int32_t) * ((size_t)T + 1));
    r->s = (int32_t *)malloc(sizeof(int32_t) * ((size_t)T + 1));
    if (!r->d || !r->c || !r->u || !r->s) return ORACLE_ERR_NOMEM;
    r->nq = fold_runs(q, T, r->d, r->u);
    r->nk = fold_runs(k, T, r->c, r->s);
    return ORACLE_OK;
}

static void runs_free(runs_t *r)
{
    free(r->d); free(r->c); free(r->u); free(r->s);
}

/* Number of key runs admissible for a query run starting at time u0: runs l  */
/* with a successor whose start s[l+1] <= u0 - g + 1 (a prefix l = 0..n-1).   */
/* Counting resumes from `from`, a count already known to be admissible.     */
static int rle_admissible(const runs_t *r, int u0, int g, int from)
{
    int n = from;
    while (n + 1 < r->nk && r->s[n + 1] <= u0 - g + 1) ++n;
    return n;
}

static int rle_brute_stream(const uint8_t *q, const uint8_t *k, const uint8_t *v, int T, int g,
                            int32_t *end_idx, int32_t *len, int32_t *sym)
{
    runs_t r;
    int rc = runs_make(&r, q, k, T);
    int32_t *prev = (int32_t *)calloc((size_t)T + 1, sizeof(int32_t));
    int32_t *cur = (int32_t *)calloc((size_t)T + 1, sizeof(int32_t));
    if (rc || !prev || !cur) { runs_free(&r); free(prev); free(cur); return ORACLE_ERR_NOMEM; }
    for (int m = 0; m < r.nq; ++m) {
        for (int l = 0; l < r.nk; ++l)
            cur[l] = (r.d[m] == r.c[l]) ? 1 + ((m > 0 && l > 0) ? prev[l - 1] : 0) : 0;
        int nadm = rle_admissible(&r, r.u[m], g, 0);
        int best = 0, best_l = -1;
        for (int l = 0; l < nadm; ++l)
            if (cur[l] > 0 && cur[l] >= best) { best = cur[l]; best_l = l; }   /* later l wins ties */
        rle_emit(r.u, r.nq, T, r.s, v, m, best_l, best, end_idx, len, sym);
        int32_t *tmp = prev; prev = cur; cur = tmp;
    }
    runs_free(&r);
    free(prev);
    free(cur);
    return ORACLE_OK;
}

int oracle_match_rle_brute(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                           int S, int T, int g, int32_t *end_idx, int32_t *len, int32_t *sym)
{
    if (S < 0 || T < 0 || g < 1 || !q || !k) return ORACLE_ERR_ARG;
    if (!v) v = k;
    for (int s = 0; s < S; ++s) {
        size_t o = (size_t)s * T;
        int rc = rle_brute_stream(q + o, k + o, v + o, T, g, end_idx + o, len + o, sym + o);
        if (rc) return rc;
    }
    return ORACLE_OK;
}

/* One matching step of (state, L) with symbol c against automaton a. */
static void sam_step(const sam_t *a, int *st, int *L, uint8_t c)
{
    while (*st != 0 && sam_get(a, *st, c) < 0) {
        *st = a->link[*st];
        *L = a->len[*st];
    }
    int nx = sam_get(a, *st, c);
    if (nx >= 0) { *st = nx; *L += 1; } else { *st = 0; *L = 0; }
}

/*
 * The automaton form (section 3.3: the automaton runs over the run-level
 * key symbols and keeps the run start times).  The online automaton holds
 * exactly the key runs admissible so far, and the matching state (state, L)
 * is the longest suffix of the query runs seen so far that occurs in it.
 * Before query run m takes its matching step, the key runs that became
 * admissible since the previous query run enter one by one; each can only
 * add occurrences that end in itself, so after inserting run l the state is
 * raised to the suffix of length D (the run-level common suffix of the query
 * runs so far and the key runs 0..l, compared directly) when D >= L: that
 * suffix is a suffix of the whole key-run prefix, so its state lies on the
 * suffix-link chain of the newest state.  Then the query run's symbol takes
 * one ordinary matching step, and last_end of the state is the most recent
 * admissible key run l*.
 */
static int rle_sam_stream(const uint8_t *q, const uint8_t *k, const uint8_t *v, int T, int g,
                          int32_t *end_idx, int32_t *len, int32_t *sym)
{
    runs_t r;
    int rc = runs_make(&r, q, k, T);
    sam_t on;
    int ro = sam_init(&on, T);
    if (rc || ro) { runs_free(&r); sam_free(&on); return ORACLE_ERR_NOMEM; }
    int st = 0, L = 0, inserted = 0;
    for (int m = 0; m < r.nq && !rc; ++m) {
        int nadm = rle_admissible(&r, r.u[m], g, inserted);
        while (inserted < nadm && !rc) {
            int l = inserted++;
            rc = sam_extend(&on, r.c[l], l);
            if (rc) break;
            int D = 0;   /* common suffix of d[0..m-1] and c[0..l] */
            while (D < m && D <= l && r.d[m - 1 - D] == r.c[l - D]) ++D;
            if (D > 0 && D >= L) {
                int x = on.last;
                while (on.link[x] > 0 && on.len[on.link[x]] >= D) x = on.link[x];
                st = x;
                L = D;
            }
        }
        if (rc) break;
        sam_step(&on, &st, &L, r.d[m]);
        rle_emit(r.u, r.nq, T, r.s, v, m, L > 0 ? on.last_end[st] : -1, L, end_idx, len, sym);
    }
    runs_free(&r);
    sam_free(&on);
    return rc;
}

typedef int (*stream_fn_t)(const uint8_t *, const uint8_t *, const uint8_t *, int, int,
                           int32_t *, int32_t *, int32_t *);

typedef struct {
    stream_fn_t fn;
    const uint8_t *q, *k, *v;
    int S, T, g, nthreads, tid;
    int32_t *end_idx, *len, *sym;
    int rc;
} gen_job_t;

static void *gen_worker(void *arg)
{
    gen_job_t *j = (gen_job_t *)arg;
    j->rc = ORACLE_OK;
    for (int s = j->tid; s < j->S; s += j->nthreads) {
        size_t o = (size_t)s * j->T;
        int rc = j->fn(j->q + o, j->k + o, j->v + o, j->T, j->g, j->end_idx + o, j->len + o, j->sym + o);
        if (rc) { j->rc = rc; break; }
    }
    return NULL;
}

/* Streams ([S, T] row-major) spread over nthreads host threads. */
static int run_streams(stream_fn_t fn, const uint8_t *q, const uint8_t *k, const uint8_t *v,
                       int S, int T, int g, int32_t *end_idx, int32_t *len, int32_t *sym, int nthreads)
{
    if (nthreads < 1) nthreads = 1;
    if (nthreads > S) nthreads = S > 0 ? S : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    gen_job_t *jobs = (gen_job_t *)malloc(sizeof(gen_job_t) * nthreads);
    if (!th || !jobs) { free(th); free(jobs); return ORACLE_ERR_NOMEM; }
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        gen_job_t jb = {fn, q, k, v, S, T, g, nthreads, i, end_idx, len, sym, 0};
        jobs[i] = jb;
        if (i == 0) continue;
        if (pthread_create(&th[i], NULL, gen_worker, &jobs[i]) != 0) break;
        started = i;
    }
    gen_worker(&jobs[0]);
    int rc = jobs[0].rc;
    for (int i = 1; i <= started; ++i) {
        pthread_join(th[i], NULL);
        if (jobs[i].rc) rc = jobs[i].rc;
    }
    for (int i = started + 1; i < nthreads; ++i) {
        gen_worker(&jobs[i]);
        if (jobs[i].rc) rc = jobs[i].rc;
    }
    free(th);
    free(jobs);
    return rc;
}

int oracle_match_rle_sam(const uint8_t *q, const uint8_t *k, const uint8_t *v,
                         int S, int T, int g, int32_t *end_idx, int32_t *len, int32_t *sym, int nthreads)
{
    if (S < 0 || T < 0 || g < 1 || !q || !k) return ORACLE_ERR_ARG;
    if (!v) v = k;
    return run_streams(rle_sam_stream, q, k, v, S, T, g, end_idx, len, sym, nthreads);
}

/* ------------------------------------------------------------------------ */
/* Read-out of the value rows at tau (appendix C.4; mask of Eq. 17).         */
/*                                                                           */
/* out[b, t, r*d + m] = V[b, tau, r*rho + m] for m < d when tau >= 0, and 0  */
/* (all-zero bits) when tau = -1, where tau = end_idx[b*R + r, t] + 1.       */
/* V: [B, T, Cv] bf16 bits with row stride Cv; out: [B, T, R*d].             */
/* ------------------------------------------------------------------------ */

int oracle_gather(const uint16_t *V, int64_t v_row_stride, int64_t rho,
                  const int32_t *end_idx, int B, int R, int T, int d, uint16_t *out)
{
    if (B < 0 || R < 0 || T < 0 || d < 0 || rho < 0) return ORACLE_ERR_ARG;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t)
            for (int r = 0; r < R; ++r) {
                int32_t e = end_idx[((size_t)b * R + r) * T + t];
                int64_t tau = (int64_t)e + 1;
                uint16_t *dst = out + ((size_t)b * T + t) * ((size_t)R * d) + (size_t)r * d;
                if (e < 0) {
                    for (int m = 0; m < d; ++m) dst[m] = 0;
                } else {
                    const uint16_t *src = V + ((size_t)b * T + (size_t)tau) * (size_t)v_row_stride
                                            + (size_t)(r * rho);
                    for (int m = 0; m < d; ++m) dst[m] = src[m];
                }
            }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Read-out embedding and injection (appendix C.3; Eq. 17 mask).             */
/*                                                                           */
/* For position (b, t) and channel c = r*M + j of route r: the recalled bit  */
/* b^ = bit j of the recalled value symbol sym[b*R + r, t], the mask         */
/* m = I[tau >= 0] (sym = -1 when nothing matched), and                      */
/*   y[b, t, c]   = m * ((1 - b^) e0[c] + b^ e1[c])                          */
/*   inj[b, t, d] = sum_c W_out[d, c] * y[b, t, c]                           */
/* in double precision.  e0, e1: [C] bf16 bits; W_out: [D, C] bf16 bits,     */
/* row-major; out: [B, T, D] doubles.                                        */
/* ------------------------------------------------------------------------ */

int oracle_inject(const int32_t *sym, const uint16_t *e0, const uint16_t *e1, const uint16_t *W,
                  int B, int R, int M, int T, int D, double *out)
{
    if (B < 0 || R < 0 || T < 0 || D < 0 || M < 1 || M > 8) return ORACLE_ERR_ARG;
    int C = R * M;
    double *y = (double *)malloc(sizeof(double) * (C > 0 ? C : 1));
    if (!y) return ORACLE_ERR_NOMEM;
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < T; ++t) {
            for (int r = 0; r < R; ++r) {
                int32_t a = sym[((size_t)b * R + r) * T + t];
                for (int j = 0; j < M; ++j) {
                    int c = r * M + j;
                    if (a < 0) {
                        y[c] = 0.0;   /* m = 0 */
                    } else {
                        int bit = (a >> j) & 1;
                        double v0 = bf16_bits_to_float(e0[c]), v1 = bf16_bits_to_float(e1[c]);
                        y[c] = (1 - bit) * v0 + bit * v1;
                    }
                }
            }
            for (int d = 0; d < D; ++d) {
                double acc = 0.0;
                for (int c = 0; c < C; ++c)
                    acc += (double)bf16_bits_to_float(W[(size_t)d * C + c]) * y[c];
                out[((size_t)b * T + t) * D + d] = acc;
            }
        }
    free(y);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------ */
/* Layer norm and projection before the threshold (section 3.2).             */
/*                                                                           */
/* U = LN(H): per row, mu = mean(h), var = mean((h - mu)^2) (population),    */
/* u = gamma * (h - mu) / sqrt(var + eps) + beta; then the projection         */
/* P = U W with W: [D, N] (the query and key projections side by side), in   */
/* double precision.  Also returns, per entry, the magnitude                 */
/* A[row, n] = sum_k |u_k W[k, n]| that bounds how far a rounded evaluation  */
/* of P can stray.  H: [rows, D] bf16 bits; gamma, beta: [D] floats (NULL:   */
/* 1 and 0); out, mag: [rows, N] doubles.                                    */
/* ------------------------------------------------------------------------ */

int oracle_ln_project(const uint16_t *H, const float *gamma, const float *beta, const uint16_t *W,
                      int rows, int D, int N, double eps, double *out, double *mag)
{
    if (rows < 0 || D < 1 || N < 0 || eps < 0.0) return ORACLE_ERR_ARG;
    double *u = (double *)malloc(sizeof(double) * D);
    if (!u) return ORACLE_ERR_NOMEM;
    for (int i = 0; i < rows; ++i) {
        const uint16_t *h = H + (size_t)i * D;
        double mu = 0.0;
        for (int k = 0; k < D; ++k) mu += bf16_bits_to_float(h[k]);
        mu /= D;
        double var = 0.0;
        for (int k = 0; k < D; ++k) {
            double x = bf16_bits_to_float(h[k]) - mu;
            var += x * x;
        }
        var /= D;
        double rstd = 1.0 / sqrt(var + eps);
        for (int k = 0; k < D; ++k) {
            double g = gamma ? gamma[k] : 1.0, bb = beta ? beta[k] : 0.0;
            u[k] = g * (bf16_bits_to_float(h[k]) - mu) * rstd + bb;
        }
        for (int n = 0; n < N; ++n) {
            double acc = 0.0, a = 0.0;
            for (int k = 0; k < D; ++k) {
                double term = u[k] * bf16_bits_to_float(W[(size_t)k * N + n]);
                acc += term;
                a += fabs(term);
            }
            out[(size_t)i * N + n] = acc;
            if (mag) mag[(size_t)i * N + n] = a;
        }
    }
    free(u);
    return ORACLE_OK;
}
