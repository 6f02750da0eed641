/*
 * CPU oracle for grouped-query split-KV decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, fp64 definition
 * that the CUDA path is checked against.  It shares no code, header, table or
 * helper with the CUDA library; only the tests, the package's smoke check and
 * the benchmark's CPU-baseline leg load it.  Nothing on the product path may
 * call it.
 *
 * What it computes (kernbench "_attention_mesh_mlo.py", the decode kernel
 * `attention_mesh_mlo_kernel`: "One-shot local partial attention", the
 * bidirectional fan-out's merge of received triplets, and "Final normalize"):
 *
 *   For batch item b, query head h (group size G = h_q / h_kv, kv head
 *   g = floor(h / G)), keys j in [0, S_b):
 *       s_j = scale * sum_d q[b][h][d] * k[row(b, j)][g][d]
 *       M   = max_j s_j
 *       l   = sum_j exp(s_j - M)
 *       O   = (sum_j exp(s_j - M) * v[row(b, j)][g][:]) / l
 *   with row(b, j) = (S_0 + ... + S_{b-1}) + j  (packed ragged cache).
 *
 *   A partial over a key range R is the triplet (m, l, o):
 *       m = max_{j in R} s_j,  l = sum_{j in R} exp(s_j - m),
 *       o = sum_{j in R} exp(s_j - m) * v_j       (unnormalised)
 *   and an empty range gives (-inf, 0, 0).
 *
 *   Two triplets merge by the page's rule:
 *       m_c = max(m, m'),  l = l e^{m - m_c} + l' e^{m' - m_c},
 *       o = o e^{m - m_c} + o' e^{m' - m_c},  m = m_c
 *   and the result is o / l.
 *
 * Readings where the page is silent or garbled:
 *   - o is the UNNORMALISED sum exp(s - m) v: the page's final o / l is only
 *     exact under this reading.
 *   - GQA mapping is contiguous: q head h reads kv head floor(h * h_kv / h_q)
 *     (tinygrad "llama speed tracking", Attention.__call__, which shards q by
 *     n_rep * head_dim next to k/v by head_dim).
 *   - The logits carry a `scale` factor (the page applies none).
 *   - An empty range is (-inf, 0, 0); merging skips such a triplet, and a
 *     row whose every range is empty has output 0.
 *   - Split i of a sequence of length S covers [i*L, min((i+1)*L, S)) with
 *     L = ceil(S / n_splits), or L = chunk_len in chunked mode.
 *
 * Prefill (causal, every position of a sequence is a query): query i of
 * sequence b (q row S_0 + ... + S_{b-1} + i) attends keys j <= i of the same
 * sequence -- the definition above with S_b replaced by i + 1.
 *
 * Everything is two-pass and unsplit: logits are stored, the maximum is taken,
 * then exponentials and sums are formed in fp64 from the exact fp64 values of
 * the stored fp32 / bf16 inputs.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

/* Exact value of element i of a fp32 or bf16 array (bf16 = top 16 bits of a
 * fp32 bit pattern). */
static double elem(const void *base, int64_t i, int dtype) {
    float f;
    if (dtype == ORACLE_BF16) {
        uint32_t u = ((uint32_t)((const uint16_t *)base)[i]) << 16;
        memcpy(&f, &u, sizeof f);
    } else {
        f = ((const float *)base)[i];
    }
    return (double)f;
}

typedef struct {
    const void *q, *k, *v;
    const int32_t *seqlens;
    const int64_t *row_off; /* packed row offset of each sequence */
    int B, h_q, h_kv, d, dtype;
    int causal;             /* prefill: q holds every position; items are (b, h, i) */
    double scale;
    /* split policy: n_splits > 0 -> L = ceil(S/n_splits); else chunk_len */
    int n_splits, chunk_len, n_out_splits;
} problem;

/* Logit s_j for query (b, h) -- at position i of the sequence when causal --
 * and key j of sequence b. */
static double logit_at(const problem *p, int b, int h, int64_t i, int64_t j) {
    int G = p->h_q / p->h_kv;
    int g = h / G;
    int64_t qrow = p->causal ? p->row_off[b] + i : (int64_t)b;
    int64_t qi = (qrow * p->h_q + h) * p->d;
    int64_t ki = ((p->row_off[b] + j) * p->h_kv + g) * p->d;
    double acc = 0.0;
    for (int t = 0; t < p->d; ++t)
        acc += elem(p->q, qi + t, p->dtype) * elem(p->k, ki + t, p->dtype);
    return p->scale * acc;
}

static double logit(const problem *p, int b, int h, int64_t j) { return logit_at(p, b, h, 0, j); }

/* Triplet of (b, h) over keys [lo, hi): the plain two-pass definition.
 * Writes m, l and o[0..d). */
static void range_triplet_at(const problem *p, int b, int h, int64_t i, int64_t lo, int64_t hi,
                             double *s_buf, double *m_out, double *l_out, double *o_out) {
    int G = p->h_q / p->h_kv;
    int g = h / G;
    for (int t = 0; t < p->d; ++t) o_out[t] = 0.0;
    if (hi <= lo) {
        *m_out = -INFINITY;
        *l_out = 0.0;
        return;
    }
    /* pass 1: logits and their maximum */
    double M = -INFINITY;
    for (int64_t j = lo; j < hi; ++j) {
        double s = logit_at(p, b, h, i, j);
        s_buf[j - lo] = s;
        if (s > M) M = s;
    }
    /* pass 2: exponentials, denominator, unnormalised weighted sum of V */
    double l = 0.0;
    for (int64_t j = lo; j < hi; ++j) {
        double w = exp(s_buf[j - lo] - M);
        l += w;
        int64_t vi = ((p->row_off[b] + j) * p->h_kv + g) * p->d;
        for (int t = 0; t < p->d; ++t) o_out[t] += w * elem(p->v, vi + t, p->dtype);
    }
    *m_out = M;
    *l_out = l;
}

static void range_triplet(const problem *p, int b, int h, int64_t lo, int64_t hi,
                          double *s_buf, double *m_out, double *l_out, double *o_out) {
    range_triplet_at(p, b, h, 0, lo, hi, s_buf, m_out, l_out, o_out);
}

/* ---- work distribution over (b, h) items ------------------------------ */

typedef struct {
    const problem *p;
    const int32_t *items; /* pairs (b, h) */
    int n_items;
    int next;             /* shared cursor */
    pthread_mutex_t lock;
    int mode;             /* 0 = full attention, 1 = partials, 2 = causal prefill */
    double *out;          /* mode 0: [n_items][d] */
    double *m, *l, *o;    /* mode 1: [n_items][n_out_splits](x d) */
    int64_t max_len;
} job;

static int take(job *jb) {
    pthread_mutex_lock(&jb->lock);
    int i = jb->next++;
    pthread_mutex_unlock(&jb->lock);
    return i < jb->n_items ? i : -1;
}

/* Key range of split i of a sequence of length S under the split policy. */
static void split_range(const problem *p, int64_t S, int i, int64_t *lo, int64_t *hi) {
    int64_t L = p->n_splits > 0 ? (S + p->n_splits - 1) / p->n_splits : p->chunk_len;
    int64_t a = (int64_t)i * L, e = a + L;
    if (a > S) a = S;
    if (e > S) e = S;
    *lo = a;
    *hi = e;
}

static void *worker(void *arg) {
    job *jb = (job *)arg;
    const problem *p = jb->p;
    double *s_buf = (double *)malloc(sizeof(double) * (size_t)(jb->max_len > 0 ? jb->max_len : 1));
    double *o_tmp = (double *)malloc(sizeof(double) * (size_t)p->d);
    int it;
    while ((it = take(jb)) >= 0) {
        if (jb->mode == 2) {
            int b = jb->items[3 * it], h = jb->items[3 * it + 1], i = jb->items[3 * it + 2];
            double m, l;
            range_triplet_at(p, b, h, i, 0, (int64_t)i + 1, s_buf, &m, &l, o_tmp);
            double *dst = jb->out + (int64_t)it * p->d;
            for (int t = 0; t < p->d; ++t) dst[t] = o_tmp[t] / l;
            continue;
        }
        int b = jb->items[2 * it], h = jb->items[2 * it + 1];
        int64_t S = p->seqlens[b];
        if (jb->mode == 0) {
            double m, l;
            range_triplet(p, b, h, 0, S, s_buf, &m, &l, o_tmp);
            double *dst = jb->out + (int64_t)it * p->d;
            for (int t = 0; t < p->d; ++t) dst[t] = l > 0.0 ? o_tmp[t] / l : 0.0;
        } else {
            for (int i = 0; i < p->n_out_splits; ++i) {
                int64_t lo, hi;
                split_range(p, S, i, &lo, &hi);
                int64_t r = (int64_t)it * p->n_out_splits + i;
                range_triplet(p, b, h, lo, hi, s_buf, jb->m + r, jb->l + r, jb->o + r * p->d);
            }
        }
    }
    free(s_buf);
    free(o_tmp);
    return NULL;
}

static int run(problem *p, const int32_t *items, int n_items, int nthreads, int mode,
               double *out, double *m, double *l, double *o) {
    if (p->h_kv <= 0 || p->h_q % p->h_kv != 0 || p->d <= 0 || p->B < 0) return 1;
    int64_t *row_off = (int64_t *)malloc(sizeof(int64_t) * (size_t)(p->B + 1));
    int64_t max_len = 0, acc = 0;
    for (int b = 0; b < p->B; ++b) {
        if (p->seqlens[b] < 0) { free(row_off); return 1; }
        row_off[b] = acc;
        acc += p->seqlens[b];
        if (p->seqlens[b] > max_len) max_len = p->seqlens[b];
    }
    row_off[p->B] = acc;
    p->row_off = row_off;
    for (int i = 0; i < n_items; ++i) {
        int w = mode == 2 ? 3 : 2;
        int b = items[w * i], h = items[w * i + 1];
        if (b < 0 || b >= p->B || h < 0 || h >= p->h_q) { free(row_off); return 1; }
        if (mode == 2 && (items[3 * i + 2] < 0 || items[3 * i + 2] >= p->seqlens[b])) {
            free(row_off);
            return 1;
        }
    }
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n_items) nthreads = n_items > 0 ? n_items : 1;

    job jb;
    jb.p = p; jb.items = items; jb.n_items = n_items; jb.next = 0; jb.mode = mode;
    jb.out = out; jb.m = m; jb.l = l; jb.o = o; jb.max_len = max_len;
    pthread_mutex_init(&jb.lock, NULL);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, worker, &jb);
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    pthread_mutex_destroy(&jb.lock);
    free(row_off);
    return 0;
}

/* Full attention output O[it][d] (fp64) for each listed (b, h) pair.
 * q: [B][h_q][d]; k, v: [sum S_b][h_kv][d] packed; dtype 0 = fp32, 1 = bf16.
 * Returns 0, or 1 on bad arguments.  nthreads <= 0 uses every online core. */
int oracle_attn(const void *q, const void *k, const void *v, const int32_t *seqlens,
                int B, int h_q, int h_kv, int d, double scale, int dtype,
                const int32_t *items, int n_items, int nthreads, double *out) {
    problem p;
    memset(&p, 0, sizeof p);
    p.q = q; p.k = k; p.v = v; p.seqlens = seqlens;
    p.B = B; p.h_q = h_q; p.h_kv = h_kv; p.d = d; p.dtype = dtype; p.scale = scale;
    return run(&p, items, n_items, nthreads, 0, out, NULL, NULL, NULL);
}

/* Partial triplets for each listed (b, h) and each of n_out_splits splits.
 * Split policy: n_splits > 0 gives L_b = ceil(S_b / n_splits); otherwise
 * chunk_len > 0 gives fixed chunks (the last one partial, later ones empty).
 * m, l: [n_items][n_out_splits]; o: [n_items][n_out_splits][d]. */
int oracle_partials(const void *q, const void *k, const void *v, const int32_t *seqlens,
                    int B, int h_q, int h_kv, int d, double scale, int dtype,
                    int n_splits, int chunk_len, int n_out_splits,
                    const int32_t *items, int n_items, int nthreads,
                    double *m, double *l, double *o) {
    if (n_splits <= 0 && chunk_len <= 0) return 1;
    if (n_out_splits <= 0) return 1;
    problem p;
    memset(&p, 0, sizeof p);
    p.q = q; p.k = k; p.v = v; p.seqlens = seqlens;
    p.B = B; p.h_q = h_q; p.h_kv = h_kv; p.d = d; p.dtype = dtype; p.scale = scale;
    p.n_splits = n_splits; p.chunk_len = chunk_len; p.n_out_splits = n_out_splits;
    return run(&p, items, n_items, nthreads, 1, NULL, m, l, o);
}

/* Merge n triplets per row with the page's pairwise rule, in split order,
 * then normalise.  m, l: [rows][n]; o: [rows][n][d]; out: [rows][d].
 * A triplet with m = -inf (empty range) contributes nothing; a row with no
 * non-empty triplet gets 0. */
void oracle_merge(const double *m, const double *l, const double *o,
                  int rows, int n, int d, double *out) {
    double *acc = (double *)malloc(sizeof(double) * (size_t)(d > 0 ? d : 1));
    for (int r = 0; r < rows; ++r) {
        double M = -INFINITY, L = 0.0;
        for (int t = 0; t < d; ++t) acc[t] = 0.0;
        for (int i = 0; i < n; ++i) {
            int64_t idx = (int64_t)r * n + i;
            double mi = m[idx];
            if (mi == -INFINITY) continue;
            const double *oi = o + idx * d;
            if (M == -INFINITY) {
                M = mi;
                L = l[idx];
                for (int t = 0; t < d; ++t) acc[t] = oi[t];
                continue;
            }
            double mc = M > mi ? M : mi;
            double a = exp(M - mc), bw = exp(mi - mc);
            L = L * a + l[idx] * bw;
            for (int t = 0; t < d; ++t) acc[t] = acc[t] * a + oi[t] * bw;
            M = mc;
        }
        for (int t = 0; t < d; ++t) out[(int64_t)r * d + t] = L > 0.0 ? acc[t] / L : 0.0;
    }
    free(acc);
}

/* Causal prefill output O[it][d] (fp64) for each listed (b, h, i): query i of
 * sequence b, head h, over keys 0..i of that sequence.  q, k, v: packed
 * [sum S_b][heads][d] (q with h_q heads, k and v with h_kv).  Returns 0, or 1
 * on bad arguments. */
int oracle_prefill(const void *q, const void *k, const void *v, const int32_t *seqlens,
                   int B, int h_q, int h_kv, int d, double scale, int dtype,
                   const int32_t *items, int n_items, int nthreads, double *out) {
    problem p;
    memset(&p, 0, sizeof p);
    p.q = q; p.k = k; p.v = v; p.seqlens = seqlens;
    p.B = B; p.h_q = h_q; p.h_kv = h_kv; p.d = d; p.dtype = dtype; p.scale = scale;
    p.causal = 1;
    return run(&p, items, n_items, nthreads, 2, out, NULL, NULL, NULL);
}
