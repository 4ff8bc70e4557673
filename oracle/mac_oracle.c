/*
 * mac_oracle.c -- plain fp64 CPU oracle of one MAC-Attention decode step.
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's
 * CPU-baseline leg are the only callers.  The CUDA library never links,
 * includes or calls anything in this directory, and this file uses nothing of
 * the CUDA library.
 *
 * Source: "MAC-Attention: a Match-Amend-Complete Scheme for Fast and Accurate
 * Attention Computation", page 1 (the abstract).  The abstract names three
 * stages and every function below cites the part it follows:
 *   Match    -- the current query is compared, before RoPE, by L2 distance
 *               with a short window of recent queries whose attention results
 *               can be reused;
 *   Amend    -- the reused attention is corrected by recomputing a small band
 *               of keys just before the match boundary;
 *   Complete -- fresh attention over the KV tail is combined with the
 *               corrected result by a numerically stable merge.
 * On a miss the step is plain decode attention over every key.
 *
 * Where the abstract is silent this file takes the plainest reading; each
 * reading is named where it is used:
 *   [mean-dist]   distance = mean over the G query heads of a KV head of the
 *                 per-head squared L2 distance of the pre-RoPE queries;
 *   [per-head]    with per-head matching every query head decides alone: its
 *                 distance is its own squared L2 distance (the mean over a
 *                 group of one), its own nearest entry, its own reuse
 *                 boundary; the keys a KV head serves are the union of its
 *                 query heads' ranges;
 *   [strict]      hit iff the smallest distance is < tau (strict), ties to the
 *                 more recent entry, NaN distances never match;
 *   [window]      the window is the W most recent previous decode steps of the
 *                 same sequence, per KV head; an entry is eligible only if its
 *                 position precedes the current one;
 *   [cut]         every step stores its prefix state over keys [0, c) with
 *                 c = max(0, p - b) (cut_mode 0: the band is the b keys
 *                 before p), or c = max(0, p + 1 - b) (cut_mode 1: the band
 *                 ends at p itself); on a hit the band [c_s, c_t) and the
 *                 tail [c_t, p_t] are recomputed with the current query;
 *   [rope]        keys in the cache are post-RoPE; the query is rotated here
 *                 with rotate-half pairs (i, i + D/2), inv_freq_i =
 *                 theta^(-2i/D), angle in fp64;
 *   [scale]       scores are q.k / sqrt(D), natural-log units;
 *   [bf16-ring]   with a bf16 window, an entry keeps its pre-RoPE query and the
 *                 normalised output o of its prefix state rounded to bf16
 *                 (round to nearest even, o first rounded to fp32, the
 *                 precision the output is computed in); m and l keep their
 *                 precision;
 *   [warm]        a window seeded from prefill holds, for each of the last n
 *                 prefill positions, its pre-RoPE query and its prefix state
 *                 over [0, c) with the query rotated at that position -- the
 *                 state a decode step at that position would have stored.
 *
 * Arithmetic is fp64 throughout; inputs are fp32 queries and bf16 keys and
 * values, read exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

typedef struct {
    int B, Hq, Hkv, D;
    int W, band;
    double tau;
    double rope_theta;
    int page_size;         /* 0: contiguous K/V [B][max_seq][Hkv][D] */
    int max_seq;           /* rows per sequence (contiguous) */
    int max_pages_per_seq; /* block table row length (paged: K/V [P][page][Hkv][D]) */
    int cut_mode;          /* [cut]: 0 or 1 */
    int per_head;          /* 0: one decision per KV head ([mean-dist]); 1: per query head ([per-head]) */
    int ring_bf16;         /* 1: entries keep q and o rounded to bf16 ([bf16-ring]) */
} ocfg_t;

typedef struct {
    ocfg_t c;
    int G, U;
    int *n;       /* [U] entries held, at most W */
    float *wq;    /* [U][W][G][D] pre-RoPE query of the entry (oldest first) */
    double *wo;   /* [U][W][G][D] normalised output of the stored prefix state */
    double *wm;   /* [U][W][G] max score of the stored prefix state */
    double *wl;   /* [U][W][G] sum of exp(score - m) of the stored prefix state */
    int *wpos;    /* [U][W] position of the entry's own token */
} ostate_t;

/* ---------------------------------------------------------------- inputs */

static double bf16_to_f64(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* [bf16-ring] The bf16 value nearest to x (ties to the even bf16), as a
 * float: keep the top 16 bits of the fp32 pattern after adding half a unit
 * of the 17th bit, plus one when the kept part is odd.  NaN stays NaN. */
static float round_bf16(float x) {
    uint32_t u;
    memcpy(&u, &x, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return x;
    u = (u + 0x7fffu + ((u >> 16) & 1u)) & 0xffff0000u;
    float r;
    memcpy(&r, &u, sizeof r);
    return r;
}

/* Row of key (or value) position k of sequence b, KV head kvh. */
static const uint16_t *kv_row(const ocfg_t *c, const uint16_t *base, const int *block_table,
                              int b, long k, int kvh) {
    size_t row;
    if (c->page_size == 0) {
        row = ((size_t)b * (size_t)c->max_seq + (size_t)k) * (size_t)c->Hkv + (size_t)kvh;
    } else {
        int page = block_table[(size_t)b * (size_t)c->max_pages_per_seq + (size_t)(k / c->page_size)];
        row = ((size_t)page * (size_t)c->page_size + (size_t)(k % c->page_size)) * (size_t)c->Hkv +
              (size_t)kvh;
    }
    return base + row * (size_t)c->D;
}

/* ------------------------------------------------------------------ RoPE */

/* [rope] Rotate a pre-RoPE query to position pos.  Pair i couples element i
 * with element i + D/2 and turns by pos * theta^(-2i/D) radians.  The match
 * stage uses the unrotated query (page 1: the match compares queries before RoPE); attention
 * uses the rotated one, since the cache holds rotated keys. */
void oracle_rope(const float *q, int D, long pos, double theta, double *out) {
    int half = D / 2;
    for (int i = 0; i < half; ++i) {
        double inv_freq = pow(theta, -2.0 * (double)i / (double)D);
        double ang = (double)pos * inv_freq;
        double cs = cos(ang), sn = sin(ang);
        double x = (double)q[i], y = (double)q[i + half];
        out[i] = x * cs - y * sn;
        out[i + half] = y * cs + x * sn;
    }
}

/* ---------------------------------------------------- attention partials */

/* Exact attention state of one query head over keys [x, y): m = max score,
 * l = sum exp(score - m), o = sum exp(score - m) v / l.  An empty range is the
 * empty state (m = -inf, l = 0, o = 0).  Two passes: scores, then weights. */
static void partial_view(const ocfg_t *c, const uint16_t *K, const uint16_t *V, const int *bt,
                         int b, int kvh, const double *qr, long x, long y,
                         double *o, double *m, double *l) {
    int D = c->D;
    memset(o, 0, sizeof(double) * (size_t)D);
    if (y <= x) {
        *m = -INFINITY;
        *l = 0.0;
        return;
    }
    double inv_sqrt_d = 1.0 / sqrt((double)D);
    double *s = (double *)malloc(sizeof(double) * (size_t)(y - x));
    double mx = -INFINITY;
    for (long k = x; k < y; ++k) {
        const uint16_t *kr = kv_row(c, K, bt, b, k, kvh);
        double dot = 0.0;
        for (int i = 0; i < D; ++i) dot += qr[i] * bf16_to_f64(kr[i]);
        s[k - x] = dot * inv_sqrt_d;
        mx = fmax(mx, s[k - x]);
    }
    double sum = 0.0;
    for (long k = x; k < y; ++k) {
        double w = exp(s[k - x] - mx);
        const uint16_t *vr = kv_row(c, V, bt, b, k, kvh);
        sum += w;
        for (int i = 0; i < D; ++i) o[i] += w * bf16_to_f64(vr[i]);
    }
    for (int i = 0; i < D; ++i) o[i] /= sum;
    *m = mx;
    *l = sum;
    free(s);
}

/* Exported for the tests: exact state of one head over keys [x, y) of a
 * contiguous [L][D] K/V pair. */
void oracle_partial(const double *qrot, const uint16_t *K, const uint16_t *V, int D, long L,
                    long x, long y, double *o, double *m, double *l) {
    ocfg_t c;
    memset(&c, 0, sizeof c);
    c.B = 1; c.Hq = 1; c.Hkv = 1; c.D = D; c.max_seq = (int)L; c.page_size = 0;
    partial_view(&c, K, V, NULL, 0, 0, qrot, x, y, o, m, l);
}

/* Stable merge (page 1, complete stage): combine two states of
 * disjoint key ranges.  Each side's weight is l_i * exp(m_i - M) with M the
 * larger max, so no exponent is positive.  The empty state is the identity. */
void oracle_merge(const double *o1, double m1, double l1, const double *o2, double m2, double l2,
                  int D, double *o, double *m, double *l) {
    int e1 = !(l1 > 0.0) && !isnan(l1), e2 = !(l2 > 0.0) && !isnan(l2);
    if (e1 && e2) {
        for (int i = 0; i < D; ++i) o[i] = 0.0;
        *m = -INFINITY;
        *l = 0.0;
        return;
    }
    if (e1) {
        for (int i = 0; i < D; ++i) o[i] = o2[i];
        *m = m2; *l = l2;
        return;
    }
    if (e2) {
        for (int i = 0; i < D; ++i) o[i] = o1[i];
        *m = m1; *l = l1;
        return;
    }
    double M = fmax(m1, m2);
    double a1 = l1 * exp(m1 - M), a2 = l2 * exp(m2 - M);
    double L = a1 + a2;
    for (int i = 0; i < D; ++i) o[i] = (a1 * o1[i] + a2 * o2[i]) / L;
    *m = M;
    *l = L;
}

/* ----------------------------------------------------------------- state */

ostate_t *oracle_create(const ocfg_t *cfg) {
    if (!cfg || cfg->Hkv <= 0 || cfg->Hq % cfg->Hkv != 0 || cfg->D <= 0 || (cfg->D & 1) || cfg->W < 0 ||
        cfg->band < 0 || cfg->B <= 0 || cfg->cut_mode < 0 || cfg->cut_mode > 1 || cfg->per_head < 0 ||
        cfg->per_head > 1 || cfg->ring_bf16 < 0 || cfg->ring_bf16 > 1)
        return NULL;
    ostate_t *s = (ostate_t *)calloc(1, sizeof(ostate_t));
    s->c = *cfg;
    s->G = cfg->Hq / cfg->Hkv;
    s->U = cfg->B * cfg->Hkv;
    size_t W = cfg->W > 0 ? (size_t)cfg->W : 1, G = (size_t)s->G, D = (size_t)cfg->D, U = (size_t)s->U;
    s->n = (int *)calloc(U, sizeof(int));
    s->wq = (float *)calloc(U * W * G * D, sizeof(float));
    s->wo = (double *)calloc(U * W * G * D, sizeof(double));
    s->wm = (double *)calloc(U * W * G, sizeof(double));
    s->wl = (double *)calloc(U * W * G, sizeof(double));
    s->wpos = (int *)calloc(U * W, sizeof(int));
    return s;
}

void oracle_free(ostate_t *s) {
    if (!s) return;
    free(s->n); free(s->wq); free(s->wo); free(s->wm); free(s->wl); free(s->wpos);
    free(s);
}

/* Empty the window of every KV head of sequence b. */
void oracle_reset(ostate_t *s, int b) {
    for (int kvh = 0; kvh < s->c.Hkv; ++kvh) s->n[b * s->c.Hkv + kvh] = 0;
}

/* Replace the match threshold.  A warm start from prefill runs its positions
 * as steps with threshold 0: every one misses and stores (q, prefix state,
 * position), i.e. the window is seeded with the prefill queries and their
 * prefix states over [0, c) ([warm]). */
void oracle_set_tau(ostate_t *s, double tau) { s->c.tau = tau; }

/* Copy out the window of unit u = b * Hkv + kvh, oldest entry first. */
int oracle_window(const ostate_t *s, int u, float *q, double *o, double *m, double *l, int *pos) {
    size_t G = (size_t)s->G, D = (size_t)s->c.D, W = (size_t)(s->c.W > 0 ? s->c.W : 1);
    int n = s->n[u];
    if (q) memcpy(q, s->wq + (size_t)u * W * G * D, sizeof(float) * (size_t)n * G * D);
    if (o) memcpy(o, s->wo + (size_t)u * W * G * D, sizeof(double) * (size_t)n * G * D);
    if (m) memcpy(m, s->wm + (size_t)u * W * G, sizeof(double) * (size_t)n * G);
    if (l) memcpy(l, s->wl + (size_t)u * W * G, sizeof(double) * (size_t)n * G);
    if (pos) memcpy(pos, s->wpos + (size_t)u * W, sizeof(int) * (size_t)n);
    return n;
}

/* ----------------------------------------------------------------- match */

/* Match (page 1): nearest entry of the window to the current pre-RoPE query
 * heads h0 .. h0 + nh - 1 of unit u's group (all G heads, or one head with
 * [per-head] matching).
 * [mean-dist] dist = (1/nh) sum_h sum_i (q[h][i] - q_e[h][i])^2.
 * [window] only entries whose position precedes p_t are candidates.
 * [strict] returns the index of the smallest distance, ties to the larger
 * position, then to the more recent entry; best and second receive the two
 * smallest distances (+inf if absent). */
static int match_unit(const ostate_t *s, int u, const float *qg, int h0, int nh, int p_t, double *best,
                      double *second) {
    int G = s->G, D = s->c.D, W = s->c.W > 0 ? s->c.W : 1;
    int n = s->n[u];
    int arg = -1;
    double b1 = INFINITY, b2 = INFINITY;
    for (int e = 0; e < n; ++e) {
        int pos = s->wpos[(size_t)u * W + e];
        if (pos >= p_t) continue;
        const float *qe = s->wq + (((size_t)u * W + e) * G) * D;
        double acc = 0.0;
        for (int h = h0; h < h0 + nh; ++h)
            for (int i = 0; i < D; ++i) {
                double dlt = (double)qg[h * D + i] - (double)qe[h * D + i];
                acc += dlt * dlt;
            }
        double dist = acc / (double)nh;
        if (isnan(dist)) continue;
        /* entries run oldest to newest, so on an exact tie of distance and
         * position the later (more recent) entry wins */
        if (dist < b1 || (dist == b1 && arg >= 0 && pos >= s->wpos[(size_t)u * W + arg])) {
            b2 = b1;
            b1 = dist;
            arg = e;
        } else if (dist < b2) {
            b2 = dist;
        }
    }
    *best = b1;
    *second = b2;
    return arg;
}

/* [window] Append (pre-RoPE query, prefix state, position) as the newest
 * entry of unit u, dropping the oldest when W entries are held. */
static void push_entry(ostate_t *s, int u, const float *qg, const double *sn, const double *snm,
                       const double *snl, int p_t) {
    int G = s->G, D = s->c.D, W = s->c.W;
    if (W <= 0) return;
    size_t gd = (size_t)G * D;
    if (s->n[u] == W) {
        memmove(s->wq + (size_t)u * W * gd, s->wq + ((size_t)u * W + 1) * gd, sizeof(float) * (W - 1) * gd);
        memmove(s->wo + (size_t)u * W * gd, s->wo + ((size_t)u * W + 1) * gd, sizeof(double) * (W - 1) * gd);
        memmove(s->wm + (size_t)u * W * G, s->wm + ((size_t)u * W + 1) * G, sizeof(double) * (W - 1) * G);
        memmove(s->wl + (size_t)u * W * G, s->wl + ((size_t)u * W + 1) * G, sizeof(double) * (W - 1) * G);
        memmove(s->wpos + (size_t)u * W, s->wpos + (size_t)u * W + 1, sizeof(int) * (W - 1));
        s->n[u] = W - 1;
    }
    int slot = s->n[u];
    memcpy(s->wq + ((size_t)u * W + slot) * gd, qg, sizeof(float) * gd);
    memcpy(s->wo + ((size_t)u * W + slot) * gd, sn, sizeof(double) * gd);
    if (s->c.ring_bf16) {
        float *q = s->wq + ((size_t)u * W + slot) * gd;
        double *o = s->wo + ((size_t)u * W + slot) * gd;
        for (size_t i = 0; i < gd; ++i) {
            q[i] = round_bf16(q[i]);
            o[i] = (double)round_bf16((float)o[i]);
        }
    }
    memcpy(s->wm + ((size_t)u * W + slot) * G, snm, sizeof(double) * (size_t)G);
    memcpy(s->wl + ((size_t)u * W + slot) * G, snl, sizeof(double) * (size_t)G);
    s->wpos[(size_t)u * W + slot] = p_t;
    s->n[u] += 1;
}

/* ------------------------------------------------------------------ step */

/* One decode step for every sequence and KV head (page 1: match, then amend
 * and complete on a hit, plain attention on a miss).
 *   q_pre     [B][Hq][D] fp32 pre-RoPE queries
 *   rope_pos  [B] position used to rotate the query
 *   K, V      bf16 bits, contiguous or paged (see ocfg_t)
 *   seq_lens  [B] keys visible (the step's own row included); p_t = len - 1
 * Outputs: out [B][Hq][D], lse [B][Hq] (natural log), hit [B*Hkv],
 * match_pos [B*Hkv] (position of the matched entry or -1), best/second
 * distances [B*Hkv] -- [B*Hq] with [per-head] matching -- and keys_read
 * (keys a unit attends freshly, the union over its heads' ranges, summed
 * over units).  Returns 0, or -1 on an invalid sequence length. */
int oracle_step(ostate_t *s, const float *q_pre, const int *rope_pos, const uint16_t *K,
                const uint16_t *V, const int *block_table, const int *seq_lens, double *out,
                double *lse, uint8_t *hit, int *match_pos, double *d_best, double *d_second,
                long *keys_read) {
    const ocfg_t *c = &s->c;
    int G = s->G, D = c->D, W = c->W > 0 ? c->W : 1;
    for (int b = 0; b < c->B; ++b)
        if (seq_lens[b] < 1) return -1;
    long total_keys = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : total_keys)
    for (int u = 0; u < s->U; ++u) {
        int b = u / c->Hkv, kvh = u % c->Hkv;
        int p_t = seq_lens[b] - 1;
        const float *qg = q_pre + ((size_t)b * c->Hq + (size_t)kvh * G) * D;

        /* Match: one decision for the group, or one per head ([per-head]). */
        const int nd = c->per_head ? G : 1, hpd = G / nd;
        int *ent = (int *)malloc(sizeof(int) * (size_t)nd);
        const long shift = c->cut_mode;
        long first_fresh = (long)p_t + 1;
        for (int d = 0; d < nd; ++d) {
            double best, second;
            int e = match_unit(s, u, qg, d * hpd, hpd, p_t, &best, &second);
            int is_hit = (e >= 0) && (best < c->tau);
            ent[d] = is_hit ? e : -1;
            int p_s = is_hit ? s->wpos[(size_t)u * W + e] : -1;
            hit[(size_t)u * nd + d] = (uint8_t)is_hit;
            match_pos[(size_t)u * nd + d] = p_s;
            if (d_best) d_best[(size_t)u * nd + d] = best;
            if (d_second) d_second[(size_t)u * nd + d] = second;
            /* [cut] the reuse boundary c_s of this decision */
            long c_s = is_hit ? (p_s - c->band + shift > 0 ? (long)(p_s - c->band + shift) : 0) : 0;
            if (c_s < first_fresh) first_fresh = c_s;
        }
        /* [cut] the prefix boundary of this step */
        long c_t = p_t - c->band + shift > 0 ? (long)(p_t - c->band + shift) : 0;
        total_keys += (long)p_t + 1 - first_fresh;

        double *qr = (double *)malloc(sizeof(double) * (size_t)D);
        double *oa = (double *)malloc(sizeof(double) * (size_t)D);
        double *ob = (double *)malloc(sizeof(double) * (size_t)D);
        double *sn = (double *)malloc(sizeof(double) * (size_t)G * D);
        double *snm = (double *)malloc(sizeof(double) * (size_t)G);
        double *snl = (double *)malloc(sizeof(double) * (size_t)G);
        for (int h = 0; h < G; ++h) {
            int hq = kvh * G + h;
            const int e = ent[h / hpd], is_hit = e >= 0;
            oracle_rope(qg + (size_t)h * D, D, rope_pos[b], c->rope_theta, qr);
            double ma, la;
            double *o_new = sn + (size_t)h * D;
            if (is_hit) {
                long p_s = s->wpos[(size_t)u * W + e];
                long c_s = p_s - c->band + shift > 0 ? p_s - c->band + shift : 0;
                /* Amend: reuse the matched entry's prefix state over [0, c_s)
                 * and recompute [c_s, c_t) with the current query. */
                const double *ro = s->wo + (((size_t)u * W + e) * G + h) * D;
                double rm = s->wm[((size_t)u * W + e) * G + h];
                double rl = s->wl[((size_t)u * W + e) * G + h];
                partial_view(c, K, V, block_table, b, kvh, qr, c_s, c_t, oa, &ma, &la);
                oracle_merge(ro, rm, rl, oa, ma, la, D, o_new, &snm[h], &snl[h]);
            } else {
                /* Miss: the prefix state is fresh attention over [0, c_t). */
                partial_view(c, K, V, block_table, b, kvh, qr, 0, c_t, o_new, &snm[h], &snl[h]);
            }
            /* Complete: fresh attention over the tail [c_t, p_t], merged. */
            partial_view(c, K, V, block_table, b, kvh, qr, c_t, (long)p_t + 1, oa, &ma, &la);
            double mo, lo;
            oracle_merge(o_new, snm[h], snl[h], oa, ma, la, D, ob, &mo, &lo);
            memcpy(out + ((size_t)b * c->Hq + hq) * D, ob, sizeof(double) * (size_t)D);
            lse[(size_t)b * c->Hq + hq] = mo + log(lo);
        }

        /* Store (pre-RoPE query, prefix state, position) as the newest entry. */
        push_entry(s, u, qg, sn, snm, snl, p_t);
        free(qr); free(oa); free(ob); free(sn); free(snm); free(snl); free(ent);
    }
    if (keys_read) *keys_read = total_keys;
    return 0;
}

/* Match stage alone, for checking decisions on long query streams without
 * the attention cost: runs the match of every unit and appends the query
 * with an empty (NaN) state.  Same outputs as oracle_step's match part. */
int oracle_match_step(ostate_t *s, const float *q_pre, const int *seq_lens, uint8_t *hit,
                      int *match_pos, double *d_best, double *d_second) {
    const ocfg_t *c = &s->c;
    int G = s->G, D = c->D, W = c->W > 0 ? c->W : 1;
    for (int b = 0; b < c->B; ++b)
        if (seq_lens[b] < 1) return -1;
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < s->U; ++u) {
        int b = u / c->Hkv, kvh = u % c->Hkv;
        int p_t = seq_lens[b] - 1;
        const float *qg = q_pre + ((size_t)b * c->Hq + (size_t)kvh * G) * D;
        const int nd = c->per_head ? G : 1, hpd = G / nd;
        for (int d = 0; d < nd; ++d) {
            double best, second;
            int e = match_unit(s, u, qg, d * hpd, hpd, p_t, &best, &second);
            int is_hit = (e >= 0) && (best < c->tau);
            hit[(size_t)u * nd + d] = (uint8_t)is_hit;
            match_pos[(size_t)u * nd + d] = is_hit ? s->wpos[(size_t)u * W + e] : -1;
            if (d_best) d_best[(size_t)u * nd + d] = best;
            if (d_second) d_second[(size_t)u * nd + d] = second;
        }
        double *sn = (double *)malloc(sizeof(double) * (size_t)G * (D + 2));
        for (size_t i = 0; i < (size_t)G * (D + 2); ++i) sn[i] = NAN;
        push_entry(s, u, qg, sn, sn + (size_t)G * D, sn + (size_t)G * D + G, p_t);
        free(sn);
    }
    return 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
