/*
 * CPU oracle for Hierarchical Global Attention (HGA) routed exact-token
 * attention.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the
 * bench's CPU-baseline leg call it; the library never does.
 *
 * Plain C99, fp64 throughout, one straightforward loop per definition, no
 * blocking or fusion.  It shares no code, header or table with the CUDA
 * library.  Sources (the HGA paper-review page "HGA: Hierarchical Global
 * Attention — Drop-In Exact-Token Routing for Pretrained Long-Context
 * Transformers", section 三 "技术架构"):
 *   - eq. (1), standard causal attention              -> or_dense
 *   - "Mixed-RoPE Routing Summaries" summary formula  -> or_set_summary
 *   - "路由策略" deterministic visibility + middle routing and the
 *     selection equation M_sel = topK_c, G_sel = topK_g -> or_route, or_visible_mark
 *   - "精确 Token 输出注意力" exact softmax over the routed set -> or_attend_row
 *   - eq. (2) token cost model (used only by the bench's byte/flop counts)
 *   - training through the routed attention (Tab. 8 "Training and Prefill
 *     Speed"; Sec. 5.9 "Fine-tuning Stability", QK fine-tuning in
 *     exact-token mode): the gradient of eq. (1) restricted to each query's
 *     visible set, with the routed groups held fixed -> or_hga_backward.
 *     The page prints no formula for it; it is the textbook derivative.
 *
 * Readings where the page is silent (all stated again in the design notes):
 *   R1 RoPE pairs are rotate-half: pair i couples dims (i, i+D/2) with
 *      omega_i = theta^(-2i/D); y_i = x_i cos a - x_{i+D/2} sin a,
 *      y_{i+D/2} = x_{i+D/2} cos a + x_i sin a, a = p * omega_i.
 *   R2 pair i is high-frequency iff its wavelength 2*pi/omega_i < hf_wavelength
 *      (default: the chunk length C); the same rule serves chunks and groups.
 *   R3 p_mid of a set is the arithmetic mean of its tokens' positions.
 *   R4 summaries are means over the set (|G| tokens), built directly from the
 *      set's own tokens.  Only closed chunks (all C tokens present) have them.
 *   R5 the routing query of a query set (a 64-token prefill block, or one
 *      decode token) and KV head h is the sum over the set's tokens and over
 *      the query heads of h of the RoPE-rotated queries.
 *   R6 scores are plain dot products (no 1/sqrt(D)).
 *   R7 middle chunks of current chunk c: closed chunks m with F <= m <= c-L-1;
 *      with L == 0 the previous chunk c-1 is forced visible and left out.
 *   R8 top-K keeps min(K, n) candidates ordered by score (descending), the
 *      lower index first on equal scores; indices are reported ascending and
 *      padded with -1.  Group candidates are the groups of the selected chunks.
 *   R9 the visible set of query token i in chunk c is the union (each token
 *      once) of: sink chunks 0..F-1, recent chunks c-L..c-1, chunk c-1, the
 *      routed groups, and the tokens c*C..i of the current chunk.
 *   R10 attention scale is exactly 1/sqrt(D); LSE is natural-log.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t C, g_s, F, L, K_c, K_g;
    double theta;
    double hf_wavelength; /* <= 0 selects the default, C */
} or_params;

static const double OR_PI = 3.14159265358979323846264338327950288;

/* ---------------------------------------------------------------- RoPE -- */

/* omega_i = theta^(-2i/D) for the D/2 rotate-half pairs (R1). */
void or_omega(int D, double theta, double *omega)
{
    for (int i = 0; i < D / 2; ++i)
        omega[i] = pow(theta, -2.0 * (double)i / (double)D);
}

/* 1 for high-frequency pairs, 0 for low ones (R2). */
void or_pair_is_high(int D, double theta, double hf_wavelength, int C, int32_t *high)
{
    double hf = hf_wavelength > 0 ? hf_wavelength : (double)C;
    for (int i = 0; i < D / 2; ++i) {
        double omega = pow(theta, -2.0 * (double)i / (double)D);
        high[i] = (2.0 * OR_PI / omega < hf) ? 1 : 0;
    }
}

/* y = R_p(x) (R1); y may not alias x. */
static void rope(const double *x, double p, int D, const double *omega, double *y)
{
    int h = D / 2;
    for (int i = 0; i < h; ++i) {
        double a = p * omega[i];
        double c = cos(a), s = sin(a);
        y[i] = x[i] * c - x[i + h] * s;
        y[i + h] = x[i + h] * c + x[i] * s;
    }
}

/* n rows of D, each rotated at its own (possibly fractional) position. */
void or_rope_rows(const double *x, const double *pos, int64_t n, int D, double theta, double *y)
{
    double *omega = (double *)malloc(sizeof(double) * (size_t)(D / 2));
    or_omega(D, theta, omega);
    for (int64_t r = 0; r < n; ++r)
        rope(x + r * D, pos[r], D, omega, y + r * D);
    free(omega);
}

/* --------------------------------------------------------- summaries -- */

/* Mixed-RoPE summary of one token set: rows K + (first + j) * row_stride,
 * positions pos[first + j], j < n.  High pairs: mean of the rotated keys.
 * Low pairs: the raw mean, rotated at p_mid (R3, R4). */
void or_set_summary(const double *K, int64_t row_stride, const int32_t *pos,
                    int64_t first, int n, int D, const double *omega,
                    const int32_t *high, double *out)
{
    int h = D / 2;
    double pmid = 0.0;
    for (int j = 0; j < n; ++j)
        pmid += (double)pos[first + j];
    pmid /= (double)n;
    double *rot = (double *)malloc(sizeof(double) * (size_t)D);
    double *raw_mean = (double *)calloc((size_t)D, sizeof(double));
    double *rot_mean = (double *)calloc((size_t)D, sizeof(double));
    for (int j = 0; j < n; ++j) {
        const double *k = K + (first + j) * row_stride;
        rope(k, (double)pos[first + j], D, omega, rot);
        for (int d = 0; d < D; ++d) {
            raw_mean[d] += k[d];
            rot_mean[d] += rot[d];
        }
    }
    for (int d = 0; d < D; ++d) {
        raw_mean[d] /= (double)n;
        rot_mean[d] /= (double)n;
    }
    rope(raw_mean, pmid, D, omega, rot); /* low pairs use this */
    for (int i = 0; i < h; ++i) {
        if (high[i]) {
            out[i] = rot_mean[i];
            out[i + h] = rot_mean[i + h];
        } else {
            out[i] = rot[i];
            out[i + h] = rot[i + h];
        }
    }
    free(rot);
    free(raw_mean);
    free(rot_mean);
}

/* Chunk and group summaries of every closed chunk (R4).
 * K [B,T,Hkv,D]; S_c [B,Hkv,NC,D]; S_g [B,Hkv,NC*C/g_s,D], NC = T / C. */
void or_build_summaries(const double *K, const int32_t *pos, int B, int T, int Hkv, int D,
                        const or_params *p, double *S_c, double *S_g)
{
    int NC = T / p->C, gpc = p->C / p->g_s, NG = NC * gpc;
    double *omega = (double *)malloc(sizeof(double) * (size_t)(D / 2));
    int32_t *high = (int32_t *)malloc(sizeof(int32_t) * (size_t)(D / 2));
    or_omega(D, p->theta, omega);
    or_pair_is_high(D, p->theta, p->hf_wavelength, p->C, high);
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < Hkv; ++h) {
            const double *Kbh = K + ((int64_t)b * T * Hkv + h) * D;
            const int32_t *pb = pos + (int64_t)b * T;
            for (int m = 0; m < NC; ++m) {
                or_set_summary(Kbh, (int64_t)Hkv * D, pb, (int64_t)m * p->C, p->C, D, omega, high,
                               S_c + (((int64_t)b * Hkv + h) * NC + m) * D);
                for (int g = 0; g < gpc; ++g)
                    or_set_summary(Kbh, (int64_t)Hkv * D, pb, (int64_t)m * p->C + (int64_t)g * p->g_s,
                                   p->g_s, D, omega, high,
                                   S_g + (((int64_t)b * Hkv + h) * NG + (int64_t)m * gpc + g) * D);
            }
        }
    free(omega);
    free(high);
}

/* ------------------------------------------------------------ routing -- */

/* Routing query (R5): sum over tokens i0..i1-1 and query heads of KV head h
 * of R_{p_i}(q_{i,h'}).  Q [B,T,Hq,D]. */
void or_route_query(const double *Q, const int32_t *pos, int T, int Hq, int Hkv, int D,
                    double theta, int b, int h, int i0, int i1, double *q_r)
{
    int G = Hq / Hkv;
    double *omega = (double *)malloc(sizeof(double) * (size_t)(D / 2));
    double *rot = (double *)malloc(sizeof(double) * (size_t)D);
    or_omega(D, theta, omega);
    for (int d = 0; d < D; ++d)
        q_r[d] = 0.0;
    for (int i = i0; i < i1; ++i)
        for (int hh = h * G; hh < (h + 1) * G; ++hh) {
            rope(Q + (((int64_t)b * T + i) * Hq + hh) * D, (double)pos[(int64_t)b * T + i], D, omega, rot);
            for (int d = 0; d < D; ++d)
                q_r[d] += rot[d];
        }
    free(omega);
    free(rot);
}

typedef struct {
    double s;
    int32_t i;
} or_cand;

/* (score descending, index ascending) — R8 */
static int cand_cmp(const void *a, const void *b)
{
    const or_cand *x = (const or_cand *)a, *y = (const or_cand *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->i < y->i) ? -1 : (x->i > y->i);
}

static int int_cmp(const void *a, const void *b)
{
    int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* Top-K of n candidates (R8): out[0..K) ascending ids, -1 padded.
 * Returns how many were kept. */
int or_topk(const double *score, const int32_t *ids, int n, int K, int32_t *out)
{
    or_cand *c = (or_cand *)malloc(sizeof(or_cand) * (size_t)(n > 0 ? n : 1));
    for (int j = 0; j < n; ++j) {
        c[j].s = score[j];
        c[j].i = ids[j];
    }
    qsort(c, (size_t)n, sizeof(or_cand), cand_cmp);
    int kept = n < K ? n : K;
    for (int j = 0; j < K; ++j)
        out[j] = j < kept ? c[j].i : -1;
    qsort(out, (size_t)kept, sizeof(int32_t), int_cmp);
    free(c);
    return kept;
}

/* Is chunk m a middle chunk for a query in chunk c? (R7) */
static int is_middle(int m, int c, const or_params *p)
{
    if (m < p->F || m > c - p->L - 1) return 0;
    if (p->L == 0 && m == c - 1) return 0;
    return 1;
}

/* Two-level routing for current chunk c (selection equation; R6-R8).
 * S_c_bh [NC,D], S_g_bh [NG,D] for this (batch, KV head).  Writes
 * sel_c[K_c], sel_g[K_g]; if non-NULL, chunk_score[NC] / group_score[NG]
 * get each candidate's score and NAN elsewhere. */
void or_route(const double *q_r, const double *S_c_bh, const double *S_g_bh, int NC, int c, int D,
              const or_params *p, int32_t *sel_c, int32_t *sel_g, double *chunk_score,
              double *group_score)
{
    int gpc = p->C / p->g_s, NG = NC * gpc;
    double *sc = (double *)malloc(sizeof(double) * (size_t)(NC > 0 ? NC : 1));
    int32_t *ids = (int32_t *)malloc(sizeof(int32_t) * (size_t)(NG > NC ? (NG > 0 ? NG : 1) : (NC > 0 ? NC : 1)));
    double *gs = (double *)malloc(sizeof(double) * (size_t)(NG > 0 ? NG : 1));
    if (chunk_score)
        for (int m = 0; m < NC; ++m) chunk_score[m] = NAN;
    if (group_score)
        for (int g = 0; g < NG; ++g) group_score[g] = NAN;
    int n = 0;
    for (int m = 0; m < NC && m < c; ++m) {
        if (!is_middle(m, c, p)) continue;
        double s = 0.0;
        for (int d = 0; d < D; ++d)
            s += q_r[d] * S_c_bh[(int64_t)m * D + d];
        sc[n] = s;
        ids[n] = m;
        ++n;
        if (chunk_score) chunk_score[m] = s;
    }
    int kc = or_topk(sc, ids, n, p->K_c, sel_c);
    n = 0;
    for (int j = 0; j < kc; ++j) {
        int m = sel_c[j];
        for (int g = 0; g < gpc; ++g) {
            int gi = m * gpc + g;
            double s = 0.0;
            for (int d = 0; d < D; ++d)
                s += q_r[d] * S_g_bh[(int64_t)gi * D + d];
            gs[n] = s;
            ids[n] = gi;
            ++n;
            if (group_score) group_score[gi] = s;
        }
    }
    or_topk(gs, ids, n, p->K_g, sel_g);
    free(sc);
    free(ids);
    free(gs);
}

/* --------------------------------------------------- visible set (R9) -- */

static void mark_range(uint8_t *mark, int64_t lo, int64_t hi, int T)
{
    if (lo < 0) lo = 0;
    if (hi > T) hi = T;
    for (int64_t j = lo; j < hi; ++j)
        mark[j] = 1;
}

/* mark[T] := 1 for every key token visible to query token i (chunk c). */
void or_visible_mark(int c, int i, int T, const int32_t *sel_g, const or_params *p, uint8_t *mark)
{
    memset(mark, 0, (size_t)T);
    for (int m = 0; m < c; ++m) {
        int fixed = (m < p->F) || (m >= c - p->L) || (m == c - 1);
        if (fixed) mark_range(mark, (int64_t)m * p->C, (int64_t)(m + 1) * p->C, T);
    }
    for (int j = 0; j < p->K_g; ++j)
        if (sel_g[j] >= 0)
            mark_range(mark, (int64_t)sel_g[j] * p->g_s, (int64_t)(sel_g[j] + 1) * p->g_s, T);
    mark_range(mark, (int64_t)c * p->C, (int64_t)i + 1, T);
}

/* ------------------------------------------------------- attention -- */

/* Exact softmax attention of one rotated query row over the marked keys
 * (eq. (1) restricted to the visible set).  Krot/V rows j at stride. */
void or_attend_row(const double *qrot, const double *Krot, const double *V, int64_t stride,
                   const uint8_t *mark, int T, int D, double *out, double *lse)
{
    double scale = 1.0 / sqrt((double)D);
    double mx = -INFINITY;
    double *s = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    for (int j = 0; j < T; ++j) {
        if (!mark[j]) continue;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += qrot[d] * Krot[(int64_t)j * stride + d];
        s[j] = dot * scale;
        if (s[j] > mx) mx = s[j];
    }
    double l = 0.0;
    for (int d = 0; d < D; ++d)
        out[d] = 0.0;
    for (int j = 0; j < T; ++j) {
        if (!mark[j]) continue;
        double e = exp(s[j] - mx);
        l += e;
        for (int d = 0; d < D; ++d)
            out[d] += e * V[(int64_t)j * stride + d];
    }
    for (int d = 0; d < D; ++d)
        out[d] /= l;
    if (lse) *lse = mx + log(l);
    free(s);
}

/* -------------------------------------------------------- the driver -- */

typedef struct {
    const double *Q, *K, *V;
    const int32_t *pos;
    int B, T, Hq, Hkv, D;
    const or_params *p;
    int route_block;
    const int32_t *units; /* pairs (b, query-set index) */
    int n_units;
    double *O, *LSE;
    int32_t *sel_c, *sel_g;
    double *cscore, *gscore;
    const int32_t *sel_g_force; /* nullable: routed groups given, not chosen */
    int do_attend;
    /* shared precomputation */
    const double *Krot, *S_c, *S_g, *omega;
    int NC, NG;
    int nthreads, tid;
} or_job;

static void run_item(const or_job *J, int item, uint8_t *mark, double *q_r, double *qrot)
{
    const or_params *p = J->p;
    int u = item / J->Hkv, h = item % J->Hkv;
    int b = J->units[2 * u], qs = J->units[2 * u + 1];
    int i0 = qs * J->route_block, i1 = i0 + J->route_block;
    if (i1 > J->T) i1 = J->T;
    int c = i0 / p->C;
    int G = J->Hq / J->Hkv, D = J->D;
    int32_t *sel_c = J->sel_c + ((int64_t)u * J->Hkv + h) * p->K_c;
    int32_t *sel_g = J->sel_g + ((int64_t)u * J->Hkv + h) * p->K_g;
    or_route_query(J->Q, J->pos, J->T, J->Hq, J->Hkv, D, p->theta, b, h, i0, i1, q_r);
    or_route(q_r, J->S_c + ((int64_t)b * J->Hkv + h) * J->NC * D,
             J->S_g + ((int64_t)b * J->Hkv + h) * J->NG * D, J->NC, c, D, p, sel_c, sel_g,
             J->cscore ? J->cscore + ((int64_t)u * J->Hkv + h) * J->NC : NULL,
             J->gscore ? J->gscore + ((int64_t)u * J->Hkv + h) * J->NG : NULL);
    if (J->sel_g_force)
        memcpy(sel_g, J->sel_g_force + ((int64_t)u * J->Hkv + h) * p->K_g,
               sizeof(int32_t) * (size_t)p->K_g);
    if (!J->do_attend) return;
    const double *Kb = J->Krot + ((int64_t)b * J->T * J->Hkv + h) * D;
    const double *Vb = J->V + ((int64_t)b * J->T * J->Hkv + h) * D;
    for (int i = i0; i < i1; ++i) {
        or_visible_mark(c, i, J->T, sel_g, p, mark);
        for (int hh = h * G; hh < (h + 1) * G; ++hh) {
            int64_t row = ((int64_t)b * J->T + i) * J->Hq + hh;
            rope(J->Q + row * D, (double)J->pos[(int64_t)b * J->T + i], D, J->omega, qrot);
            or_attend_row(qrot, Kb, Vb, (int64_t)J->Hkv * D, mark, J->T, D, J->O + row * D,
                          J->LSE ? &J->LSE[((int64_t)b * J->Hq + hh) * J->T + i] : NULL);
        }
    }
}

static void *worker(void *arg)
{
    or_job *J = (or_job *)arg;
    uint8_t *mark = (uint8_t *)malloc((size_t)J->T + 1);
    double *q_r = (double *)malloc(sizeof(double) * (size_t)J->D);
    double *qrot = (double *)malloc(sizeof(double) * (size_t)J->D);
    int n_items = J->n_units * J->Hkv;
    for (int it = J->tid; it < n_items; it += J->nthreads)
        run_item(J, it, mark, q_r, qrot);
    free(mark);
    free(q_r);
    free(qrot);
    return NULL;
}

/* Full HGA over a list of query sets.  A query set is the tokens
 * [s*route_block, min(T,(s+1)*route_block)) of batch row b (route_block = C
 * for prefill blocks, 1 for decode-style per-token routing); it must lie in
 * one chunk.  units = n_units pairs (b, s).  Outputs for every unit u:
 * O rows [B,T,Hq,D] and LSE [B,Hq,T] (rows of the unit only; LSE nullable),
 * sel_c [n_units,Hkv,K_c], sel_g [n_units,Hkv,K_g], and if non-NULL the
 * candidate scores cscore [n_units,Hkv,NC], gscore [n_units,Hkv,NG].
 * Summaries are rebuilt here from K (a "full recompute").  If sel_g_force
 * is non-NULL ([n_units,Hkv,K_g]) the attention uses those routed groups
 * instead of its own choice (sel_g still reports the oracle's choice's
 * replacement: the forced ids).  With do_attend == 0 only routing runs.
 * Returns 0, or -1 on a malformed argument. */
int or_hga(const double *Q, const double *K, const double *V, const int32_t *pos, int B, int T,
           int Hq, int Hkv, int D, const or_params *p, int route_block, const int32_t *units,
           int n_units, int nthreads, double *O, double *LSE, int32_t *sel_c, int32_t *sel_g,
           double *cscore, double *gscore, const int32_t *sel_g_force, int do_attend)
{
    if (Hq % Hkv || D % 2 || p->C % p->g_s || route_block < 1 || p->C % route_block) return -1;
    int NC = T / p->C, NG = NC * (p->C / p->g_s);
    int64_t nk = (int64_t)B * T * Hkv;
    double *Krot = (double *)malloc(sizeof(double) * (size_t)(nk * D));
    double *S_c = (double *)malloc(sizeof(double) * (size_t)((int64_t)B * Hkv * (NC > 0 ? NC : 1) * D));
    double *S_g = (double *)malloc(sizeof(double) * (size_t)((int64_t)B * Hkv * (NG > 0 ? NG : 1) * D));
    double *omega = (double *)malloc(sizeof(double) * (size_t)(D / 2));
    or_omega(D, p->theta, omega);
    for (int64_t r = 0; r < nk; ++r)
        rope(K + r * D, (double)pos[r / Hkv], D, omega, Krot + r * D);
    or_build_summaries(K, pos, B, T, Hkv, D, p, S_c, S_g);
    if (nthreads < 1) nthreads = 1;
    or_job *jobs = (or_job *)malloc(sizeof(or_job) * (size_t)nthreads);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        or_job J = {Q, K, V, pos, B, T, Hq, Hkv, D, p, route_block, units, n_units, O, LSE,
                    sel_c, sel_g, cscore, gscore, sel_g_force, do_attend, Krot, S_c, S_g,
                    omega, NC, NG, nthreads, t};
        jobs[t] = J;
    }
    for (int t = 1; t < nthreads; ++t)
        pthread_create(&th[t], NULL, worker, &jobs[t]);
    worker(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    free(jobs);
    free(th);
    free(Krot);
    free(S_c);
    free(S_g);
    free(omega);
    return 0;
}

/* Dense causal attention, eq. (1): every key j <= i, RoPE on q and k. */
int or_dense(const double *Q, const double *K, const double *V, const int32_t *pos, int B, int T,
             int Hq, int Hkv, int D, double theta, double *O, double *LSE)
{
    if (Hq % Hkv || D % 2) return -1;
    int G = Hq / Hkv;
    double *omega = (double *)malloc(sizeof(double) * (size_t)(D / 2));
    double *qrot = (double *)malloc(sizeof(double) * (size_t)D);
    double *Krot = (double *)malloc(sizeof(double) * (size_t)((int64_t)B * T * Hkv * D));
    uint8_t *mark = (uint8_t *)malloc((size_t)T + 1);
    or_omega(D, theta, omega);
    for (int64_t r = 0; r < (int64_t)B * T * Hkv; ++r)
        rope(K + r * D, (double)pos[r / Hkv], D, omega, Krot + r * D);
    for (int b = 0; b < B; ++b)
        for (int i = 0; i < T; ++i) {
            for (int j = 0; j < T; ++j)
                mark[j] = (uint8_t)(j <= i);
            for (int hh = 0; hh < Hq; ++hh) {
                int64_t row = ((int64_t)b * T + i) * Hq + hh;
                int h = hh / G;
                rope(Q + row * D, (double)pos[(int64_t)b * T + i], D, omega, qrot);
                or_attend_row(qrot, Krot + ((int64_t)b * T * Hkv + h) * D,
                              V + ((int64_t)b * T * Hkv + h) * D, (int64_t)Hkv * D, mark, T, D,
                              O + row * D, LSE ? &LSE[((int64_t)b * Hq + hh) * T + i] : NULL);
            }
        }
    free(omega);
    free(qrot);
    free(Krot);
    free(mark);
    return 0;
}

/* ---------------------------------------------------------- backward -- */

/* x = R_p^T(y), the adjoint of R1's rotation (rotation by -p); x may not
 * alias y. */
static void rope_adjoint(const double *y, double p, int D, const double *omega, double *x)
{
    int h = D / 2;
    for (int i = 0; i < h; ++i) {
        double a = p * omega[i];
        double c = cos(a), s = sin(a);
        x[i] = y[i] * c + y[i + h] * s;
        x[i + h] = y[i + h] * c - y[i] * s;
    }
}

typedef struct {
    const double *Q, *K, *V, *dO;
    const int32_t *pos, *sel_g;
    int B, T, Hq, Hkv, D, NB;
    const or_params *p;
    double *dQ, *dK, *dV;
    const double *omega;
    int nthreads, tid;
} or_bwd_job;

/* One (sequence b, KV head h): every query row of h's query heads, in
 * order; dK and dV rows of (b, h) and dQ rows of those heads belong to this
 * item alone. */
static void bwd_item(const or_bwd_job *J, int b, int h)
{
    const or_params *p = J->p;
    int T = J->T, D = J->D, G = J->Hq / J->Hkv;
    int64_t ks = (int64_t)J->Hkv * D; /* key row stride */
    double scale = 1.0 / sqrt((double)D);
    double *krot = (double *)malloc(sizeof(double) * (size_t)((int64_t)(T > 0 ? T : 1) * D));
    double *dkrot = (double *)calloc((size_t)((int64_t)(T > 0 ? T : 1) * D), sizeof(double));
    double *pr = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
    uint8_t *mark = (uint8_t *)malloc((size_t)T + 1);
    double *qrot = (double *)malloc(sizeof(double) * (size_t)D);
    double *o = (double *)malloc(sizeof(double) * (size_t)D);
    double *dqrot = (double *)malloc(sizeof(double) * (size_t)D);
    const double *Kb = J->K + ((int64_t)b * T * J->Hkv + h) * D;
    const double *Vb = J->V + ((int64_t)b * T * J->Hkv + h) * D;
    double *dKb = J->dK + ((int64_t)b * T * J->Hkv + h) * D;
    double *dVb = J->dV + ((int64_t)b * T * J->Hkv + h) * D;
    for (int j = 0; j < T; ++j) {
        rope(Kb + (int64_t)j * ks, (double)J->pos[(int64_t)b * T + j], D, J->omega,
             krot + (int64_t)j * D);
        for (int d = 0; d < D; ++d)
            dVb[(int64_t)j * ks + d] = 0.0;
    }
    for (int i = 0; i < T; ++i) {
        /* A query row whose dO is zero adds nothing to any gradient (every
         * term it contributes carries a factor dO_i, including dO_i . O_i)
         * and its own dq is zero: such rows are skipped. */
        int live = 0;
        for (int hh = h * G; hh < (h + 1) * G && !live; ++hh) {
            const double *dO = J->dO + (((int64_t)b * T + i) * J->Hq + hh) * D;
            for (int d = 0; d < D; ++d)
                if (dO[d] != 0.0) { live = 1; break; }
        }
        if (!live) {
            for (int hh = h * G; hh < (h + 1) * G; ++hh)
                memset(J->dQ + (((int64_t)b * T + i) * J->Hq + hh) * D, 0, sizeof(double) * (size_t)D);
            continue;
        }
        int c = i / p->C;
        or_visible_mark(c, i, T, J->sel_g + (((int64_t)b * J->NB + c) * J->Hkv + h) * p->K_g, p,
                        mark);
        double pi = (double)J->pos[(int64_t)b * T + i];
        for (int hh = h * G; hh < (h + 1) * G; ++hh) {
            int64_t row = ((int64_t)b * T + i) * J->Hq + hh;
            const double *dO = J->dO + row * D;
            rope(J->Q + row * D, pi, D, J->omega, qrot);
            /* forward again: P_j and O_i */
            double mx = -INFINITY;
            for (int j = 0; j < T; ++j) {
                if (!mark[j]) continue;
                double dot = 0.0;
                for (int d = 0; d < D; ++d)
                    dot += qrot[d] * krot[(int64_t)j * D + d];
                pr[j] = dot * scale;
                if (pr[j] > mx) mx = pr[j];
            }
            double l = 0.0;
            for (int j = 0; j < T; ++j)
                if (mark[j]) {
                    pr[j] = exp(pr[j] - mx);
                    l += pr[j];
                }
            for (int d = 0; d < D; ++d)
                o[d] = 0.0;
            for (int j = 0; j < T; ++j) {
                if (!mark[j]) continue;
                pr[j] /= l;
                for (int d = 0; d < D; ++d)
                    o[d] += pr[j] * Vb[(int64_t)j * ks + d];
            }
            /* D_i = dO_i . O_i, then the gradients through P */
            double di = 0.0;
            for (int d = 0; d < D; ++d)
                di += dO[d] * o[d];
            for (int d = 0; d < D; ++d)
                dqrot[d] = 0.0;
            for (int j = 0; j < T; ++j) {
                if (!mark[j]) continue;
                double dp = 0.0;
                for (int d = 0; d < D; ++d)
                    dp += dO[d] * Vb[(int64_t)j * ks + d];
                double ds = pr[j] * (dp - di);
                for (int d = 0; d < D; ++d) {
                    dVb[(int64_t)j * ks + d] += pr[j] * dO[d];
                    dqrot[d] += ds * scale * krot[(int64_t)j * D + d];
                    dkrot[(int64_t)j * D + d] += ds * scale * qrot[d];
                }
            }
            rope_adjoint(dqrot, pi, D, J->omega, J->dQ + row * D);
        }
    }
    for (int j = 0; j < T; ++j)
        rope_adjoint(dkrot + (int64_t)j * D, (double)J->pos[(int64_t)b * T + j], D, J->omega,
                     dKb + (int64_t)j * ks);
    free(krot);
    free(dkrot);
    free(pr);
    free(mark);
    free(qrot);
    free(o);
    free(dqrot);
}

static void *bwd_worker(void *arg)
{
    or_bwd_job *J = (or_bwd_job *)arg;
    for (int it = J->tid; it < J->B * J->Hkv; it += J->nthreads)
        bwd_item(J, it / J->Hkv, it % J->Hkv);
    return NULL;
}

/* Backward of the exact attention of HGA prefill (eq. (1) restricted to each
 * query token's visible set, blocks of C query tokens).  Routing is a
 * discrete choice, so no gradient reaches the summaries: the routed groups
 * are an input, sel_g [B, NB, Hkv, K_g] (NB = ceil(T / C)), the ones the
 * forward attended.  Given dO [B,T,Hq,D], writes the gradients of the loss
 * with respect to the RAW (pre-RoPE) q and k and to v:
 *   S_ij = R_{p_i}(q_i) . R_{p_j}(k_j) / sqrt(D), P_ij = softmax_j S_ij over
 *   j in V(i), O_i = sum_j P_ij v_j,
 *   dv_j = sum_i P_ij dO_i,
 *   dS_ij = P_ij (dO_i . v_j - dO_i . O_i),
 *   dq_i = R_{p_i}^T sum_j dS_ij R_{p_j}(k_j) / sqrt(D),
 *   dk_j = R_{p_j}^T sum_i dS_ij R_{p_i}(q_i) / sqrt(D),
 * where i runs over the query rows of every query head of k_j's KV head.
 * dQ [B,T,Hq,D], dK and dV [B,T,Hkv,D].  Returns 0, or -1 on a malformed
 * argument. */
int or_hga_backward(const double *Q, const double *K, const double *V, const int32_t *pos,
                    const double *dO, int B, int T, int Hq, int Hkv, int D, const or_params *p,
                    const int32_t *sel_g, int nthreads, double *dQ, double *dK, double *dV)
{
    if (Hq % Hkv || D % 2 || p->C % p->g_s || p->C < 1 || T < 0 || B < 1) return -1;
    int NB = (T + p->C - 1) / p->C;
    double *omega = (double *)malloc(sizeof(double) * (size_t)(D / 2));
    or_omega(D, p->theta, omega);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > B * Hkv) nthreads = B * Hkv;
    or_bwd_job *jobs = (or_bwd_job *)malloc(sizeof(or_bwd_job) * (size_t)nthreads);
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int t = 0; t < nthreads; ++t) {
        or_bwd_job J = {Q, K, V, dO, pos, sel_g, B, T, Hq, Hkv, D, NB, p, dQ, dK, dV, omega,
                        nthreads, t};
        jobs[t] = J;
    }
    for (int t = 1; t < nthreads; ++t)
        pthread_create(&th[t], NULL, bwd_worker, &jobs[t]);
    bwd_worker(&jobs[0]);
    for (int t = 1; t < nthreads; ++t)
        pthread_join(th[t], NULL);
    free(jobs);
    free(th);
    free(omega);
    return 0;
}
