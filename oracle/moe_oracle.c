/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle of the masked routed-expert
 * MoE layer.  TEST INFRASTRUCTURE ONLY: it is called by the tests, by the
 * smoke check and by the benchmark's CPU-baseline leg, never by the product
 * path.  It shares no code with the CUDA library.
 *
 * Source of the definition: "Uncovering Intra-expert Activation Sparsity for
 * Efficient Mixture-of-Expert Model Execution" (technical summary page),
 * Methodology item 3 and its four bullets, and the Hindi summary of the same
 * paper, section "How they did it: the skip-list system".  Per token:
 *
 *   router      logits_e = x . Wr[e];  p = softmax(logits) over all E;
 *               the k experts with the largest p are selected, ties going to
 *               the lower expert index; the routing weight is p itself
 *               (the router is kept unchanged, Methodology item 3).
 *   gate        g_j = sum_i x_i Wg[e][i][j]  for every neuron j  (dense,
 *               "Gate projection" bullet).
 *   score/mask  s_j = |silu(g_j)|,  silu(z) = z / (1 + exp(-z));  neuron j
 *               is active iff s_j >= tau  -- one threshold pass, no sort
 *               ("Activation masking" bullet).
 *   up/down     for active j only: u_j = sum_i x_i Wu[e][i][j],
 *               h_j = silu(g_j) u_j,  y += p_e h_j Wd[e][j][:]
 *               ("Fused up-down projection" bullet; inactive neurons are not
 *               loaded, Hindi summary "The skip").
 *   shared      y += sum_j silu(gs_j) us_j Wds[j][:]  over the neurons of each
 *               shared expert, not weighted (shared experts are always on and
 *               their execution is unchanged, Methodology items 1-3).  By
 *               default every shared neuron counts; a separate shared
 *               threshold tau_s > 0 keeps only shared neurons with
 *               |silu(gs_j)| >= tau_s (Methodology item 1: shared neurons
 *               matter more per neuron than routed ones, so they take their
 *               own, looser threshold).
 *
 * Precision: bf16 inputs are widened exactly; every product and sum is in
 * double.  The mask decision compares the score rounded to float with the
 * float tau, the precision the CUDA path decides in.
 *
 * Layout (x @ W convention): x [T][d], Wr [E][d], Wg/Wu [E][d][f],
 * Wd [E][f][d], Wsg/Wsu [S][d][f], Wsd [S][f][d]; all bf16 bit patterns.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double silu(double z)
{
    return z / (1.0 + exp(-z));
}

/* Router for one token: logits, softmax over all experts, top-k selection.
 * Selection repeats "take the largest remaining p, lower index on ties"
 * k times; that is the definition of an ordered top-k. */
static void route_token(const uint16_t *xt, int d, const uint16_t *wr, int E, int k,
                        double *logit, double *p, int *idx, double *w)
{
    double mx = -INFINITY, sum = 0.0;
    for (int e = 0; e < E; ++e) {
        double acc = 0.0;
        for (int i = 0; i < d; ++i)
            acc += bf16_to_double(xt[i]) * bf16_to_double(wr[(size_t)e * d + i]);
        logit[e] = acc;
        if (acc > mx) mx = acc;
    }
    for (int e = 0; e < E; ++e) {
        p[e] = exp(logit[e] - mx);
        sum += p[e];
    }
    for (int e = 0; e < E; ++e) p[e] /= sum;
    for (int r = 0; r < k; ++r) {
        int best = -1;
        for (int e = 0; e < E; ++e) {
            int taken = 0;
            for (int q = 0; q < r; ++q) taken |= (idx[q] == e);
            if (taken) continue;
            if (best < 0 || p[e] > p[best]) best = e;   /* strict: ties keep the lower index */
        }
        idx[r] = best;
        w[r] = p[best];
    }
}

/* One SwiGLU projection pair for one expert: g = x Wg, u = x Wu (all f columns). */
static void gate_up(const uint16_t *xt, int d, int f, const uint16_t *wg, const uint16_t *wu,
                    double *g, double *u)
{
    for (int j = 0; j < f; ++j) { g[j] = 0.0; if (u) u[j] = 0.0; }
    for (int i = 0; i < d; ++i) {
        double xi = bf16_to_double(xt[i]);
        const uint16_t *rg = wg + (size_t)i * f;
        for (int j = 0; j < f; ++j) g[j] += xi * bf16_to_double(rg[j]);
        if (u) {
            const uint16_t *ru = wu + (size_t)i * f;
            for (int j = 0; j < f; ++j) u[j] += xi * bf16_to_double(ru[j]);
        }
    }
}

/* The full layer.  Outputs (any may be NULL except y):
 *   y          [T][d]   layer output, double
 *   topk_idx   [T][k]   selected experts in rank order
 *   topk_w     [T][k]   their routing weights p
 *   logits     [T][E]   router logits
 *   score      [T][k][f] s = |silu(g)| of each selected pair
 *   active     [T][k][f] 1 where s >= tau (decided in float)
 *   score_shared [T][S][f] |silu(gs)| of each shared neuron
 * tau_shared: shared neuron j counts iff (float)|silu(gs_j)| >= tau_shared;
 * tau_shared <= 0 keeps every shared neuron (the default layer).
 * Optional input:
 *   active_in  [T][k][f] when not NULL, neuron j of the pair (t, rank r) is
 *              active iff active_in[t][r][j] != 0, in place of the threshold
 *              decision (tau is then unused).  This evaluates the layer under
 *              a given mask, e.g. one whose neurons at the threshold went the
 *              other way; `active` then echoes active_in.
 * Returns 0, or -1 on bad sizes / allocation failure. */
int oracle_moe_forward(const uint16_t *x, int T, int d, int f, int E, int k, int S,
                       const uint16_t *wr, const uint16_t *wg, const uint16_t *wu,
                       const uint16_t *wd, const uint16_t *wsg, const uint16_t *wsu,
                       const uint16_t *wsd, float tau, float tau_shared, int nthreads,
                       double *y, int *topk_idx, double *topk_w, double *logits,
                       double *score, uint8_t *active, const uint8_t *active_in, double *score_shared)
{
    if (T < 0 || d <= 0 || f <= 0 || E <= 0 || k <= 0 || k > E || S < 0) return -1;
    if (S > 0 && (!wsg || !wsu || !wsd)) return -1;
    int bad = 0;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
#else
    (void)nthreads;
#endif
    for (int t = 0; t < T; ++t) {
        const uint16_t *xt = x + (size_t)t * d;
        double *lg = malloc(sizeof(double) * E), *p = malloc(sizeof(double) * E);
        double *g = malloc(sizeof(double) * f), *u = malloc(sizeof(double) * f);
        int *idx = malloc(sizeof(int) * k);
        double *w = malloc(sizeof(double) * k);
        double *yt = y + (size_t)t * d;
        if (!lg || !p || !g || !u || !idx || !w) {
            bad |= 1;
        } else {
            for (int i = 0; i < d; ++i) yt[i] = 0.0;
            route_token(xt, d, wr, E, k, lg, p, idx, w);
            if (logits) memcpy(logits + (size_t)t * E, lg, sizeof(double) * E);
            if (topk_idx) memcpy(topk_idx + (size_t)t * k, idx, sizeof(int) * k);
            if (topk_w) memcpy(topk_w + (size_t)t * k, w, sizeof(double) * k);
            /* shared experts: SwiGLU, unweighted; every neuron unless a
               shared threshold is given */
            for (int s = 0; s < S; ++s) {
                gate_up(xt, d, f, wsg + (size_t)s * d * f, wsu + (size_t)s * d * f, g, u);
                const uint16_t *down = wsd + (size_t)s * f * d;
                for (int j = 0; j < f; ++j) {
                    double as = silu(g[j]);
                    double ss = fabs(as);
                    if (score_shared) score_shared[((size_t)t * S + s) * f + j] = ss;
                    if (!((float)ss >= tau_shared)) continue;
                    double h = as * u[j];
                    for (int i = 0; i < d; ++i) yt[i] += h * bf16_to_double(down[(size_t)j * d + i]);
                }
            }
            /* routed experts: dense gate, threshold mask, up/down on active neurons */
            for (int r = 0; r < k; ++r) {
                int e = idx[r];
                gate_up(xt, d, f, wg + (size_t)e * d * f, wu + (size_t)e * d * f, g, u);
                const uint16_t *down = wd + (size_t)e * f * d;
                for (int j = 0; j < f; ++j) {
                    double a = silu(g[j]);
                    double s = fabs(a);
                    size_t o = ((size_t)t * k + r) * f + j;
                    int on = ((float)s >= tau);
                    if (active_in) on = (active_in[o] != 0);
                    if (score) score[o] = s;
                    if (active) active[o] = (uint8_t)on;
                    if (!on) continue;
                    double h = a * u[j];
                    for (int i = 0; i < d; ++i)
                        yt[i] += w[r] * h * bf16_to_double(down[(size_t)j * d + i]);
                }
            }
        }
        free(lg); free(p); free(g); free(u); free(idx); free(w);
    }
    return bad ? -1 : 0;
}

static int cmp_double(const void *a, const void *b)
{
    double x = *(const double *)a, y = *(const double *)b;
    return (x > y) - (x < y);
}

/* Threshold for a target sparsity q: sort the N scores ascending and take the
 * one at position floor(q*N); q <= 0 gives 0 (keep all), floor(q*N) >= N gives
 * +inf (keep none).  At least N - floor(q*N) scores are >= tau, so the kept
 * fraction is within 1/N of 1 - q when scores are distinct. */
double oracle_calibrate_tau(const double *s, long n, double q)
{
    if (q <= 0.0 || n <= 0) return 0.0;
    long m = (long)floor(q * (double)n);
    if (m >= n) return INFINITY;
    double *c = malloc(sizeof(double) * (size_t)n);
    if (!c) return NAN;
    memcpy(c, s, sizeof(double) * (size_t)n);
    qsort(c, (size_t)n, sizeof(double), cmp_double);
    double tau = c[m];
    free(c);
    return tau;
}

/* Rank budget per pair (technical summary, Methodology item 1: the
 * lowest-scoring neurons of an expert are zeroed progressively, as an
 * alternative to one threshold): of each pair's f scores keep the r largest.
 * The scores are compared rounded to float, the precision the threshold is
 * decided in; equal scores go to the lower neuron index; a NaN score is never
 * kept (it ranks below every number), so a pair keeps min(r, its non-NaN
 * scores) neurons.  The definition is written as a sort of the pair's
 * (score, index) entries by score descending, index ascending, the first r
 * entries being kept.
 *   s     [n_pairs][f] scores (e.g. the `score` output above)
 *   mask  [n_pairs][f] out: 1 kept, 0 not
 * Returns 0, or -1 on bad sizes / allocation failure. */
typedef struct {
    double v;
    int j;
} rank_entry;

static int cmp_rank(const void *pa, const void *pb)
{
    const rank_entry *a = (const rank_entry *)pa, *b = (const rank_entry *)pb;
    const float va = (float)a->v, vb = (float)b->v;
    if (va > vb) return -1;
    if (va < vb) return 1;
    return (a->j > b->j) - (a->j < b->j);
}

int oracle_rank_mask(const double *s, long n_pairs, int f, int r, uint8_t *mask)
{
    if (n_pairs < 0 || f < 1 || !s || !mask) return -1;
    rank_entry *e = (rank_entry *)malloc(sizeof(rank_entry) * (size_t)f);
    if (!e) return -1;
    for (long p = 0; p < n_pairs; ++p) {
        const double *sp = s + p * (long)f;
        uint8_t *mp = mask + p * (long)f;
        int n = 0;
        for (int j = 0; j < f; ++j) {
            mp[j] = 0;
            if (sp[j] == sp[j]) {   /* not NaN */
                e[n].v = sp[j];
                e[n].j = j;
                ++n;
            }
        }
        qsort(e, (size_t)n, sizeof(rank_entry), cmp_rank);
        for (int q = 0; q < n && q < r; ++q) mp[e[q].j] = 1;
    }
    free(e);
    return 0;
}

/* Capacity-aware token drop ("Capacity-Aware Inference" page, section
 * "Capacity-Aware Token Drop"): an expert holds at most C of the (token,
 * expert) pairs routed to it.  When more are routed to it, it keeps the C
 * pairs with the largest routing weight p (the post-softmax gate score),
 * compared rounded to float as the CUDA path decides it, equal weights going
 * to the lower token index; the other pairs are dropped and contribute
 * nothing.  Kept pairs keep their weights (no renormalisation) and the
 * token's other experts are unaffected.  Written as its definition: a pair is
 * kept iff fewer than C pairs of the same expert beat it.
 *   idx, w  [T][k] the router's selection and weights (rank order)
 *   keep    [T][k] out: 1 kept, 0 dropped
 * C < 0 keeps every pair.  Returns 0, or -1 on bad sizes. */
int oracle_capacity_keep(const int *idx, const double *w, int T, int k, int E, int C, uint8_t *keep)
{
    if (T < 0 || k <= 0 || E <= 0 || !idx || !w || !keep) return -1;
    const long P = (long)T * k;
    for (long p = 0; p < P; ++p) {
        if (C < 0) {
            keep[p] = 1;
            continue;
        }
        const int e = idx[p];
        const float wp = (float)w[p];
        const long tp = p / k;
        long better = 0;
        for (long q = 0; q < P; ++q) {
            if (q == p || idx[q] != e) continue;
            const float wq = (float)w[q];
            if (wq > wp || (wq == wp && q / k < tp)) ++better;
        }
        keep[p] = (uint8_t)(better < C);
    }
    return 0;
}
