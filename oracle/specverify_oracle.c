/*
 * specverify_oracle.c -- plain, slow, single-threaded fp64 reference of the
 * speculative-decoding verification sampler.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or constant with the
 * CUDA implementation; the two meet only through the seeded synthetic inputs.
 *
 * Sources (cited by short name below):
 *   [Sonar]     Licker & McKnight, "Accelerating Sonar through speculation",
 *               Perplexity blog, 2025.  Sections "Speculative decoding" (the
 *               four stages), "Target-Draft" (acceptance compares the full
 *               draft and target distributions; the target always yields one
 *               more set of logits after the accepted prefix), "EAGLE"
 *               (tree drafts: longest suitable sequence plus one target
 *               token).
 *   [Explainer] "Speculative decoding explained: how any LLM can get 3x
 *               faster inference".  Section "Draft and verification loop"
 *               (the probabilistic acceptance rule and the corrected token
 *               drawn from an adjusted distribution; the output keeps the
 *               target's distribution) and "Best and worst case" (all drafts
 *               plus one extra token; first draft rejected).
 *   [Leviathan] Leviathan, Kalman & Matias, "Fast inference from
 *               transformers via speculative decoding" (the first reference
 *               of [Sonar]): accept with min(1, p(x)/q(x)), on rejection
 *               resample from norm(max(0, p - q)).
 *   [Philox]    Salmon, Moraes, Dror & Shaw, "Parallel random numbers: as
 *               easy as 1, 2, 3", SC'11, section 4 (the Philox S-box and key
 *               schedule).
 *
 * Readings taken where the pages are silent (each one is listed in the
 * design notes as well):
 *   - temperature T divides both target and draft logits before the softmax;
 *   - the accept test is strict: accept <=> u * q(x) < p(x), u in [0, 1);
 *   - inverse CDF: token = smallest v with C_v > u * Z, C accumulated left to
 *     right; if rounding leaves no such v, the largest v with w_v > 0;
 *   - if the residual mass is exactly zero, sample the target row instead;
 *   - a tree node is accepted when its parent is accepted and its own test
 *     passes; the deepest accepted node wins, ties to the lowest index; the
 *     bonus comes from that node's target row (no residual in tree mode).
 *
 * Precision: every probability, sum and comparison is fp64.  Input logits
 * are fp32 or bf16 and are widened exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* request error bits (same meaning as the library's status bits) */
#define ORC_ERR_TOKEN 1   /* a draft/node token outside [0, V)            */
#define ORC_ERR_TREE 2    /* malformed parent array or depth > max_depth  */
#define ORC_ERR_LOGIT 4   /* NaN logit, or a row whose normaliser is bad  */

/* ------------------------------------------------------------------------ */
/* [Philox] Philox4x32-10.                                                  */
/* Counter-based generator: a 4-word counter is pushed through ten rounds   */
/* of a multiply/xor S-box keyed by a 2-word key that is bumped by two Weyl */
/* constants between rounds.                                                */
/* ------------------------------------------------------------------------ */
static const uint32_t PHILOX_MUL_A = 0xD2511F53u;
static const uint32_t PHILOX_MUL_B = 0xCD9E8D57u;
static const uint32_t PHILOX_WEYL_A = 0x9E3779B9u; /* golden ratio          */
static const uint32_t PHILOX_WEYL_B = 0xBB67AE85u; /* sqrt(3) - 1           */

void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        uint64_t pa = (uint64_t)PHILOX_MUL_A * (uint64_t)x0;
        uint64_t pb = (uint64_t)PHILOX_MUL_B * (uint64_t)x2;
        uint32_t hi_a = (uint32_t)(pa >> 32), lo_a = (uint32_t)pa;
        uint32_t hi_b = (uint32_t)(pb >> 32), lo_b = (uint32_t)pb;
        uint32_t y0 = hi_b ^ x1 ^ k0;
        uint32_t y1 = lo_b;
        uint32_t y2 = hi_a ^ x3 ^ k1;
        uint32_t y3 = lo_a;
        x0 = y0; x1 = y1; x2 = y2; x3 = y3;
        k0 += PHILOX_WEYL_A;
        k1 += PHILOX_WEYL_B;
    }
    out[0] = x0; out[1] = x1; out[2] = x2; out[3] = x3;
}

/* Uniform in [0, 1 - 2^-24] drawn from counter (request, position, purpose,
 * offset) under key (seed low word, seed high word): the top 24 bits of the
 * first output word times 2^-24 (exact in fp32 and fp64). */
double orc_uniform(uint64_t seed, uint32_t request, uint32_t position, uint32_t purpose,
                   uint32_t offset)
{
    uint32_t ctr[4] = {request, position, purpose, offset};
    uint32_t key[2] = {(uint32_t)(seed & 0xFFFFFFFFu), (uint32_t)(seed >> 32)};
    uint32_t out[4];
    orc_philox4x32_10(ctr, key, out);
    return (double)(out[0] >> 8) * (1.0 / 16777216.0);
}

/* out[b * count + i] = U(seed, b, first_position + i, purpose, offset) */
void orc_fill_uniforms(uint64_t seed, uint32_t offset, uint32_t purpose, int batch, int count,
                       int first_position, double *out)
{
    for (int b = 0; b < batch; ++b)
        for (int i = 0; i < count; ++i)
            out[(int64_t)b * count + i] =
                orc_uniform(seed, (uint32_t)b, (uint32_t)(first_position + i), purpose, offset);
}

/* ------------------------------------------------------------------------ */
/* Logit access: dtype 0 = fp32, 1 = bf16 (upper half of an fp32).          */
/* ------------------------------------------------------------------------ */
static double logit_at(const void *base, int dtype, int64_t index)
{
    if (dtype == 0) return (double)((const float *)base)[index];
    uint32_t bits = (uint32_t)((const uint16_t *)base)[index] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* A target or draft row after temperature scaling:
 *   p(v) = exp((l_v - m) / T) / S,   m = max_v l_v,   S = sum_v exp((l_v - m) / T).
 * [Sonar] "Target-Draft": acceptance compares the full distributions, so
 * every row needs its whole-vocabulary normaliser. */
typedef struct {
    double m;  /* row maximum                                  */
    double S;  /* normaliser relative to the maximum          */
    int bad;   /* NaN / +inf present, or no finite maximum    */
} row_stats;

static row_stats softmax_stats(const void *base, int dtype, int64_t row_off, int V, double T)
{
    row_stats r;
    r.m = -INFINITY;
    r.S = 0.0;
    r.bad = 0;
    for (int v = 0; v < V; ++v) {
        double l = logit_at(base, dtype, row_off + v);
        if (isnan(l) || (isinf(l) && l > 0)) r.bad = 1;
        if (l > r.m) r.m = l;
    }
    if (r.bad || !isfinite(r.m)) {
        r.bad = 1;
        return r;
    }
    for (int v = 0; v < V; ++v) r.S += exp((logit_at(base, dtype, row_off + v) - r.m) / T);
    return r;
}

/* log p(v) for one token, exact in fp64 without underflow */
static double log_prob(const void *base, int dtype, int64_t row_off, row_stats st, int v, double T)
{
    return (logit_at(base, dtype, row_off + v) - st.m) / T - log(st.S);
}

/* Greedy argmax, ties to the lowest index; *nan_seen set on a NaN. */
static int row_argmax(const void *base, int dtype, int64_t row_off, int V, int *nan_seen)
{
    int best = 0;
    double bv = logit_at(base, dtype, row_off);
    if (isnan(bv)) *nan_seen = 1;
    for (int v = 1; v < V; ++v) {
        double l = logit_at(base, dtype, row_off + v);
        if (isnan(l)) *nan_seen = 1;
        if (l > bv) {
            bv = l;
            best = v;
        }
    }
    return best;
}

/* ------------------------------------------------------------------------ */
/* [Explainer] "Draft and verification loop" / [Leviathan]: accept draft x  */
/* when u * q(x) < p(x).  Evaluated in the log domain so that neither side  */
/* underflows: p(x) == 0 rejects, q(x) == 0 (p > 0) accepts, u == 0 (p > 0) */
/* accepts, otherwise log u + log q < log p.                                */
/* margin = |u - p/q| when p/q < 1, +inf when the outcome cannot depend on  */
/* u (p/q >= 1, p == 0 or q == 0).                                          */
/* ------------------------------------------------------------------------ */
static int accept_test(double lp, double lq, double u, double *margin)
{
    if (lp == -INFINITY) {
        *margin = INFINITY;
        return 0;
    }
    if (lq == -INFINITY || lp >= lq) {
        *margin = INFINITY;
        return 1;
    }
    double ratio = exp(lp - lq); /* in (0, 1) */
    *margin = fabs(u - ratio);
    if (u == 0.0) return 1;
    return log(u) + lq < lp;
}

/* Inverse CDF over non-negative weights w[0..V): smallest v with
 * C_v > u*Z (C_v = w_0 + ... + w_v, left to right).  If rounding leaves no
 * such v, the largest v with w_v > 0.  margin = distance of u*Z from the
 * nearer edge of the chosen bucket, divided by the bucket width. */
static int inverse_cdf(const double *w, int V, double u, double *margin)
{
    double Z = 0.0;
    for (int v = 0; v < V; ++v) Z += w[v];
    double target = u * Z;
    double C = 0.0;
    for (int v = 0; v < V; ++v) {
        double prev = C;
        C += w[v];
        if (C > target) {
            double lo = target - prev, hi = C - target;
            *margin = (lo < hi ? lo : hi) / w[v];
            return v;
        }
    }
    for (int v = V - 1; v >= 0; --v)
        if (w[v] > 0.0) {
            *margin = 0.0;
            return v;
        }
    *margin = 0.0;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Linear verification with given uniforms.                                 */
/*   tl [B][k+1][stride], dl [B][k][stride], x [B][k]                       */
/*   u_acc [B][k]   : u_j for the accept test of draft j                    */
/*   u_smp [B][k+1] : u for the final sample when it happens at position j  */
/* Outputs: out [B][k+1] (-1 padded), acc [B], logp/logq [B][k],            */
/*   acc_margin [B][k], smp_margin [B], err [B].                            */
/* Steps ([Sonar] "Speculative decoding": acceptance, then target           */
/* generation):                                                             */
/*   1. softmax normalisers of all 2k+1 rows;                               */
/*   2. n = first j whose accept test fails, else k;                        */
/*   3. n < k: residual w = max(0, p_n - q_n); n == k: bonus w = exp((l-m)/T)*/
/*      over target row k ([Sonar] "Target-Draft": the target always gives */
/*      one more set of logits after the accepted drafts);                  */
/*   4. out = x_0..x_{n-1}, sampled token, then -1.                         */
/* ------------------------------------------------------------------------ */
int orc_verify_linear_u(const void *tl, const void *dl, int dtype, int64_t stride,
                        const int32_t *x, int B, int k, int V, double T, const double *u_acc,
                        const double *u_smp, int32_t *out, int32_t *acc, double *logp,
                        double *logq, double *acc_margin, double *smp_margin, int32_t *err)
{
    if (B < 0 || k < 1 || V < 1 || !(T > 0.0)) return -1;
    row_stats *ts = (row_stats *)malloc(sizeof(row_stats) * (size_t)(k + 1));
    row_stats *ds = (row_stats *)malloc(sizeof(row_stats) * (size_t)k);
    double *w = (double *)malloc(sizeof(double) * (size_t)V);
    if (!ts || !ds || !w) {
        free(ts); free(ds); free(w);
        return -2;
    }
    for (int b = 0; b < B; ++b) {
        int32_t e = 0;
        const int32_t *xb = x + (int64_t)b * k;
        for (int j = 0; j < k; ++j)
            if (xb[j] < 0 || xb[j] >= V) e |= ORC_ERR_TOKEN;
        for (int j = 0; j <= k; ++j) {
            ts[j] = softmax_stats(tl, dtype, ((int64_t)b * (k + 1) + j) * stride, V, T);
            if (ts[j].bad) e |= ORC_ERR_LOGIT;
        }
        for (int j = 0; j < k; ++j) {
            ds[j] = softmax_stats(dl, dtype, ((int64_t)b * k + j) * stride, V, T);
            if (ds[j].bad) e |= ORC_ERR_LOGIT;
        }
        err[b] = e;
        if (e) {
            for (int j = 0; j <= k; ++j) out[(int64_t)b * (k + 1) + j] = -1;
            acc[b] = -1;
            for (int j = 0; j < k; ++j) {
                logp[(int64_t)b * k + j] = NAN;
                logq[(int64_t)b * k + j] = NAN;
                acc_margin[(int64_t)b * k + j] = INFINITY;
            }
            smp_margin[b] = INFINITY;
            continue;
        }
        int n = k;
        for (int j = 0; j < k; ++j) {
            int64_t toff = ((int64_t)b * (k + 1) + j) * stride;
            int64_t doff = ((int64_t)b * k + j) * stride;
            double lp = log_prob(tl, dtype, toff, ts[j], xb[j], T);
            double lq = log_prob(dl, dtype, doff, ds[j], xb[j], T);
            logp[(int64_t)b * k + j] = lp;
            logq[(int64_t)b * k + j] = lq;
            int ok = accept_test(lp, lq, u_acc[(int64_t)b * k + j], &acc_margin[(int64_t)b * k + j]);
            if (!ok && n == k) n = j;
        }
        int64_t trow = ((int64_t)b * (k + 1) + n) * stride;
        if (n < k) {
            /* [Leviathan] residual norm(max(0, p_n - q_n)) */
            int64_t drow = ((int64_t)b * k + n) * stride;
            double Z = 0.0;
            for (int v = 0; v < V; ++v) {
                double p = exp((logit_at(tl, dtype, trow + v) - ts[n].m) / T) / ts[n].S;
                double q = exp((logit_at(dl, dtype, drow + v) - ds[n].m) / T) / ds[n].S;
                w[v] = p > q ? p - q : 0.0;
                Z += w[v];
            }
            if (!(Z > 0.0)) /* zero residual mass: sample the target row */
                for (int v = 0; v < V; ++v)
                    w[v] = exp((logit_at(tl, dtype, trow + v) - ts[n].m) / T);
        } else {
            for (int v = 0; v < V; ++v)
                w[v] = exp((logit_at(tl, dtype, trow + v) - ts[n].m) / T);
        }
        int tok = inverse_cdf(w, V, u_smp[(int64_t)b * (k + 1) + n], &smp_margin[b]);
        int32_t *ob = out + (int64_t)b * (k + 1);
        for (int j = 0; j < n; ++j) ob[j] = xb[j];
        ob[n] = tok;
        for (int j = n + 1; j <= k; ++j) ob[j] = -1;
        acc[b] = n;
    }
    free(ts); free(ds); free(w);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Greedy (argmax-match) verification.  [Sonar] "Target-Draft": the draft   */
/* samples its top token at each step; the accepted length is the longest   */
/* prefix where the draft equals the target's top token, and the target's   */
/* top token at the first mismatch (or at row k) is emitted.                */
/*   tl [B][k+1][stride], x [B][k]; out [B][k+1], acc [B], err [B].         */
/* ------------------------------------------------------------------------ */
int orc_verify_greedy(const void *tl, int dtype, int64_t stride, const int32_t *x, int B, int k,
                      int V, int32_t *out, int32_t *acc, int32_t *err)
{
    if (B < 0 || k < 1 || V < 1) return -1;
    int *g = (int *)malloc(sizeof(int) * (size_t)(k + 1));
    if (!g) return -2;
    for (int b = 0; b < B; ++b) {
        int32_t e = 0;
        const int32_t *xb = x + (int64_t)b * k;
        for (int j = 0; j < k; ++j)
            if (xb[j] < 0 || xb[j] >= V) e |= ORC_ERR_TOKEN;
        for (int j = 0; j <= k; ++j) {
            int nan_seen = 0;
            g[j] = row_argmax(tl, dtype, ((int64_t)b * (k + 1) + j) * stride, V, &nan_seen);
            if (nan_seen) e |= ORC_ERR_LOGIT;
        }
        err[b] = e;
        int32_t *ob = out + (int64_t)b * (k + 1);
        if (e) {
            for (int j = 0; j <= k; ++j) ob[j] = -1;
            acc[b] = -1;
            continue;
        }
        int n = k;
        for (int j = 0; j < k; ++j)
            if (xb[j] != g[j]) {
                n = j;
                break;
            }
        for (int j = 0; j < n; ++j) ob[j] = xb[j];
        ob[n] = g[n];
        for (int j = n + 1; j <= k; ++j) ob[j] = -1;
        acc[b] = n;
    }
    free(g);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Tree verification ([Sonar] "EAGLE": a tree of top-K candidates; the      */
/* longest acceptable root-to-node sequence is kept plus one target token). */
/*   node 0 is the root (the last committed token, no draft); parents[0]=-1,*/
/*   0 <= parents[i] < i.  Target row i = distribution after node i; draft  */
/*   row i = the draft distribution node i's children were drawn from.      */
/*   test(i), i >= 1, par = parents[i], t = tokens[i]:                      */
/*     greedy:     t == argmax(target row par)                              */
/*     stochastic: u_acc[i] * q_par(t) < p_par(t)                            */
/*   accepted(0) = true; accepted(i) = accepted(par) and test(i).           */
/*   d = deepest accepted node (ties: lowest index); out = tokens on the    */
/*   path root->d (root excluded), then the bonus from target row d        */
/*   (greedy: argmax; stochastic: inverse CDF of exp((l-m)/T) with          */
/*   u_smp[d]), then -1.  acc = depth(d).  path[j] = node at depth j.       */
/*   u_acc [B][N] (entry 0 unused), u_smp [B][N].                           */
/*   acc_margin [B][N] holds each node's test margin (+inf for node 0).     */
/* ------------------------------------------------------------------------ */
int orc_verify_tree_u(const void *tl, const void *dl, int dtype, int64_t stride,
                      const int32_t *tokens, const int32_t *parents, int B, int N, int max_depth,
                      int V, int stochastic, double T, const double *u_acc, const double *u_smp,
                      int32_t *out, int32_t *acc, int32_t *path, double *acc_margin,
                      double *smp_margin, int32_t *err)
{
    if (B < 0 || N < 1 || V < 1 || max_depth < 1) return -1;
    if (stochastic && !(T > 0.0)) return -1;
    int *depth = (int *)malloc(sizeof(int) * (size_t)N);
    int *accd = (int *)malloc(sizeof(int) * (size_t)N);
    int *has_child = (int *)malloc(sizeof(int) * (size_t)N);
    int *g = (int *)malloc(sizeof(int) * (size_t)N);
    row_stats *ts = (row_stats *)malloc(sizeof(row_stats) * (size_t)N);
    row_stats *ds = (row_stats *)malloc(sizeof(row_stats) * (size_t)N);
    double *w = (double *)malloc(sizeof(double) * (size_t)V);
    if (!depth || !accd || !has_child || !g || !ts || !ds || !w) {
        free(depth); free(accd); free(has_child); free(g); free(ts); free(ds); free(w);
        return -2;
    }
    const int W = max_depth + 1;
    for (int b = 0; b < B; ++b) {
        const int32_t *tk = tokens + (int64_t)b * N;
        const int32_t *pa = parents + (int64_t)b * N;
        int32_t e = 0;
        smp_margin[b] = INFINITY;
        for (int i = 0; i < N; ++i) acc_margin[(int64_t)b * N + i] = INFINITY;
        /* structure */
        if (pa[0] != -1) e |= ORC_ERR_TREE;
        depth[0] = 0;
        for (int i = 0; i < N; ++i) has_child[i] = 0;
        for (int i = 1; i < N; ++i) {
            if (pa[i] < 0 || pa[i] >= i) {
                e |= ORC_ERR_TREE;
                depth[i] = 0;
                continue;
            }
            depth[i] = depth[pa[i]] + 1;
            if (depth[i] > max_depth) e |= ORC_ERR_TREE;
            has_child[pa[i]] = 1;
            if (tk[i] < 0 || tk[i] >= V) e |= ORC_ERR_TOKEN;
        }
        /* rows */
        if (!(e & ORC_ERR_TREE)) {
            for (int i = 0; i < N; ++i) {
                int64_t off = ((int64_t)b * N + i) * stride;
                if (stochastic) {
                    ts[i] = softmax_stats(tl, dtype, off, V, T);
                    if (ts[i].bad) e |= ORC_ERR_LOGIT;
                    if (has_child[i]) {
                        ds[i] = softmax_stats(dl, dtype, off, V, T);
                        if (ds[i].bad) e |= ORC_ERR_LOGIT;
                    }
                } else {
                    int nan_seen = 0;
                    g[i] = row_argmax(tl, dtype, off, V, &nan_seen);
                    if (nan_seen) e |= ORC_ERR_LOGIT;
                }
            }
        }
        err[b] = e;
        int32_t *ob = out + (int64_t)b * W;
        int32_t *pb = path ? path + (int64_t)b * W : NULL;
        if (e) {
            for (int j = 0; j < W; ++j) {
                ob[j] = -1;
                if (pb) pb[j] = -1;
            }
            acc[b] = -1;
            continue;
        }
        /* per-node tests and acceptance, in index order (parents come first) */
        accd[0] = 1;
        for (int i = 1; i < N; ++i) {
            int par = pa[i], t = tk[i];
            int ok;
            if (stochastic) {
                int64_t off = ((int64_t)b * N + par) * stride;
                double lp = log_prob(tl, dtype, off, ts[par], t, T);
                double lq = log_prob(dl, dtype, off, ds[par], t, T);
                ok = accept_test(lp, lq, u_acc[(int64_t)b * N + i], &acc_margin[(int64_t)b * N + i]);
            } else {
                ok = (t == g[par]);
            }
            accd[i] = accd[par] && ok;
        }
        int d = 0;
        for (int i = 1; i < N; ++i)
            if (accd[i] && depth[i] > depth[d]) d = i;
        /* path root -> d */
        int D = depth[d];
        for (int j = 0; j < W; ++j) {
            ob[j] = -1;
            if (pb) pb[j] = -1;
        }
        for (int node = d; node != 0; node = pa[node]) {
            ob[depth[node] - 1] = tk[node];
            if (pb) pb[depth[node]] = node;
        }
        if (pb) pb[0] = 0;
        int bonus;
        if (stochastic) {
            int64_t off = ((int64_t)b * N + d) * stride;
            for (int v = 0; v < V; ++v) w[v] = exp((logit_at(tl, dtype, off + v) - ts[d].m) / T);
            bonus = inverse_cdf(w, V, u_smp[(int64_t)b * N + d], &smp_margin[b]);
        } else {
            bonus = g[d];
        }
        ob[D] = bonus;
        acc[b] = D;
    }
    free(depth); free(accd); free(has_child); free(g); free(ts); free(ds); free(w);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Distribution-exact tree verification: recursive rejection over siblings. */
/* The pages give the tree ([Sonar] "EAGLE") and the single-draft rule      */
/* ([Leviathan], [Explainer] "Draft and verification loop"); this mode      */
/* applies that rule to one sibling after another.  Walk from the root; at  */
/* node u, with p the current target distribution (first p_u) and q_u the   */
/* draft distribution u's children were drawn from, test u's children in    */
/* index order against the current p:                                       */
/*   child c, token t, accepted <=> u_acc[c] * q_u(t) < p(t);               */
/*   accepted: c becomes the node (p = p_c) and its children are tested;    */
/*   rejected: p = norm(max(0, p - q_u)) ([Leviathan]'s residual), and the  */
/*   next sibling is tested against it.                                     */
/* When u has no child left (or none), the final token is drawn from the    */
/* current p by the inverse CDF with u_smp[u].  If the children of every    */
/* node are independent draws from q_u, the emitted tokens follow the       */
/* target's distribution, each rejection round being one speculative-       */
/* sampling step against the residual of the last.  Readings: a zero        */
/* residual mass (reachable only through rounding) leaves p unchanged; the  */
/* uniforms are those of orc_verify_tree_u (test of node c: u_acc[c]; draw  */
/* at node d: u_smp[d]).  p is kept as unnormalised weights and their sum,  */
/* so that on a chain every number equals the linear mode's.                */
/* Inputs, checks and outputs as orc_verify_tree_u (stochastic);            */
/* acc_margin[c] holds the margin of every tested child (+inf untested).    */
/* ------------------------------------------------------------------------ */
int orc_verify_tree_exact_u(const void *tl, const void *dl, int dtype, int64_t stride,
                            const int32_t *tokens, const int32_t *parents, int B, int N,
                            int max_depth, int V, double T, const double *u_acc,
                            const double *u_smp, int32_t *out, int32_t *acc, int32_t *path,
                            double *acc_margin, double *smp_margin, int32_t *err)
{
    if (B < 0 || N < 1 || V < 1 || max_depth < 1 || !(T > 0.0)) return -1;
    int *depth = (int *)malloc(sizeof(int) * (size_t)N);
    int *has_child = (int *)malloc(sizeof(int) * (size_t)N);
    row_stats *ts = (row_stats *)malloc(sizeof(row_stats) * (size_t)N);
    row_stats *ds = (row_stats *)malloc(sizeof(row_stats) * (size_t)N);
    double *cur = (double *)malloc(sizeof(double) * (size_t)V);
    double *w = (double *)malloc(sizeof(double) * (size_t)V);
    if (!depth || !has_child || !ts || !ds || !cur || !w) {
        free(depth); free(has_child); free(ts); free(ds); free(cur); free(w);
        return -2;
    }
    const int W = max_depth + 1;
    for (int b = 0; b < B; ++b) {
        const int32_t *tk = tokens + (int64_t)b * N;
        const int32_t *pa = parents + (int64_t)b * N;
        int32_t e = 0;
        smp_margin[b] = INFINITY;
        for (int i = 0; i < N; ++i) acc_margin[(int64_t)b * N + i] = INFINITY;
        if (pa[0] != -1) e |= ORC_ERR_TREE;
        depth[0] = 0;
        for (int i = 0; i < N; ++i) has_child[i] = 0;
        for (int i = 1; i < N; ++i) {
            if (pa[i] < 0 || pa[i] >= i) {
                e |= ORC_ERR_TREE;
                depth[i] = 0;
                continue;
            }
            depth[i] = depth[pa[i]] + 1;
            if (depth[i] > max_depth) e |= ORC_ERR_TREE;
            has_child[pa[i]] = 1;
            if (tk[i] < 0 || tk[i] >= V) e |= ORC_ERR_TOKEN;
        }
        if (!(e & ORC_ERR_TREE)) {
            for (int i = 0; i < N; ++i) {
                int64_t off = ((int64_t)b * N + i) * stride;
                ts[i] = softmax_stats(tl, dtype, off, V, T);
                if (ts[i].bad) e |= ORC_ERR_LOGIT;
                if (has_child[i]) {
                    ds[i] = softmax_stats(dl, dtype, off, V, T);
                    if (ds[i].bad) e |= ORC_ERR_LOGIT;
                }
            }
        }
        err[b] = e;
        int32_t *ob = out + (int64_t)b * W;
        int32_t *pb = path ? path + (int64_t)b * W : NULL;
        for (int j = 0; j < W; ++j) {
            ob[j] = -1;
            if (pb) pb[j] = -1;
        }
        if (e) {
            acc[b] = -1;
            continue;
        }
        int u = 0;
        for (;;) {
            /* p = target row of u: weights exp((l - m)/T), total S */
            int64_t toff = ((int64_t)b * N + u) * stride;
            for (int v = 0; v < V; ++v) cur[v] = exp((logit_at(tl, dtype, toff + v) - ts[u].m) / T);
            double Zc = ts[u].S;
            int residual = 0; /* cur holds a residual (not the target row) */
            int next = -1;
            for (int c = u + 1; c < N && next < 0; ++c) {
                if (pa[c] != u) continue;
                int t = tk[c];
                double lq = log_prob(dl, dtype, toff, ds[u], t, T);
                double lp = residual ? log(cur[t] / Zc) : log_prob(tl, dtype, toff, ts[u], t, T);
                if (accept_test(lp, lq, u_acc[(int64_t)b * N + c], &acc_margin[(int64_t)b * N + c])) {
                    next = c;
                    break;
                }
                /* [Leviathan] residual of the current p against q_u */
                double Z = 0.0;
                for (int v = 0; v < V; ++v) {
                    double pv = cur[v] / Zc;
                    double qv = exp((logit_at(dl, dtype, toff + v) - ds[u].m) / T) / ds[u].S;
                    w[v] = pv > qv ? pv - qv : 0.0;
                    Z += w[v];
                }
                if (Z > 0.0) { /* zero residual mass (rounding only): p unchanged */
                    for (int v = 0; v < V; ++v) cur[v] = w[v];
                    Zc = Z;
                    residual = 1;
                }
            }
            if (next < 0) break;
            u = next;
        }
        int D = depth[u];
        for (int node = u; node != 0; node = pa[node]) {
            ob[depth[node] - 1] = tk[node];
            if (pb) pb[depth[node]] = node;
        }
        if (pb) pb[0] = 0;
        ob[D] = inverse_cdf(cur, V, u_smp[(int64_t)b * N + u], &smp_margin[b]);
        acc[b] = D;
    }
    free(depth); free(has_child); free(ts); free(ds); free(cur); free(w);
    return 0;
}

/* Row statistics helper exposed for tests: log-softmax of one row. */
int orc_log_softmax_row(const void *row, int dtype, int V, double T, double *out_logp)
{
    row_stats st = softmax_stats(row, dtype, 0, V, T);
    if (st.bad) return -1;
    for (int v = 0; v < V; ++v) out_logp[v] = log_prob(row, dtype, 0, st, v, T);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* [Sonar] "MTP schedule for one token": after verification a kernel plugs  */
/* the next target tokens into their positions, so that the accepted count  */
/* never has to reach the CPU before the next step; "MTP": the draft reads  */
/* the target's input tokens shifted one step left of its hidden states    */
/* (the token at position i is the one that follows position i).           */
/*                                                                          */
/* Per request b with n = acc[b] and emitted tokens e_0..e_n = out[b][0..n]: */
/*   next[b][i] = in[b][i + 1] for i < k, i != n (the shifted input; for    */
/*                i > n these are drafts after the first rejection, a       */
/*                don't-care the next draft run processes and discards);    */
/*   next[b][n] = e_n (the drawn token plugged at its position);            */
/*   next[b][k] = e_n when n < k (no shifted token is left there: a pad);   */
/*   seq[b][len[b] + j] = e_j for j <= n, then len[b] += n + 1.             */
/* n = -1 (a request the verification reported as an error): no change to  */
/* seq, next[b][*] = -1.  n outside [-1, k]: the same, plus the token error  */
/* bit.  A sequence without room for n + 1 more tokens (or a negative        */
/* length): seq and len unchanged, next as above, plus ORC_ERR_CAPACITY.    */
/* next and seq may be NULL (then that part is skipped).  Returns the OR of */
/* the error bits (0: none).                                                */
#define ORC_ERR_CAPACITY 16
int orc_plug_tokens(const int32_t *in, const int32_t *out, const int32_t *acc, int B, int k,
                    int32_t *next, int32_t *seq, int32_t *len, int capacity)
{
    int bits = 0;
    for (int b = 0; b < B; ++b) {
        const int32_t *inb = in + (int64_t)b * (k + 1);
        const int32_t *e = out + (int64_t)b * (k + 1);
        int32_t *nb = next ? next + (int64_t)b * (k + 1) : NULL;
        const int n = acc[b];
        if (n < 0 || n > k) {
            if (n != -1) bits |= ORC_ERR_TOKEN;
            if (nb)
                for (int i = 0; i <= k; ++i) nb[i] = -1;
            continue;
        }
        if (nb) {
            for (int i = 0; i < k; ++i) nb[i] = inb[i + 1];
            nb[k] = e[n];
            nb[n] = e[n];
        }
        if (seq) {
            const int L = len[b];
            if (L < 0 || (int64_t)L + n + 1 > (int64_t)capacity) {
                bits |= ORC_ERR_CAPACITY;
                continue;
            }
            int32_t *sb = seq + (int64_t)b * capacity;
            for (int j = 0; j <= n; ++j) sb[L + j] = e[j];
            len[b] = L + n + 1;
        }
    }
    return bits;
}
