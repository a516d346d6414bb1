/*
 * CPU oracle for the forward pass of a sparse, noisy, top-k, capacity-limited
 * Mixture-of-Experts layer.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg load this file's library.  The CUDA path never
 * calls it and shares no code with it.
 *
 * Plain loops and double accumulation, written from the method's definition:
 *   - "Mixture of Experts (MoE) 12段階極小ビジュアル解剖シミュレーター",
 *     STEP 2 (router logits s_raw = W_g x), STEP 4 (s = s_raw + eps),
 *     STEP 5 (KeepTopK: -inf outside the top k), STEP 6 (softmax over the
 *     masked scores), STEP 8-10 (W_up, ReLU, W_down), STEP 11-12 (gate
 *     scaling and weighted sum).
 *   - "nanoMoEの深層解剖", slide 11 (router in full precision, autocast off),
 *     slides 12-13 (topk, -inf scatter, softmax), slide 14 and slides 15-23
 *     (one_hot + cumsum slot rank with all first choices ranked before all
 *     second choices, capacity drop), slides 24-29 and 38-40 (combine with
 *     the pre-drop gate, dropped pairs contribute nothing), slide 32 (the
 *     MLPExperts variant: biases, GELU), slide 14 (used_capacity, extended to
 *     per-expert load statistics).
 *
 * Readings where the pages leave a step open:
 *   - noise: s = fl32(s_raw + fl32(sigma * eps)) with eps ~ N(0,1) supplied;
 *   - top-k order: descending score, ties to the lower expert index;
 *   - capacity: C = min(N, ceil(cf * N * k / E)), cf = +inf means C = N;
 *   - no gate renormalisation after drops; a token with every choice
 *     dropped gets y = 0.
 *
 * Inputs are read at their exact values: fp32 arrays as float, bf16 arrays as
 * their bit patterns widened exactly to float.  Build with -ffp-contract=off
 * so that the two fp32 roundings of the noise step stay separate.
 */
#pragma STDC FP_CONTRACT OFF

#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1 };

static double elem(const void *p, int dt, size_t i)
{
    if (dt == ORACLE_BF16) {
        uint32_t u = (uint32_t)((const uint16_t *)p)[i] << 16;
        float f;
        memcpy(&f, &u, sizeof f);
        return (double)f;
    }
    return (double)((const float *)p)[i];
}

/* STEP 2 / slide 11: s_raw[t][e] = W_g[e] . x[t], summed in double, rounded
 * once to fp32; then the router bias (if any) is added in fp32. */
void oracle_router_logits(const void *x, int dt, const float *W_g, const float *b_g,
                          int64_t N, int d, int E, float *s_raw)
{
    for (int64_t t = 0; t < N; ++t) {
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i)
                acc += elem(x, dt, (size_t)t * d + i) * (double)W_g[(size_t)e * d + i];
            float s = (float)acc;
            if (b_g)
                s = s + b_g[e];
            s_raw[(size_t)t * E + e] = s;
        }
    }
}

/* Order used for KeepTopK: higher score first, equal scores by lower index. */
static const float *g_sort_scores;
static int before(const void *a, const void *b)
{
    int ia = *(const int *)a, ib = *(const int *)b;
    float sa = g_sort_scores[ia], sb = g_sort_scores[ib];
    if (sa > sb) return -1;
    if (sa < sb) return 1;
    return (ia < ib) ? -1 : (ia > ib);
}

/* STEP 3-6 / slides 12-13, starting from the router logits:
 *   s      = fl32(s_raw + fl32(sigma * eps))        (noise; skipped if eps is NULL)
 *   TopK   = the k experts first in (s desc, index asc) order, in that order
 *   gates  = exp(s_j - s_top) / sum_l exp(s_l - s_top) over the kept experts
 *            (the -inf entries contribute exp(-inf) = 0), in double, stored fp32.
 * s_noisy (nullable) receives s. */
void oracle_route_from_logits(const float *s_raw, const float *noise, float sigma,
                              int64_t N, int E, int k,
                              int32_t *topk_idx, float *gates, float *s_noisy)
{
    float *s = (float *)malloc(sizeof(float) * (size_t)E);
    int *idx = (int *)malloc(sizeof(int) * (size_t)E);
    for (int64_t t = 0; t < N; ++t) {
        for (int e = 0; e < E; ++e) {
            float v = s_raw[(size_t)t * E + e];
            if (noise) {
                float scaled = sigma * noise[(size_t)t * E + e];
                v = v + scaled;
            }
            s[e] = v;
            idx[e] = e;
            if (s_noisy)
                s_noisy[(size_t)t * E + e] = v;
        }
        g_sort_scores = s;
        qsort(idx, (size_t)E, sizeof(int), before);
        double top = (double)s[idx[0]];
        double denom = 0.0;
        for (int j = 0; j < k; ++j)
            denom += exp((double)s[idx[j]] - top);
        for (int j = 0; j < k; ++j) {
            topk_idx[(size_t)t * k + j] = idx[j];
            gates[(size_t)t * k + j] = (float)(exp((double)s[idx[j]] - top) / denom);
        }
    }
    free(s);
    free(idx);
}

/* Expert capacity C = min(N, ceil(cf * N * k / E)); cf = +inf gives N.
 * Returns -1 for invalid arguments (cf <= 0 or NaN, k or E out of range). */
int64_t oracle_capacity(int64_t N, int E, int k, double cf)
{
    if (N < 0 || E < 1 || k < 1 || k > E || !(cf > 0.0))
        return -1;
    if (isinf(cf))
        return N;
    double c = ceil(cf * (double)N * (double)k / (double)E);
    if (c > (double)N)
        return N;
    return (int64_t)c;
}

/* Slides 14-23: an assignment's place in its expert's queue is the number of
 * earlier assignments to the same expert, where every token's j-th choice
 * comes before every token's (j+1)-th choice and tokens keep their order
 * within one choice rank.  Places >= C are dropped (slot -1).
 * counts[e] is the number of kept assignments of expert e (used_capacity). */
void oracle_assign_slots(const int32_t *topk_idx, int64_t N, int E, int k, int64_t C,
                         int32_t *slot, int32_t *counts)
{
    int64_t *queue = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    for (int j = 0; j < k; ++j) {
        for (int64_t t = 0; t < N; ++t) {
            int e = topk_idx[(size_t)t * k + j];
            int64_t place = queue[e]++;
            slot[(size_t)t * k + j] = (place < C) ? (int32_t)place : -1;
        }
    }
    for (int e = 0; e < E; ++e)
        counts[e] = (int32_t)(queue[e] < C ? queue[e] : C);
    free(queue);
}

/* Backward of the layer for a given routing.  "Mixture of Experts (MoE)
 * 12段階極小ビジュアル解剖シミュレーター" STEP 6 (the -inf mask keeps the kept
 * experts' softmax differentiable and gives the others gate 0) and STEP 11
 * (g_i E_i(x) carries the gradient to the router); the top-k indices and the
 * slots are piecewise constant and carry none.  With L = sum over t, i of
 * dy[t, i] y[t, i]:
 *   kept (t, j), e = topk[t, j]:  z = W_up[e] x_t,  h = ReLU(z),  o = W_down[e] h
 *     dg_j = dy_t . o,   d_o = g_j dy_t
 *     dW_down[e] += d_o h^T,  dz = (W_down[e]^T d_o) * [z > 0],
 *     dW_up[e] += dz x_t^T,   dx_t += W_up[e]^T dz
 *   dropped (t, j): dg_j = 0 (its gate multiplies nothing)
 *   every chosen (t, j): ds_j = g_j (dg_j - sum_l g_l dg_l)   (softmax over the k
 *     chosen scores, capacity drops included, as the gates are formed before the cut)
 *     db_g[e] += ds_j,  dW_g[e] += ds_j x_t,  dx_t += ds_j W_g[e]
 * s [N, E] fp32 are the noisy scores the gates came from (s = s_raw + sigma eps:
 * ds_raw = ds); the gates are recomputed from them in double.  dy [N, d] double.
 * relu_mask (nullable, [N, k, d_ff] bytes): the ReLU decisions [z > 0] of the
 * kept pairs taken from elsewhere (another implementation's rounding of z),
 * replayed in place of the sign of this oracle's own z: h = mask ? z : 0 and
 * dz = mask ? W_down^T d_o : 0.  With NULL the oracle decides.
 * Outputs are double and overwritten: dx [N, d], dW_g [E, d], db_g [E],
 * dW_up [E, d_ff, d], dW_down [E, d, d_ff]. */
void oracle_backward(const void *x, int dt, const float *W_g, const void *W_up, const void *W_down,
                     const float *s, const int32_t *topk_idx, const int32_t *slot, const double *dy,
                     int64_t N, int d, int E, int d_ff, int k, const uint8_t *relu_mask,
                     double *dx, double *dW_g, double *db_g, double *dW_up, double *dW_down)
{
    memset(dx, 0, sizeof(double) * (size_t)N * d);
    memset(dW_g, 0, sizeof(double) * (size_t)E * d);
    memset(db_g, 0, sizeof(double) * (size_t)E);
    memset(dW_up, 0, sizeof(double) * (size_t)E * d_ff * d);
    memset(dW_down, 0, sizeof(double) * (size_t)E * d * d_ff);
    double *g = (double *)malloc(sizeof(double) * (size_t)k);
    double *dg = (double *)malloc(sizeof(double) * (size_t)k);
    double *z = (double *)malloc(sizeof(double) * (size_t)d_ff);
    double *h = (double *)malloc(sizeof(double) * (size_t)d_ff);
    double *dz = (double *)malloc(sizeof(double) * (size_t)d_ff);
    double *o = (double *)malloc(sizeof(double) * (size_t)d);
    for (int64_t t = 0; t < N; ++t) {
        const int32_t *ti = topk_idx + (size_t)t * k;
        const double top = (double)s[(size_t)t * E + ti[0]];
        double denom = 0.0;
        for (int j = 0; j < k; ++j)
            denom += exp((double)s[(size_t)t * E + ti[j]] - top);
        for (int j = 0; j < k; ++j)
            g[j] = exp((double)s[(size_t)t * E + ti[j]] - top) / denom;
        const double *dyt = dy + (size_t)t * d;
        double *dxt = dx + (size_t)t * d;
        for (int j = 0; j < k; ++j) {
            dg[j] = 0.0;
            if (slot[(size_t)t * k + j] < 0)
                continue;
            const int e = ti[j];
            const uint8_t *mk = relu_mask ? relu_mask + ((size_t)t * k + j) * d_ff : NULL;
            for (int f = 0; f < d_ff; ++f) {
                double acc = 0.0;
                for (int i = 0; i < d; ++i)
                    acc += elem(W_up, dt, ((size_t)e * d_ff + f) * d + i) * elem(x, dt, (size_t)t * d + i);
                z[f] = acc;
                const int on = mk ? (mk[f] != 0) : (acc > 0.0);
                h[f] = on ? acc : 0.0;
            }
            for (int i = 0; i < d; ++i) {
                double acc = 0.0;
                for (int f = 0; f < d_ff; ++f)
                    acc += elem(W_down, dt, ((size_t)e * d + i) * d_ff + f) * h[f];
                o[i] = acc;
                dg[j] += dyt[i] * acc;
            }
            for (int f = 0; f < d_ff; ++f) {
                double acc = 0.0;
                for (int i = 0; i < d; ++i) {
                    const double d_o = g[j] * dyt[i];
                    dW_down[((size_t)e * d + i) * d_ff + f] += d_o * h[f];
                    acc += elem(W_down, dt, ((size_t)e * d + i) * d_ff + f) * d_o;
                }
                dz[f] = (mk ? (mk[f] != 0) : (z[f] > 0.0)) ? acc : 0.0;
            }
            for (int f = 0; f < d_ff; ++f)
                for (int i = 0; i < d; ++i) {
                    dW_up[((size_t)e * d_ff + f) * d + i] += dz[f] * elem(x, dt, (size_t)t * d + i);
                    dxt[i] += elem(W_up, dt, ((size_t)e * d_ff + f) * d + i) * dz[f];
                }
        }
        double sum = 0.0;
        for (int j = 0; j < k; ++j)
            sum += g[j] * dg[j];
        for (int j = 0; j < k; ++j) {
            const double ds = g[j] * (dg[j] - sum);
            const int e = ti[j];
            db_g[e] += ds;
            for (int i = 0; i < d; ++i) {
                dW_g[(size_t)e * d + i] += ds * elem(x, dt, (size_t)t * d + i);
                dxt[i] += ds * (double)W_g[(size_t)e * d + i];
            }
        }
    }
    free(g);
    free(dg);
    free(z);
    free(h);
    free(dz);
    free(o);
}

/* ------------------------------------------------------------------ sampled backward
 * The quantities of oracle_backward at listed places only, for batches where
 * the whole backward is too slow on a CPU: dx rows of listed tokens, rows f of
 * dW_up[e] and columns f of dW_down[e] for listed (e, f), and all of dW_g and
 * db_g.  Each listed value is summed in the same order as in oracle_backward
 * (tokens ascending, then choices), so the two agree exactly.
 *   tokens [n_tokens] -> dx_rows [n_tokens, d]
 *   ef [n_ef, 2] (expert, f) -> dW_up_rows [n_ef, d] (= dW_up[e][f][:]) and
 *                               dW_down_cols [n_ef, d] (= dW_down[e][:][f])
 * The gate gradients of every kept pair (dg = dy . o) need every expert
 * output, which is the expensive part: it runs on nthreads threads, split over
 * tokens; the listed rows and columns are split over threads the same way. */
struct bwd_ctx {
    const void *x, *W_up, *W_down;
    int dt;
    const float *W_g, *s;
    const int32_t *topk_idx, *slot;
    const double *dy;
    int64_t N;
    int d, E, d_ff, k;
    const uint8_t *relu_mask;
    double *g, *dg, *ds;           /* [N, k] */
    const int64_t *tokens;
    const int32_t *ef;
    double *dx_rows, *dW_up_rows, *dW_down_cols;
};

struct bwd_job {
    struct bwd_ctx *c;
    int64_t begin, end;
};

static int relu_on(const struct bwd_ctx *c, int64_t t, int j, int f, double z)
{
    if (c->relu_mask)
        return c->relu_mask[((size_t)t * c->k + j) * c->d_ff + f] != 0;
    return z > 0.0;
}

static double up_dot(const struct bwd_ctx *c, int e, int f, int64_t t)
{
    double acc = 0.0;
    for (int i = 0; i < c->d; ++i)
        acc += elem(c->W_up, c->dt, ((size_t)e * c->d_ff + f) * c->d + i) * elem(c->x, c->dt, (size_t)t * c->d + i);
    return acc;
}

/* gates (recomputed in double from s) and dg = dy . o of every kept pair */
static void *bwd_gate_grads(void *arg)
{
    struct bwd_job *jb = (struct bwd_job *)arg;
    struct bwd_ctx *c = jb->c;
    double *h = (double *)malloc(sizeof(double) * (size_t)c->d_ff);
    for (int64_t t = jb->begin; t < jb->end; ++t) {
        const int32_t *ti = c->topk_idx + (size_t)t * c->k;
        const double top = (double)c->s[(size_t)t * c->E + ti[0]];
        double denom = 0.0;
        for (int j = 0; j < c->k; ++j)
            denom += exp((double)c->s[(size_t)t * c->E + ti[j]] - top);
        for (int j = 0; j < c->k; ++j)
            c->g[(size_t)t * c->k + j] = exp((double)c->s[(size_t)t * c->E + ti[j]] - top) / denom;
        const double *dyt = c->dy + (size_t)t * c->d;
        for (int j = 0; j < c->k; ++j) {
            double dgj = 0.0;
            if (c->slot[(size_t)t * c->k + j] >= 0) {
                const int e = ti[j];
                for (int f = 0; f < c->d_ff; ++f) {
                    const double z = up_dot(c, e, f, t);
                    h[f] = relu_on(c, t, j, f, z) ? z : 0.0;
                }
                for (int i = 0; i < c->d; ++i) {
                    double acc = 0.0;
                    for (int f = 0; f < c->d_ff; ++f)
                        acc += elem(c->W_down, c->dt, ((size_t)e * c->d + i) * c->d_ff + f) * h[f];
                    dgj += dyt[i] * acc;
                }
            }
            c->dg[(size_t)t * c->k + j] = dgj;
        }
    }
    free(h);
    return NULL;
}

/* dx rows of the listed tokens, in oracle_backward's order */
static void *bwd_dx_rows(void *arg)
{
    struct bwd_job *jb = (struct bwd_job *)arg;
    struct bwd_ctx *c = jb->c;
    const int d = c->d, d_ff = c->d_ff, k = c->k;
    double *z = (double *)malloc(sizeof(double) * (size_t)d_ff);
    double *dz = (double *)malloc(sizeof(double) * (size_t)d_ff);
    for (int64_t r = jb->begin; r < jb->end; ++r) {
        const int64_t t = c->tokens[r];
        const int32_t *ti = c->topk_idx + (size_t)t * k;
        const double *dyt = c->dy + (size_t)t * d;
        double *dxt = c->dx_rows + (size_t)r * d;
        for (int i = 0; i < d; ++i)
            dxt[i] = 0.0;
        for (int j = 0; j < k; ++j) {
            if (c->slot[(size_t)t * k + j] < 0)
                continue;
            const int e = ti[j];
            const double gj = c->g[(size_t)t * k + j];
            for (int f = 0; f < d_ff; ++f)
                z[f] = up_dot(c, e, f, t);
            for (int f = 0; f < d_ff; ++f) {
                double acc = 0.0;
                for (int i = 0; i < d; ++i)
                    acc += elem(c->W_down, c->dt, ((size_t)e * d + i) * d_ff + f) * (gj * dyt[i]);
                dz[f] = relu_on(c, t, j, f, z[f]) ? acc : 0.0;
            }
            for (int f = 0; f < d_ff; ++f)
                for (int i = 0; i < d; ++i)
                    dxt[i] += elem(c->W_up, c->dt, ((size_t)e * d_ff + f) * d + i) * dz[f];
        }
        for (int j = 0; j < k; ++j) {
            const double dsj = c->ds[(size_t)t * k + j];
            const int e = ti[j];
            for (int i = 0; i < d; ++i)
                dxt[i] += dsj * (double)c->W_g[(size_t)e * d + i];
        }
    }
    free(z);
    free(dz);
    return NULL;
}

/* row f of dW_up[e] and column f of dW_down[e] for the listed (e, f) */
static void *bwd_weight_rows(void *arg)
{
    struct bwd_job *jb = (struct bwd_job *)arg;
    struct bwd_ctx *c = jb->c;
    const int d = c->d, d_ff = c->d_ff, k = c->k;
    for (int64_t q = jb->begin; q < jb->end; ++q) {
        const int e = c->ef[2 * q], f = c->ef[2 * q + 1];
        double *wu = c->dW_up_rows + (size_t)q * d;
        double *wd = c->dW_down_cols + (size_t)q * d;
        for (int i = 0; i < d; ++i)
            wu[i] = wd[i] = 0.0;
        for (int64_t t = 0; t < c->N; ++t) {
            for (int j = 0; j < k; ++j) {
                if (c->topk_idx[(size_t)t * k + j] != e || c->slot[(size_t)t * k + j] < 0)
                    continue;
                const double gj = c->g[(size_t)t * k + j];
                const double *dyt = c->dy + (size_t)t * d;
                const double z = up_dot(c, e, f, t);
                const int on = relu_on(c, t, j, f, z);
                const double hf = on ? z : 0.0;
                double acc = 0.0;
                for (int i = 0; i < d; ++i) {
                    const double d_o = gj * dyt[i];
                    wd[i] += d_o * hf;
                    acc += elem(c->W_down, c->dt, ((size_t)e * d + i) * d_ff + f) * d_o;
                }
                const double dzf = on ? acc : 0.0;
                for (int i = 0; i < d; ++i)
                    wu[i] += dzf * elem(c->x, c->dt, (size_t)t * d + i);
            }
        }
    }
    return NULL;
}

static void bwd_run(void *(*fn)(void *), struct bwd_ctx *c, int64_t n, int nthreads)
{
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > n)
        nthreads = n > 0 ? (int)n : 1;
    struct bwd_job *jobs = (struct bwd_job *)calloc((size_t)nthreads, sizeof *jobs);
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof *th);
    for (int w = 0; w < nthreads; ++w) {
        jobs[w].c = c;
        jobs[w].begin = n * w / nthreads;
        jobs[w].end = n * (w + 1) / nthreads;
    }
    if (nthreads == 1) {
        fn(&jobs[0]);
    } else {
        for (int w = 0; w < nthreads; ++w)
            pthread_create(&th[w], NULL, fn, &jobs[w]);
        for (int w = 0; w < nthreads; ++w)
            pthread_join(th[w], NULL);
    }
    free(jobs);
    free(th);
}

void oracle_backward_sampled(const void *x, int dt, const float *W_g, const void *W_up, const void *W_down,
                             const float *s, const int32_t *topk_idx, const int32_t *slot, const double *dy,
                             int64_t N, int d, int E, int d_ff, int k, const uint8_t *relu_mask,
                             const int64_t *tokens, int64_t n_tokens, const int32_t *ef, int64_t n_ef,
                             int nthreads, double *dx_rows, double *dW_g, double *db_g, double *dW_up_rows,
                             double *dW_down_cols)
{
    struct bwd_ctx c;
    memset(&c, 0, sizeof c);
    c.x = x; c.W_up = W_up; c.W_down = W_down; c.dt = dt; c.W_g = W_g; c.s = s;
    c.topk_idx = topk_idx; c.slot = slot; c.dy = dy; c.N = N; c.d = d; c.E = E; c.d_ff = d_ff; c.k = k;
    c.relu_mask = relu_mask; c.tokens = tokens; c.ef = ef;
    c.dx_rows = dx_rows; c.dW_up_rows = dW_up_rows; c.dW_down_cols = dW_down_cols;
    c.g = (double *)malloc(sizeof(double) * (size_t)(N * k + 1));
    c.dg = (double *)malloc(sizeof(double) * (size_t)(N * k + 1));
    c.ds = (double *)malloc(sizeof(double) * (size_t)(N * k + 1));
    bwd_run(bwd_gate_grads, &c, N, nthreads);
    /* router gradients, in oracle_backward's order */
    memset(dW_g, 0, sizeof(double) * (size_t)E * d);
    memset(db_g, 0, sizeof(double) * (size_t)E);
    for (int64_t t = 0; t < N; ++t) {
        double sum = 0.0;
        for (int j = 0; j < k; ++j)
            sum += c.g[(size_t)t * k + j] * c.dg[(size_t)t * k + j];
        for (int j = 0; j < k; ++j) {
            const double dsj = c.g[(size_t)t * k + j] * (c.dg[(size_t)t * k + j] - sum);
            c.ds[(size_t)t * k + j] = dsj;
            const int e = topk_idx[(size_t)t * k + j];
            db_g[e] += dsj;
            for (int i = 0; i < d; ++i)
                dW_g[(size_t)e * d + i] += dsj * elem(x, dt, (size_t)t * d + i);
        }
    }
    bwd_run(bwd_dx_rows, &c, n_tokens, nthreads);
    bwd_run(bwd_weight_rows, &c, n_ef, nthreads);
    free(c.g);
    free(c.dg);
    free(c.ds);
}

/* Per-expert load of one routed batch ("nanoMoEの深層解剖" slide 14: the
 * router's used_capacity counts each expert's rows that survive the capacity
 * cut).  load[e]: choices (t, j) that picked e, before the cut; used[e] =
 * min(load[e], C); importance[e] (skipped if gates or importance is NULL):
 * the sum of those choices' gates, each gate taken as the nearest multiple of
 * 2^-32 (ties to even), summed exactly in 64-bit integers, then scaled back. */
void oracle_load_stats(const int32_t *topk_idx, const float *gates, int64_t N, int E, int k, int64_t C,
                       int32_t *load, int32_t *used, double *importance)
{
    int64_t *q = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    int64_t *mass = (int64_t *)calloc((size_t)E, sizeof(int64_t));
    for (int64_t t = 0; t < N; ++t) {
        for (int j = 0; j < k; ++j) {
            int e = topk_idx[(size_t)t * k + j];
            if (e < 0 || e >= E)
                continue;
            q[e] += 1;
            if (gates)
                mass[e] += llrint(ldexp((double)gates[(size_t)t * k + j], 32));
        }
    }
    for (int e = 0; e < E; ++e) {
        load[e] = (int32_t)q[e];
        used[e] = (int32_t)(q[e] < C ? q[e] : C);
        if (gates && importance)
            importance[e] = ldexp((double)mass[e], -32);
    }
    free(q);
    free(mass);
}

/* The nanoMoE expert variant ("nanoMoEの深層解剖" slide 32, MLPExperts): an
 * optional bias after each projection and GELU in place of ReLU.  GELU is the
 * exact form x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2)), in double.
 *   z = W_up[e] x + b_up[e],  h = act(z),  o = W_down[e] h + b_down[e]
 * act: 1 = ReLU, 2 = GELU.  b_up [E][d_ff] and b_down [E][d] are fp32 or NULL. */
void oracle_expert_ffn_ex(const void *x, int dt, const void *W_up, const void *W_down,
                          const float *b_up, const float *b_down, int act,
                          int64_t t, int e, int d, int d_ff, double *h, double *o)
{
    for (int f = 0; f < d_ff; ++f) {
        double z = 0.0;
        size_t wrow = ((size_t)e * d_ff + f) * d;
        for (int i = 0; i < d; ++i)
            z += elem(W_up, dt, wrow + i) * elem(x, dt, (size_t)t * d + i);
        if (b_up)
            z += (double)b_up[(size_t)e * d_ff + f];
        if (act == 2)
            h[f] = 0.5 * z * (1.0 + erf(z / sqrt(2.0)));
        else
            h[f] = z > 0.0 ? z : 0.0;
    }
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        size_t wrow = ((size_t)e * d + i) * d_ff;
        for (int f = 0; f < d_ff; ++f)
            acc += elem(W_down, dt, wrow + f) * h[f];
        if (b_down)
            acc += (double)b_down[(size_t)e * d + i];
        o[i] = acc;
    }
}

/* STEP 8-10 for one token and one expert, in double:
 *   z = W_up[e] x,  h = max(0, z),  o = W_down[e] h. */
void oracle_expert_ffn(const void *x, int dt, const void *W_up, const void *W_down,
                       int64_t t, int e, int d, int d_ff, double *h, double *o)
{
    oracle_expert_ffn_ex(x, dt, W_up, W_down, NULL, NULL, 1, t, e, d, d_ff, h, o);
}

struct combine_job {
    const void *x, *W_up, *W_down;
    const float *b_up, *b_down;
    int act;
    int dt;
    const int32_t *topk_idx, *slot;
    const float *gates;
    int d, d_ff, k;
    const int64_t *tokens;
    int64_t begin, end;
    double *y;
};

/* STEP 11-12 / slides 38-40: y[t] = sum over kept choices j of
 * gates[t][j] * E_{e_j}(x[t]); a dropped choice adds nothing and the kept
 * gates are not renormalised. */
static void *combine_range(void *arg)
{
    struct combine_job *jb = (struct combine_job *)arg;
    double *h = (double *)malloc(sizeof(double) * (size_t)jb->d_ff);
    double *o = (double *)malloc(sizeof(double) * (size_t)jb->d);
    for (int64_t r = jb->begin; r < jb->end; ++r) {
        int64_t t = jb->tokens[r];
        double *yt = jb->y + (size_t)r * jb->d;
        for (int i = 0; i < jb->d; ++i)
            yt[i] = 0.0;
        for (int j = 0; j < jb->k; ++j) {
            if (jb->slot[(size_t)t * jb->k + j] < 0)
                continue;
            int e = jb->topk_idx[(size_t)t * jb->k + j];
            double g = (double)jb->gates[(size_t)t * jb->k + j];
            oracle_expert_ffn_ex(jb->x, jb->dt, jb->W_up, jb->W_down, jb->b_up, jb->b_down, jb->act, t, e,
                                 jb->d, jb->d_ff, h, o);
            for (int i = 0; i < jb->d; ++i)
                yt[i] += g * o[i];
        }
    }
    free(h);
    free(o);
    return NULL;
}

/* Layer output for the listed tokens (y rows in list order, double), with the
 * expert variant of oracle_expert_ffn_ex (act 1 = ReLU, 2 = GELU; biases nullable).
 * Work is split over tokens across nthreads plain threads; each token's
 * arithmetic is the same as with one thread. */
void oracle_ffn_combine_ex(const void *x, int dt, const void *W_up, const void *W_down,
                           const float *b_up, const float *b_down, int act,
                           const int32_t *topk_idx, const float *gates, const int32_t *slot,
                           int d, int d_ff, int k, const int64_t *tokens, int64_t n_tokens,
                           double *y, int nthreads)
{
    if (nthreads < 1)
        nthreads = 1;
    if (nthreads > n_tokens)
        nthreads = n_tokens > 0 ? (int)n_tokens : 1;
    struct combine_job *jobs = (struct combine_job *)calloc((size_t)nthreads, sizeof *jobs);
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof *th);
    for (int w = 0; w < nthreads; ++w) {
        struct combine_job *jb = &jobs[w];
        jb->x = x; jb->W_up = W_up; jb->W_down = W_down; jb->dt = dt;
        jb->b_up = b_up; jb->b_down = b_down; jb->act = act;
        jb->topk_idx = topk_idx; jb->slot = slot; jb->gates = gates;
        jb->d = d; jb->d_ff = d_ff; jb->k = k; jb->tokens = tokens; jb->y = y;
        jb->begin = n_tokens * w / nthreads;
        jb->end = n_tokens * (w + 1) / nthreads;
    }
    if (nthreads == 1) {
        combine_range(&jobs[0]);
    } else {
        for (int w = 0; w < nthreads; ++w)
            pthread_create(&th[w], NULL, combine_range, &jobs[w]);
        for (int w = 0; w < nthreads; ++w)
            pthread_join(th[w], NULL);
    }
    free(jobs);
    free(th);
}

/* The layer as the walkthrough defines it: ReLU experts, no biases. */
void oracle_ffn_combine(const void *x, int dt, const void *W_up, const void *W_down,
                        const int32_t *topk_idx, const float *gates, const int32_t *slot,
                        int d, int d_ff, int k, const int64_t *tokens, int64_t n_tokens,
                        double *y, int nthreads)
{
    oracle_ffn_combine_ex(x, dt, W_up, W_down, NULL, NULL, 1, topk_idx, gates, slot, d, d_ff, k,
                          tokens, n_tokens, y, nthreads);
}
