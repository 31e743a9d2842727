/*
 * fp64 CPU oracle for gated triangle self-attention with pair bias.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or load
 * this file; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do. It shares no code, header or constant with the CUDA library.
 *
 * What it computes. The pages describe the operation only in words: triangle
 * attention lets the model use a third residue when it reasons about a pair,
 * at a cost cubic in the crop size, and its backward yields gradients for
 * query, key, value and pair bias ("TurboPairFormer accelera fino a 1,73×
 * l'addestramento di OpenFold3 nei test", section "Dove si impiega il tempo").
 * No page prints a formula. This file takes the standard AlphaFold-family
 * definition of gated triangle self-attention with pair bias, the gate applied
 * per channel; for every attention row r, head h and query x:
 *
 *   s_y  = c^-1/2 * sum_c q[r,x,h,c] k[r,y,h,c] + b[h,x,y] + mu(r,y)
 *   lse  = log sum_y exp(s_y)             (plain two-pass: max, then sum)
 *   p_y  = exp(s_y - lse)
 *   u    = sum_y p_y v[r,y,h,:]
 *   out  = sigmoid(g[r,x,h,:]) * u
 *
 * mu(r,y) is 0 when mask[r*mask_row_stride + y] != 0 and -inf otherwise; a row
 * whose keys are all masked has lse = -inf, p = 0, u = 0 and contributes
 * nothing to any gradient.
 *
 * Backward of L = sum(dout * out), written from the chain rule:
 *   du    = dout * sigmoid(g)              dgate = dout * u * s(1 - s)
 *   D_x   = sum_c du_x u_x                 dp_xy = sum_c du_x v_y
 *   ds_xy = p_xy (dp_xy - D_x)
 *   dq_x  = c^-1/2 sum_y ds_xy k_y         dk_y  = c^-1/2 sum_x ds_xy q_x
 *   dv_y  = sum_x p_xy du_x                dbias[h,x,y] = sum_r ds_xy
 *
 * Variants. "Starting node": row r = i, query x = j, key y = k, so pair
 * tensors are read at [r, x] and the bias at [h, x, y]. "Ending node" is the
 * same computation on the transposed pair layout: pair tensors are read at
 * [x, r], the bias at [h, y, x] and dbias is written back transposed. The key
 * mask and lse are always indexed in the variant's own frame (row r, key y /
 * row r, head h, query x).
 *
 * All floating-point inputs arrive as float32 (which holds bf16 values exactly);
 * all arithmetic is fp64 with libm exp/log.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <omp.h>

typedef struct {
    int64_t N;
    int H, C, variant;
    const float *q, *k, *v, *bias, *gate, *dout;
    const uint8_t *mask;
    int64_t mask_row_stride;
} prob_t;

/* Offset of element [.., c=0] of the pair tensor entry (row r, query/key x). */
static int64_t pair_at(const prob_t *p, int64_t r, int64_t x, int h)
{
    int64_t a = (p->variant == 0) ? r : x;
    int64_t b = (p->variant == 0) ? x : r;
    return ((a * p->N + b) * p->H + h) * (int64_t)p->C;
}

/* Offset of the bias entry used by query x and key y of head h. */
static int64_t bias_at(const prob_t *p, int h, int64_t x, int64_t y)
{
    if (p->variant == 0) return ((int64_t)h * p->N + x) * p->N + y;
    return ((int64_t)h * p->N + y) * p->N + x;
}

static int key_kept(const prob_t *p, int64_t r, int64_t y)
{
    if (!p->mask) return 1;
    return p->mask[r * p->mask_row_stride + y] != 0;
}

static double sigmoid(double g) { return 1.0 / (1.0 + exp(-g)); }

/*
 * One query of one attention row: fills prob[0..N) with p_y, u[0..C) with the
 * ungated output and returns lse (-INFINITY when every key is masked).
 */
static double query_forward(const prob_t *p, int64_t r, int h, int64_t x,
                            double *prob, double *u)
{
    const int64_t N = p->N;
    const int C = p->C;
    const double scale = 1.0 / sqrt((double)C);
    const float *qx = p->q + pair_at(p, r, x, h);
    int any = 0;
    double m = -INFINITY;
    for (int64_t y = 0; y < N; ++y) {
        if (!key_kept(p, r, y)) { prob[y] = 0.0; continue; }
        const float *ky = p->k + pair_at(p, r, y, h);
        double dot = 0.0;
        for (int c = 0; c < C; ++c) dot += (double)qx[c] * (double)ky[c];
        double s = scale * dot + (double)p->bias[bias_at(p, h, x, y)];
        prob[y] = s;                      /* holds the logit for now */
        if (!any || s > m) m = s;
        any = 1;
    }
    for (int c = 0; c < C; ++c) u[c] = 0.0;
    if (!any) return -INFINITY;
    double z = 0.0;
    for (int64_t y = 0; y < N; ++y)
        if (key_kept(p, r, y)) z += exp(prob[y] - m);
    const double lse = m + log(z);
    for (int64_t y = 0; y < N; ++y) {
        if (!key_kept(p, r, y)) continue;
        prob[y] = exp(prob[y] - lse);
        const float *vy = p->v + pair_at(p, r, y, h);
        for (int c = 0; c < C; ++c) u[c] += prob[y] * (double)vy[c];
    }
    return lse;
}

static prob_t make_prob(int64_t N, int H, int C, int variant, const float *q,
                        const float *k, const float *v, const float *bias,
                        const float *gate, const float *dout, const uint8_t *mask,
                        int64_t mask_row_stride)
{
    prob_t p;
    p.N = N; p.H = H; p.C = C; p.variant = variant;
    p.q = q; p.k = k; p.v = v; p.bias = bias; p.gate = gate; p.dout = dout;
    p.mask = mask; p.mask_row_stride = mask_row_stride;
    return p;
}

static int check(int64_t N, int H, int C, int variant)
{
    if (N < 0 || H <= 0 || C <= 0 || (variant != 0 && variant != 1)) return 1;
    return 0;
}

int tri_oracle_version(void) { return 1; }

/*
 * Forward for the listed attention rows (variant frame). Outputs are compact:
 * out[n][x][h][c] and lse[n][h][x] for n in [0, n_rows).
 */
int tri_oracle_fwd(int64_t N, int H, int C, int variant, const float *q,
                   const float *k, const float *v, const float *bias,
                   const float *gate, const uint8_t *mask, int64_t mask_row_stride,
                   const int64_t *rows, int64_t n_rows, double *out, double *lse)
{
    if (check(N, H, C, variant)) return 1;
    prob_t p = make_prob(N, H, C, variant, q, k, v, bias, gate, NULL, mask,
                         mask_row_stride);
    const int64_t units = n_rows * H * N;
#pragma omp parallel
    {
        double *prob = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        double *u = (double *)malloc(sizeof(double) * (size_t)C);
#pragma omp for schedule(static)
        for (int64_t w = 0; w < units; ++w) {
            const int64_t n = w / (H * N);
            const int h = (int)((w / N) % H);
            const int64_t x = w % N;
            const int64_t r = rows[n];
            const double l = query_forward(&p, r, h, x, prob, u);
            const float *gx = gate + pair_at(&p, r, x, h);
            double *o = out + ((n * N + x) * H + h) * (int64_t)C;
            for (int c = 0; c < C; ++c) o[c] = sigmoid((double)gx[c]) * u[c];
            lse[(n * H + h) * N + x] = l;
        }
        free(prob);
        free(u);
    }
    return 0;
}

/* Probabilities p[x][y] of one attention row r and head h (small N only). */
int tri_oracle_probs(int64_t N, int H, int C, int variant, const float *q,
                     const float *k, const float *v, const float *bias,
                     const uint8_t *mask, int64_t mask_row_stride, int64_t r, int h,
                     double *P)
{
    if (check(N, H, C, variant)) return 1;
    prob_t p = make_prob(N, H, C, variant, q, k, v, bias, NULL, NULL, mask,
                         mask_row_stride);
    double *u = (double *)malloc(sizeof(double) * (size_t)C);
    for (int64_t x = 0; x < N; ++x) query_forward(&p, r, h, x, P + x * N, u);
    free(u);
    return 0;
}

/*
 * Backward for the listed attention rows. dq, dk, dv, dgate are compact
 * [n][x][h][c] in the variant frame; dbias (storage layout [H][N][N]) receives
 * the sum over the listed rows only (all rows gives the full dbias). The sum
 * over rows is taken per thread over a static partition and the partial sums
 * are added in thread order.
 */
int tri_oracle_bwd(int64_t N, int H, int C, int variant, const float *q,
                   const float *k, const float *v, const float *bias,
                   const float *gate, const uint8_t *mask, int64_t mask_row_stride,
                   const float *dout, const int64_t *rows, int64_t n_rows,
                   double *dq, double *dk, double *dv, double *dgate, double *dbias)
{
    if (check(N, H, C, variant)) return 1;
    prob_t p = make_prob(N, H, C, variant, q, k, v, bias, gate, dout, mask,
                         mask_row_stride);
    const double scale = 1.0 / sqrt((double)C);
    const int64_t units = n_rows * H;
    const int64_t nb = (int64_t)H * N * N;
    int nthreads = omp_get_max_threads();
    if (nthreads < 1) nthreads = 1;
    double *part = (double *)calloc((size_t)nthreads * (size_t)(nb > 0 ? nb : 1),
                                    sizeof(double));
    if (!part) return 2;
#pragma omp parallel num_threads(nthreads)
    {
        const int t = omp_get_thread_num();
        double *acc = part + (int64_t)t * nb;
        double *P = (double *)malloc(sizeof(double) * (size_t)(N * N > 0 ? N * N : 1));
        double *u = (double *)malloc(sizeof(double) * (size_t)(N * C > 0 ? N * C : 1));
        double *du = (double *)malloc(sizeof(double) * (size_t)(N * C > 0 ? N * C : 1));
        double *D = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
#pragma omp for schedule(static)
        for (int64_t w = 0; w < units; ++w) {
            const int64_t n = w / H;
            const int h = (int)(w % H);
            const int64_t r = rows[n];
            /* forward of the whole row: probabilities and ungated outputs */
            for (int64_t x = 0; x < N; ++x) query_forward(&p, r, h, x, P + x * N, u + x * C);
            /* gate: du, dgate and D */
            for (int64_t x = 0; x < N; ++x) {
                const float *gx = gate + pair_at(&p, r, x, h);
                const float *ox = dout + pair_at(&p, r, x, h);
                double *dg = dgate + ((n * N + x) * H + h) * (int64_t)C;
                double d = 0.0;
                for (int c = 0; c < C; ++c) {
                    const double s = sigmoid((double)gx[c]);
                    du[x * C + c] = (double)ox[c] * s;
                    dg[c] = (double)ox[c] * u[x * C + c] * s * (1.0 - s);
                    d += du[x * C + c] * u[x * C + c];
                }
                D[x] = d;
            }
            /* zero this row's pair gradients */
            for (int64_t x = 0; x < N; ++x)
                for (int c = 0; c < C; ++c) {
                    const int64_t o = ((n * N + x) * H + h) * (int64_t)C + c;
                    dq[o] = 0.0; dk[o] = 0.0; dv[o] = 0.0;
                }
            for (int64_t x = 0; x < N; ++x) {
                const float *qx = q + pair_at(&p, r, x, h);
                double *dqx = dq + ((n * N + x) * H + h) * (int64_t)C;
                for (int64_t y = 0; y < N; ++y) {
                    const double pxy = P[x * N + y];
                    if (pxy == 0.0 && !key_kept(&p, r, y)) continue;
                    const float *vy = v + pair_at(&p, r, y, h);
                    const float *ky = k + pair_at(&p, r, y, h);
                    double dp = 0.0;
                    for (int c = 0; c < C; ++c) dp += du[x * C + c] * (double)vy[c];
                    const double ds = pxy * (dp - D[x]);
                    double *dky = dk + ((n * N + y) * H + h) * (int64_t)C;
                    double *dvy = dv + ((n * N + y) * H + h) * (int64_t)C;
                    for (int c = 0; c < C; ++c) {
                        dqx[c] += scale * ds * (double)ky[c];
                        dky[c] += scale * ds * (double)qx[c];
                        dvy[c] += pxy * du[x * C + c];
                    }
                    acc[bias_at(&p, h, x, y)] += ds;
                }
            }
        }
        free(P); free(u); free(du); free(D);
    }
    for (int64_t e = 0; e < nb; ++e) {
        double s = 0.0;
        for (int t = 0; t < nthreads; ++t) s += part[(int64_t)t * nb + e];
        dbias[e] = s;
    }
    free(part);
    return 0;
}

/*
 * Selected dbias entries summed over ALL N rows, for sizes where the full
 * backward is too slow. ent holds n_ent triples (h, a, b) in storage layout
 * dbias[h][a][b]; out[e] receives that entry.
 */
int tri_oracle_dbias_entries(int64_t N, int H, int C, int variant, const float *q,
                             const float *k, const float *v, const float *bias,
                             const float *gate, const uint8_t *mask,
                             int64_t mask_row_stride, const float *dout,
                             const int64_t *ent, int64_t n_ent, double *out)
{
    if (check(N, H, C, variant)) return 1;
    prob_t p = make_prob(N, H, C, variant, q, k, v, bias, gate, dout, mask,
                         mask_row_stride);
#pragma omp parallel
    {
        double *prob = (double *)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        double *u = (double *)malloc(sizeof(double) * (size_t)C);
#pragma omp for schedule(dynamic, 1)
        for (int64_t e = 0; e < n_ent; ++e) {
            const int h = (int)ent[3 * e];
            const int64_t a = ent[3 * e + 1], b = ent[3 * e + 2];
            const int64_t x = (variant == 0) ? a : b;   /* query in the variant frame */
            const int64_t y = (variant == 0) ? b : a;   /* key in the variant frame */
            double sum = 0.0;
            for (int64_t r = 0; r < N; ++r) {
                query_forward(&p, r, h, x, prob, u);
                if (prob[y] == 0.0) continue;
                const float *gx = gate + pair_at(&p, r, x, h);
                const float *ox = dout + pair_at(&p, r, x, h);
                const float *vy = v + pair_at(&p, r, y, h);
                double d = 0.0, dp = 0.0;
                for (int c = 0; c < C; ++c) {
                    const double du = (double)ox[c] * sigmoid((double)gx[c]);
                    d += du * u[c];
                    dp += du * (double)vy[c];
                }
                sum += prob[y] * (dp - d);
            }
            out[e] = sum;
        }
        free(prob);
        free(u);
    }
    return 0;
}
