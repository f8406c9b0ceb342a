/*
 * hstu_ref.c -- fp64 CPU oracle for HSTU causal pointwise aggregated attention.
 *
 * TEST INFRASTRUCTURE ONLY: used by the tests, the smoke check and the
 * benchmark's CPU-baseline leg; never by the product path.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * What it computes (the plain definition, nothing approximated):
 *
 *   For each sequence b (tokens s = off[b] .. off[b+1]-1, length n = n_b),
 *   each local row i < n, each head h and each local column j <= i:
 *
 *     S_ij = q_i . k_j + rab_pos[h][(i-j)+L-1] + rab_time[h][bucket(t_i - t_j)]
 *     A_ij = SiLU(S_ij) / N_b,           SiLU(x) = x / (1 + exp(-x))
 *     O_i  = sum_{j<=i} A_ij v_j         (heads concatenated to width D = H*dv)
 *     Y_i  = (gamma * LayerNorm_D(O_i) + beta) * SiLU(U_i)
 *
 * Sources:
 *  - score without 1/sqrt(d), SiLU instead of softmax, divide by the length,
 *    lower-triangular mask (diagonal kept), A.V per head and concatenation of
 *    heads: "HSTU (Generative Recommender)" model card, Exported PyTorch,
 *    HSTUBlock.forward (the `attn = (F.silu(q @ k^T) / t).tril()` and
 *    `attn @ vh` steps).
 *  - no softmax normalisation and a causal mask: the HSTU reproduction note
 *    (daiwk.github.io, "核心公式" / key formula section).
 *  - relative position and time biases inside the pointwise attention:
 *    "HSTU Hierarchical Sequential Transduction Units" (briansu.co),
 *    §1 The key contribution and §3 How it works; the position bias is also
 *    listed in the reproduction note's fidelity line.
 *  - post-pooling normalisation followed by the U gate: the reproduction
 *    note's flowchart; the gate `o * F.silu(u)`: the model card's
 *    HSTUBlock.forward.
 *  - LayerNorm with biased variance, eps 1e-5 and an elementwise affine
 *    gamma, beta over the D features (the model card's block norms with
 *    nn.LayerNorm, whose weight and bias start at ones and zeros: NULL
 *    tables mean exactly that unit affine); the time bucket
 *    min(NB-1, floor(ln(max(1,|dt|))/0.301)); the position index (i-j)+L-1
 *    into a [H, 2L-1] table; normalisation by a fixed N or by each sequence's
 *    own length: readings taken where the pages print no formula (their
 *    equation sections lost the equations in extraction).
 *
 * The backward is the chain rule of the same definition, in fp64:
 *   g = SiLU(U), dU = dY * (gamma xhat + beta) * SiLU'(U),
 *   dxhat = dY * g * gamma, d_gamma = sum_t dY * g * xhat, d_beta = sum_t dY * g,
 *   dO = rstd * (dxhat - mean_D(dxhat) - xhat * mean_D(dxhat * xhat)),
 *   dV_j = sum_{i>=j} A_ij dO_i,  dA_ij = dO_i . v_j,
 *   dS_ij = dA_ij * SiLU'(S_ij) / N_b,  dQ_i = sum_j dS_ij k_j,
 *   dK_j = sum_i dS_ij q_i,  d_rab_pos[h][(i-j)+L-1] += dS_ij,
 *   d_rab_time[h][bucket] += dS_ij,
 *   with SiLU'(x) = sigma(x) (1 + x (1 - sigma(x))).
 *
 * Summation order is fixed (ascending j, ascending c); there are no atomics,
 * so results are bit-identical for any thread count.
 */
#include "hstu_ref.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double ref_silu(double x) { return x / (1.0 + exp(-x)); }

static double ref_sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

static double ref_silu_grad(double x) {
    double s = ref_sigmoid(x);
    return s * (1.0 + x * (1.0 - s));
}

int32_t hstu_ref_time_bucket(int64_t dt, int32_t num_time_buckets) {
    /* |dt| with max(1, .): INT64_MIN has no positive counterpart; it is far
     * beyond the last bucket anyway. */
    double a;
    if (dt == INT64_MIN) a = 9223372036854775808.0;
    else a = (double)(dt < 0 ? -dt : dt);
    if (a < 1.0) a = 1.0;
    double b = floor(log(a) / 0.301);
    if (b > (double)(num_time_buckets - 1)) b = (double)(num_time_buckets - 1);
    return (int32_t)b;
}

static int validate(const hstu_ref_problem *p) {
    if (!p || !p->offsets || p->batch < 0 || p->num_heads <= 0 || p->d_qk <= 0 || p->d_v <= 0)
        return -1;
    if (p->offsets[0] != 0) return -2;
    for (int b = 0; b < p->batch; ++b) {
        int32_t n = p->offsets[b + 1] - p->offsets[b];
        if (n < 0) return -3;
        if (p->rab_pos && n > p->rab_pos_len) return -4;
        if (p->norm_len < 0) return -5;
    }
    if (p->rab_time && (!p->timestamps || p->num_time_buckets <= 0)) return -6;
    return 0;
}

/* Bias of (local row i, local column j) of the sequence starting at token s. */
static double ref_bias(const hstu_ref_problem *p, int h, int64_t s, int i, int j) {
    double bias = 0.0;
    if (p->rab_pos) {
        int64_t L = p->rab_pos_len;
        bias += p->rab_pos[(int64_t)h * (2 * L - 1) + (i - j) + L - 1];
    }
    if (p->rab_time) {
        int32_t bk = hstu_ref_time_bucket(p->timestamps[s + i] - p->timestamps[s + j],
                                          p->num_time_buckets);
        bias += p->rab_time[(int64_t)h * p->num_time_buckets + bk];
    }
    return bias;
}

static double ref_dot(const double *a, const double *b, int n) {
    double acc = 0.0;
    for (int c = 0; c < n; ++c) acc += a[c] * b[c];
    return acc;
}

static int seq_of_token(const hstu_ref_problem *p, int64_t t) {
    int lo = 0, hi = p->batch - 1;
    while (lo < hi) {   /* last b with offsets[b] <= t; then offsets[b+1] > t */
        int mid = (lo + hi + 1) / 2;
        if (p->offsets[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

/* One output row: global token t.  Writes o_row [D], y_row [D], *mean, *rstd. */
static void fwd_row(const hstu_ref_problem *p, const double *q, const double *k,
                    const double *v, const double *u, int64_t t, double *o_row,
                    double *y_row, double *mean_out, double *rstd_out) {
    const int H = p->num_heads, dqk = p->d_qk, dv = p->d_v, D = H * dv;
    int b = seq_of_token(p, t);
    int64_t s = p->offsets[b];
    int n = p->offsets[b + 1] - p->offsets[b];
    int i = (int)(t - s);
    double Nn = p->norm_len > 0 ? (double)p->norm_len : (double)n;

    for (int c = 0; c < D; ++c) o_row[c] = 0.0;
    for (int h = 0; h < H; ++h) {
        const double *qi = q + (t * H + h) * dqk;
        double *oh = o_row + h * dv;
        for (int j = 0; j <= i; ++j) {
            const double *kj = k + ((s + j) * H + h) * dqk;
            double S = ref_dot(qi, kj, dqk) + ref_bias(p, h, s, i, j);
            double A = ref_silu(S) / Nn;
            const double *vj = v + ((s + j) * H + h) * dv;
            for (int c = 0; c < dv; ++c) oh[c] += A * vj[c];
        }
    }
    /* LayerNorm over the D concatenated head outputs, biased variance. */
    double mu = 0.0;
    for (int c = 0; c < D; ++c) mu += o_row[c];
    mu /= (double)D;
    double var = 0.0;
    for (int c = 0; c < D; ++c) var += (o_row[c] - mu) * (o_row[c] - mu);
    var /= (double)D;
    double rstd = 1.0 / sqrt(var + p->ln_eps);
    const double *ur = u + t * D;
    for (int c = 0; c < D; ++c) {
        double w = p->ln_weight ? p->ln_weight[c] : 1.0;
        double bb = p->ln_bias ? p->ln_bias[c] : 0.0;
        y_row[c] = ((o_row[c] - mu) * rstd * w + bb) * ref_silu(ur[c]);
    }
    *mean_out = mu;
    *rstd_out = rstd;
}

int hstu_ref_fwd_rows(const hstu_ref_problem *p, const double *q, const double *k,
                      const double *v, const double *u, const int64_t *rows,
                      int64_t nrows, double *y, double *o, double *mean,
                      double *rstd, int num_threads) {
    int rc = validate(p);
    if (rc) return rc;
    const int64_t T = p->offsets[p->batch];
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= T) return -7;
    const int D = p->num_heads * p->d_v;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel
    {
        double *o_tmp = (double *)malloc(sizeof(double) * D);
        double *y_tmp = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < nrows; ++r) {
            double mu, rs;
            fwd_row(p, q, k, v, u, rows[r], o_tmp, y_tmp, &mu, &rs);
            if (y) memcpy(y + r * D, y_tmp, sizeof(double) * D);
            if (o) memcpy(o + r * D, o_tmp, sizeof(double) * D);
            if (mean) mean[r] = mu;
            if (rstd) rstd[r] = rs;
        }
        free(o_tmp);
        free(y_tmp);
    }
    return 0;
}

int hstu_ref_fwd(const hstu_ref_problem *p, const double *q, const double *k,
                 const double *v, const double *u, double *y, double *o,
                 double *mean, double *rstd, int num_threads) {
    int rc = validate(p);
    if (rc) return rc;
    const int64_t T = p->offsets[p->batch];
    int64_t *rows = (int64_t *)malloc(sizeof(int64_t) * (T > 0 ? T : 1));
    /* Longest rows first so the dynamic schedule balances the causal triangle. */
    int64_t w = 0;
    for (int b = 0; b < p->batch; ++b)
        for (int64_t t = p->offsets[b + 1] - 1; t >= p->offsets[b]; --t) rows[w++] = t;
    const int D = p->num_heads * p->d_v;
    size_t cap = (size_t)(T > 0 ? T : 1);
    double *yy = (double *)malloc(sizeof(double) * cap * D);
    double *oo = (double *)malloc(sizeof(double) * cap * D);
    double *mm = (double *)malloc(sizeof(double) * cap);
    double *rr = (double *)malloc(sizeof(double) * cap);
    rc = hstu_ref_fwd_rows(p, q, k, v, u, rows, T, yy, oo, mm, rr, num_threads);
    for (int64_t r = 0; r < T && rc == 0; ++r) {   /* scatter back to token order */
        int64_t t = rows[r];
        if (y) memcpy(y + t * D, yy + r * D, sizeof(double) * D);
        if (o) memcpy(o + t * D, oo + r * D, sizeof(double) * D);
        if (mean) mean[t] = mm[r];
        if (rstd) rstd[t] = rr[r];
    }
    free(yy); free(oo); free(mm); free(rr);
    free(rows);
    return rc;
}

int hstu_ref_bwd(const hstu_ref_problem *p, const double *q, const double *k,
                 const double *v, const double *u, const double *dy,
                 double *dq, double *dk, double *dv, double *du,
                 double *d_rab_pos, double *d_rab_time, double *d_ln_weight,
                 double *d_ln_bias, int num_threads) {
    int rc = validate(p);
    if (rc) return rc;
    if (!dy || !dq || !dk || !dv || !du) return -8;
    const int B = p->batch, H = p->num_heads, dqk = p->d_qk, dvv = p->d_v, D = H * dvv;
    const int64_t T = p->offsets[B];
    const int64_t L = p->rab_pos_len, NB = p->num_time_buckets;
    const int64_t npos = p->rab_pos ? (2 * L - 1) : 0;
    const int64_t ntime = p->rab_time ? NB : 0;

    /* 1. Forward statistics of every row. */
    double *o = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * D);
    double *mean = (double *)malloc(sizeof(double) * (T > 0 ? T : 1));
    double *rstd = (double *)malloc(sizeof(double) * (T > 0 ? T : 1));
    double *dO = (double *)malloc(sizeof(double) * (size_t)(T > 0 ? T : 1) * D);
    rc = hstu_ref_fwd(p, q, k, v, u, NULL, o, mean, rstd, num_threads);
    if (rc) { free(o); free(mean); free(rstd); free(dO); return rc; }

#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#endif
    /* 2. LayerNorm + gate backward, per row. */
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const double *orow = o + t * D, *dyr = dy + t * D, *ur = u + t * D;
        double *dur = du + t * D, *dOr = dO + t * D;
        double m1 = 0.0, m2 = 0.0;   /* mean(dxhat), mean(dxhat * xhat) */
        for (int c = 0; c < D; ++c) {
            double w = p->ln_weight ? p->ln_weight[c] : 1.0;
            double bb = p->ln_bias ? p->ln_bias[c] : 0.0;
            double xhat = (orow[c] - mean[t]) * rstd[t];
            double g = ref_silu(ur[c]);
            dur[c] = dyr[c] * (w * xhat + bb) * ref_silu_grad(ur[c]);
            double dxh = dyr[c] * g * w;
            m1 += dxh;
            m2 += dxh * xhat;
        }
        m1 /= (double)D;
        m2 /= (double)D;
        for (int c = 0; c < D; ++c) {
            double w = p->ln_weight ? p->ln_weight[c] : 1.0;
            double xhat = (orow[c] - mean[t]) * rstd[t];
            double dxh = dyr[c] * ref_silu(ur[c]) * w;
            dOr[c] = rstd[t] * (dxh - m1 - xhat * m2);
        }
    }
    /* LayerNorm affine gradients: sums over every token, in token order. */
    if (d_ln_weight || d_ln_bias) {
        for (int c = 0; c < D; ++c) {
            if (d_ln_weight) d_ln_weight[c] = 0.0;
            if (d_ln_bias) d_ln_bias[c] = 0.0;
        }
        for (int64_t t = 0; t < T; ++t) {
            const double *orow = o + t * D, *dyr = dy + t * D, *ur = u + t * D;
            for (int c = 0; c < D; ++c) {
                double xhat = (orow[c] - mean[t]) * rstd[t];
                double dyg = dyr[c] * ref_silu(ur[c]);
                if (d_ln_weight) d_ln_weight[c] += dyg * xhat;
                if (d_ln_bias) d_ln_bias[c] += dyg;
            }
        }
    }

    /* 3. Attention backward, one (b, h) pair per task; bias gradients go to
     *    per-(b,h) partials reduced afterwards in a fixed order. */
    for (int64_t t = 0; t < T * H * dqk; ++t) { dq[t] = 0.0; dk[t] = 0.0; }
    for (int64_t t = 0; t < T * H * dvv; ++t) dv[t] = 0.0;
    size_t part_sz = (size_t)B * H;
    double *pos_part = npos ? (double *)calloc(part_sz * npos, sizeof(double)) : NULL;
    double *time_part = ntime ? (double *)calloc(part_sz * ntime, sizeof(double)) : NULL;

#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < (int64_t)B * H; ++bh) {
        int b = (int)(bh / H), h = (int)(bh % H);
        int64_t s = p->offsets[b];
        int n = p->offsets[b + 1] - p->offsets[b];
        double Nn = p->norm_len > 0 ? (double)p->norm_len : (double)n;
        double *pp = pos_part ? pos_part + bh * npos : NULL;
        double *tp = time_part ? time_part + bh * ntime : NULL;
        for (int i = 0; i < n; ++i) {
            const double *qi = q + ((s + i) * H + h) * dqk;
            const double *dOi = dO + (s + i) * D + h * dvv;
            double *dqi = dq + ((s + i) * H + h) * dqk;
            for (int j = 0; j <= i; ++j) {
                const double *kj = k + ((s + j) * H + h) * dqk;
                const double *vj = v + ((s + j) * H + h) * dvv;
                double S = ref_dot(qi, kj, dqk) + ref_bias(p, h, s, i, j);
                double A = ref_silu(S) / Nn;
                double dA = ref_dot(dOi, vj, dvv);
                double dS = dA * ref_silu_grad(S) / Nn;
                double *dvj = dv + ((s + j) * H + h) * dvv;
                for (int c = 0; c < dvv; ++c) dvj[c] += A * dOi[c];
                double *dkj = dk + ((s + j) * H + h) * dqk;
                for (int c = 0; c < dqk; ++c) {
                    dqi[c] += dS * kj[c];
                    dkj[c] += dS * qi[c];
                }
                if (pp) pp[(i - j) + L - 1] += dS;
                if (tp) {
                    int32_t bk = hstu_ref_time_bucket(p->timestamps[s + i] - p->timestamps[s + j],
                                                      p->num_time_buckets);
                    tp[bk] += dS;
                }
            }
        }
    }
    if (d_rab_pos && npos) {
        for (int h = 0; h < H; ++h)
            for (int64_t x = 0; x < npos; ++x) {
                double acc = 0.0;
                for (int b = 0; b < B; ++b) acc += pos_part[((int64_t)b * H + h) * npos + x];
                d_rab_pos[h * npos + x] = acc;
            }
    }
    if (d_rab_time && ntime) {
        for (int h = 0; h < H; ++h)
            for (int64_t x = 0; x < ntime; ++x) {
                double acc = 0.0;
                for (int b = 0; b < B; ++b) acc += time_part[((int64_t)b * H + h) * ntime + x];
                d_rab_time[h * ntime + x] = acc;
            }
    }
    free(pos_part);
    free(time_part);
    free(o); free(mean); free(rstd); free(dO);
    return 0;
}

/* ------------------------------------------------------------------------
 * Projections either side of the attention.
 *
 * UVQK: the model card's `self.uvqk(x).split([h*dv, h*dv, h*dqk, h*dqk])`
 * (nn.Linear: x W^T + b), optionally followed by SiLU as in the reproduction
 * note's key formula SiLU(Norm(X) W_UVQK).  Output: the model card's
 * `self.norm(x + self.out(...))`, nn.Linear then nn.LayerNorm over E.
 * Plain loops, fp64, fixed order (c ascending).
 * ------------------------------------------------------------------------ */
int hstu_ref_uvqk(int64_t T, int32_t E, int32_t H, int32_t dqk, int32_t dv, int32_t act,
                  const double *x, const double *w, const double *b,
                  double *u, double *v, double *q, double *k) {
    if (T < 0 || E <= 0 || H <= 0 || dqk <= 0 || dv <= 0 || !x || !w) return -1;
    const int64_t Nu = (int64_t)H * dv, Nq = (int64_t)H * dqk;
    const int64_t N = 2 * Nu + 2 * Nq;
#pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        const double *xr = x + t * E;
        for (int64_t n = 0; n < N; ++n) {
            const double *wr = w + n * E;
            double acc = 0.0;
            for (int c = 0; c < E; ++c) acc += xr[c] * wr[c];
            if (b) acc += b[n];
            if (act) acc = ref_silu(acc);
            if (n < Nu) u[t * Nu + n] = acc;
            else if (n < 2 * Nu) v[t * Nu + (n - Nu)] = acc;
            else if (n < 2 * Nu + Nq) q[t * Nq + (n - 2 * Nu)] = acc;
            else k[t * Nq + (n - 2 * Nu - Nq)] = acc;
        }
    }
    return 0;
}

int hstu_ref_out(int64_t T, int32_t E, int32_t Dy, const double *y, const double *x,
                 const double *w, const double *b, const double *gamma, const double *beta,
                 double eps, double *z, double *mean, double *rstd) {
    if (T < 0 || E <= 0 || Dy <= 0 || !y || !x || !w || !z) return -1;
#pragma omp parallel
    {
        double *r = (double *)malloc(sizeof(double) * E);
#pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            const double *yr = y + t * Dy, *xr = x + t * E;
            for (int e = 0; e < E; ++e) {
                const double *wr = w + (int64_t)e * Dy;
                double acc = 0.0;
                for (int c = 0; c < Dy; ++c) acc += yr[c] * wr[c];
                r[e] = xr[e] + acc + (b ? b[e] : 0.0);
            }
            double mu = 0.0;
            for (int e = 0; e < E; ++e) mu += r[e];
            mu /= (double)E;
            double var = 0.0;
            for (int e = 0; e < E; ++e) var += (r[e] - mu) * (r[e] - mu);
            var /= (double)E;
            double rs = 1.0 / sqrt(var + eps);
            for (int e = 0; e < E; ++e)
                z[t * E + e] = (r[e] - mu) * rs * (gamma ? gamma[e] : 1.0) + (beta ? beta[e] : 0.0);
            if (mean) mean[t] = mu;
            if (rstd) rstd[t] = rs;
        }
        free(r);
    }
    return 0;
}

/* ------------------------------------------------------------------------
 * Candidate scoring against a cached history ("HSTU Hierarchical Sequential
 * Transduction Units", §6 Why it works: M-FALCON, micro-batched candidate
 * scoring with key/value reuse).  The pages give no formula.  Reading taken:
 * candidate c of user b is the token that follows the user's n_b history
 * tokens, on its own: it attends to every history token j < n_b and to itself,
 * never to another candidate.  Its local row index is n_b, its time is its
 * own timestamp, and its normaliser is norm_len (> 0) or n_b + 1, the length
 * of (history, c).  Micro-batching and the reuse of the history's keys and
 * values change the cost, not the result, so neither appears here.
 * ------------------------------------------------------------------------ */
int hstu_ref_mfalcon(const hstu_ref_problem *p, const double *k_hist, const double *v_hist,
                     const int32_t *cand_offsets, const int64_t *cand_ts, const double *qc,
                     const double *kc, const double *vc, const double *uc, double *y,
                     double *o, double *mean, double *rstd, int num_threads) {
    int rc = validate(p);
    if (rc != 0) return rc;
    if (!cand_offsets || cand_offsets[0] != 0) return -7;
    if (p->rab_time && !cand_ts) return -8;
    for (int b = 0; b < p->batch; ++b) {
        if (cand_offsets[b + 1] < cand_offsets[b]) return -9;
        /* the candidate's position index n_b must be in the table */
        if (p->rab_pos && p->offsets[b + 1] - p->offsets[b] + 1 > p->rab_pos_len) return -4;
    }
    const int H = p->num_heads, dqk = p->d_qk, dv = p->d_v, D = H * dv;
    const int64_t C = cand_offsets[p->batch];
    const int64_t L = p->rab_pos_len, NB = p->num_time_buckets;
    if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel
    {
        double *orow = (double *)malloc(sizeof(double) * D);
#pragma omp for schedule(dynamic, 4)
        for (int64_t c = 0; c < C; ++c) {
            int b = 0;
            while (cand_offsets[b + 1] <= c) ++b;
            const int64_t s = p->offsets[b];
            const int n = p->offsets[b + 1] - p->offsets[b];
            const double Nn = p->norm_len > 0 ? (double)p->norm_len : (double)(n + 1);
            for (int e = 0; e < D; ++e) orow[e] = 0.0;
            for (int h = 0; h < H; ++h) {
                const double *q = qc + (c * H + h) * dqk;
                double *oh = orow + h * dv;
                /* history tokens j < n, relative position n - j */
                for (int j = 0; j < n; ++j) {
                    double S = ref_dot(q, k_hist + ((s + j) * H + h) * dqk, dqk);
                    if (p->rab_pos) S += p->rab_pos[h * (2 * L - 1) + (n - j) + L - 1];
                    if (p->rab_time)
                        S += p->rab_time[h * NB + hstu_ref_time_bucket(cand_ts[c] - p->timestamps[s + j],
                                                                       p->num_time_buckets)];
                    const double A = ref_silu(S) / Nn;
                    const double *vj = v_hist + ((s + j) * H + h) * dv;
                    for (int e = 0; e < dv; ++e) oh[e] += A * vj[e];
                }
                /* the candidate itself: relative position 0, time difference 0 */
                double S = ref_dot(q, kc + (c * H + h) * dqk, dqk);
                if (p->rab_pos) S += p->rab_pos[h * (2 * L - 1) + L - 1];
                if (p->rab_time) S += p->rab_time[h * NB + hstu_ref_time_bucket(0, p->num_time_buckets)];
                const double A = ref_silu(S) / Nn;
                const double *vs = vc + (c * H + h) * dv;
                for (int e = 0; e < dv; ++e) oh[e] += A * vs[e];
            }
            double mu = 0.0;
            for (int e = 0; e < D; ++e) mu += orow[e];
            mu /= (double)D;
            double var = 0.0;
            for (int e = 0; e < D; ++e) var += (orow[e] - mu) * (orow[e] - mu);
            var /= (double)D;
            const double rs = 1.0 / sqrt(var + p->ln_eps);
            for (int e = 0; e < D; ++e) {
                const double w = p->ln_weight ? p->ln_weight[e] : 1.0;
                const double bb = p->ln_bias ? p->ln_bias[e] : 0.0;
                y[c * D + e] = ((orow[e] - mu) * rs * w + bb) * ref_silu(uc[c * D + e]);
                if (o) o[c * D + e] = orow[e];
            }
            if (mean) mean[c] = mu;
            if (rstd) rstd[c] = rs;
        }
        free(orow);
    }
    return 0;
}
