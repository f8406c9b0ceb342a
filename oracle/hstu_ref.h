/*
 * hstu_ref.h -- fp64 CPU oracle for HSTU causal pointwise aggregated attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path includes, links or
 * calls this; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code with the CUDA library.
 *
 * All floating inputs are fp64 host arrays holding the (already rounded) values
 * of the run; every computation is plain fp64 loops in a fixed order.
 */
#ifndef HSTU_REF_H
#define HSTU_REF_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int32_t batch;              /* B                                               */
    int32_t num_heads;          /* H                                               */
    int32_t d_qk, d_v;          /* per-head widths                                 */
    const int32_t *offsets;     /* [B+1], offsets[0] = 0, non-decreasing, = T      */
    const int64_t *timestamps;  /* [T] or NULL (no time bias)                      */
    const double *rab_pos;      /* [H, 2L-1] or NULL                               */
    int32_t rab_pos_len;        /* L                                               */
    const double *rab_time;     /* [H, num_time_buckets] or NULL                   */
    int32_t num_time_buckets;   /* 128 in the workloads                            */
    int32_t norm_len;           /* >0: divide by it; 0: divide by each n_b         */
    double ln_eps;              /* LayerNorm epsilon (1e-5)                        */
    const double *ln_weight;    /* [H*dv] LayerNorm scale, or NULL (all ones)      */
    const double *ln_bias;      /* [H*dv] LayerNorm shift, or NULL (all zeros)     */
} hstu_ref_problem;

/* Time bucket of a timestamp difference: min(NB-1, floor(ln(max(1,|dt|))/0.301)). */
int32_t hstu_ref_time_bucket(int64_t dt, int32_t num_time_buckets);

/* Forward on every token.  q,k: [T,H,dqk]; v: [T,H,dv]; u: [T,H*dv].
 * Writes y [T,H*dv]; o [T,H*dv], mean [T], rstd [T] when non-NULL.
 * Returns 0 on success, a negative code on invalid arguments. */
int hstu_ref_fwd(const hstu_ref_problem *p, const double *q, const double *k,
                 const double *v, const double *u, double *y, double *o,
                 double *mean, double *rstd, int num_threads);

/* Forward on the listed global token rows only (rows[r] in [0,T)).  Outputs
 * are compact: y [nrows, H*dv], o [nrows, H*dv], mean/rstd [nrows]. */
int hstu_ref_fwd_rows(const hstu_ref_problem *p, const double *q, const double *k,
                      const double *v, const double *u, const int64_t *rows,
                      int64_t nrows, double *y, double *o, double *mean,
                      double *rstd, int num_threads);

/* Backward from dy [T,H*dv].  Writes dq, dk [T,H,dqk], dv [T,H,dv],
 * du [T,H*dv]; d_rab_pos [H,2L-1], d_rab_time [H,NB], d_ln_weight and
 * d_ln_bias [H*dv] are overwritten (not accumulated) when non-NULL.  The
 * forward is recomputed internally. */
int hstu_ref_bwd(const hstu_ref_problem *p, const double *q, const double *k,
                 const double *v, const double *u, const double *dy,
                 double *dq, double *dk, double *dv, double *du,
                 double *d_rab_pos, double *d_rab_time, double *d_ln_weight,
                 double *d_ln_bias, int num_threads);

/* The projections either side of the attention (one HSTU block, "HSTU
 * (Generative Recommender)" model card, HSTUBlock):
 *
 * UVQK: P = X W^T + b over the T rows of X [T, E], W [H(2dv+2dqk), E],
 * b [H(2dv+2dqk)] or NULL; with act = 1, P = SiLU(P) (the reproduction note's
 * SiLU(Norm(X) W_UVQK)).  P's columns split, in order, into u [T, H*dv],
 * v [T, H*dv], q [T, H*dqk], k [T, H*dqk].  Returns 0, or < 0 for bad sizes. */
int hstu_ref_uvqk(int64_t T, int32_t E, int32_t H, int32_t dqk, int32_t dv, int32_t act,
                  const double *x, const double *w, const double *b,
                  double *u, double *v, double *q, double *k);

/* Output: Z = LayerNorm_E(X + Y W_out^T + b_out) with weight gamma and bias
 * beta (NULL: ones, zeros), biased variance and eps.  Y [T, Dy] (Dy = H*dv),
 * X [T, E] (the residual), W_out [E, Dy], b_out [E] or NULL.  Writes z [T, E]
 * and, when non-NULL, the row mean and rstd [T]. */
int hstu_ref_out(int64_t T, int32_t E, int32_t Dy, const double *y, const double *x,
                 const double *w, const double *b, const double *gamma, const double *beta,
                 double eps, double *z, double *mean, double *rstd);

/* Candidate scoring against a cached history (M-FALCON).  p describes the
 * history: offsets [B+1] over T_h history tokens, timestamps [T_h].  k_hist
 * [T_h,H,dqk], v_hist [T_h,H,dv]; cand_offsets [B+1] over C candidates with
 * timestamps cand_ts [C] (or NULL without a time table); qc, kc [C,H,dqk],
 * vc [C,H,dv], uc [C,H*dv].  Candidate c of user b attends to the user's
 * history and to itself only, as row n_b of (history, c).  Writes y
 * [C,H*dv]; o [C,H*dv], mean, rstd [C] when non-NULL. */
int hstu_ref_mfalcon(const hstu_ref_problem *p, const double *k_hist, const double *v_hist,
                     const int32_t *cand_offsets, const int64_t *cand_ts, const double *qc,
                     const double *kc, const double *vc, const double *uc, double *y,
                     double *o, double *mean, double *rstd, int num_threads);

#ifdef __cplusplus
}
#endif
#endif
