/*
 * hstu.h -- C ABI of libhstu: HSTU causal pointwise aggregated attention on
 * NVIDIA B200 (sm_100a).
 *
 * The operation (one HSTU layer's spatial aggregation and gated output; see
 * "HSTU (Generative Recommender)" model card, Exported PyTorch,
 * HSTUBlock.forward; "HSTU Hierarchical Sequential Transduction Units",
 * §1 The key contribution and §3 How it works; the HSTU reproduction note's
 * flowchart and key-formula section):
 *
 *   for every sequence b (tokens s..s+n_b-1 of the packed token axis), every
 *   head h and every local row i, over local columns j <= i:
 *     S_ij = q_i . k_j + rab_pos[h][(i-j)+L-1] + rab_time[h][bucket(t_i - t_j)]
 *     A_ij = SiLU(S_ij) / N_b        (no softmax; N_b = norm_len or n_b)
 *     O_i  = sum_{j<=i} A_ij v_j     (heads concatenated: width D = H*d_v)
 *     Y_i  = (gamma * LayerNorm_D(O_i) + beta) * SiLU(U_i)   (biased variance, eps)
 *   bucket(dt) = min(NB-1, floor(ln(max(1,|dt|)) / 0.301)).
 *
 * Layouts (row-major, token-major, packed over the B sequences):
 *   q, k  [T, H, d_qk]    v [T, H, d_v]    u, y, dy [T, H*d_v]
 *   offsets int32 [B+1] (offsets[0] = 0, non-decreasing, offsets[B] = T)
 *   timestamps int64 [T]; rab_pos fp32 [H, 2L-1]; rab_time fp32 [H, NB];
 *   ln_weight, ln_bias fp32 [H*d_v] (gamma, beta; NULL = ones, zeros)
 *
 * Ownership: the caller owns every buffer.  Device pointers must point to
 * memory of the current CUDA device; the library allocates nothing, and all
 * work is enqueued asynchronously on `stream` (a cudaStream_t; NULL = the
 * legacy default stream).
 *
 * Errors: argument checks are synchronous and return HSTU_ERR_INVALID_ARG,
 * HSTU_ERR_UNSUPPORTED or HSTU_ERR_WORKSPACE without enqueueing anything.  A
 * failed launch returns HSTU_ERR_CUDA.  Problems found on the device (offsets
 * that contradict the sizes, a bounded wait that ran out) are recorded in a
 * status word at the start of the workspace and reported by hstu_attn_check.
 * No C++ exception crosses this boundary.
 */
#ifndef HSTU_H
#define HSTU_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define HSTU_API __attribute__((visibility("default")))
#else
#define HSTU_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HSTU_OK = 0,
  HSTU_ERR_INVALID_ARG = 1,  /* NULL/misaligned pointer, bad sizes, bad offsets  */
  HSTU_ERR_UNSUPPORTED = 2,  /* valid problem outside the implemented shapes     */
  HSTU_ERR_CUDA = 3,         /* a CUDA call or launch failed                     */
  HSTU_ERR_TIMEOUT = 4,      /* a bounded device-side wait ran out               */
  HSTU_ERR_WORKSPACE = 5,    /* workspace NULL or smaller than required          */
  HSTU_ERR_BOUNDS = 6        /* an index check of a HSTU_DEBUG_BOUNDS build failed */
} hstu_status_t;

typedef enum { HSTU_F32 = 0, HSTU_BF16 = 1 } hstu_dtype_t;

/* Problem description, passed by const pointer; read during the call only. */
typedef struct {
  hstu_dtype_t dtype;         /* q, k, v, u, y, dy and the gradients dq..du       */
  int32_t batch;              /* B >= 0                                           */
  int32_t total_tokens;       /* T = offsets[B]                                   */
  int32_t max_seq_len;        /* >= every n_b; sizes the launch grid              */
  int32_t num_heads;          /* H >= 1                                           */
  int32_t d_qk, d_v;          /* per-head widths                                  */
  const int32_t *offsets;     /* device [B+1]                                     */
  const int32_t *offsets_host;/* optional host copy of offsets: full validation   */
  const int64_t *timestamps;  /* device [T], or NULL when rab_time is NULL        */
  const float *rab_pos;       /* device [H, 2L-1] or NULL (no position bias)      */
  int32_t rab_pos_len;        /* L >= max_seq_len when rab_pos is given           */
  const float *rab_time;      /* device [H, NB] or NULL (no time bias)            */
  int32_t num_time_buckets;   /* NB in [1, 128] when rab_time is given            */
  int32_t norm_len;           /* > 0: divide by it; 0: divide by each n_b         */
  float ln_eps;               /* LayerNorm epsilon, > 0 (1e-5)                    */
  const float *ln_weight;     /* device [H*d_v] LayerNorm weight, or NULL (ones)  */
  const float *ln_bias;       /* device [H*d_v] LayerNorm bias, or NULL (zeros)   */
} hstu_problem_t;

/*
 * Bytes of device workspace the call needs (is_bwd = 0: forward; 1: backward).
 * With a time table the bf16 calls also keep there the shapes of their
 * time-bias plans, 4 bytes per token and 32-column block of max_seq_len
 * (rounded up to 128) for the forward, twice that for the backward, and 96
 * bytes per token of per-element buckets near the diagonal:
 * T * (16 * ceil(max_seq_len / 128) + 96) bytes (forward),
 * T * (32 * ceil(max_seq_len / 128) + 96) bytes (backward), each rounded up to 256.
 * The workspace must be 256-byte aligned and zero-filled before its first use;
 * its first word is the device status that hstu_attn_check reads and re-arms.
 * Words 16 and 17 hold the bf16 forward's work counters: each launch hands its
 * (sequence, query tile) items out through them and the last cluster to
 * finish returns them to zero.  Calls that share a workspace must therefore
 * run one after another (same stream or ordered by events), never overlapped.
 */
HSTU_API size_t hstu_attn_workspace_size(const hstu_problem_t *p, int is_bwd);

/*
 * Forward.  q, k, v, u: inputs (dtype, layouts above, 16-byte aligned).
 * y: output [T, H*d_v] (dtype).  o_save [T, H*d_v], ln_mean [T], ln_rstd [T]:
 * optional fp32 outputs kept for the backward (all three or none; NULL = skip).
 * Supported: bf16 with d_qk = d_v = 128, 1 <= H <= 8 and
 * 2 * batch * ceil(max_seq_len / 128) <= 2^31 - 256 (tcgen05 path); fp32 with
 * d_qk, d_v <= 128 and H*d_v <= 1024 (true-fp32 SIMT path).
 */
HSTU_API hstu_status_t hstu_attn_fwd(const hstu_problem_t *p, const void *q, const void *k,
                            const void *v, const void *u, void *y, float *o_save,
                            float *ln_mean, float *ln_rstd, void *workspace,
                            size_t workspace_bytes, void *stream);

/*
 * Backward of hstu_attn_fwd.  dy [T, H*d_v] (dtype) is the upstream gradient;
 * o_save, ln_mean, ln_rstd are the forward's saved fp32 outputs (required).
 * Writes dq, dk [T,H,d_qk], dv [T,H,d_v], du [T,H*d_v] (dtype); d_rab_pos
 * [H,2L-1], d_rab_time [H,NB], d_ln_weight and d_ln_bias [H*d_v] (fp32) are
 * overwritten, not accumulated, when non-NULL (entries with i-j < 0 are
 * zero); each needs its table in the problem.  The bias and LayerNorm
 * gradients are sums over all tokens taken with fp32 atomics, so their last
 * bits may differ between runs.  Supported shapes are those of hstu_attn_fwd.
 */
HSTU_API hstu_status_t hstu_attn_bwd(const hstu_problem_t *p, const void *dy, const void *q,
                            const void *k, const void *v, const void *u,
                            const float *o_save, const float *ln_mean, const float *ln_rstd,
                            void *dq, void *dk, void *dv, void *du, float *d_rab_pos,
                            float *d_rab_time, float *d_ln_weight, float *d_ln_bias,
                            void *workspace, size_t workspace_bytes, void *stream);

/*
 * Waits for `stream`, reads the device status word of `workspace`, resets it
 * to zero and returns it (HSTU_OK, HSTU_ERR_INVALID_ARG for offsets found
 * inconsistent on the device, HSTU_ERR_TIMEOUT for an expired wait,
 * HSTU_ERR_BOUNDS when a library built with -DHSTU_DEBUG_BOUNDS found an
 * index outside its buffer: it recorded the first failing check site in
 * word 6 and its index in word 7 and used index 0 instead), or
 * HSTU_ERR_CUDA when the stream itself reports an error.
 */
HSTU_API hstu_status_t hstu_attn_check(void *workspace, void *stream);

/* Static, NUL-terminated description of a status code. */
HSTU_API const char *hstu_status_string(hstu_status_t s);

/*
 * Host utility: writes the library's time-bucket thresholds, out[k-1] = the
 * smallest |dt| with bucket(dt) >= k for k = 1..num_buckets-1.  Returns the
 * number written, or -1 for num_buckets outside [1, 128].
 */
HSTU_API int32_t hstu_time_bucket_thresholds(int64_t *out, int32_t num_buckets);

/*
 * Self-test of the device error path: launches one thread that waits on an
 * mbarrier nothing arrives on, with the library's bounded wait limited to
 * budget_ns (1 ns .. 5 s).  When the budget runs out the kernel sets the
 * timeout bit of the workspace status word and returns; hstu_attn_check then
 * reports HSTU_ERR_TIMEOUT and the context remains usable.  Returns
 * HSTU_ERR_WORKSPACE for a NULL or unaligned workspace (256 bytes suffice).
 */
HSTU_API hstu_status_t hstu_selftest_wait_timeout(void *workspace, uint64_t budget_ns,
                                                  void *stream);

/*
 * Backward without a caller-provided workspace.  The HSTU model card and
 * papers define no such call; it exists for callers that cannot allocate
 * device memory themselves
 * (for example when another allocator already owns the free device memory,
 * or a host framework forbids direct CUDA allocation).
 *
 * Same arguments, results and synchronous errors as hstu_attn_bwd, minus the
 * workspace: the scratch lives in a fixed 16 MiB array in device global memory
 * that the library reserves on every device it is loaded on and keeps until
 * the process exits.  The argument checks of hstu_attn_bwd run first and
 * return the same codes; then problems whose backward workspace
 * (hstu_attn_workspace_size(p, 1)) is larger than the array return
 * HSTU_ERR_WORKSPACE.  A rejected call enqueues nothing.  The function calls no allocation routine.  The first
 * call on a device looks up the array's device address (with that device
 * current) and caches it.  All calls share the one array: calls that may
 * overlap on the GPU (different streams, no ordering between them) race on it
 * and must be serialised by the caller.  Each call clears the device status
 * word at the start of the array; device-side findings (offsets contradicting
 * the sizes, an expired wait) stay in that word and are not reported by this
 * entry point, so pass offsets_host to have the offsets checked on the host.
 */
HSTU_API hstu_status_t hstu_attn_bwd_noalloc(const hstu_problem_t *p, const void *dy,
                                             const void *q, const void *k, const void *v,
                                             const void *u, const float *o_save,
                                             const float *ln_mean, const float *ln_rstd,
                                             void *dq, void *dk, void *dv, void *du,
                                             float *d_rab_pos, float *d_rab_time,
                                             float *d_ln_weight, float *d_ln_bias, void *stream);

/*
 * The projections either side of the attention in an HSTU layer ("HSTU
 * (Generative Recommender)" model card, Exported PyTorch, HSTUBlock: the
 * uvqk linear split into u, v, q, k, and norm(x + out(y)); the reproduction
 * note's key formulas: U, V, Q, K = Split(SiLU(Norm(X) W_UVQK)) and the
 * residual around the layer).  Both are bf16 GEMMs on the tcgen05 tensor
 * cores with fp32 accumulation and a fused epilogue; outputs are rounded to
 * bf16 once.  All matrices are row-major bf16, 16-byte aligned; fp32 vectors
 * 16-byte aligned.  `workspace` (>= 256 bytes, 256-byte aligned, zero-filled
 * before first use) holds only the device status word that hstu_attn_check
 * reads.  Argument checks are synchronous (HSTU_ERR_INVALID_ARG,
 * HSTU_ERR_UNSUPPORTED, HSTU_ERR_WORKSPACE) and enqueue nothing; T = 0 is a
 * no-op.
 */

/*
 * UVQK projection: P = act(X W^T + bias), X [T, E], W [N, E] (the nn.Linear
 * weight layout), N = 2*H*d_v + 2*H*d_qk, bias fp32 [N] or NULL, act 0 =
 * identity, 1 = SiLU.  Columns [0, Hd_v) go to u [T, H*d_v], [Hd_v, 2Hd_v)
 * to v [T, H, d_v], the next H*d_qk to q [T, H, d_qk] and the last H*d_qk to
 * k [T, H, d_qk] -- the layouts hstu_attn_fwd reads.  Supported: E a
 * multiple of 64; H*d_v and H*d_qk multiples of 256; T <= 8388480.
 */
HSTU_API hstu_status_t hstu_uvqk_fwd(int32_t T, int32_t E, int32_t H, int32_t d_qk, int32_t d_v,
                                     int32_t act, const void *x, const void *w, const float *bias,
                                     void *u, void *v, void *q, void *k, void *workspace,
                                     size_t workspace_bytes, void *stream);

/*
 * Output projection, residual and LayerNorm over E:
 *   R = X + Y W^T + bias,  Z = (R - mean(R)) * rstd * ln_weight + ln_bias,
 *   rstd = 1 / sqrt(biased variance of R + eps).
 * Y [T, D] (the attention output, D = H*d_v), W [E, D] (nn.Linear layout),
 * X [T, E] the residual (the layer input), bias, ln_weight, ln_bias fp32 [E]
 * or NULL (zeros, ones, zeros); z [T, E] bf16 output; mean, rstd fp32 [T]
 * (both or neither) receive the row statistics of R.  Supported: E in
 * {256, 512}; D a multiple of 64.
 */
HSTU_API hstu_status_t hstu_out_fwd(int32_t T, int32_t E, int32_t D, const void *y, const void *w,
                                    const void *x, const float *bias, const float *ln_weight,
                                    const float *ln_bias, float eps, void *z, float *mean,
                                    float *rstd, void *workspace, size_t workspace_bytes,
                                    void *stream);

/*
 * Candidate scoring against cached histories (M-FALCON: "HSTU Hierarchical
 * Sequential Transduction Units", §6 Why it works, micro-batched candidate
 * scoring with key/value reuse; the pages print no formula).  Reading taken:
 * candidate c of user b is the token that follows the user's n_b history
 * tokens, on its own -- it attends to every history token j < n_b (relative
 * position n_b - j, time bucket of t_c - t_j) and to itself (relative
 * position 0, time difference 0), never to another candidate; the
 * normaliser is norm_len (> 0) or n_b + 1.  Y_c is thus the last row of
 * hstu_attn_fwd over the sequence (history of b, c).  Each history key and
 * value tile is read once per micro-batch of 128 candidates and head.
 *
 * p describes the histories: batch, total_tokens (history tokens T_h),
 * max_seq_len (>= every n_b), offsets, timestamps (history), the bias tables
 * (rab_pos_len >= max_seq_len + 1, as a candidate sits at position n_b),
 * norm_len, ln_eps, ln_weight/ln_bias.  k_hist, v_hist [T_h, H, 128]: the
 * cached keys and values.  cand_offsets device int32 [B+1] over total_cands
 * candidates (at most max_cands per user); cand_timestamps device int64
 * [total_cands] (required with rab_time).  q, k, v [C, H, 128], u [C, H*128]:
 * the candidates' projections; y [C, H*128] output.  Supported: bf16,
 * d_qk = d_v = 128, 1 <= H <= 16.  workspace: hstu_cand_workspace_size bytes
 * for the same problem (with a time table it also holds the time-plan shape
 * of every candidate against every 32-event block of its user's history:
 * 16 * ceil(max_seq_len / 128) bytes per candidate), 256-byte aligned,
 * zero-filled before its first use (its per-micro-batch counters return to
 * zero after each call); candidate offsets found inconsistent on the device
 * are reported by hstu_attn_check.
 */
HSTU_API size_t hstu_cand_workspace_size(const hstu_problem_t *p, int32_t total_cands,
                                         int32_t max_cands);
HSTU_API hstu_status_t hstu_cand_fwd(const hstu_problem_t *p, const void *k_hist,
                                     const void *v_hist, const int32_t *cand_offsets,
                                     int32_t total_cands, int32_t max_cands,
                                     const int64_t *cand_timestamps, const void *q, const void *k,
                                     const void *v, const void *u, void *y, void *workspace,
                                     size_t workspace_bytes, void *stream);

#ifdef __cplusplus
}
#endif
#endif /* HSTU_H */
