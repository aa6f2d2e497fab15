/*
 * bi_isloss.h -- C ABI of the batch-invariant token-logprob + unclipped IS REINFORCE loss library.
 *
 * The operation (sources are page titles and sections):
 *   "Zero Mismatch, Simple Async RL", section "Only one probability gap comes from old weights":
 *       the learner/rollout log-ratio  log pi_theta_k - log mu_v  and the D3 statistic, the
 *       per-update token mean of  w - 1 - log w.
 *   "Zero Mismatch, Simple Async RL", section "Alignment permits a simpler learning path":
 *       bit-identical rollout and learner logprobs for the same weights and tokens; unclipped
 *       token-level importance weight  w = pi_learner / mu_rollout; advantage = response reward
 *       minus its group mean; tokens averaged within each response; no rejection gate.
 *   "REINFORCE-Zero: kernel alignment + unclipped IS ...", "Core insight": no ratio clipping;
 *       kernel mismatch comes from batch composition, prefill/decode paths and float ordering.
 *
 * Definitions computed by the library (T rows, hidden size H, vocabulary V):
 *   z_t     = W h_t                          (LM-head logits; never written to memory unless the
 *                                            caller opts in to the P store, BI_LOSS_STORE_P)
 *   lse_t   = log sum_v exp(z_tv)
 *   logpi_t = z_{t,y_t} - lse_t
 *   w_t     = exp(logpi_t - logmu_t)         (no clipping)
 *   d3_t    = w_t - 1 - log w_t
 *   A_i     = r_i - mean_{j in group(i)} r_j
 *   c_i     = A_i / (R* n_i)                 n_i = scored rows of response i, R* = R or the caller's value
 *   L       = -sum_i c_i sum_{t in i} w_t    (ratio form; its gradient equals the REINFORCE form's)
 *   dL/dH   = dZ W,  dL/dW = dZ^T H,   dZ_tv = -c_i w_t (1[v = y_t] - softmax(z_t)_v)
 *
 * Batch invariance: every per-row output (logpi, lse, w, token loss, grad_hidden row) has the same
 * bits whatever batch the row sits in, at whatever position, and whether it is scored alone
 * (T = 1 per call) or packed: one tile shape, a fixed K order and a fixed vocabulary-chunk order,
 * independent of T; no atomics in any reduction.
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE memory owned by the caller; the library allocates nothing and
 *     keeps no state between calls.  bf16 arrays are passed as uint16_t bit patterns, row-major.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream) and returns
 *     without synchronising.
 *   - The return value reports errors that the host can see before launching: a NULL pointer,
 *     an unsupported shape, a misaligned pointer (16 bytes for hidden, w_lm, grad_hidden, grad_w),
 *     a workspace that is too small, or a failed launch (BI_ERR_CUDA).  Nothing is launched when
 *     the return value is not BI_OK.
 *   - Errors found on the device are written to *dev_status (int32, caller-owned, device memory):
 *     the library first sets it to BI_OK, then kernels may raise it to BI_ERR_BAD_TARGET (a target
 *     outside [0, V)), BI_ERR_BAD_OFFSETS (inconsistent offsets), BI_ERR_NONFINITE (a non-finite
 *     weight, D3 term or loss) or BI_ERR_TIMEOUT (a bounded wait inside a kernel ran out; the
 *     kernel returned early and its outputs are undefined).  Read it after synchronising.
 *     Kernels never trap.
 *   - Supported shapes: H a multiple of 64 such that H / C is a multiple of 64 and at most 384
 *     for some C in 1..8 (e.g. 128, 1536, 2048, 2560, 3072); 1 <= V < 2^31; 0 <= T < 2^31.
 */
#ifndef BI_ISLOSS_H
#define BI_ISLOSS_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BI_API __attribute__((visibility("default")))
#else
#define BI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BI_OK = 0,
  BI_ERR_INVALID_ARG = 1,       /* NULL pointer, negative size, misaligned pointer */
  BI_ERR_UNSUPPORTED_SHAPE = 2, /* H not supported (see above) */
  BI_ERR_WORKSPACE = 3,         /* ws == NULL or ws_bytes below the size the call needs */
  BI_ERR_CUDA = 4,              /* a CUDA runtime call or launch failed */
  BI_ERR_TIMEOUT = 5,           /* device: a bounded wait ran out */
  BI_ERR_BAD_TARGET = 6,        /* device: a target id outside [0, V) */
  BI_ERR_NONFINITE = 7,         /* device: non-finite IS weight, D3 term or loss */
  BI_ERR_BAD_OFFSETS = 8        /* device: offsets not monotone / not covering the rows */
} bi_status;

/* Diagnostics of one call, written by the library to device memory.
 *   mean, max, count, n_nonfinite: D3 statistics ("Zero Mismatch", section "Only one probability
 *     gap ..."): mean and max of d3_t = w_t - 1 - log w_t over the scored tokens, the number of
 *     scored tokens and the number of non-finite terms; mean and max are non-finite when any term
 *     is.
 *   k1_mean, k2_mean: the other sampled estimators of the rollout-to-learner KL(mu || pi) from the
 *     rollout's tokens (the pages plot a "sampled estimate" of this KL): means of -delta and of
 *     delta^2 / 2, delta = log pi - log mu.  D3 is the third one, k3.
 *   n_clipped: tokens whose gradient the PPO clip removed (BI_LOSS_PPO_CLIP), else 0.
 *   n_rejected: responses the sequence gate rejected (BI_LOSS_SEQ_GATE), else 0.
 * bi_d3_stats fills mean ... k2_mean and sets both counters to 0. */
typedef struct {
  float mean;
  float max;
  int64_t count;
  int64_t n_nonfinite;
  float k1_mean;
  float k2_mean;
  int32_t n_clipped;
  int32_t n_rejected;
} bi_d3;

/* Loss of bi_is_loss_fwd_bwd.  The method is the unclipped one; the two others are the baselines
 * the pages compare it with ("Zero Mismatch", section "Alignment permits a simpler learning path":
 * clipping suppresses excursions but biases, rejection gates discard samples).  The pages give no
 * formula for either; the readings:
 *   BI_LOSS_UNCLIPPED  l_t = -c_i w_t, c_i = A_i / (R* n_i)
 *   BI_LOSS_PPO_CLIP   l_t = -min(w_t A_i, clip(w_t, 1 - eps_low, 1 + eps_high) A_i) / (R* n_i),
 *                      differentiated through w_t only (no gradient where the clipped term is the
 *                      smaller one)
 *   BI_LOSS_SEQ_GATE   the unclipped terms, except that response i contributes nothing (loss and
 *                      gradient) when its mean token log-ratio rho_i = mean_t (log pi_t - log mu_t)
 *                      has |rho_i| > gate or is not finite; it still counts in R*. */
typedef enum { BI_LOSS_UNCLIPPED = 0, BI_LOSS_PPO_CLIP = 1, BI_LOSS_SEQ_GATE = 2 } bi_loss_variant;

/* bi_loss_cfg.flags.  BI_LOSS_STORE_P opts in to the P store: the forward writes every bf16 tile
 * e^{z - m} of the exponentiated logits to the workspace (about 2 T (V + 384) bytes, 23 GB for
 * T = 76,000 rows of a 151,936-token vocabulary; size from bi_workspace_bytes_pstore) and dW is
 * one GEMM over those tiles instead of a second pass over the logits.  This MATERIALISES THE
 * T x V LOGITS (as probabilities) IN DEVICE MEMORY; without the flag nothing of size T x V is
 * ever written.  Both paths give the same bits for every output except grad_w, where they differ
 * by rounding only. */
#define BI_LOSS_STORE_P 1

typedef struct {
  int32_t variant;  /* bi_loss_variant */
  float eps_low;    /* PPO_CLIP: >= 0 */
  float eps_high;   /* PPO_CLIP: >= 0 */
  float gate;       /* SEQ_GATE: >= 0 (may be +inf) */
  int32_t flags;    /* 0 or BI_LOSS_STORE_P; other bits: BI_ERR_INVALID_ARG */
} bi_loss_cfg;

/* Size in bytes of the scratch workspace for these sizes (R = number of responses; pass 0 for
 * bi_logprob_fwd / bi_d3_stats).  Deterministic and free of side effects; the caller allocates
 * the workspace (256-byte aligned) and may reuse it across calls on the same stream.
 * Nothing in it has T x V entries.  For bi_is_loss_fwd_bwd it holds O(T) per-row arrays, a compact
 * copy of the scored hidden rows (T H bf16), per-response coefficients and a fixed-size scratch for
 * the tiles the cluster passes between its CTAs; dW recomputes the logits tile by tile.
 * For bi_logprob_fwd with 1 <= T <= 128 rows (decode-style scoring) it also holds what the all-SM
 * path keeps: each row's maximum over every 128-column sub-tile (64-column where 128 does not
 * divide the logit-tile width; one 8-byte word each), each step's reference and the 32-column
 * partial sums of e^{z - m} (about 4 T V / 18 bytes at H = 1536, V = 151936: 1/18 of the rows'
 * fp32 logits), so that the call runs on every SM instead of one cluster; the bits are the same
 * either way. */
BI_API size_t bi_workspace_bytes(int64_t T, int32_t H, int32_t V, int32_t R);

/* Smallest workspace accepted.  For bi_is_loss_fwd_bwd it equals bi_workspace_bytes.  For R = 0 it
 * is the per-CTA partials only: bi_logprob_fwd accepts it for any T (with T <= 128 it then scores
 * the rows on one cluster, with the same bits). */
BI_API size_t bi_workspace_bytes_min(int64_t T, int32_t H, int32_t V, int32_t R);

/* Workspace of bi_is_loss_fwd_bwd with BI_LOSS_STORE_P in cfg->flags (R >= 1; 0 otherwise): the
 * default workspace plus the P store, the per-step reference history ([ceil(V / 128)][T'] float)
 * and the scaled hidden states of the dW GEMM ([T'][H] bf16), T' = T rounded up to 128. */
BI_API size_t bi_workspace_bytes_pstore(int64_t T, int32_t H, int32_t V, int32_t R);

/* Token log-probabilities log pi(y_t | h_t) under the LM head W (definition above).
 *   hidden   [T, H] bf16      rows to score (row-major, 16-byte aligned)
 *   w_lm     [V, H] bf16      LM-head weight (row-major, 16-byte aligned)
 *   targets  [T]    int32     token ids; an id outside [0, V) sets BI_ERR_BAD_TARGET and NaN
 *   logprob  [T]    float     out: z_{t,y_t} - lse_t
 *   lse      [T]    float     out (may be NULL): log-sum-exp of the row's logits
 * A row gets identical bits whether it is scored alone (T = 1, decode style) or packed.  Packed
 * batches run on the cluster kernel (one cluster sweeps the vocabulary for each 128-row tile).
 * With 1 <= T <= 128 and a workspace of bi_workspace_bytes(T, H, V, 0) bytes the rows are scored
 * on every SM instead, in one cooperative pass over W: the logits of 128-column sub-tiles with the
 * cluster kernel's per-column instruction sequence give the row maxima, every CTA advances the
 * reference chain once the maxima of the tiles it needs are stored, forms the 32-column partial
 * sums against each step's reference, and a per-row combine follows the cluster kernel's class
 * order, which reproduces its bits ("Zero Mismatch, Simple Async RL", section "Alignment permits a
 * simpler learning path").  Without cooperative launch support the rows go to the cluster kernel,
 * with the same bits. */
BI_API bi_status bi_logprob_fwd(const uint16_t* hidden, const uint16_t* w_lm, const int32_t* targets,
                         int64_t T, int32_t H, int32_t V, float* logprob, float* lse,
                         int32_t* dev_status, void* ws, size_t ws_bytes, void* stream);

/* bi_logprob_fwd for callers that cannot allocate device memory.  The source pages have no
 * counterpart of this entry point; it exists for code that runs inside a host framework which
 * owns every device allocation (a serving engine's fixed memory pool, a plugin given no allocator
 * handle) and so cannot pass a workspace.  Arguments and results are those of bi_logprob_fwd
 * without the workspace; the forward's per-CTA partials live in a fixed device array inside the
 * library (480 KB, one [2][3][128] float block per CTA of a full-device grid, held by every GPU
 * that loads the library until the process exits).  Its size does not depend on T: any T that
 * bi_logprob_fwd accepts is accepted, and the results are bit-identical to bi_logprob_fwd's
 * (it always runs the cluster kernel, whose bits both of bi_logprob_fwd's paths have).
 *   - The call allocates nothing (no cudaMalloc, no library allocator).  Its first call on a
 *     device looks up the array's device address with that device current; make that first call
 *     before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents (every value read is
 *     written first by the same call).  Calls whose kernels overlap on the GPU -- different
 *     streams or host threads without ordering between them -- race on it and must be serialised
 *     by the caller. */
BI_API bi_status bi_logprob_fwd_noalloc(const uint16_t* hidden, const uint16_t* w_lm,
                                        const int32_t* targets, int64_t T, int32_t H, int32_t V,
                                        float* logprob, float* lse, int32_t* dev_status,
                                        void* stream);

/* Fused forward + backward of the token-level IS REINFORCE loss (unclipped unless cfg says
 * otherwise).
 *   hidden, w_lm, targets, T, H, V   as in bi_logprob_fwd (T = all packed rows)
 *   rollout_logprob [T] float   log mu of each row's target under the rollout policy
 *   rewards        [R] float    one reward per response
 *   resp_offsets [R+1] int64    rows of response i are [resp_offsets[i], resp_offsets[i+1]);
 *                               resp_offsets[0] = 0, resp_offsets[R] = T, non-decreasing
 *   group_offsets [G+1] int32   responses of group k are [group_offsets[k], group_offsets[k+1]);
 *                               group_offsets[0] = 0, group_offsets[G] = R, non-decreasing
 *   prompt_lens      [R] int32  (may be NULL) the first prompt_lens[i] rows of response i are not
 *                               scored (0 <= prompt_lens[i] <= its length)
 *   resp_normalizer  R* in c_i = A_i / (R* n_i); 0 means R.  Data-parallel callers pass the
 *                               global number of responses.
 *   cfg              (may be NULL: BI_LOSS_UNCLIPPED, no flags) host pointer, read during the
 *                               call; with BI_LOSS_STORE_P in cfg->flags ws_bytes must be at least
 *                               bi_workspace_bytes_pstore(T, H, V, R), else BI_ERR_WORKSPACE
 * Outputs (device):
 *   loss        [1]    float   L (sum over scored tokens in a fixed order, float64 accumulation)
 *   logprob     [T]    float   log pi_t on scored rows, 0 on prompt rows
 *   is_weight   [T]    float   (may be NULL) w_t, 0 on prompt rows
 *   token_loss  [T]    float   (may be NULL) l_t of the loss variant, 0 on prompt rows
 *   d3          [1]    bi_d3   (may be NULL) D3, KL estimators and variant counters
 *   grad_hidden [T, H] bf16    dL/dh_t (zero rows for prompt rows)
 *   grad_w      [V, H] float   dL/dW, overwritten (not accumulated)
 * A response with no scored row contributes 0 and still counts in R*. */
BI_API bi_status bi_is_loss_fwd_bwd(const uint16_t* hidden, const uint16_t* w_lm, const int32_t* targets,
                             const float* rollout_logprob, const float* rewards,
                             const int64_t* resp_offsets, const int32_t* group_offsets,
                             const int32_t* prompt_lens, int32_t R, int32_t G,
                             double resp_normalizer, const bi_loss_cfg* cfg, int64_t T, int32_t H,
                             int32_t V, float* loss, float* logprob, float* is_weight, float* token_loss,
                             bi_d3* d3, uint16_t* grad_hidden, float* grad_w,
                             int32_t* dev_status, void* ws, size_t ws_bytes, void* stream);

/* D3 statistics from two logprob arrays ("Zero Mismatch", "Only one probability gap ..."):
 *   learner_logprob [T] float, rollout_logprob [T] float, mask [T] uint8 (may be NULL: all rows;
 *   otherwise rows with mask != 0).  out [1] bi_d3 in device memory.  Sets BI_ERR_NONFINITE in
 *   *dev_status when a term is non-finite.  The terms are summed in float64 in a fixed order:
 *   per block of 8192 rows, then over the blocks (16-byte loads when the two arrays are 16-byte
 *   aligned and the mask 4-byte aligned, element loads otherwise, with the same sums). */
BI_API bi_status bi_d3_stats(const float* learner_logprob, const float* rollout_logprob,
                      const uint8_t* mask, int64_t T, bi_d3* out, int32_t* dev_status, void* ws,
                      size_t ws_bytes, void* stream);

/* Static, NUL-terminated name of a status code ("BI_OK", ...); "BI_UNKNOWN" otherwise. */
BI_API const char* bi_status_string(bi_status s);

/* Library version as an integer (major * 10000 + minor * 100 + patch). */
BI_API int32_t bi_version(void);

/* Test hook, not for production use: the next call of bi_logprob_fwd on this host thread makes
 * one epilogue wait in the forward kernel wait on a barrier that nothing signals, with the given
 * limit in nanoseconds, so that the bounded-wait path (BI_ERR_TIMEOUT, early return, TMEM freed)
 * can be exercised without hanging the GPU.  0 disables the hook. */
BI_API void bi_debug_force_timeout_once(uint64_t limit_ns);

/* Kernel timing for measurement tools (not needed for correctness).  bi_profile_enable(1) makes
 * every later call on this host thread record a CUDA event pair around each kernel launch on the
 * call's stream and accumulate the elapsed times; bi_profile_enable(0) stops it.
 * bi_profile_read(names_out, ms_out, launches_out, max_kernels) synchronises on the recorded events,
 * writes up to max_kernels entries (kernel name as a static string, total milliseconds, number of
 * launches) and returns the number of kernel kinds; bi_profile_reset() clears the totals.
 * Returns -1 if a CUDA event call failed. */
BI_API void bi_profile_enable(int32_t on);
BI_API void bi_profile_reset(void);
BI_API int32_t bi_profile_read(const char** names_out, double* ms_out, int64_t* launches_out,
                               int32_t max_kernels);

#ifdef __cplusplus
}
#endif

#endif /* BI_ISLOSS_H */
