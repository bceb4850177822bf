/*
 * rkl.h -- C ABI of librkl.so: exact full-vocabulary reverse-KL distillation
 * loss on NVIDIA B200 (sm_100a).
 *
 * The operation (NeMo RL PR #3978, "feat(mopd): add full-vocabulary on-policy
 * distillation", description):
 *
 *     L_t = sum_v p_s(v) * (log p_s(v) - log p_t(v)),   p = softmax(z)
 *
 * for every trainable position t of a [B, S-1] batch, where the student logits
 * are z_s = h_s W_s^T and the teacher logits are either z_t = h_t W_t^T
 * (hidden-state payload) or shipped directly (logits payload) -- same page,
 * payload bullets.  Only the N loss-masked rows are projected ("fix(megatron):
 * compact actor logits before projection", slime PR #2310, Summary).  The
 * backward is the shared one of PR #3978's first implementation note,
 * dL/dz_s = p_s * (w - L) with w = log p_s - log p_t, recomputing the
 * log-softmaxes instead of caching [N, V].
 *
 * Conventions for every entry point:
 *  - Row-major tensors.  T = B * Sm1 token rows; row r = b * Sm1 + t predicts
 *    token t + 1 of sequence b.  h_* are [T, H]; W_* are [V, H]; teacher logits
 *    are [T, V]; the mask and the per-token loss are [B, Sm1].
 *  - All pointers are DEVICE pointers unless stated, owned by the caller.  The
 *    library never allocates device memory: scratch comes from the caller's
 *    workspace (size from rkl_workspace_size).  Teacher inputs are read-only
 *    and get no gradient (PR #3978, implementation note 5: the teacher LM head
 *    is held outside the trained parameters).
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *    enqueued on it; no entry point synchronises the host except
 *    rkl_device_error.
 *  - Errors are returned, never thrown or aborted on.  Arguments are checked
 *    before any launch; on error nothing is enqueued and rkl_last_error()
 *    (thread-local) describes the problem.
 *  - Data pointers must be 16-byte aligned (RKL_ERR_ALIGN).  For RKL_BF16, H
 *    must be a multiple of 64 and, on the logits payload, V a multiple of 8
 *    (row pitch of 16 bytes); RKL_FP32 accepts any H and V >= 1.
 *  - Results are deterministic: the same inputs give bitwise-equal outputs,
 *    and a row's loss and dH row do not depend on which other rows are in the
 *    batch.
 *  - The trainable-row count.  Every entry point that takes `int32_t N` also
 *    takes `const int32_t* n_dev` (device, 4-byte aligned, nullable):
 *      n_dev == NULL: N is the exact count (a host value, e.g. read back
 *                     from rkl_compact_rows);
 *      n_dev != NULL: N is an upper bound (normally B*Sm1; the workspace and
 *                     `saved` are sized for it) and the kernels read the
 *                     count from *n_dev when they run, clamped to [0, N].
 *    With n_dev a whole step (compaction, forward, backward) is enqueued with
 *    no host synchronisation and no device-to-host copy; the mask may change
 *    from step to step.  Outputs are the same in both modes; the device mode
 *    always gathers the trainable rows (the host mode skips the gather when
 *    N = B*Sm1).  `saved` offsets (the top-k entry points' second block) are
 *    taken from N in both modes, so forward and backward must be given the
 *    same N.
 */
#ifndef RKL_H
#define RKL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum rkl_status {
  RKL_OK = 0,
  RKL_ERR_NULL = 1,        /* a required pointer is NULL */
  RKL_ERR_SHAPE = 2,       /* a size is out of range or inconsistent */
  RKL_ERR_DTYPE = 3,       /* unknown dtype / payload / reduction enum value */
  RKL_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned */
  RKL_ERR_WORKSPACE = 5,   /* workspace NULL or smaller than rkl_workspace_size */
  RKL_ERR_UNSUPPORTED = 6, /* option with no code path (rejected, not ignored) */
  RKL_ERR_CUDA = 7,        /* a CUDA runtime/driver call failed */
  RKL_ERR_DEVICE = 8       /* a kernel's bounded wait ran out (rkl_device_error) */
} rkl_status;

typedef enum rkl_dtype { RKL_BF16 = 0, RKL_FP32 = 1 } rkl_dtype;

/* PR #3978, second implementation note: token-level mean, or the nested
 * per-sequence average under token_level_loss=false.  NONE returns only the
 * per-token tensor. */
typedef enum rkl_reduction {
  RKL_REDUCE_NONE = 0,
  RKL_REDUCE_TOKEN_MEAN = 1,        /* sum_k L_k / N            (0 when N = 0) */
  RKL_REDUCE_SEQ_MEAN_NESTED = 2    /* mean over sequences with n_b > 0 of
                                       sum_{t in b} L_t / n_b   (0 when N = 0) */
} rkl_reduction;

/* PR #3978, payload bullets: full.teacher_payload = hidden_states | logits.
 * LOGITS_PAIR: the student's logits are given too (rkl_*_logits_pair).
 * TOPK_HIDDEN / TOPK_LOGITS: only for rkl_workspace_size, the workspaces of
 * rkl_forward_topk_hidden / rkl_backward_topk_hidden and
 * rkl_forward_topk_logits / rkl_backward_topk_logits. */
typedef enum rkl_payload {
  RKL_PAYLOAD_HIDDEN = 0,
  RKL_PAYLOAD_LOGITS = 1,
  RKL_PAYLOAD_LOGITS_PAIR = 2,
  RKL_PAYLOAD_TOPK_HIDDEN = 3,
  RKL_PAYLOAD_TOPK_LOGITS = 4
} rkl_payload;

/* Library version string (static storage). */
const char* rkl_version(void);

/* Description of the last error on the calling thread ("" if none). */
const char* rkl_last_error(void);

/* Bytes of device workspace that rkl_forward_* and rkl_backward need for at
 * most n_max trainable rows (n_max <= B*Sm1) of the given problem.  The same
 * workspace may be reused by consecutive calls on one stream; calls that run
 * concurrently need separate workspaces.  Content need not be initialised. */
rkl_status rkl_workspace_size(rkl_payload payload, rkl_dtype dtype, int64_t n_max,
                              int64_t B, int64_t Sm1, int64_t H, int64_t V,
                              size_t* bytes /* host out */);

/* S1, compaction (slime PR #2310, Summary: project only the N loss-masked
 * rows).  row_idx[k] = flattened index b*Sm1+t of the k-th nonzero entry of
 * mask [B, Sm1] (uint8, nonzero = trainable), strictly ascending; *n_dev = N.
 * row_idx must hold B*Sm1 int32.  Bit-exact, deterministic.  The next calls
 * either take N from the host (one 4-byte device-to-host copy after this
 * call) or read *n_dev on the device (pass n_dev to them, see the
 * conventions above). */
rkl_status rkl_compact_rows(const uint8_t* mask, int64_t B, int64_t Sm1,
                            int32_t* row_idx, int32_t* n_dev, void* stream);

/* S2-S4, forward on the hidden-state payload (PR #3978, payload bullet 1).
 * h_s, h_t [T, H]; W_s, W_t [V, H]; dtype of all four.  row_idx/N from
 * rkl_compact_rows.  Outputs (fp32):
 *   loss_tok [B, Sm1]  per-token loss, exact 0 at masked positions (nullable)
 *   loss     [1]       reduced loss (nullable; ignored for RKL_REDUCE_NONE)
 *   saved    [N, 3]    per-row (lse_s, lse_t, L) kept for rkl_backward
 * N = 0 gives loss 0 and all-zero loss_tok without NaN (slime PR #2310, Summary:
 * an empty mask still yields a well-defined zero gradient). */
rkl_status rkl_forward_hidden(const void* h_s, const void* h_t,
                              const void* W_s, const void* W_t, rkl_dtype dtype,
                              int64_t B, int64_t Sm1, int64_t H, int64_t V,
                              const int32_t* row_idx, int32_t N, const int32_t* n_dev,
                              rkl_reduction reduction,
                              float* loss_tok, float* loss, float* saved,
                              void* workspace, size_t workspace_bytes, void* stream);

/* S2-S4 + S8, forward on the logits payload (PR #3978, payload bullet 2: the
 * teacher ships full-vocabulary logits and needs no LM head).  teacher_logits
 * [T, V] of `dtype`, used as given (only rows in row_idx are read).  Same
 * outputs as rkl_forward_hidden. */
rkl_status rkl_forward_logits(const void* h_s, const void* W_s,
                              const void* teacher_logits, rkl_dtype dtype,
                              int64_t B, int64_t Sm1, int64_t H, int64_t V,
                              const int32_t* row_idx, int32_t N, const int32_t* n_dev,
                              rkl_reduction reduction,
                              float* loss_tok, float* loss, float* saved,
                              void* workspace, size_t workspace_bytes, void* stream);

/* rkl_forward_hidden / rkl_forward_logits plus per-token statistics of the
 * student distribution from the same pass (PR #3978, implementation note 1:
 * the kernels sit beside a chunked entropy kernel; slime PR #2310, Summary:
 * log-probability / entropy on the compacted rows, scattered back):
 *   targets        [B, Sm1] int32 target token id per position (nullable;
 *                  required for target_logprob; ids outside [0, V) give NaN)
 *   entropy        [B, Sm1] fp32 H(p_s) = -sum_v p_s log p_s (nullable)
 *   target_logprob [B, Sm1] fp32 log p_s(targets) (nullable)
 * Both outputs are exactly 0 at masked positions.  The loss outputs are
 * identical to those of the plain entry points. */
rkl_status rkl_forward_hidden_ex(const void* h_s, const void* h_t,
                                 const void* W_s, const void* W_t, rkl_dtype dtype,
                                 int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                 const int32_t* row_idx, int32_t N, const int32_t* n_dev,
                                 rkl_reduction reduction,
                                 float* loss_tok, float* loss, float* saved,
                                 const int32_t* targets, float* entropy, float* target_logprob,
                                 void* workspace, size_t workspace_bytes, void* stream);
rkl_status rkl_forward_logits_ex(const void* h_s, const void* W_s,
                                 const void* teacher_logits, rkl_dtype dtype,
                                 int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                 const int32_t* row_idx, int32_t N, const int32_t* n_dev,
                                 rkl_reduction reduction,
                                 float* loss_tok, float* loss, float* saved,
                                 const int32_t* targets, float* entropy, float* target_logprob,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* S5-S7, backward of either payload (PR #3978, first implementation note:
 * dL/dz_s = p_s (w - L), log-softmaxes recomputed, nothing [N, V] kept).
 *   payload   RKL_PAYLOAD_HIDDEN: teacher = h_t [T, H], W_t [V, H]
 *             RKL_PAYLOAD_LOGITS: teacher = teacher logits [T, V], W_t NULL
 *   saved     [N, 3] from the matching forward call on the same inputs
 *   grad_loss [1] dLoss upstream gradient of the reduced loss (nullable = 0;
 *             ignored for RKL_REDUCE_NONE)
 *   grad_tok  [B, Sm1] upstream gradient of loss_tok (nullable = 0)
 * Row weight of trainable row k: g_k = grad_tok[row] + grad_loss * w_k, with
 * w_k = 1/N (token mean) or 1/(B_eff * n_b) (nested mean).  Outputs (fp32,
 * overwritten): dH_s [T, H] with exact zero rows at masked positions, and
 * dW_s [V, H].  No gradient is produced for the teacher inputs. */
rkl_status rkl_backward(rkl_payload payload,
                        const void* h_s, const void* teacher,
                        const void* W_s, const void* W_t, rkl_dtype dtype,
                        int64_t B, int64_t Sm1, int64_t H, int64_t V,
                        const int32_t* row_idx, int32_t N, const int32_t* n_dev,
                        rkl_reduction reduction, const float* saved,
                        const float* grad_loss, const float* grad_tok,
                        float* dH_s, float* dW_s,
                        void* workspace, size_t workspace_bytes, void* stream);

/* Both sides as logits: the student's logits [T, V] are given as well as the
 * teacher's (the logits payload of PR #3978's payload bullet 2, meant for
 * numerical checks, with the student side also materialised).  Same loss
 * and saved scalars as rkl_forward_logits; bandwidth bound (reads 2 N V
 * elements).  Any V >= 1; rows are read with 16-byte loads when the row
 * pitch allows.  Workspace: rkl_workspace_size(RKL_PAYLOAD_LOGITS_PAIR, ...)
 * (H is ignored). */
rkl_status rkl_forward_logits_pair(const void* student_logits, const void* teacher_logits,
                                   rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t V,
                                   const int32_t* row_idx, int32_t N, const int32_t* n_dev,
                                   rkl_reduction reduction,
                                   float* loss_tok, float* loss, float* saved,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* Backward of rkl_forward_logits_pair: dz [T, V] of `dtype` (overwritten) =
 * dLoss/dz_s = g_k p_s (w - L) on trainable rows (row weight g_k as in
 * rkl_backward), exact zeros on masked rows.  Reads 2 N V and writes T V
 * elements. */
rkl_status rkl_backward_logits_pair(const void* student_logits, const void* teacher_logits,
                                    rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t V,
                                    const int32_t* row_idx, int32_t N, const int32_t* n_dev,
                                    rkl_reduction reduction, const float* saved,
                                    const float* grad_loss, const float* grad_tok, void* dz,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * Top-k estimator, both sides as [T, V] logits.  PR #3978, description: the
 * exact objective is the K = V limit of the top-k MOPD estimator, whose
 * score-function tail term vanishes when the support spans the vocabulary.
 * The page does not write the estimator out; this library's reading:
 *   S      = the k largest student logits of the row (ties: lower token id
 *            first); k = 0 gives an empty support, k >= V the whole row;
 *   L_hat  = sum_{v in S} p_s(v) w(v) + [y not in S] w(y), w = log p_s -
 *            log p_t, y = the position's sampled token (targets);
 *   dz_s   = g (p_s ([v in S](w + 1) - C) + [v = y] a), a = [y not in S]
 *            (w(y) + 1), C = sum_S p_s w + sum_S p_s + a.
 * Averaged over y ~ p_s, L_hat and dz_s are the exact loss and gradient; at
 * k = 0, L_hat is the sampled-token gap w(y); at k >= V they are the exact
 * ones.  Bandwidth bound: the forward reads the student row twice and the
 * teacher row once (plus the few teacher entries of S); rows whose k-th
 * logit sits in a run of more than 4096 near-equal logits take extra exact
 * passes.  The backward reads both rows once and writes dz once.
 * ------------------------------------------------------------------------ */

/* Forward of the top-k estimator.  targets [B, Sm1] int32 (device): the
 * sampled token of every position (only trainable positions are read; an id
 * outside [0, V) gives NaN for that row).  loss_tok / loss as
 * rkl_forward_logits_pair with L = L_hat.  saved [7 N] floats: [N, 3]
 * (lse_s, lse_t, L_hat) followed by [N, 4] (C, a, and the bit patterns of
 * the k-th key and of the last tied token id taken into S), for
 * rkl_backward_topk_pair.  k >= 0 (RKL_ERR_SHAPE otherwise).  Workspace:
 * rkl_workspace_size(RKL_PAYLOAD_LOGITS_PAIR, ...). */
rkl_status rkl_forward_topk_pair(const void* student_logits, const void* teacher_logits,
                                 rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t V,
                                 const int32_t* row_idx, int32_t N, const int32_t* n_dev, int64_t k,
                                 const int32_t* targets, rkl_reduction reduction,
                                 float* loss_tok, float* loss, float* saved,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* The same estimator on the hidden-state payload (bf16 only; RKL_FP32 gives
 * RKL_ERR_UNSUPPORTED): z_s = h_s W_s^T and z_t = h_t W_t^T as in
 * rkl_forward_hidden.  The forward writes the fp32 logits of at most 2048
 * compacted rows at a time into the workspace and selects / estimates on
 * them; the backward recomputes the logits tile by tile (bitwise the same
 * fp32 values, so the support is the forward's) and runs the gradient GEMMs
 * of rkl_backward.  Arguments as rkl_forward_hidden / rkl_backward plus k and
 * targets as rkl_forward_topk_pair; saved [7 N] as there; workspace:
 * rkl_workspace_size(RKL_PAYLOAD_TOPK_HIDDEN, ...).  Outputs dH_s [T, H] and
 * dW_s [V, H] as rkl_backward. */
rkl_status rkl_forward_topk_hidden(const void* h_s, const void* h_t,
                                   const void* W_s, const void* W_t, rkl_dtype dtype,
                                   int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                   const int32_t* row_idx, int32_t N, const int32_t* n_dev, int64_t k,
                                   const int32_t* targets, rkl_reduction reduction,
                                   float* loss_tok, float* loss, float* saved,
                                   void* workspace, size_t workspace_bytes, void* stream);

rkl_status rkl_backward_topk_hidden(const void* h_s, const void* h_t,
                                    const void* W_s, const void* W_t, rkl_dtype dtype,
                                    int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                    const int32_t* row_idx, int32_t N, const int32_t* n_dev,
                                    const int32_t* targets,
                                    rkl_reduction reduction, const float* saved,
                                    const float* grad_loss, const float* grad_tok,
                                    float* dH_s, float* dW_s,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* The same estimator on the logits payload (PR #3978, payload bullet 2: the
 * teacher ships its full-vocabulary logits), bf16 only: z_s = h_s W_s^T by
 * the tensor core, z_t the shipped teacher_logits [T, V] (V a multiple of 8)
 * as in rkl_forward_logits.  The forward writes the fp32 z_s of at most 2048
 * compacted rows at a time into the workspace, beside an exact fp32 copy of
 * those rows' teacher logits, and selects / estimates on them; the backward
 * recomputes z_s tile by tile (bitwise the same fp32 values) and runs the
 * gradient GEMMs of rkl_backward.  Arguments as rkl_forward_logits /
 * rkl_backward (payload RKL_PAYLOAD_LOGITS) plus k and targets as
 * rkl_forward_topk_pair; saved [7 N]; workspace:
 * rkl_workspace_size(RKL_PAYLOAD_TOPK_LOGITS, ...). */
rkl_status rkl_forward_topk_logits(const void* h_s, const void* W_s,
                                   const void* teacher_logits, rkl_dtype dtype,
                                   int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                   const int32_t* row_idx, int32_t N, const int32_t* n_dev, int64_t k,
                                   const int32_t* targets, rkl_reduction reduction,
                                   float* loss_tok, float* loss, float* saved,
                                   void* workspace, size_t workspace_bytes, void* stream);

rkl_status rkl_backward_topk_logits(const void* h_s, const void* W_s,
                                    const void* teacher_logits, rkl_dtype dtype,
                                    int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                    const int32_t* row_idx, int32_t N, const int32_t* n_dev,
                                    const int32_t* targets, rkl_reduction reduction, const float* saved,
                                    const float* grad_loss, const float* grad_tok,
                                    float* dH_s, float* dW_s,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* Backward of the top-k estimator: dz [T, V] of `dtype` (overwritten) with
 * exact zero rows at masked positions; row weights g as rkl_backward; saved
 * and targets from the matching forward call. */
rkl_status rkl_backward_topk_pair(const void* student_logits, const void* teacher_logits,
                                  rkl_dtype dtype, int64_t B, int64_t Sm1, int64_t V,
                                  const int32_t* row_idx, int32_t N, const int32_t* n_dev,
                                  const int32_t* targets,
                                  rkl_reduction reduction, const float* saved,
                                  const float* grad_loss, const float* grad_tok, void* dz,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------------
 * A teacher per row (hidden-state payload).  PR #3978, first-version limits:
 * the first version takes one teacher checkpoint and lays out the payload so
 * that a per-row teacher index can be added.  Here every position carries
 * the index k in [0, n_teachers) of its teacher, and the teacher logits of a
 * trainable row r are z_t = h_t[r] W_t[k_r]^T, with W_t the stacked teacher
 * heads [n_teachers, V, H] (all teachers share V and H).  The loss, the saved
 * scalars, the reductions and the gradients are those of the one-teacher
 * entry points.  1 <= n_teachers <= 16.
 *
 * Internally the compacted rows are regrouped by teacher into whole 256-row
 * tiles (padding rows between groups cost at most 255 rows per teacher of
 * extra tensor-core work), so every tile projects with one teacher head.
 * That layout is planned on the host from the per-teacher counts, so these
 * entry points take the exact N and counts from the host (no n_dev).
 * ------------------------------------------------------------------------ */

/* S1 with teacher counts.  teacher_idx [B, Sm1] int32 (device; entries at
 * masked positions are never read).  Writes row_idx / *n_dev exactly as
 * rkl_compact_rows, and counts [n_teachers + 1] (device): counts[g] = number
 * of trainable rows of teacher g, counts[n_teachers] = number of trainable
 * rows whose index lies outside [0, n_teachers) (such rows make the forward
 * and backward fail with RKL_ERR_SHAPE).  The caller reads counts back (a
 * (n_teachers + 1)-int copy) together with N. */
rkl_status rkl_compact_rows_multi(const uint8_t* mask, const int32_t* teacher_idx,
                                  int64_t B, int64_t Sm1, int32_t n_teachers,
                                  int32_t* row_idx, int32_t* n_dev, int32_t* counts, void* stream);

/* Workspace bytes of rkl_forward_hidden_multi / rkl_backward_hidden_multi
 * for up to n_max trainable rows. */
rkl_status rkl_workspace_size_multi(rkl_dtype dtype, int64_t n_max, int32_t n_teachers,
                                    int64_t B, int64_t Sm1, int64_t H, int64_t V, size_t* bytes);

/* Forward with a teacher per row.  Arguments as rkl_forward_hidden, plus:
 *   W_t          [n_teachers, V, H] stacked teacher heads (device)
 *   teacher_idx  [B, Sm1] int32 (device), the array given to compaction
 *   counts       [n_teachers] int32, HOST copy of the counts written by
 *                rkl_compact_rows_multi; they must add up to N
 *                (RKL_ERR_SHAPE otherwise).  Counts that do not belong to
 *                teacher_idx and the mask give unspecified (memory-safe)
 *                results.
 * Per-row entropy / target log-prob outputs are not offered in this mode. */
rkl_status rkl_forward_hidden_multi(const void* h_s, const void* h_t,
                                   const void* W_s, const void* W_t,
                                   int32_t n_teachers, const int32_t* teacher_idx,
                                   const int32_t* counts, rkl_dtype dtype,
                                   int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                   const int32_t* row_idx, int32_t N,
                                   rkl_reduction reduction,
                                   float* loss_tok, float* loss, float* saved,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* Backward with a teacher per row; arguments as rkl_backward (hidden
 * payload) plus those of rkl_forward_hidden_multi.  dH_s [T, H] and dW_s
 * [V, H] as rkl_backward; no gradient for any teacher input. */
rkl_status rkl_backward_hidden_multi(const void* h_s, const void* h_t,
                                    const void* W_s, const void* W_t,
                                    int32_t n_teachers, const int32_t* teacher_idx,
                                    const int32_t* counts, rkl_dtype dtype,
                                    int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                    const int32_t* row_idx, int32_t N,
                                    rkl_reduction reduction, const float* saved,
                                    const float* grad_loss, const float* grad_tok,
                                    float* dH_s, float* dW_s,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* rkl_forward_hidden without a caller workspace, for callers that cannot
 * allocate device memory when they call: a runtime that plans all device
 * memory up front and forbids allocation afterwards, code that runs where
 * cudaMalloc is not allowed or would stall (it can synchronise the device and
 * can fail under memory pressure), or a host with no device allocator of its
 * own.  The pages have no counterpart to this entry point; it is a packaging
 * convenience of this library.
 *
 * Arguments and outputs are those of rkl_forward_hidden.  The scratch is a
 * fixed 32 MiB array inside the library's device image: every GPU on which
 * the library is loaded holds it until the process exits.  A problem whose
 * forward needs more scratch (rows x hidden x dtype of the compacted student
 * and teacher rows, plus the partial statistics) is rejected with
 * RKL_ERR_WORKSPACE and a message giving both sizes; nothing is enqueued.
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.
 * This entry point allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library call.  All calls share the one array and each call
 * overwrites what it uses, so calls whose work can overlap on the GPU (other
 * streams, other host threads) race and must be serialised by the caller. */
rkl_status rkl_forward_hidden_noalloc(const void* h_s, const void* h_t,
                                      const void* W_s, const void* W_t, rkl_dtype dtype,
                                      int64_t B, int64_t Sm1, int64_t H, int64_t V,
                                      const int32_t* row_idx, int32_t N,
                                      rkl_reduction reduction,
                                      float* loss_tok, float* loss, float* saved,
                                      void* stream);

/* Synchronises the current device, then reports and clears the library's
 * device error word: *code = 0 if no kernel's bounded wait ran out since the
 * last call, else a nonzero bit set naming the wait (the kernel returned
 * early and its outputs are invalid).  Returns RKL_ERR_DEVICE when *code != 0. */
rkl_status rkl_device_error(int32_t* code /* host out */);

/* Measurement hooks (used by bench.py).  When enabled, every kernel launch of
 * the library is bracketed by CUDA events on the launching stream;
 * rkl_profile_read synchronises and returns, per kernel id, the summed device
 * time and the launch count since the last rkl_profile_reset. */
int32_t rkl_kernel_count(void);                 /* number of kernel ids */
const char* rkl_kernel_name(int32_t kernel_id); /* NULL if out of range */
rkl_status rkl_profile_enable(int32_t enable);
rkl_status rkl_profile_reset(void);
rkl_status rkl_profile_read(int32_t kernel_id, double* total_ms, int64_t* launches);
/* Total kernel launches issued by the library since load (host counter). */
int64_t rkl_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* RKL_H */
