/*
 * streamkl.h — C ABI of the fused attention-distillation KL divergence on
 * NVIDIA B200 (sm_100a).
 *
 * The operation ("StreamKL: Fast and Memory-Efficient KL Divergence for
 * Boosting Attention Distillation", abstract): one attention distribution,
 * the teacher P = softmax(scale_t * Q_t K_t^T), is compared with another, the
 * student Q = softmax(scale_s * Q_s K_s^T), row by row through their KL
 * divergence KL_i = sum_j P_ij (log P_ij - log Q_ij) (teacher in the first
 * slot, "Lecture 05 - Where It All Lands ...", section 3.1), and the loss is
 * the mean of KL_i over every (batch, head, query row).  The forward is one
 * pass over key tiles held on chip, keeping an online per-row state for both
 * distributions; the backward recomputes both distributions tile by tile from
 * the saved per-row log-sum-exps.  Neither pass writes an N_Q x N_K buffer,
 * and the library never allocates device memory: every buffer is the
 * caller's.
 *
 * Conventions shared by every entry point
 *  - Tensors are dense row-major with the head dimension innermost:
 *      Q_t [B, H, N_Q, d_t]   K_t [B, H, N_K, d_t]     (teacher, bf16)
 *      Q_s [B, H, N_Q, d_s]   K_s [B, H, N_K, d_s]     (student, bf16)
 *    per-row vectors are fp32 [B, H, N_Q]; gradients are fp32 and shaped like
 *    the tensor they belong to.
 *  - Every pointer is a DEVICE pointer on the current CUDA device, 16-byte
 *    aligned, unless stated otherwise.  Inputs are read only.  A pointer to
 *    an array with no elements (B*H*N_Q or B*H*N_K zero) may be NULL.
 *  - d_t and d_s must each be 64 or 128 (other sizes: STREAMKL_ERR_UNSUPPORTED).
 *    N_Q, N_K need not be multiples of any tile size.
 *  - causal: key j is visible to query i iff j <= i + (N_K - N_Q) (the mask's
 *    diagonal ends at the bottom-right corner); causal with N_Q > N_K is
 *    rejected (rows without a visible key).  Non-causal needs N_K >= 1.
 *  - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and is asynchronous: a return of STREAMKL_OK means the launch was
 *    accepted.  Errors found on the device (a bounded wait that gave up) are
 *    recorded in the caller's workspace and reported by streamkl_check().
 *  - `workspace` is device memory owned by the caller, at least 256 bytes,
 *    cleared once with streamkl_workspace_init() before first use.  Its first
 *    256 bytes hold a sticky device status word that kernels set when a
 *    bounded wait gives up; streamkl_check() reads and clears it.  A
 *    workspace of streamkl_workspace_size() bytes (more than 256 only for
 *    problems with few query tiles and long key ranges) also lets the
 *    forward and the query-side backward split each query tile's keys across
 *    several CTAs (partial results go to the bytes after the status word and
 *    are combined in a fixed order, so results are the same run to run;
 *    they match the unsplit path up to rounding).  Calls that share a
 *    256-byte workspace may overlap on the GPU (the word is only OR-ed);
 *    calls that share a larger one must be ordered (one stream), since their
 *    partial results would collide.
 *  - No entry point aborts, prints, or allocates; on an argument error nothing
 *    is launched.
 */
#ifndef STREAMKL_H
#define STREAMKL_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    STREAMKL_OK = 0,
    STREAMKL_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad shape or flag */
    STREAMKL_ERR_UNSUPPORTED = 2,   /* valid problem the kernels do not cover (d not 64/128, no sm_100 device) */
    STREAMKL_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
    STREAMKL_ERR_TIMEOUT = 4,       /* a kernel gave up on a bounded wait (see streamkl_check) */
    STREAMKL_ERR_WORKSPACE = 5,     /* workspace NULL or smaller than streamkl_workspace_size() */
    STREAMKL_ERR_BOUNDS = 6         /* bounds-checked build only: a kernel skipped an access outside its tensor */
} streamkl_status;

/* Bytes of device workspace that let streamkl_fwd and streamkl_bwd run this
 * problem on their fastest path on the current device: 256 (the status word)
 * plus, when the problem has too few 128-row query tiles to fill the GPU and
 * long enough key ranges, room for the partial results of key splits
 * (5 floats per row and split for the forward, d_s + d_t floats per row and
 * split for the query-side backward; at most a few tens of MB).  Any
 * workspace of at least 256 bytes is accepted; a smaller one than this
 * value only turns splitting off.  Arguments as in streamkl_fwd. */
size_t streamkl_workspace_size(int B, int H, int N_Q, int N_K, int d_t, int d_s, int causal);

/*
 * Forward.  For every (b, h, i) writes
 *   lse_t[b,h,i] = log sum_j exp(scale_t <Q_t[i], K_t[j]>)   (visible j, natural log)
 *   lse_s[b,h,i] = the same for the student
 *   kl[b,h,i]    = sum_j P_ij (log P_ij - log Q_ij)           (nats, not clamped)
 * and, if loss_mean != NULL, the device scalar loss_mean = mean over all
 * B*H*N_Q rows of kl (a deterministic reduction).
 * Source: the abstract's single one-pass forward kernel with the online
 * formulation of the coupled two-distribution KL reduction.
 * kl, lse_t, lse_s: required, fp32 [B,H,N_Q].  They are what streamkl_bwd needs.
 */
streamkl_status streamkl_fwd(const void *q_t, const void *k_t, const void *q_s, const void *k_s,
                             int B, int H, int N_Q, int N_K, int d_t, int d_s,
                             float scale_t, float scale_s, int causal,
                             float *kl, float *lse_t, float *lse_s, float *loss_mean,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * Backward.  With the upstream gradient g_i = dL/dKL_i taken from `dkl`
 * ([B,H,N_Q] fp32) or, when dkl == NULL, g_i = dloss / (B*H*N_Q) (the
 * gradient of loss_mean scaled by dloss), writes
 *   dq_s = dL/dQ_s, dk_s = dL/dK_s                (always; fp32)
 *   dq_t = dL/dQ_t, dk_t = dL/dK_t                (only if both are non-NULL)
 * where, per visible (i, j),
 *   dS_s = g_i (Q_ij - P_ij),  dS_t = g_i P_ij (log P_ij - log Q_ij - KL_i),
 *   dQ = scale * dS K,  dK = scale * dS^T Q   (teacher side with scale_t).
 * Source: the abstract's backward, which recomputes the attention
 * probabilities tile by tile instead of storing quadratic intermediates.
 * kl, lse_t, lse_s must be the outputs of streamkl_fwd on the same inputs.
 * Gradient outputs are overwritten (not accumulated).  dq_t and dk_t must be
 * both NULL (student gradients only) or both non-NULL.
 */
streamkl_status streamkl_bwd(const void *q_t, const void *k_t, const void *q_s, const void *k_s,
                             int B, int H, int N_Q, int N_K, int d_t, int d_s,
                             float scale_t, float scale_s, int causal,
                             const float *kl, const float *lse_t, const float *lse_s,
                             const float *dkl, float dloss,
                             float *dq_s, float *dk_s, float *dq_t, float *dk_t,
                             void *workspace, size_t workspace_bytes, void *stream);

/*
 * The two halves of streamkl_bwd, for callers that need only one side (a
 * frozen query or key projection) or that schedule them separately.  Same
 * arguments and meaning as streamkl_bwd.  streamkl_bwd_dk writes dk_s (and
 * dk_t if non-NULL); streamkl_bwd_dq writes dq_s (and dq_t if non-NULL).
 * Each recomputes both distributions on its own.
 */
streamkl_status streamkl_bwd_dk(const void *q_t, const void *k_t, const void *q_s, const void *k_s,
                                int B, int H, int N_Q, int N_K, int d_t, int d_s,
                                float scale_t, float scale_s, int causal,
                                const float *kl, const float *lse_t, const float *lse_s,
                                const float *dkl, float dloss, float *dk_s, float *dk_t,
                                void *workspace, size_t workspace_bytes, void *stream);
streamkl_status streamkl_bwd_dq(const void *q_t, const void *k_t, const void *q_s, const void *k_s,
                                int B, int H, int N_Q, int N_K, int d_t, int d_s,
                                float scale_t, float scale_s, int causal,
                                const float *kl, const float *lse_t, const float *lse_s,
                                const float *dkl, float dloss, float *dq_s, float *dq_t,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * streamkl_bwd with the scalar upstream gradient in DEVICE memory, so that a
 * caller such as an autograd engine never reads it back to the host:
 *   g_i = dkl[i]                       if dkl != NULL
 *   g_i = dloss_scale * (*dloss_dev)   otherwise (dloss_dev: device fp32 scalar)
 * e.g. dloss_scale = 1 / (B*H*N_Q) for the gradient of the mean loss, or
 * T^2 / (B*H*N_Q) for the temperature-scaled distillation loss
 * T^2 * mean KL ("Lecture 05 - Where It All Lands ...", section 3.3).
 * Every other argument, result and error as streamkl_bwd; both dkl and
 * dloss_dev NULL is STREAMKL_ERR_INVALID_ARG.
 */
streamkl_status streamkl_bwd_dloss_device(const void *q_t, const void *k_t, const void *q_s, const void *k_s,
                                          int B, int H, int N_Q, int N_K, int d_t, int d_s,
                                          float scale_t, float scale_s, int causal,
                                          const float *kl, const float *lse_t, const float *lse_s,
                                          const float *dkl, const float *dloss_dev, float dloss_scale,
                                          float *dq_s, float *dk_s, float *dq_t, float *dk_t,
                                          void *workspace, size_t workspace_bytes, void *stream);

/* loss_mean (device scalar) = mean of kl[0..n_rows) in a fixed summation
 * order (so repeated calls give identical bits); the same reduction
 * streamkl_fwd runs when its loss_mean argument is non-NULL. */
streamkl_status streamkl_loss_mean(const float *kl, long long n_rows, float *loss_mean, void *stream);

/* out (device scalar) = factor * sum of kl[0..n_rows), same fixed order and
 * fp64 accumulation as streamkl_loss_mean; factor = T^2 gives the summed
 * temperature-scaled loss, T^2 / n_rows its mean.  A NaN factor is
 * STREAMKL_ERR_INVALID_ARG. */
streamkl_status streamkl_loss_reduce(const float *kl, long long n_rows, double factor, float *out, void *stream);

/* Clears the workspace (enqueued on `stream`).  Needed once per workspace. */
streamkl_status streamkl_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/* Synchronises `stream` and returns STREAMKL_ERR_TIMEOUT if a kernel of an
 * earlier call on this workspace gave up on a bounded wait,
 * STREAMKL_ERR_INVALID_ARG if a kernel met a per-batch key length outside
 * [0, N_K] (streamkl_fwd_ex / streamkl_bwd_ex; the length was clamped),
 * STREAMKL_ERR_BOUNDS if (in the bounds-checked build, libstreamkl_checked.so)
 * a kernel found a TMA coordinate or global index outside its tensor and
 * skipped the access, STREAMKL_ERR_CUDA if the stream reports a CUDA error,
 * else STREAMKL_OK.  `code_out` (host pointer, nullable) receives the raw
 * device status word (0 = clean; bit 0 timeout, bit 1 bad length, bit 2
 * bounds, bits 8..15 which wait, bits 16..23 which checked access). */
streamkl_status streamkl_check(const void *workspace, void *stream, unsigned int *code_out);

/*
 * Padded batches and grouped key heads.
 * Source: the abstract of "StreamKL: ..." names sparse-attention LLM training
 * and long-context distillation as the uses; both feed batches of sequences
 * padded to a common length and models whose keys have fewer heads than their
 * queries.  The pages give no formula for either, so these take the plain
 * readings:
 *  - K_t is [B, H_kt, N_K, d_t] and K_s is [B, H_ks, N_K, d_s], H_kt and H_ks
 *    each >= 1 and dividing H (else STREAMKL_ERR_INVALID_ARG); query head h of
 *    batch b reads key head b * H_k + h / (H / H_k).  Q_t, Q_s and every
 *    per-row vector keep H heads.  dk_t and dk_s have their key tensor's shape:
 *    a key head's gradient is the sum over the query heads that read it
 *    (computed as one partial per query head in the workspace, then summed in
 *    a fixed order, so the result is the same run to run).
 *  - kv_len: DEVICE int32 [B] (4-byte aligned), or NULL for no padding.  Key j
 *    is visible to row i of batch b iff the causal rule above allows it AND
 *    j < kv_len[b] (the causal diagonal stays at N_K - N_Q).  A row with no
 *    visible key (kv_len[b] = 0) gets kl = 0, lse_t = lse_s = -inf and zero
 *    gradients; keys at and past kv_len[b] get zero dK rows.  Lengths are read
 *    on the device: one outside [0, N_K] is clamped to it and sets a bit that
 *    streamkl_check() reports as STREAMKL_ERR_INVALID_ARG.
 * With H_kt = H_ks = H and kv_len = NULL these are streamkl_fwd, streamkl_bwd.
 */

/* Workspace bytes for streamkl_fwd_ex / streamkl_bwd_ex on the current
 * device: streamkl_workspace_size plus, for the key gradients of grouped key
 * heads, B * H * N_K floats per grouped side (d_s for the student; d_t for
 * the teacher when teacher_grads != 0).  That part is REQUIRED by
 * streamkl_bwd_ex (a smaller workspace is STREAMKL_ERR_WORKSPACE); the rest
 * only enables key splits, as for streamkl_bwd. */
size_t streamkl_workspace_size_ex(int B, int H, int H_kt, int H_ks, int N_Q, int N_K, int d_t, int d_s, int causal,
                                  int teacher_grads);

/* streamkl_fwd with grouped key heads and padding (see above).  Arguments,
 * results and errors otherwise as streamkl_fwd; loss_mean is the mean over all
 * B*H*N_Q rows (rows of padded queries included: leave them out of a mean
 * with the per-row kl and weights). */
streamkl_status streamkl_fwd_ex(const void *q_t, const void *k_t, const void *q_s, const void *k_s,
                                int B, int H, int H_kt, int H_ks, int N_Q, int N_K, int d_t, int d_s,
                                float scale_t, float scale_s, int causal, const int *kv_len,
                                float *kl, float *lse_t, float *lse_s, float *loss_mean,
                                void *workspace, size_t workspace_bytes, void *stream);

/* streamkl_bwd with grouped key heads and padding (see above), taking every
 * form of the upstream gradient and either half of the backward:
 *   g_i = dkl[i]                      if dkl != NULL
 *   g_i = dloss * (*dloss_dev)        else if dloss_dev != NULL (device scalar)
 *   g_i = dloss / (B*H*N_Q)           otherwise
 * parts: 1 = key gradients (dk_s, dk_t), 2 = query gradients (dq_s, dq_t),
 * 3 = both (other values: STREAMKL_ERR_INVALID_ARG); the pointers of a part
 * not asked for are ignored.  The teacher pair of a part asked for must be
 * both NULL or both given (for parts = 3: all four teacher pointers alike).
 * kl, lse_t, lse_s must come from streamkl_fwd_ex with the same arguments. */
streamkl_status streamkl_bwd_ex(const void *q_t, const void *k_t, const void *q_s, const void *k_s,
                                int B, int H, int H_kt, int H_ks, int N_Q, int N_K, int d_t, int d_s,
                                float scale_t, float scale_s, int causal, const int *kv_len,
                                const float *kl, const float *lse_t, const float *lse_s,
                                const float *dkl, float dloss, const float *dloss_dev,
                                float *dq_s, float *dk_s, float *dq_t, float *dk_t, int parts,
                                void *workspace, size_t workspace_bytes, void *stream);

/*
 * Forward with no device memory from the caller beyond inputs and outputs.
 * (An addition of this library; the paper has no counterpart.)
 *
 * For callers that cannot allocate device memory at all, not even the small
 * workspace of streamkl_fwd: plug-in hosts that hand a library only buffers
 * they planned in advance, runtimes that forbid allocation once serving, and
 * programs whose memory pool owns the whole device.  Same arguments, results
 * and errors as streamkl_fwd, but the status word lives in a fixed 256-byte
 * array inside the library (a file-scope __device__ array that every GPU
 * loading the library keeps until the process exits).  Nothing is allocated:
 * no cudaMalloc, no cudaFree, no allocating library call.
 *  - The first call in each CUDA context (for runtime-API callers: once per
 *    device, in its primary context) looks up that array's device address
 *    with cudaGetSymbolAddress, with the context current, and caches it under
 *    the context's unique id; make that first call before any stream capture.
 *  - Arguments are checked before any CUDA call; a rejected call enqueues
 *    nothing and leaves the array as it was.  Each accepted call clears the
 *    status word at its start.  All calls in a context share the one array
 *    and it keeps the last call's contents, so calls that overlap on the GPU
 *    (different streams, no ordering) race on it.
 *  - The array holds the 256-byte minimum workspace that every problem runs
 *    with; the forward then does not split key ranges across CTAs (that
 *    needs the larger workspace streamkl_workspace_size reports), so no
 *    problem is rejected for size.
 *  - status_out (host pointer): if non-NULL the call synchronises `stream`,
 *    stores the device status word there (0 = clean) and returns
 *    STREAMKL_ERR_TIMEOUT if a bounded wait gave up; if NULL the call returns
 *    as soon as the work is enqueued.
 */
streamkl_status streamkl_fwd_noalloc(const void *q_t, const void *k_t, const void *q_s, const void *k_s,
                                     int B, int H, int N_Q, int N_K, int d_t, int d_s,
                                     float scale_t, float scale_s, int causal,
                                     float *kl, float *lse_t, float *lse_s, float *loss_mean,
                                     void *stream, unsigned int *status_out);

/*
 * Self-test of device failure reporting.  Launches one warp that waits, with
 * the same bounded wait every kernel of the library uses, on a barrier that is
 * never signalled; after budget_ns (1 ms .. 2 s, else STREAMKL_ERR_INVALID_ARG)
 * the wait gives up, ORs STREAMKL's timeout bit and the waiter id 63 (bits
 * 8..15) into the workspace status word, and the kernel returns normally.  A
 * following streamkl_check() on the same workspace then returns
 * STREAMKL_ERR_TIMEOUT and clears the word; the CUDA context stays usable.
 * Nothing faults and nothing hangs.  For tests of callers' error handling.
 */
streamkl_status streamkl_selftest_timeout(void *workspace, size_t workspace_bytes, unsigned long long budget_ns,
                                          void *stream);

/* Static, human-readable name of a status. */
const char *streamkl_strerror(streamkl_status status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int streamkl_version(void);

#ifdef __cplusplus
}
#endif

#endif /* STREAMKL_H */
