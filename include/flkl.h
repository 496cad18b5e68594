/*
 * flkl.h - C ABI of the fused linear-head + KL-divergence loss on B200 (sm_100a).
 *
 * The operation (the "Add FusedLinearKLDivLoss" pull-request page of the
 * Liger-Kernel mirror, sections Summary and Details): given hidden states
 * X[BT,H], a vocabulary head W[V,H] with optional bias b[V] and an explicit
 * teacher distribution Q[BT,V],
 *
 *     z   = X W^T + b,   u = z / T,   log p = log_softmax(u) per row,
 *     l_r = sum_v q_rv (log max(q_rv, eps) - log p_rv)   (q == 0 contributes 0)
 *     loss = sum over kept rows of l_r / D
 *
 * with D = N_valid (batchmean), N_valid * V (mean) or 1 (sum); a row is dropped
 * when its shift label equals ignore_index.  The gradients are produced in the
 * same call ("gradient in forward", page Details, third bullet):
 *
 *     G_r = (S_r p_r - q_r) / (T D)  on kept rows, 0 on dropped rows,
 *     S_r = sum_v q_rv,   dX = G W,   dW = G^T X,   db = sum_r G_r,
 *
 * and dW / db only when asked for (the frozen-head change of the GRPO page,
 * section Summary).  The BT x V logits are never written to device memory as
 * a whole: the library computes them tile by tile in two passes (statistics,
 * then the gradient per vocabulary chunk, recomputing the logits) and stages
 * only a bounded BT x Vc block of G (Vc about V/6, rounded up to the tile
 * width); on the bf16 path pass 1 keeps the fp32 logits of the first chunk
 * only (at most 256 MiB), from which that chunk's G is formed without a
 * second GEMM.
 *
 * Declared below, besides that call: the same path with a one-hot teacher
 * (cross-entropy) and as per-token log-probabilities with a separate backward
 * (selective log-probability), the Jensen-Shannon divergence against a
 * teacher head, a data-parallel form (whole-batch divisor), RMSNorm /
 * LayerNorm backward with frozen-parameter flags, an allocation-free variant,
 * workspace sizes, status and wait-limit helpers.
 *
 * Conventions for every entry point:
 *  - Pointers named "device" are CUDA device pointers on the current device;
 *    the caller owns and allocates all of them (inputs, outputs, workspace).
 *    The library allocates no device memory and keeps no per-call state.
 *  - Tensors are dense and row-major.  Every tensor base pointer must be
 *    16-byte aligned and H and V must be multiples of 8 (bf16) or 4 (fp32);
 *    otherwise the call returns FLKL_ERR_UNSUPPORTED without launching.
 *  - Calls are asynchronous on `stream` (a cudaStream_t, may be NULL for the
 *    legacy default stream).  A host-side argument error returns before any
 *    launch.  A device-side error (a bounded wait that ran out) is recorded
 *    in the workspace and read with flkl_device_status().
 *  - No entry point throws, traps or aborts.
 */
#ifndef FLKL_H_
#define FLKL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FLKL_ABI_VERSION 1

#if defined(__GNUC__)
#define FLKL_API __attribute__((visibility("default")))
#else
#define FLKL_API
#endif

/* Reductions.  Same meaning as torch.nn.KLDivLoss, restricted to kept rows
 * (page Details, first bullet).  FLKL_REDUCTION_NONE is refused with
 * FLKL_ERR_UNSUPPORTED: the gradient is computed with the loss and needs a
 * scalar loss (page Details, fourth bullet). */
typedef enum {
  FLKL_REDUCTION_BATCHMEAN = 0,
  FLKL_REDUCTION_MEAN = 1,
  FLKL_REDUCTION_SUM = 2,
  FLKL_REDUCTION_NONE = 3
} flkl_reduction;

/* Element type shared by X, W, b and Q (and of dX). */
typedef enum { FLKL_DTYPE_F32 = 0, FLKL_DTYPE_BF16 = 1 } flkl_dtype;

typedef enum {
  FLKL_OK = 0,
  FLKL_ERR_INVALID_ARG = 1, /* null/inconsistent pointer, bad size or scalar */
  FLKL_ERR_UNSUPPORTED = 2, /* reduction NONE, misalignment, size limits     */
  FLKL_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed          */
  FLKL_ERR_TIMEOUT = 4,     /* device: a bounded wait ran out (kernel quit)  */
  FLKL_ERR_WORKSPACE = 5,   /* workspace missing, misaligned or too small    */
  FLKL_ERR_TOO_LARGE = 6    /* sizes need more than FLKL_NOALLOC_SCRATCH_BYTES */
} flkl_status;

/* Version of this ABI (FLKL_ABI_VERSION of the built library). */
FLKL_API int flkl_abi_version(void);

/* Bytes of device workspace flkl_forward_backward needs for these sizes.
 * Returns 0 for invalid sizes.  The workspace must be 256-byte aligned; its
 * contents need no initialisation and are scratch between calls, except the
 * status word read by flkl_device_status(). */
FLKL_API size_t flkl_workspace_size(int64_t BT, int64_t H, int64_t V, int dtype, int compute_dW,
                           int compute_db);

/* Loss and gradients of the fused linear + KL(Q||P) loss, in one call.
 *
 *  X            device, [BT,H], dtype.
 *  W            device, [V,H], dtype.
 *  b            device, [V], dtype, or NULL (no bias).
 *  Q            device, [BT,V], dtype: teacher probabilities, used as given
 *               (not renormalised; rows need not sum to 1).
 *  shift_labels device, [BT] int64, or NULL (every row kept).  Only equality
 *               with ignore_index matters.
 *  ignore_index label value that drops a row (usually -100).
 *  BT, H, V     sizes; BT >= 0, H >= 1, V >= 1, each below 2^31.
 *  dtype        flkl_dtype.  BF16 runs on the tensor cores with fp32
 *               accumulation; F32 runs fp32 FMA throughout.
 *  temperature  T > 0, divides the student logits only.
 *  eps          >= 0; clamp inside log q only.
 *  reduction    flkl_reduction.
 *  compute_dW   nonzero: write dW; then dW must be non-NULL, else NULL.
 *  compute_db   nonzero: write db; needs b and a non-NULL db, else db NULL.
 *  accum_fp32   nonzero: dW and db are fp32; zero: they have `dtype`.
 *  loss         device, one fp32 (written).
 *  dX           device, [BT,H], dtype (overwritten).
 *  dW           device, [V,H] (overwritten) or NULL.
 *  db           device, [V] (overwritten) or NULL.
 *  workspace    device, flkl_workspace_size(...) bytes, 256-byte aligned.
 *  stream       cudaStream_t.
 *
 * Outputs are overwritten, never accumulated, and are gradients of the loss
 * itself (an autograd wrapper multiplies them by the incoming gradient).
 * Returns FLKL_OK once every kernel is enqueued.  With N_valid = 0 the loss
 * and every gradient are 0.  BT = 0 writes loss 0 (and zero dW/db). */
FLKL_API flkl_status flkl_forward_backward(const void* X, const void* W, const void* b, const void* Q,
                                  const int64_t* shift_labels, int64_t ignore_index, int64_t BT,
                                  int64_t H, int64_t V, int dtype, float temperature, float eps,
                                  int reduction, int compute_dW, int compute_db, int accum_fp32,
                                  float* loss, void* dX, void* dW, void* db, void* workspace,
                                  size_t workspace_bytes, void* stream);

/* Fused linear-head + cross-entropy loss: flkl_forward_backward with a
 * one-hot teacher at target[r], i.e. KL(onehot || P) = -log p_{r, target[r]}
 * (the cross-entropy of fused_linear_cross_entropy, which the
 * FusedLinearKLDivLoss page names in its Summary as the source of its chunk
 * geometry).  No teacher tensor is read.
 *
 *  target  device, [BT] int64: the class of each row; a row whose target
 *          equals ignore_index is dropped (it is the row mask too).  A
 *          target outside [0, V) that is not ignore_index gives its row no
 *          teacher mass: the row's loss and dX are 0 (such targets are not
 *          validated).
 *  Other arguments, outputs, workspace (flkl_workspace_size with the same
 *  sizes), reductions (batchmean divides by the kept rows, which is torch's
 *  cross_entropy "mean"), temperature and errors: as flkl_forward_backward;
 *  eps does not apply.  Loss = sum over kept rows of
 *  (logsumexp(z_r/T) - z_{r,target}/T) / D, dz = (p - onehot) / (T D). */
FLKL_API flkl_status flkl_ce_forward_backward(const void* X, const void* W, const void* b,
                                              const int64_t* target, int64_t ignore_index,
                                              int64_t BT, int64_t H, int64_t V, int dtype,
                                              float temperature, int reduction, int compute_dW,
                                              int compute_db, int accum_fp32, float* loss,
                                              void* dX, void* dW, void* db, void* workspace,
                                              size_t workspace_bytes, void* stream);

/* Selective log-probability (the GRPO frozen-head page, Summary: the chunked
 * per-token log-probability of the policy head, whose weight and bias
 * gradients are computed only when they are asked for).  Two calls on the
 * same workspace:
 *
 * flkl_selective_logprob_forward: logp[r] = z_{r,t}/T - logsumexp_v(z_{r,v}/T)
 *   with z = X W^T (+ b) and t = target[r]; 0 on rows whose target is
 *   ignore_index or outside [0, V).  logp: device fp32 [BT].  compute_dW /
 *   compute_db size the workspace (flkl_workspace_size with the same flags)
 *   for the backward call; nothing else is written.  The workspace keeps the
 *   row statistics for the backward call: do not use it for another call in
 *   between.
 * flkl_selective_logprob_backward: for upstream gradients dlogp [BT] (device
 *   fp32), dz_r = dlogp[r] (onehot(t) - softmax(z_r/T)) / T, and dX = dz W,
 *   dW = dz^T X (compute_dW), db = column sums of dz (compute_db), written as
 *   in flkl_forward_backward.  X, W, b, target, ignore_index, sizes, dtype,
 *   temperature and the flags must be those of the forward call.
 * Errors, alignment and asynchrony as flkl_forward_backward. */
FLKL_API flkl_status flkl_selective_logprob_forward(
    const void* X, const void* W, const void* b, const int64_t* target, int64_t ignore_index,
    int64_t BT, int64_t H, int64_t V, int dtype, float temperature, int compute_dW,
    int compute_db, float* logp, void* workspace, size_t workspace_bytes, void* stream);
FLKL_API flkl_status flkl_selective_logprob_backward(
    const void* X, const void* W, const void* b, const int64_t* target, int64_t ignore_index,
    int64_t BT, int64_t H, int64_t V, int dtype, float temperature, const float* dlogp,
    int compute_dW, int compute_db, int accum_fp32, void* dX, void* dW, void* db,
    void* workspace, size_t workspace_bytes, void* stream);

/* Fused linear Jensen-Shannon divergence (the FusedLinearKLDivLoss page,
 * Summary, names LigerFusedLinearJSD as the sibling loss whose teacher side
 * has its own projection; the pages print no formula, the generalized JSD is
 * the reading used).  Student P = softmax((X W^T + b)/T), teacher
 * Q = softmax((Xt Wt^T + bt)/T), M = beta P + (1 - beta) Q:
 *   loss = sum over kept rows of [beta KL(P||M) + (1 - beta) KL(Q||M)] / D
 * with the divisors, row mask (shift_labels), outputs, flags and errors of
 * flkl_forward_backward; only the student gets gradients,
 *   dz_rv = beta p_rv (log(p_rv / m_rv) - KL(P_r||M_r)) / (T D).
 *  Xt [BT, Ht], Wt [V, Ht], bt [V] (nullable): teacher hidden states and head,
 *  `dtype` like X; Ht a multiple of 8 (bf16) or 4 (fp32).  0 < beta < 1.
 *  workspace: flkl_jsd_workspace_size bytes (no BT x V buffer: two
 *  staging blocks of one vocabulary chunk and, on the tensor-core path, each
 *  side's fp32 logits of the first chunk, kept by its statistics pass when
 *  they fit 256 MiB, so that neither sweep recomputes them).  The
 *  probabilities of a chunk are staged in the input dtype (bf16 on the
 *  tensor-core path). */
FLKL_API size_t flkl_jsd_workspace_size(int64_t BT, int64_t H, int64_t Ht, int64_t V, int dtype,
                                        int compute_dW, int compute_db);
FLKL_API flkl_status flkl_jsd_forward_backward(
    const void* X, const void* W, const void* b, const void* Xt, const void* Wt, const void* bt,
    const int64_t* shift_labels, int64_t ignore_index, int64_t BT, int64_t H, int64_t Ht,
    int64_t V, int dtype, float temperature, float beta, int reduction, int compute_dW,
    int compute_db, int accum_fp32, float* loss, void* dX, void* dW, void* db, void* workspace,
    size_t workspace_bytes, void* stream);

/* Data-parallel use: the batch is split by rows over ranks that share the
 * head W, b (the row sharding of the scope table's multi-GPU row).  Each rank
 * calls flkl_count_valid on its labels (or targets), all-reduces the int64
 * count (sum) into `n_valid_total`, calls the _dp entry below, then
 * all-reduces loss, dW and db (sum); dX needs no exchange.  The _dp entries
 * are flkl_forward_backward / flkl_ce_forward_backward with the divisor of
 * the reduction taken from *n_valid_total (device int64, 8-byte aligned,
 * read on the device, non-NULL) instead of this call's kept rows, so the
 * per-rank results add up to the whole batch's.  No collective runs in the
 * library.
 *
 * flkl_count_valid: *count (device int64) = rows r < BT with labels[r] !=
 * ignore_index (labels NULL: BT).  Asynchronous on `stream`. */
FLKL_API flkl_status flkl_count_valid(const int64_t* labels, int64_t BT, int64_t ignore_index,
                                      int64_t* count, void* stream);
FLKL_API flkl_status flkl_forward_backward_dp(
    const void* X, const void* W, const void* b, const void* Q, const int64_t* shift_labels,
    int64_t ignore_index, int64_t BT, int64_t H, int64_t V, int dtype, float temperature,
    float eps, int reduction, int compute_dW, int compute_db, int accum_fp32, float* loss,
    void* dX, void* dW, void* db, void* workspace, size_t workspace_bytes, void* stream,
    const int64_t* n_valid_total);
FLKL_API flkl_status flkl_ce_forward_backward_dp(
    const void* X, const void* W, const void* b, const int64_t* target, int64_t ignore_index,
    int64_t BT, int64_t H, int64_t V, int dtype, float temperature, int reduction,
    int compute_dW, int compute_db, int accum_fp32, float* loss, void* dX, void* dW, void* db,
    void* workspace, size_t workspace_bytes, void* stream, const int64_t* n_valid_total);

/* Overlap of the data-parallel dW exchange with the remaining chunks.
 *
 * flkl_vocab_chunks: the vocabulary chunks of a call with these sizes and
 * flags; returns their number n (0 for invalid sizes or BT = 0) and, when
 * `bounds` is non-NULL, writes bounds[0..min(n, capacity)] (host int64):
 * chunk c covers dW / db rows [bounds[c], bounds[c+1]).
 *
 * The _dp_events entries are flkl_forward_backward_dp /
 * flkl_ce_forward_backward_dp that also record chunk_done[c] (a
 * cudaEvent_t created by the caller) on `stream` as soon as the dW rows of
 * chunk c are final, for c < n_events; a caller can then all-reduce those
 * rows on another stream (after cudaStreamWaitEvent) while the later chunks
 * run.  db and the loss are final only when the whole call is. */
FLKL_API int flkl_vocab_chunks(int64_t BT, int64_t H, int64_t V, int dtype, int compute_dW,
                               int compute_db, int64_t* bounds, int capacity);
FLKL_API flkl_status flkl_forward_backward_dp_events(
    const void* X, const void* W, const void* b, const void* Q, const int64_t* shift_labels,
    int64_t ignore_index, int64_t BT, int64_t H, int64_t V, int dtype, float temperature,
    float eps, int reduction, int compute_dW, int compute_db, int accum_fp32, float* loss,
    void* dX, void* dW, void* db, void* workspace, size_t workspace_bytes, void* stream,
    const int64_t* n_valid_total, void** chunk_done, int n_events);
FLKL_API flkl_status flkl_ce_forward_backward_dp_events(
    const void* X, const void* W, const void* b, const int64_t* target, int64_t ignore_index,
    int64_t BT, int64_t H, int64_t V, int dtype, float temperature, int reduction,
    int compute_dW, int compute_db, int accum_fp32, float* loss, void* dX, void* dW, void* db,
    void* workspace, size_t workspace_bytes, void* stream, const int64_t* n_valid_total,
    void** chunk_done, int n_events);

/* Gradient-in-forward scaling for autograd (the FusedLinearKLDivLoss page,
 * Details, bullet 3: the gradients come from the forward call; the backward
 * only applies the incoming gradient of the loss):
 *   dst[i] = dst_dtype(src[i] * *scale),  0 <= i < n
 * with the multiplication skipped when *scale == 1 (bitwise copy / cast).
 *  src, dst    device, 16-byte aligned; may be the same pointer only when
 *              src_dtype == dst_dtype (in place).  FLKL_DTYPE_F32 or
 *              FLKL_DTYPE_BF16 each (bf16 results rounded to nearest even).
 *  scale       device fp32 scalar read on the device (no host
 *              synchronisation), or NULL for 1.
 *  Asynchronous on `stream`.  n < 0, a bad dtype or a null src/dst with
 *  n > 0 gives FLKL_ERR_INVALID_ARG; misaligned pointers
 *  FLKL_ERR_UNSUPPORTED. */
FLKL_API flkl_status flkl_scale_cast(const void* src, int src_dtype, void* dst, int dst_dtype,
                                     int64_t n, const float* scale, void* stream);

/* Kinds of launches reported by flkl_forward_backward_profiled. */
typedef enum {
  FLKL_LAUNCH_PREPARE = 0,  /* valid-row count and divisor                   */
  FLKL_LAUNCH_STATS = 1,    /* pass 1: logits GEMM + softmax/KL statistics    */
  FLKL_LAUNCH_COMBINE = 2,  /* per-row log-sum-exp and row loss              */
  FLKL_LAUNCH_LOSS = 3,     /* reduction of the row losses                   */
  FLKL_LAUNCH_GRAD = 4,     /* pass 2 of one chunk: G staging (the logits     */
                            /* again, or the kept first-chunk logits)         */
  FLKL_LAUNCH_DW = 5,       /* dW chunk GEMM (fp32 path)                     */
  FLKL_LAUNCH_DX = 6,       /* dX chunk GEMM (fp32 path)                     */
  FLKL_LAUNCH_DB = 7,       /* db column reduction                           */
  FLKL_LAUNCH_ZERO = 8,     /* zero fill (BT = 0)                            */
  FLKL_LAUNCH_CHUNK = 9     /* bf16 path, one per vocabulary chunk c: dX(c), */
                            /* pass 2 of chunk c+1 and dW(c) in one launch   */
} flkl_launch_kind;

/* flkl_forward_backward with a timing record of every launch, for profiling.
 * `events` holds 2*capacity cudaEvent_t created by the caller; launch i
 * (i < capacity) is bracketed by events[2i] and events[2i+1], recorded on
 * `stream`; its flkl_launch_kind is written to the host array kinds[i] and
 * its GEMM FLOPs (2*M*N*K summed over the launch's problems, 0 for launches
 * without a GEMM) to the host array flops[i].  *n_launches (host) receives
 * the number of launches of the call (which may exceed capacity; the extra
 * ones are not recorded).  Same results and errors as
 * flkl_forward_backward, plus FLKL_ERR_INVALID_ARG for a null
 * events/kinds/flops/n_launches or a negative capacity.  With ce_target
 * non-NULL (and Q and shift_labels NULL) it profiles flkl_ce_forward_backward
 * instead (eps ignored). */
FLKL_API flkl_status flkl_forward_backward_profiled(
    const void* X, const void* W, const void* b, const void* Q, const int64_t* shift_labels,
    int64_t ignore_index, int64_t BT, int64_t H, int64_t V, int dtype, float temperature,
    float eps, int reduction, int compute_dW, int compute_db, int accum_fp32, float* loss,
    void* dX, void* dW, void* db, void* workspace, size_t workspace_bytes, void* stream,
    void** events, int* kinds, double* flops, int capacity, int* n_launches,
    const int64_t* ce_target);

/* Size of the fixed device scratch used by flkl_forward_backward_noalloc. */
#define FLKL_NOALLOC_SCRATCH_BYTES (128u << 20)

/* flkl_forward_backward for callers that cannot allocate device memory.
 *
 * No counterpart on the pages: this is a library convenience.  Some callers
 * cannot call cudaMalloc or hand over a workspace: code that runs inside a
 * host framework whose allocator owns every device byte (a plugin or
 * extension interface that passes in tensors but no scratch), or a
 * latency-critical loop where cudaMalloc's implicit device synchronisation
 * is not acceptable.  This entry point takes the same arguments minus the
 * workspace and uses a fixed scratch array of FLKL_NOALLOC_SCRATCH_BYTES
 * (128 MiB) that lives in the library itself: every GPU that loads the
 * library holds those 128 MiB until the process exits.  The caller still
 * passes every input and output.
 *
 *  - It allocates nothing and calls no allocating routine.
 *  - When flkl_workspace_size() exceeds FLKL_NOALLOC_SCRATCH_BYTES the call
 *    leaves out the first vocabulary chunk's kept logits and recomputes
 *    that chunk (the same results; BT=1024, H=4096, V=128256 with dW runs
 *    so in 119.8 MiB); sizes that need more even then return
 *    FLKL_ERR_TOO_LARGE before any launch.
 *  - Every call looks up the scratch address on the current device (a
 *    host-side lookup, so a device reset cannot leave a stale address); the
 *    first call on a device also loads the library's device code there, so
 *    make that first call before any stream capture.
 *  - Every call on a device shares the one scratch array, which keeps the
 *    previous call's contents (the call initialises what it reads).  Calls
 *    that can overlap on the GPU (different streams, or different host
 *    threads) race on it and give wrong results: serialise them.
 *  - A device-side wait that runs out is recorded in the shared scratch and
 *    cannot be read back through this entry point; use
 *    flkl_forward_backward with a workspace when that status is needed. */
FLKL_API flkl_status flkl_forward_backward_noalloc(
    const void* X, const void* W, const void* b, const void* Q, const int64_t* shift_labels,
    int64_t ignore_index, int64_t BT, int64_t H, int64_t V, int dtype, float temperature,
    float eps, int reduction, int compute_dW, int compute_db, int accum_fp32, float* loss,
    void* dX, void* dW, void* db, void* stream);

/* RMSNorm / LayerNorm backward with frozen-parameter flags (the LoRA
 * normalization pull-request page, Key Changes: COMPUTE_DW for RMSNorm,
 * COMPUTE_DW / COMPUTE_DB for LayerNorm; with a frozen parameter its gradient
 * is neither accumulated nor reduced and dX is unchanged).
 *
 *   RMSNorm:   y = w * x / sqrt(mean(x^2) + eps)
 *   LayerNorm: y = w * (x - mean(x)) / sqrt(var(x) + eps) + b  (biased var)
 *
 * over the last dimension of x [rows, H], for the incoming gradient dY
 * [rows, H]; the row statistics are recomputed from X.
 *
 *  dY, X, W     device; dY and X [rows, H], W [H]; all `dtype`.
 *  rows, H      rows >= 0; 1 <= H <= 8192 and H a multiple of 8.
 *  eps          >= 0.
 *  compute_dW   nonzero: write dW [H] (dW non-NULL), else dW must be NULL.
 *  compute_db   (LayerNorm) nonzero: write db [H] = sum of dY over rows.
 *  accum_fp32   nonzero: dW / db are fp32, else `dtype`.
 *  dX           device [rows, H], `dtype` (overwritten).
 *  workspace    device, flkl_norm_workspace_size(...) bytes, 256-byte aligned
 *               (may be NULL when that size is 0, i.e. both flags are 0).
 *  Pointers 16-byte aligned (else FLKL_ERR_UNSUPPORTED).  Asynchronous on
 *  `stream`; host-side errors as flkl_forward_backward.  A device-side wait
 *  that gives up (flkl_set_wait_limit_ms) leaves dX undefined and is reported
 *  by flkl_norm_device_status.  Deterministic on a given device: dW and db
 *  are summed in a fixed order (per-CTA partial rows, then in CTA order).
 *  The workspace holds one fp32 partial row of H per CTA and per gradient
 *  asked for; its size depends on the current device's SM count. */
FLKL_API size_t flkl_norm_workspace_size(int64_t rows, int64_t H, int compute_dW,
                                         int compute_db);
FLKL_API flkl_status flkl_rms_norm_backward(const void* dY, const void* X, const void* W,
                                            int64_t rows, int64_t H, int dtype, float eps,
                                            int compute_dW, int accum_fp32, void* dX, void* dW,
                                            void* workspace, size_t workspace_bytes,
                                            void* stream);
FLKL_API flkl_status flkl_layer_norm_backward(const void* dY, const void* X, const void* W,
                                              int64_t rows, int64_t H, int dtype, float eps,
                                              int compute_dW, int compute_db, int accum_fp32,
                                              void* dX, void* dW, void* db, void* workspace,
                                              size_t workspace_bytes, void* stream);
/* Synchronises `stream` and returns the status word of the norm-backward
 * kernels of the current device (FLKL_OK, or FLKL_ERR_TIMEOUT when one of
 * their waits gave up since the last call), then clears it. */
FLKL_API flkl_status flkl_norm_device_status(void* stream);

/* Synchronises `stream`, then returns the device status recorded by the last
 * flkl_forward_backward call that used `workspace` (FLKL_OK or
 * FLKL_ERR_TIMEOUT), or FLKL_ERR_CUDA if the copy or the synchronisation
 * fails. */
FLKL_API flkl_status flkl_device_status(const void* workspace, void* stream);

/* Upper bound, in milliseconds, of every wait inside the kernels (default
 * 4000).  After it a kernel records FLKL_ERR_TIMEOUT, drains its own copies,
 * frees its tensor memory and returns.  Applies to later launches of this
 * process; 0 restores the default. */
FLKL_API void flkl_set_wait_limit_ms(unsigned int ms);

/* Self-check of the bounded wait: launches one block that waits on an
 * mbarrier which nothing ever completes, with a limit of `limit_ms`, and
 * writes the resulting status code (FLKL_ERR_TIMEOUT expected) to the device
 * int *status_out.  Touches no other memory. */
FLKL_API flkl_status flkl_wait_selftest(int* status_out, unsigned int limit_ms, void* stream);

/* Measurement helper (not part of the loss): one thread samples the SM
 * clock counter and the global nanosecond timer every interval_ns,
 * n_samples times, writing (globaltimer, clock64) pairs to out[2i],
 * out[2i+1] (device uint64 [2 * n_samples]).  Launched on `stream`, usually
 * a side stream next to the kernels whose SM clock is wanted; it holds one
 * thread of one SM for n_samples * interval_ns and ends by itself.
 * n_samples in [1, 2^24], interval_ns in [1000, 10^8]. */
FLKL_API flkl_status flkl_clock_trace(uint64_t* out, int n_samples, unsigned int interval_ns,
                                      void* stream);

/* SMs (CTAs, one per SM) that every GEMM launch of the library's tensor-core
 * kernel occupies on the current device: as many CTA pairs (clusters of two)
 * as are resident at once, times two; 0 without a usable device. */
FLKL_API int flkl_gemm_ctas(void);

/* Static text for a status code. */
FLKL_API const char* flkl_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* FLKL_H_ */
