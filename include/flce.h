/*
 * flce.h -- exact fused linear cross-entropy on NVIDIA B200 (sm_100a), C ABI.
 *
 * The operation is the one stated in "分块交叉熵 / Output projection / exact
 * cross entropy" (glenzli.com), §01 equation:
 *
 *   Z_ij = H_i W_j^T + b_j                       (never stored: tiles live on chip)
 *   a_i  = 1[mask_i] * 1[y_i != ignore_index],   C = sum_i a_i
 *   L    = (1/C) sum_{i: a_i=1} ( (m_i - Z_{i,y_i}) + log s_i )       (§02)
 *
 * with m_i = max_j Z_ij and s_i = sum_j exp(Z_ij - m_i) over the full
 * vocabulary (the running statistics of §02), and the gradients of §04:
 *
 *   p_ij = exp((Z_ij - m_i) - log s_i)
 *   G_ij = (lambda a_i / C) (p_ij - 1[j = y_i])
 *   dH = G W,   dW = G^T H,   db = sum_i G_i
 *
 * C = 0 gives the zero sentinel loss and zero gradients (§01).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All arrays are DEVICE pointers, dense, row-major, owned by the caller.
 *    The library never allocates, frees or writes its inputs.  It never
 *    synchronises the stream, except in flce_device_status().
 *  - 16-bit tensors (H, W, b) are bf16 or fp16 per `dtype`; both operands of
 *    one call have the same type.  H and W must be 16-byte aligned and D a
 *    multiple of 8 (rows of 16-byte multiples, needed by the TMA engine).
 *  - labels are int64 [N]; mask is uint8 [N] (nonzero = position takes part)
 *    or NULL (all positions take part).  Arrays with N entries (H, labels,
 *    m, logs, dH, idx) may be NULL when N == 0.
 *  - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and runs asynchronously.  Argument errors are returned before
 *    anything is enqueued.  Errors found on the device (a supervised label
 *    outside [0, V), a pipeline wait that ran past its time limit, a
 *    non-finite statistic) are recorded in an error word inside the
 *    workspace, make the loss NaN, and are reported by flce_device_status().
 *  - The workspace is caller-allocated device memory of at least
 *    flce_workspace_bytes(N, D, V, dtype) bytes, 256-byte aligned (the
 *    forward alone uses only its leading part and accepts a shorter buffer;
 *    the size returned is always enough).  Calls are stateless: the
 *    workspace carries nothing from one call to the next, but two calls in
 *    flight at the same time must not share one workspace.
 *  - Only the current CUDA device is used; it must be compute capability
 *    10.0 (sm_100a).
 */
#ifndef FLCE_H_
#define FLCE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define FLCE_API __attribute__((visibility("default")))
#else
#define FLCE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FLCE_OK = 0,
  FLCE_ERR_NULL = 1,        /* a required pointer is NULL                        */
  FLCE_ERR_SHAPE = 2,       /* N, D or V out of range                            */
  FLCE_ERR_DTYPE = 3,       /* dtype is not FLCE_BF16 / FLCE_FP16                */
  FLCE_ERR_ALIGN = 4,       /* pointer or D not aligned as required              */
  FLCE_ERR_WORKSPACE = 5,   /* workspace smaller than flce_workspace_bytes()     */
  FLCE_ERR_CUDA = 6,        /* a CUDA runtime call failed                        */
  FLCE_ERR_LABEL = 7,       /* device: a supervised label is outside [0, V)      */
  FLCE_ERR_TIMEOUT = 8,     /* device: a pipeline wait ran past its time limit   */
  FLCE_ERR_NONFINITE = 9,   /* device: a non-finite per-row statistic            */
  FLCE_ERR_DEVICE = 10,     /* current device is not sm_100 / cannot run kernels */
  FLCE_ERR_ARG = 11,        /* an argument value is invalid (e.g. the reduction) */
  FLCE_ERR_SHARD = 12       /* device: a supervised label is held by no
                               vocabulary slice, or by several (shard combine) */
} flce_status;

typedef enum { FLCE_BF16 = 0, FLCE_FP16 = 1 } flce_dtype;

/* A cudaStream_t, passed without the CUDA headers. */
typedef void* flce_stream;

/* Bytes of device workspace needed for problem size (N, D, V).  Returns 0
 * when the sizes are out of range (same limits as FLCE_ERR_SHAPE).  For
 * D <= 64 it includes the single-kernel backward's partial sums (see
 * flce_backward): (8 * V + 160 * N) * D * 4 bytes, rounded up, in the space
 * the panel form's buffers take otherwise. */
FLCE_API size_t flce_workspace_bytes(int64_t N, int64_t D, int64_t V, int dtype);

/*
 * Supervised-row compaction (a_i and C of §01; "filter: keep only labels !=
 * -100" of "ChunkedLinearCrossEntropy (Qwen3.5 training memory peak)").
 *
 * Writes idx[0..C) = the supervised rows in ascending order (int32, device,
 * capacity N) and *C_out (int32, device).  Labels of supervised rows outside
 * [0, V) set FLCE_ERR_LABEL in the workspace error word.
 */
FLCE_API flce_status flce_compact(const int64_t* labels, const uint8_t* mask, int64_t ignore_index,
                         int64_t N, int64_t V, int32_t* idx, int32_t* C_out,
                         void* ws, size_t ws_bytes, flce_stream stream);

/*
 * Forward (§01 objective, §02 running statistics).
 *
 *   H [N x D], W [V x D], b [V] or NULL (absent bias means b = 0)
 *   loss  : device float scalar, the mean over the C supervised rows; 0 when C = 0
 *   m     : device float [N], per-row max logit; -inf for unsupervised rows
 *   logs  : device float [N], per-row log s;     -inf for unsupervised rows
 *
 * m and logs are the saved statistics that flce_backward() consumes.
 */
FLCE_API flce_status flce_forward(const void* H, const void* W, const void* b,
                         const int64_t* labels, const uint8_t* mask, int64_t ignore_index,
                         int64_t N, int64_t D, int64_t V, int dtype,
                         float* loss, float* m, float* logs,
                         void* ws, size_t ws_bytes, flce_stream stream);

/*
 * Backward (§04 reconstruction and accumulation).
 *
 *   m, logs   : the statistics written by flce_forward() for the same inputs
 *   lambda    : upstream gradient dJ/dL (host float), used when lambda_dev is NULL
 *   lambda_dev: optional device float scalar holding lambda (lets an autograd
 *               caller pass its gradient without a host round trip)
 *   dH [N x D], dW [V x D] : float32 outputs, fully overwritten; rows of dH
 *               for unsupervised positions are zero
 *   db [V]    : float32 output, required iff b is not NULL
 *
 * dH, dW and db are deterministic: every output element is reduced in a
 * fixed order independent of scheduling.
 *
 * Two forms of the same computation.  D > 64 (or FLCE_FLAG_PANEL_BACKWARD):
 * the gradient of the logits is staged in 16 bits, one vocabulary panel of
 * 8192 ids at a time, and read by the dW and dH contractions.  D <= 64: one
 * kernel per call does the score tile, the gradient and both contractions
 * per 256-row x 128-id tile (§04's single fused pass: dH of the row block
 * accumulates across the vocabulary on chip; dW is added up per group of
 * row blocks in row-block order, and the groups' sums by a second kernel in
 * a fixed order).
 */
FLCE_API flce_status flce_backward(const void* H, const void* W, const void* b,
                          const int64_t* labels, const uint8_t* mask, int64_t ignore_index,
                          int64_t N, int64_t D, int64_t V, int dtype,
                          const float* m, const float* logs,
                          float lambda, const float* lambda_dev,
                          float* dH, float* dW, float* db,
                          void* ws, size_t ws_bytes, flce_stream stream);

/* Bytes of the fixed scratch buffer that flce_forward_noalloc() uses. */
#define FLCE_NOALLOC_SCRATCH_BYTES (32u << 20)

/*
 * Forward that needs no workspace from the caller and allocates nothing.
 * The pages have no counterpart of this entry point; it exists for callers.
 *
 * Some callers cannot provide device scratch memory: a plug-in running inside
 * a host framework that owns every device allocation and allows no
 * cudaMalloc outside its own pool, or code on a latency-critical path where
 * cudaMalloc (which can synchronise the whole device) is not acceptable.
 * This call computes the same loss, m and logs as flce_forward(), with its
 * scratch in a FLCE_NOALLOC_SCRATCH_BYTES buffer compiled into the library
 * (a static device array: every GPU that loads libflce.so holds it until the
 * process exits).  It calls no cudaMalloc, cudaFree or other allocating
 * routine.  The caller still passes all inputs and outputs.
 *
 *  - Size limit: the forward's scratch, about (N rounded up to 256) x
 *    (2 D + 8 ceil(V / 256) + 20) bytes, must fit in FLCE_NOALLOC_SCRATCH_BYTES
 *    (the small workload, N=2048 D=512 V=32000, needs about 4 MiB; the
 *    16k-row, 248320-vocabulary case needs about 154 MiB and does not fit);
 *    larger problems get FLCE_ERR_WORKSPACE before anything is enqueued.
 *  - Every call looks up the buffer's device address on the current device
 *    (cudaGetSymbolAddress, which allocates nothing; no address is kept
 *    between calls, so a reset of the device's primary context, which loads
 *    the library's module and the buffer again, cannot leave a stale one).
 *    The first call on a device also loads the kernels there: make that
 *    first call before any stream capture.
 *  - All calls on a device share the one buffer, which keeps the previous
 *    call's contents; the call clears what has to start at zero.  Calls that
 *    overlap on the GPU (different streams or host threads) race on the
 *    buffer and must be serialised by the caller.
 *  - A device-side error (bad label, wait timeout) shows up as a NaN loss;
 *    the error word lives in the shared buffer and is not returned.
 */
FLCE_API flce_status flce_forward_noalloc(const void* H, const void* W, const void* b,
                                          const int64_t* labels, const uint8_t* mask,
                                          int64_t ignore_index, int64_t N, int64_t D, int64_t V,
                                          int dtype, float* loss, float* m, float* logs,
                                          flce_stream stream);

/*
 * Reductions of the per-row losses l_i = (m_i - Z_{i,y_i}) + log s_i, with
 * optional per-row weights w_i (1 when `weight` is NULL).  MEAN is the
 * objective of the page's §01; SUM and NONE are the reductions of NeMo's
 * ChunkedCrossEntropy ("reduction", "num_label_tokens", "loss_weights"):
 *   FLCE_REDUCE_MEAN  L = (1/C) sum_i w_i l_i
 *   FLCE_REDUCE_SUM   L = (1/denom) sum_i w_i l_i   (denom <= 0 means 1)
 *   FLCE_REDUCE_NONE  loss_rows[i] = w_i l_i, 0 for unsupervised rows
 */
typedef enum { FLCE_REDUCE_MEAN = 0, FLCE_REDUCE_SUM = 1, FLCE_REDUCE_NONE = 2 } flce_reduction;

/* Option bits of the _ex calls.
 * FLCE_FLAG_ROUND_LOGITS: each logit (after the bias) is rounded from fp32 to
 *   the input dtype before the loss, as a projection that outputs the model
 *   dtype does (NeMo "logits_dtype"; the bf16 logits of the
 *   ChunkedLinearCrossEntropy article).  The backward treats the rounding as
 *   the identity.  Pass the same flags to the forward and the backward. */
#define FLCE_FLAG_ROUND_LOGITS 1u
/* FLCE_FLAG_ACCUMULATE_DH (backward calls only): dH += this call's dH instead
 *   of dH = this call's dH (rows of unsupervised positions are left as they
 *   are).  With it the dH terms of several vocabulary slices, or of several
 *   losses on one hidden state, sum in place. */
#define FLCE_FLAG_ACCUMULATE_DH 2u
/* FLCE_FLAG_REUSE_FORWARD (backward calls only): the workspace still holds
 *   what a forward call (flce_forward, flce_forward_ex or flce_shard_forward)
 *   left there for the same H, labels, mask, ignore_index, N, D and V (the
 *   supervised-row list, C, the gathered rows H_c and the row map), and
 *   nothing has written to the workspace since: the backward skips the
 *   compaction and the gather and uses them.  The caller guarantees that
 *   H, labels and mask did not change in between; the result is undefined
 *   otherwise.  A device error recorded by that forward stays recorded. */
#define FLCE_FLAG_REUSE_FORWARD 4u
/* FLCE_FLAG_PANEL_BACKWARD (backward calls only): use the panel form of the
 *   backward where the single-kernel form would apply (D <= 64); the results
 *   agree within rounding (see flce_backward).  Gradient filtering always
 *   uses the panel form. */
#define FLCE_FLAG_PANEL_BACKWARD 8u

/*
 * Forward with a reduction.  weight: device float [N] or NULL.  loss: device
 * scalar, required for MEAN and SUM (ignored for NONE); loss_rows: device
 * float [N], required for NONE (ignored otherwise).  m and logs as in
 * flce_forward().  flags: FLCE_FLAG_* bits (0 for none).  flce_forward() is
 * this call with weight NULL, MEAN and no flags.
 */
FLCE_API flce_status flce_forward_ex(const void* H, const void* W, const void* b,
                                     const int64_t* labels, const uint8_t* mask,
                                     int64_t ignore_index, int64_t N, int64_t D, int64_t V,
                                     int dtype, const float* weight, int reduction, float denom,
                                     unsigned flags, float* loss, float* loss_rows, float* m,
                                     float* logs,
                                     void* ws, size_t ws_bytes, flce_stream stream);

/*
 * Backward of flce_forward_ex() (§04 with G_ij = s_i (p_ij - 1[j = y_i])):
 *   MEAN  s_i = lambda w_i / C        SUM  s_i = lambda w_i / denom
 *   NONE  s_i = grad_rows[i] w_i      (grad_rows: device float [N], the
 *                                      upstream gradient of each row's loss)
 * lambda / lambda_dev as in flce_backward() (unused for NONE).
 * flags as given to the forward.  flce_backward() is this call with weight
 * NULL, MEAN and no flags.
 */
FLCE_API flce_status flce_backward_ex(const void* H, const void* W, const void* b,
                                      const int64_t* labels, const uint8_t* mask,
                                      int64_t ignore_index, int64_t N, int64_t D, int64_t V,
                                      int dtype, const float* m, const float* logs,
                                      const float* weight, int reduction, float denom,
                                      unsigned flags, float lambda, const float* lambda_dev,
                                      const float* grad_rows, float* dH, float* dW, float* db,
                                      void* ws, size_t ws_bytes, flce_stream stream);

/*
 * Backward with opt-in gradient filtering, an approximation: the
 * "分块交叉熵 / Output projection / exact cross entropy" page (§07, on Apple's
 * Cut Cross-Entropy) describes skipping the blocks of the softmax whose
 * probabilities are all negligible in the backward contractions.  Here a
 * block is 128 consecutive supervised rows (ascending row order) by 64
 * consecutive vocabulary ids, aligned to multiples of 128 and 64; a block
 * whose every |p_ij - 1[j = y_i]| is below filter_eps contributes nothing to
 * dH and dW (the dW / dH contractions skip it), while db keeps every entry.
 * The test is made in fp32 on the kernel's p.  filter_eps = 0 is the exact
 * backward, identical to flce_backward_ex(); filter_eps < 0 or not finite:
 * FLCE_ERR_ARG.  Every other argument as in flce_backward_ex().  The result is
 * reported against the exact oracle in the tests; how far it departs from the
 * exact gradient depends on the inputs (for logits with a few dominant
 * entries per row, little; for flat logits, p ~ 1 / V everywhere, it drops
 * almost everything off the target entries).
 */
FLCE_API flce_status flce_backward_filtered(const void* H, const void* W, const void* b,
                                            const int64_t* labels, const uint8_t* mask,
                                            int64_t ignore_index, int64_t N, int64_t D,
                                            int64_t V, int dtype, const float* m,
                                            const float* logs, const float* weight,
                                            int reduction, float denom, unsigned flags,
                                            float lambda, const float* lambda_dev,
                                            const float* grad_rows, float filter_eps, float* dH,
                                            float* dW, float* db, void* ws, size_t ws_bytes,
                                            flce_stream stream);

/*
 * Vocabulary-sharded (tensor-parallel over V) form.
 *
 * The vocabulary [0, V_total) is cut into disjoint slices; the caller that
 * holds the slice [v0, v0 + V_slice) passes W_slice = rows v0 .. v0+V_slice-1
 * of W ([V_slice x D]) and the same slice of b.  Labels stay global ids in
 * [0, V_total).  One step is:
 *
 *   1. flce_shard_forward on every slice   -> stats_r [N] (float4 per row)
 *   2. exchange: every caller obtains all slices' stats, stacked [P x N]
 *      (an all-gather of P x N x 16 bytes)
 *   3. flce_shard_combine                  -> loss, m, logs (full vocabulary)
 *   4. flce_shard_backward on every slice  -> dW_slice, db_slice, dH_r
 *   5. exchange: dH = sum_r dH_r (an all-reduce of N x D floats)
 *
 * The merge in step 3 is the two-state online-softmax merge ("数学基础"
 * maths-basics page, worked example 9.4, and "分块交叉熵" §02), exact in the
 * reals for any partition of the vocabulary; the need for a cross-device
 * aggregation when the vocabulary is tensor-parallel is the maths-basics
 * page's §5.9 remark.  With the merged statistics each slice forms its own
 * columns of G (§04), so step 4 needs nothing from the other slices.  The
 * library does no communication: steps 2 and 5 are the caller's (e.g. NCCL).
 */

/*
 * Per-row partial statistics of one slice.
 *   stats : device float4 [N] (16-byte aligned), per row
 *           (m_r, log s_r, t_r, o_r) = the slice's max logit, the log of its
 *           sum of exp(Z - m_r), the target logit when the slice holds the
 *           label (else 0) and the ownership flag 1[v0 <= y < v0 + V_slice].
 *           Unsupervised rows get (-inf, -inf, 0, 0).
 *   0 <= v0, v0 + V_slice <= V_total <= the V limit; labels are checked
 *   against V_total (FLCE_ERR_LABEL).  Workspace: flce_workspace_bytes(N, D,
 *   V_slice, dtype).  flags: FLCE_FLAG_* as in flce_forward_ex().
 */
FLCE_API flce_status flce_shard_forward(const void* H, const void* W_slice, const void* b_slice,
                                        const int64_t* labels, const uint8_t* mask,
                                        int64_t ignore_index, int64_t N, int64_t D,
                                        int64_t V_slice, int64_t v0, int64_t V_total, int dtype,
                                        unsigned flags, float* stats, void* ws, size_t ws_bytes,
                                        flce_stream stream);

/* Bytes of device workspace flce_shard_combine() needs for N rows. */
FLCE_API size_t flce_shard_combine_workspace_bytes(int64_t N);

/*
 * Merge of P slices' statistics into the full-vocabulary result.
 *   stats_all : device float4 [P x N] (16-byte aligned), slice r's stats at
 *               rows r*N .. r*N+N-1, slices in any order
 *   labels, mask, ignore_index : as given to flce_shard_forward (same on
 *               every slice); weight, reduction, denom, loss, loss_rows as in
 *               flce_forward_ex(); m, logs : device float [N], the merged
 *               statistics that flce_shard_backward() consumes.
 * A supervised row held by no slice or by several records FLCE_ERR_SHARD
 * (loss NaN).  Workspace: flce_shard_combine_workspace_bytes(N).
 */
FLCE_API flce_status flce_shard_combine(const float* stats_all, int P, const int64_t* labels,
                                        const uint8_t* mask, int64_t ignore_index, int64_t N,
                                        const float* weight, int reduction, float denom,
                                        float* loss, float* loss_rows, float* m, float* logs,
                                        void* ws, size_t ws_bytes, flce_stream stream);

/*
 * This slice's share of the backward: with the merged m and logs from
 * flce_shard_combine(), dW_slice [V_slice x D] and db_slice [V_slice] (iff
 * b_slice) are the slice's rows of dW and db, and dH [N x D] is this slice's
 * term G_r W_slice of dH = sum_r G_r W_r (float32, fully overwritten; the
 * caller sums the slices' dH).  Other arguments as in flce_backward_ex() and
 * flce_shard_forward().  Workspace: flce_workspace_bytes(N, D, V_slice, dtype).
 */
FLCE_API flce_status flce_shard_backward(const void* H, const void* W_slice,
                                         const void* b_slice, const int64_t* labels,
                                         const uint8_t* mask, int64_t ignore_index, int64_t N,
                                         int64_t D, int64_t V_slice, int64_t v0, int64_t V_total,
                                         int dtype, const float* m, const float* logs,
                                         const float* weight, int reduction, float denom,
                                         unsigned flags, float lambda, const float* lambda_dev,
                                         const float* grad_rows, float* dH, float* dW_slice,
                                         float* db_slice, void* ws, size_t ws_bytes,
                                         flce_stream stream);

/* Synchronises `stream`, then reads and returns the device error word of the
 * workspace (FLCE_OK when no device error was recorded by the last call). */
FLCE_API flce_status flce_device_status(const void* ws, flce_stream stream);

/* Static, human-readable name of a status code. */
FLCE_API const char* flce_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* FLCE_H_ */
