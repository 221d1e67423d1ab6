/*
 * flce.h -- C ABI of the B200 (sm_100a) fused linear cross-entropy library.
 *
 * The operation is the language-model-head loss that PyTorch PR #126348
 * ("[AOTAutograd] tweak min-cut partitioner to avoid saving softmax output")
 * describes as four steps -- a matmul producing softmax_input, a row max, a
 * row sum, and a normalised softmax_output -- fused so that neither the
 * logits nor the softmax is ever stored in full:
 *
 *   z      = X W^T                  X: BT x H hidden states, W: V x H weight
 *                                   of a bias-free nn.Linear(H, V) (the PR's
 *                                   test fragment: nn.Linear(C, V, bias=False))
 *   y      = c tanh(z / c)          optional Gemma2 logit softcap c (Liger-Kernel
 *                                   issue #227, "Gemma2 softcap logits")
 *   lse_i  = log sum_j exp(y_ij)    steps 2-3 of the PR summary
 *   loss   = mean over rows with label_i != ignore_index of (lse_i - y_i,label_i)
 *                                   (the loss_fn(logits, labels) call of torchtune
 *                                   issue #1228)
 *   G      = (softmax(y) - onehot(label)) * dy/dz * dloss / N_valid, rows with
 *            ignored labels zero; the softmax is recomputed from X, W and the
 *            saved lse (PR #126348, point b: the softmax is rebuilt, not saved),
 *            or, in flce_fused for BT >= 512, rebuilt from the bf16
 *            exp(y - m) the forward kept for one chunk of rows at a time
 *   dX     = G W,    dW = G^T X
 *
 * N_valid is the number of rows whose label is not ignore_index.  When every
 * row is ignored the loss is 0 and dX, dW are 0.
 *
 * Conventions for every entry point:
 *   - All array arguments are DEVICE pointers (memory the caller allocated on
 *     the current CUDA device), row-major: X is BT x H with row stride ldx
 *     elements, W is V x H with row stride ldw, dX is BT x H with row stride
 *     lddx, dW is V x H with row stride lddw (each 0 = H, dense).  A stride
 *     lets X be a slice of a wider activation (hidden[:, a:a+H]), W a slice
 *     of a padded or tied weight, and the gradients land inside wider
 *     buffers, with no copy.  Every row must start on a 16-byte boundary:
 *     X, W, dX and dW 16-byte aligned and each stride times the element size
 *     a multiple of 16 (else FLCE_ERR_MISALIGNED); a stride below H is
 *     FLCE_ERR_INVALID_ARG.  labels is dense, 8-byte aligned.
 *     labels is int64 [BT]: per-row labels, or token ids that the op shifts
 *     itself when flce_problem_t.shift_seq_len > 0.
 *   - Element type: FLCE_BF16 (bfloat16 X/W/dX/dW, fp32 accumulation, the
 *     tensor-core path) or FLCE_FP32 (fp32 throughout, CUDA-core path).
 *     loss and lse are always fp32.
 *   - H must be a multiple of 8 (each row a whole number of 16-byte units).
 *   - The library allocates nothing.  Scratch space is the caller's
 *     workspace `ws` of at least flce_workspace_size() bytes, 256-byte
 *     aligned.  Outputs (loss, lse, dX, dW) are overwritten, never
 *     accumulated into.
 *   - All work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and the calls return without waiting for it.  Calls that run
 *     concurrently must use different workspaces.
 *   - Errors found on the host (bad sizes, NULL or misaligned pointers, a
 *     workspace that is too small, unsupported dtype) are returned before
 *     anything is enqueued.  Errors found on the device (a label outside
 *     [0, V) that is not ignore_index, a pipeline wait that timed out) are
 *     recorded in the workspace's status word; the remaining kernels of the
 *     call then skip their work and the outputs are unspecified.  Read it
 *     with flce_get_device_status().  No kernel traps or asserts.
 */
#ifndef FLCE_H_
#define FLCE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t is struct CUstream_st* */
struct CUevent_st;  /* cudaEvent_t is struct CUevent_st* */

#if defined(__GNUC__)
#define FLCE_API __attribute__((visibility("default")))
#else
#define FLCE_API
#endif

typedef enum {
  FLCE_OK = 0,
  FLCE_ERR_INVALID_ARG = 1,        /* negative/zero size, NULL pointer, bad op */
  FLCE_ERR_UNSUPPORTED = 2,        /* dtype or size the library does not handle */
  FLCE_ERR_MISALIGNED = 3,         /* pointer alignment or H % 8 != 0 */
  FLCE_ERR_WORKSPACE_TOO_SMALL = 4,
  FLCE_ERR_LABEL_OUT_OF_RANGE = 5, /* device-detected: label not in [0,V), not ignored */
  FLCE_ERR_TIMEOUT = 6,            /* device-detected: a pipeline wait gave up */
  FLCE_ERR_CUDA = 7                /* a CUDA runtime/driver call failed */
} flce_status_t;

typedef enum { FLCE_BF16 = 0, FLCE_FP32 = 1 } flce_dtype_t;

typedef enum { FLCE_OP_FORWARD = 0, FLCE_OP_BACKWARD = 1, FLCE_OP_FUSED = 2 } flce_op_t;

/* Problem description.  softcap <= 0, NaN or +inf means "no softcap".
 * Size limits (else FLCE_ERR_UNSUPPORTED): BT, H, V < 2^31; strides < 2^31;
 * ceil(BT/128) * ceil(V/256) < 2^28 (32-bit tile ids); fp32 problems
 * BT <= 65535 * 32. */
typedef struct {
  int64_t BT;           /* rows (batch x sequence), >= 0 */
  int64_t H;            /* hidden size, > 0, multiple of 8 */
  int64_t V;            /* vocabulary size, > 0 */
  int32_t dtype;        /* flce_dtype_t */
  int32_t shift_seq_len; /* 0, or T > 0: labels holds token ids of B = BT/T
                           sequences of T positions, and position t of a
                           sequence is scored against id t+1 (its last
                           position is ignored); BT must be a multiple of T */
  int64_t ignore_index; /* label value that marks a row as ignored (e.g. -100) */
  float softcap;        /* Gemma2-style logit cap c, or <= 0 for none */
  int32_t dw_fp32;      /* 0: dW has X's element type; 1: dW is fp32 (V x H
                           float, row stride lddw) whatever X's type, for a
                           gradient kept, or summed over ranks, in fp32.  With
                           bf16 inputs the fused-in-forward schedule then keeps
                           its running sum of dW in dW itself instead of the
                           workspace.  Other values: FLCE_ERR_INVALID_ARG */
  int64_t ldx;          /* row stride of X in elements; 0 = H */
  int64_t ldw;          /* row stride of W in elements; 0 = H */
  int64_t lddx;         /* row stride of dX in elements; 0 = H */
  int64_t lddw;         /* row stride of dW in elements; 0 = H */
} flce_problem_t;

/* Bytes of workspace `op` (flce_op_t) needs for problem `p`, or 0 when `p`
 * is invalid.  Never allocates; callable without a GPU. */
FLCE_API size_t flce_workspace_size(const flce_problem_t* p, int op);

/* Forward: loss (device fp32 scalar) and lse (device fp32 [BT], the per-row
 * log-sum-exp that flce_backward needs).  Steps 1-3 of the PR #126348
 * summary with the target-logit gather in place of step 4 (the PR's point
 * a: the NLL needs one entry of each softmax row, not the whole tensor). */
FLCE_API flce_status_t flce_forward(const flce_problem_t* p, const void* X, const void* W,
                           const int64_t* labels, float* loss, float* lse, void* ws,
                           size_t ws_bytes, struct CUstream_st* stream);

/* Backward: dX and dW from the saved lse and the upstream gradient dloss
 * (device fp32 scalar; a training loop that divides the loss by its
 * gradient-accumulation count passes that factor here).  Recomputes the
 * logits tile by tile instead of reading a saved softmax (PR #126348, b.). */
FLCE_API flce_status_t flce_backward(const flce_problem_t* p, const void* X, const void* W,
                            const int64_t* labels, const float* lse, const float* dloss,
                            void* dX, void* dW, void* ws, size_t ws_bytes,
                            struct CUstream_st* stream);

/* Forward and backward in one call, dloss given by value (1.0 for a plain
 * loss.backward()).  Writes loss (device fp32 scalar), dX and dW; the lse
 * lives in the workspace. */
FLCE_API flce_status_t flce_fused(const flce_problem_t* p, const void* X, const void* W,
                         const int64_t* labels, float dloss, float* loss, void* dX, void* dW,
                         void* ws, size_t ws_bytes, struct CUstream_st* stream);

/* Data parallelism over rows (each rank holds its own rows of X and labels
 * and the same W).  The pages train with a mean loss over the batch (torchtune
 * issue #1228: loss_fn(logits, labels) then loss / grad-accumulation steps);
 * split over ranks, that mean needs the count of non-ignored labels of all
 * ranks before any G is formed, and dW is the sum of every rank's G^T X.
 *
 * flce_count_valid: *n_valid (device int64) = number of rows of problem p
 * whose label (after the shift when p->shift_seq_len > 0) is not
 * p->ignore_index (out-of-range labels are counted; the loss call reports
 * them).  labels and n_valid 8-byte aligned device pointers.  The caller
 * then sums n_valid over its ranks (e.g. an NCCL all-reduce).
 *
 * flce_fused_global: flce_fused with the mean's divisor read from
 * *n_valid_global (device int64, the all-rank count) instead of this call's
 * own count.  loss = this rank's sum of NLL / N_global (its share of the
 * global mean: the ranks' losses sum to it); dX = this rank's rows of the
 * global-mean gradient; dW = this rank's G^T X, to be summed over ranks by
 * the caller.  N_global = 0 gives loss 0 and zero gradients.
 * flce_get_device_status then reports N_global.  Same workspace as
 * flce_fused; the same errors, plus FLCE_ERR_INVALID_ARG for a NULL
 * n_valid_global.  The pages describe no counterpart of these two calls;
 * they exist for running one rank per GPU. */
FLCE_API flce_status_t flce_count_valid(const flce_problem_t* p, const int64_t* labels,
                                        int64_t* n_valid, struct CUstream_st* stream);
FLCE_API flce_status_t flce_fused_global(const flce_problem_t* p, const void* X, const void* W,
                                         const int64_t* labels, const int64_t* n_valid_global,
                                         float dloss, float* loss, void* dX, void* dW, void* ws,
                                         size_t ws_bytes, struct CUstream_st* stream);

/* flce_fused_global_sliced: flce_fused_global (or flce_fused, when
 * n_valid_global is NULL) that hands dW over in n_slices vocabulary slices,
 * so the caller can start reducing dW over its ranks (torchtune issue #1228's
 * data-parallel recipes: an all-reduce, or a reduce-scatter under FSDP)
 * while the rest of dW is still being computed.  Slice s is rows
 * [s * r, min(V, (s + 1) * r)) of dW, r = flce_dw_slice_rows(V, n_slices)
 * (a multiple of 256; trailing slices may be empty).  slice_done[s] is a
 * caller-created CUDA event (no timing needed); the call records it on
 * `stream` once slice s of dW holds its final values, and writes nothing to
 * those rows afterwards.  With the fused-in-forward schedule the last row
 * chunk's dW GEMM runs slice by slice, each event recorded as its slice's
 * launch ends; with the recompute schedule every event is recorded after
 * the last launch.  1 <= n_slices <= 64, every event non-NULL (else
 * FLCE_ERR_INVALID_ARG); otherwise as flce_fused_global. */
FLCE_API flce_status_t flce_fused_global_sliced(const flce_problem_t* p, const void* X,
                                                const void* W, const int64_t* labels,
                                                const int64_t* n_valid_global, float dloss,
                                                float* loss, void* dX, void* dW, void* ws,
                                                size_t ws_bytes, int32_t n_slices,
                                                struct CUevent_st* const* slice_done,
                                                struct CUstream_st* stream);
/* Rows of dW per slice for flce_fused_global_sliced (0 when V <= 0 or
 * n_slices is outside [1, 64]). */
FLCE_API int64_t flce_dw_slice_rows(int64_t V, int32_t n_slices);

/* Vocabulary parallelism: W split over the vocabulary across ranks, rank r
 * holding rows [v_offset, v_offset + p->V) of a V_total-row W and all of X
 * and the labels (global vocabulary ids).  The mean loss needs, per row, the
 * log-sum-exp over the whole vocabulary, so each rank reduces its slice to
 * three numbers per row, the ranks exchange them, and the backward then
 * needs only the global lse: dX is a sum over the ranks' slices, dW stays
 * with its rank.  The pages' distributed setting is data parallel (torchtune
 * issue #1228's FSDP recipes); this is the other split the loss allows.
 *
 * flce_vp_forward: stats (device fp32 [BT][3]) = per row, over this rank's
 *   slice, the largest y log2(e), the sum of exp2(y log2(e) - that), and y at
 *   the label when the label lies in the slice (else 0).  Labels are checked
 *   against [0, v_total).  Workspace: flce_vp_workspace_size(p,
 *   FLCE_OP_FORWARD).
 * flce_vp_combine: with p->V = v_total, stats_all (device fp32
 *   [n_ranks][BT][3], the ranks' stats in rank order) -> lse (device fp32
 *   [BT]) and loss (device fp32 scalar, the mean over non-ignored rows),
 *   combined in rank order (identical on every rank).  Workspace: any
 *   forward workspace of this BT (>= 256 + 2 * ceil256(4 * BT) bytes).
 * flce_vp_backward: dX (device fp32, BT x H, row stride p->lddx or H; this
 *   rank's share, to be summed over the ranks) and dW (this rank's V rows,
 *   as in flce_backward) from the global lse and dloss (device fp32 scalar).
 *   Workspace: flce_vp_workspace_size(p, FLCE_OP_BACKWARD).
 * p->shift_seq_len must be 0 (FLCE_ERR_UNSUPPORTED otherwise); v_offset < 0
 * or v_offset + p->V > v_total: FLCE_ERR_INVALID_ARG. */
FLCE_API size_t flce_vp_workspace_size(const flce_problem_t* p, int op);
FLCE_API flce_status_t flce_vp_forward(const flce_problem_t* p, int64_t v_offset,
                                       int64_t v_total, const void* X, const void* W,
                                       const int64_t* labels, float* stats, void* ws,
                                       size_t ws_bytes, struct CUstream_st* stream);
FLCE_API flce_status_t flce_vp_combine(const flce_problem_t* p, int32_t n_ranks,
                                       const float* stats_all, const int64_t* labels,
                                       float* loss, float* lse, void* ws, size_t ws_bytes,
                                       struct CUstream_st* stream);
FLCE_API flce_status_t flce_vp_backward(const flce_problem_t* p, int64_t v_offset,
                                        int64_t v_total, const void* X, const void* W,
                                        const int64_t* labels, const float* lse,
                                        const float* dloss, float* dX, void* dW, void* ws,
                                        size_t ws_bytes, struct CUstream_st* stream);

/* Size in bytes of the fixed scratch array behind flce_fused_noalloc. */
#define FLCE_NOALLOC_SCRATCH_BYTES (64u << 20)

/* flce_fused without a caller-supplied workspace, for callers that cannot
 * allocate device memory themselves (for example a plugin whose host program
 * owns all GPU memory, or a foreign-language caller that can only pass the
 * tensors it was given).  The pages have no counterpart: this exists for
 * callers of the library, not for the method.
 *
 * Arguments and results are those of flce_fused.  Scratch space is a
 * module-level device array of FLCE_NOALLOC_SCRATCH_BYTES (64 MiB) that every
 * GPU which loads it keeps until the process exits; the call allocates
 * nothing.  Problems whose fused workspace (flce_workspace_size(p,
 * FLCE_OP_FUSED)) is larger are rejected with FLCE_ERR_WORKSPACE_TOO_SMALL
 * before any work is enqueued.  Every call looks up the array's address in
 * the current device's context; the first call on a device may load the
 * library's device code to do so, so it must not be made while `stream` is
 * being captured into a CUDA graph (it then returns FLCE_ERR_INVALID_ARG
 * without enqueueing anything).  All calls on a device share the one array and it keeps
 * the previous call's contents; the computation overwrites every scratch
 * byte before reading it, so nothing needs clearing, but calls whose GPU
 * work overlaps race on the array: serialise them.  The device status of a
 * call is not readable through flce_get_device_status (the array is not
 * exposed); check the outputs or use flce_fused when that is needed. */
FLCE_API flce_status_t flce_fused_noalloc(const flce_problem_t* p, const void* X, const void* W,
                                          const int64_t* labels, float dloss, float* loss,
                                          void* dX, void* dW, struct CUstream_st* stream);

/* ---------------- cross-entropy for callers that hold the logits -------------
 *
 * PyTorch PR #126348's own case: the caller already has softmax_input (the
 * logits, BT x V), e.g. from its own LM-head matmul.  The PR's summary lists
 * the unfused loss as a matmul then three passes over the logits (row max,
 * row sum, a normalised softmax_output saved for backward) and observes that
 * (a.) the forward needs only the label's entry of the softmax and (b.) the
 * backward can rebuild the softmax from the logits and the small row
 * statistics.  flce_ce_forward reads the logits once and keeps only
 * lse [BT]; flce_ce_backward reads them once more and writes the gradient,
 * rebuilding the softmax from the logits and that lse.  Nothing else of size
 * BT x V is read or written.
 *
 *   y     = c tanh(z / c) under a softcap c, else z       (z: the logits)
 *   lse_i = log sum_j exp(y_ij)
 *   loss  = mean over rows with label_i != ignore_index of (lse_i - y_i,label_i)
 *   dZ_ij = (exp(y_ij - lse_i) - [j == label_i]) * dy/dz * dloss / N_valid,
 *           rows with ignored labels zero
 *
 * Same conventions as the FLCE calls above (labels, shift_seq_len,
 * ignore_index, softcap, the all-ignored case, device status word, stream,
 * caller-owned workspace), except the layout:
 *   - logits and dlogits are DEVICE arrays of BT rows of V entries (bf16 or
 *     fp32, `dtype`), row i at element i*ld (resp. i*ld_grad); ld = 0 means
 *     V.  Rows need not be 16-byte aligned (a dense bf16 tensor with odd V is
 *     fine); the pointers must be aligned to the element size.
 *   - dlogits may be the logits array itself (ld_grad == ld): the gradient
 *     then overwrites the logits in place.  Any other overlap is undefined.
 * Size limits: BT, V < 2^31; ld, ld_grad < 2^40 (else FLCE_ERR_UNSUPPORTED);
 * ld or ld_grad below V is FLCE_ERR_INVALID_ARG. */
typedef struct {
  int64_t BT;            /* rows, >= 0 */
  int64_t V;             /* classes (vocabulary), > 0 */
  int32_t dtype;         /* flce_dtype_t of logits and dlogits */
  int32_t shift_seq_len; /* as in flce_problem_t */
  int64_t ignore_index;
  float softcap;         /* <= 0, NaN or inf: none */
  int32_t reserved1;     /* must be 0 */
  int64_t ld;            /* row stride of logits in elements; 0 = V */
  int64_t ld_grad;       /* row stride of dlogits in elements; 0 = V */
} flce_ce_problem_t;

/* Workspace bytes for op FLCE_OP_FORWARD, FLCE_OP_BACKWARD or FLCE_OP_FUSED
 * (flce_ce_fused) (0 when the problem or op is invalid): a 256-byte header,
 * [BT] fp32 per-row losses (forward, fused), [BT] int64 shifted labels
 * (shift_seq_len > 0). */
FLCE_API size_t flce_ce_workspace_size(const flce_ce_problem_t* p, int op);

/* loss (device fp32 scalar) and lse (device fp32 [BT], kept for
 * flce_ce_backward) from the logits: one read of them. */
FLCE_API flce_status_t flce_ce_forward(const flce_ce_problem_t* p, const void* logits,
                                       const int64_t* labels, float* loss, float* lse, void* ws,
                                       size_t ws_bytes, struct CUstream_st* stream);

/* dlogits from the logits, the forward's lse and the upstream gradient dloss
 * (device fp32 scalar): one read of the logits, one write of dlogits. */
FLCE_API flce_status_t flce_ce_backward(const flce_ce_problem_t* p, const void* logits,
                                        const int64_t* labels, const float* lse,
                                        const float* dloss, void* dlogits, void* ws,
                                        size_t ws_bytes, struct CUstream_st* stream);

/* Forward and backward together, for a training step that holds the logits
 * (dloss by value, as flce_fused): loss (device fp32 scalar), optionally lse
 * (device fp32 [BT], or NULL) and dlogits, reading each row of the logits
 * from HBM once: one read and one write of the BT x V tensor in all, instead
 * of flce_ce_forward's read plus flce_ce_backward's read and write.  Rows of
 * at most 112 KB (V <= 57344 bf16, e.g. 50257; V <= 28672 fp32) go through
 * one persistent block per SM that holds two rows in shared memory: the next
 * row arrives by a bulk asynchronous copy while the current one is reduced
 * and its gradient written.  Longer rows take one block per row, whose
 * second read comes mostly from L2.  Workspace:
 * flce_ce_workspace_size(p, FLCE_OP_FUSED).  dlogits may be the logits
 * array itself. */
FLCE_API flce_status_t flce_ce_fused(const flce_ce_problem_t* p, const void* logits,
                                     const int64_t* labels, float dloss, float* loss, float* lse,
                                     void* dlogits, void* ws, size_t ws_bytes,
                                     struct CUstream_st* stream);

/* How flce_fused schedules its work (bf16 problems; fp32 always recomputes).
 *  FLCE_SCHEDULE_RECOMPUTE: forward pass for lse and loss, then per
 *    vocabulary chunk recompute the logits, form G and run dX and dW
 *    (8*BT*H*V FLOP; workspace < one BT x V bf16 tensor by far).
 *  FLCE_SCHEDULE_FUSED_FORWARD: per row chunk (at least two; at most
 *    1 GiB of q, 2 GiB when an fp32 V x H array exceeds 1 GiB, and 46 MiB
 *    of X rows each) the forward GEMM keeps q = exp(y) dy/dz in bf16 against
 *    one exponent reference per row; the chunk's lse and row factors follow;
 *    dX for the chunk is q W scaled per row, and the chunk's dW is added
 *    into an fp32 V x H running sum (6*BT*H*V FLOP; workspace: a chunk's q
 *    plus that sum, or only the q when dW is fp32).
 *  FLCE_SCHEDULE_AUTO: fused-in-forward when BT >= 512, else recompute. */
typedef enum {
  FLCE_SCHEDULE_AUTO = 0,
  FLCE_SCHEDULE_RECOMPUTE = 1,
  FLCE_SCHEDULE_FUSED_FORWARD = 2
} flce_schedule_t;

/* Set the process-wide flce_fused schedule (also used by
 * flce_workspace_size for FLCE_OP_FUSED); returns the previous one, or -1
 * for an unknown value. */
FLCE_API int32_t flce_set_schedule(int32_t schedule);

/* Process-wide cap, in bytes, on the workspace flce_fused plans under
 * FLCE_SCHEDULE_AUTO (0 = none, the default; also used by
 * flce_workspace_size for FLCE_OP_FUSED).  Under the cap AUTO takes the
 * fused-in-forward schedule only when its workspace fits, else the
 * recompute schedule with its vocabulary chunk narrowed (down to 256
 * columns) until the workspace fits; when nothing fits it plans the
 * smallest recompute workspace.  A cap of one bf16 BT x V tensor (2*BT*V
 * bytes) keeps every plan below the logits' size.  The forced schedules
 * ignore it.  Returns the previous cap. */
FLCE_API uint64_t flce_set_workspace_limit(uint64_t bytes);

/* Synchronise `stream`, then read the device status word and the valid-row
 * count of the last call that used workspace `ws`.  Either output pointer
 * may be NULL.  Returns FLCE_ERR_CUDA if the copy fails. */
FLCE_API flce_status_t flce_get_device_status(const void* ws, struct CUstream_st* stream,
                                     int32_t* device_status, int64_t* n_valid);

/* Static description of a status code; never NULL. */
FLCE_API const char* flce_status_string(flce_status_t s);

/* Limit, in nanoseconds, on every pipeline wait inside the kernels (default
 * 2e9).  A wait that exceeds it records FLCE_ERR_TIMEOUT and the kernel
 * returns.  Process-wide; returns the previous value.  0 restores the
 * default. */
FLCE_API uint64_t flce_set_wait_limit_ns(uint64_t ns);

/* Number of kernel launches (and memsets) the last call on this host
 * thread enqueued (for launch accounting). */
FLCE_API int32_t flce_last_launch_count(void);

/* Failure-path self-test.  Enqueues one tiny kernel that waits, with the
 * same bounded wait the GEMM pipelines use, on a barrier nothing signals.
 * After limit_ns it gives up and records FLCE_ERR_TIMEOUT in the status word
 * of workspace `ws` (>= 256 bytes, 256-byte aligned; the word is cleared
 * first).  Read it with flce_get_device_status; the context stays usable. */
FLCE_API flce_status_t flce_selftest_wait_timeout(void* ws, uint64_t limit_ns,
                                                  struct CUstream_st* stream);

/* Accuracy self-test of the two approximations the GEMM epilogues use in
 * place of library calls: for each of the n fp32 inputs x[i] (device),
 * out[4i .. 4i+3] (device fp32) = the epilogues' tanh (1 - 2 / (2^(2x log2 e)
 * + 1) on the hardware exp2), CUDA's tanhf, the epilogues' exp2 (the
 * ex2.approx.ftz instruction) and CUDA's exp2f, so a test can bound the
 * difference.  Enqueued on `stream`. */
FLCE_API flce_status_t flce_selftest_approx(const float* x, int64_t n, float* out,
                                            struct CUstream_st* stream);

/* Per-launch timing for profiling.  flce_profile_start(n) creates 2n CUDA
 * events; until flce_profile_stop, every kernel the library launches records
 * one event just before it and one just after it on the call's stream (the
 * first n launches only).  flce_profile_stop synchronises on the last event,
 * writes each launch's duration in milliseconds and its kind (see
 * flce_kernel_name) for up to max_out launches, destroys the events and
 * returns the number written, or -1 on error.  Not for use while another
 * thread calls the library. */
FLCE_API flce_status_t flce_profile_start(int32_t n);
FLCE_API int32_t flce_profile_stop(float* ms, int32_t* kinds, int32_t max_out);

/* Name of a kernel kind reported by flce_profile_stop ("lse_gemm",
 * "grad_gemm", "dx_gemm", "dw_gemm", ...); never NULL. */
FLCE_API const char* flce_kernel_name(int32_t kind);

#ifdef __cplusplus
}
#endif

#endif /* FLCE_H_ */
