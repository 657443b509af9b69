/*
 * flce.h -- C ABI of the fused LM-head linear + softcapped cross-entropy for B200 (sm_100a).
 *
 * The operation (little-lm 3.8B write-ups):
 *   - the untied LM head W [Vpad, d] (154.5M = 50304 x 3072 parameters; "Setup" table);
 *   - logits z = X W^T with a logit softcap s = cap * tanh(z / cap), cap = 15 (the config
 *     appendix sets a softcap of 15 for the model and its fused loss; the pages print no
 *     formula, cap*tanh(z/cap) is the reading used);
 *   - a vocabulary of Vreal = 50257 tokens padded to Vpad = 50304, a multiple of 64, for the
 *     tensor cores ("Increasing throughput", vocabulary padding; config appendix).  Padded
 *     columns j >= Vreal take no part in the softmax and get zero gradient;
 *   - cross entropy averaged over the rows whose target is not ignore_index;
 *   - fused: the lm_head matmul is computed in chunks inside the loss, so the full
 *     (B*T, vocab) logits are never materialised ("Increasing throughput", fused linear
 *     cross-entropy).
 *
 *   loss   = (1/Nv) * sum_{i in V} (lse_i - s_{i, t_i}),   lse_i = log sum_{j < Vreal} exp(s_ij)
 *   dz_ij  = g/Nv * (softmax(s_i)_j - [j = t_i]) * (1 - tanh^2(z_ij / cap))    (0 for j >= Vreal)
 *   dX     = dz W,   dW = dz^T X
 * with V = {i : t_i != ignore_index and 0 <= t_i < Vreal}, Nv = |V|.  Nv = 0 gives loss 0 and
 * zero gradients.
 *
 * Conventions for every entry point:
 *   - Data pointers are DEVICE pointers owned by the caller; the library never allocates or
 *     frees memory.  Scratch space is the caller's `workspace` (see flce_workspace_bytes).
 *   - Layouts are row-major and dense: X [N, d] bf16, W [Vpad, d] bf16, targets [N] int64,
 *     lse [N] fp32, loss [1] fp32, dX [N, d] bf16, dW [Vpad, d] fp32 or bf16 (dW_dtype).
 *   - Every array pointer must be 16-byte aligned except loss and lse (4-byte aligned); d and
 *     Vpad must be multiples of 8 (the tensor-memory-accelerator row stride must be a multiple
 *     of 16 bytes).
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Calls are
 *     stream-ordered and asynchronous; calls on different streams are independent when their
 *     workspaces and outputs differ.
 *   - Argument errors are detected on the host before anything is launched and returned as a
 *     negative flce_status.  Targets outside [0, Vreal) that are not ignore_index are not an
 *     argument error: the row is treated as ignored and the device status word gets
 *     FLCE_DEV_BAD_TARGET (read it with flce_read_status).  No kernel ever traps.
 *   - Every wait inside a kernel is bounded; a wait that runs out sets FLCE_DEV_TIMEOUT.
 *   - Results are bitwise reproducible from call to call (fixed reduction orders).
 *   - The device must be compute capability 10.0 (B200, sm_100a).
 */
#ifndef FLCE_H_
#define FLCE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FLCE_OK = 0,
  FLCE_ERR_ARG = -1,       /* null pointer, bad size, inconsistent shape */
  FLCE_ERR_ALIGN = -2,     /* pointer not 16-byte aligned, or d / Vpad not a multiple of 8 */
  FLCE_ERR_WORKSPACE = -3, /* workspace smaller than flce_workspace_bytes() */
  FLCE_ERR_DEVICE = -4,    /* current device is not compute capability 10.0 */
  FLCE_ERR_CUDA = -5,      /* a CUDA runtime call or kernel launch failed */
  FLCE_ERR_TIMEOUT = -6    /* reserved: a device wait ran out (reported via the status word) */
} flce_status;

/* Bits of the device status word (flce_read_status). */
enum { FLCE_DEV_BAD_TARGET = 1u, FLCE_DEV_TIMEOUT = 2u };

/* Element type of the dW output (dW_dtype arguments). */
enum { FLCE_DTYPE_F32 = 0, FLCE_DTYPE_BF16 = 1 };

typedef struct {
  int64_t N;            /* tokens (rows of X, targets); N = 0 is allowed and gives loss 0 */
  int64_t d;            /* hidden size; multiple of 8 */
  int64_t Vpad;         /* rows of W; multiple of 8 */
  int64_t Vreal;        /* real vocabulary, 1 <= Vreal <= Vpad */
  float cap;            /* logit softcap; <= 0 disables it */
  int64_t ignore_index; /* target value that leaves a row out of the loss (e.g. -1) */
  int64_t chunk_rows;   /* rows per fused chunk (bounds the scratch); 0 = automatic: 8192 */
} flce_shape;

/*
 * Bytes of device scratch the calls below need for this shape.  want_grads = 0: the
 * statistics-only forward; want_grads = 1: the forward that also forms the gradients, and the
 * recomputing backward.  The scratch grows with chunk_rows * Vpad (the per-chunk gradient
 * operand) and linearly with N; it never holds an N x Vpad buffer.  Returns 0 when the shape is
 * invalid.
 */
size_t flce_workspace_bytes(const flce_shape* shape, int want_grads);

/*
 * Forward.  Writes loss[0] (mean over rows in the loss) and lse[i] for every row (ignored rows
 * included).  With want_grads = 1 it also forms, in the same pass over the logits, the
 * gradients of g * loss for the upstream gradient g = *grad_scale (a device float; NULL means
 * g = 1): dX [N, d] bf16 is written, and dW [Vpad, d] is written (accumulate_dW = 0) or added to
 * (accumulate_dW = 1).  Gradient accumulation over micro-batches (the pages accumulate over 7
 * per optimizer step) with each micro-batch's loss divided by the number of micro-batches m is
 * accumulate_dW = 1 with *grad_scale = 1/m on every call: each call adds only its own scaled
 * contribution.
 *   dW_dtype: FLCE_DTYPE_F32 (fp32 dW) or FLCE_DTYPE_BF16 (bf16 dW, for bf16 master weights;
 *     each chunk's contribution is added to the stored values in fp32 and rounded to bf16 once).
 * With want_grads = 0, grad_scale, dX and dW may be NULL and are not touched.  When N = 0, X,
 * targets, lse and dX may be NULL.
 * workspace: device scratch of at least flce_workspace_bytes(shape, want_grads) bytes,
 * 256-byte aligned; its contents on entry are ignored.
 */
int flce_forward(const flce_shape* shape, const void* X, const void* W, const int64_t* targets,
                 float* loss, float* lse, int want_grads, const float* grad_scale, void* dX,
                 void* dW, int dW_dtype, int accumulate_dW, void* workspace,
                 size_t workspace_bytes, void* stream);

/*
 * Backward.
 *   grads_precomputed = 1: dX and dW were formed by flce_forward(want_grads = 1) with
 *     accumulate_dW = 0 and grad_scale NULL; both are multiplied in place by the device scalar
 *     *grad_out (nothing runs when grad_out is NULL; the kernel returns at once when
 *     *grad_out == 1).  accumulate_dW must be 0 here (FLCE_ERR_ARG otherwise): a dW that holds
 *     earlier micro-batches cannot be scaled after the fact -- pass g to the forward as
 *     grad_scale instead.
 *   grads_precomputed = 0: recomputes the logits chunk by chunk from X and W, using lse from
 *     flce_forward, and forms dX (written) and dW (written, or added to when
 *     accumulate_dW = 1) for upstream gradient *grad_out (1 when grad_out is NULL).
 * dW_dtype as in flce_forward.  workspace: at least flce_workspace_bytes(shape, 1) bytes
 * (unused when grads_precomputed = 1).
 */
int flce_backward(const flce_shape* shape, const void* X, const void* W, const int64_t* targets,
                  const float* lse, const float* grad_out, void* dX, void* dW, int dW_dtype,
                  int accumulate_dW, int grads_precomputed, void* workspace,
                  size_t workspace_bytes, void* stream);

/*
 * Forward without any caller-provided scratch: loss[0] and lse[N] exactly as flce_forward with
 * want_grads = 0, but the scratch lives in a device array of FLCE_NOALLOC_SCRATCH_BYTES inside the
 * library, so the call allocates nothing and needs no workspace.  It is meant for callers that
 * cannot obtain device memory at call time: a plugin whose host framework owns every device
 * allocation and hands it no allocator, or a latency-critical caller that must not risk the
 * implicit device synchronisation of cudaMalloc.  The write-ups describe no such entry point.
 *   - The array is a file-scope __device__ object: every GPU that loads the library holds it
 *     until the process exits.
 *   - The first call on each device looks up the array's device address with that device
 *     current (cudaGetSymbolAddress); make that first call before any stream capture.
 *   - Shapes whose scratch exceeds the array are rejected with FLCE_ERR_WORKSPACE before
 *     anything runs (chunk_rows = 0 picks the largest chunk of 4096, 2048, ..., 128 rows that
 *     fits; at d = 3072, Vpad = 50304 that admits N up to several hundred thousand rows).
 *   - All calls share the array and it keeps the last call's contents (nothing in it needs to
 *     start at zero).  Calls that overlap on the GPU (different streams, or different host
 *     threads without ordering) race on it and must not be issued.
 *   - The device status word and the count of rows in the loss of the last call on the current
 *     device are read with flce_read_status(NULL, ...), like a workspace's.
 * Same argument rules as flce_forward with want_grads = 0 otherwise.
 */
#define FLCE_NOALLOC_SCRATCH_BYTES (16u << 20)
int flce_forward_noalloc(const flce_shape* shape, const void* X, const void* W,
                         const int64_t* targets, float* loss, float* lse, void* stream);

/*
 * Data-parallel training (the write-ups train with plain DDP on 8 GPUs, gradient all-reduce; the
 * "distributed strategy" paragraph).  Every rank holds W and its own rows.  To make the result
 * equal to one call on the union of all ranks' rows:
 *   1. flce_count_valid writes this rank's number of rows in the loss to *n_valid_out (device
 *      int64, 8-byte aligned);
 *   2. the caller sums it over ranks (an all-reduce) into a device int64 n_valid_total;
 *   3. flce_forward_dp runs flce_forward but normalises by *n_valid_total: loss[0] is this rank's
 *      share of the global mean and dX / dW are the gradients of the global mean (dW: this
 *      rank's contribution, written or accumulated as in flce_forward);
 *   4. the caller sums loss and dW over ranks (all-reduces); dX stays with its rows.
 * flce_forward_dp takes the same arguments as flce_forward plus n_valid_total.
 */
int flce_count_valid(const flce_shape* shape, const int64_t* targets, int64_t* n_valid_out,
                     void* stream);
int flce_forward_dp(const flce_shape* shape, const void* X, const void* W, const int64_t* targets,
                    const int64_t* n_valid_total, float* loss, float* lse, int want_grads,
                    const float* grad_scale, void* dX, void* dW, int dW_dtype,
                    int accumulate_dW, void* workspace, size_t workspace_bytes, void* stream);

/*
 * flce_forward_dp (want_grads = 1) whose dW becomes final in vocabulary buckets, so that the
 * caller's dW all-reduce (step 4) can overlap the rest of the computation: the gradient
 * contractions of the last chunk run as n_buckets launches; launch b completes dW rows
 * [bucket_bounds[b], bucket_bounds[b + 1]) (whole 256-row vocabulary tiles; the last bucket
 * also carries dX), after which the library records bucket_events[b] on `stream`.
 *   n_buckets: 1 .. min(64, ceil(Vpad / 256)).
 *   bucket_events: n_buckets cudaEvent_t handles created by the caller (none NULL).
 *   bucket_bounds: host array of n_buckets + 1 int64, written before the call returns.
 * A caller exchanges bucket b by making its communication stream wait on bucket_events[b] and
 * all-reducing those dW rows there.  The write-ups train with unmodified DDP ("distributed
 * strategy" paragraph), which all-reduces gradients in buckets that overlap the backward pass;
 * this is that overlap for the head's gradient, which the fused forward forms.
 */
int flce_forward_dp_bucketed(const flce_shape* shape, const void* X, const void* W,
                             const int64_t* targets, const int64_t* n_valid_total, float* loss,
                             float* lse, const float* grad_scale, void* dX, void* dW,
                             int dW_dtype, int accumulate_dW, int n_buckets,
                             void* const* bucket_events, int64_t* bucket_bounds,
                             void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward with FP8 logits: the logits contraction z = X W^T reads e4m3 operands with dynamic
 * tensorwise scales (x ~ X8 * *scale_x, w ~ W8 * *scale_w; the scales are device scalars) on the
 * tensor cores' fp8 path, with both scales applied to z before the softcap.  This follows the
 * write-ups' FP8 training ("Increasing throughput": GEMMs in FP8 with dynamic tensorwise scaling
 * through torch._scaled_mm, one forward and two backward GEMMs per layer).
 * With want_grads = 1 the softmax gradient is formed from those logits and the two gradient
 * contractions run
 *   grad_fp8 = 0: in bf16, on the bf16 copies X [N, d] and W [Vpad, d] (dX = dz W, dW = dz^T X);
 *   grad_fp8 = 1: in FP8 as well: the normalised gradient dz * Nv/g (|.| <= 1) times 2^15 is
 *     encoded in e5m2 (a fixed power-of-two scale suffices: no amax pass) and multiplied with the
 *     e4m3 operands, dX = g/(Nv 2^15) * scale_w * (q W8) and dW = g/(Nv 2^15) * scale_x *
 *     (q^T X8), on the tensor cores' 8-bit path.  Needs 0 < cap <= 32; X and W may be NULL.
 * With want_grads = 0 (or grad_fp8 = 1) X and W may be NULL.
 *   X8 [N, d], W8 [Vpad, d]: e4m3 bytes, row-major; d must be a multiple of 16.
 * Outputs, grad_scale, dW_dtype, workspace (flce_workspace_bytes of the same shape) and errors as
 * flce_forward.
 */
int flce_forward_fp8(const flce_shape* shape, const void* X8, const void* W8,
                     const float* scale_x, const float* scale_w, const void* X, const void* W,
                     const int64_t* targets, float* loss, float* lse, int want_grads, int grad_fp8,
                     const float* grad_scale, void* dX, void* dW, int dW_dtype,
                     int accumulate_dW, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Dynamic tensorwise e4m3 quantisation of n bf16 values: *scale_out = amax(|src|) / 448
 * (1 when all values are 0) and dst[i] = e4m3(src[i] / *scale_out), rounded to nearest even and
 * saturated to the finite e4m3 range.  scale_out is a device float; it also serves as the
 * amax accumulator while the call runs.  Four small kernels on `stream`.
 */
int flce_quantize_e4m3(const void* src, int64_t n, void* dst, float* scale_out, void* stream);

/*
 * The model's final RMSNorm, whose output feeds the head (the write-ups' model is Llama-style
 * with RMSNorm; config appendix: rms_norm_eps = 1.0e-6):
 *   x_i = h_i * rstd_i * gamma,  rstd_i = 1 / sqrt(mean_k h_ik^2 + eps)   (fp32 arithmetic)
 * H [N, d] bf16, gamma [d] bf16, X [N, d] bf16 (out), rstd [N] fp32 (out).  d % 8 == 0.
 * H, gamma, X, dX, dH 16-byte aligned; rstd and dgamma 4-byte aligned.
 * Backward, for dX = dL/dx from the loss (e.g. flce_forward's dX):
 *   dH = rstd * (g - xh * mean_k(g * xh)),  dgamma = sum_i dX * xh,  xh = h * rstd, g = dX * gamma
 * dH [N, d] bf16 (out); dgamma [d] fp32 written, or added to with accumulate_dgamma = 1.  The
 * dgamma reduction is deterministic (fixed-order partial sums in `workspace`, at least
 * flce_rmsnorm_workspace_bytes(N, d) bytes, 16-byte aligned).
 */
int flce_rmsnorm_forward(const void* H, const void* gamma, float eps, int64_t N, int64_t d,
                         void* X, float* rstd, void* stream);
size_t flce_rmsnorm_workspace_bytes(int64_t N, int64_t d);
int flce_rmsnorm_backward(const void* H, const void* gamma, const float* rstd, const void* dX,
                          int64_t N, int64_t d, void* dH, float* dgamma, int accumulate_dgamma,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * The final RMSNorm and the head as one training step (the write-ups' model: final RMSNorm,
 * then the untied head and the softcapped loss).  H [N, d] bf16 holds the rows before the norm;
 * the head reads x = h rstd gamma, rounded to bf16 (written to the workspace), and the call
 * returns what flce_forward returns for that x, with dH and dgamma in place of dX:
 *   dH = rstd (gamma . dX - xh c),  c_i = mean_k x_ik dX_ik,  dgamma = sum_i dX_i . xh_i,
 * dX the gradient of g * loss with respect to x (never stored when 0 < cap <= 32) and
 * xh = h rstd.  With 0 < cap <= 32 the backward of the norm is folded into the dX contraction:
 * c_i equals (1/d) sum_j dz_ij z_ij, which the logits pass sums next to the softmax, so the dX
 * epilogue writes dH rows directly and per 32 rows the column sums that make dgamma (summed in
 * row-block order: deterministic).  Otherwise dX goes to the workspace and separate row
 * kernels follow.
 *   eps >= 0 (the write-ups' config: 1e-6).  H, gamma, W, targets, dH, dW 16-byte aligned;
 *   dgamma [d] fp32, 4-byte aligned.  want_grads = 0: loss and lse only (dH, dgamma, dW unused).
 *   grad_scale, dW_dtype: as in flce_forward.  accumulate = 1 adds into both dW and dgamma (the
 *   parameters), 0 writes them; dH is always written.
 *   workspace: flce_workspace_bytes_rmsnorm(shape, want_grads) bytes, 256-byte aligned.
 *   Errors: as flce_forward; FLCE_ERR_ARG also for eps < 0 or a null gamma, or a null dgamma
 *   with want_grads.
 * flce_scale_grads_rmsnorm multiplies dH, dgamma and dW in place by the device scalar *grad_out
 * (nothing when it is 1, or when grad_out is NULL): the upstream gradient applied to gradients
 * that flce_forward_rmsnorm formed with g = 1 and accumulate = 0.
 */
size_t flce_workspace_bytes_rmsnorm(const flce_shape* shape, int want_grads);
int flce_forward_rmsnorm(const flce_shape* shape, const void* H, const void* gamma, float eps,
                         const void* W, const int64_t* targets, float* loss, float* lse,
                         int want_grads, const float* grad_scale, void* dH, float* dgamma,
                         void* dW, int dW_dtype, int accumulate, void* workspace,
                         size_t workspace_bytes, void* stream);
int flce_scale_grads_rmsnorm(const flce_shape* shape, const float* grad_out, void* dH,
                             float* dgamma, void* dW, int dW_dtype, void* stream);
/*
 * flce_forward_rmsnorm for one data-parallel rank: the loss and gradients are normalised by
 * *n_valid_total (device int64, 8-byte aligned: the rows in the loss over all ranks, e.g. the
 * all-reduced flce_count_valid), as flce_forward_dp does for the head alone.  The loss is this
 * rank's share of the global mean; dgamma and dW are its contributions, to be summed over ranks.
 */
int flce_forward_rmsnorm_dp(const flce_shape* shape, const void* H, const void* gamma, float eps,
                            const void* W, const int64_t* targets, const int64_t* n_valid_total,
                            float* loss, float* lse, int want_grads, const float* grad_scale,
                            void* dH, float* dgamma, void* dW, int dW_dtype, int accumulate,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * Self-test of failure detection (no counterpart on the pages): runs the library's bounded
 * pipeline wait on a barrier that nothing arrives at, with a limit of limit_ns (1 ns .. 10 s).
 * The wait runs out, FLCE_DEV_TIMEOUT is or-ed into the status word of `workspace` (read it with
 * flce_read_status), and the kernel returns normally, leaving the context usable.  workspace
 * needs 256 bytes and is otherwise untouched.
 */
int flce_selftest_wait_timeout(void* workspace, uint64_t limit_ns, void* stream);

/*
 * Host-side check of the persistent tile schedule (no counterpart on the pages; runs on the CPU,
 * no GPU needed): `pairs` SM pairs share T0 tiles of cost c0 and T1 tiles of cost c1 (costs in
 * k-blocks) with the same assignment the contraction kernels use.  Returns FLCE_OK when every
 * tile of both problems goes to exactly one (pair, slot); FLCE_ERR_ARG for bad sizes
 * (pairs < 1 or > 4096, T0, T1 < 0 or above 2^24, c0, c1 < 1) or a tile that is missing,
 * repeated or out of range.  max_cost / min_cost (either may be NULL) receive the largest
 * and smallest per-pair sum of tile costs.
 */
int flce_check_pair_schedule(int pairs, int T0, int c0, int T1, int c1, int64_t* max_cost,
                             int64_t* min_cost);

/*
 * Reads the device status word (FLCE_DEV_* bits) and the number of rows in the loss from the
 * workspace of the last call on `stream`; workspace = NULL reads those of the last
 * flce_forward_noalloc call on the current device.  Synchronises that stream.  Either output
 * may be NULL.
 */
int flce_read_status(const void* workspace, uint32_t* dev_status_out, int64_t* n_valid_out,
                     void* stream);

/*
 * Instrumentation (not part of the computation).  flce_instrument(1) resets the counters and
 * starts recording: every kernel the library launches is counted, and each tensor-core
 * contraction launch (kind 0: logits; kind 1: dX and dW, which share one launch; kind 2 is not
 * used) is bracketed by CUDA events on its own stream.  flce_instrument(0) stops recording.  flce_instrument_read waits for the recorded
 * events and fills `out` with the totals since the last reset.  Process-wide; host-thread safe.
 */
typedef struct {
  int64_t launches_total;      /* all kernels launched while recording */
  int64_t gemm_launches[3];    /* contraction launches by kind */
  double gemm_ms[3];           /* summed event-timed durations by kind, milliseconds */
  double gemm_flop[3];         /* 2*M*N*K of the launched extents, summed over those launches;
                                  the gradient launches run over the rows in the loss only, so
                                  with ignored rows they compute less than this */
} flce_kernel_stats;

int flce_instrument(int enable);
int flce_instrument_read(flce_kernel_stats* out);

/* Human-readable name of an flce_status value. */
const char* flce_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* FLCE_H_ */
