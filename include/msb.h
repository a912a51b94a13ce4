/*
 * msb.h -- C ABI of the sparse-MoE block decode library (libmsb.so).
 *
 * One decode step of one sparse-MoE block with calibration-free top-k channel
 * selection.  For each token the router picks the top-K experts; for each
 * (token, routed expert) every intermediate channel is scored with a ternary
 * sketch of the gate weights, exactly the k best channels are kept, only those
 * channels' BF16 gate row, up row and down column are read, SwiGLU is applied,
 * a rank-r term A_e (B_e x) compensates the skipped channels, and the expert
 * outputs are combined by router weight.
 *
 * Sources (web pages, by title and section):
 *  - "KAIST drops calibration from MoE decoding, speeds up blocks by up to
 *    2.69x over vLLM": opening paragraph (small-batch MoE decode is bound by
 *    loading the routed experts' weights), "Top-k instead of a threshold"
 *    (keep each token's k highest-scoring channels; the read budget is known
 *    in advance), "A reader built from weights alone" (ternary sketch filter,
 *    low-rank compensation, both built from the weights only).
 *  - "Calibration-free top-k MoE selector saves tuning": BF16 weights.
 *  - "MoE top_k override (--moe-top-k)", "Ce que ca fait": top-K routing and
 *    the gated expert MLP.
 *  - Ternary Weight Networks (Li, Zhang, Liu 2016): the sketch's threshold
 *    0.7*mean|W| and scale alpha = mean |W| over the kept entries.
 *
 * Conventions for every entry point:
 *  - Device pointers point to memory of the current CUDA device; host pointers
 *    are named *_host.  All device buffers are owned by the caller; the library
 *    allocates nothing on the call path.
 *  - BF16 values are passed as 16-bit patterns (void* / uint16_t*).
 *  - Every device entry point is asynchronous on `stream` (a cudaStream_t; NULL
 *    means the legacy default stream) and returns after enqueueing.
 *  - Return value: MSB_OK (0) or a negative MSB_E* code.  Argument errors are
 *    detected on the host before anything is enqueued.  Kernel-side problems
 *    (a bounded wait that ran out, a non-finite router logit) set a sticky word
 *    in the workspace that msb_check() reports after the stream has been
 *    synchronised.
 *  - Inputs must be finite (no NaN/Inf); a non-finite router logit makes that
 *    call's output undefined (reported as MSB_ENONFINITE) and leaves the
 *    workspace ready for the next call.
 */
#ifndef MSB_H_
#define MSB_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ------------------------------------------------------------------ status */
#define MSB_OK 0
#define MSB_EINVAL (-1)        /* null pointer, size out of range, misalignment,
                                  workspace too small, out aliasing x */
#define MSB_EUNSUPPORTED (-2)  /* sizes beyond the compiled limits below */
#define MSB_ECUDA (-3)         /* a CUDA launch or runtime call failed */
#define MSB_ETIMEOUT (-4)      /* (msb_check) a kernel's bounded wait ran out */
#define MSB_ENONFINITE (-5)    /* (msb_check) the router met NaN/Inf logits: x or W_router
                                  is not finite (invalid input; the output is undefined) */
#define MSB_EINTERNAL (-6)     /* (msb_check) a kernel's internal consistency check failed
                                  (e.g. a channel selection of the wrong size); the access
                                  it guarded was skipped and the output is undefined */

/* ------------------------------------------------------------------ limits */
#define MSB_MAX_D 8192         /* hidden size d: multiple of 64, 64..8192 */
#define MSB_MAX_INTER 4096     /* intermediate size I per expert: 1..4096 */
#define MSB_MAX_EXPERTS 512    /* E: 1..512 */
#define MSB_MAX_TOP_E 16       /* routed experts per token K: 1..min(E,16) */
#define MSB_MAX_RANK 128       /* low-rank rank r: 0..128 */
#define MSB_MAX_BATCH 256      /* tokens per call B: 1..256 */

/* ------------------------------------------------------------------ flags */
#define MSB_FLAG_GENERAL 1u    /* use the multi-kernel path at every batch size */
#define MSB_FLAG_SINGLE 4u     /* batches up to 16 tokens: the single-launch kernel even
                                  where the multi-kernel path is faster (ignored with
                                  MSB_FLAG_GENERAL) */
#define MSB_FLAG_X_READY 2u    /* x is complete when the call is enqueued: nothing earlier on
                                  the stream writes it (activations the host produced), so
                                  the single-launch kernel may fetch it while the previous
                                  launch on the stream still runs.  Wrong results if a
                                  kernel or copy earlier on the stream does write x. */

/* Block dimensions.  renorm = 1: the K kept router probabilities are rescaled
 * to sum to one; 0: they are used as they are. */
typedef struct msb_dims {
  int32_t d;        /* hidden size */
  int32_t inter;    /* intermediate channels per expert, I */
  int32_t experts;  /* E */
  int32_t top_e;    /* routed experts per token, K */
  int32_t rank;     /* low-rank rank r (0 = no compensation term) */
  int32_t renorm;   /* 0 or 1 */
} msb_dims;

/* Optional per-call record of routing and selection (device pointers; any may
 * be NULL).  Token t's routed experts are in rank order (highest logit first).
 *   expert_ids  int32 [B][K]
 *   expert_w    float [B][K]      combine weight of each routed expert
 *   sel         uint16 [B][K][k]  top-k mode: the kept channels, ascending
 *                                 (threshold mode: capacity I, first sel_count used)
 *   sel_count   int32 [B][K]      channels kept per (token, expert)
 *   union_count int32 [E]         channels read per expert (union over the
 *                                 batch's tokens); 0 for unused experts
 *   scores      float [B][K][Ipad] channel scores (Ipad = I rounded up to 16);
 *                                 not written on the dense path (k == I) */
typedef struct msb_trace {
  int32_t* expert_ids;
  float* expert_w;
  uint16_t* sel;
  int32_t* sel_count;
  int32_t* union_count;
  float* scores;
} msb_trace;

/* ------------------------------------------------------------------ packed weights
 * The packer (msb_pack) turns model-layout BF16 weights into the layout the
 * kernels read.  Ipad = I rounded up to a multiple of 16.
 *
 *  router_t  bf16  [E][d]        W_router transposed: one contiguous row per expert.
 *  records   bf16  [E][I][3d]    channel record of (e, j): gate row j | up row j |
 *                                down column j.  One selected channel = one
 *                                contiguous 6d-byte read (16-byte aligned).
 *  sketch    u32   msb_sketch_words(dims) words: ternary sketch of W_gate at
 *                                exactly 2 bits per weight, in tensor-core tile
 *                                order (16-row tiles x 64-column chunks, 256 B each).
 *  alpha     f32   [E][Ipad]     per-row sketch scale (0 on padding rows).
 *  lr_a      bf16  [E][d][r]     A_e, model layout (not repacked).
 *  lr_b      bf16  [E][r][d]     B_e, model layout (not repacked).
 */
/* Sizes of the sketch (u32 words) and alpha (floats) outputs for these dims; 0 when
 * the dims are invalid (any limit below, or top_e > experts). */
size_t msb_sketch_words(const msb_dims* dims);
size_t msb_alpha_count(const msb_dims* dims);

/* Offline packer, host memory only (no CUDA).  Inputs in model layout:
 *   gate_host, up_host  bf16 [E][I][d];  down_host bf16 [E][d][I];  router_host bf16 [d][E].
 * Outputs (caller-allocated host buffers): records_host [E][I][3d], sketch_host
 * (msb_sketch_words), alpha_host (msb_alpha_count), router_t_host [E][d].
 * The sketch of row W = W_gate[e][j] is T_i = sign(W_i) * [|W_i| > 0.7*mean|W|]
 * (strict; evaluated exactly as 10*d*|W_i| > 7*sum|W| in double precision) and
 * alpha = mean |W_i| over the kept entries (0 if none), rounded to float.
 * Uses up to `threads` host threads (<= 0: all hardware threads).
 * Returns MSB_OK, or MSB_EINVAL / MSB_EUNSUPPORTED for a null pointer or dims that
 * msb_sketch_words rejects (checked before anything is written). */
int32_t msb_pack(const uint16_t* gate_host, const uint16_t* up_host, const uint16_t* down_host,
                 const uint16_t* router_host, const msb_dims* dims, uint16_t* records_host,
                 uint32_t* sketch_host, float* alpha_host, uint16_t* router_t_host,
                 int32_t threads);

/* ------------------------------------------------------------------ workspace
 * Bytes of device workspace a call with up to max_batch tokens needs (0 for
 * invalid dims or max_batch outside 1..MSB_MAX_BATCH).  The
 * workspace must be zero-filled once before its first use (msb_workspace_init);
 * every call leaves it ready for the next.  Calls that share a workspace must
 * not overlap on the GPU (same stream, or ordered by events). */
size_t msb_workspace_size(const msb_dims* dims, int32_t max_batch);
int32_t msb_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Synchronises `stream`, reads and clears the workspace's sticky error word.
 * Returns MSB_OK, MSB_EINTERNAL, MSB_ETIMEOUT, MSB_ENONFINITE (in that order of
 * precedence when several were flagged), or MSB_ECUDA if the stream itself failed. */
int32_t msb_check(void* workspace, void* stream);

const char* msb_strerror(int32_t status);

/* Diagnostics: the path moe_sparse_block takes for these arguments on the
 * current device.  Small batches run on the single-launch kernel when it fits
 * (one cluster per (token, routed expert) pair, each pair reading its own k
 * channels): up to 12 (2048 / d)^2 tokens (1..16; the measured crossover: 12 at
 * d = 2048, 3 at d = 4096), up to 16 with MSB_FLAG_SINGLE or 4-bit records.
 * Larger batches, MSB_FLAG_GENERAL, and batches above 1 whose trace asks for the
 * per-expert union count take the multi-kernel path, which reads each expert's
 * union of channels once.  Fills info (host, 8 int32):
 *   {path (1 = single launch, 2 = multi-kernel), cluster size, clusters per
 *    routed expert, channel-record ring slots, dynamic shared-memory bytes,
 *    resident 16-CTA clusters, resident 8-CTA clusters, 0}.
 * Returns MSB_OK, MSB_EINVAL / MSB_EUNSUPPORTED for bad sizes, or MSB_ECUDA. */
int32_t msb_path_info(const msb_dims* dims, int32_t batch, int32_t k, uint32_t flags,
                      int32_t* info);

/* ------------------------------------------------------------------ the block
 * out[t] = sum over the K routed experts e of token t of
 *          w_{t,e} * ( sum_{j in S_{t,e}} silu(gate_j . x_t) * (up_j . x_t) * down[:, j]
 *                      + A_e (B_e x_t) )
 * with S_{t,e} the k channels of highest score alpha_j * |T_j . x_t| (ties: lower j).
 *
 *  x        bf16 [batch][d] device, 16-byte aligned.
 *  batch    1..MSB_MAX_BATCH tokens (one decode step of `batch` sequences).
 *  router_t, records, sketch, alpha, lr_a, lr_b: packed weights (see above);
 *           lr_a / lr_b may be NULL when dims->rank == 0.
 *  k        channels kept per (token, expert), 1..I.  k == I is the dense
 *           path: no sketch is read and every channel is used (the low-rank
 *           term is still added when rank > 0; pass rank 0 for the dense block).
 *  out      bf16 [batch][d] device, must not overlap x.  Rounded once from the
 *           FP32 accumulation (nearest even).
 *  dims     block dimensions (host struct).
 *  workspace, workspace_bytes: device scratch of at least
 *           msb_workspace_size(dims, batch) bytes, zero-filled before first use.
 *  trace    optional host struct of device pointers (NULL: no trace).
 *  flags    0 or an OR of MSB_FLAG_GENERAL, MSB_FLAG_SINGLE, MSB_FLAG_X_READY.
 *  stream   cudaStream_t.
 * FP32 accumulation throughout; channel scores in FP32. */
int32_t moe_sparse_block(const void* x, int32_t batch, const void* router_t, const void* records,
                         const uint32_t* sketch, const float* alpha, int32_t k, const void* lr_a,
                         const void* lr_b, void* out, const msb_dims* dims, void* workspace,
                         size_t workspace_bytes, const msb_trace* trace, uint32_t flags,
                         void* stream);

/* The block with the router's expert count overridden ("MoE top_k override
 * (--moe-top-k)", section "Ce que ca fait"): each token is routed to its top_e
 * highest-scoring experts instead of the dims->top_e the model was trained with.
 * 1 <= top_e <= dims->top_e; a count above the trained one is rejected with
 * MSB_EINVAL.  With dims->renorm the top_e weights are renormalised over the
 * chosen experts; without it they are the softmax over all E.  The workspace is
 * sized for the trained dims; the trace buffers hold top_e entries per token.
 * Otherwise identical to moe_sparse_block (channel top-k with budget k). */
int32_t moe_sparse_block_top_e(const void* x, int32_t batch, const void* router_t,
                               const void* records, const uint32_t* sketch, const float* alpha,
                               int32_t k, int32_t top_e, const void* lr_a, const void* lr_b,
                               void* out, const msb_dims* dims, void* workspace,
                               size_t workspace_bytes, const msb_trace* trace, uint32_t flags,
                               void* stream);

/* The block on activations in host memory, everything enqueued on `stream` (no
 * synchronisation: the host buffers must stay valid, and out_host unread, until the
 * stream has passed the call).
 *  - batches on the single-launch path (see msb_path_info) with x_host and out_host
 *    pinned, mapped into the current device's address space (cudaHostAlloc / torch
 *    pin_memory under unified addressing) and 16-byte aligned: the kernel itself
 *    reads x_host and writes out_host across the host link, so consecutive calls
 *    keep their launch overlap; the staging buffers are not touched.
 *  - otherwise: copies x_host to x_dev, runs moe_sparse_block(x_dev -> out_dev) and
 *    copies out_dev to out_host with cudaMemcpyAsync (pinned memory makes the copies
 *    asynchronous).
 *  x_host, out_host  bf16 [batch][d] host memory, not overlapping each other.
 *  x_dev, out_dev    bf16 [batch][d] device staging buffers (as x and out of
 *                    moe_sparse_block: 16-byte aligned, not overlapping).
 * The other arguments are those of moe_sparse_block (no trace).  Every argument is
 * checked before anything is enqueued; on an error nothing is copied. */
int32_t moe_sparse_block_host(const void* x_host, void* x_dev, int32_t batch, const void* router_t,
                              const void* records, const uint32_t* sketch, const float* alpha,
                              int32_t k, const void* lr_a, const void* lr_b, void* out_dev,
                              void* out_host, const msb_dims* dims, void* workspace,
                              size_t workspace_bytes, uint32_t flags, void* stream);

/* The calibrated-threshold selector that the pages compare top-k against
 * ("The threshold promises a budget but does not keep it"): identical to
 * moe_sparse_block except S_{t,e} = { j : score_j > tau }, so the number of
 * channels read varies per (token, expert).  Always the multi-kernel path. */
int32_t moe_sparse_block_threshold(const void* x, int32_t batch, const void* router_t,
                                   const void* records, const uint32_t* sketch,
                                   const float* alpha, float tau, const void* lr_a,
                                   const void* lr_b, void* out, const msb_dims* dims,
                                   void* workspace, size_t workspace_bytes,
                                   const msb_trace* trace, void* stream);

/* The batch-1 block for callers that cannot allocate device memory.  The source
 * pages have no counterpart to this entry point: it serves callers that own no
 * device allocator -- a plugin that its host framework hands only input and
 * output buffers, or code running where a cudaMalloc would synchronise the
 * device or is not permitted.  Such a caller passes only the inputs and the
 * output; nothing else is allocated.
 *
 * Same arguments and result as moe_sparse_block with batch = 1 and no
 * workspace.  The scratch (error word, arrival counters, a d-float FP32
 * accumulator) is a static device array of the library, about 37 KB, held on
 * every GPU that loads the library until the process exits.  Limits: d <=
 * MSB_NOALLOC_MAX_D, and the shapes must fit the single-launch kernel; otherwise
 * MSB_EUNSUPPORTED (argument errors give MSB_EINVAL, as for moe_sparse_block).
 * The first call on a device looks up the array's device address (do that
 * first call before any stream capture).  Every call clears the part of the
 * array it uses on `stream` and then launches; all calls share the array, so
 * calls that overlap on the GPU (unordered streams) race.  What the kernel
 * flags (a non-finite router logit, a bounded wait that ran out, a failed
 * consistency check; the output of such a call is undefined) stays in the
 * array's error word until the next call clears it: read it with
 * msb_noalloc_check before that next call. */
#define MSB_NOALLOC_MAX_D 8192
int32_t moe_sparse_block_noalloc(const void* x, const void* router_t, const void* records,
                                 const uint32_t* sketch, const float* alpha, int32_t k,
                                 const void* lr_a, const void* lr_b, void* out,
                                 const msb_dims* dims, const msb_trace* trace, void* stream);

/* Status of the last moe_sparse_block_noalloc call on the current device: synchronises
 * `stream`, reads the static array's error word and clears it.  Returns MSB_OK,
 * MSB_EINTERNAL, MSB_ETIMEOUT, MSB_ENONFINITE (as msb_check), or MSB_ECUDA.  Call it
 * after the call whose status is wanted and before the next allocation-free call. */
int32_t msb_noalloc_check(void* stream);

/* Stack glue between decode layers (attention omitted):
 *   h[t] += y[t]            (h float [batch][d], y bf16 [batch][d]; y may be NULL: no add)
 *   x_next[t] = BF16( h[t] / sqrt(mean(h[t]^2) + eps) )   (RMSNorm, unit weight)
 * h is updated in place; x_next bf16 [batch][d]. */
int32_t msb_residual_rmsnorm(float* h, const void* y, void* x_next, int32_t batch, int32_t d,
                             float eps, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MSB_H_ */
