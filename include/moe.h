/*
 * moe.h -- C ABI of the B200 top-k routed mixture-of-experts FFN forward.
 *
 * The operation (sources are the pages on the MoE FFN, by title and item):
 *   "ClikaRT::nn::QMoEWoQ", forward(): one fused MoE step, x [T, H] and the
 *     caller-computed router_logits [T, E] -> [T, H] in x's dtype; an optional
 *     shared_output [T, H] folds into the routed combine.
 *   "Struct MoeSpec" fields: router_bias (added to every logit before scoring),
 *     score (softmax over every logit, or each logit's own sigmoid),
 *     selection_bias (choose by score + B[e], weigh by score alone), groups
 *     (only the best groups' experts are eligible), renormalize (kept weights
 *     rescaled to sum to one, the sum clamped at 2^-14 per sum_can_clamp),
 *     scale (every kept weight times S, after renormalization), weigh_inputs
 *     (the weight scales the expert's input instead of its output), biases
 *     (gate, up and down bias rows per expert), act (the gated activation).
 *   "MoE" graph-op page: fc1 [E, 2*inter, hidden] (fused gate||up, interleaved
 *     or not per swiglu_fusion), fc2 [E, hidden, inter], activation_alpha,
 *     activation_beta, swiglu_limit, k, normalize_routing_weights.
 *   "Struct Moe": shared experts (shared_dff) with an optional sigmoid gate
 *     sigma(x . g); groups scored by their two best experts.
 *   "ClikaRT::nn::QMoEWoQ" class notes: weight-only quantized (MXFP4) expert
 *     stacks decoded block by block inside the GEMM, never as a dense copy.
 *
 * Readings where the pages are silent: ties go to the lower expert (group)
 * index; a group's score is the sum of its two best keys; the renormalizing sum
 * is max(sum, 2^-14); SiLU gating is h = g*sigmoid(alpha*g) * (u + beta) with
 * limit L > 0 applying g <- min(g, L), u <- clamp(u, -L, L); gate rows come
 * first (concat) or at even indices (interleaved).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are caller-owned CUDA device memory of the current
 *     device; the library allocates no device memory.  Row-major layouts.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *     stream).  After validation every call is asynchronous on that stream,
 *     performs no host synchronisation and may be captured in a CUDA graph.
 *   - Validation is synchronous and happens before any launch; a rejected call
 *     launches nothing, returns a nonzero moe_status and sets a thread-local
 *     message readable with moe_last_error().
 *   - Thread-safe and reentrant: no global mutable state except the
 *     thread-local error message and a per-device cache of kernel attributes.
 */
#ifndef MOE_B200_MOE_H
#define MOE_B200_MOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---- */
typedef enum {
  MOE_OK = 0,
  MOE_ERR_NULL = 1,        /* a required pointer is NULL */
  MOE_ERR_SHAPE = 2,       /* a size is out of range or inconsistent */
  MOE_ERR_DTYPE = 3,       /* unknown dtype code or unsupported combination */
  MOE_ERR_ALIGN = 4,       /* a pointer is not 16-byte aligned (TMA requirement) */
  MOE_ERR_UNSUPPORTED = 5, /* valid per the pages but not built here */
  MOE_ERR_WORKSPACE = 6,   /* workspace NULL or smaller than moe_workspace_size() */
  MOE_ERR_CUDA = 7,        /* a CUDA runtime call failed (message has the name) */
  MOE_ERR_TIMEOUT = 8,     /* a device-side bounded wait gave up (moe_debug_status) */
  MOE_ERR_ARG = 9          /* an option value is out of range */
} moe_status;

/* ---- dtype codes ---- */
enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_MXFP4 = 2 };
/* ---- scoring ("Struct MoeSpec" score) ---- */
enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 };
/* ---- gated activation ("Struct MoeSpec" act; graph-op activation_type) ---- */
enum { MOE_ACT_SILU = 0, MOE_ACT_GELU_ERF = 1, MOE_ACT_GELU_TANH = 2, MOE_ACT_RELU = 3,
       MOE_ACT_IDENTITY = 4 };
/* ---- gate/up layout (graph-op swiglu_fusion: 2 = fused concat, 1 = fused interleaved,
 *      0 = not fused: the gate rows in their own stack, "MoE" set_weights gate_experts) ---- */
enum { MOE_GU_CONCAT = 0, MOE_GU_INTERLEAVED = 1, MOE_GU_UNFUSED = 2 };
/* ---- expert FFN form (graph-op fc1 fusion_size: 2 = gated, 1 = plain) ---- */
enum { MOE_FFN_GATED = 0, MOE_FFN_PLAIN = 1 };

/*
 * Problem sizes.  T tokens (a 3-D x [B, S, d] is passed as T = B*S), d hidden,
 * F expert dff, E routed experts, k experts per token (1 <= k <= E), Fs the
 * shared expert's dff (0 = no shared expert).
 * Supported dtype combinations (act_dtype, w_dtype): (F32, F32), (BF16, BF16),
 * (BF16, MXFP4).  logit_dtype is F32 or BF16.
 */
typedef struct {
  int64_t T, d, F, E, k, Fs;
  int32_t act_dtype;   /* x, y, expert biases, shared weights, shared gate, shared_output */
  int32_t w_dtype;     /* routed expert stacks */
  int32_t logit_dtype; /* router_logits and router_bias */
  int32_t reserved;    /* must be 0 */
} moe_shape;

/* Routing and activation options.  Initialise with moe_options_init(). */
typedef struct {
  int32_t score;       /* MOE_SCORE_*                                   default SOFTMAX */
  int32_t renormalize; /* 0/1; w <- w / max(sum_kept w, 2^-14)           default 0       */
  float routed_scale;  /* S, applied after renormalization               default 1       */
  int32_t n_group;     /* 0 = no group limit; else E % n_group == 0      default 0       */
  int32_t topk_group;  /* groups kept; topk_group * E/n_group >= k        default 0       */
  int32_t weigh_inputs;/* 0/1: weight scales the expert input (Llama 4)   default 0       */
  int32_t act;         /* MOE_ACT_*                                      default SILU    */
  float alpha;         /* SiLU slope: g * sigmoid(alpha * g)             default 1       */
  float beta;          /* h = act(g) * (u + beta)                        default 0       */
  float limit;         /* SiLU clamp; 0 = none                           default 0       */
  int32_t gu_layout;   /* MOE_GU_*                                       default CONCAT  */
  int32_t shared_gate; /* 0/1: shared expert output times sigmoid(x . g) default 0       */
  int32_t ffn;         /* MOE_FFN_GATED: h = act(g) * (u + beta);        default GATED   */
                       /* MOE_FFN_PLAIN: h = act(fc1 x + b1), one matrix (graph-op       */
                       /* activation_type relu/gelu/silu/identity with fusion_size 1;    */
                       /* alpha for SiLU, no beta, no limit)                             */
} moe_options;

/*
 * Tensors (device pointers; NULL = absent where marked optional).
 *   x               [T, d] act_dtype
 *   router_logits   [T, E] logit_dtype
 *   router_bias     [E] logit_dtype, optional; l' = fp32(l) + fp32(bias)
 *   selection_bias  [E] fp32, optional
 *   gate_up         [E, 2F, d] w_dtype; MXFP4: e2m1 codes [E, 2F, d/2] u8, two per
 *                   byte, the even k in the low nibble
 *   gate_up_scales  MXFP4 only: e8m0 block scales [E, 2F, d/32] u8 (blocks of 32 along d)
 *   gate_up_bias    [E, 2F] act_dtype, optional (same row order as gate_up)
 *   down            [E, d, F] w_dtype; MXFP4: codes [E, d, F/2]
 *   down_scales     MXFP4 only: [E, d, F/32]
 *   down_bias       [E, d] act_dtype, optional
 *   shared_gate_up  [2Fs, d] act_dtype (required when Fs > 0; same layout option)
 *   shared_down     [d, Fs] act_dtype (required when Fs > 0)
 *   shared_gate_vec [d] act_dtype (required when shared_gate)
 *   shared_output   [T, d] act_dtype, optional; added to y
 *   y               [T, d] act_dtype, output (must not alias any input)
 *   topk_idx        [T, k] int32, optional output: chosen experts, best first
 *   topk_w          [T, k] fp32, optional output: their weights
 *   gate            MOE_GU_UNFUSED only: the gate rows [E, F, d] w_dtype (MXFP4: codes
 *                   [E, F, d/2] with gate_scales [E, F, d/32]); gate_up then holds the
 *                   up rows [E, F, d] and gate_up_bias their bias [E, F]
 *   gate_bias       [E, F] act_dtype, optional (MOE_GU_UNFUSED)
 *   router_weight   [d, E] act_dtype ("Struct MoeSpec" wr, wr[(i-1)E + e]): with
 *                   router_logits NULL the layer computes the logits x Wr itself
 *                   (fp32 accumulation) and routes on them without storing them
 *   logits_out      [T, E] fp32, optional output (router_weight only): the logits
 *                   the layer computed, before router_bias
 * With MOE_FFN_PLAIN, gate_up is fc1 [E, F, d] (bias [E, F]) and shared_gate_up
 * [Fs, d].  The shared expert of an unfused layer keeps one stack [2Fs, d], gate
 * rows first.
 */
typedef struct {
  const void *x, *router_logits, *router_bias;
  const float *selection_bias;
  const void *gate_up;
  const uint8_t *gate_up_scales;
  const void *gate_up_bias;
  const void *down;
  const uint8_t *down_scales;
  const void *down_bias;
  const void *shared_gate_up, *shared_down, *shared_gate_vec, *shared_output;
  void *y;
  int32_t *topk_idx;
  float *topk_w;
  const void *gate;
  const uint8_t *gate_scales;
  const void *gate_bias;
  const void *router_weight;
  float *logits_out;
} moe_tensors;

/* Fill `opts` with the defaults listed in moe_options (the graph-op page's
 * defaults: alpha 1, beta 0, limit 0, k from the shape; renormalize off). */
MOE_API void moe_options_init(moe_options *opts);

/*
 * Bytes of device workspace moe_forward / moe_route need for this problem
 * (0 if the arguments are invalid; moe_last_error() then says why).
 * The workspace holds the routing, the expert-sorted row permutation and the
 * intermediate activations; its contents do not persist between calls.
 */
MOE_API size_t moe_workspace_size(const moe_shape *shape, const moe_options *opts);

/*
 * The whole forward ("ClikaRT::nn::QMoEWoQ" forward(); "Struct MoeSpec"):
 * route -> sort rows by expert -> gate_up GEMM + bias + gated activation ->
 * down GEMM + bias + routing weight -> deterministic combine (+ shared expert,
 * + shared_output) -> y [T, d] in act_dtype.
 * workspace: device memory of at least moe_workspace_size() bytes, 256-byte
 * aligned, used exclusively by this call until it completes on `stream`.
 * Errors: MOE_ERR_NULL / SHAPE / DTYPE / ALIGN / ARG / UNSUPPORTED / WORKSPACE
 * before any launch; MOE_ERR_CUDA if a launch fails.  T == 0 is a no-op.
 * Results are bitwise reproducible run to run for the same inputs.
 * Kernel choice (environment variables read at every call; set them before
 * moe_workspace_size, the choices may need different workspace sizes):
 *   - bf16 weights, T*k > 4096, fused or plain layout: CTA pairs with the weight
 *     rows as the MMA's M (256 over two SMs) and the token rows as N, padded to 16
 *     (MOE_B200_SWAP_GEMM=0 turns them off);
 *   - otherwise bf16: token tiles, on CTA pairs (256 rows over two SMs) when the
 *     experts average >= 512 routed rows and T*k > 4096, else one CTA per 128-row
 *     tile, with split-K for small batches (MOE_B200_PAIR_GEMM=0 or =1 forces
 *     one or the other); for T <= 64 gate_up reads x in place and, unless
 *     MOE_B200_FUSED_FFN=0 or MOE_B200_INTERLEAVE=1, gate_up and down run as one
 *     launch whose down tiles start once their expert's h rows are complete (a
 *     cooperative launch; where its CTAs cannot all be resident, two launches);
 *   - MXFP4 weights: one CTA per tile; MOE_B200_PAIR_FP4=1 picks CTA pairs with
 *     256 decoded weight rows (slower on the shapes measured);
 *   - MOE_B200_INTERLEAVE=1: the bf16 GEMMs visit the experts largest first,
 *     alternating with the smallest (results unchanged);
 *   - MOE_B200_GEMV=N (N <= 4): bf16 batches of at most N tokens with E <= 256 and d,
 *     F, Fs multiples of 64 run the whole forward in one cooperative launch (routing
 *     inside it unless router_weight is given, then after the router kernel): each
 *     warp streams weight tiles with TMA and multiplies them by the token rows with
 *     warp-level mma.sync; off by default (slower on the shapes measured).
 * Launches: every kernel after the first may be scheduled while its
 * predecessor in the stream still runs (programmatic dependent launch) and
 * waits on the device for the predecessor's results; MOE_B200_PDL=0, read
 * once per process, turns this off.
 */
MOE_API int moe_forward(const moe_shape *shape, const moe_options *opts, const moe_tensors *t,
                void *workspace, size_t workspace_bytes, void *stream);

/*
 * Routing only ("Struct MoeSpec" score, selection_bias, groups, renormalize,
 * scale): writes t->topk_idx [T, k] and t->topk_w [T, k] (both required here).
 * Only x (when shared_gate or router_weight), router_logits or router_weight,
 * router_bias and selection_bias are read.  Same workspace rules as moe_forward.
 */
MOE_API int moe_route(const moe_shape *shape, const moe_options *opts, const moe_tensors *t,
              void *workspace, size_t workspace_bytes, void *stream);

/*
 * moe_forward that also records caller-created CUDA events (cudaEvent_t passed
 * as void*) on `stream` at the stage boundaries, for per-kernel timing:
 *   events[0] before routing          events[4] after the gate_up GEMM
 *   events[1] after routing           events[5] after the down GEMM
 *   events[2] after sort/scan/scatter events[6] after the combine
 *   events[3] after the row gather
 * (events[4] and events[5] both after the one launch of the two GEMMs when
 * moe_forward_fused_gemms says they are fused.)
 * n_events <= MOE_STAGE_EVENTS; NULL entries are skipped.  Same results,
 * errors and workspace rules as moe_forward.  Called under stream capture,
 * the events become event-record nodes of the graph and time every replay.
 */
#define MOE_STAGE_EVENTS 7
MOE_API int moe_forward_events(const moe_shape *shape, const moe_options *opts, const moe_tensors *t,
                               void *workspace, size_t workspace_bytes, void *stream,
                               void *const *events, int n_events);

/*
 * moe_forward without a caller workspace, for callers that cannot allocate
 * device memory (a plugin inside a runtime that owns all device memory and
 * offers no allocator; a request path that must not call cudaMalloc).  It is
 * not an operation of the pages (they have no counterpart): the forward is
 * the same as moe_forward, run on a static scratch array of
 * MOE_NOALLOC_WORKSPACE_BYTES inside the library, held by every GPU that
 * loads the library until the process exits.
 *   - The first call in each CUDA context (the device's primary context, or a
 *     caller's own context current on the calling thread) looks up the array's
 *     device address there (cudaGetSymbolAddress, with that device current) and
 *     caches it for that context; make that first call before any stream
 *     capture.
 *   - Problems whose moe_workspace_size() exceeds the array are rejected with
 *     MOE_ERR_WORKSPACE (nothing is launched); use moe_forward for them.
 *   - All calls share the array and it keeps the last call's contents: calls
 *     that overlap on the GPU (other streams or threads) race and give wrong
 *     results; serialise them.
 *   - It calls no cudaMalloc or cudaFree.  Other errors as moe_forward; the
 *     device status word lives in the array, read it with
 *     moe_noalloc_debug_status.
 */
#define MOE_NOALLOC_WORKSPACE_BYTES (64u << 20)
MOE_API int moe_forward_noalloc(const moe_shape *shape, const moe_options *opts, const moe_tensors *t,
                                void *stream);

/* moe_debug_status for moe_forward_noalloc: synchronises `stream` and reads the
 * device status word the last call on the current context left in the static
 * array (no counterpart on the pages). */
MOE_API int moe_noalloc_debug_status(void *stream);

/* Size in bytes of the static scratch array (MOE_NOALLOC_WORKSPACE_BYTES of the
 * library as built). */
MOE_API size_t moe_noalloc_workspace_bytes(void);

/* Number of CUDA kernels one moe_forward of this problem launches (-1 if the
 * arguments are invalid; 0 for T == 0).  For launch accounting; with router_logits
 * (the few-token kernel adds the router kernel when router_weight is given). */
MOE_API int moe_forward_kernel_count(const moe_shape *shape, const moe_options *opts);

/* The split-K factors moe_forward uses for the gate_up and down GEMMs of this
 * problem (1 = K not split; more only for bf16 batches of at most 4096 routed rows
 * on the single-CTA GEMMs, when the tiles alone would leave SMs idle).  Returns
 * MOE_OK or the argument error of moe_forward. */
MOE_API int moe_forward_split_k(const moe_shape *shape, const moe_options *opts, int *splits_gate_up,
                                int *splits_down);

/* 1 if moe_forward of this problem runs gate_up and down as one kernel launch
 * (batches of at most 64 tokens with bf16 weights; MOE_B200_FUSED_FFN=0 turns it
 * off), 2 if it runs the whole forward as one launch of the few-token kernel
 * (MOE_B200_GEMV), 0 if neither, -1 if the arguments are invalid.  Stage events 4
 * and 5 are then both recorded after that launch (with 2, events 1-3 before it and
 * 4-6 after it). */
MOE_API int moe_forward_fused_gemms(const moe_shape *shape, const moe_options *opts);

/* Message of the last failed call on this thread ("" if none). */
MOE_API const char *moe_last_error(void);

/*
 * Synchronises `stream` and reads the device status word a previous call left
 * in `workspace` (MOE_OK, or MOE_ERR_TIMEOUT if a bounded device wait gave up,
 * MOE_ERR_SHAPE if a device-side consistency check failed).  Intended for tests.
 */
MOE_API int moe_debug_status(const void *workspace, void *stream);

/* Library version string. */
MOE_API const char *moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_MOE_H */
