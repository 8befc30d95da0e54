/*
 * moe.h -- C ABI of the B200 (sm_100a) stacked Mixture-of-Experts FFN
 * forward pass.
 *
 * The layer (max.nn.moe.StackedMoE page, class signature and "Weight tensor
 * shapes"):
 *
 *   1. router      logits -> expert_indices [T,k], expert_weights [T,k]
 *                  (softmax top-k, or the fused sigmoid gate with sink lanes
 *                  of the Mojo sink_gate_router_kernel page);
 *   2. bucketing   expert_indices -> per-expert CSR offsets [E+1] and the
 *                  permutation of the T*k routed slots (moe_create_indices,
 *                  named on the sink_gate_router_kernel page; NeMo
 *                  _permute_tokens_for_grouped_mm);
 *   3. grouped gate_up GEMM over gate_up_proj [E, H, 2D] with the gated
 *      activation of the max.nn.moe.GatedActivation page fused in;
 *   4. grouped down GEMM over down_proj [E, D, H]; the router weight is
 *      applied after the expert (StackedMoE apply_router_weight_first=False),
 *      including to the down bias (NeMo _apply_bias), and the k routed rows
 *      of each token are summed back in token order.
 *
 * Notation: T tokens, H hidden_dim, E routed experts, S sink lanes, k top_k,
 * D moe_dim, R = T*k routed slots.  Slot s = t*k + j is the j-th choice of
 * token t.
 *
 * Conventions for every entry point:
 *   - Every tensor pointer is a DEVICE pointer owned by the caller.  All
 *     tensors are dense row-major (C order) except the logits, whose row
 *     stride is logits_row_stride elements.
 *   - bf16 tensors are passed as `const void*` and hold IEEE bfloat16 values.
 *   - x, gate_up_w, down_w, out and the workspace must be 16-byte aligned
 *     (they are read or written by the Tensor Memory Accelerator).
 *   - The library allocates nothing, frees nothing and never synchronizes
 *     inside these calls: work is enqueued on `stream` in order and the call
 *     returns.  Every buffer must stay valid until that work completes.
 *   - Arguments are validated on the host before anything is enqueued.  A
 *     non-OK status means nothing was enqueued, except MOE_ERR_CUDA, which
 *     reports a failed launch (the stream may hold part of the work).
 *   - Faults found while the kernels run (an index out of range in caller-
 *     provided routing, an inconsistent CSR, a pipeline wait that timed out)
 *     are recorded as bits in a status word at the start of the workspace and
 *     the offending access is skipped; read them with moe_device_status().
 *   - Requires a compute-capability 10.0 device (B200); other devices get
 *     MOE_ERR_UNSUPPORTED.
 */
#ifndef MOE_B200_MOE_H_
#define MOE_B200_MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream.  NULL is the legacy default stream. */
typedef struct CUstream_st* moe_stream_t;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARGUMENT = 1,    /* bad size, null required pointer, misalignment, bad alpha/limit */
  MOE_ERR_UNSUPPORTED = 2,         /* valid by the pages but outside what this library implements */
  MOE_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes < moe_workspace_size() */
  MOE_ERR_CUDA = 4,                /* a CUDA runtime call or launch failed */
  MOE_ERR_DEVICE_TIMEOUT = 5       /* moe_device_status() found a timed-out pipeline wait */
} moe_status_t;

/* Router kinds.  SOFTMAX_TOPK: the k largest logits (ties to the lowest
 * expert index, ordered by descending logit), weights = softmax over the k
 * selected logits.  SIGMOID_SINK: the sink_gate_router_kernel page's fused
 * chain -- selection on sigmoid(logit) + expert_bias (the bias is used for
 * selection only), weights = softmax over [log sigmoid(z_selected),
 * log sigmoid(z_sink)] of the RAW logits, times route_scale * global_scale. */
typedef enum { MOE_ROUTER_SOFTMAX_TOPK = 0, MOE_ROUTER_SIGMOID_SINK = 1 } moe_router_t;

/* Column layout of the 2*D gate_up output (StackedMoE gate_up_format).
 * CONCATENATED: [gate | up], gate = columns 0..D-1, up = D..2D-1.
 * INTERLEAVED:  gate = even columns, up = odd columns (NeMo quick_geglu). */
typedef enum { MOE_GATE_UP_CONCATENATED = 0, MOE_GATE_UP_INTERLEAVED = 1 } moe_gate_up_format_t;

/* GatedActivation fused_activation:
 * SILU:      silu(g) * u; with limit > 0, g = min(g, limit), u = clamp(u, +-limit).
 * SWIGLUOAI: g * sigmoid(alpha * g) * (u + 1), same clamps when limit > 0.
 * GELU_TANH: 0.5 g (1 + tanh(0.7978845608028654 (g + 0.044715 g^3))) * u. */
typedef enum { MOE_ACT_SILU = 0, MOE_ACT_SWIGLUOAI = 1, MOE_ACT_GELU_TANH = 2 } moe_activation_t;

typedef enum { MOE_DTYPE_BF16 = 0, MOE_DTYPE_F32 = 1 } moe_dtype_t;

/* One layer configuration.  Field names follow the StackedMoE constructor
 * (hidden_dim, num_experts, num_experts_per_token -> top_k, moe_dim,
 * gate_up_format, has_bias), the GatedActivation fields (alpha, limit) and
 * the sink_gate_router_kernel parameters (n_shared_experts -> num_sink,
 * route_scale). */
typedef struct {
  int32_t num_tokens;          /* T >= 0 (T = 0 is a no-op) */
  int32_t hidden_dim;          /* H, multiple of 8 */
  int32_t num_experts;         /* E, 1..1024 */
  int32_t top_k;               /* k, 1..min(E, 32) */
  int32_t moe_dim;             /* D, multiple of 8 */
  int32_t num_sink;            /* S >= 0; must be 0 for SOFTMAX_TOPK */
  moe_router_t router;
  moe_dtype_t logits_dtype;    /* BF16 or F32 */
  int64_t logits_row_stride;   /* elements between logits rows, >= E + S; a wider row's tail is not read */
  float route_scale;           /* SIGMOID_SINK only: host scalar multiplied into every weight */
  moe_gate_up_format_t gate_up_format;
  moe_activation_t activation;
  float alpha;                 /* sigmoid scale of SWIGLUOAI; must be 0 for the others */
  float limit;                 /* clamp bound, >= 0; 0 = no clamp; must be 0 for GELU_TANH */
  int32_t has_bias;            /* 1: gate_up_b [E,2D] and down_b [E,H] given; 0: both NULL */
} moe_config_t;

/* Device-side fault bits reported by moe_device_status(). */
#define MOE_DEVICE_ERR_EXPERT_INDEX   0x1  /* an expert index outside [0, E): slot ignored */
#define MOE_DEVICE_ERR_CSR            0x2  /* offsets not a CSR of R slots, or a permutation entry out of range */
#define MOE_DEVICE_ERR_TIMEOUT_GEMM1  0x4  /* a gate_up GEMM pipeline wait gave up */
#define MOE_DEVICE_ERR_TIMEOUT_GEMM2  0x8  /* a down GEMM pipeline wait gave up */
#define MOE_DEVICE_ERR_TIMEOUT_CSR    0x10 /* the one-launch CSR build's grid barrier gave up */
#define MOE_DEVICE_ERR_LAUNCH         0x20 /* a CTA-pair kernel ran without clusters of two CTAs: nothing computed */
/* (a wait that gives up inside the single-launch FFN sets both GEMM bits) */

/* Number of events moe_forward_timed() records (one before each stage and
 * one after the last). */
#define MOE_NUM_STAGE_EVENTS 9

const char* moe_status_string(moe_status_t status);

/* Bytes of device workspace that any call below needs for this
 * configuration.  Host only, no CUDA calls.  The workspace holds the device
 * status word, the CSR scratch, the gathered rows Xp [R,H], the activations
 * h [R,D] and the unreduced expert outputs Y [R,H] (bf16), and the
 * single-launch FFN's per-piece arrival counters. */
moe_status_t moe_workspace_size(const moe_config_t* cfg, size_t* bytes);

/* Stage 1, the router (sink_gate_router_kernel page, Args; softmax top-k
 * reading above).  One warp per token.
 *   logits         [T, logits_row_stride] of logits_dtype; routed columns
 *                  0..E-1, then the S sink columns E..E+S-1.
 *   expert_bias    [E] fp32, SIGMOID_SINK only (NULL = zero); selection only.
 *   global_scale   device [1] fp32, SIGMOID_SINK only (NULL = 1).
 *   expert_indices [T, k] int32 out, descending score, ties to lowest index.
 *   expert_weights [T, k] fp32 out (fp32 whatever the logits dtype).
 *   sink_weights   [T, S] fp32 out, required when S > 0.
 * SIGMOID_SINK requires k + S to be a power of two <= 32 (the page's
 * contract for its single warp-level normalisation); otherwise
 * MOE_ERR_UNSUPPORTED. */
moe_status_t moe_route(const moe_config_t* cfg, const void* logits, const float* expert_bias,
                       const float* global_scale, int32_t* expert_indices, float* expert_weights,
                       float* sink_weights, moe_stream_t stream);

/* Stage 2, moe_create_indices: per-expert CSR of the R = T*k slots.
 *   expert_indices [T, k] int32 in [0, E) (out-of-range entries are skipped
 *                  and flagged MOE_DEVICE_ERR_EXPERT_INDEX).
 *   expert_offsets [E+1] int32 out: exclusive prefix sum of per-expert counts.
 *   permutation    [R] int32 out: slot ids sorted by expert, ascending slot
 *                  within one expert (stable; token of slot s is s / k).
 *   inverse        [R] int32 out or NULL: position of slot s in permutation.
 * The result is deterministic (no atomics decide any order). */
moe_status_t moe_create_indices(const moe_config_t* cfg, const int32_t* expert_indices,
                                int32_t* expert_offsets, int32_t* permutation, int32_t* inverse,
                                void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* Stages 3 and 4 given a routing: gather the routed rows, grouped gate_up GEMM
 * + bias + activation (tcgen05 tensor cores), grouped down GEMM + bias, times
 * the routing weight, and the per-token sum over the k slots.  By default
 * the two GEMMs run as ONE persistent cooperative launch (the MegaFFN page's
 * single launch: a down tile of a 128-row piece starts as soon as every
 * gate_up tile of that piece has stored its h, signalled through per-piece
 * arrival counters in the workspace, every wait bounded); the environment
 * variable MOE_B200_SINGLE_LAUNCH=0 selects two launches instead (same
 * results bit for bit; see moe_single_launch_ffn).
 *   x              [T, H] bf16.
 *   gate_up_w      [E, H, 2D] bf16 (StackedMoE gate_up_proj layout).
 *   gate_up_b      [E, 2D] bf16 or NULL (per has_bias).
 *   down_w         [E, D, H] bf16 (StackedMoE down_proj layout).
 *   down_b         [E, H] bf16 or NULL (per has_bias).
 *   expert_offsets [E+1], permutation [R]: as produced by moe_create_indices.
 *   expert_weights [T, k] fp32 routing weights (slot order).
 *   out            [T, H] bf16, fully overwritten.
 * Numerics: bf16 operands, fp32 accumulation, fp32 epilogues; h and the
 * per-slot expert outputs are rounded to bf16; the k-way sum is in fp32 in
 * slot order j = 0..k-1 (deterministic). */
moe_status_t moe_grouped_ffn(const moe_config_t* cfg, const void* x, const void* gate_up_w,
                             const void* gate_up_b, const void* down_w, const void* down_b,
                             const int32_t* expert_offsets, const int32_t* permutation,
                             const float* expert_weights, void* out, void* workspace,
                             size_t workspace_bytes, moe_stream_t stream);

/* The whole layer: moe_route -> moe_create_indices -> moe_grouped_ffn, with
 * the routing kept in the workspace.  expert_indices_out [T,k],
 * expert_weights_out [T,k] and sink_weights_out [T,S] are optional copies of
 * the routing (NULL = not returned; sink_weights_out is written only when
 * S > 0).  Seven kernel launches (four when T*k <= 2048 and E <= 512: the
 * router and the CSR build then share one single-CTA kernel; one more each
 * with MOE_B200_SINGLE_LAUNCH=0), no host
 * synchronisation, no allocation, so the call can be captured in a CUDA
 * graph. */
moe_status_t moe_forward(const moe_config_t* cfg, const void* x, const void* logits,
                         const float* expert_bias, const float* global_scale, const void* gate_up_w,
                         const void* gate_up_b, const void* down_w, const void* down_b, void* out,
                         int32_t* expert_indices_out, float* expert_weights_out, float* sink_weights_out,
                         void* workspace, size_t workspace_bytes, moe_stream_t stream);

/* moe_forward that also records stage_events[0..MOE_NUM_STAGE_EVENTS-1]
 * (cudaEvent_t handles created by the caller) on `stream` before router,
 * CSR count, CSR scan, CSR scatter, gather, gate_up GEMM, down GEMM and
 * combine, and after the combine, so a caller can time each kernel on the
 * stream it runs on.  With the single-launch FFN the "gate_up GEMM" stage
 * is the fused launch and the "down GEMM" stage is empty.  A NULL entry of
 * the array is skipped (so a caller can time one stage alone); a NULL array
 * is MOE_ERR_INVALID_ARGUMENT.  Under stream capture the events become
 * external event-record nodes, so each replay of the graph records them. */
/* *enabled = 1 if moe_grouped_ffn / moe_forward / moe_forward_ex called now
 * in this process run the two GEMMs as one launch, 0 if as two (the
 * MOE_B200_SINGLE_LAUNCH setting, read at each call). */
moe_status_t moe_single_launch_ffn(int32_t* enabled);

moe_status_t moe_forward_timed(const moe_config_t* cfg, const void* x, const void* logits,
                               const float* expert_bias, const float* global_scale, const void* gate_up_w,
                               const void* gate_up_b, const void* down_w, const void* down_b, void* out,
                               int32_t* expert_indices_out, float* expert_weights_out,
                               float* sink_weights_out, void* workspace, size_t workspace_bytes,
                               moe_stream_t stream, void* const* stage_events);

/* Copies the workspace's device status word to *device_status (a bitwise OR
 * of MOE_DEVICE_ERR_* since the last call that reset it), synchronizing
 * `stream`.  moe_forward resets the word in its first kernel;
 * moe_create_indices and moe_grouped_ffn reset it before their first kernel.
 * Returns MOE_ERR_DEVICE_TIMEOUT if a timeout bit is set, MOE_OK otherwise
 * (other bits are reported through *device_status only). */
moe_status_t moe_device_status(const void* workspace, int32_t* device_status, moe_stream_t stream);

/* Extensions of the layer beyond the core path (moe_forward_ex).  A zeroed
 * struct (or a NULL pointer) means none of them.
 *   token_mask     [T] uint8 or NULL (NeMo GroupedExperts.forward token_mask):
 *                  a token whose byte is 0 is still routed (its routing is
 *                  returned) but goes through no expert and its output row
 *                  is zero.
 *   apply_router_weight_first  0 or 1 (StackedMoE apply_router_weight_first):
 *                  1 scales each routed copy of x by its routing weight
 *                  before the expert (rounded to bf16), so the expert's down
 *                  bias is not weighted; 0 weights the expert's output.
 *   num_shared, shared_dim, shared_*  (StackedMoE has_shared_experts,
 *                  shared_experts_dim): num_shared dense experts that every
 *                  token goes through, weights laid out like the routed ones:
 *                  shared_gate_up_w [Ns, H, 2*Ds], shared_down_w [Ns, Ds, H],
 *                  biases [Ns, 2*Ds] / [Ns, H] per has_bias (same gate/up
 *                  format and activation as the routed experts).  With the
 *                  sink router their gates are the sink weights (the sink
 *                  lanes are gated shared experts, so num_shared must equal
 *                  num_sink); with the softmax router their gate is 1.
 *                  shared_dim must be a multiple of 8. */
typedef struct {
  const uint8_t* token_mask;
  int32_t apply_router_weight_first;
  int32_t num_shared;
  int32_t shared_dim;
  const void* shared_gate_up_w;
  const void* shared_gate_up_b;
  const void* shared_down_w;
  const void* shared_down_b;
} moe_extras_t;

/* Events moe_forward_ex() records when given stage_events: router, CSR
 * count, scan, scatter, gather, gate_up GEMM, down GEMM, shared index,
 * shared gather, shared gate_up GEMM, shared down GEMM, combine, end.
 * Stages that do not run record back to back. */
#define MOE_NUM_STAGE_EVENTS_EX 13

/* Workspace for moe_forward_ex with these extensions (adds, with shared
 * experts, the [T*Ns] slot CSR, Xp_s/Y_s [T*Ns, H] and h_s [T*Ns, Ds]). */
moe_status_t moe_workspace_size_ex(const moe_config_t* cfg, const moe_extras_t* extras, size_t* bytes);

/* moe_forward with the extensions above.  Same arguments and conventions as
 * moe_forward, plus `extras` (NULL = none) and stage_events (NULL, or
 * MOE_NUM_STAGE_EVENTS_EX caller-created cudaEvent_t, NULL entries skipped).  The output is
 *   out[t] = mask[t] * ( sum_j  w_tj * FFN_e(tj)(x_t)          (or FFN(w_tj x_t))
 *                      + sum_i  g_ti * SharedFFN_i(x_t) )      (or SharedFFN_i(g_ti x_t))
 * summed in fp32 (routed slots j ascending, then shared i ascending). */
moe_status_t moe_forward_ex(const moe_config_t* cfg, const moe_extras_t* extras, const void* x, const void* logits,
                            const float* expert_bias, const float* global_scale, const void* gate_up_w,
                            const void* gate_up_b, const void* down_w, const void* down_b, void* out,
                            int32_t* expert_indices_out, float* expert_weights_out, float* sink_weights_out,
                            void* workspace, size_t workspace_bytes, moe_stream_t stream, void* const* stage_events);

/* moe_create_indices without a workspace.  This entry point has no
 * counterpart on the documentation pages; it exists for callers that cannot
 * allocate device memory at the point where they build the routing: code
 * embedded in a host runtime that owns all device memory through its own pool
 * (for instance a serving engine that reserves almost all of HBM for its
 * caches and gives plugins no allocator), and latency-critical paths where
 * the implicit synchronisation of cudaMalloc/cudaFree is not acceptable.
 *
 * It computes exactly what moe_create_indices computes (same arguments
 * without workspace/workspace_bytes), with its scratch -- the device status
 * word and the per-chunk histogram and base tables -- in one file-scope
 * device array of 524,544 bytes that every GPU loading this library holds
 * until the process exits.  Capacity: ceil(T*k / 2048) * E <= 65,536 (for
 * example up to 1,048,576 routed slots with E = 128); larger problems get
 * MOE_ERR_WORKSPACE_TOO_SMALL before anything is enqueued.  The call itself
 * allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *
 * The first call on each device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current) and caches it for the
 * life of the process.  Under lazy module loading (CUDA_MODULE_LOADING=LAZY,
 * the default) that lookup also loads the library module that holds the
 * array, which places the 524,544 bytes in device memory and may
 * synchronize the device: make the first call on each device once at
 * initialisation, outside any stream capture and off the latency-critical
 * path; later calls allocate and synchronize nothing.  The cached address
 * belongs to the device's current primary context: after cudaDeviceReset
 * (or anything else that destroys that context) it is stale, so no call may
 * follow a context reset in the same process.  Every call shares the one array, which keeps
 * the last call's contents (the status word is cleared at the start of each
 * call, the tables are rewritten): calls that overlap on the GPU -- on two
 * streams, or from two threads -- race and give undefined results.  Device
 * fault bits (MOE_DEVICE_ERR_EXPERT_INDEX) land in the array's status word,
 * which no entry point reads back; out-of-range indices are skipped as in
 * moe_create_indices. */
moe_status_t moe_create_indices_noalloc(const moe_config_t* cfg, const int32_t* expert_indices,
                                        int32_t* expert_offsets, int32_t* permutation, int32_t* inverse,
                                        moe_stream_t stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* MOE_B200_MOE_H_ */
