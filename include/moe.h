/*
 * moe.h -- C ABI of libmoe.so: a capacity-limited top-k sparse
 * mixture-of-experts layer for NVIDIA B200 (sm_100a).
 *
 * Sources of the operations (page title, then section):
 *   [P1] "Sparse MoE Layer in NumPy -- Token Drop, Exact Dispatch/Combine,
 *        Aux Loss & Backward": sections 1 (root causes), 2 (implementation),
 *        4 (usage).
 *   [P2] "Top-k MoE Router with Load Statistics": problem statement,
 *        Requirements, Constraints.
 *   [P3] "Module 7. Mixture of Experts": route_logits, expert_capacity,
 *        dispatch_with_capacity, switch_auxiliary_loss, swiglu_expert,
 *        EducationalMoE.
 *   [P4] "32. Sparse MoE Token Dispatch & Combine (Capacity-Limited)":
 *        Problem, Step-by-Step Approach.
 *   [P5] "mixture-of-experts/3": Expert, TopKMoE, _load_balancing_loss.
 *
 * General conventions (apply to every entry point):
 *   - Pointers marked "device" must point to memory of the current CUDA
 *     device; pointers marked "host" to host memory.  The caller owns every
 *     buffer.  The library never allocates device memory: scratch space is
 *     a caller-provided device workspace whose minimum size is returned by
 *     the matching *_workspace_size function.
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t; NULL
 *     is the legacy default stream).  No entry point synchronises, except
 *     moe_read_status.
 *   - Matrices are row-major.  "Row stride" arguments (ld*) count elements.
 *     bf16 operands that feed the tensor-core path need 16-byte aligned
 *     base pointers and row strides that are multiples of 8 elements.
 *   - Inputs are never modified ([P2] Requirements).
 *   - Return value: MOE_OK, or an error from moe_status for a problem
 *     detected on the host before anything was enqueued (nothing is
 *     enqueued then).  Problems that depend on device data (an expert index
 *     outside [0,E), a non-finite logit, a wait that exceeded its time
 *     limit) are written by the kernels into the device status word
 *     `dev_status` (may be NULL to ignore them): the first error wins, the
 *     word is never reset by a kernel.  Clear it with moe_clear_status and
 *     read it with moe_read_status.
 *   - Expert weights use the (out, in) layout of nn.Linear ([P5] Expert):
 *     a matrix that maps K_in features to N_out features is stored
 *     (N_out, K_in), one such matrix per expert, experts outermost.  The
 *     pages' x @ W matrices (E, K_in, N_out) ([P1] section 2, [P3]
 *     EducationalMoE, [P4]) are the transposes; moe_transpose_weights
 *     converts them once.
 */
#ifndef MOE_H_
#define MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

typedef struct CUstream_st* moe_stream_t; /* identical to cudaStream_t */
typedef struct CUevent_st* moe_event_t;   /* identical to cudaEvent_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1, /* bad size, NULL pointer, k outside [1,E], capacity_factor <= 0 */
    MOE_ERR_UNSUPPORTED = 2, /* valid per the pages but outside this build's limits */
    MOE_ERR_CUDA = 3,        /* a CUDA runtime or driver call failed */
    MOE_ERR_BAD_INDEX = 4,   /* device: an expert index outside [0, E) */
    MOE_ERR_NONFINITE = 5,   /* device: a non-finite router logit */
    MOE_ERR_TIMEOUT = 6,     /* device: a bounded wait gave up */
    MOE_ERR_WORKSPACE = 7    /* workspace NULL or smaller than required */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* What the combine adds the gated expert outputs to ([P1] section 1 item 4:
 * the input row; [P2]: the shared output; [P4]/[P5]: nothing). */
typedef enum { MOE_BASE_ZERO = 0, MOE_BASE_INPUT = 1, MOE_BASE_TENSOR = 2 } moe_base;

/* Expert function: [P1]/[P4] linear x @ W; [P5] fc2(gelu(fc1 x)) with
 * biases and exact (erf) GELU; [P3] swiglu_expert (silu(x Wg) * x Wu) Wd. */
typedef enum { MOE_FFN_LINEAR = 0, MOE_FFN_GELU_MLP = 1, MOE_FFN_SWIGLU = 2 } moe_ffn_kind;

/* Router weight layout: (D, E) as on [P2]; (E, D) as nn.Linear in [P5]. */
typedef enum { MOE_ROUTER_DE = 0, MOE_ROUTER_ED = 1 } moe_router_layout;

/* Clean router scores ([P3] route_logits): softmax over the experts, or an
 * independent logistic sigmoid per expert. */
typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_scoring;

/* Static string for a moe_status value. */
MOE_API const char* moe_status_string(int status);

/* Library ABI version (major * 100 + minor). */
MOE_API int moe_version(void);

/*
 * moe_capacity -- per-expert capacity C = ceil(capacity_factor * T * k / E),
 * at least 1 ([P3] expert_capacity; [P1] section 1 item 2).  Evaluated in
 * IEEE double in the order capacity_factor * T * k / E.
 *   T, k, E  : tokens, experts per token, experts; T >= 1, 1 <= k <= E.
 *   capacity_factor : finite and > 0, else MOE_ERR_INVALID_ARG ([P3]
 *              rejects a zero factor).
 *   C_out    : host; receives C.
 * A caller that wants C = 0 (every assignment dropped, [P1] section 3 edge
 * checks) passes C = 0 directly to moe_dispatch.
 */
MOE_API int moe_capacity(int64_t T, int32_t k, int32_t E, double capacity_factor, int64_t* C_out);

/*
 * moe_route -- router scores, softmax, stable top-k, renormalised gates,
 * pre-drop counts and probability sums for T tokens.
 *
 * Computes, per token t ([P2] problem statement; [P1] section 2
 * top_k_gating; [P3] route_logits, stable_softmax, _deterministic_top_k;
 * [P5] TopKMoE.forward):
 *   s[t,e]   = x_t . w_e (+ logit_bias[e])    (fp32 accumulation)
 *   p[t,:]   = softmax(s[t,:]) in fp32, maximum subtracted first
 *   selected = the k experts with the largest s, in descending order, an
 *              exact tie going to the lower expert index
 *   gate_j   = exp(s_j - s_max) / sum_r exp(s_r - s_max) over the selected
 *              experts (= p_j / sum_r p_r)
 *   counts[e]   = #{(t,j) : selected[t,j] = e}      (before any drop)
 *   prob_sum[e] = sum_t p[t,e]                      (fixed-order reduction)
 *
 * Arguments:
 *   x          device; (T, D) activations with row stride ldx, dtype `dtype`.
 *              If w_router is NULL, x instead holds the (T, E) router logits
 *              (row stride ldx, dtype `dtype`) and D is ignored.
 *   w_router   device or NULL; router weight in `layout`, dtype `dtype`.
 *              bf16 scores are computed on the tensor cores (fp32
 *              accumulate); fp32 scores on the tensor cores as split-tf32
 *              products (fp32 accuracy).
 *   logit_bias device fp32 (E) or NULL.
 *   k          1 <= k <= E; this build requires k <= 64 and E <= 1024.
 *   logits_out device fp32 (T, E) or NULL; receives s.
 *   selected   device int64 (T, k).
 *   gates      device (T, k) in `dtype` or NULL ([P2]: results in x's dtype).
 *   gates_f32  device fp32 (T, k) or NULL.
 *   counts     device int32 (E).
 *   prob_sum   device fp32 (E).
 *   dev_status device int32 or NULL: MOE_ERR_NONFINITE if a logit is not
 *              finite (that token's outputs are then unspecified, [P3]
 *              rejects such input).
 *   workspace  device, >= moe_route_workspace_size(...) bytes.
 */
MOE_API size_t moe_route_workspace_size(int64_t T, int64_t D, int32_t E, moe_dtype dtype,
                                int has_router_weight, moe_router_layout layout);
MOE_API int moe_route(const void* x, moe_dtype dtype, int64_t T, int64_t D, int64_t ldx,
              const void* w_router, moe_router_layout layout, int32_t E, const float* logit_bias,
              int32_t k, float* logits_out, int64_t* selected, void* gates, float* gates_f32,
              int32_t* counts, float* prob_sum, int32_t* dev_status, void* workspace,
              size_t workspace_bytes, moe_stream_t stream);

/*
 * moe_route_ex -- moe_route with the router variants of [P3] route_logits.
 *   scoring        MOE_SCORE_SOFTMAX: clean scores p = softmax(s); gates =
 *                  softmax of the selected logits (moe_route's behaviour).
 *                  MOE_SCORE_SIGMOID: clean scores sigmoid(s) per expert;
 *                  gates = the selected sigmoids divided by their sum,
 *                  computed as a softmax of log-sigmoids so that it stays
 *                  finite when every sigmoid underflows.
 *   selection_bias device fp32 (E) or NULL.  When given, the top-k ranks the
 *                  clean score plus this bias (the bias moves the selection
 *                  only; gates still come from the clean scores); otherwise the
 *                  ranking uses the logits themselves.  Ties -> lower index.
 *                  The ranking is decided in fp32.
 *   prob_sum[e]    sum over tokens of the clean score of expert e.
 *   z_loss         device fp32 (1) or NULL: the router z-loss
 *                  mean_t logsumexp(s_t)^2 ([P3] router_z_loss), fixed-order.
 * Other arguments as moe_route; the workspace size is the same.
 */
MOE_API int moe_route_ex(const void* x, moe_dtype dtype, int64_t T, int64_t D, int64_t ldx,
                         const void* w_router, moe_router_layout layout, int32_t E,
                         const float* logit_bias, int32_t k, moe_scoring scoring,
                         const float* selection_bias, float* logits_out, int64_t* selected,
                         void* gates, float* gates_f32, int32_t* counts, float* prob_sum,
                         float* z_loss, int32_t* dev_status, void* workspace,
                         size_t workspace_bytes, moe_stream_t stream);

/*
 * moe_router_backward -- gradients of the router scores s = x W (+ b) for a
 * given dL/ds (dlogits, e.g. from moe_backward or moe_backward_swiglu):
 *   dx_router[t,d] = sum_e dlogits[t,e] W(e,d)           fp32 (T, D)
 *   dw_router      = x^T dlogits in w_router's layout     fp32 ((E,D) or (D,E))
 *   db_router[e]   = sum_t dlogits[t,e]                   fp32 (E), fixed order
 * ([P2] s = x . w_e is linear in x, w and b.)  The layer's full input
 * gradient is the expert backward's dx plus dx_router.  Both products run on
 * the tensor cores with fp32 accuracy: for bf16 x and w with E and D multiples
 * of 64, dlogits is split into three bf16 parts (24 mantissa bits; each
 * product with a bf16 x or w is exact in the fp32 accumulator) and bf16 GEMMs
 * take them; otherwise as split-tf32.  Any of the three outputs may be NULL to
 * skip it.
 *   x          device (T, D), row stride ldx, dtype `dtype`.
 *   w_router   device, layout `layout`, dtype `dtype`.
 *   dlogits    device fp32 (T, E).
 *   workspace  device, >= moe_router_backward_workspace_size(T, D, E, dtype, layout).
 */
MOE_API size_t moe_router_backward_workspace_size(int64_t T, int64_t D, int32_t E, moe_dtype dtype,
                                                  moe_router_layout layout);
MOE_API int moe_router_backward(moe_dtype dtype, const void* x, int64_t T, int64_t D, int64_t ldx,
                                const void* w_router, moe_router_layout layout, int32_t E, const float* dlogits,
                                float* dx_router, float* dw_router, float* db_router, int32_t* dev_status,
                                void* workspace, size_t workspace_bytes, moe_stream_t stream);

/*
 * moe_renormalize_kept_gates -- [P3] dispatch_with_capacity with
 * renormalize_kept_gates: out[t,j] = gates[t,j] / sum of token t's kept gates
 * for kept assignments (slot[t,j] >= 0), 0 for dropped ones, and all zeros for
 * a token with nothing kept.  gates_f32, out: device fp32 (T, k); slot: device
 * int64 (T, k) from moe_dispatch.  The default layer keeps the pre-drop gates
 * ([P1] section 1 item 4); pass this output to moe_combine for the other policy.
 */
MOE_API int moe_renormalize_kept_gates(const float* gates_f32, const int64_t* slot, int64_t T,
                                       int32_t k, float* out, moe_stream_t stream);

/*
 * moe_dispatch -- greedy position-priority slot assignment and the gather
 * into expert-major buffers.
 *
 * Over the assignment stream ordered by token t ascending, then route slot
 * j ascending (selection order = descending gate), an assignment (t,j) to
 * expert e is kept iff fewer than C earlier assignments to e were kept
 * ([P1] section 2 position_priority_dispatch; [P3] dispatch_with_capacity;
 * [P4] step 2, the exclusive running count).  Computed as a single-pass
 * per-expert prefix count with decoupled look-back; the result is unique.
 *   slot[t,j]          rank of (t,j) among e's kept rows, -1 if dropped
 *   kept[t,j]          1 kept / 0 dropped
 *   used[e]            min(count_e, C)
 *   overflow[e]        count_e - used[e] ([P1] section 1 item 3)
 *   drops_per_token[t] dropped assignments of token t ([P1] section 4)
 *   token_of_slot[e,c] token in slot c of expert e, -1 for c >= used[e]
 *   xbuf[e,c,:]        = x[token_of_slot[e,c], :] for c < used[e]
 *                      ([P4] step 5 gather); rows c >= used[e] untouched.
 *
 * Arguments:
 *   selected  device int64 (T, k) expert indices (from moe_route, or given
 *             as in [P4]); an index outside [0, E) sets MOE_ERR_BAD_INDEX
 *             in dev_status and is treated as dropped.
 *   T, k, E, C : T >= 1, 1 <= k <= 64, 1 <= E <= 2048, C >= 0; T * k < 2^30.
 *   x         device (T, D) row stride ldx, dtype `dtype`, or NULL to skip
 *             the gather (then xbuf is ignored).
 *   xbuf      device (E, C, D) contiguous, dtype `dtype`.
 *   slot, kept, used, overflow, drops_per_token, token_of_slot : device
 *             outputs as above (int64, uint8, int32, int32, int32, int32).
 *   workspace device, >= moe_dispatch_workspace_size(T, k, E) bytes.
 */
MOE_API size_t moe_dispatch_workspace_size(int64_t T, int32_t k, int32_t E);
MOE_API int moe_dispatch(const int64_t* selected, int64_t T, int32_t k, int32_t E, int64_t C,
                 const void* x, moe_dtype dtype, int64_t D, int64_t ldx, int64_t* slot,
                 uint8_t* kept, int32_t* used, int32_t* overflow, int32_t* drops_per_token,
                 int32_t* token_of_slot, void* xbuf, int32_t* dev_status, void* workspace,
                 size_t workspace_bytes, moe_stream_t stream);

/*
 * moe_dispatch_static -- moe_dispatch for callers that cannot allocate device
 * memory.  The pages have no counterpart: this is an interface variant of
 * moe_dispatch with the same results, not a different computation.
 *
 * Who needs it: code that a host framework calls with nothing but input and
 * output pointers (a plugin or custom-operator interface that manages the
 * device memory budget itself) may not call cudaMalloc or cudaFree, which
 * would synchronise the device and bypass that budget, so it cannot provide
 * the workspace that moe_dispatch asks for.
 *
 * This entry point takes no workspace.  The slot scan's look-back state lives
 * in one fixed file-scope device array of moe_dispatch_static_max_state_bytes()
 * bytes (4 MiB) that every GPU which loads the library holds until the process
 * exits.  The call allocates nothing: no cudaMalloc, cudaFree or allocating
 * library routine.
 *
 * Arguments and outputs: as moe_dispatch, without workspace/workspace_bytes.
 * Limit: ceil(T/128) * E * 4 + 4 bytes of state, rounded up to 256, must fit in
 * the array (E = 256 allows T <= 524160); a larger problem returns
 * MOE_ERR_UNSUPPORTED and enqueues nothing.
 * Set-up: the first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and keeps it for the life
 * of the process; make that first call before any stream capture.  A device
 * reset (cudaDeviceReset, or anything else that destroys the device's primary
 * context) makes the kept address stale: do not call this entry point on that
 * device after such a reset.
 * Sharing: all calls on a device use the same array; each call clears, in
 * stream order, the part it uses before the scan, so a later call never sees
 * an earlier call's state.  Calls that can overlap on the GPU (different
 * streams not ordered by events) race on the array and must not be issued.
 */
MOE_API size_t moe_dispatch_static_max_state_bytes(void);
MOE_API int moe_dispatch_static(const int64_t* selected, int64_t T, int32_t k, int32_t E, int64_t C,
                                const void* x, moe_dtype dtype, int64_t D, int64_t ldx, int64_t* slot,
                                uint8_t* kept, int32_t* used, int32_t* overflow, int32_t* drops_per_token,
                                int32_t* token_of_slot, void* xbuf, int32_t* dev_status,
                                moe_stream_t stream);

/*
 * moe_expert_ffn -- every expert applied to its own rows of an expert-major
 * buffer (grouped GEMM over variable-occupancy experts).
 *
 * For each expert e and row c < rows(e) (rows(e) = used[e], or C when used
 * is NULL):  ybuf[e,c,:] = Expert_e(xbuf[e,c,:]) with
 *   LINEAR   : x W1_e^T                      W1 (E, Dout, D)       [P1], [P4]
 *   GELU_MLP : gelu(x W1_e^T + b1_e) W2_e^T + b2_e                  [P5]
 *              W1 (E, F, D), b1 (E, F), W2 (E, Dout, F), b2 (E, Dout)
 *   SWIGLU   : (silu(x W1_e^T) * (x W3_e^T)) W2_e^T                 [P3]
 *              W1 = gate (E, F, D), W3 = up (E, F, D), W2 = down (E, Dout, F)
 * bf16: tcgen05 tensor cores, fp32 accumulation, the intermediate
 * activation rounded to bf16, outputs bf16.  fp32: tcgen05 tensor cores on
 * split-tf32 operands (x = hi + lo, three tf32 products per term, fp32
 * accumulation), which keeps fp32 accuracy; the split operands live in the
 * workspace.
 * Rows c >= rows(e) of ybuf are not written.  With C = 0 nothing is read or
 * written (the buffer and weight pointers may then be NULL).  An always-on
 * shared expert ([P3] EducationalMoE) is this call with E = 1, C = T,
 * used = NULL and the token matrix as xbuf.
 *
 * Arguments:
 *   xbuf      device (E, C, D) contiguous, dtype `dtype`.
 *   used      device int32 (E) or NULL.
 *   w1,b1,w2,b2,w3 device, layouts above, dtype `dtype` (biases too);
 *             unused ones may be NULL.
 *   ybuf      device (E, C, Dout) contiguous, dtype `dtype`.
 *   workspace device, >= moe_expert_ffn_workspace_size(kind, dtype, E, C, D, F, Dout)
 *             bytes (0 for bf16 LINEAR; fp32 needs room for the split operands).
 */
MOE_API size_t moe_expert_ffn_workspace_size(moe_ffn_kind kind, moe_dtype dtype, int32_t E, int64_t C,
                                             int64_t D, int64_t F, int64_t Dout);
MOE_API int moe_expert_ffn(moe_ffn_kind kind, moe_dtype dtype, const void* xbuf, const int32_t* used,
                   int32_t E, int64_t C, int64_t D, int64_t F, int64_t Dout, const void* w1,
                   const void* b1, const void* w2, const void* b2, const void* w3, void* ybuf,
                   int32_t* dev_status, void* workspace, size_t workspace_bytes,
                   moe_stream_t stream);

/*
 * moe_expert_ffn_gathered -- moe_expert_ffn (SwiGLU, bf16) reading each
 * expert's rows straight from the token matrix through the dispatch's
 * inverse map, without the expert-major copy:
 *   ybuf[e,c,:] = Expert_e(x[token_of_slot[e,c], :])   for c < used[e]
 * which equals moe_dispatch's gather into xbuf followed by moe_expert_ffn
 * ([P4] steps 5 and 6 fused; [P3] swiglu_expert).  The gate/up kernel copies
 * the token rows into the tensor-core tiles itself, so the (E, C, D) buffer
 * is neither written nor read.
 *
 * Arguments:
 *   kind, dtype   MOE_FFN_SWIGLU and MOE_BF16 only (else MOE_ERR_UNSUPPORTED).
 *   x             device bf16 (T, D), row stride ldx (multiple of 8, 16-byte
 *                 aligned base); D a multiple of 8.
 *   token_of_slot device int32 (E, C) from moe_dispatch; an entry outside
 *                 [0, T) for c < used[e] sets MOE_ERR_BAD_INDEX and reads a zero row.
 *   used          device int32 (E) from moe_dispatch (required).
 *   w1 = gate (E, F, D), w3 = up (E, F, D), w2 = down (E, Dout, F), bf16.
 *   ybuf          device bf16 (E, C, Dout); rows c >= used[e] are not written.
 *   workspace     device, >= moe_expert_ffn_workspace_size(MOE_FFN_SWIGLU, MOE_BF16, E, C, D, F, Dout).
 */
MOE_API int moe_expert_ffn_gathered(moe_ffn_kind kind, moe_dtype dtype, const void* x, int64_t T, int64_t ldx,
                                    const int32_t* token_of_slot, const int32_t* used, int32_t E, int64_t C,
                                    int64_t D, int64_t F, int64_t Dout, const void* w1, const void* w2,
                                    const void* w3, void* ybuf, int32_t* dev_status, void* workspace,
                                    size_t workspace_bytes, moe_stream_t stream);

/*
 * moe_expert_ffn_save -- moe_expert_ffn for bf16 SwiGLU experts that also
 * keeps what the backward needs: saved_ab[e, c] = [a | b] with a = xbuf[e,c]
 * Wg_e^T and b = xbuf[e,c] Wu_e^T (the gate and up pre-activations, fp32
 * accumulation rounded to bf16), for c < used[e] (other rows are not
 * written).  Pass it to moe_backward_swiglu, which then skips recomputing
 * them.  ([P3] swiglu_expert; the usual store-for-backward trade of memory
 * for a GEMM.)
 *   xbuf bf16 (E, C, D); used int32 (E) (required); w_gate, w_up bf16 (E, F, D);
 *   w_down bf16 (E, Dout, F); ybuf bf16 (E, C, Dout); saved_ab bf16 (E, C, 2F).
 *   workspace >= moe_expert_ffn_workspace_size(MOE_FFN_SWIGLU, MOE_BF16, E, C, D, F, Dout).
 */
MOE_API int moe_expert_ffn_save(const void* xbuf, const int32_t* used, int32_t E, int64_t C, int64_t D, int64_t F,
                                int64_t Dout, const void* w_gate, const void* w_down, const void* w_up, void* ybuf,
                                void* saved_ab, int32_t* dev_status, void* workspace, size_t workspace_bytes,
                                moe_stream_t stream);

/*
 * moe_combine -- gate-weighted combine back to token order.
 *   y[t,:] = base[t,:] + sum_{j : slot[t,j] >= 0} gate[t,j] * ybuf[e_{t,j}, slot[t,j], :]
 * ([P1] section 1 item 4: y = x + sum over kept; [P2] y = shared + sum;
 * [P4] step 6 and [P5]: no base, a dropped token gives a zero row).  The
 * sum runs over j in ascending order in fp32 for every element, with no
 * atomics, so the result is deterministic.
 *
 * Arguments:
 *   ybuf      device (E, C, N) contiguous, dtype `dtype`.
 *   selected, slot : device int64 (T, k), as produced by moe_route / moe_dispatch.
 *   gates     device (T, k) of dtype `gate_dtype`, or NULL for all-ones.
 *   base_kind MOE_BASE_ZERO (base ignored), MOE_BASE_INPUT or MOE_BASE_TENSOR
 *             (base = device (T, N), row stride ldbase, dtype `dtype`).
 *   y         device (T, N) row stride ldy, dtype `dtype`.
 *   dev_status: MOE_ERR_BAD_INDEX for a kept assignment whose expert or slot
 *             lies outside (E, C); such a term is skipped.
 */
MOE_API int moe_combine(const void* ybuf, const int64_t* selected, const int64_t* slot, const void* gates,
                moe_dtype gate_dtype, int64_t T, int32_t k, int32_t E, int64_t C, int64_t N,
                moe_base base_kind, const void* base, int64_t ldbase, void* y, int64_t ldy,
                moe_dtype dtype, int32_t* dev_status, moe_stream_t stream);

/*
 * moe_aux_stats -- load statistics and the Switch auxiliary loss.
 *   f[e] = counts[e] / T                         ([P2] token_fraction, sums to k)
 *   P[e] = prob_sum[e] / T                       ([P2] probability_mass, sums to 1)
 *   aux[0] = E * sum_e (counts[e] / (T * kn)) * P[e]
 *            kn = k if normalize_by_k ([P1] section 1 item 6, [P3]
 *            switch_auxiliary_loss: 1 at uniform routing), else kn = 1 ([P5])
 *   aux[1] = aux_coef * aux[0]
 * f and P are written in `out_dtype`; aux in fp32.  Fixed-order reduction.
 * All pointers device: counts int32 (E), prob_sum fp32 (E), f (E), P (E),
 * aux fp32 (2).
 */
MOE_API int moe_aux_stats(const int32_t* counts, const float* prob_sum, int64_t T, int32_t E, int32_t k,
                  int normalize_by_k, float aux_coef, void* f, void* P, moe_dtype out_dtype,
                  float* aux, moe_stream_t stream);

/*
 * moe_swiglu_layer_forward -- the whole layer forward in one call: [P3]
 * EducationalMoE with SwiGLU routed experts and an optional always-on shared
 * SwiGLU expert, softmax router with a per-expert logit bias ([P2] problem
 * statement), capacity-limited greedy dispatch ([P1] section 2
 * position_priority_dispatch), gate-weighted combine onto the shared output
 * ([P2] y = shared + sum), and the load statistics with the Switch aux loss.
 * It runs moe_route, moe_dispatch, moe_expert_ffn (routed, and shared on the
 * side stream), moe_combine and moe_aux_stats on buffers carved from one
 * workspace; the results equal that sequence of calls exactly.
 *
 * Layer description (all weights device bf16, (out, in) layout):
 *   T, H          tokens and hidden size; E experts, k per token, C capacity
 *                 (moe_capacity; 0 drops everything), F / F_shared the routed
 *                 and shared intermediate sizes (F_shared = 0: no shared
 *                 expert, y = sum of the gated outputs).
 *   w_router (E, H); router_bias fp32 (E) or NULL; w_gate, w_up (E, F, H);
 *   w_down (E, H, F); s_gate, s_up (1, F_shared, H); s_down (1, H, F_shared).
 *   aux_coef      scales aux[1].
 *
 * Arguments:
 *   x     (T, H) bf16, contiguous: device memory, or host memory (pinned for
 *         an asynchronous copy) that the call copies into the workspace with
 *         one cudaMemcpyAsync on copy_in_stream.
 *   y     (T, H) bf16 output, device or host; a host y is copied back with one
 *         cudaMemcpyAsync on copy_out_stream after the layer.
 *   aux   fp32 (2): {aux loss, aux_coef * aux loss}, device or host, or NULL.
 *   dev_status   device status word or NULL (as for the calls above).
 *   workspace    device, >= moe_swiglu_layer_workspace_size(L) bytes.  It
 *         holds the device copies of x and y, every routing and dispatch
 *         output and the expert buffers; the call owns it until it is done.
 *   stream       the layer's kernels; side_stream (or NULL: stream) the
 *         shared expert; copy_in_stream / copy_out_stream (or NULL: stream)
 *         the host copies.
 *   x_free, y_free  cudaEvent_t handles or NULL, one pair per workspace.
 *         x_free: the call waits for it before its first use of the workspace
 *         (the copy-in of a host x, else the first kernel) and records it on
 *         `stream` after its last kernel.  y_free: before writing the y
 *         staging of a host y the call waits for it, and records it after the
 *         copy-out.  With two workspaces used in turn, each with its own pair,
 *         one batch's copy-in, the previous batch's copy-out and the kernels
 *         in between overlap.  When x_free is NULL, a host copy-in waits for
 *         all work already on `stream`.
 * Results: with host outputs, y and aux are complete when copy_out_stream
 * (or `stream`) reaches the end of the call's work; synchronise it (or the
 * event) before reading them.  Returns MOE_ERR_WORKSPACE / _INVALID_ARG /
 * _UNSUPPORTED / _CUDA for host-detected problems, nothing enqueued then
 * except possibly the copy-in.
 */
typedef struct moe_swiglu_layer {
    int64_t T, H, F, F_shared, C;
    int32_t E, k;
    float aux_coef;
    const void* w_router;
    const float* router_bias;
    const void* w_gate;
    const void* w_up;
    const void* w_down;
    const void* s_gate;
    const void* s_up;
    const void* s_down;
} moe_swiglu_layer;

MOE_API size_t moe_swiglu_layer_workspace_size(const moe_swiglu_layer* L);
MOE_API int moe_swiglu_layer_forward(const moe_swiglu_layer* L, const void* x, void* y, float* aux,
                                     int32_t* dev_status, void* workspace, size_t workspace_bytes,
                                     moe_stream_t stream, moe_stream_t side_stream, moe_stream_t copy_in_stream,
                                     moe_stream_t copy_out_stream, moe_event_t x_free, moe_event_t y_free);

/*
 * moe_backward -- backward of the linear-expert layer, the kept mask and the
 * drops held constant ([P1] section 1 item 7 and section 2 moe_backward).
 * fp32 linear experts (kind MOE_FFN_LINEAR, dtype MOE_F32); the bf16 SwiGLU
 * experts have moe_backward_swiglu.
 *
 * With out_{t,j} = x_t W_e^T (e = selected[t,j], kept) and the loss
 * L = sum_t dy_t . y_t + aux_coef * aux:
 *   dgate[t,j]    = kept ? dy_t . out_{t,j} : 0
 *   dlogits[t,i]  = gate_i (dgate_i - sum_j gate_j dgate_j) on the selected
 *                   experts, 0 elsewhere (gate = softmax of the selected
 *                   logits), plus, when aux_coef != 0,
 *                   aux_coef * E / (T*T*kn) * p[t,e] * (counts[e] - sum_e' counts[e'] p[t,e'])
 *   dW[e]         = sum_{kept (t,j) -> e} gate * dy_t^T x_t      (E, Dout, D)
 *   dx[t]         = [dy_t] + sum_{kept j} gate_j dy_t W_e        (T, D)
 * The residual term [dy_t] needs Dout == D.
 *
 * Arguments (device unless noted):
 *   dy (T, Dout), x (T, D), logits fp32 (T, E), selected int64 (T, k),
 *   gates fp32 (T, k), slot int64 (T, k), used int32 (E),
 *   token_of_slot int32 (E, C), xbuf (E, C, D) and ybuf (E, C, Dout) from
 *   the forward (ybuf = ungated expert outputs), W (E, Dout, D),
 *   counts int32 (E) (read only when aux_coef != 0).
 *   Outputs dx (T, D), dW (E, Dout, D), dlogits fp32 (T, E), dgate fp32 (T, k).
 *   workspace >= moe_backward_workspace_size(...) bytes.
 */
MOE_API size_t moe_backward_workspace_size(int32_t E, int64_t C, int64_t D, int64_t Dout);
MOE_API int moe_backward(moe_ffn_kind kind, moe_dtype dtype, const void* dy, const void* x,
                 const float* logits, const int64_t* selected, const float* gates,
                 const int64_t* slot, const int32_t* used, const int32_t* token_of_slot,
                 const void* xbuf, const void* ybuf, const void* W, int64_t T, int32_t k,
                 int32_t E, int64_t C, int64_t D, int64_t Dout, int use_residual, float aux_coef,
                 int normalize_by_k, const int32_t* counts, void* dx, void* dW, float* dlogits,
                 float* dgate, int32_t* dev_status, void* workspace, size_t workspace_bytes,
                 moe_stream_t stream);

/*
 * moe_backward_swiglu -- backward of the SwiGLU-expert layer ([P3]
 * swiglu_expert, [P3] EducationalMoE routed experts) under the same rules as
 * moe_backward: kept mask and drops constant, gates = softmax of the selected
 * logits.  bf16 activations and weights, fp32 accumulation; weight gradients
 * in fp32.  For a kept (t,j) -> e with a = x_t Wg_e^T, b = x_t Wu_e^T,
 * h = silu(a) * b, o = h Wd_e^T:
 *   dgate[t,j] = dy_t . o        (o read from the forward's ybuf)
 *   dlogits    as in moe_backward
 *   do = gate dy_t,  dh = do Wd_e,  s = sigmoid(a),
 *   da = dh * b * s * (1 + a (1 - s)),  db = dh * a * s
 *   dw_down[e] += do^T h         (E, H, F)
 *   dw_gate[e] += da^T x_t       (E, F, H)
 *   dw_up[e]   += db^T x_t       (E, F, H)
 *   dx[t]      = [dy_t] + sum_kept (da Wg_e + db Wu_e)     (T, H), bf16
 * a and b are recomputed from xbuf (fp32), or read from saved_ab when the
 * forward ran moe_expert_ffn_save (bf16, which saves that GEMM); h, da, db are
 * rounded to bf16 before the weight-gradient and dx products.
 *
 * Arguments (device): dy bf16 (T, H); logits fp32 (T, E); selected int64,
 *   gates fp32, slot int64 (T, k); used int32 (E); xbuf bf16 (E, C, H) and
 *   ybuf bf16 (E, C, H) from the forward; saved_ab bf16 (E, C, 2F) from
 *   moe_expert_ffn_save, or NULL; w_gate, w_up bf16 (E, F, H);
 *   w_down bf16 (E, H, F); counts int32 (E) when aux_coef != 0.
 *   H and F multiples of 8, k <= 64, dtype MOE_BF16 (else MOE_ERR_UNSUPPORTED).
 *   Outputs: dx bf16 (T, H); dw_gate, dw_up fp32 (E, F, H); dw_down fp32
 *   (E, H, F); dlogits fp32 (T, E); dgate fp32 (T, k).
 *   workspace >= moe_backward_swiglu_workspace_size(E, C, H, F) bytes.
 */
MOE_API size_t moe_backward_swiglu_workspace_size(int32_t E, int64_t C, int64_t H, int64_t F);
MOE_API int moe_backward_swiglu(moe_dtype dtype, const void* dy, const float* logits, const int64_t* selected,
                                const float* gates, const int64_t* slot, const int32_t* used, const void* xbuf,
                                const void* ybuf, const void* saved_ab, const void* w_gate, const void* w_up, const void* w_down,
                                int64_t T, int32_t k, int32_t E, int64_t C, int64_t H, int64_t F, int use_residual,
                                float aux_coef, int normalize_by_k, const int32_t* counts, void* dx,
                                float* dw_gate, float* dw_up, float* dw_down, float* dlogits, float* dgate,
                                int32_t* dev_status, void* workspace, size_t workspace_bytes,
                                moe_stream_t stream);

/*
 * moe_backward_gelu -- backward of the GELU-MLP-expert layer ([P5] Expert:
 * fc2(gelu(fc1(x))) with biases, exact erf GELU) under the same rules as
 * moe_backward: kept mask and drops constant, gates = softmax of the
 * selected logits.  fp32 throughout; the products run on the tensor cores as
 * split-tf32 (fp32 accuracy).  For a kept (t,j) -> e with
 * z = x_t W1_e^T + b1_e, h = gelu(z), o = h W2_e^T + b2_e:
 *   dgate[t,j] = dy_t . o        (o read from the forward's ybuf)
 *   dlogits    as in moe_backward
 *   do = gate dy_t,  dh = do W2_e,  dz = dh * gelu'(z),
 *   gelu'(z) = Phi(z) + z phi(z)  (standard normal CDF and density)
 *   dw2[e] += do^T h   (E, Dout, F)     db2[e] += do   (E, Dout)
 *   dw1[e] += dz^T x_t (E, F, D)        db1[e] += dz   (E, F)
 *   dx[t]   = [dy_t] + sum_kept dz W1_e                 (T, D)
 * z is recomputed from xbuf.  Bias gradients are summed over the kept rows
 * of each expert in slot order.
 *
 * Arguments (device): dy (T, Dout); logits fp32 (T, E); selected int64,
 *   gates fp32, slot int64 (T, k); used int32 (E); xbuf (E, C, D) and ybuf
 *   (E, C, Dout) from the forward; w1 (E, F, D), b1 (E, F), w2 (E, Dout, F)
 *   as for moe_expert_ffn (b2 does not enter the gradients); counts int32
 *   (E) when aux_coef != 0.  dtype MOE_F32 (else MOE_ERR_UNSUPPORTED), k <= 64.
 *   The residual term [dy_t] needs Dout == D.
 *   Outputs: dx (T, D); dw1 (E, F, D); db1 (E, F); dw2 (E, Dout, F);
 *   db2 (E, Dout); dlogits fp32 (T, E); dgate fp32 (T, k).
 *   workspace >= moe_backward_gelu_workspace_size(E, C, D, F, Dout) bytes.
 */
MOE_API size_t moe_backward_gelu_workspace_size(int32_t E, int64_t C, int64_t D, int64_t F, int64_t Dout);
MOE_API int moe_backward_gelu(moe_dtype dtype, const void* dy, const float* logits, const int64_t* selected,
                              const float* gates, const int64_t* slot, const int32_t* used, const void* xbuf,
                              const void* ybuf, const void* w1, const void* b1, const void* w2, int64_t T,
                              int32_t k, int32_t E, int64_t C, int64_t D, int64_t F, int64_t Dout,
                              int use_residual, float aux_coef, int normalize_by_k, const int32_t* counts,
                              void* dx, float* dw1, float* db1, float* dw2, float* db2, float* dlogits,
                              float* dgate, int32_t* dev_status, void* workspace, size_t workspace_bytes,
                              moe_stream_t stream);

/*
 * Expert parallelism over R ranks (one process per GPU).  Rank r holds T_r
 * tokens and experts [r E/R, (r+1) E/R) with their weights.  The layer over
 * the R ranks equals the layer over the whole batch with the tokens in rank
 * order: expert e keeps at most C assignments, C = ceil(cf * T * k / E) for
 * the global T, which is also ceil(cf * T_r * k / (E/R)) when every rank has
 * T_r = T / R tokens ([P1] section 1 item 2: the capacity does not change
 * with the expert-parallel world size).  Greedy position priority across
 * ranks: rank r's assignments to expert e take the slots after those of
 * ranks 0..r-1.  [P3]'s expert-parallel payload (T k D values each way) is
 * moved by moe_ep_dispatch and moe_ep_combine themselves, reading and
 * writing the other ranks' buffers through peer memory.
 *
 * One step on rank r:
 *   1. moe_route on the local tokens -> selected, gates, counts (E).
 *   2. gather every rank's counts into counts_all (R, E) (caller: e.g. an
 *      NCCL all-gather), then moe_ep_plan.
 *   3. moe_ep_dispatch: slots and rows into the owner ranks' xbuf.
 *   4. barrier (every rank's rows have landed).
 *   5. moe_expert_ffn on the local (E/R, C, D) xbuf with used + r E/R.
 *   6. barrier (every expert output is written).
 *   7. moe_ep_combine from the owner ranks' ybuf.
 * Barrier 4 of the next step also orders this step's combine reads before
 * the next expert FFN overwrites ybuf.  The buffers of the other ranks are
 * mapped once with moe_ipc_export / moe_ipc_import.
 */

/*
 * moe_ep_plan -- from every rank's pre-drop counts, this rank's slot base per
 * expert and the global per-expert statistics.
 *   counts_all   device int32 (R, E): row q = rank q's counts from moe_route.
 *   rank_base    device int32 (E): sum_{q < rank} counts_all[q][e].
 *   used         device int32 (E) or NULL: min(sum_q counts_all[q][e], C).
 *   overflow     device int32 (E) or NULL: sum - used.
 *   counts_total device int32 (E) or NULL: sum_q counts_all[q][e] (the global
 *                counts for moe_aux_stats).
 * Sums saturate at 2^31 - 1.
 */
MOE_API int moe_ep_plan(const int32_t* counts_all, int32_t R, int32_t rank, int32_t E, int64_t C,
                        int32_t* rank_base, int32_t* used, int32_t* overflow, int32_t* counts_total,
                        moe_stream_t stream);

/*
 * moe_ep_dispatch -- moe_dispatch for rank `rank` of an expert-parallel group:
 * slot[t,j] = rank_base[e] + #{earlier local assignments to e}, kept iff
 * slot < C; each kept row x[t] is written to row (e mod E/R) * C + slot of
 * the expert-major buffer of rank e / (E/R).
 *   selected     device int64 (T, k) local assignments; rank_base from
 *                moe_ep_plan; token_base = global index of local token 0
 *                (recorded in token_of_slot).
 *   x            device (T, D), row stride ldx, dtype `dtype`; NULL skips the
 *                row movement.
 *   xbuf_ranks   HOST array of R device pointers: rank q's (E/R, C, D) buffer,
 *                as mapped into this process (this rank's own buffer at q =
 *                rank).  Rows are written with 16-byte vectors when every
 *                pointer and the row pitch allow it.
 *   slot (T, k) int64, kept (T, k) uint8, drops_per_token (T) int32: as
 *                moe_dispatch, with global slots.
 *   token_of_slot device int32 (E, C) or NULL: filled with -1, then
 *                token_base + t at the slots this rank's tokens hold.
 *   workspace    >= moe_dispatch_workspace_size(T, k, E) bytes.
 * E must be a multiple of R; R <= 64; E <= 2048, k <= 64.
 */
MOE_API int moe_ep_dispatch(const int64_t* selected, int64_t T, int32_t k, int32_t E, int64_t C,
                            const int32_t* rank_base, int64_t token_base, const void* x, moe_dtype dtype,
                            int64_t D, int64_t ldx, void* const* xbuf_ranks, int32_t R, int64_t* slot,
                            uint8_t* kept, int32_t* drops_per_token, int32_t* token_of_slot, int32_t* dev_status,
                            void* workspace, size_t workspace_bytes, moe_stream_t stream);

/*
 * moe_ep_combine -- moe_combine reading each kept row from the owner rank:
 *   y[t] = base[t] + sum_{j kept, ascending} gate[t,j] * ybuf_{e / (E/R)}[e mod E/R, slot[t,j]]
 *   ybuf_ranks   HOST array of R device pointers to every rank's (E/R, C, N)
 *                expert output buffer, as mapped into this process.
 * Other arguments and the status word as moe_combine (E is the global
 * expert count, a multiple of R).
 */
MOE_API int moe_ep_combine(const void* const* ybuf_ranks, int32_t R, const int64_t* selected, const int64_t* slot,
                           const void* gates, moe_dtype gate_dtype, int64_t T, int32_t k, int32_t E, int64_t C,
                           int64_t N, moe_base base_kind, const void* base, int64_t ldbase, void* y, int64_t ldy,
                           moe_dtype dtype, int32_t* dev_status, moe_stream_t stream);

/*
 * Peer mapping of device buffers between processes (CUDA IPC).
 * moe_ipc_export: handle (host, MOE_IPC_HANDLE_BYTES) of the device
 *   allocation holding dev_ptr, and the byte offset of dev_ptr in it.  The
 *   memory must come from cudaMalloc (PyTorch's default allocator).
 * moe_ipc_import: maps another process's allocation into this one; the
 *   buffer is at *mapping + offset.  Release with moe_ipc_close(*mapping).
 * Errors are returned as MOE_ERR_CUDA (nothing is left pending).
 */
#define MOE_IPC_HANDLE_BYTES 64
MOE_API int moe_ipc_export(const void* dev_ptr, void* handle, int64_t* offset);
MOE_API int moe_ipc_import(const void* handle, void** mapping);
MOE_API int moe_ipc_close(void* mapping);

/*
 * moe_transpose_weights -- convert expert matrices from the pages' x @ W
 * layout (E, K_in, N_out) to this library's (E, N_out, K_in), on device.
 * src and dst must not overlap.  dtype f32 or bf16.
 */
MOE_API int moe_transpose_weights(const void* src, void* dst, int32_t E, int64_t K_in, int64_t N_out,
                          moe_dtype dtype, moe_stream_t stream);

/*
 * moe_wait_probe -- the failure-detection path of the library's device-side
 * waits (slot-scan look-back, GEMM pipeline barriers), on a flag the caller
 * controls: one thread waits until the device word *flag becomes non-zero,
 * or records MOE_ERR_TIMEOUT in dev_status once limit_ns nanoseconds have
 * passed and returns, leaving the context usable.  0 < limit_ns <= 4e9.
 *   flag, dev_status: device.
 */
MOE_API int moe_wait_probe(const uint32_t* flag, int64_t limit_ns, int32_t* dev_status, moe_stream_t stream);

/* Set the device status word to MOE_OK (stream-ordered). */
MOE_API int moe_clear_status(int32_t* dev_status, moe_stream_t stream);

/* Synchronise `stream`, then copy the device status word into *host_status
 * (host pointer).  Returns MOE_ERR_CUDA if the synchronisation failed. */
MOE_API int moe_read_status(const int32_t* dev_status, moe_stream_t stream, int32_t* host_status);

#ifdef __cplusplus
}
#endif

#endif /* MOE_H_ */
