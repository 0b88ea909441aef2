/*
 * moe.h -- C ABI of the B200 (sm_100a) top-k routed Mixture-of-Experts FFN
 * layer forward pass.
 *
 * What is computed (page title, section):
 *   - the router picks a fixed set of k experts per token ("PCoMoE" summary,
 *     "The Limitation of Monolithic Expert Selection"); gates are the softmax
 *     of the selected logits (renormalised over the k);
 *   - routing decisions are flattened into a task list, grouped by expert id
 *     and sorted by token id inside each group, then run as a grouped GEMM
 *     that loads each block of expert weights once for a batch of tokens
 *     ("OmniMoE" technical summary, 2.2 Expert-Centric Scheduling);
 *   - experts: SwiGLU FFN experts y = W_down (silu(W_gate x) * (W_up x));
 *     always-on shared experts ("OmniMoE" 2.1, Shared Dense MLP); MoE++
 *     zero (output 0), copy (output x) and constant (a1 x + a2 v) experts,
 *     and gating residuals that add the previous layer's logits ("MoE++"
 *     summary, "Approach"); OmniMoE atomic experts
 *     E_i(x) = GELU(x . u_i) v_i found by a Cartesian-product router that
 *     scores the row and column halves of a 2-D expert grid separately
 *     ("OmniMoE" 2.1 Atomic Experts, 2.2 Cartesian Product Router).
 *
 * Conventions (all entry points):
 *   - Ownership: the caller owns every buffer.  Pointers to tensors are
 *     DEVICE pointers (cudaMalloc / PyTorch CUDA memory) unless stated; the
 *     descriptor and weight structs are read on the host during the call.
 *     The library allocates no device memory: scratch space is the
 *     caller's `workspace` of at least the size the *_workspace_size calls
 *     return (256-byte aligned).  The library keeps host-side caches of TMA
 *     descriptors only.
 *   - Layout: row-major, C order.  d_model: a multiple of 64 (bf16) or 8 (fp32).  Expert weights are K-contiguous:
 *     w_gate, w_up [n_ffn, hidden, d_model]; w_down [n_ffn, d_model, hidden].
 *     Every tensor base must be 16-byte aligned.
 *   - Types: x, weights and y are `dtype` (fp32 or bf16); accumulation is
 *     fp32; routing outputs are fp32 / int32.
 *   - Asynchrony: every call only enqueues kernels on `stream` (a
 *     cudaStream_t; NULL = legacy default stream) and returns; nothing is
 *     synchronised.
 *   - Errors: argument errors are detected on the host and returned at
 *     once (nothing enqueued).  Errors found by the kernels (an expert id
 *     out of range, a wait that timed out) are recorded in a per-device
 *     status word and returned by moe_get_device_status().  No kernel traps.
 *   - Expert ids: 0..n_ffn-1 are FFN experts, then n_zero zero experts,
 *     n_copy copy experts, n_const constant experts.  Atomic experts have ids
 *     r * pk_cols + c for grid row r and column c.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

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

typedef void* moe_stream_t; /* a cudaStream_t */

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,   /* bad descriptor, null or misaligned pointer   */
    MOE_ERR_UNSUPPORTED = 2,   /* valid but not implemented (shape limits)     */
    MOE_ERR_WORKSPACE = 3,     /* workspace smaller than required              */
    MOE_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed            */
    MOE_ERR_DEVICE_BOUNDS = 5, /* a kernel saw an index out of range           */
    MOE_ERR_TIMEOUT = 6        /* a kernel wait exceeded its time limit        */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;
typedef enum { MOE_EXPERT_SWIGLU = 0, MOE_EXPERT_ATOMIC_GELU = 1 } moe_expert_kind;

/* Sizes of one layer.  Unused fields must be 0. */
typedef struct moe_layer_desc {
    int32_t T;             /* tokens in the batch (>= 0)                          */
    int32_t d_model;       /* width of x and y                                    */
    int32_t top_k;         /* experts per token (atomic: K of the product router) */
    int32_t dtype;         /* moe_dtype of x, weights and y                       */
    int32_t kind;          /* moe_expert_kind                                     */
    int32_t n_ffn;         /* routed SwiGLU experts                               */
    int32_t hidden;        /* their hidden width H                                */
    int32_t n_shared;      /* always-on SwiGLU experts (weight 1); atomic kind:   *
                            * 0 or 1 shared dense branch (the full OmniMoE layer) */
    int32_t hidden_shared; /* their hidden width (SwiGLU kind: equal to hidden;   *
                            * atomic kind: a multiple of 128)                     */
    int32_t n_zero;        /* MoE++ zero experts                                  */
    int32_t n_copy;        /* MoE++ copy experts                                  */
    int32_t n_const;       /* MoE++ constant experts                              */
    int32_t pk_rows;       /* atomic: grid rows N_r (row sub-keys)                */
    int32_t pk_cols;       /* atomic: grid columns N_c (column sub-keys)          */
    int32_t pk_topk_half;  /* atomic: sub-keys kept per half                      */
    int32_t d_query;       /* atomic: query width (two halves of d_query / 2)     */
    int32_t out_f32;       /* 0: y is `dtype`; 1: y is fp32 (the fp32 combine     *
                            * before its final rounding; the dtype output is its *
                            * round-to-nearest-even)                              */
    int32_t expert_fp8;    /* 1: FP8 experts ("PCoMoE" summary, Improvements 3,  *
                            * Mixed Precision Execution): the SwiGLU experts'     *
                            * weights are e4m3 codes with an fp32 scale per      *
                            * output row (moe_layer_weights s_*), the expert     *
                            * GEMMs run on e4m3 activations (each row divided by *
                            * the smallest power of two s with 448 s >= its      *
                            * max |value| and rounded to nearest, s kept); the  *
                            * router and the combine stay in `dtype` (bf16,     *
                            * required), as do h between its rounding to bf16   *
                            * and its quantization.  d_model a multiple of 256, *
                            * hidden of 128.  0: weights in `dtype`.             */
} moe_layer_desc;

/* Device pointers to the layer's parameters (NULL where the layer has none). */
typedef struct moe_layer_weights {
    const void* w_router;     /* [n_ffn + n_zero + n_copy + n_const, d_model]            */
    const float* router_bias; /* [same rows] fp32, added to the logits; nullable         */
    const void* w_const_mix;  /* [n_const, 2, d_model]: (a1, a2) = softmax(W_c x)        */
    const void* const_vec;    /* [n_const, d_model]: the constant experts' vectors v     */
    const void* w_gate;       /* [n_ffn, hidden, d_model]                                */
    const void* w_up;         /* [n_ffn, hidden, d_model]                                */
    const void* w_down;       /* [n_ffn, d_model, hidden]                                */
    const void* ws_gate;      /* [n_shared, hidden_shared, d_model]                      */
    const void* ws_up;        /* [n_shared, hidden_shared, d_model]                      */
    const void* ws_down;      /* [n_shared, d_model, hidden_shared]                      */
    const void* w_query;      /* atomic: [d_query, d_model]                              */
    const void* subkeys_row;  /* atomic: [pk_rows, d_query / 2]                          */
    const void* subkeys_col;  /* atomic: [pk_cols, d_query / 2]                          */
    const void* u;            /* atomic: [pk_rows * pk_cols, d_model] input vectors      */
    const void* v;            /* atomic: [pk_rows * pk_cols, d_model] output vectors     */
    /* expert_fp8: w_gate, w_up, w_down (and ws_*) hold e4m3 codes; these are
     * the fp32 scales of their rows (the weight is code * scale):            */
    const float* s_gate;      /* [n_ffn, hidden]                                         */
    const float* s_up;        /* [n_ffn, hidden]                                         */
    const float* s_down;      /* [n_ffn, d_model]                                        */
    const float* ss_gate;     /* [n_shared, hidden_shared]                               */
    const float* ss_up;       /* [n_shared, hidden_shared]                               */
    const float* ss_down;     /* [n_shared, d_model]                                     */
} moe_layer_weights;

/* Number of expert groups of the grouped step: n_ffn + n_shared (SwiGLU) or
 * pk_rows * pk_cols (atomic).  expert_offsets has groups + 1 entries. */
MOE_API int64_t moe_num_groups(const moe_layer_desc* desc);

/* Row capacity of x_sorted / y_sorted / token_of: T*top_k + n_shared*T
 * (SwiGLU) or T*top_k (atomic). */
MOE_API int64_t moe_row_capacity(const moe_layer_desc* desc);

/* Scratch bytes needed by moe_route, moe_permute and moe_grouped_ffn (the
 * largest of the three); -1 for an invalid descriptor. */
MOE_API int64_t moe_workspace_size(const moe_layer_desc* desc);

/* Bytes needed by moe_layer_forward: all intermediates plus the scratch. */
MOE_API int64_t moe_layer_workspace_size(const moe_layer_desc* desc);

/*
 * Router ("PCoMoE" summary, top-k selection; "MoE++" Approach, gating
 * residuals; "OmniMoE" 2.2 Cartesian Product Router).
 * SwiGLU kind: z[t] = W_router x_t + router_bias + prev_logits[t] (fp32);
 *   topk_idx[t] = the k largest z in descending order, ties to the lower id;
 *   topk_gate[t, j] = exp(z_sel[j] - z_sel[0]) / sum over the k selected;
 *   const_mix[t, c] = softmax(W_c,c x_t) for each constant expert.
 * Atomic kind: q = W_query x_t (fp32), s_row = subkeys_row q[:dq/2],
 *   s_col = subkeys_col q[dq/2:]; the pk_topk_half best of each half; the
 *   pk_topk_half^2 candidates (r, c) score s_row[r] + s_col[c] (compared
 *   exactly, ties to the lower id r*pk_cols + c); the top_k best with softmax
 *   gates.
 * x [T, d_model]; prev_logits [T, rows of w_router] fp32 nullable;
 * logits_out (nullable): SwiGLU [T, rows of w_router] fp32 z; atomic
 *   [T, pk_rows + pk_cols] fp32 (s_row then s_col);
 * topk_idx [T, top_k] int32; topk_gate [T, top_k] fp32;
 * const_mix [T, n_const, 2] fp32 (required iff n_const > 0).
 */
MOE_API moe_status moe_route(const moe_layer_desc* desc, const moe_layer_weights* w, const void* x,
                     const float* prev_logits, float* logits_out, int32_t* topk_idx,
                     float* topk_gate, float* const_mix, void* workspace, size_t ws_bytes,
                     moe_stream_t stream);

/*
 * Expert-centric grouping ("OmniMoE" 2.2: task collection, grouping by
 * expert id, sorting by token id within each group): a per-expert
 * histogram, an exclusive prefix sum and a stable permutation.
 * expert_offsets [groups + 1]: group g holds rows [off[g], off[g+1]).
 *   SwiGLU: groups 0..n_ffn-1 are the FFN experts' tasks in (expert, token)
 *   order; group n_ffn + s holds all T tokens in order for shared expert s.
 *   Zero-computation slots are not grouped.
 * row_of [T*top_k]: row of slot (t, j), -1 for a zero-computation expert.
 * token_of [row capacity]: SwiGLU: token of each row; atomic: flat slot id
 *   t*top_k + j of each task.
 * x_sorted [row capacity, d_model]: SwiGLU only, x_sorted[r] = x[token_of[r]]
 *   (expert_fp8: the rows' e4m3 codes [row capacity, d_model] bytes, then at
 *   byte offset align256(capacity * d_model) their fp32 scales [row capacity]);
 *   NULL for the atomic kind, and may be NULL for the SwiGLU kind (no copy
 *   made) when the fused expert step gathers the rows itself.  Rows past
 *   expert_offsets[groups] are untouched.
 * An id outside [0, n_ffn + n_zero + n_copy + n_const) (or the atomic grid)
 * sets MOE_ERR_DEVICE_BOUNDS in the device status and is skipped.
 * Both kinds run as a cooperative launch (every block resident, grid barriers
 * on a counter in the workspace, cleared first on `stream`; each wait bounded,
 * MOE_ERR_TIMEOUT in the device status if one gives up), so two calls must
 * not share a workspace while both may run.
 */
MOE_API moe_status moe_permute(const moe_layer_desc* desc, const int32_t* topk_idx, const void* x,
                       int32_t* expert_offsets, int32_t* row_of, int32_t* token_of,
                       void* x_sorted, void* workspace, size_t ws_bytes, moe_stream_t stream);

/*
 * Grouped expert step ("OmniMoE" 2.2 Grouped GEMM; 2.1 Atomic Experts).
 * SwiGLU: y_sorted[r] = W_down[e] (silu(W_gate[e] x_sorted[r]) * (W_up[e]
 *   x_sorted[r])) for r in group e (shared groups use the ws_* weights),
 *   on tcgen05 tensor cores (bf16) or fp32 SIMT cores (fp32); the hidden
 *   activation is rounded to dtype in the workspace, the expert outputs are
 *   kept in fp32.  y_sorted [row capacity, d_model] fp32.  token_of, x,
 *   topk_gate unused.
 * Atomic: c[s] = topk_gate[s] * GELU(u_e . x_t) for each task s = t*K + j of
 *   expert e, over the expert-sorted task order in units of 16 tasks whose
 *   dot products are one tensor-core tile (each touched u_e read once per
 *   unit); y_sorted is float c[T*K] in slot order.  x_sorted unused.  The
 *   workspace holds the expert of each task (T*top_k int32).  With a shared
 *   dense branch ("OmniMoE" 2.1, Shared Dense MLP; n_shared = 1) the call
 *   also computes ys = Ws_down (silu(Ws_gate x_t) * (Ws_up x_t)) for every
 *   token (two grouped GEMMs, the hidden activation rounded to bf16 in the
 *   workspace) into y_sorted after c, at byte offset align256(T*K*4), as
 *   [T, d_model] fp32.
 */
MOE_API moe_status moe_grouped_ffn(const moe_layer_desc* desc, const moe_layer_weights* w,
                           const void* x_sorted, const int32_t* expert_offsets,
                           const int32_t* token_of, const void* x, const float* topk_gate,
                           void* y_sorted, void* workspace, size_t ws_bytes,
                           moe_stream_t stream);

/*
 * The two grouped GEMMs of the SwiGLU step, one per call (same arguments as
 * moe_grouped_ffn): phase 1 writes the hidden activation h into the
 * workspace, phase 2 reads it and writes y_sorted.  Calling phase 1 then
 * phase 2 on the same workspace equals moe_grouped_ffn.  Atomic kind with a
 * shared dense branch: phase 1 and 2 are that branch's two GEMMs (x_sorted
 * is x itself, expert_offsets unused); moe_grouped_ffn = the atomic step
 * followed by both.
 */
MOE_API moe_status moe_grouped_ffn_phase(const moe_layer_desc* desc, const moe_layer_weights* w,
                                 int phase, const void* x_sorted,
                                 const int32_t* expert_offsets, void* y_sorted,
                                 void* workspace, size_t ws_bytes, moe_stream_t stream);

/*
 * Gate-weighted combine back to token order ("OmniMoE" 2.1 Dynamic Expert
 * Assembly; "MoE++" Approach).
 * SwiGLU: y_t = sum_s y_sorted[off[n_ffn + s] + t]
 *             + sum_j topk_gate[t, j] * O_j, with O_j = y_sorted[row_of[t, j]]
 *   (y_sorted fp32 as written by moe_grouped_ffn)
 *   for an FFN expert, 0 for a zero expert, x_t for a copy expert and
 *   a1 x_t + a2 v_c for constant expert c (const_mix, w->const_vec);
 *   accumulated in fp32 in slot order, rounded once to dtype.
 * Atomic: y_t = sum_j c[t*K + j] * v_{topk_idx[t, j]} (+ the shared branch's
 *   row of y_sorted when n_shared = 1), fp32, rounded once.
 * y [T, d_model] in dtype, or fp32 if desc->out_f32.
 */
MOE_API moe_status moe_combine(const moe_layer_desc* desc, const moe_layer_weights* w,
                       const void* y_sorted, const int32_t* expert_offsets,
                       const int32_t* row_of, const int32_t* topk_idx, const float* topk_gate,
                       const float* const_mix, const void* x, void* y, moe_stream_t stream);

/*
 * The expert step with the permutation and the combine fused into the two
 * grouped GEMMs ("OmniMoE" technical summary, 2.2 Expert-Centric
 * Scheduling: the expert weights of a block are loaded once for the tokens of
 * the expert's group; 2.1 Dynamic Expert Assembly: the routed outputs are
 * assembled per token).  Same result as moe_grouped_ffn + moe_combine, with no
 * x_sorted and no y_sorted in memory:
 *   phase 1: h[r] = silu(W_gate[e] x[token_of[r]]) * (W_up[e] x[token_of[r]])
 *            for the rows r of expert e's group, the token rows read from
 *            moe_permute's x_sorted, or, with x_sorted NULL, gathered from x
 *            by the GEMM's own loads (tile::gather4 of single rows; each row
 *            is then fetched once per weight block, which measured 3x slower
 *            than the gather copy on the Mixtral-shaped layer, so the layer
 *            path passes x_sorted); the same kernel zeroes the fp32
 *            accumulator rows of the groups' tokens;
 *   phase 2: acc[t] += g(t, e) * (W_down[e] h[r]) for t = token_of[r], by
 *            the GEMM's epilogue with vector atomics.  A token has at most
 *            two FFN slots, and two fp32 additions into zero give the same sum
 *            in either order, so the result does not depend on timing;
 *   phase 3: y_t = acc[t] (if the token has an FFN slot) + the zero-
 *            computation slots' terms in slot order (as in moe_combine),
 *            rounded once to the output type.
 *   phase 0: the three in order.
 * Layers it applies to (else MOE_ERR_UNSUPPORTED, nothing enqueued): SwiGLU
 * kind, bf16, n_ffn > 0, no shared experts, top_k <= 2, d_model a multiple
 * of 256, hidden a multiple of 128.  moe_layer_forward keeps the two-pass
 * step (moe_grouped_ffn + moe_combine): on B200 it measured faster on the
 * Mixtral-shaped and MoE++ layers, because zeroing the accumulator and the
 * atomic epilogue cost more inside the GEMMs than the y_sorted round trip.
 * Arguments as moe_route / moe_permute produce them (expert_offsets [n_ffn +
 * 1], row_of [T, top_k], token_of [T * top_k], x_sorted [row capacity,
 * d_model] or NULL); x [T, d_model]; y [T, d_model] (bf16, or fp32 if
 * desc->out_f32).  workspace: at least
 * moe_fused_workspace_size(desc) bytes (h, then the accumulator at byte
 * align256(cap * hidden * 2)); phases 1-3 called one by one must share it.
 * moe_fused_workspace_size returns -1 for a descriptor the step does not
 * apply to.
 */
MOE_API int64_t moe_fused_workspace_size(const moe_layer_desc* desc);
MOE_API moe_status moe_fused_ffn_combine(const moe_layer_desc* desc, const moe_layer_weights* w, int phase,
                                         const void* x, const void* x_sorted, const int32_t* topk_idx,
                                         const float* topk_gate,
                                         const float* const_mix, const int32_t* expert_offsets,
                                         const int32_t* row_of, const int32_t* token_of, void* y,
                                         void* workspace, size_t ws_bytes, moe_stream_t stream);

/*
 * The whole layer: moe_route, moe_permute, moe_grouped_ffn and moe_combine
 * on `stream`, intermediates in `workspace` (moe_layer_workspace_size bytes).
 * x [T, d_model]; y [T, d_model] (dtype, or fp32 if desc->out_f32);
 * prev_logits nullable; logits_out nullable (as in moe_route).
 */
MOE_API moe_status moe_layer_forward(const moe_layer_desc* desc, const moe_layer_weights* w,
                             const void* x, const float* prev_logits, void* y,
                             float* logits_out, void* workspace, size_t ws_bytes,
                             moe_stream_t stream);

/*
 * The whole layer from host memory to host memory, for a caller whose tokens
 * arrive on the host (a serving loop).  The T tokens are processed in
 * `chunks` consecutive token ranges (0: automatic, max(2, (T + 2048) / 3584)
 * for T >= 4096, else 1; at most 8; with three or more, the first and the last
 * are half as long as the others); the host->device copy of range c + 1 and
 * the device->host copy of range c - 1 run on two internal copy streams while
 * range c is computed on `stream`, so PCIe transfers overlap the layer.  Every
 * token's result equals moe_layer_forward's bit for bit (tokens are
 * independent).  The pages (OmniMoE's serving scenario) name no such call.
 * x_host [T, d_model] (dtype), prev_logits_host [T, rows of w_router] fp32
 * (nullable), y_host [T, d_model] (dtype, or fp32 if desc->out_f32): host
 * memory, page-locked for the copies to overlap (pageable memory works but
 * serialises).  workspace: device, moe_layer_host_workspace_size bytes.
 * Asynchronous on `stream`: y_host is complete when `stream` reaches this
 * point (the internal streams are joined back into `stream`, so the call can
 * be captured in a CUDA graph).  Calls from several host threads on one
 * device share the internal streams and events: a per-device lock orders
 * their enqueueing, so they are correct but their copies do not overlap
 * each other.
 */
MOE_API int64_t moe_layer_host_workspace_size(const moe_layer_desc* desc, int chunks);
MOE_API moe_status moe_layer_forward_host(const moe_layer_desc* desc, const moe_layer_weights* w,
                                          const void* x_host, const float* prev_logits_host,
                                          void* y_host, int chunks, void* workspace,
                                          size_t ws_bytes, moe_stream_t stream);

/*
 * moe_permute without a workspace, for callers that cannot allocate device
 * memory: for example a plugin inside a host framework that owns all device
 * memory and offers the plugin no allocator, or a service whose device
 * memory budget is fixed and fully committed at start-up.  (The pages have
 * no counterpart: this is a property of the library, not of the method.)
 * Same arguments, results and errors as moe_permute for the SwiGLU kind,
 * minus the workspace: the per-block expert counts live in a fixed array in
 * the library's own device memory (256 KiB, held by every GPU that loads the
 * library until the process exits).  The call allocates nothing (no
 * cudaMalloc / cudaFree, no allocating library routine).
 * Limit: ceil(T / 256) * n_ffn <= 65536 (e.g. T <= 65536 with 256 experts,
 *   T <= 2,097,152 with 8 experts); beyond it, or for the atomic kind, the
 *   call returns MOE_ERR_UNSUPPORTED and enqueues nothing.
 * The first call on a device (and the first after a cudaDeviceReset, which
 *   gives the device a new context) looks up the array's device address with
 *   that device current and may fail with MOE_ERR_CUDA; make that first call
 *   before any stream capture.
 * Every call on a device shares the one array and it keeps the last call's
 *   contents (nothing needs clearing: each call overwrites every entry it
 *   reads).  Calls whose kernels overlap on the GPU -- on two streams at once,
 *   or from two host threads -- race on it and give wrong results; order them.
 */
MOE_API moe_status moe_permute_static(const moe_layer_desc* desc, const int32_t* topk_idx, const void* x,
                                      int32_t* expert_offsets, int32_t* row_of, int32_t* token_of,
                                      void* x_sorted, moe_stream_t stream);

/*
 * Expert parallelism (host functions; no device work).  With the routed
 * experts split over G ranks, each rank routes, permutes and combines its own
 * tokens, and the rows of expert e are computed by the rank that owns e.
 * Ownership follows the grouping of tasks by contiguous ranges of expert ids
 * ("OmniMoE" technical summary, 2.2 Expert-Centric Scheduling): rank r owns
 * experts [r*E/G, (r+1)*E/G) (integer division; a rank may own none when
 * E < G).  A rank's rows of expert e are rows [off[e], off[e+1]) of its
 * x_sorted (moe_permute's expert_offsets); it sends that block to the owner,
 * which lays the blocks it receives out expert-major with the source rank
 * inside, so its owned experts are ordinary groups of the grouped GEMM; the
 * results go back block by block to the rows they came from, and the combine
 * is the single-rank one.  The exchange itself (NCCL send/receive of the
 * blocks, in increasing expert order between every pair of ranks) is the
 * caller's.  The pages describe expert parallelism only as prior art for
 * other hardware; the split and layout here are this library's.
 *
 * moe_ep_expert_range: the experts [*lo, *hi) that `rank` owns.
 * moe_ep_owner: the rank that owns `expert` (-1 for invalid arguments).
 * moe_ep_plan: counts [G, E] host int32, counts[q*E + e] = rows of rank q
 *   routed to expert e (the differences of every rank's expert_offsets).
 *   For this rank's owned experts i = e - lo (n_own = hi - lo):
 *   recv_offsets[i*G + q], recv_counts[i*G + q] (host int32, n_own*G each):
 *   where the block of (expert e, source rank q) lands in the receive buffer
 *   and its rows; local_offsets [n_own + 1] (host int32): the group offsets
 *   of the owned experts in the receive buffer.  Returns the number of rows
 *   received (>= 0), or -1 for invalid arguments, a negative count or a total
 *   of 2^31 rows or more.  All buffers are the caller's.
 */
MOE_API moe_status moe_ep_expert_range(int G, int E, int rank, int32_t* lo, int32_t* hi);
MOE_API int32_t moe_ep_owner(int G, int E, int expert);
MOE_API int64_t moe_ep_plan(const int32_t* counts, int G, int E, int rank, int32_t* recv_offsets,
                            int32_t* recv_counts, int32_t* local_offsets);

/*
 * Self-test of the kernels' bounded waits (no counterpart on the pages): a
 * one-thread kernel waits on an mbarrier that nothing arrives on, giving up
 * after limit_ns nanoseconds (0 < limit_ns <= 2e9) the way every wait in the
 * library does -- it writes 0 to *waited_ok (device int) and records
 * MOE_ERR_TIMEOUT in the status word, and the CUDA context stays usable.
 */
MOE_API moe_status moe_selftest_wait_timeout(uint64_t limit_ns, int32_t* waited_ok, moe_stream_t stream);

/* Synchronises `stream`, returns the current device's status word in *out
 * (MOE_OK if no kernel reported an error) and clears it if reset != 0. */
MOE_API moe_status moe_get_device_status(moe_status* out, int reset, moe_stream_t stream);

/* Static description of a status code. */
MOE_API const char* moe_status_string(moe_status s);

/* Number of kernels the last call on this host thread enqueued. */
MOE_API int32_t moe_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
