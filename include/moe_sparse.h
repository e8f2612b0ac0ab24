/*
 * moe_sparse.h -- C ABI of a B200 (sm_100a) Mixture-of-Experts feed-forward
 * layer that skips inactive neurons inside each routed expert.
 *
 * The operation, per batch of T tokens x[T][d_model]:
 *
 *   1. Router. logits = x W_router^T (+ router_bias), softmax over all E
 *      experts, the top_k experts by probability (ties go to the lower
 *      expert index), weights p_sel / sum(p_sel) when desc.renormalize,
 *      else p_sel. The pages keep the dense model's router as it is
 *      [gist.science EN "Uncovering Intra-expert Activation Sparsity for
 *      Efficient Mixture-of-Expert Model Execution", Technical Summary >
 *      Methodology > System Implementation in vLLM].
 *   2. Dense gate and up projections of every routed (token, expert) pair
 *      [same list, "Gate Projection": the gate projection runs densely to
 *      produce the activation scores] and the SwiGLU value
 *      h = SiLU(x W_gate[e]^T) * (x W_up[e]^T)
 *      [mlsanity.com page, "Builds on": GLU Variants Improve Transformer].
 *   3. Threshold mask in one pass, no sort: neuron j is active iff
 *      |h_j| > tau; at or below tau it is inactive
 *      [same list, "Activation Masking"]. The test is taken on the fp32 h
 *      before any rounding.
 *   4. Down projection that reads only the W_down rows of active neurons
 *      [same list, "Fused Up-Down Projection": gather the active neurons'
 *      weights, pack them densely, multiply densely]; y = sum_{j active}
 *      h_j W_down[e][j, :].
 *   5. Combine out[t] = sum_i w[t,i] y[t,i] + sum_s y_shared[s,t]; shared
 *      experts are always active with weight 1 and their own threshold
 *      [gist.science EN, Technical Summary > Methodology > "Empirical
 *      Analysis": routed vs always-active shared experts].
 *   The sparse/dense codepath choice by batch size [same list, "Dynamic
 *   Switching"] is made per expert token group on the device from the
 *   group's token count and the size of its active-row union.
 *
 * Gate score (desc.score = MOE_SCORE_GATE), the pages' own system: step 3
 * tests the gate projection alone, neuron j is active iff |SiLU(g_j)| > tau
 * [same list, "Gate Projection" and "Activation Masking"], and for the
 * small expert token groups (the GEMV path) the up projection of step 2 is
 * computed only for the group's active-row union, reading only those W_up
 * rows [same list, "Fused Up-Down Projection": only the active neurons'
 * up and down weights are fetched]. An active neuron still contributes its
 * full h_j = SiLU(g_j) u_j. Larger groups compute the up projection densely
 * and apply the same gate-score mask.
 *
 * Conventions shared by every entry point
 *   - Tensors are DEVICE pointers on desc.device, contiguous, row-major,
 *     16-byte aligned, in desc.dtype (x, weights, out), except router_bias
 *     (float32) and out when desc.out_f32 is set (float32). The caller owns them; the library never frees them.
 *       x         [T][d_model]
 *       W_router  [n_experts][d_model]            logits = x W_router^T
 *       W_gate    [n_experts][d_ff][d_model]      row j: neuron j's input weights
 *       W_up      [n_experts][d_ff][d_model]
 *       W_down    [n_experts][d_ff][d_model]      row j: neuron j's output vector
 *       out       [T][d_model]
 *   - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - The context owns a device workspace sized at init for max_tokens and
 *     top_k_max; moe_sparse_forward never allocates and never synchronises
 *     the host.
 *   - Argument errors return synchronously before any launch. Launch
 *     errors return MOE_ERR_CUDA. Errors found by kernels (a bounded wait
 *     that ran out) are recorded in a device status word read by
 *     moe_sparse_get_status.
 *   - One context serves one stream at a time.
 *   - Shapes: d_model % 256 == 0 and d_ff % 128 == 0 for MOE_BF16;
 *     d_model % 128 == 0 and d_ff % 32 == 0 for MOE_F32; 1 <= n_experts <= 256;
 *     1 <= top_k <= min(n_experts, 16); 1 <= max_tokens <= 65536.
 */
#ifndef MOE_SPARSE_H
#define MOE_SPARSE_H

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

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID = 1,        /* bad argument, null pointer, size out of range */
  MOE_ERR_UNSUPPORTED = 2,    /* valid but not implemented (shape, dtype, device) */
  MOE_ERR_CUDA = 3,           /* a CUDA runtime/driver call failed */
  MOE_ERR_NOMEM = 4,          /* device allocation failed in init */
  MOE_ERR_DEVICE_TIMEOUT = 5  /* a kernel's bounded wait ran out (status word) */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

typedef enum {
  MOE_SCORE_H = 0,            /* active iff |h| > tau, h = SiLU(g) u */
  MOE_SCORE_GATE = 1          /* active iff |SiLU(g)| > tau; sparse up projection */
} moe_score;

typedef enum {
  MOE_PATH_AUTO = 0,          /* threshold on; per group: row stream (GEMV; inside the gate/up
                                 kernel when every gate/up tile of the batch has its own CTA),
                                 gathered TC or all-rows TC; small groups join the all-rows TC
                                 groups when those are at least half of the batch and all
                                 groups fit one tensor-core wave */
  MOE_PATH_DENSE = 1,         /* no threshold: every neuron active (the dense baseline; same
                                 kernels and per-group rules as AUTO) */
  MOE_PATH_SPARSE_GEMV = 2,   /* threshold on; every group on the CUDA-core row-stream kernel
                                 (never fused into the gate/up kernel) */
  MOE_PATH_SPARSE_TC = 3,     /* threshold on; gathered-row tensor-core path (groups <= 64 tokens) */
  MOE_PATH_SPARSE_TC_ALLROWS = 4 /* threshold on; tensor cores over all rows with masked h */
} moe_path;

typedef struct {
  int32_t d_model;
  int32_t d_ff;
  int32_t n_experts;
  int32_t top_k_max;
  int32_t max_tokens;
  int32_t renormalize;        /* 1: w = p_sel / sum(p_sel); 0: w = p_sel */
  int32_t n_shared;           /* always-on shared experts, 0..8 */
  int32_t d_ff_shared;        /* their d_ff (same divisibility as d_ff); ignored if n_shared == 0 */
  int32_t dtype;              /* moe_dtype */
  int32_t path;               /* moe_path */
  int32_t debug;              /* 1: keep per-pair active bitmaps for moe_sparse_get_debug */
  int32_t device;             /* CUDA device ordinal */
  int32_t gemv_max_tokens;    /* AUTO: groups with <= this many tokens use the GEMV path.
                                 0: automatic -- groups of <= 4 tokens on the GEMV path, and
                                 (|h| score, bf16) groups of 5..8 tokens choose after gate/up:
                                 the GEMV path if their active-row union is <= 0.8 x d_ff,
                                 else all rows on the tensor cores; in batches whose groups
                                 all hold <= 8 tokens (T <= 8), every group uses the GEMV
                                 path (either score) */
  float gather_max_density;   /* AUTO (bf16): a tensor-core group of <= 64 tokens whose
                                 active-row union is <= this fraction of d_ff reads only
                                 the union rows (gathered copies, packed in shared memory)
                                 instead of all rows; 0: never. The Python binding's
                                 default is 0.5 (the gathered stream runs at about 2/3 of
                                 the all-rows stream's bandwidth) */
  int32_t score;              /* moe_score (0: MOE_SCORE_H) */
  int32_t out_f32;            /* 1: out is float32 [T][d_model] for either dtype (the combine's
                                 fp32 sums, not rounded; for partial outputs that are summed
                                 afterwards, e.g. over d_ff shards); 0: out is in dtype */
} moe_sparse_desc;

typedef struct {
  int64_t n_routed_h;         /* routed (token, expert) pairs x d_ff: h values tested */
  int64_t n_routed_active;    /* of those, |h| > tau */
  int64_t n_shared_h;
  int64_t n_shared_active;
  int64_t down_rows_read;     /* W_down rows streamed by the down projection, all groups */
  int64_t n_groups;           /* expert token groups (routed + shared) */
  int64_t n_groups_gemv;
  int64_t n_groups_tc_gather;
  int64_t n_groups_tc_allrows;
  int64_t n_experts_touched;  /* routed experts with at least one token */
  int64_t up_rows_read;       /* W_up rows streamed by the sparse up projection (gate score) */
  int64_t gate_up_rows_read;  /* W_gate + W_up rows loaded by the gate/up projection */
  int64_t down_rows_gemv;     /* of down_rows_read, the rows streamed by the row-stream (GEMV)
                                 kernel, once per pass of up to 8 tokens */
  int64_t down_rows_fused;    /* of down_rows_read, the rows read by the gate/up kernel's fused
                                 down projection (row-stream groups of <= 4 tokens, bf16):
                                 per 128-neuron tile, the tile's active rows */
  int64_t up_rows_fused;      /* of up_rows_read, the rows read by the gate/up kernel's fused
                                 up + down projection (gate score, one-token groups) */
} moe_stats;

typedef struct moe_sparse_ctx moe_sparse_ctx;

/* Host-only check of a descriptor (no CUDA call). MOE_OK if init would accept it. */
MOE_API moe_status moe_sparse_validate_desc(const moe_sparse_desc* desc);

/* Device workspace bytes init allocates for desc (host-only, no CUDA call). */
MOE_API moe_status moe_sparse_workspace_bytes(const moe_sparse_desc* desc, size_t* bytes);

/* Create a context on desc->device: validates desc, allocates the workspace.
 * On failure *ctx is NULL and nothing is left allocated. */
MOE_API moe_status moe_sparse_init(const moe_sparse_desc* desc, moe_sparse_ctx** ctx);

/* Always-on shared experts (desc.n_shared > 0): W*_s are device pointers
 * [n_shared][d_ff_shared][d_model] in desc.dtype, kept by pointer (the caller
 * keeps them alive); tau_shared is their own threshold. A negative tau_shared
 * keeps every shared neuron active, so the shared experts run dense while the
 * routed experts stay sparse (the configuration of the paper's system, which
 * leaves shared-expert execution unchanged [gist.science EN "Uncovering
 * Intra-expert Activation Sparsity for Efficient Mixture-of-Expert Model
 * Execution", Technical Summary > Methodology > System Implementation in
 * vLLM]). Must be called before the first forward of a context with shared
 * experts. */
MOE_API moe_status moe_sparse_set_shared(moe_sparse_ctx* ctx, const void* Wg_s, const void* Wu_s,
                                 const void* Wd_s, float tau_shared);

/* One layer forward, steps 1-5 above, enqueued on stream. 0 <= T <= max_tokens
 * (T == 0 launches nothing); 1 <= top_k <= top_k_max; router_bias may be NULL.
 * tau is ignored by MOE_PATH_DENSE. out is fully overwritten. */
MOE_API moe_status moe_sparse_forward(moe_sparse_ctx* ctx, const void* x, int32_t T,
                              const void* W_router, const float* router_bias,
                              const void* W_gate, const void* W_up, const void* W_down,
                              float tau, int32_t top_k, void* out, void* stream);

/* Routing and active sets of the last forward, in pair order p = t*top_k + i,
 * copied into caller DEVICE buffers on stream (any pointer may be NULL):
 *   topk_idx [T][top_k] int32, topk_w [T][top_k] float32,
 *   active_bits [T*top_k][ceil(d_ff/32)] uint32 (bit j%32 of word j/32 = neuron j active;
 *              needs desc.debug = 1),
 *   active_bits_shared [n_shared][T][ceil(d_ff_shared/32)] (needs desc.debug = 1). */
MOE_API moe_status moe_sparse_get_debug(moe_sparse_ctx* ctx, int32_t* topk_idx, float* topk_w,
                                uint32_t* active_bits, uint32_t* active_bits_shared,
                                void* stream);

/* Counters of the last forward (synchronises stream, then copies to the host struct). */
MOE_API moe_status moe_sparse_get_stats(moe_sparse_ctx* ctx, moe_stats* stats, void* stream);

/* Reads and clears the device status word (synchronises the device).
 * *device_err receives MOE_OK or MOE_ERR_DEVICE_TIMEOUT. */
MOE_API moe_status moe_sparse_get_status(moe_sparse_ctx* ctx, int32_t* device_err);

/* Per-stage timing of later forwards with CUDA events recorded on the
 * forward's stream between its kernels. ring > 0 keeps event sets for the
 * last `ring` forwards (at most 4096); 0 turns timing off. */
MOE_API moe_status moe_sparse_set_timing(moe_sparse_ctx* ctx, int32_t ring);

/* Milliseconds of each stage of the last timed forward (synchronises its
 * events). Stages: 0 route, 1 permute, 2 gate_up, 3 union_scan, 4 down_gemv,
 * 5 down_tc, 6 combine; a stage that launched nothing reports 0. */
MOE_API moe_status moe_sparse_get_timing(moe_sparse_ctx* ctx, float* ms, int32_t n);

/* Stage milliseconds of every timed forward since the last call, oldest
 * first: ms[f * n_stages + s] for f < *n_forwards (at most max_forwards and
 * at most the ring size; older ones are dropped). Synchronises the events and
 * restarts the collection. */
MOE_API moe_status moe_sparse_get_timing_all(moe_sparse_ctx* ctx, float* ms, int32_t n_stages,
                                             int32_t max_forwards, int32_t* n_forwards);

/* Kernels this context has launched since init (host-side count). */
MOE_API moe_status moe_sparse_launch_count(const moe_sparse_ctx* ctx, int64_t* n);

/* Name of stage i (static string), or NULL. */
MOE_API const char* moe_sparse_stage_name(int32_t i);

/* Last error message of ctx (or of the last failed init if ctx is NULL). */
MOE_API const char* moe_sparse_last_error(const moe_sparse_ctx* ctx);

/* Routing only, for callers that must not allocate device memory: plug-ins
 * living inside another framework's fixed memory plan (where a private
 * cudaMalloc breaks the host's accounting or fragments its pool), and serving
 * loops that reserve all device memory up front and treat any later
 * allocation as a failure. The paper has no counterpart: it is an
 * allocation-free variant of the forward's router kernel, not a step of the
 * method.
 * It computes what moe_sparse_forward's router computes for x [T][d_model]
 * and W_router [n_experts][d_model] (device pointers, dtype, 16-byte aligned;
 * router_bias [n_experts] float32 or NULL) into caller DEVICE buffers:
 *   topk_idx [T][top_k] int32, topk_w [T][top_k] float32 (as in get_debug);
 *   expert_offsets [n_experts+1]: pairs of expert e hold positions
 *     expert_offsets[e] .. expert_offsets[e+1]-1 (no padding);
 *   slot_of [T*top_k]: position of pair p = t*top_k + i; perm [T*top_k]: token
 *     at each position; within an expert, positions follow pair order.
 * Its scratch is a 1 MiB array in device memory that every GPU which loads the
 * library holds until exit, so it allocates nothing and launches one kernel
 * (plus a 256-byte cudaMemsetAsync that clears its completion counter).
 * Limits: T <= 4096, n_experts <= 256, top_k <= 16, d_model a multiple of 256
 * (bf16) or 128 (fp32); larger sizes return MOE_ERR_UNSUPPORTED with a message.
 * The first call on a device looks the scratch address up (set-up): make that
 * first call before any stream capture. All calls share the one scratch array,
 * so calls whose kernels overlap on the GPU (different streams, or different
 * host threads on one device) race and must be serialised by the caller.
 * Runs on the current device, enqueued on stream. */
MOE_API moe_status moe_sparse_route_noalloc(const void* x, int32_t T, int32_t d_model,
                                            const void* W_router, const float* router_bias,
                                            int32_t n_experts, int32_t top_k,
                                            int32_t renormalize, int32_t dtype,
                                            int32_t* topk_idx, float* topk_w,
                                            int32_t* expert_offsets, int32_t* slot_of,
                                            int32_t* perm, void* stream);

/* Frees the workspace and the context. NULL is accepted. */
MOE_API moe_status moe_sparse_destroy(moe_sparse_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* MOE_SPARSE_H */
