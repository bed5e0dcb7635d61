/*
 * moe.h - C ABI of libmoe_b200: the forward pass of one Mixture-of-Experts
 * layer on one NVIDIA B200 (sm_100a).
 *
 * The layer has four stages, each exposed as its own entry point and fused
 * in moe_layer_forward:
 *
 *   1. router   logits l = W_g x (+ b), top-k expert selection and gate weights
 *               ("moe communication costs", Router design; "Advanced GPU
 *               Optimization ... Part 5", section 1.1 The Router Kernel)
 *   2. dispatch tokens grouped into expert-contiguous rows with capacity
 *               dropping, plus the aux-loss statistics ("MoE: what it costs to
 *               train and serve", Expert parallelism and two all-to-alls, step 1;
 *               "moe communication costs", Capacity factor and token dropping,
 *               Load balancing)
 *   3. experts  the expert FFNs as one grouped GEMM over the variable-size
 *               expert segments (same page, step 2)
 *   4. combine  y = sum over the selected experts i of G(x)_i E_i(x)
 *               ("moe communication costs", Router design; same page, step 3)
 *
 * Conventions for every entry point:
 *   - Pointer arguments named as device buffers are device pointers that the
 *     caller owns; the library never allocates or frees device memory.
 *   - Every call only enqueues work on `stream` (a cudaStream_t; NULL means the
 *     legacy default stream) and returns without synchronising, except
 *     moe_check_status.
 *   - Arguments are validated on the host before anything is enqueued; on a
 *     validation failure the call returns an error and writes nothing.
 *   - Launch failures return MOE_ERR_CUDA (the CUDA error string is available
 *     from moe_last_error_string).
 *   - Problems only the device can see (an expert index out of range, a
 *     bounded wait that gave up) are recorded in a status word at the start of
 *     the workspace; no kernel traps.  moe_check_status reads and clears it.
 *   - Layouts are row-major; "[A, B]" means A rows of B contiguous elements.
 *   - Element types: x, weights and y are all MOE_F32 or all MOE_BF16
 *     (bf16 stored as its 16-bit pattern).  Accumulation is fp32 or wider.
 *   - Weight layout (experts stacked on the leading axis, reduction axis
 *     contiguous):
 *        W1, W3 [N, H, d]   row h of expert e holds column h of the d x H
 *                           matrix applied to x (x W1)
 *        W2     [N, d, H]   row i of expert e holds column i of the H x d matrix
 *        Wg     [N, d]      router matrix W_g
 *        Ws1, Ws3 [Hs, d], Ws2 [d, Hs]  the always-on shared expert
 *   - The workspace is one device buffer of at least moe_workspace_bytes(cfg)
 *     bytes, 256-byte aligned, zero-filled by the caller once before its first
 *     use (the status word must start at zero).  One workspace serves every
 *     entry point for that configuration.  Calls that share a workspace must
 *     be ordered on one stream.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum moe_status {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = 1,    /* bad shape, null pointer, misalignment, k > N ... */
    MOE_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. FP8 dispatch with f32) */
    MOE_ERR_WORKSPACE = 3,      /* workspace missing, misaligned or too small */
    MOE_ERR_CUDA = 4,           /* a CUDA runtime / driver call failed */
    MOE_ERR_DEVICE_STATUS = 5,  /* moe_check_status: a kernel recorded an anomaly */
    MOE_ERR_TIMEOUT = 6         /* moe_check_status: a bounded device wait gave up */
} moe_status;

enum { MOE_F32 = 0, MOE_BF16 = 1, MOE_FP8_E4M3 = 2 };

/* Gate modes.
 *  MOE_GATE_TOPK_THEN_SOFTMAX ("mode R"): softmax over the k selected logits
 *    only, as the page-3 router does for its top-2 ("Advanced GPU Optimization
 *    ... Part 5", section 1.1).
 *  MOE_GATE_SOFTMAX_THEN_TOPK ("mode F"): G(x) = softmax over all N logits and
 *    the k largest G(x)_i are the mixture coefficients ("moe communication
 *    costs", Router design); with renormalize != 0 they are divided by their sum.
 * In both modes the k experts are the k largest logits in descending order,
 * equal logits ordered by lower expert index first. */
enum { MOE_GATE_TOPK_THEN_SOFTMAX = 0, MOE_GATE_SOFTMAX_THEN_TOPK = 1 };

/* Expert FFN forms: ReLU: y = max(x W1, 0) W2.
 *                   SwiGLU: y = (silu(x W1) * (x W3)) W2, silu(a) = a / (1 + e^-a). */
enum { MOE_ACT_RELU = 0, MOE_ACT_SWIGLU = 1 };

/* What happens to (token, slot) pairs an expert cannot take under its
 * capacity C ("moe communication costs", Capacity factor and token dropping:
 * overflowing tokens are either dropped or re-routed to a shared fallback
 * expert).
 *  MOE_OVERFLOW_DROP: dropped (they contribute nothing).
 *  MOE_OVERFLOW_FALLBACK: re-routed, with their gate weight, to a fallback
 *    expert stored as expert N after the routed ones (W1, W3, W2 then hold
 *    N + 1 expert blocks); it has no capacity limit and takes the overflow of
 *    every expert in the order the pairs are taken. */
enum { MOE_OVERFLOW_DROP = 0, MOE_OVERFLOW_FALLBACK = 1 };

typedef struct moe_config {
    int64_t T;               /* tokens, >= 0 */
    int32_t d;               /* hidden size; multiple of 8 (bf16) or 4 (f32) */
    int32_t N;               /* routed experts, 1..256 */
    int32_t k;               /* experts per token, 1..min(N, 8) */
    int32_t H;               /* routed expert hidden size */
    int32_t H_shared;        /* shared-expert hidden size, 0 = no shared expert */
    float   capacity_factor; /* C = floor(capacity_factor * T / N); <= 0: no limit */
    int32_t gate_mode;       /* MOE_GATE_* */
    int32_t renormalize;     /* mode F only */
    int32_t act;             /* MOE_ACT_* */
    int32_t dtype;           /* MOE_F32 or MOE_BF16 for x, weights, y */
    int32_t dispatch_dtype;  /* == dtype, or MOE_FP8_E4M3 (bf16 layers only) */
    float   aux_alpha;       /* alpha of L_aux = alpha * N * sum_i f_i p_i */
    /* Node-limited routing ("MoE: what it costs to train and serve", Limit how
     * many machines a token touches: a token may go to at most a few nodes,
     * chosen by the sum of the highest expert scores on each node).  With
     * n_groups > 1 and topk_groups < n_groups the N experts sit on n_groups
     * nodes of N / n_groups consecutive experts; a token uses at most
     * topk_groups of them, those with the largest sums of their
     * ceil(k / topk_groups) highest router probabilities (equal sums: lower
     * node first), and its top-k is taken among those nodes' experts.
     * Requires N % n_groups == 0, n_groups <= 32, 1 <= topk_groups,
     * k <= topk_groups * N / n_groups, and gate mode R or renormalised mode F
     * (plain mode F with nodes: MOE_ERR_UNSUPPORTED).  The aux statistics
     * still use the softmax over all N.  0 / 0: no nodes. */
    int32_t n_groups;
    int32_t topk_groups;
    int32_t overflow;        /* MOE_OVERFLOW_*; only matters with a capacity limit */
    int32_t slot_priority;   /* 0: capacity is filled token by token (t, then slot j);
                              * 1: slot by slot, every token's first choice before any
                              * token's second (priority for the top choices when k > 1) */
} moe_config;

/* Bytes of workspace every entry point below needs for `cfg` (0 on an invalid
 * configuration).  Host only, no CUDA calls. */
size_t moe_workspace_bytes(const moe_config *cfg);

/* Where moe_layer_forward keeps its intermediate dispatch results inside the
 * workspace, as byte offsets from the workspace start, so that a caller can
 * read the dispatch of the fused call ("MoE: what it costs to train and
 * serve", Expert parallelism step 1, as a local permutation) without running
 * the stages separately.  After a moe_layer_forward on that workspace has
 * completed on its stream, the regions hold that call's values, laid out as
 * the outputs of moe_dispatch of the same name; any later call on the
 * workspace may overwrite them.  topk_idx, topk_w and counts are filled only
 * when the caller passed NULL for the corresponding output of
 * moe_layer_forward.  Host only, no CUDA calls; MOE_ERR_INVALID_ARG on an
 * invalid configuration or a NULL `out`. */
typedef struct moe_workspace_regions {
    size_t topk_idx;   /* [T, k] int32 */
    size_t topk_w;     /* [T, k] fp32 */
    size_t counts;     /* [N] int32, before capacity */
    size_t offsets;    /* [N+1] int32 ([N+2] with MOE_OVERFLOW_FALLBACK) */
    size_t perm;       /* [T*k] int32, rows < R meaningful */
    size_t inv_row;    /* [T*k] int32, -1 for a dropped pair */
    size_t drop;       /* [T*k] uint8 */
    size_t x_scale;    /* [T*k] fp32 per kept row (FP8 dispatch only) */
    size_t x_gemm;     /* [T*k, d] the expert-ordered rows the expert GEMMs read, rows < R
                          meaningful: x's rows (dtype), or for FP8 dispatch the E4M3 codes'
                          values as bf16 (x_gemm * x_scale per row = the dequantised row) */
    size_t total;      /* = moe_workspace_bytes(cfg) */
} moe_workspace_regions;
moe_status moe_workspace_layout(const moe_config *cfg, moe_workspace_regions *out);

/* Stage 1, router ("moe communication costs", Router design; "Advanced GPU
 * Optimization ... Part 5", section 1.1).
 *   x        [T, d]  dtype
 *   Wg       [N, d]  dtype
 *   bias     [N] fp32 added to the logits, or NULL
 *   logits   [T, N] fp32 out, or NULL
 *   topk_idx [T, k] int32 out: slot 0 = largest logit
 *   topk_w   [T, k] fp32 out: gate weights of the selected experts
 *   p_mean   [N] fp32 out, or NULL: mean over tokens of the full softmax over
 *            N (the p_i of the aux loss)
 * Routing decisions are taken on logits accurate to about 1e-12 relative
 * (fp64 accumulation of the selected candidates), so ties are broken as the
 * exact arithmetic would break them. */
moe_status moe_router(const moe_config *cfg, const void *x, const void *Wg, const float *bias,
                      float *logits, int32_t *topk_idx, float *topk_w, float *p_mean,
                      void *workspace, size_t workspace_bytes, void *stream);

/* Stage 2, dispatch ("MoE: what it costs to train and serve", Expert
 * parallelism step 1, done as a local permutation; "moe communication costs",
 * Capacity factor and token dropping, Load balancing).
 *   x             [T, d] dtype
 *   topk_idx      [T, k] int32, values in [0, N) and distinct per token
 *   expert_counts [N] int32 out: pairs routed to each expert before dropping
 *   expert_offsets[N+1] int32 out: exclusive prefix sum of min(count, C); with
 *                 MOE_OVERFLOW_FALLBACK [N+2], the fallback expert's rows being
 *                 [offsets[N], offsets[N+1]) (R = offsets[N+1] = the pairs kept)
 *   perm          [T*k] int32 out: perm[row] = t*k + j for rows < R = offsets[N]
 *   inv_row       [T*k] int32 out: row of pair (t, j), or -1 if dropped
 *   drop_mask     [T*k] uint8 out: 1 if dropped (never with the fallback expert)
 *   x_perm        [T*k, d] out: row r = x[perm[r] / k]; dispatch_dtype
 *                 (FP8: E4M3 codes, one byte each)
 *   x_scale       [T*k] fp32 out for FP8 dispatch (per-token amax / 448), else NULL
 *   p_mean        [N] fp32 in (from moe_router) or NULL
 *   f             [N] fp32 out or NULL: count / (T*k)
 *   aux_loss      [1] fp32 out or NULL (needs p_mean): alpha * N * sum f_i p_mean_i
 * Within an expert, pairs are ordered by token index (slot_priority: by slot,
 * then token); when an expert gets more than C pairs the first C in that order
 * are kept, the rest dropped or (fallback) appended to the fallback expert's
 * rows in the same order.  Rows >= R of perm and x_perm are left untouched. */
moe_status moe_dispatch(const moe_config *cfg, const void *x, const int32_t *topk_idx,
                        int32_t *expert_counts, int32_t *expert_offsets, int32_t *perm,
                        int32_t *inv_row, uint8_t *drop_mask, void *x_perm, float *x_scale,
                        const float *p_mean, float *f, float *aux_loss,
                        void *workspace, size_t workspace_bytes, void *stream);

/* Dispatch without a workspace, for callers that cannot allocate device
 * memory for one: a host framework that owns all device memory through its
 * own pool, or a runtime with a fixed memory budget set up front, or a call
 * path where cudaMalloc/cudaFree are not acceptable because they may
 * synchronise the device.  (The pages have no counterpart to this entry
 * point; it is a deployment variant of moe_dispatch.)
 *
 * Arguments and results are those of moe_dispatch without the workspace.
 * The scratch the dispatch kernels keep between their launches (per-block
 * expert counts and a status word) lives instead in an array of about
 * 128 KiB compiled into this library, which every GPU that loads the library
 * holds until the process exits.  Limits: T*k <= 262144 pairs and N <= 256
 * experts; larger calls return MOE_ERR_WORKSPACE before anything is enqueued.
 * The library allocates nothing: no cudaMalloc, cudaFree or allocating
 * library routine.  The first call on each device looks up the device
 * address of the array (cudaGetSymbolAddress, with that device current), so
 * make that first call before any stream capture.  All calls on one device
 * share the array: calls that may run at the same time on the GPU (unordered
 * streams, several host threads) race and must be serialised by the caller.
 * An out-of-range expert index is dropped as in moe_dispatch but is not
 * reported, since there is no workspace status word to read. */
moe_status moe_dispatch_noalloc(const moe_config *cfg, const void *x, const int32_t *topk_idx,
                                int32_t *expert_counts, int32_t *expert_offsets, int32_t *perm,
                                int32_t *inv_row, uint8_t *drop_mask, void *x_perm,
                                float *x_scale, const float *p_mean, float *f, float *aux_loss,
                                void *stream);

/* Stage 3, expert FFNs as one grouped GEMM ("MoE: what it costs to train and
 * serve", Expert parallelism step 2).
 *   x_perm         [T*k, d] dispatch_dtype (rows >= offsets[N] are ignored)
 *   x_scale        [T*k] fp32 for FP8 dispatch, else NULL
 *   expert_offsets [N+1] int32 (device), segment e = rows [offsets[e], offsets[e+1]);
 *                  [N+2] with MOE_OVERFLOW_FALLBACK (expert N = the fallback)
 *   W1, W3, W2     stacked expert weights (W3 NULL for ReLU)
 *   y_perm         [T*k, d] dtype out; rows >= offsets[N] untouched
 * The hidden activations live in the workspace (bf16 for bf16 layers). */
moe_status moe_expert_ffn(const moe_config *cfg, const void *x_perm, const float *x_scale,
                          const int32_t *expert_offsets, const void *W1, const void *W3,
                          const void *W2, void *y_perm,
                          void *workspace, size_t workspace_bytes, void *stream);

/* Stage 3 for rows that arrive from several ranks ("MoE: what it costs to
 * train and serve", Expert parallelism and two all-to-alls, step 2: each GPU
 * runs its local experts on the tokens the first all-to-all brought it).
 * cfg->N is the number of experts held here; the rows come as n_src blocks,
 * one per sending rank, each grouped by these N experts.
 *   x_rows   [rows_cap, d] dispatch_dtype (FP8: E4M3 codes)
 *   x_scale  [rows_cap] fp32 for FP8 rows, else NULL
 *   offsets  [n_src*N + 1] int32 (device): the rows of source s for expert e
 *            are [offsets[s*N + e], offsets[s*N + e + 1]); group (s, e) uses
 *            weight block e of W1, W3, W2 (laid out as for moe_expert_ffn)
 *   y_rows   [rows_cap, d] dtype out; rows >= offsets[n_src*N] untouched
 *   rows_cap rows allocated in x_rows and y_rows, at most cfg->T * cfg->k (the
 *            workspace holds the hidden activations of that many rows: size
 *            cfg->T for the rows this rank can receive)
 * Requires 1 <= n_src and n_src * N <= 1024.  With MOE_OVERFLOW_FALLBACK in
 * cfg: MOE_ERR_UNSUPPORTED (place the fallback among the N local experts).
 * The pages have no counterpart to this entry point beyond the step above: it
 * exists so that the expert-parallel flow can run the local experts on rows
 * received from every rank in one launch per projection. */
moe_status moe_expert_ffn_multi(const moe_config *cfg, int32_t n_src, int64_t rows_cap,
                                const void *x_rows, const float *x_scale,
                                const int32_t *offsets, const void *W1, const void *W3,
                                const void *W2, void *y_rows, void *workspace,
                                size_t workspace_bytes, void *stream);

/* Stage 4, combine ("moe communication costs", Router design, the weighted
 * sum; "MoE: what it costs to train and serve", step 3).
 *   y_perm   [T*k, d] dtype
 *   inv_row  [T*k] int32 from moe_dispatch
 *   topk_w   [T, k] fp32
 *   y_shared [T, d] dtype added with coefficient 1, or NULL
 *   y        [T, d] dtype out: sum_j topk_w[t,j] * y_perm[inv_row[t*k+j]] over
 *            kept slots, in slot order, fp32 accumulation; a token whose slots
 *            are all dropped gets 0 (+ y_shared). */
moe_status moe_combine(const moe_config *cfg, const void *y_perm, const int32_t *inv_row,
                       const float *topk_w, const void *y_shared, void *y,
                       void *workspace, size_t workspace_bytes, void *stream);

/* All four stages, plus the shared expert when cfg->H_shared > 0 (run on the
 * unquantised x and added with coefficient 1).
 *   optional outputs (NULL to skip): topk_idx [T,k], topk_w [T,k],
 *   expert_counts [N], f [N], p_mean [N], aux_loss [1] (device). */
moe_status moe_layer_forward(const moe_config *cfg, const void *x, const void *Wg,
                             const float *bias, const void *W1, const void *W3, const void *W2,
                             const void *Ws1, const void *Ws3, const void *Ws2, void *y,
                             int32_t *topk_idx, float *topk_w, int32_t *expert_counts,
                             float *f, float *p_mean, float *aux_loss,
                             void *workspace, size_t workspace_bytes, void *stream);

/* Synchronises `stream`, reads and clears the device status word of the
 * workspace.  Returns MOE_OK, MOE_ERR_DEVICE_STATUS or MOE_ERR_TIMEOUT;
 * *detail (if not NULL) receives the raw word (bit meanings in the source). */
moe_status moe_check_status(void *workspace, void *stream, uint32_t *detail);

/* Static description of a status code. */
const char *moe_status_string(moe_status s);

/* Text of the last CUDA error seen by a call on this host thread. */
const char *moe_last_error_string(void);

/* ---- observability --------------------------------------------------- */

/* Number of CUDA kernels this library has launched in this process so far
 * (all entry points, all devices).  Host only. */
uint64_t moe_launch_count(void);

/* Per-stage timing of moe_layer_forward with CUDA events recorded on the
 * caller's stream between the stages.  moe_profile_begin(max_steps) starts
 * recording for up to max_steps calls (host only; creates the events);
 * moe_profile_end synchronises on the recorded events, writes the summed
 * milliseconds of each stage into stage_ms[MOE_PROFILE_STAGES] and the
 * number of recorded calls into *steps, and stops recording.  Stages:
 * 0 router, 1 dispatch, 2 expert up-projection (+ activation), 3 expert
 * down-projection, 4 shared expert, 5 combine. */
#define MOE_PROFILE_STAGES 6
moe_status moe_profile_begin(int max_steps);
moe_status moe_profile_end(float *stage_ms, int *steps);

/* Library version, e.g. "moe_b200 1.0 sm_100a". */
const char *moe_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
