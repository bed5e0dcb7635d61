// Host-side launchers of the libmoe_b200 kernels (internal interface between
// the C ABI layer and the kernel files).
#pragma once

#include <cstdint>
#include <mutex>
#include <utility>
#include <cuda_runtime.h>

namespace moe {

// Every kernel of the library is launched with programmatic dependent launch:
// it may be scheduled while the previous kernel on the stream drains, and it
// waits (griddepcontrol.wait, first thing in every kernel) until that kernel
// has completed and its writes are visible.  This hides the launch gap
// between the short kernels of a layer forward.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_k(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                           cudaStream_t stream, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Count of kernel launches made by the library (reported by moe_launch_count).
void count_launches(int n);

// One-time set-up per device.  CUDA keeps function attributes (the dynamic
// shared-memory bound) and occupancy for each device separately, so a value
// cached for the first device a process used is wrong on a second one.
// device_once runs init(&value) the first time it is reached with a given
// device current, under a lock, and afterwards returns that device's value.
constexpr int kMaxDeviceSlots = 64;
struct DeviceOnce {
    std::mutex mu;
    bool done[kMaxDeviceSlots] = {};
    int value[kMaxDeviceSlots] = {};
};
template <typename F>
inline cudaError_t device_once(DeviceOnce &once, int *value_out, F init)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDeviceSlots)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(once.mu);
    if (!once.done[dev]) {
        int v = 0;
        e = init(&v);
        if (e != cudaSuccess)
            return e;
        once.value[dev] = v;
        once.done[dev] = true;
    }
    if (value_out)
        *value_out = once.value[dev];
    return cudaSuccess;
}

enum EpiKind { EPI_STORE = 0, EPI_RELU = 1, EPI_SWIGLU = 2 };

// Grouped GEMM on tcgen05 tensor cores: see gemm_tc.cu.
struct GemmLaunch {
    int epi;                 // EpiKind
    bool out_f32;            // fp32 output (router logits) instead of bf16
    const void *A;           // [a_rows, K] bf16
    int64_t a_rows;
    int32_t K;
    const void *B;           // [b_rows, K] bf16 (groups stacked: g * n_out + n)
    const void *B2;          // second weight (W3) for SwiGLU, same shape as B
    int64_t b_rows;
    const int32_t *offsets;  // [G+1] device row offsets, or null for one group of rows_single
    int32_t rows_single;
    int32_t G;
    int32_t w_blocks;        // weight blocks in B: group g uses block g % w_blocks (0: g)
    int32_t n_out;
    void *out;               // [out_rows, ld_out]
    int64_t out_rows;
    int64_t ld_out;
    const float *row_scale;  // [a_rows] or null
    int32_t ksplit;          // >1: K split into ksplit slices (fp32 partial outputs)
    int64_t split_stride;    // elements between the partial outputs of two slices
    uint32_t *status;
    // One-CTA kernel: weights of groups of at most two m tiles are read once or
    // twice in a row: load them evict-first from L2 and the rows evict-last.
    int32_t stream_hint;
};
// K slices the router GEMM uses so that its tiles cover the SMs, at most
// router_ksplit_cap(T, N) (which sizes the workspace's partial-logit buffer).
int router_ksplit(int64_t T, int32_t N, int32_t d);
constexpr int kRouterMaxSplit = 32;
constexpr int64_t kRouterPartialBudget = int64_t(1) << 24;   // fp32 partial logits
inline int router_ksplit_cap(int64_t T, int32_t N)
{
    const int64_t tn = T * N;
    if (tn <= 0)
        return 1;
    int64_t c = kRouterPartialBudget / tn;
    if (c > kRouterMaxSplit)
        c = kRouterMaxSplit;
    return c < 1 ? 1 : static_cast<int>(c);
}
cudaError_t launch_grouped_gemm(const GemmLaunch &L, cudaStream_t stream);
// Same contract on CTA pairs (256-row tiles, tcgen05 cta_group::2), bf16 output,
// no K split: see gemm_tc2.cu.  For compute-bound shapes (many rows per group).
cudaError_t launch_grouped_gemm_pair(const GemmLaunch &L, cudaStream_t stream);
// Rows per group from which the pair kernel is used.
constexpr int64_t kPairMinRowsPerGroup = 512;
// Same contract on CTA pairs with the weights as the MMA's M (tiles of up to
// 160 rows of one group against 512 weight rows), for the HBM-bound grouped
// projections below kPairMinRowsPerGroup; needs offsets: see gemm_tc2t.cu.
cudaError_t launch_grouped_gemm_pairt(const GemmLaunch &L, cudaStream_t stream);

// fp32 CUDA-core grouped GEMM (fp32 layers): see ffn_simt.cu.
cudaError_t launch_simt_gemm_f32(int epi, const float *A, int64_t rows_cap, int32_t K,
                                 const float *B, const float *B2, int32_t n_out,
                                 const int32_t *offsets, int32_t G, int32_t w_blocks,
                                 int32_t rows_single, float *out, cudaStream_t stream);

// The whole forward of a small fp32 layer in one launch: see layer_small.cu.
// Used for fp32 layers without a capacity limit when layer_small_fits().
struct LayerSmallLaunch {
    const float *x, *Wg, *bias, *W1, *W3, *W2, *Ws1, *Ws3, *Ws2;   // W3 / Ws*: may be null
    float *y;
    int64_t T;
    int32_t d, N, k, H, Hs;
    int32_t gate_mode, renormalize, n_groups, topk_groups, swiglu, slot_priority;
    float alpha;
    int32_t *topk_idx;
    float *topk_w;
    double *p_part;          // [blocks, N] workspace
    uint32_t *ticket;        // workspace word, 0 between calls
    int32_t *counts, *offsets, *perm, *inv_row;
    uint8_t *drop;
    float *p_mean, *f, *aux_loss;   // may be null
    uint32_t *status;
};
constexpr int64_t kSmallMaxPairs = 8192;
constexpr size_t kSmallMaxSmem = 96 * 1024;
bool layer_small_fits(const LayerSmallLaunch &L);
cudaError_t launch_layer_small(const LayerSmallLaunch &L, cudaStream_t stream);

// Router: see router.cu.
struct RouterLaunch {
    int dtype;               // MOE_F32 / MOE_BF16
    const void *x;
    const void *Wg;
    const float *bias;
    int64_t T;
    int32_t d, N, k;
    int32_t gate_mode, renormalize;
    int32_t n_groups, topk_groups;   // node-limited routing (0 / 0: off), checked by the ABI
    const float *logits_in;  // large-N path: fp32 partial logits [ksplit][T][N] from the GEMM
    int32_t ksplit;          // number of partial logit slices
    float *logits_out;       // optional fp32 logits (small-N path)
    int32_t *topk_idx;
    float *topk_w;
    double *p_part;          // [router_blocks, N] per-block sums of the full softmax
    int32_t *p_blocks;       // out: number of blocks used (host value, written by launcher)
    uint32_t *status;
};
constexpr int kRouterMaxBlocks = 1184;
constexpr int kRouterSmallMaxN = 16;
cudaError_t launch_router_small(RouterLaunch &L, cudaStream_t stream);
cudaError_t launch_router_select(RouterLaunch &L, cudaStream_t stream);
// p_mean[e] = sum over blocks of p_part[b][e] / T, summed in block order.
cudaError_t launch_p_finalize(const double *p_part, int32_t p_blocks, int32_t N, int64_t T,
                              float *p_mean, cudaStream_t stream);

// Dispatch: see dispatch.cu.
constexpr int kDispChunk = 2048;      // (token, slot) pairs per block
// Batches of at most kFusedMaxPairs pairs over at most kFusedMaxN experts are
// sorted by one block in one launch (expert ids staged in shared memory).
constexpr int64_t kFusedMaxPairs = 8192;
constexpr int kFusedMaxN = 256;
struct DispatchLaunch {
    int dtype;                // element type of x
    int fp8;                  // quantise rows to E4M3 + per-row scale
    const void *x;
    int64_t T;
    int32_t d, N, k;
    int64_t capacity;         // -1 = unlimited
    int fallback;             // pairs over capacity go to group N (offsets has N + 2 entries)
    int slot_priority;        // pairs taken slot by slot instead of token by token
    const int32_t *topk_idx;
    int32_t *block_base;      // [nblk, N] workspace, then [nblk] fallback bases
    int32_t *counts;          // [N]
    int32_t *offsets;         // [N+1]
    int32_t *perm;            // [T*k]
    int32_t *inv_row;         // [T*k]
    uint8_t *drop;            // [T*k]
    void *x_perm;             // [T*k, d]
    float *x_scale;           // [T*k] (fp8)
    void *x_bf16_copy;        // optional [T*k, d] bf16 of the fp8 codes (GEMM operand)
    const float *p_mean;      // optional in [N] (router output), needed for aux_loss
    float *f;                 // optional out [N]
    float *aux_loss;          // optional out [1]
    float aux_alpha;
    uint32_t *status;
};
cudaError_t launch_dispatch(const DispatchLaunch &L, cudaStream_t stream);
// FP8 payload of token t written to every kept row r = inv_row[t k + j]:
// out[r] = E4M3 codes of x[t] / scale as bf16, out_scale[r] = scale = amax/448.
cudaError_t launch_quantize_scatter(const void *x, int64_t T, int32_t d, int32_t k,
                                    const int32_t *inv_row, void *out, float *out_scale,
                                    cudaStream_t stream);
// E4M3 codes -> bf16 (exact) for rows < offsets[N].
cudaError_t launch_fp8_to_bf16(const uint8_t *q, int64_t rows_cap, int32_t d,
                               const int32_t *offsets, int32_t N, void *out, cudaStream_t stream);

// Combine: see combine.cu.
cudaError_t launch_combine(int dtype, const void *y_perm, const int32_t *inv_row,
                           const float *topk_w, const void *y_shared, void *y, int64_t T,
                           int32_t d, int32_t k, uint32_t *status, cudaStream_t stream);

}  // namespace moe
