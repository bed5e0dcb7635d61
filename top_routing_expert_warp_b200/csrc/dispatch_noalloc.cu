// moe_dispatch_noalloc: the dispatch stage for callers that cannot hand the
// library a workspace allocated with cudaMalloc.
//
// Some callers own every byte of device memory through their own pool (a
// host framework whose allocator must account for all memory, or a runtime
// with a fixed memory budget decided up front), and others cannot afford
// cudaMalloc/cudaFree on their call path because those calls may synchronise
// the device.  This variant therefore needs no workspace: the per-block
// expert counts that the dispatch kernels keep between their launches live in
// a fixed-size array compiled into this library.  The caller still passes all
// inputs and outputs.
//
// Limits and sharing: the array holds the counts of at most
// kNoAllocMaxPairs (token, slot) pairs for up to 256 experts (and the
// fallback expert's per-block bases), about 128 KiB per GPU, and every GPU that loads the library keeps it until the process
// exits.  All calls on a device share the one array, so calls whose work
// overlaps on the GPU (different streams without ordering, or several host
// threads at once) race with each other and must be serialised by the caller.
#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"

namespace {

constexpr int64_t kNoAllocMaxPairs = 1 << 18;   // T * k
constexpr int kNoAllocMaxExperts = 256;
constexpr int kNoAllocMaxBlocks = static_cast<int>(kNoAllocMaxPairs / moe::kDispChunk);
constexpr int kStatusInts = 64;                 // status word, padded to 256 bytes

// [0]: device status word; [kStatusInts ...]: per-block expert counts / bases,
// then per-block bases of the fallback expert's rows.
static __device__ __align__(256) int32_t
    g_noalloc_scratch[kStatusInts + kNoAllocMaxBlocks * kNoAllocMaxExperts + kNoAllocMaxBlocks];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t *g_scratch_ptr[kMaxDevices] = {};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" moe_status moe_dispatch_noalloc(const moe_config *cfg, const void *x,
                                           const int32_t *topk_idx, int32_t *expert_counts,
                                           int32_t *expert_offsets, int32_t *perm,
                                           int32_t *inv_row, uint8_t *drop_mask, void *x_perm,
                                           float *x_scale, const float *p_mean, float *f,
                                           float *aux_loss, void *stream)
{
    // configuration: same rules as moe_dispatch (workspace_bytes is 0 when invalid)
    if (!cfg || moe_workspace_bytes(cfg) == 0)
        return MOE_ERR_INVALID_ARG;
    if (!expert_counts || !expert_offsets)
        return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (!x || !topk_idx || !perm || !inv_row || !drop_mask || !x_perm ||
                       !aligned16(x) || !aligned16(x_perm)))
        return MOE_ERR_INVALID_ARG;
    if (cfg->dispatch_dtype == MOE_FP8_E4M3 && cfg->T > 0 && !x_scale)
        return MOE_ERR_INVALID_ARG;
    if (aux_loss && !p_mean)
        return MOE_ERR_INVALID_ARG;
    const int64_t pairs = cfg->T * cfg->k;
    if (pairs > kNoAllocMaxPairs || cfg->N > kNoAllocMaxExperts)
        return MOE_ERR_WORKSPACE;  // the built-in scratch is too small for this batch
    cudaStream_t s = static_cast<cudaStream_t>(stream);

    // once per device, with that device current: the device address of the array
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return MOE_ERR_CUDA;
    int32_t *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_scratch_ptr[dev]) {
            void *p = nullptr;
            if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess)
                return MOE_ERR_CUDA;
            g_scratch_ptr[dev] = static_cast<int32_t *>(p);
        }
        scratch = g_scratch_ptr[dev];
    }

    const int fallback = cfg->overflow == MOE_OVERFLOW_FALLBACK ? 1 : 0;
    if (pairs == 0) {
        if (cudaMemsetAsync(expert_counts, 0, cfg->N * sizeof(int32_t), s) != cudaSuccess ||
            cudaMemsetAsync(expert_offsets, 0, (cfg->N + 1 + fallback) * sizeof(int32_t), s) !=
                cudaSuccess ||
            (f && cudaMemsetAsync(f, 0, cfg->N * sizeof(float), s) != cudaSuccess) ||
            (aux_loss && cudaMemsetAsync(aux_loss, 0, sizeof(float), s) != cudaSuccess))
            return MOE_ERR_CUDA;
        return MOE_OK;
    }
    // the array keeps the previous call's contents: the status word must start
    // at zero (the per-block counts are fully rewritten before they are read)
    if (cudaMemsetAsync(scratch, 0, sizeof(int32_t), s) != cudaSuccess)
        return MOE_ERR_CUDA;

    moe::DispatchLaunch D{};
    D.dtype = cfg->dtype;
    D.fp8 = cfg->dispatch_dtype == MOE_FP8_E4M3;
    D.x = x;
    D.T = cfg->T;
    D.d = cfg->d;
    D.N = cfg->N;
    D.k = cfg->k;
    D.capacity = -1;
    if (cfg->capacity_factor > 0.0f)
        D.capacity = static_cast<int64_t>(static_cast<double>(cfg->capacity_factor) *
                                          static_cast<double>(cfg->T) /
                                          static_cast<double>(cfg->N));
    D.fallback = fallback;
    D.slot_priority = cfg->slot_priority;
    D.topk_idx = topk_idx;
    D.block_base = scratch + kStatusInts;
    D.counts = expert_counts;
    D.offsets = expert_offsets;
    D.perm = perm;
    D.inv_row = inv_row;
    D.drop = drop_mask;
    D.x_perm = x_perm;
    D.x_scale = x_scale;
    D.x_bf16_copy = nullptr;
    D.p_mean = p_mean;
    D.f = f;
    D.aux_loss = aux_loss;
    D.aux_alpha = cfg->aux_alpha;
    D.status = reinterpret_cast<uint32_t *>(scratch);
    if (moe::launch_dispatch(D, s) != cudaSuccess)
        return MOE_ERR_CUDA;
    return MOE_OK;
}
