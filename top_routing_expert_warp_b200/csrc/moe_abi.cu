// C ABI of libmoe_b200 (declared in include/moe.h): argument validation,
// workspace layout and the launch sequence of each stage.  No kernel code.
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"

namespace moe {
static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n)); }
}  // namespace moe

namespace {

thread_local char g_last_error[256] = "";

// Stage timing of moe_layer_forward (moe_profile_begin / moe_profile_end).
// Boundary b of a call is recorded before stage b starts; boundary 6 after
// the combine.  Stages that a call does not run record back-to-back events.
constexpr int kMarks = MOE_PROFILE_STAGES + 1;
struct Profiler {
    std::mutex mu;
    bool on = false;
    int max_steps = 0;
    int steps = 0;
    std::vector<cudaEvent_t> ev;
};
Profiler g_prof;

void prof_mark(int boundary, cudaStream_t s)
{
    if (!g_prof.on || g_prof.steps >= g_prof.max_steps)
        return;
    cudaEventRecord(g_prof.ev[static_cast<size_t>(g_prof.steps) * kMarks + boundary], s);
}

moe_status cuda_fail(cudaError_t e)
{
    std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e),
                  cudaGetErrorString(e));
    return MOE_ERR_CUDA;
}

#define MOE_CUDA(call)                          \
    do {                                        \
        cudaError_t e_ = (call);                \
        if (e_ != cudaSuccess)                  \
            return cuda_fail(e_);               \
    } while (0)

size_t up256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

int elem_size(int dt) { return dt == MOE_F32 ? 4 : (dt == MOE_BF16 ? 2 : 1); }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Offsets of the workspace regions (bytes from the workspace start).
struct Layout {
    size_t status, p_part, logits, topk_idx, topk_w, p_mean, counts, offsets, block_base, perm,
        inv_row, drop, x_scale, x_gemm, h, y_perm, hs, ys, total;
};

// Node-limited routing in effect: more than one node and fewer allowed.
bool node_limited(const moe_config &c)
{
    return c.n_groups > 1 && c.topk_groups < c.n_groups;
}

// Pairs over capacity go to the fallback expert N (one more expert group).
bool has_fallback(const moe_config &c)
{
    return c.overflow == MOE_OVERFLOW_FALLBACK;
}

// Expert groups of the FFN: the routed experts, plus the fallback.
int32_t ffn_groups(const moe_config &c)
{
    return c.N + (has_fallback(c) ? 1 : 0);
}

bool config_ok(const moe_config *c)
{
    if (!c)
        return false;
    if (c->T < 0 || c->d <= 0 || c->N < 1 || c->N > 256 || c->k < 1 || c->k > 8 || c->k > c->N ||
        c->H <= 0 || c->H_shared < 0)
        return false;
    if (c->dtype != MOE_F32 && c->dtype != MOE_BF16)
        return false;
    if (c->dispatch_dtype != c->dtype &&
        !(c->dispatch_dtype == MOE_FP8_E4M3 && c->dtype == MOE_BF16))
        return false;
    if (c->act != MOE_ACT_RELU && c->act != MOE_ACT_SWIGLU)
        return false;
    if (c->gate_mode != MOE_GATE_TOPK_THEN_SOFTMAX && c->gate_mode != MOE_GATE_SOFTMAX_THEN_TOPK)
        return false;
    if (c->renormalize != 0 && c->renormalize != 1)
        return false;
    const int align = (c->dtype == MOE_BF16) ? 8 : 4;
    if (c->d % align || c->H % align || c->H_shared % align)
        return false;
    if (c->T * c->k > 0x7FFFFFFFll)
        return false;
    if (c->n_groups < 0 || c->topk_groups < 0)
        return false;
    if ((c->overflow != MOE_OVERFLOW_DROP && c->overflow != MOE_OVERFLOW_FALLBACK) ||
        (c->slot_priority != 0 && c->slot_priority != 1))
        return false;
    if (node_limited(*c)) {
        if (c->n_groups > 32 || c->N % c->n_groups != 0 || c->topk_groups < 1 ||
            c->k > c->topk_groups * (c->N / c->n_groups))
            return false;
    }
    if (c->dtype == MOE_F32) {
        // fp32 layers: CUDA-core router (N <= 16) and a row-staged SIMT GEMM
        if (c->N > moe::kRouterSmallMaxN || c->d > 12288 || c->H > 12288 || c->H_shared > 12288)
            return false;
    }
    return true;
}

Layout layout_of(const moe_config &c)
{
    Layout L{};
    const size_t T = static_cast<size_t>(c.T), N = c.N, k = c.k, d = c.d, H = c.H;
    const size_t rows = T * k;
    const size_t es = elem_size(c.dtype);
    const size_t nblk = (rows + moe::kDispChunk - 1) / moe::kDispChunk;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o += up256(bytes);
        return at;
    };
    L.status = take(256);
    L.p_part = take(static_cast<size_t>(moe::kRouterMaxBlocks) * N * sizeof(double));
    L.logits = take(c.dtype == MOE_BF16
                        ? static_cast<size_t>(moe::router_ksplit_cap(c.T, c.N)) * T * N * 4 : 0);
    L.topk_idx = take(rows * 4);
    L.topk_w = take(rows * 4);
    L.p_mean = take(N * 4);
    L.counts = take(N * 4);
    L.offsets = take((N + 2) * 4);
    L.block_base = take(nblk * N * 4 + nblk * 4);   // per-block expert bases, fallback bases
    L.perm = take(rows * 4);
    L.inv_row = take(rows * 4);
    L.drop = take(rows);
    L.x_scale = take(rows * 4);
    const bool fp8 = c.dispatch_dtype == MOE_FP8_E4M3;
    L.x_gemm = take(rows * d * (fp8 ? 2 : static_cast<size_t>(elem_size(c.dtype))));  // GEMM rows
    L.h = take(rows * H * es);
    L.y_perm = take(rows * d * es);
    L.hs = take(c.H_shared > 0 ? T * static_cast<size_t>(c.H_shared) * es : 0);
    L.ys = take(c.H_shared > 0 ? T * d * es : 0);
    L.total = o;
    return L;
}

struct Ws {
    uint8_t *base;
    Layout L;
    template <typename P>
    P *at(size_t off) const
    {
        return reinterpret_cast<P *>(base + off);
    }
    uint32_t *status() const { return at<uint32_t>(L.status); }
};

moe_status check_ws(const moe_config *c, void *ws, size_t ws_bytes, Ws *out)
{
    if (!ws || !aligned(ws, 256))
        return MOE_ERR_WORKSPACE;
    Layout L = layout_of(*c);
    if (ws_bytes < L.total)
        return MOE_ERR_WORKSPACE;
    out->base = static_cast<uint8_t *>(ws);
    out->L = L;
    return MOE_OK;
}

// ---------------------------------------------------------------- stages
moe_status run_router(const moe_config &c, const void *x, const void *Wg, const float *bias,
                      float *logits, int32_t *topk_idx, float *topk_w, float *p_mean,
                      const Ws &w, cudaStream_t s)
{
    // with nodes, plain mode F would weigh excluded experts' tensor-core logits in
    // its softmax denominator without recomputing them
    if (node_limited(c) && c.gate_mode == MOE_GATE_SOFTMAX_THEN_TOPK && !c.renormalize)
        return MOE_ERR_UNSUPPORTED;
    if (c.T == 0) {
        if (p_mean)
            MOE_CUDA(cudaMemsetAsync(p_mean, 0, c.N * sizeof(float), s));
        return MOE_OK;
    }
    moe::RouterLaunch R{};
    int32_t blocks = 0;
    R.dtype = c.dtype;
    R.x = x;
    R.Wg = Wg;
    R.bias = bias;
    R.T = c.T;
    R.d = c.d;
    R.N = c.N;
    R.k = c.k;
    R.gate_mode = c.gate_mode;
    R.renormalize = c.renormalize;
    R.n_groups = node_limited(c) ? c.n_groups : 0;
    R.topk_groups = node_limited(c) ? c.topk_groups : 0;
    R.topk_idx = topk_idx;
    R.topk_w = topk_w;
    R.p_part = w.at<double>(w.L.p_part);
    R.p_blocks = &blocks;
    R.status = w.status();
    if (c.dtype == MOE_F32) {
        // fp32 layers (small N): CUDA cores, exact fp64 products
        R.logits_out = logits;
        MOE_CUDA(moe::launch_router_small(R, s));
    } else {
        // logits = sum of ksplit fp32 partial GEMMs over slices of d (so the
        // tiles cover the SMs), summed in slice order by the selection kernel
        float *part = w.at<float>(w.L.logits);
        const int ks = moe::router_ksplit(c.T, c.N, c.d);
        moe::GemmLaunch G{};
        G.epi = moe::EPI_STORE;
        G.out_f32 = true;
        G.A = x;
        G.a_rows = c.T;
        G.K = c.d;
        G.B = Wg;
        G.B2 = nullptr;
        G.b_rows = c.N;
        G.offsets = nullptr;
        G.rows_single = static_cast<int32_t>(c.T);
        G.G = 1;
        G.n_out = c.N;
        G.out = part;
        G.out_rows = c.T;
        G.ld_out = c.N;
        G.row_scale = nullptr;
        G.ksplit = ks;
        G.split_stride = c.T * c.N;
        G.status = w.status();
        MOE_CUDA(moe::launch_grouped_gemm(G, s));
        R.logits_in = part;
        R.ksplit = ks;
        R.logits_out = logits;
        MOE_CUDA(moe::launch_router_select(R, s));
    }
    if (p_mean)
        MOE_CUDA(moe::launch_p_finalize(R.p_part, blocks, c.N, c.T, p_mean, s));
    return MOE_OK;
}

moe_status run_dispatch(const moe_config &c, const void *x, const int32_t *topk_idx,
                        int32_t *counts, int32_t *offsets, int32_t *perm, int32_t *inv_row,
                        uint8_t *drop, void *x_perm, float *x_scale, void *x_bf16_copy,
                        const float *p_mean, float *f, float *aux_loss, const Ws &w,
                        cudaStream_t s)
{
    if (c.T == 0) {
        MOE_CUDA(cudaMemsetAsync(counts, 0, c.N * sizeof(int32_t), s));
        MOE_CUDA(cudaMemsetAsync(offsets, 0, (ffn_groups(c) + 1) * sizeof(int32_t), s));
        if (f)
            MOE_CUDA(cudaMemsetAsync(f, 0, c.N * sizeof(float), s));
        if (aux_loss)
            MOE_CUDA(cudaMemsetAsync(aux_loss, 0, sizeof(float), s));
        return MOE_OK;
    }
    moe::DispatchLaunch D{};
    D.dtype = c.dtype;
    D.fp8 = c.dispatch_dtype == MOE_FP8_E4M3;
    D.x = x;
    D.T = c.T;
    D.d = c.d;
    D.N = c.N;
    D.k = c.k;
    D.capacity = -1;
    if (c.capacity_factor > 0.0f)
        D.capacity = static_cast<int64_t>(static_cast<double>(c.capacity_factor) *
                                          static_cast<double>(c.T) / static_cast<double>(c.N));
    D.fallback = has_fallback(c) ? 1 : 0;
    D.slot_priority = c.slot_priority;
    D.topk_idx = topk_idx;
    D.block_base = w.at<int32_t>(w.L.block_base);
    D.counts = counts;
    D.offsets = offsets;
    D.perm = perm;
    D.inv_row = inv_row;
    D.drop = drop;
    D.x_perm = x_perm;
    D.x_scale = x_scale;
    D.x_bf16_copy = x_bf16_copy;
    D.p_mean = p_mean;
    D.f = f;
    D.aux_loss = aux_loss;
    D.aux_alpha = c.aux_alpha;
    D.status = w.status();
    MOE_CUDA(moe::launch_dispatch(D, s));
    return MOE_OK;
}

// Whether the expert FFN of `rows_cap` rows over G groups runs on CTA pairs.
bool ffn_on_pairs(int64_t rows_cap, int32_t G)
{
    return rows_cap >= moe::kPairMinRowsPerGroup * G;
}

// Dense FFN over grouped rows: up (with activation) into h, down into out.
// Group g of the rows uses weight block g % w_blocks (w_blocks = 0: block g).
moe_status run_ffn(const moe_config &c, const void *A, const float *row_scale, int64_t rows_cap,
                   const int32_t *offsets, int32_t G, int32_t rows_single, int32_t H,
                   const void *W1, const void *W3, const void *W2, void *h, void *out,
                   uint32_t *status, cudaStream_t s, int mark_between = -1, int32_t w_blocks = 0)
{
    if (rows_cap == 0)
        return MOE_OK;
    const int32_t wb = w_blocks > 0 ? w_blocks : G;
    const int epi = c.act == MOE_ACT_SWIGLU ? moe::EPI_SWIGLU : moe::EPI_RELU;
    if (c.dtype == MOE_F32) {
        MOE_CUDA(moe::launch_simt_gemm_f32(epi, static_cast<const float *>(A), rows_cap, c.d,
                                           static_cast<const float *>(W1),
                                           static_cast<const float *>(W3), H, offsets, G, wb,
                                           rows_single, static_cast<float *>(h), s));
        if (mark_between >= 0)
            prof_mark(mark_between, s);
        MOE_CUDA(moe::launch_simt_gemm_f32(moe::EPI_STORE, static_cast<const float *>(h), rows_cap,
                                           H, static_cast<const float *>(W2), nullptr, c.d,
                                           offsets, G, wb, rows_single, static_cast<float *>(out),
                                           s));
        return MOE_OK;
    }
    moe::GemmLaunch U{};
    U.epi = epi;
    U.out_f32 = false;
    U.A = A;
    U.a_rows = rows_cap;
    U.K = c.d;
    U.B = W1;
    U.B2 = W3;
    U.b_rows = static_cast<int64_t>(wb) * H;
    U.offsets = offsets;
    U.rows_single = rows_single;
    U.G = G;
    U.w_blocks = wb;
    U.n_out = H;
    U.out = h;
    U.out_rows = rows_cap;
    U.ld_out = H;
    U.row_scale = row_scale;
    U.status = status;
    // compute-bound expert projections (many rows per expert) run on CTA pairs;
    // grouped HBM-bound ones on transposed CTA pairs (weights as the MMA's M),
    // except with a fallback expert: its one group of thousands of rows runs
    // faster on the one-CTA kernel (m tiles sharing each weight tile through
    // L2, which the evict-first weights of the small groups leave it)
    const bool pair = ffn_on_pairs(rows_cap, G);
    const bool pairt = !pair && offsets != nullptr && !has_fallback(c);
    // the down-projection's K is H, often short: with experts of more than 64
    // rows on average, many transposed tiles hold both TMEM slots (129-160
    // rows) through their epilogue, which then weighs on tiles of few K steps;
    // the one-CTA kernel's double buffer was faster there (DeepSeek-shaped
    // down-projection 1.59 -> 1.53 ms)
    const bool pairt_down = pairt && rows_cap <= 64 * static_cast<int64_t>(G);
    auto launch = [&](const moe::GemmLaunch &L, bool t) {
        return pair ? moe::launch_grouped_gemm_pair(L, s)
                    : (t ? moe::launch_grouped_gemm_pairt(L, s) : moe::launch_grouped_gemm(L, s));
    };
    // groups of at most two 128-row tiles read their weight tiles once or twice
    // in a row: stream those weights past L2 (evict-first)
    const int32_t hint = (!pair && offsets != nullptr && rows_cap <= 256 * static_cast<int64_t>(G))
                             ? 1 : 0;
    U.stream_hint = hint;
    MOE_CUDA(launch(U, pairt));
    if (mark_between >= 0)
        prof_mark(mark_between, s);
    moe::GemmLaunch Dn{};
    Dn.epi = moe::EPI_STORE;
    Dn.out_f32 = false;
    Dn.A = h;
    Dn.a_rows = rows_cap;
    Dn.K = H;
    Dn.B = W2;
    Dn.B2 = nullptr;
    Dn.b_rows = static_cast<int64_t>(wb) * c.d;
    Dn.offsets = offsets;
    Dn.rows_single = rows_single;
    Dn.G = G;
    Dn.w_blocks = wb;
    Dn.n_out = c.d;
    Dn.out = out;
    Dn.out_rows = rows_cap;
    Dn.ld_out = c.d;
    Dn.row_scale = nullptr;
    Dn.status = status;
    Dn.stream_hint = hint;
    MOE_CUDA(launch(Dn, pairt_down));
    return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_workspace_bytes(const moe_config *cfg)
{
    if (!config_ok(cfg))
        return 0;
    return layout_of(*cfg).total;
}

moe_status moe_workspace_layout(const moe_config *cfg, moe_workspace_regions *out)
{
    if (!config_ok(cfg) || !out)
        return MOE_ERR_INVALID_ARG;
    const Layout L = layout_of(*cfg);
    out->topk_idx = L.topk_idx;
    out->topk_w = L.topk_w;
    out->counts = L.counts;
    out->offsets = L.offsets;
    out->perm = L.perm;
    out->inv_row = L.inv_row;
    out->drop = L.drop;
    out->x_scale = L.x_scale;
    out->x_gemm = L.x_gemm;
    out->total = L.total;
    return MOE_OK;
}

moe_status moe_router(const moe_config *cfg, const void *x, const void *Wg, const float *bias,
                      float *logits, int32_t *topk_idx, float *topk_w, float *p_mean,
                      void *workspace, size_t workspace_bytes, void *stream)
{
    if (!config_ok(cfg))
        return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (!x || !Wg || !topk_idx || !topk_w || !aligned(x, 16) || !aligned(Wg, 16)))
        return MOE_ERR_INVALID_ARG;
    if (logits && !aligned(logits, 16))
        return MOE_ERR_INVALID_ARG;
    Ws w;
    moe_status st = check_ws(cfg, workspace, workspace_bytes, &w);
    if (st != MOE_OK)
        return st;
    return run_router(*cfg, x, Wg, bias, logits, topk_idx, topk_w, p_mean, w,
                      static_cast<cudaStream_t>(stream));
}

moe_status moe_dispatch(const moe_config *cfg, const void *x, const int32_t *topk_idx,
                        int32_t *expert_counts, int32_t *expert_offsets, int32_t *perm,
                        int32_t *inv_row, uint8_t *drop_mask, void *x_perm, float *x_scale,
                        const float *p_mean, float *f, float *aux_loss,
                        void *workspace, size_t workspace_bytes, void *stream)
{
    if (!config_ok(cfg))
        return MOE_ERR_INVALID_ARG;
    if (!expert_counts || !expert_offsets)
        return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (!x || !topk_idx || !perm || !inv_row || !drop_mask || !x_perm ||
                       !aligned(x, 16) || !aligned(x_perm, 16)))
        return MOE_ERR_INVALID_ARG;
    if (cfg->dispatch_dtype == MOE_FP8_E4M3 && cfg->T > 0 && !x_scale)
        return MOE_ERR_INVALID_ARG;
    if (aux_loss && !p_mean)
        return MOE_ERR_INVALID_ARG;
    Ws w;
    moe_status st = check_ws(cfg, workspace, workspace_bytes, &w);
    if (st != MOE_OK)
        return st;
    return run_dispatch(*cfg, x, topk_idx, expert_counts, expert_offsets, perm, inv_row,
                        drop_mask, x_perm, x_scale, nullptr, p_mean, f, aux_loss, w,
                        static_cast<cudaStream_t>(stream));
}

moe_status moe_expert_ffn(const moe_config *cfg, const void *x_perm, const float *x_scale,
                          const int32_t *expert_offsets, const void *W1, const void *W3,
                          const void *W2, void *y_perm,
                          void *workspace, size_t workspace_bytes, void *stream)
{
    if (!config_ok(cfg))
        return MOE_ERR_INVALID_ARG;
    const bool swiglu = cfg->act == MOE_ACT_SWIGLU;
    if (cfg->T > 0 && (!x_perm || !expert_offsets || !W1 || !W2 || !y_perm || (swiglu && !W3) ||
                       !aligned(x_perm, 16) || !aligned(W1, 16) || !aligned(W2, 16) ||
                       (swiglu && !aligned(W3, 16)) || !aligned(y_perm, 16)))
        return MOE_ERR_INVALID_ARG;
    const bool fp8 = cfg->dispatch_dtype == MOE_FP8_E4M3;
    if (fp8 && cfg->T > 0 && !x_scale)
        return MOE_ERR_INVALID_ARG;
    Ws w;
    moe_status st = check_ws(cfg, workspace, workspace_bytes, &w);
    if (st != MOE_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t rows_cap = cfg->T * cfg->k;
    const void *A = x_perm;
    if (fp8 && rows_cap > 0) {
        MOE_CUDA(moe::launch_fp8_to_bf16(static_cast<const uint8_t *>(x_perm), rows_cap, cfg->d,
                                         expert_offsets, ffn_groups(*cfg), w.at<void>(w.L.x_gemm),
                                         s));
        A = w.at<void>(w.L.x_gemm);
    }
    return run_ffn(*cfg, A, fp8 ? x_scale : nullptr, rows_cap, expert_offsets, ffn_groups(*cfg), 0,
                   cfg->H,
                   W1, swiglu ? W3 : nullptr, W2, w.at<void>(w.L.h), y_perm, w.status(), s);
}

moe_status moe_expert_ffn_multi(const moe_config *cfg, int32_t n_src, int64_t rows_cap,
                                const void *x_rows, const float *x_scale,
                                const int32_t *offsets, const void *W1, const void *W3,
                                const void *W2, void *y_rows, void *workspace,
                                size_t workspace_bytes, void *stream)
{
    if (!config_ok(cfg))
        return MOE_ERR_INVALID_ARG;
    if (n_src < 1 || static_cast<int64_t>(n_src) * cfg->N > 1024 || rows_cap < 0 ||
        rows_cap > cfg->T * cfg->k)
        return MOE_ERR_INVALID_ARG;
    if (has_fallback(*cfg))
        return MOE_ERR_UNSUPPORTED;
    const bool swiglu = cfg->act == MOE_ACT_SWIGLU;
    if (rows_cap > 0 && (!x_rows || !offsets || !W1 || !W2 || !y_rows || (swiglu && !W3) ||
                         !aligned(x_rows, 16) || !aligned(W1, 16) || !aligned(W2, 16) ||
                         (swiglu && !aligned(W3, 16)) || !aligned(y_rows, 16)))
        return MOE_ERR_INVALID_ARG;
    const bool fp8 = cfg->dispatch_dtype == MOE_FP8_E4M3;
    if (fp8 && rows_cap > 0 && !x_scale)
        return MOE_ERR_INVALID_ARG;
    Ws w;
    moe_status st = check_ws(cfg, workspace, workspace_bytes, &w);
    if (st != MOE_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int32_t groups = n_src * cfg->N;
    const void *A = x_rows;
    if (fp8 && rows_cap > 0) {
        MOE_CUDA(moe::launch_fp8_to_bf16(static_cast<const uint8_t *>(x_rows), rows_cap, cfg->d,
                                         offsets, groups, w.at<void>(w.L.x_gemm), s));
        A = w.at<void>(w.L.x_gemm);
    }
    return run_ffn(*cfg, A, fp8 ? x_scale : nullptr, rows_cap, offsets, groups, 0, cfg->H, W1,
                   swiglu ? W3 : nullptr, W2, w.at<void>(w.L.h), y_rows, w.status(), s, -1,
                   cfg->N);
}

moe_status moe_combine(const moe_config *cfg, const void *y_perm, const int32_t *inv_row,
                       const float *topk_w, const void *y_shared, void *y,
                       void *workspace, size_t workspace_bytes, void *stream)
{
    if (!config_ok(cfg))
        return MOE_ERR_INVALID_ARG;
    if (cfg->T > 0 && (!y_perm || !inv_row || !topk_w || !y || !aligned(y_perm, 16) ||
                       !aligned(y, 16) || (y_shared && !aligned(y_shared, 16))))
        return MOE_ERR_INVALID_ARG;
    Ws w;
    moe_status st = check_ws(cfg, workspace, workspace_bytes, &w);
    if (st != MOE_OK)
        return st;
    MOE_CUDA(moe::launch_combine(cfg->dtype, y_perm, inv_row, topk_w, y_shared, y, cfg->T, cfg->d,
                                 cfg->k, w.status(), static_cast<cudaStream_t>(stream)));
    return MOE_OK;
}

moe_status moe_layer_forward(const moe_config *cfg, const void *x, const void *Wg,
                             const float *bias, const void *W1, const void *W3, const void *W2,
                             const void *Ws1, const void *Ws3, const void *Ws2, void *y,
                             int32_t *topk_idx, float *topk_w, int32_t *expert_counts,
                             float *f, float *p_mean, float *aux_loss,
                             void *workspace, size_t workspace_bytes, void *stream)
{
    if (!config_ok(cfg))
        return MOE_ERR_INVALID_ARG;
    const moe_config &c = *cfg;
    const bool swiglu = c.act == MOE_ACT_SWIGLU;
    const bool shared = c.H_shared > 0;
    if (c.T > 0) {
        if (!x || !Wg || !W1 || !W2 || !y || (swiglu && !W3))
            return MOE_ERR_INVALID_ARG;
        if (!aligned(x, 16) || !aligned(Wg, 16) || !aligned(W1, 16) || !aligned(W2, 16) ||
            (swiglu && !aligned(W3, 16)) || !aligned(y, 16))
            return MOE_ERR_INVALID_ARG;
        if (shared && (!Ws1 || !Ws2 || (swiglu && !Ws3) || !aligned(Ws1, 16) ||
                       !aligned(Ws2, 16) || (swiglu && !aligned(Ws3, 16))))
            return MOE_ERR_INVALID_ARG;
    }
    Ws w;
    moe_status st = check_ws(cfg, workspace, workspace_bytes, &w);
    if (st != MOE_OK)
        return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t *idx = topk_idx ? topk_idx : w.at<int32_t>(w.L.topk_idx);
    float *gw = topk_w ? topk_w : w.at<float>(w.L.topk_w);
    int32_t *counts = expert_counts ? expert_counts : w.at<int32_t>(w.L.counts);
    float *pm = p_mean ? p_mean : ((aux_loss != nullptr) ? w.at<float>(w.L.p_mean) : nullptr);
    const bool fp8 = c.dispatch_dtype == MOE_FP8_E4M3;
    int32_t *offsets = w.at<int32_t>(w.L.offsets);

    // small fp32 layers without a capacity limit: the whole forward in one launch
    if (c.dtype == MOE_F32 && c.capacity_factor <= 0.0f && c.T > 0 &&
        !(node_limited(c) && c.gate_mode == MOE_GATE_SOFTMAX_THEN_TOPK && !c.renormalize)) {
        moe::LayerSmallLaunch S{};
        S.x = static_cast<const float *>(x);
        S.Wg = static_cast<const float *>(Wg);
        S.bias = bias;
        S.W1 = static_cast<const float *>(W1);
        S.W3 = swiglu ? static_cast<const float *>(W3) : nullptr;
        S.W2 = static_cast<const float *>(W2);
        S.Ws1 = shared ? static_cast<const float *>(Ws1) : nullptr;
        S.Ws3 = (shared && swiglu) ? static_cast<const float *>(Ws3) : nullptr;
        S.Ws2 = shared ? static_cast<const float *>(Ws2) : nullptr;
        S.y = static_cast<float *>(y);
        S.T = c.T;
        S.d = c.d;
        S.N = c.N;
        S.k = c.k;
        S.H = c.H;
        S.Hs = c.H_shared;
        S.gate_mode = c.gate_mode;
        S.renormalize = c.renormalize;
        S.n_groups = node_limited(c) ? c.n_groups : 0;
        S.topk_groups = node_limited(c) ? c.topk_groups : 0;
        S.swiglu = swiglu ? 1 : 0;
        S.slot_priority = c.slot_priority;
        S.alpha = c.aux_alpha;
        S.topk_idx = idx;
        S.topk_w = gw;
        S.p_part = w.at<double>(w.L.p_part);
        S.ticket = w.status() + 1;
        S.counts = counts;
        S.offsets = offsets;
        S.perm = w.at<int32_t>(w.L.perm);
        S.inv_row = w.at<int32_t>(w.L.inv_row);
        S.drop = w.at<uint8_t>(w.L.drop);
        S.p_mean = pm;
        S.f = f;
        S.aux_loss = aux_loss;
        S.status = w.status();
        if (moe::layer_small_fits(S)) {
            // one kernel: its time is reported as the expert stage
            prof_mark(0, s);
            prof_mark(1, s);
            prof_mark(2, s);
            MOE_CUDA(moe::launch_layer_small(S, s));
            for (int b = 3; b < kMarks; ++b)
                prof_mark(b, s);
            if (g_prof.on && g_prof.steps < g_prof.max_steps)
                ++g_prof.steps;
            return MOE_OK;
        }
    }
    prof_mark(0, s);
    st = run_router(c, x, Wg, bias, nullptr, idx, gw, pm, w, s);
    if (st != MOE_OK)
        return st;
    prof_mark(1, s);
    // dispatch: counts, capacity, permutation, then the expert-ordered GEMM
    // rows.  FP8 dispatch quantises each token once (codes as bf16 + scale)
    // and writes them to the token's kept rows, instead of quantising every
    // (token, slot) copy.
    void *xg = w.at<void>(w.L.x_gemm);
    st = run_dispatch(c, x, idx, counts, offsets, w.at<int32_t>(w.L.perm),
                      w.at<int32_t>(w.L.inv_row), w.at<uint8_t>(w.L.drop), fp8 ? nullptr : xg,
                      nullptr, nullptr, pm, f, aux_loss, w, s);
    if (st != MOE_OK)
        return st;
    if (fp8 && c.T > 0)
        MOE_CUDA(moe::launch_quantize_scatter(x, c.T, c.d, c.k, w.at<int32_t>(w.L.inv_row), xg,
                                              w.at<float>(w.L.x_scale), s));
    prof_mark(2, s);
    if (c.T == 0) {
        for (int b = 3; b < kMarks; ++b)
            prof_mark(b, s);
        if (g_prof.on && g_prof.steps < g_prof.max_steps)
            ++g_prof.steps;
        return MOE_OK;
    }
    const int64_t rows_cap = c.T * c.k;
    st = run_ffn(c, xg, fp8 ? w.at<float>(w.L.x_scale) : nullptr, rows_cap, offsets, ffn_groups(c),
                 0, c.H,
                 W1, swiglu ? W3 : nullptr, W2, w.at<void>(w.L.h), w.at<void>(w.L.y_perm),
                 w.status(), s, 3);
    if (st != MOE_OK)
        return st;
    prof_mark(4, s);
    void *ys = nullptr;
    if (shared) {
        ys = w.at<void>(w.L.ys);
        st = run_ffn(c, x, nullptr, c.T, nullptr, 1, static_cast<int32_t>(c.T), c.H_shared, Ws1,
                     swiglu ? Ws3 : nullptr, Ws2, w.at<void>(w.L.hs), ys, w.status(), s);
        if (st != MOE_OK)
            return st;
    }
    prof_mark(5, s);
    MOE_CUDA(moe::launch_combine(c.dtype, w.at<void>(w.L.y_perm), w.at<int32_t>(w.L.inv_row), gw,
                                 ys, y, c.T, c.d, c.k, w.status(), s));
    prof_mark(6, s);
    if (g_prof.on && g_prof.steps < g_prof.max_steps)
        ++g_prof.steps;
    return MOE_OK;
}

moe_status moe_check_status(void *workspace, void *stream, uint32_t *detail)
{
    if (!workspace || !aligned(workspace, 256))
        return MOE_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    MOE_CUDA(cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s));
    MOE_CUDA(cudaStreamSynchronize(s));
    if (word != 0) {
        MOE_CUDA(cudaMemsetAsync(workspace, 0, sizeof(word), s));
        MOE_CUDA(cudaStreamSynchronize(s));
    }
    if (detail)
        *detail = word;
    if (word & moe::DEV_TIMEOUT_ANY)
        return MOE_ERR_TIMEOUT;
    return word ? MOE_ERR_DEVICE_STATUS : MOE_OK;
}

const char *moe_status_string(moe_status s)
{
    switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_STATUS: return "a kernel recorded an anomaly in the status word";
    case MOE_ERR_TIMEOUT: return "a bounded device wait gave up";
    }
    return "unknown status";
}

const char *moe_last_error_string(void) { return g_last_error; }

uint64_t moe_launch_count(void) { return moe::g_launches.load(); }

moe_status moe_profile_begin(int max_steps)
{
    std::lock_guard<std::mutex> lk(g_prof.mu);
    if (max_steps <= 0 || g_prof.on)
        return MOE_ERR_INVALID_ARG;
    const size_t need = static_cast<size_t>(max_steps) * kMarks;
    while (g_prof.ev.size() < need) {
        cudaEvent_t e;
        MOE_CUDA(cudaEventCreate(&e));
        g_prof.ev.push_back(e);
    }
    g_prof.max_steps = max_steps;
    g_prof.steps = 0;
    g_prof.on = true;
    return MOE_OK;
}

moe_status moe_profile_end(float *stage_ms, int *steps)
{
    std::lock_guard<std::mutex> lk(g_prof.mu);
    if (!g_prof.on)
        return MOE_ERR_INVALID_ARG;
    g_prof.on = false;
    double acc[MOE_PROFILE_STAGES] = {0};
    for (int st = 0; st < g_prof.steps; ++st) {
        MOE_CUDA(cudaEventSynchronize(g_prof.ev[static_cast<size_t>(st) * kMarks + kMarks - 1]));
        for (int b = 0; b < MOE_PROFILE_STAGES; ++b) {
            float ms = 0.0f;
            MOE_CUDA(cudaEventElapsedTime(&ms, g_prof.ev[static_cast<size_t>(st) * kMarks + b],
                                          g_prof.ev[static_cast<size_t>(st) * kMarks + b + 1]));
            acc[b] += ms;
        }
    }
    if (stage_ms)
        for (int b = 0; b < MOE_PROFILE_STAGES; ++b)
            stage_ms[b] = static_cast<float>(acc[b]);
    if (steps)
        *steps = g_prof.steps;
    return MOE_OK;
}

const char *moe_version(void) { return "moe_b200 1.0 sm_100a"; }

}  // extern "C"
