// The whole forward of a small fp32 MoE layer in one launch.
//
// For fp32 layers with few experts (N <= 16), no capacity limit and small
// hidden sizes, the four stages take microseconds of arithmetic, and a chain
// of separate launches (router, dispatch, two GEMMs, combine) costs several
// times more than the work.  Here each CTA takes kTokPerBlock tokens and runs
// the layer for them end to end:
//
//   router   logits l = W_g x (+ b) as fp64 dot products of the fp32 operands,
//            top-k (lowest index first on a tie) and the gates, by the same
//            helpers and in the same order as the small-N router kernel, so
//            the routing is bit-identical ("moe communication costs", Router
//            design; "Advanced GPU Optimization ... Part 5", section 1.1);
//   experts  for every (token, slot) pair, one warp computes
//            h = act(x W1_e) and then h W2_e (fp32, in the order of the fp32
//            grouped GEMM), token-major: without a capacity limit no pair is
//            dropped, so no permutation is needed for the output;
//   combine  y = sum over slots, in slot order, of g_j E_j(x) (+ the shared
//            expert) ("moe communication costs", Router design).
//
// The dispatch results the layer also reports (expert counts, offsets, the
// permutation and inverse rows of "MoE: what it costs to train and serve",
// Expert parallelism step 1, f, p and L_aux of "moe communication costs",
// Load balancing) depend on every token: the last CTA to finish (a ticket
// counter in the workspace, reset by that CTA for the next call) builds them
// with a counting sort over chunks of 32 pairs.
#include "common.cuh"
#include "kernels.h"
#include "moe.h"
#include "router_small.cuh"

namespace moe {

namespace {

using namespace rsel;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTokPerBlock = 4;

struct SmallParams {
    const float *x, *Wg, *bias, *W1, *W3, *W2, *Ws1, *Ws3, *Ws2;
    float *y;
    int64_t T;
    int d, N, k, H, Hs;
    int gate_mode, renorm, n_groups, topk_groups, swiglu, slot_priority;
    float alpha;
    int32_t *topk_idx;
    float *topk_w;
    double *p_part;        // [gridDim.x, N]
    uint32_t *ticket;      // CTAs finished; 0 between calls
    int32_t *counts, *offsets, *perm, *inv_row;
    uint8_t *drop;
    float *p_mean, *f, *aux_loss;
    uint32_t *status;
};

// Dot products of a (shared memory) with rows w0 and w1 (global, n fp32
// each, n a multiple of 4), each summed in order as an fmaf chain; the loads
// of 8 float4 of each row are issued before they are used, so the two rows'
// L2 latencies overlap.  w1 may equal w0 (then *d1 repeats *d0).
__device__ __forceinline__ void dot2_f32(const float *__restrict__ a, const float *__restrict__ w0,
                                         const float *__restrict__ w1, int n, float *d0,
                                         float *d1)
{
    float acc0 = 0.0f, acc1 = 0.0f;
    constexpr int B = 8;   // float4 per row per batch
    for (int i0 = 0; i0 < n; i0 += 4 * B) {
        float4 u[B], v[B];
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const int i = i0 + 4 * b;
            u[b] = i < n ? __ldg(reinterpret_cast<const float4 *>(w0 + i)) : make_float4(0, 0, 0, 0);
            v[b] = i < n ? __ldg(reinterpret_cast<const float4 *>(w1 + i)) : make_float4(0, 0, 0, 0);
        }
#pragma unroll
        for (int b = 0; b < B; ++b) {
            const int i = i0 + 4 * b;
            if (i < n) {
                acc0 = fmaf(a[i], u[b].x, acc0);
                acc0 = fmaf(a[i + 1], u[b].y, acc0);
                acc0 = fmaf(a[i + 2], u[b].z, acc0);
                acc0 = fmaf(a[i + 3], u[b].w, acc0);
                acc1 = fmaf(a[i], v[b].x, acc1);
                acc1 = fmaf(a[i + 1], v[b].y, acc1);
                acc1 = fmaf(a[i + 2], v[b].z, acc1);
                acc1 = fmaf(a[i + 3], v[b].w, acc1);
            }
        }
    }
    *d0 = acc0;
    *d1 = acc1;
}

// Pair taken at position pos: token by token, or slot by slot.
__device__ __forceinline__ int64_t pair_of(int64_t pos, int64_t T, int k, int slot_priority)
{
    return slot_priority ? (pos % T) * k + pos / T : pos;
}

template <int NMAX>
__global__ void __launch_bounds__(kThreads) layer_small_f32_kernel(SmallParams p)
{
    grid_dep_wait();
    extern __shared__ float s_dyn[];
    __shared__ double s_p[kWarps][NMAX];
    __shared__ int32_t s_idx[kTokPerBlock * kMaxK];
    __shared__ float s_g[kTokPerBlock * kMaxK];
    __shared__ int32_t s_tot[NMAX], s_off[NMAX + 1];
    __shared__ float s_pm[NMAX];
    __shared__ int s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int d = p.d, k = p.k, N = p.N;
    const int64_t T = p.T;
    const int npair = k + (p.Hs > 0 ? 1 : 0);   // per token: its k slots (+ the shared expert)
    const int Hmax = p.H > p.Hs ? p.H : p.Hs;
    float *s_x = s_dyn;                               // [kTokPerBlock, d]
    float *s_h = s_x + kTokPerBlock * d;              // [kWarps, Hmax]
    float *s_y = s_h + kWarps * Hmax;                 // [kTokPerBlock, npair, d]
    int32_t *s_cnt = reinterpret_cast<int32_t *>(s_y + kTokPerBlock * npair * d);  // tail

    const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kTokPerBlock;
    const int ntok = static_cast<int>(T - t0 < kTokPerBlock ? T - t0 : kTokPerBlock);
    for (int i = threadIdx.x; i < ntok * d; i += kThreads)
        s_x[i] = p.x[t0 * d + i];
    __syncthreads();

    // ---- router: warp w takes token t0 + w
    double my_psum = 0.0;
    if (warp < ntok) {
        const int64_t t = t0 + warp;
        const int chunks = d / 4;
        DotAcc da[NMAX];
        const uint4 *xr = reinterpret_cast<const uint4 *>(s_x + warp * d);
        for (int c = lane; c < chunks; c += 32) {
            float xf[8];
            unpack_chunk<false>(xr[c], xf);
#pragma unroll
            for (int e = 0; e < NMAX; ++e)
                if (e < N)
                    chunk_dot<false>(xf, __ldg(reinterpret_cast<const uint4 *>(
                                                   p.Wg + static_cast<int64_t>(e) * d) + c),
                                     da[e]);
        }
        double acc[NMAX];
#pragma unroll
        for (int e = 0; e < NMAX; ++e) {
            acc[e] = warp_sum(da[e].value(false));
            if (p.bias != nullptr && e < N)
                acc[e] += static_cast<double>(p.bias[e]);
        }
        small_select<NMAX>(acc, t, N, k, p.gate_mode, p.renorm, p.n_groups, p.topk_groups, lane,
                           p.topk_idx, p.topk_w, &my_psum);
    }
    if (lane < NMAX)
        s_p[warp][lane] = my_psum;
    __syncthreads();   // the block's routing (global writes above) is visible to the block
    for (int e = threadIdx.x; e < N; e += kThreads) {
        double s = 0.0;
        for (int wi = 0; wi < kWarps; ++wi)
            s += s_p[wi][e];
        p.p_part[static_cast<int64_t>(blockIdx.x) * N + e] = s;
    }
    for (int i = threadIdx.x; i < ntok * k; i += kThreads) {
        s_idx[i] = p.topk_idx[t0 * k + i];
        s_g[i] = p.topk_w[t0 * k + i];
    }
    __syncthreads();

    // ---- experts, token-major: warp per (token, slot) pair
    for (int q = warp; q < ntok * npair; q += kWarps) {
        const int tt = q / npair, j = q - tt * npair;
        const bool shared = j == k;
        const float *w1, *w3, *w2;
        int H;
        if (shared) {
            w1 = p.Ws1;
            w3 = p.Ws3;
            w2 = p.Ws2;
            H = p.Hs;
        } else {
            const int e = s_idx[tt * k + j];
            float *yq = s_y + static_cast<int64_t>(q) * d;
            if (e < 0 || e >= N) {    // cannot come from the router; guards the weights
                if (lane == 0)
                    set_status(p.status, DEV_BAD_EXPERT);
                for (int c = lane; c < d; c += 32)
                    yq[c] = 0.0f;
                continue;
            }
            H = p.H;
            w1 = p.W1 + static_cast<int64_t>(e) * H * d;
            w3 = p.swiglu ? p.W3 + static_cast<int64_t>(e) * H * d : nullptr;
            w2 = p.W2 + static_cast<int64_t>(e) * d * H;
        }
        const float *xr = s_x + tt * d;
        float *h = s_h + warp * Hmax;
        if (p.swiglu) {
            // the W1 and W3 rows of hidden unit c together
            for (int c = lane; c < H; c += 32) {
                float a, b;
                dot2_f32(xr, w1 + static_cast<int64_t>(c) * d, w3 + static_cast<int64_t>(c) * d, d,
                         &a, &b);
                h[c] = a / (1.0f + expf(-a)) * b;
            }
        } else {
            // hidden units c and c + 32 together
            for (int c = lane; c < H; c += 64) {
                const int c2 = c + 32 < H ? c + 32 : c;
                float a, b;
                dot2_f32(xr, w1 + static_cast<int64_t>(c) * d, w1 + static_cast<int64_t>(c2) * d,
                         d, &a, &b);
                h[c] = fmaxf(a, 0.0f);
                if (c + 32 < H)
                    h[c + 32] = fmaxf(b, 0.0f);
            }
        }
        __syncwarp();
        float *yq = s_y + static_cast<int64_t>(q) * d;
        for (int c = lane; c < d; c += 64) {
            const int c2 = c + 32 < d ? c + 32 : c;
            float a, b;
            dot2_f32(h, w2 + static_cast<int64_t>(c) * H, w2 + static_cast<int64_t>(c2) * H, H, &a,
                     &b);
            yq[c] = a;
            if (c + 32 < d)
                yq[c + 32] = b;
        }
        __syncwarp();
    }
    __syncthreads();

    // ---- combine, slots in order, then the shared expert
    for (int i = threadIdx.x; i < ntok * d; i += kThreads) {
        const int tt = i / d, c = i - tt * d;
        float acc = 0.0f;
        for (int j = 0; j < k; ++j) {
            const int e = s_idx[tt * k + j];
            if (e >= 0 && e < N)
                acc = fmaf(s_g[tt * k + j], s_y[(static_cast<int64_t>(tt) * npair + j) * d + c],
                           acc);
        }
        if (p.Hs > 0)
            acc += s_y[(static_cast<int64_t>(tt) * npair + k) * d + c];
        p.y[(t0 + tt) * d + c] = acc;
    }

    // ---- the last CTA: p, counts, offsets, permutation, f and L_aux
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0)
        s_last = atomicAdd(p.ticket, 1u) == gridDim.x - 1;
    __syncthreads();
    if (!s_last)
        return;
    __threadfence();
    // p: warp e sums expert e's partials, lanes over the blocks, then a
    // fixed-order butterfly (the same result on every run)
    for (int e = warp; e < N; e += kWarps) {
        double s = 0.0;
        for (unsigned b = lane; b < gridDim.x; b += 32)
            s += p.p_part[static_cast<int64_t>(b) * N + e];
        s = warp_sum(s);
        if (lane == 0) {
            const float pm = T > 0 ? static_cast<float>(s / static_cast<double>(T)) : 0.0f;
            s_pm[e] = pm;
            if (p.p_mean != nullptr)
                p.p_mean[e] = pm;
        }
    }
    const int64_t n_pairs = T * k;
    const int chunks = static_cast<int>((n_pairs + 31) / 32);
    // per chunk of 32 positions: the count of each expert
    for (int ch = warp; ch < chunks; ch += kWarps) {
        const int64_t pos = static_cast<int64_t>(ch) * 32 + lane;
        int e = -1;
        if (pos < n_pairs) {
            e = p.topk_idx[pair_of(pos, T, k, p.slot_priority)];
            if (e < 0 || e >= N)
                e = -1;
        }
        for (int ee = 0; ee < N; ++ee) {
            const uint32_t bal = __ballot_sync(0xffffffffu, e == ee);
            if (lane == 0)
                s_cnt[ch * N + ee] = __popc(bal);
        }
    }
    __syncthreads();
    // column scan over the chunks: each chunk's base inside every expert
    if (threadIdx.x < N) {
        const int ee = threadIdx.x;
        int32_t run = 0;
        for (int ch = 0; ch < chunks; ++ch) {
            const int32_t v = s_cnt[ch * N + ee];
            s_cnt[ch * N + ee] = run;
            run += v;
        }
        s_tot[ee] = run;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        int32_t o = 0;
        double aux = 0.0;
        for (int ee = 0; ee < N; ++ee) {
            s_off[ee] = o;
            o += s_tot[ee];
            aux += static_cast<double>(s_tot[ee]) / static_cast<double>(n_pairs) *
                   static_cast<double>(s_pm[ee]);
        }
        s_off[N] = o;
        if (p.aux_loss != nullptr)
            p.aux_loss[0] = static_cast<float>(static_cast<double>(p.alpha) * N * aux);
    }
    __syncthreads();
    for (int ee = threadIdx.x; ee <= N; ee += kThreads) {
        p.offsets[ee] = s_off[ee];
        if (ee < N) {
            p.counts[ee] = s_tot[ee];
            if (p.f != nullptr)
                p.f[ee] = static_cast<float>(static_cast<double>(s_tot[ee]) /
                                             static_cast<double>(n_pairs));
        }
    }
    // ranks: chunk base + earlier lanes of the chunk with the same expert
    for (int ch = warp; ch < chunks; ch += kWarps) {
        const int64_t pos = static_cast<int64_t>(ch) * 32 + lane;
        int64_t i = -1;
        int e = -1;
        if (pos < n_pairs) {
            i = pair_of(pos, T, k, p.slot_priority);
            e = p.topk_idx[i];
            if (e < 0 || e >= N) {
                set_status(p.status, DEV_BAD_EXPERT);
                e = -1;
            }
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        if (i >= 0) {
            if (e < 0) {
                p.drop[i] = 1;
                p.inv_row[i] = -1;
            } else {
                const int32_t row = s_off[e] + s_cnt[ch * N + e] + __popc(peers & lanemask_lt());
                p.perm[row] = static_cast<int32_t>(i);
                p.inv_row[i] = row;
                p.drop[i] = 0;
            }
        }
    }
    if (threadIdx.x == 0)
        *p.ticket = 0;   // every CTA has taken its ticket: ready for the next call
}

size_t small_smem_bytes(const LayerSmallLaunch &L)
{
    const int npair = L.k + (L.Hs > 0 ? 1 : 0);
    const int Hmax = L.H > L.Hs ? L.H : L.Hs;
    const int64_t chunks = (L.T * L.k + 31) / 32;
    return sizeof(float) * (static_cast<size_t>(kTokPerBlock) * L.d + kWarps * Hmax +
                            static_cast<size_t>(kTokPerBlock) * npair * L.d) +
           sizeof(int32_t) * static_cast<size_t>(chunks) * L.N;
}

}  // namespace

bool layer_small_fits(const LayerSmallLaunch &L)
{
    return L.T > 0 && L.N <= 16 && L.k <= kMaxK && L.T * L.k <= kSmallMaxPairs &&
           (L.T + kTokPerBlock - 1) / kTokPerBlock <= kRouterMaxBlocks && L.d % 4 == 0 &&
           L.H % 4 == 0 && L.Hs % 4 == 0 && small_smem_bytes(L) <= kSmallMaxSmem;
}

cudaError_t launch_layer_small(const LayerSmallLaunch &L, cudaStream_t stream)
{
    if (!layer_small_fits(L))
        return cudaErrorInvalidValue;
    SmallParams p;
    p.x = L.x;
    p.Wg = L.Wg;
    p.bias = L.bias;
    p.W1 = L.W1;
    p.W3 = L.W3;
    p.W2 = L.W2;
    p.Ws1 = L.Ws1;
    p.Ws3 = L.Ws3;
    p.Ws2 = L.Ws2;
    p.y = L.y;
    p.T = L.T;
    p.d = L.d;
    p.N = L.N;
    p.k = L.k;
    p.H = L.H;
    p.Hs = L.Hs;
    p.gate_mode = L.gate_mode;
    p.renorm = L.renormalize;
    p.n_groups = L.n_groups;
    p.topk_groups = L.topk_groups;
    p.swiglu = L.swiglu;
    p.slot_priority = L.slot_priority;
    p.alpha = L.alpha;
    p.topk_idx = L.topk_idx;
    p.topk_w = L.topk_w;
    p.p_part = L.p_part;
    p.ticket = L.ticket;
    p.counts = L.counts;
    p.offsets = L.offsets;
    p.perm = L.perm;
    p.inv_row = L.inv_row;
    p.drop = L.drop;
    p.p_mean = L.p_mean;
    p.f = L.f;
    p.aux_loss = L.aux_loss;
    p.status = L.status;
    const int grid = static_cast<int>((L.T + kTokPerBlock - 1) / kTokPerBlock);
    const size_t smem = small_smem_bytes(L);
    static DeviceOnce attr_once;   // per device: function attributes are per device
    cudaError_t e = device_once(attr_once, nullptr, [](int *) {
        cudaError_t r = cudaFuncSetAttribute(layer_small_f32_kernel<8>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmallMaxSmem);
        if (r == cudaSuccess)
            r = cudaFuncSetAttribute(layer_small_f32_kernel<16>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kSmallMaxSmem);
        return r;
    });
    if (e != cudaSuccess)
        return e;
    if (L.N <= 8)
        e = launch_k(layer_small_f32_kernel<8>, grid, kThreads, smem, stream, p);
    else
        e = launch_k(layer_small_f32_kernel<16>, grid, kThreads, smem, stream, p);
    count_launches(1);
    return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace moe
