// Router: logits l = W_g x (+ b), top-k selection with lowest-index
// tie-break, gate weights in both modes, per-block sums of the full softmax.
//
// Definitions followed:
//   "moe communication costs", Router design: G(x) = softmax(W_g x), the k
//     largest entries select the experts and are the mixture coefficients
//     (mode F, optionally renormalised over the k).
//   "Advanced GPU Optimization: How to tech an LLM with CUDA and ROCm? - Part 5",
//     section 1.1: the top-2 is kept by strict comparisons (so the lowest index
//     wins a tie, slot 0 is the largest) and the softmax is taken over the
//     selected scores only, shifted by the largest (mode R).
//   "MoE: what it costs to train and serve", Numerical precision: the router
//     is computed at higher precision than the rest of the layer.
//
// Unlike the page-3 kernel (one thread per token looping over all experts
// and all of d), the work here is spread over a warp per token with 16-byte
// loads, and routing decisions are taken on fp64 logits:
//   - small N (<= 16): router_small computes every logit with exact products
//     and compensated accumulation (fp64-level accuracy), then selects;
//   - large N: the logits come from the tcgen05 GEMM (fp32 accumulation);
//     router_select takes the best few candidates on those, recomputes the
//     candidates in fp64 and decides among them, so near-ties are resolved as
//     exact arithmetic resolves them.
#include "common.cuh"
#include "kernels.h"
#include "moe.h"
#include "router_small.cuh"

namespace moe {

namespace {

using namespace rsel;

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxCand = 10;
constexpr int kMaxPerLane = 8;  // large-N path: N <= 256

// Small-N router: a warp takes kTokPerWarp tokens at a time and kUnroll
// 16-byte chunks per lane per pass, so several loads of x (from HBM) and of
// W_g (L1-resident) are in flight per lane and each W_g chunk serves every
// token of the warp.
constexpr int kTokPerWarp = 2;
constexpr int kUnroll = 4;

template <bool BF16, int NMAX>
__global__ void __launch_bounds__(kThreads)
    router_small_kernel(const void *__restrict__ xv, const void *__restrict__ wv,
                        const float *__restrict__ bias, int64_t T, int d, int N, int k,
                        int gate_mode, int renorm, int n_groups, int topk_groups,
                        float *__restrict__ logits_out, int32_t *__restrict__ topk_idx,
                        float *__restrict__ topk_w, double *__restrict__ p_part)
{
    grid_dep_wait();
    __shared__ double s_p[kWarps][NMAX];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int esz = BF16 ? 2 : 4;
    const int chunks = d * esz / 16;
    const uint8_t *x = static_cast<const uint8_t *>(xv);
    const uint8_t *w = static_cast<const uint8_t *>(wv);
    double my_psum = 0.0;  // lane e: this warp's sum of p_e over its tokens

    const int64_t step = static_cast<int64_t>(gridDim.x) * kWarps * kTokPerWarp;
    for (int64_t t0 = (static_cast<int64_t>(blockIdx.x) * kWarps + warp) * kTokPerWarp; t0 < T;
         t0 += step) {
        DotAcc da[kTokPerWarp][NMAX];
        const uint4 *xr[kTokPerWarp];
#pragma unroll
        for (int q = 0; q < kTokPerWarp; ++q) {
            const int64_t tq = (t0 + q < T) ? t0 + q : t0;   // a missing token re-reads t0
            xr[q] = reinterpret_cast<const uint4 *>(x + tq * static_cast<int64_t>(d) * esz);
        }
        for (int c0 = lane; c0 < chunks; c0 += 32 * kUnroll) {
            float xf[kTokPerWarp][kUnroll][8];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int c = c0 + 32 * u;
#pragma unroll
                for (int q = 0; q < kTokPerWarp; ++q) {
                    uint4 v = make_uint4(0, 0, 0, 0);
                    if (c < chunks)
                        v = __ldg(xr[q] + c);
                    unpack_chunk<BF16>(v, xf[q][u]);
                }
            }
#pragma unroll
            for (int e = 0; e < NMAX; ++e) {
                if (e < N) {
                    const uint4 *wr = reinterpret_cast<const uint4 *>(
                        w + static_cast<int64_t>(e) * d * esz);
#pragma unroll
                    for (int u = 0; u < kUnroll; ++u) {
                        const int c = c0 + 32 * u;
                        if (c < chunks) {
                            const uint4 wa = __ldg(wr + c);
#pragma unroll
                            for (int q = 0; q < kTokPerWarp; ++q)
                                chunk_dot<BF16>(xf[q][u], wa, da[q][e]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int q = 0; q < kTokPerWarp; ++q) {
            const int64_t t = t0 + q;
            double acc[NMAX];
#pragma unroll
            for (int e = 0; e < NMAX; ++e) {
                acc[e] = warp_sum(da[q][e].value(BF16));
                if (bias != nullptr && e < N)
                    acc[e] += static_cast<double>(bias[e]);
            }
            if (t >= T)
                continue;
            if (logits_out != nullptr) {
#pragma unroll
                for (int e = 0; e < NMAX; ++e)
                    if (e < N && lane == e)
                        logits_out[t * N + e] = static_cast<float>(acc[e]);
            }
            small_select<NMAX>(acc, t, N, k, gate_mode, renorm, n_groups, topk_groups, lane,
                               topk_idx, topk_w, &my_psum);
        }
    }
    if (lane < NMAX)
        s_p[warp][lane] = my_psum;
    __syncthreads();
    for (int e = threadIdx.x; e < N; e += kThreads) {
        double s = 0.0;
        for (int wi = 0; wi < kWarps; ++wi)
            s += s_p[wi][e];
        p_part[static_cast<int64_t>(blockIdx.x) * N + e] = s;
    }
}

// Unsigned key with the order of the float values (-0 counts as +0, so that
// equal values get equal keys): larger key = larger value.
__device__ __forceinline__ uint32_t order_key(float v)
{
    const uint32_t u = __float_as_uint(v + 0.0f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float a key was made from.
__device__ __forceinline__ float key_value(uint32_t key)
{
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Compensated fp32 accumulator (hi + lo) of bf16 dot products; see DotAcc.
struct Comp {
    float hi = 0.0f, lo = 0.0f;
    __device__ __forceinline__ void add(float s)
    {
        const float t = hi + s;
        const float bp = t - hi;
        lo += (hi - (t - bp)) + (s - bp);
        hi = t;
    }
};

// The 8 bf16 values of a 16-byte chunk as 4 packed fp32 pairs (element 2i in
// the low half, 2i + 1 in the high half of pair i).
__device__ __forceinline__ void unpack_pairs(const uint4 a, uint64_t (&p)[4])
{
    const uint32_t av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
        p[i] = static_cast<uint64_t>(av[i] << 16) |
               (static_cast<uint64_t>(av[i] & 0xFFFF0000u) << 32);
}

// Sum of the 8 exact bf16 x bf16 products of a chunk with packed fp32 FMAs
// (two lanes of partial sums: even and odd elements), then the two added.
__device__ __forceinline__ float chunk_dot8_x2(const uint64_t (&xp)[4], const uint4 b)
{
    uint64_t wp[4];
    unpack_pairs(b, wp);
    uint64_t acc;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(acc) : "l"(xp[0]), "l"(wp[0]));
#pragma unroll
    for (int i = 1; i < 4; ++i)
        asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(xp[i]), "l"(wp[i]));
    return __uint_as_float(static_cast<uint32_t>(acc)) +
           __uint_as_float(static_cast<uint32_t>(acc >> 32));
}

// Selection from the tensor-core logits (bf16 layers, any N <= 256): one warp
// per token.  The logits are the K-slice partial sums of the router GEMM,
// added in slice order.  The KC best become candidates; their logits are
// recomputed from x and W_g with exact products and compensated sums, the
// candidates are re-ranked on those values (descending, lower index first)
// and the gates are taken from them.  The full softmax for p (aux loss) uses
// the recomputed candidates and fp32 exponentials of the other logits.
// Stages of the per-warp copy ring of the candidate recomputation: deep
// enough to keep several 512-byte steps of x and every candidate row in
// flight per warp, within the shared memory of one 8-warp block per SM for
// the 8- and 10-candidate forms.
template <int KCM>
struct Ring {
    static constexpr int kStages = KCM >= 8 ? 3 : 4;
    static constexpr int kBytes = kWarps * kStages * (1 + KCM) * 512;
};

// NPL: logits per lane (N <= 32 NPL); KCM: bound on the candidate count.
// Both are compile-time so that every loop below has a fixed trip count and
// the instantiation used by a layer stays small.
template <int NPL, int KCM>
__global__ void __launch_bounds__(kThreads, NPL >= 8 ? 2 : 3)
    router_select_kernel(const float *__restrict__ part, int ksplit,
                         float *__restrict__ logits_out, const uint16_t *__restrict__ x,
                         const uint16_t *__restrict__ w, const float *__restrict__ bias, int64_t T,
                         int d, int N, int k, int gate_mode, int renorm, int n_groups,
                         int topk_groups, int32_t *__restrict__ topk_idx,
                         float *__restrict__ topk_w, double *__restrict__ p_part)
{
    grid_dep_wait();
    constexpr int kRing = Ring<KCM>::kStages;
    extern __shared__ __align__(16) uint8_t s_sel[];
    uint8_t *s_ring = s_sel;                             // [kWarps][kRing][1 + KCM][32 x 16 B]
    double *s_pdyn = reinterpret_cast<double *>(s_sel);  // [kWarps][N], after the tokens
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int chunks = d / 8;
    // candidates recomputed at fp64-level accuracy: the k selected experts,
    // whose logits alone set the gates in modes R and renormalised F; two more
    // in plain mode F, whose softmax denominator also weighs the runners-up
    const bool mode_f_raw = (gate_mode == MOE_GATE_SOFTMAX_THEN_TOPK) && !renorm;
    int KC = mode_f_raw ? k + 2 : k;
    if (KC > N)
        KC = N;
    if (KC > KCM)
        KC = KCM;

    float psum[NPL];
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        psum[i] = 0.0f;
    // node-limited routing: node of each of this lane's experts
    int grp[NPL];
    const int S = n_groups > 1 ? N / n_groups : N;
#pragma unroll
    for (int i = 0; i < NPL; ++i)
        grp[i] = (lane + 32 * i) / S;
    const int m_node = n_groups > 1 ? (k + topk_groups - 1) / topk_groups : 0;

    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kWarps + warp; t < T;
         t += static_cast<int64_t>(gridDim.x) * kWarps) {
        float lv[NPL];
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            lv[i] = -INFINITY;
            if (e < N) {
                float v = 0.0f;  // K-slice partial logits, summed in slice order
                for (int sl = 0; sl < ksplit; ++sl)
                    v += part[static_cast<int64_t>(sl) * T * N + t * N + e];
                if (bias != nullptr)
                    v += bias[e];
                if (logits_out != nullptr)
                    logits_out[t * N + e] = v;
                lv[i] = v;
            }
        }
        // node-limited routing: node g's score is the sum of its m_node
        // highest probabilities (as exp(l - max), largest first), picked by
        // warp reductions; lane g keeps it.  The topk_groups best nodes (lower
        // node first on equal scores) hold the experts that may be chosen.
        uint32_t allow = 0xffffffffu;   // bit i: expert lane + 32 i may be chosen
        if (n_groups > 1) {
            float lm = lv[0];
#pragma unroll
            for (int i = 1; i < NPL; ++i)
                lm = fmaxf(lm, lv[i]);
            const float gm = key_value(__reduce_max_sync(0xffffffffu, order_key(lm)));
            float my_gs = -1.0f;
#pragma unroll 1
            for (int g = 0; g < n_groups; ++g) {
                uint32_t tk = 0;
                float sum = 0.0f;
#pragma unroll 1
                for (int r = 0; r < m_node; ++r) {
                    float bv = -INFINITY;
                    int be = -1;
#pragma unroll
                    for (int i = 0; i < NPL; ++i) {
                        const int e = lane + 32 * i;
                        if (e < N && grp[i] == g && !((tk >> i) & 1u) && (be < 0 || lv[i] > bv)) {
                            bv = lv[i];
                            be = e;
                        }
                    }
                    const uint32_t key = be >= 0 ? order_key(bv) : 0u;
                    const uint32_t top = __reduce_max_sync(0xffffffffu, key);
                    const uint32_t eb = __reduce_min_sync(
                        0xffffffffu, (be >= 0 && key == top) ? static_cast<uint32_t>(be) : 0xffffffffu);
                    if (static_cast<int>(eb & 31u) == lane)
                        tk |= 1u << (eb >> 5);
                    sum += expf(key_value(top) - gm);
                }
                if (lane == g)
                    my_gs = sum;
            }
            uint32_t gtaken = 0;
#pragma unroll 1
            for (int j = 0; j < topk_groups; ++j) {
                const bool live = lane < n_groups && !((gtaken >> lane) & 1u);
                const uint32_t key = live ? order_key(my_gs) : 0u;
                const uint32_t top = __reduce_max_sync(0xffffffffu, key);
                const uint32_t gi = __reduce_min_sync(
                    0xffffffffu, (live && key == top) ? static_cast<uint32_t>(lane) : 0xffffffffu);
                gtaken |= 1u << gi;
            }
            allow = 0;
#pragma unroll
            for (int i = 0; i < NPL; ++i)
                if (lane + 32 * i < N && ((gtaken >> grp[i]) & 1u))
                    allow |= 1u << i;
        }
        // candidates: the KC best logits, best first.  Each round takes the
        // lane's best untaken logit (lowest index on a tie), then the warp's
        // largest (two warp reductions: the largest value, then the lowest
        // expert index holding it)
        int cand[KCM];
        uint32_t taken = 0;
#pragma unroll
        for (int c = 0; c < KCM; ++c) {
            cand[c] = 0;
            if (c < KC) {
                float bv = -INFINITY;
                int be = -1;
#pragma unroll
                for (int i = 0; i < NPL; ++i) {
                    const int e = lane + 32 * i;
                    if (e < N && ((allow >> i) & 1u) && !((taken >> i) & 1u) &&
                        (be < 0 || lv[i] > bv)) {
                        bv = lv[i];
                        be = e;
                    }
                }
                const uint32_t key = be >= 0 ? order_key(bv) : 0u;
                const uint32_t top = __reduce_max_sync(0xffffffffu, key);
                be = static_cast<int>(__reduce_min_sync(
                    0xffffffffu, (be >= 0 && key == top) ? static_cast<uint32_t>(be) : 0xffffffffu));
                cand[c] = be;
                if ((be & 31) == lane)
                    taken |= 1u << (be >> 5);
            }
        }
        // recomputation of the candidates
        // Each lane streams its own 16-byte chunks (chunk lane + 32 i at step
        // i) of x and of the KC candidate rows through a ring of kRing stages
        // in shared memory with cp.async, kRing - 1 steps ahead of the
        // arithmetic; it reads back only what it copied, so no warp barrier.
        Comp da[KCM];
        {
            const uint4 *xr = reinterpret_cast<const uint4 *>(x + t * static_cast<int64_t>(d));
            const int steps = (chunks + 31) / 32;
            uint8_t *ring = s_ring + static_cast<size_t>(warp) * kRing * (1 + KCM) * 512 + lane * 16;
            auto issue = [&](int i) {
                const int ch = lane + 32 * i;
                const bool live = i < steps && ch < chunks;
                uint8_t *slot = ring + (i % kRing) * (1 + KCM) * 512;
                cp_async_16(smem_u32(slot), xr + (live ? ch : 0), live ? 16u : 0u);
#pragma unroll
                for (int c = 0; c < KCM; ++c)
                    if (c < KC)
                        cp_async_16(smem_u32(slot + (1 + c) * 512),
                                    reinterpret_cast<const uint4 *>(
                                        w + static_cast<int64_t>(cand[c]) * d) + (live ? ch : 0),
                                    live ? 16u : 0u);
                cp_async_commit();   // one group per step (empty past the end)
            };
#pragma unroll
            for (int i = 0; i < kRing - 1; ++i)
                issue(i);
            for (int i = 0; i < steps; ++i) {
                issue(i + kRing - 1);
                cp_async_wait<kRing - 1>();   // step i's copies of this lane have landed
                const int ch = lane + 32 * i;
                if (ch < chunks) {
                    const uint8_t *slot = ring + (i % kRing) * (1 + KCM) * 512;
                    uint64_t xp[4];
                    unpack_pairs(*reinterpret_cast<const uint4 *>(slot), xp);
#pragma unroll
                    for (int c = 0; c < KCM; ++c)
                        if (c < KC)
                            da[c].add(chunk_dot8_x2(
                                xp, *reinterpret_cast<const uint4 *>(slot + (1 + c) * 512)));
                }
            }
            cp_async_wait_all();
        }
        double acc[KCM];
#pragma unroll
        for (int c = 0; c < KCM; ++c) {
            acc[c] = 0.0;
            if (c < KC) {   // KC is the same on every lane
                acc[c] = warp_sum(static_cast<double>(da[c].hi) + static_cast<double>(da[c].lo));
                if (bias != nullptr)
                    acc[c] += static_cast<double>(bias[cand[c]]);
            }
        }
        // order candidates by (recomputed value desc, index asc); fixed-shape
        // exchange sort so that every index is a compile-time constant
#pragma unroll
        for (int pass = 0; pass < KCM - 1; ++pass) {
            if (pass + 1 >= KC)
                break;
#pragma unroll
            for (int c = 0; c + 1 < KCM - pass; ++c) {
                if (c + 1 < KC - pass) {
                    const bool sw = (acc[c] < acc[c + 1]) ||
                                    (acc[c] == acc[c + 1] && cand[c] > cand[c + 1]);
                    if (sw) {
                        const double tv = acc[c];
                        acc[c] = acc[c + 1];
                        acc[c + 1] = tv;
                        const int te = cand[c];
                        cand[c] = cand[c + 1];
                        cand[c + 1] = te;
                    }
                }
            }
        }
        const double mx = acc[0];
        const float mxf = static_cast<float>(mx);
        // candidates' exponentials in fp64, candidate c on lane c, then
        // broadcast; the other experts' in fp32 on their lanes
        double my_acc = 0.0;
#pragma unroll
        for (int c = 0; c < KCM; ++c)
            if (c == lane)
                my_acc = acc[c];
        const double my_ec = (lane < KC) ? exp(my_acc - mx) : 0.0;
        double ec[KCM];
        double zc = 0.0, gs = 0.0;
#pragma unroll
        for (int c = 0; c < KCM; ++c) {
            ec[c] = (c < KC) ? __shfl_sync(0xffffffffu, my_ec, c) : 0.0;
            zc += ec[c];
            if (c < k)
                gs += ec[c];
        }
        float ev[NPL];
        float zl = 0.0f;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            bool is_c = false;
#pragma unroll
            for (int c = 0; c < KCM; ++c)
                is_c |= (c < KC && cand[c] == e);
            ev[i] = (e < N && !is_c) ? expf(lv[i] - mxf) : 0.0f;
            zl += ev[i];
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            zl += __shfl_xor_sync(0xffffffffu, zl, o);
        const double Z = static_cast<double>(zl) + zc;
        const double zinv = 1.0 / Z;
#pragma unroll
        for (int i = 0; i < NPL; ++i) {
            const int e = lane + 32 * i;
            float pv = ev[i] * static_cast<float>(zinv);
#pragma unroll
            for (int c = 0; c < KCM; ++c)
                if (c < KC && cand[c] == e)
                    pv = static_cast<float>(ec[c] * zinv);
            psum[i] += pv;
        }
        // gates: slot j = the j-th recomputed candidate (lane j writes it)
        double gj = 0.0;
        int ej = 0;
#pragma unroll
        for (int c = 0; c < KCM; ++c)
            if (c == lane) {
                gj = ec[c];
                ej = cand[c];
            }
        const bool norm = (gate_mode == MOE_GATE_TOPK_THEN_SOFTMAX) || renorm;
        if (lane < k) {
            topk_idx[t * k + lane] = ej;
            topk_w[t * k + lane] = static_cast<float>(norm ? gj / gs : gj * zinv);
        }
    }
    __syncthreads();   // every warp is done with its ring before it holds the sums
#pragma unroll
    for (int i = 0; i < NPL; ++i) {
        const int e = lane + 32 * i;
        if (e < N)
            s_pdyn[warp * N + e] = static_cast<double>(psum[i]);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < N; e += kThreads) {
        double s = 0.0;
        for (int wi = 0; wi < kWarps; ++wi)
            s += s_pdyn[wi * N + e];
        p_part[static_cast<int64_t>(blockIdx.x) * N + e] = s;
    }
}

// p_mean[e] = (sum over router blocks b of p_part[b][e]) / T; one block per
// expert, fixed-order tree so the result is the same on every run.
__global__ void __launch_bounds__(256)
    p_finalize_kernel(const double *__restrict__ p_part, int nblk, int N, int64_t T,
                      float *__restrict__ p_mean)
{
    grid_dep_wait();
    __shared__ double s[256];
    const int e = blockIdx.x;
    double acc = 0.0;
    for (int b = threadIdx.x; b < nblk; b += 256)
        acc += p_part[static_cast<int64_t>(b) * N + e];
    s[threadIdx.x] = acc;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w)
            s[threadIdx.x] += s[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0)
        p_mean[e] = T > 0 ? static_cast<float>(s[0] / static_cast<double>(T)) : 0.0f;
}

int router_grid(int64_t T, int tok_per_warp)
{
    int64_t want = (T + kWarps * tok_per_warp - 1) / (kWarps * tok_per_warp);
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t cap = static_cast<int64_t>(sms) * 8;
    if (cap > kRouterMaxBlocks)
        cap = kRouterMaxBlocks;
    if (want > cap)
        want = cap;
    return want < 1 ? 1 : static_cast<int>(want);
}

}  // namespace

cudaError_t launch_router_small(RouterLaunch &L, cudaStream_t stream)
{
    const int grid = router_grid(L.T, kTokPerWarp);
    *L.p_blocks = grid;
    if (L.dtype == MOE_BF16) {
        if (L.N <= 8)
            launch_k(router_small_kernel<true, 8>, grid, kThreads, 0, stream, 
                L.x, L.Wg, L.bias, L.T, L.d, L.N, L.k, L.gate_mode, L.renormalize, L.n_groups,
                L.topk_groups, L.logits_out, L.topk_idx, L.topk_w, L.p_part);
        else
            launch_k(router_small_kernel<true, 16>, grid, kThreads, 0, stream, 
                L.x, L.Wg, L.bias, L.T, L.d, L.N, L.k, L.gate_mode, L.renormalize, L.n_groups,
                L.topk_groups, L.logits_out, L.topk_idx, L.topk_w, L.p_part);
    } else {
        if (L.N <= 8)
            launch_k(router_small_kernel<false, 8>, grid, kThreads, 0, stream, 
                L.x, L.Wg, L.bias, L.T, L.d, L.N, L.k, L.gate_mode, L.renormalize, L.n_groups,
                L.topk_groups, L.logits_out, L.topk_idx, L.topk_w, L.p_part);
        else
            launch_k(router_small_kernel<false, 16>, grid, kThreads, 0, stream, 
                L.x, L.Wg, L.bias, L.T, L.d, L.N, L.k, L.gate_mode, L.renormalize, L.n_groups,
                L.topk_groups, L.logits_out, L.topk_idx, L.topk_w, L.p_part);
    }
    count_launches(1);
    return cudaGetLastError();
}

template <int NPL, int KCM>
cudaError_t select_launch(RouterLaunch &L, int grid, size_t smem_sums, cudaStream_t stream)
{
    const size_t smem = smem_sums > static_cast<size_t>(Ring<KCM>::kBytes)
                            ? smem_sums : static_cast<size_t>(Ring<KCM>::kBytes);
    static DeviceOnce attr_once;   // per device: function attributes are per device
    cudaError_t e = device_once(attr_once, nullptr, [](int *) {
        return cudaFuncSetAttribute(router_select_kernel<NPL, KCM>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    static_cast<int>(227 * 1024));
    });
    if (e != cudaSuccess)
        return e;
    return launch_k(router_select_kernel<NPL, KCM>, grid, kThreads, smem, stream,
        L.logits_in, L.ksplit, L.logits_out, static_cast<const uint16_t *>(L.x),
        static_cast<const uint16_t *>(L.Wg), L.bias, L.T, L.d, L.N, L.k, L.gate_mode,
        L.renormalize, L.n_groups, L.topk_groups, L.topk_idx, L.topk_w, L.p_part);
}

template <int NPL>
cudaError_t select_launch_kc(RouterLaunch &L, int kc, int grid, size_t smem, cudaStream_t stream)
{
    if (kc <= 2)
        return select_launch<NPL, 2>(L, grid, smem, stream);
    if (kc <= 4)
        return select_launch<NPL, 4>(L, grid, smem, stream);
    if (kc <= 8)
        return select_launch<NPL, 8>(L, grid, smem, stream);
    return select_launch<NPL, kMaxCand>(L, grid, smem, stream);
}

cudaError_t launch_router_select(RouterLaunch &L, cudaStream_t stream)
{
    if (L.dtype != MOE_BF16 || L.N > 32 * kMaxPerLane || L.k > kMaxCand)
        return cudaErrorInvalidValue;
    const int grid = router_grid(L.T, 1);
    *L.p_blocks = grid;
    const size_t smem = static_cast<size_t>(kWarps) * L.N * sizeof(double);
    const bool mode_f_raw = (L.gate_mode == MOE_GATE_SOFTMAX_THEN_TOPK) && !L.renormalize;
    int kc = mode_f_raw ? L.k + 2 : L.k;
    if (kc > L.N)
        kc = L.N;
    cudaError_t e;
    if (L.N <= 32)
        e = select_launch_kc<1>(L, kc, grid, smem, stream);
    else if (L.N <= 64)
        e = select_launch_kc<2>(L, kc, grid, smem, stream);
    else if (L.N <= 128)
        e = select_launch_kc<4>(L, kc, grid, smem, stream);
    else
        e = select_launch_kc<kMaxPerLane>(L, kc, grid, smem, stream);
    count_launches(1);
    return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_p_finalize(const double *p_part, int32_t p_blocks, int32_t N, int64_t T,
                              float *p_mean, cudaStream_t stream)
{
    launch_k(p_finalize_kernel, N, 256, 0, stream, p_part, p_blocks, N, T, p_mean);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
