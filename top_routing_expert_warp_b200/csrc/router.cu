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
//     and fp64 accumulation, then selects;
//   - large N: the logits come from the tcgen05 GEMM (fp32 accumulation);
//     router_select takes the best few candidates on those, recomputes the
//     candidates in fp64 and decides among them, so near-ties are resolved as
//     exact arithmetic resolves them.
#include "common.cuh"
#include "kernels.h"
#include "moe.h"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxK = 8;
constexpr int kMaxCand = 10;
constexpr int kMaxPerLane = 8;  // large-N path: N <= 256

__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// fp64 dot of 16-byte chunks: bf16 (8 values) or fp32 (4 values); each
// product is exact in fp64.
template <bool BF16>
__device__ __forceinline__ double chunk_dot(const uint4 a, const uint4 b, double acc)
{
    const uint32_t av[4] = {a.x, a.y, a.z, a.w};
    const uint32_t bv[4] = {b.x, b.y, b.z, b.w};
    if (BF16) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc = fma(static_cast<double>(__uint_as_float(av[i] << 16)),
                      static_cast<double>(__uint_as_float(bv[i] << 16)), acc);
            acc = fma(static_cast<double>(__uint_as_float(av[i] & 0xFFFF0000u)),
                      static_cast<double>(__uint_as_float(bv[i] & 0xFFFF0000u)), acc);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            acc = fma(static_cast<double>(__uint_as_float(av[i])),
                      static_cast<double>(__uint_as_float(bv[i])), acc);
    }
    return acc;
}

template <bool BF16, int NMAX>
__global__ void __launch_bounds__(kThreads)
    router_small_kernel(const void *__restrict__ xv, const void *__restrict__ wv,
                        const float *__restrict__ bias, int64_t T, int d, int N, int k,
                        int gate_mode, int renorm, float *__restrict__ logits_out,
                        int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                        double *__restrict__ p_part)
{
    __shared__ double s_p[kWarps][NMAX];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int esz = BF16 ? 2 : 4;
    const int chunks = d * esz / 16;
    const uint8_t *x = static_cast<const uint8_t *>(xv);
    const uint8_t *w = static_cast<const uint8_t *>(wv);

    double psum[NMAX];
#pragma unroll
    for (int e = 0; e < NMAX; ++e)
        psum[e] = 0.0;

    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kWarps + warp; t < T;
         t += static_cast<int64_t>(gridDim.x) * kWarps) {
        double acc[NMAX];
#pragma unroll
        for (int e = 0; e < NMAX; ++e)
            acc[e] = 0.0;
        const uint4 *xr = reinterpret_cast<const uint4 *>(x + t * static_cast<int64_t>(d) * esz);
        for (int c = lane; c < chunks; c += 32) {
            const uint4 xa = __ldg(xr + c);
#pragma unroll
            for (int e = 0; e < NMAX; ++e) {
                if (e < N) {
                    const uint4 wa = __ldg(reinterpret_cast<const uint4 *>(
                                               w + static_cast<int64_t>(e) * d * esz) +
                                           c);
                    acc[e] = chunk_dot<BF16>(xa, wa, acc[e]);
                }
            }
        }
#pragma unroll
        for (int e = 0; e < NMAX; ++e) {
            acc[e] = warp_sum(acc[e]);
            if (bias != nullptr && e < N)
                acc[e] += static_cast<double>(bias[e]);
        }
        if (logits_out != nullptr) {
#pragma unroll
            for (int e = 0; e < NMAX; ++e)
                if (e < N && lane == e)
                    logits_out[t * N + e] = static_cast<float>(acc[e]);
        }
        // top-k: strict comparison in ascending expert order -> lowest index wins
        uint32_t taken = 0;
        int sel[kMaxK];
        double val[kMaxK];
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            sel[j] = 0;
            val[j] = 0.0;
            if (j < k) {
                int bi = -1;
                double bv = 0.0;
#pragma unroll
                for (int e = 0; e < NMAX; ++e) {
                    if (e < N && !((taken >> e) & 1u) && (bi < 0 || acc[e] > bv)) {
                        bi = e;
                        bv = acc[e];
                    }
                }
                taken |= 1u << bi;
                sel[j] = bi;
                val[j] = bv;
            }
        }
        // full softmax over N (aux statistic p, and mode F gates)
        const double mx = val[0];
        double Z = 0.0;
        double pe[NMAX];
#pragma unroll
        for (int e = 0; e < NMAX; ++e) {
            pe[e] = (e < N) ? exp(acc[e] - mx) : 0.0;
            Z += pe[e];
        }
#pragma unroll
        for (int e = 0; e < NMAX; ++e) {
            pe[e] /= Z;
            psum[e] += pe[e];
        }
        double g[kMaxK];
        double gs = 0.0;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            g[j] = 0.0;
            if (j < k) {
                if (gate_mode == MOE_GATE_TOPK_THEN_SOFTMAX) {
                    g[j] = exp(val[j] - mx);
                } else {
                    double pj = 0.0;
#pragma unroll
                    for (int e = 0; e < NMAX; ++e)
                        if (e == sel[j])
                            pj = pe[e];
                    g[j] = pj;
                }
                gs += g[j];
            }
        }
        const bool norm = (gate_mode == MOE_GATE_TOPK_THEN_SOFTMAX) || renorm;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            if (j < k && lane == j) {
                topk_idx[t * k + j] = sel[j];
                topk_w[t * k + j] = static_cast<float>(norm ? g[j] / gs : g[j]);
            }
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int e = 0; e < NMAX; ++e)
            s_p[warp][e] = psum[e];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < N; e += kThreads) {
        double s = 0.0;
        for (int wi = 0; wi < kWarps; ++wi)
            s += s_p[wi][e];
        p_part[static_cast<int64_t>(blockIdx.x) * N + e] = s;
    }
}

// (value, index) ordering: larger value first, then lower index.
__device__ __forceinline__ bool better(float v1, int e1, float v2, int e2)
{
    return (v1 > v2) || (v1 == v2 && e1 < e2 && e1 >= 0) || (e2 < 0 && e1 >= 0);
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads)
    router_select_kernel(float *__restrict__ logits, const void *__restrict__ xv,
                         const void *__restrict__ wv, const float *__restrict__ bias, int64_t T,
                         int d, int N, int k, int gate_mode, int renorm,
                         int32_t *__restrict__ topk_idx, float *__restrict__ topk_w,
                         double *__restrict__ p_part)
{
    extern __shared__ double s_pdyn[];  // [kWarps][N]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int esz = BF16 ? 2 : 4;
    const int chunks = d * esz / 16;
    const uint8_t *x = static_cast<const uint8_t *>(xv);
    const uint8_t *w = static_cast<const uint8_t *>(wv);
    const int npl = (N + 31) / 32;
    const bool mode_f_raw = (gate_mode == MOE_GATE_SOFTMAX_THEN_TOPK) && !renorm;
    int KC = k + 2;
    if (mode_f_raw && KC < 8)
        KC = 8;
    if (KC > N)
        KC = N;
    if (KC > kMaxCand)
        KC = kMaxCand;

    double psum[kMaxPerLane];
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i)
        psum[i] = 0.0;

    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kWarps + warp; t < T;
         t += static_cast<int64_t>(gridDim.x) * kWarps) {
        float lv[kMaxPerLane];
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i) {
            const int e = lane + 32 * i;
            lv[i] = -INFINITY;
            if (i < npl && e < N) {
                float v = logits[t * N + e];
                if (bias != nullptr) {
                    v += bias[e];
                    logits[t * N + e] = v;
                }
                lv[i] = v;
            }
        }
        // candidates: the KC best fp32 logits, best first
        int cand[kMaxCand];
        uint32_t taken = 0;
#pragma unroll
        for (int c = 0; c < kMaxCand; ++c) {
            cand[c] = 0;
            if (c < KC) {
                float bv = -INFINITY;
                int be = -1;
#pragma unroll
                for (int i = 0; i < kMaxPerLane; ++i) {
                    const int e = lane + 32 * i;
                    if (i < npl && e < N && !((taken >> i) & 1u) &&
                        (be < 0 || lv[i] > bv)) {
                        bv = lv[i];
                        be = e;
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
                    const int oe = __shfl_xor_sync(0xffffffffu, be, o);
                    if (better(ov, oe, bv, be)) {
                        bv = ov;
                        be = oe;
                    }
                }
                cand[c] = be;
                if ((be & 31) == lane)
                    taken |= 1u << (be >> 5);
            }
        }
        // fp64 recomputation of the candidates
        double acc[kMaxCand];
#pragma unroll
        for (int c = 0; c < kMaxCand; ++c)
            acc[c] = 0.0;
        const uint4 *xr = reinterpret_cast<const uint4 *>(x + t * static_cast<int64_t>(d) * esz);
        for (int ch = lane; ch < chunks; ch += 32) {
            const uint4 xa = __ldg(xr + ch);
#pragma unroll
            for (int c = 0; c < kMaxCand; ++c) {
                if (c < KC) {
                    const uint4 wa = __ldg(reinterpret_cast<const uint4 *>(
                                               w + static_cast<int64_t>(cand[c]) * d * esz) +
                                           ch);
                    acc[c] = chunk_dot<BF16>(xa, wa, acc[c]);
                }
            }
        }
#pragma unroll
        for (int c = 0; c < kMaxCand; ++c) {
            acc[c] = warp_sum(acc[c]);
            if (bias != nullptr && c < KC)
                acc[c] += static_cast<double>(bias[cand[c]]);
        }
        // order candidates by (fp64 value desc, index asc); fixed-shape
        // exchange sort so that every index is a compile-time constant
#pragma unroll
        for (int pass = 0; pass < kMaxCand - 1; ++pass) {
#pragma unroll
            for (int c = 0; c + 1 < kMaxCand; ++c) {
                if (c + 1 < KC) {
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
        // full softmax over N: candidates use fp64 logits, the rest fp32 ones
        double Z = 0.0;
        double ev[kMaxPerLane];
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i) {
            const int e = lane + 32 * i;
            ev[i] = 0.0;
            if (i < npl && e < N) {
                double l = static_cast<double>(lv[i]);
#pragma unroll
                for (int c = 0; c < kMaxCand; ++c)
                    if (c < KC && cand[c] == e)
                        l = acc[c];
                ev[i] = exp(l - mx);
                Z += ev[i];
            }
        }
        Z = warp_sum(Z);
#pragma unroll
        for (int i = 0; i < kMaxPerLane; ++i)
            psum[i] += ev[i] / Z;
        double g[kMaxK];
        double gs = 0.0;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            g[j] = 0.0;
            if (j < k) {
                g[j] = exp(acc[j] - mx);
                gs += g[j];
            }
        }
        const bool norm = (gate_mode == MOE_GATE_TOPK_THEN_SOFTMAX) || renorm;
#pragma unroll
        for (int j = 0; j < kMaxK; ++j) {
            if (j < k && lane == j) {
                topk_idx[t * k + j] = cand[j];
                topk_w[t * k + j] = static_cast<float>(norm ? g[j] / gs : g[j] / Z);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < kMaxPerLane; ++i) {
        const int e = lane + 32 * i;
        if (i < npl && e < N)
            s_pdyn[warp * N + e] = psum[i];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < N; e += kThreads) {
        double s = 0.0;
        for (int wi = 0; wi < kWarps; ++wi)
            s += s_pdyn[wi * N + e];
        p_part[static_cast<int64_t>(blockIdx.x) * N + e] = s;
    }
}

__global__ void p_finalize_kernel(const double *__restrict__ p_part, int nblk, int N, int64_t T,
                                  float *__restrict__ p_mean)
{
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < N; e += gridDim.x * blockDim.x) {
        double s = 0.0;
        for (int b = 0; b < nblk; ++b)
            s += p_part[static_cast<int64_t>(b) * N + e];
        p_mean[e] = T > 0 ? static_cast<float>(s / static_cast<double>(T)) : 0.0f;
    }
}

int router_grid(int64_t T)
{
    int64_t want = (T + kWarps - 1) / kWarps;
    int sms = 148;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t cap = static_cast<int64_t>(sms) * 4;
    if (cap > kRouterMaxBlocks)
        cap = kRouterMaxBlocks;
    if (want > cap)
        want = cap;
    return want < 1 ? 1 : static_cast<int>(want);
}

}  // namespace

cudaError_t launch_router_small(RouterLaunch &L, cudaStream_t stream)
{
    const int grid = router_grid(L.T);
    *L.p_blocks = grid;
    if (L.dtype == MOE_BF16) {
        if (L.N <= 8)
            router_small_kernel<true, 8><<<grid, kThreads, 0, stream>>>(
                L.x, L.Wg, L.bias, L.T, L.d, L.N, L.k, L.gate_mode, L.renormalize,
                L.logits_out, L.topk_idx, L.topk_w, L.p_part);
        else
            router_small_kernel<true, 16><<<grid, kThreads, 0, stream>>>(
                L.x, L.Wg, L.bias, L.T, L.d, L.N, L.k, L.gate_mode, L.renormalize,
                L.logits_out, L.topk_idx, L.topk_w, L.p_part);
    } else {
        if (L.N <= 8)
            router_small_kernel<false, 8><<<grid, kThreads, 0, stream>>>(
                L.x, L.Wg, L.bias, L.T, L.d, L.N, L.k, L.gate_mode, L.renormalize,
                L.logits_out, L.topk_idx, L.topk_w, L.p_part);
        else
            router_small_kernel<false, 16><<<grid, kThreads, 0, stream>>>(
                L.x, L.Wg, L.bias, L.T, L.d, L.N, L.k, L.gate_mode, L.renormalize,
                L.logits_out, L.topk_idx, L.topk_w, L.p_part);
    }
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_router_select(RouterLaunch &L, cudaStream_t stream)
{
    const int grid = router_grid(L.T);
    *L.p_blocks = grid;
    const size_t smem = static_cast<size_t>(kWarps) * L.N * sizeof(double);
    if (L.dtype == MOE_BF16)
        router_select_kernel<true><<<grid, kThreads, smem, stream>>>(
            const_cast<float *>(L.logits_in), L.x, L.Wg, L.bias, L.T, L.d, L.N, L.k,
            L.gate_mode, L.renormalize, L.topk_idx, L.topk_w, L.p_part);
    else
        router_select_kernel<false><<<grid, kThreads, smem, stream>>>(
            const_cast<float *>(L.logits_in), L.x, L.Wg, L.bias, L.T, L.d, L.N, L.k,
            L.gate_mode, L.renormalize, L.topk_idx, L.topk_w, L.p_part);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_p_finalize(const double *p_part, int32_t p_blocks, int32_t N, int64_t T,
                              float *p_mean, cudaStream_t stream)
{
    p_finalize_kernel<<<1, 256, 0, stream>>>(p_part, p_blocks, N, T, p_mean);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
