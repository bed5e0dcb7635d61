// Routing helpers shared by the small-N router (router.cu) and the
// single-launch small fp32 layer (layer_small.cu): logits as compensated or
// fp64 dot products, top-k with the lowest-index tie-break, and the gates.
//
// "moe communication costs", Router design (G(x) = softmax(W_g x), the k
// largest entries select the experts, mode F); "Advanced GPU Optimization:
// How to tech an LLM with CUDA and ROCm? - Part 5", section 1.1 (strict
// comparisons keep the lowest index on a tie; softmax over the selected
// scores only, mode R); "MoE: what it costs to train and serve", Limit how
// many machines a token touches (node-limited routing).
#pragma once

#include "common.cuh"
#include "moe.h"

namespace moe {
namespace rsel {

constexpr int kMaxK = 8;

__device__ __forceinline__ double warp_sum(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Accumulator of a dot product: a compensated fp32 pair (hi + lo) for bf16
// operands, whose products are exact in fp32 (8-bit significands); plain fp64
// for fp32 operands.  Each 16-byte chunk (8 bf16 products) is summed in fp32,
// then added to (hi, lo) with Knuth's branch-free TwoSum, so no rounding
// error accumulates across chunks and the result is as accurate as an fp64
// sum of the chunk sums, without fp64 or conversion instructions in the loop.
struct DotAcc {
    float hi = 0.0f, lo = 0.0f;
    double d = 0.0;
    __device__ __forceinline__ void add_chunk_sum(float s)
    {
        const float t = hi + s;
        const float bp = t - hi;
        lo += (hi - (t - bp)) + (s - bp);
        hi = t;
    }
    __device__ __forceinline__ double value(bool bf16) const
    {
        return bf16 ? static_cast<double>(hi) + static_cast<double>(lo) : d;
    }
};

template <bool BF16>
__device__ __forceinline__ void chunk_dot(const float (&xf)[8], const uint4 b, DotAcc &acc)
{
    const uint32_t bv[4] = {b.x, b.y, b.z, b.w};
    if (BF16) {
        float s = xf[0] * __uint_as_float(bv[0] << 16);
        s = fmaf(xf[1], __uint_as_float(bv[0] & 0xFFFF0000u), s);
#pragma unroll
        for (int i = 1; i < 4; ++i) {
            s = fmaf(xf[2 * i], __uint_as_float(bv[i] << 16), s);
            s = fmaf(xf[2 * i + 1], __uint_as_float(bv[i] & 0xFFFF0000u), s);
        }
        acc.add_chunk_sum(s);
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
            acc.d = fma(static_cast<double>(xf[i]), static_cast<double>(__uint_as_float(bv[i])),
                        acc.d);
    }
}

// The 8 (bf16) or 4 (fp32) values of a 16-byte chunk as floats.
template <bool BF16>
__device__ __forceinline__ void unpack_chunk(const uint4 a, float (&xf)[8])
{
    const uint32_t av[4] = {a.x, a.y, a.z, a.w};
    if (BF16) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            xf[2 * i] = __uint_as_float(av[i] << 16);
            xf[2 * i + 1] = __uint_as_float(av[i] & 0xFFFF0000u);
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            xf[i] = __uint_as_float(av[i]);
            xf[4 + i] = 0.0f;
        }
    }
}

// Selection and gates of one token from its N logits (fp64, every lane holds
// all of them).  Lane e accumulates the softmax probability of expert e into
// *my_psum.
template <int NMAX>
__device__ __forceinline__ void small_select(const double (&acc)[NMAX], int64_t t, int N, int k,
                                             int gate_mode, int renorm, int n_groups,
                                             int topk_groups, int lane,
                                             int32_t *__restrict__ topk_idx,
                                             float *__restrict__ topk_w, double *my_psum)
{
    // node-limited routing: lane g scores node g (sum of its m highest
    // probabilities, as exp(l - max), largest first), then the topk_groups
    // best nodes (lower node first on equal scores) are the allowed ones
    uint32_t allowed = 0xffffffffu;
    if (n_groups > 1) {
        const int S = N / n_groups;
        const int m = (k + topk_groups - 1) / topk_groups;
        double gmx = acc[0];
#pragma unroll
        for (int e = 1; e < NMAX; ++e)
            if (e < N && acc[e] > gmx)
                gmx = acc[e];
        double gs = -1.0;
        if (lane < n_groups) {
            gs = 0.0;
            uint32_t tk = 0;
#pragma unroll 1
            for (int r = 0; r < m; ++r) {
                int bi = -1;
                double bv = 0.0;
#pragma unroll
                for (int e = 0; e < NMAX; ++e) {
                    if (e < N && e / S == lane && !((tk >> e) & 1u) && (bi < 0 || acc[e] > bv)) {
                        bi = e;
                        bv = acc[e];
                    }
                }
                tk |= 1u << bi;
                gs += exp(bv - gmx);
            }
        }
        uint32_t gtaken = 0;
#pragma unroll 1
        for (int j = 0; j < topk_groups; ++j) {
            double v = (lane < n_groups && !((gtaken >> lane) & 1u)) ? gs : -1.0;
            int gi = v >= 0.0 ? lane : 32;
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const double ov = __shfl_xor_sync(0xffffffffu, v, o);
                const int oi = __shfl_xor_sync(0xffffffffu, gi, o);
                if (ov > v || (ov == v && oi < gi)) {
                    v = ov;
                    gi = oi;
                }
            }
            gtaken |= 1u << gi;
        }
        allowed = 0;
#pragma unroll
        for (int e = 0; e < NMAX; ++e)
            if (e < N && ((gtaken >> (e / S)) & 1u))
                allowed |= 1u << e;
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
                if (e < N && ((allowed >> e) & 1u) && !((taken >> e) & 1u) &&
                    (bi < 0 || acc[e] > bv)) {
                    bi = e;
                    bv = acc[e];
                }
            }
            taken |= 1u << bi;
            sel[j] = bi;
            val[j] = bv;
        }
    }
    // full softmax over N, one expert per lane (aux statistic p, mode F gates)
    const double mx = val[0];
    double my_l = 0.0;
#pragma unroll
    for (int e = 0; e < NMAX; ++e)
        if (e == lane)
            my_l = acc[e];
    const double my_ev = (lane < N) ? exp(my_l - mx) : 0.0;
    const double Z = warp_sum(my_ev);
    *my_psum += my_ev / Z;
    // gates: lane j < k computes slot j
    double gj = 0.0;
    int sj = 0;
#pragma unroll
    for (int j = 0; j < kMaxK; ++j)
        if (j == lane) {
            sj = sel[j];
            gj = val[j];
        }
    if (lane < k)
        gj = (gate_mode == MOE_GATE_TOPK_THEN_SOFTMAX) ? exp(gj - mx) : exp(gj - mx) / Z;
    else
        gj = 0.0;
    const double gs = warp_sum(gj);
    const bool norm = (gate_mode == MOE_GATE_TOPK_THEN_SOFTMAX) || renorm;
    if (lane < k) {
        topk_idx[t * k + lane] = sj;
        topk_w[t * k + lane] = static_cast<float>(norm ? gj / gs : gj);
    }
}

}  // namespace rsel
}  // namespace moe
