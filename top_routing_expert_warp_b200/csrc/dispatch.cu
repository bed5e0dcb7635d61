// Dispatch as an on-device permutation of (token, slot) pairs into
// expert-contiguous rows.
//
// On one GPU the first all-to-all of the expert-parallel flow ("MoE: what it
// costs to train and serve", Expert parallelism and two all-to-alls, step 1)
// becomes a counting sort of the pairs by expert.  Capacity follows "moe
// communication costs", Capacity factor and token dropping: expert e keeps
// at most C = floor(capacity_factor * T / N) pairs, the first C in token
// order; the rest are dropped.  The aux-loss statistics follow the same
// page's Load balancing paragraph: f_i = pairs routed to i (before dropping)
// / (T k), L_aux = alpha N sum_i f_i p_i.
//
// Kernels (one stream, no host synchronisation):
//   count  - per block of 2048 pairs, per-expert counts with warp-aggregated
//            shared-memory atomics (__match_any_sync groups equal experts);
//   scan   - one block: per expert, exclusive scan over blocks (block bases),
//            counts, kept = min(count, C), offsets = exclusive scan of kept,
//            f and L_aux in a fixed summation order;
//   rank   - stable rank of every pair inside its expert: block base +
//            earlier warps of the block + earlier lanes of the warp; writes
//            perm / inv_row / drop;
//   gather - one warp per kept row copies x[token] with 16-byte accesses,
//            or quantises it to FP8 E4M3 with a per-row fp32 scale
//            (amax / 448) as the page's FP8 dispatch payload does ("MoE: what
//            it costs to train and serve", Worked example: bytes per token).
#include <cuda_fp8.h>

#include "common.cuh"
#include "kernels.h"
#include "moe.h"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kPerWarp = kDispChunk / kWarps;  // 256 pairs, 8 rounds of 32

// Pair index at position p of the order in which pairs are taken: token by
// token (p itself), or slot by slot (every token's first choice first).
__device__ __forceinline__ int64_t pair_at(int64_t p, int64_t T, int k, int slot_priority)
{
    return slot_priority ? (p % T) * k + p / T : p;
}

__global__ void __launch_bounds__(kThreads)
    dispatch_count_kernel(const int32_t *__restrict__ idx, int64_t T, int k, int slot_priority,
                          int N, int32_t *__restrict__ block_base, uint32_t *status)
{
    grid_dep_wait();
    extern __shared__ int32_t s_cnt[];
    for (int e = threadIdx.x; e < N; e += kThreads)
        s_cnt[e] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t n_pairs = T * k;
    const int64_t base = static_cast<int64_t>(blockIdx.x) * kDispChunk;
    constexpr int R = kDispChunk / kThreads;
    int ev[R];   // every load of the thread issued before the first is used
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t p = base + r * kThreads + threadIdx.x;
        ev[r] = p < n_pairs ? idx[pair_at(p, T, k, slot_priority)] : -1;
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t p = base + r * kThreads + threadIdx.x;
        int e = ev[r];
        if (p < n_pairs && (e < 0 || e >= N)) {
            set_status(status, DEV_BAD_EXPERT);
            e = -1;
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(peers) - 1)
            atomicAdd(&s_cnt[e], __popc(peers));
    }
    __syncthreads();
    for (int e = threadIdx.x; e < N; e += kThreads)
        block_base[static_cast<int64_t>(blockIdx.x) * N + e] = s_cnt[e];
}

// Per expert e (thread e of a 1024-thread block, e < N): total count `run`,
// kept = min(run, C), offsets = exclusive scan of kept over experts, f and
// L_aux = alpha N sum_e f_e p_e summed in a fixed tree order; with a fallback
// expert also offsets[N + 1] = offsets[N] + the pairs over capacity.  Also
// leaves offsets[0..N] in s_off when it is given.  Every thread of the block
// calls it.
__device__ __forceinline__ void expert_offsets_and_aux(int e, int32_t run, int N, int64_t n_pairs,
                                                       int64_t C, int fallback,
                                                       int32_t *__restrict__ counts,
                                                       int32_t *__restrict__ offsets,
                                                       const float *__restrict__ p_mean,
                                                       float *__restrict__ f,
                                                       float *__restrict__ aux_loss, float alpha,
                                                       int32_t *s_off)
{
    __shared__ int32_t s_warp[32];
    __shared__ int32_t s_over[32];
    __shared__ double s_aux[1024];
    const int lane = e & 31, warp = e >> 5;
    int32_t kept = 0;
    if (e < N) {
        counts[e] = run;
        kept = (C >= 0 && run > C) ? static_cast<int32_t>(C) : run;
        if (f != nullptr)
            f[e] = static_cast<float>(static_cast<double>(run) / static_cast<double>(n_pairs));
    }
    // exclusive scan of kept over experts; sum of the overflow
    int32_t incl = kept;
    int32_t over = run - kept;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o)
            incl += v;
        over += __shfl_xor_sync(0xffffffffu, over, o);
    }
    if (lane == 31)
        s_warp[warp] = incl;
    if (lane == 0)
        s_over[warp] = over;
    __syncthreads();
    if (warp == 0) {
        int32_t w = s_warp[lane];
        int32_t wi = w;
        int32_t ov = s_over[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t v = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o)
                wi += v;
            ov += __shfl_xor_sync(0xffffffffu, ov, o);
        }
        s_warp[lane] = wi - w;  // exclusive warp base
        if (lane == 0)
            s_over[0] = ov;
    }
    __syncthreads();
    const int32_t excl = s_warp[warp] + incl - kept;
    if (e < N) {
        offsets[e] = excl;
        if (s_off != nullptr)
            s_off[e] = excl;
    }
    if (e == N - 1) {
        offsets[N] = excl + kept;
        if (s_off != nullptr)
            s_off[N] = excl + kept;
        if (fallback)
            offsets[N + 1] = excl + kept + s_over[0];
    }
    // L_aux = alpha N sum_e f_e p_e, summed in a fixed tree order
    if (aux_loss != nullptr && p_mean != nullptr) {
        double term = 0.0;
        if (e < N)
            term = static_cast<double>(run) / static_cast<double>(n_pairs) *
                   static_cast<double>(p_mean[e]);
        s_aux[e] = term;
        __syncthreads();
        for (int st = 512; st > 0; st >>= 1) {
            if (e < st)
                s_aux[e] += s_aux[e + st];
            __syncthreads();
        }
        if (e == 0)
            *aux_loss = static_cast<float>(static_cast<double>(alpha) * N * s_aux[0]);
    }
}

// Exclusive prefix sum of v[0..n) in place by one 1024-thread block.
__device__ void block_exclusive_scan(int32_t *v, int n)
{
    __shared__ int32_t s_part[32];
    __shared__ int32_t s_carry;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0)
        s_carry = 0;
    __syncthreads();
    for (int c0 = 0; c0 < n; c0 += 1024) {
        const int i = c0 + static_cast<int>(threadIdx.x);
        const int32_t x = i < n ? v[i] : 0;
        int32_t incl = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += y;
        }
        if (lane == 31)
            s_part[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int32_t w = s_part[lane];
            int32_t wi = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int32_t y = __shfl_up_sync(0xffffffffu, wi, o);
                if (lane >= o)
                    wi += y;
            }
            s_part[lane] = wi - w;
        }
        __syncthreads();
        const int32_t carry = s_carry;
        if (i < n)
            v[i] = carry + s_part[warp] + incl - x;
        __syncthreads();
        if (threadIdx.x == 1023)
            s_carry = carry + s_part[31] + incl;
        __syncthreads();
    }
}

__global__ void __launch_bounds__(1024)
    dispatch_scan_kernel(int nblk, int N, int64_t n_pairs, int64_t C, int fallback,
                         int32_t *__restrict__ block_base, int32_t *__restrict__ counts,
                         int32_t *__restrict__ offsets, const float *__restrict__ p_mean,
                         float *__restrict__ f, float *__restrict__ aux_loss, float alpha)
{
    grid_dep_wait();
    const int e = threadIdx.x;
    // fallback: pairs of block b over capacity, then their exclusive scan
    int32_t *fb_base = block_base + static_cast<int64_t>(nblk) * N;
    const bool fb = fallback && C >= 0;
    if (fb)
        for (int b = threadIdx.x; b < nblk; b += 1024)
            fb_base[b] = 0;
    __syncthreads();
    int32_t run = 0;
    if (e < N) {
        constexpr int B = 8;   // the counts of B blocks loaded together
        for (int b0 = 0; b0 < nblk; b0 += B) {
            int32_t vb[B];
#pragma unroll
            for (int u = 0; u < B; ++u)
                vb[u] = b0 + u < nblk ? block_base[static_cast<int64_t>(b0 + u) * N + e] : 0;
#pragma unroll
            for (int u = 0; u < B; ++u) {
                const int b = b0 + u;
                if (b >= nblk)
                    break;
                const int32_t v = vb[u];
                block_base[static_cast<int64_t>(b) * N + e] = run;
                if (fb) {
                    // pairs of this block past the first C of the expert
                    int64_t over = static_cast<int64_t>(run) + v - C;
                    over = over < 0 ? 0 : (over > v ? v : over);
                    if (over > 0)
                        atomicAdd(&fb_base[b], static_cast<int32_t>(over));
                }
                run += v;
            }
        }
    }
    __syncthreads();
    if (fb)
        block_exclusive_scan(fb_base, nblk);
    expert_offsets_and_aux(e, run, N, n_pairs, C, fallback, counts, offsets, p_mean, f, aux_loss,
                           alpha, nullptr);
}

// The whole sort in one block, for batches of at most kFusedMaxPairs pairs and
// N <= kFusedMaxN experts: each of the 32 warps takes a contiguous range of
// positions (in the order pairs are taken), counts its experts, a column scan
// over the warps gives every warp its base inside each expert, and a second
// walk (expert ids kept in shared memory) ranks each pair stably; with a
// fallback expert a third walk places the pairs over capacity.  Same results
// as count + scan + rank, in one launch without a workspace.
constexpr int kFusedThreads = 1024;
constexpr int kFusedWarps = kFusedThreads / 32;

__global__ void __launch_bounds__(kFusedThreads)
    dispatch_fused_kernel(const int32_t *__restrict__ idx, int64_t T, int k, int slot_priority,
                          int N, int64_t C, int fallback, int32_t *__restrict__ counts,
                          int32_t *__restrict__ offsets, int32_t *__restrict__ perm,
                          int32_t *__restrict__ inv_row, uint8_t *__restrict__ drop,
                          const float *__restrict__ p_mean, float *__restrict__ f,
                          float *__restrict__ aux_loss, float alpha, uint32_t *status)
{
    grid_dep_wait();
    extern __shared__ int32_t s_fz[];
    int32_t *s_cnt = s_fz;                                              // [32][N]
    int16_t *s_e = reinterpret_cast<int16_t *>(s_fz + kFusedWarps * N);  // [n_pairs], by position
    __shared__ int32_t s_off[kFusedMaxN + 1];
    __shared__ int32_t s_fbw[kFusedWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_pairs = T * k;
    for (int i = threadIdx.x; i < kFusedWarps * N; i += kFusedThreads)
        s_cnt[i] = 0;
    __syncthreads();
    // positions per warp, a multiple of 32
    const int64_t per_w = (n_pairs + 32 * kFusedWarps - 1) / (32 * kFusedWarps) * 32;
    const int64_t wb = warp * per_w;
    int32_t *mine = s_cnt + warp * N;
    constexpr int U = 4;   // rounds whose loads are issued together
    for (int64_t r0 = 0; r0 < per_w; r0 += 32 * U) {
        int ev[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t p = wb + r0 + 32 * u + lane;
            ev[u] = (r0 + 32 * u < per_w && p < n_pairs) ? idx[pair_at(p, T, k, slot_priority)]
                                                         : -1;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            if (r0 + 32 * u >= per_w)
                break;
            const int64_t p = wb + r0 + 32 * u + lane;
            int e = ev[u];
            if (p < n_pairs) {
                if (e < 0 || e >= N) {
                    set_status(status, DEV_BAD_EXPERT);
                    e = -1;
                }
                s_e[p] = static_cast<int16_t>(e);
            }
            const uint32_t peers = __match_any_sync(0xffffffffu, e);
            if (e >= 0 && lane == __ffs(peers) - 1)
                mine[e] += __popc(peers);
            __syncwarp();
        }
    }
    __syncthreads();
    // column scan: warp w's base inside expert e = pairs of e in warps < w
    int32_t run = 0;
    if (threadIdx.x < N) {
        const int e = threadIdx.x;
        for (int w = 0; w < kFusedWarps; ++w) {
            const int32_t v = s_cnt[w * N + e];
            s_cnt[w * N + e] = run;
            run += v;
        }
    }
    expert_offsets_and_aux(threadIdx.x, run, N, n_pairs, C, fallback, counts, offsets, p_mean, f,
                           aux_loss, alpha, s_off);
    __syncthreads();
    // walk again in order; rank = warp base + earlier rounds + earlier lanes
    int32_t n_over = 0;   // this warp's pairs over capacity (fallback)
    for (int64_t r = 0; r < per_w; r += 32) {
        const int64_t p = wb + r + lane;
        const int e = p < n_pairs ? static_cast<int>(s_e[p]) : -1;
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        int32_t rank = 0;
        if (e >= 0)
            rank = mine[e] + __popc(peers & lanemask_lt());
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1)
            mine[e] += __popc(peers);
        __syncwarp();
        const bool over = e >= 0 && C >= 0 && rank >= C;
        n_over += __popc(__ballot_sync(0xffffffffu, over && fallback));
        if (p < n_pairs) {
            const int64_t i = pair_at(p, T, k, slot_priority);
            if (e < 0 || (over && !fallback)) {
                drop[i] = 1;
                inv_row[i] = -1;
            } else if (over) {
                s_e[p] = -2;   // placed by the walk below
            } else {
                const int32_t row = s_off[e] + rank;
                perm[row] = static_cast<int32_t>(i);
                inv_row[i] = row;
                drop[i] = 0;
            }
        }
    }
    if (!fallback)
        return;
    // fallback rows: offsets[N] + the overflow of earlier warps + earlier rounds and lanes
    if (lane == 0)
        s_fbw[warp] = n_over;
    __syncthreads();
    if (warp == 0) {
        const int32_t w = s_fbw[lane];
        int32_t wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int32_t y = __shfl_up_sync(0xffffffffu, wi, o);
            if (lane >= o)
                wi += y;
        }
        s_fbw[lane] = wi - w;
    }
    __syncthreads();
    int32_t pos = s_off[N] + s_fbw[warp];
    for (int64_t r = 0; r < per_w; r += 32) {
        const int64_t p = wb + r + lane;
        const bool mark = p < n_pairs && s_e[p] == -2;
        const uint32_t bal = __ballot_sync(0xffffffffu, mark);
        if (mark) {
            const int64_t i = pair_at(p, T, k, slot_priority);
            const int32_t row = pos + __popc(bal & lanemask_lt());
            perm[row] = static_cast<int32_t>(i);
            inv_row[i] = row;
            drop[i] = 0;
        }
        pos += __popc(bal);
    }
}

__global__ void __launch_bounds__(kThreads)
    dispatch_rank_kernel(const int32_t *__restrict__ idx, int64_t T, int k, int slot_priority,
                         int N, int64_t C, int fallback, const int32_t *__restrict__ block_base,
                         const int32_t *__restrict__ offsets, int32_t *__restrict__ perm,
                         int32_t *__restrict__ inv_row, uint8_t *__restrict__ drop)
{
    grid_dep_wait();
    extern __shared__ int32_t s_w[];  // [kWarps][N]
    __shared__ uint8_t s_over[kDispChunk];   // fallback: position over capacity
    __shared__ int32_t s_fbw[kWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t n_pairs = T * k;
    const int nblk = static_cast<int>((n_pairs + kDispChunk - 1) / kDispChunk);
    for (int i = threadIdx.x; i < kWarps * N; i += kThreads)
        s_w[i] = 0;
    __syncthreads();
    const int64_t wbase = static_cast<int64_t>(blockIdx.x) * kDispChunk + warp * kPerWarp;
    int32_t *mine = s_w + warp * N;
    // this lane's experts of the warp's rounds, loaded once for both walks
    constexpr int R = kPerWarp / 32;
    int ev[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t p = wbase + r * 32 + lane;
        int e = p < n_pairs ? idx[pair_at(p, T, k, slot_priority)] : -1;
        ev[r] = (e < 0 || e >= N) ? -1 : e;
    }
    // phase 1: per-warp counts
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int e = ev[r];
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        if (e >= 0 && lane == __ffs(peers) - 1)
            mine[e] += __popc(peers);
        __syncwarp();
    }
    __syncthreads();
    // phase 2: warp bases = block base + counts of earlier warps
    for (int e = threadIdx.x; e < N; e += kThreads) {
        int32_t run = block_base[static_cast<int64_t>(blockIdx.x) * N + e];
        for (int w = 0; w < kWarps; ++w) {
            const int32_t v = s_w[w * N + e];
            s_w[w * N + e] = run;
            run += v;
        }
    }
    __syncthreads();
    // phase 3: walk the pairs in order; rank = warp base + earlier lanes
    int32_t n_over = 0;
#pragma unroll
    for (int r = 0; r < R; ++r) {
        const int64_t p = wbase + r * 32 + lane;
        const int e = ev[r];
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        int32_t rank = 0;
        if (e >= 0)
            rank = mine[e] + __popc(peers & lanemask_lt());
        __syncwarp();
        if (e >= 0 && lane == __ffs(peers) - 1)
            mine[e] += __popc(peers);
        __syncwarp();
        const bool over = e >= 0 && C >= 0 && rank >= C;
        n_over += __popc(__ballot_sync(0xffffffffu, over && fallback));
        s_over[warp * kPerWarp + r * 32 + lane] = (over && fallback) ? 1 : 0;
        if (p < n_pairs) {
            const int64_t i = pair_at(p, T, k, slot_priority);
            if (e < 0 || (over && !fallback)) {
                drop[i] = 1;
                inv_row[i] = -1;
            } else if (!over) {
                const int32_t row = offsets[e] + rank;
                perm[row] = static_cast<int32_t>(i);
                inv_row[i] = row;
                drop[i] = 0;
            }
        }
    }
    if (!fallback)
        return;
    // phase 4 (fallback): this block's pairs over capacity, in order, after
    // those of earlier blocks (scan kernel) and earlier warps
    if (lane == 0)
        s_fbw[warp] = n_over;
    __syncthreads();
    if (threadIdx.x == 0) {
        int32_t run = offsets[N] + block_base[static_cast<int64_t>(nblk) * N + blockIdx.x];
        for (int w = 0; w < kWarps; ++w) {
            const int32_t v = s_fbw[w];
            s_fbw[w] = run;
            run += v;
        }
    }
    __syncthreads();
    int32_t pos = s_fbw[warp];
    for (int r = 0; r < kPerWarp / 32; ++r) {
        const int64_t p = wbase + r * 32 + lane;
        const bool mark = s_over[warp * kPerWarp + r * 32 + lane] != 0;
        const uint32_t bal = __ballot_sync(0xffffffffu, mark);
        if (mark) {
            const int64_t i = pair_at(p, T, k, slot_priority);
            const int32_t row = pos + __popc(bal & lanemask_lt());
            perm[row] = static_cast<int32_t>(i);
            inv_row[i] = row;
            drop[i] = 0;
        }
        pos += __popc(bal);
    }
}

// One warp per kept row.  BF16 in -> copy (or FP8 quantise); F32 in -> copy.
template <bool BF16, bool FP8>
__global__ void __launch_bounds__(kThreads)
    dispatch_gather_kernel(const uint8_t *__restrict__ x, int d, int k,
                           const int32_t *__restrict__ perm, const int32_t *__restrict__ R_ptr,
                           uint8_t *__restrict__ x_perm, float *__restrict__ x_scale,
                           __nv_bfloat16 *__restrict__ x_bf16_copy)
{
    grid_dep_wait();
    const int lane = threadIdx.x & 31;
    const int64_t R = *R_ptr;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
    const int esz = BF16 ? 2 : 4;
    const int chunks = d * esz / 16;
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5); r < R;
         r += nwarps) {
        const int64_t t = perm[r] / k;
        const uint4 *src = reinterpret_cast<const uint4 *>(x + t * static_cast<int64_t>(d) * esz);
        if (!FP8) {
            uint4 *dst = reinterpret_cast<uint4 *>(x_perm + r * static_cast<int64_t>(d) * esz);
            constexpr int U = 4;  // loads in flight per lane
            for (int c0 = lane; c0 < chunks; c0 += 32 * U) {
                uint4 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (c0 + 32 * u < chunks)
                        v[u] = __ldg(src + c0 + 32 * u);
#pragma unroll
                for (int u = 0; u < U; ++u)
                    if (c0 + 32 * u < chunks)
                        dst[c0 + 32 * u] = v[u];
            }
        } else {
            float amax = 0.0f;
            for (int c = lane; c < chunks; c += 32) {
                const uint4 v = __ldg(src + c);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    amax = fmaxf(amax, fabsf(__uint_as_float(w[i] << 16)));
                    amax = fmaxf(amax, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
                }
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1)
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
            const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
            if (lane == 0)
                x_scale[r] = scale;
            uint2 *dq = reinterpret_cast<uint2 *>(x_perm + r * static_cast<int64_t>(d));
            uint4 *db = x_bf16_copy
                            ? reinterpret_cast<uint4 *>(x_bf16_copy + r * static_cast<int64_t>(d))
                            : nullptr;
            for (int c = lane; c < chunks; c += 32) {
                const uint4 v = __ldg(src + c);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                uint32_t q[2] = {0u, 0u};
                uint32_t b[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float lo = __fdiv_rn(__uint_as_float(w[i] << 16), scale);
                    const float hi = __fdiv_rn(__uint_as_float(w[i] & 0xFFFF0000u), scale);
                    const __nv_fp8_storage_t qlo = __nv_cvt_float_to_fp8(lo, __NV_SATFINITE, __NV_E4M3);
                    const __nv_fp8_storage_t qhi = __nv_cvt_float_to_fp8(hi, __NV_SATFINITE, __NV_E4M3);
                    q[i >> 1] |= (static_cast<uint32_t>(qlo) | (static_cast<uint32_t>(qhi) << 8))
                                 << (16 * (i & 1));
                    if (db) {
                        __nv_fp8_e4m3 flo, fhi;
                        flo.__x = qlo;
                        fhi.__x = qhi;
                        b[i] = pack_bf16x2(static_cast<float>(flo), static_cast<float>(fhi));
                    }
                }
                dq[c] = make_uint2(q[0], q[1]);
                if (db)
                    db[c] = make_uint4(b[0], b[1], b[2], b[3]);
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads)
    fp8_to_bf16_kernel(const uint8_t *__restrict__ q, int d, const int32_t *__restrict__ R_ptr,
                       __nv_bfloat16 *__restrict__ out)
{
    grid_dep_wait();
    const int lane = threadIdx.x & 31;
    const int64_t R = *R_ptr;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
    const int chunks = d / 8;
    for (int64_t r = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5); r < R;
         r += nwarps) {
        const uint2 *src = reinterpret_cast<const uint2 *>(q + r * static_cast<int64_t>(d));
        uint4 *dst = reinterpret_cast<uint4 *>(out + r * static_cast<int64_t>(d));
        for (int c = lane; c < chunks; c += 32) {
            const uint2 v = src[c];
            const uint32_t w[2] = {v.x, v.y};
            uint32_t b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                __nv_fp8_e4m3 lo, hi;
                lo.__x = static_cast<__nv_fp8_storage_t>((w[i >> 1] >> (16 * (i & 1))) & 0xFF);
                hi.__x = static_cast<__nv_fp8_storage_t>((w[i >> 1] >> (16 * (i & 1) + 8)) & 0xFF);
                b[i] = pack_bf16x2(static_cast<float>(lo), static_cast<float>(hi));
            }
            dst[c] = make_uint4(b[0], b[1], b[2], b[3]);
        }
    }
}

// FP8 payload of the fused layer path, written straight into the expert-
// ordered GEMM rows: one warp per token computes scale = amax / 448 (1 for an
// all-zero row) and codes = E4M3(x / scale), as the gather kernel above does
// per row, and writes the codes' values as bf16 (exact) to every kept row of
// the token (inv_row), with the scale beside each row for the GEMM epilogue.
// Each token is read twice from L2 and quantised once.
template <int KM>
__global__ void __launch_bounds__(kThreads)
    quantize_scatter_kernel(const uint8_t *__restrict__ x, int64_t T, int d, int k,
                            const int32_t *__restrict__ inv_row, uint8_t *__restrict__ out,
                            float *__restrict__ out_scale)
{
    grid_dep_wait();
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
    const int chunks = d / 8;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5); t < T;
         t += nwarps) {
        int32_t rows[KM];
        const int32_t my_row = lane < k ? inv_row[t * k + lane] : -1;
#pragma unroll
        for (int j = 0; j < KM; ++j)
            rows[j] = __shfl_sync(0xffffffffu, my_row, j);
        const uint4 *src = reinterpret_cast<const uint4 *>(x + t * static_cast<int64_t>(d) * 2);
        float amax = 0.0f;
        for (int c = lane; c < chunks; c += 32) {
            const uint4 v = __ldg(src + c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                amax = fmaxf(amax, fabsf(__uint_as_float(w[i] << 16)));
                amax = fmaxf(amax, fabsf(__uint_as_float(w[i] & 0xFFFF0000u)));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        if (lane < k && my_row >= 0)
            out_scale[my_row] = scale;
        for (int c = lane; c < chunks; c += 32) {
            const uint4 v = __ldg(src + c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                __nv_fp8_e4m3 lo, hi;
                lo.__x = __nv_cvt_float_to_fp8(__fdiv_rn(__uint_as_float(w[i] << 16), scale),
                                               __NV_SATFINITE, __NV_E4M3);
                hi.__x = __nv_cvt_float_to_fp8(__fdiv_rn(__uint_as_float(w[i] & 0xFFFF0000u), scale),
                                               __NV_SATFINITE, __NV_E4M3);
                b[i] = pack_bf16x2(static_cast<float>(lo), static_cast<float>(hi));
            }
            const uint4 o = make_uint4(b[0], b[1], b[2], b[3]);
#pragma unroll
            for (int j = 0; j < KM; ++j)
                if (j < k && rows[j] >= 0)
                    reinterpret_cast<uint4 *>(out + static_cast<int64_t>(rows[j]) * d * 2)[c] = o;
        }
    }
}

// The same with the token's first pass (the amax) issuing all of a lane's CPL
// 16-byte loads (chunks lane + 32 i) at once, so the row's reads are in flight
// together; the second pass finds the row in L1.
template <int KM, int CPL>
__global__ void __launch_bounds__(kThreads)
    quantize_scatter_wide_kernel(const uint8_t *__restrict__ x, int64_t T, int d, int k,
                                 const int32_t *__restrict__ inv_row, uint8_t *__restrict__ out,
                                 float *__restrict__ out_scale)
{
    grid_dep_wait();
    const int lane = threadIdx.x & 31;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
    const int chunks = d / 8;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5); t < T;
         t += nwarps) {
        int32_t rows[KM];
        const int32_t my_row = lane < k ? inv_row[t * k + lane] : -1;
#pragma unroll
        for (int j = 0; j < KM; ++j)
            rows[j] = __shfl_sync(0xffffffffu, my_row, j);
        const uint4 *src = reinterpret_cast<const uint4 *>(x + t * static_cast<int64_t>(d) * 2);
        float amax = 0.0f;
        {
            uint4 v[CPL];
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const int c = lane + 32 * i;
                v[i] = c < chunks ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int i = 0; i < CPL; ++i) {
                const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    amax = fmaxf(amax, fabsf(__uint_as_float(w[q] << 16)));
                    amax = fmaxf(amax, fabsf(__uint_as_float(w[q] & 0xFFFF0000u)));
                }
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        const float scale = amax > 0.0f ? __fdiv_rn(amax, 448.0f) : 1.0f;
        if (lane < k && my_row >= 0)
            out_scale[my_row] = scale;
#pragma unroll 1
        for (int c = lane; c < chunks; c += 32) {
            const uint4 v = __ldg(src + c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t b[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                __nv_fp8_e4m3 lo, hi;
                lo.__x = __nv_cvt_float_to_fp8(__fdiv_rn(__uint_as_float(w[q] << 16), scale),
                                               __NV_SATFINITE, __NV_E4M3);
                hi.__x = __nv_cvt_float_to_fp8(__fdiv_rn(__uint_as_float(w[q] & 0xFFFF0000u), scale),
                                               __NV_SATFINITE, __NV_E4M3);
                b[q] = pack_bf16x2(static_cast<float>(lo), static_cast<float>(hi));
            }
            const uint4 o = make_uint4(b[0], b[1], b[2], b[3]);
#pragma unroll
            for (int j = 0; j < KM; ++j)
                if (j < k && rows[j] >= 0)
                    reinterpret_cast<uint4 *>(out + static_cast<int64_t>(rows[j]) * d * 2)[c] = o;
        }
    }
}

int gather_grid(int64_t rows)
{
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t want = (rows + kWarps - 1) / kWarps;
    const int64_t cap = static_cast<int64_t>(sms) * 8;
    if (want > cap)
        want = cap;
    return want < 1 ? 1 : static_cast<int>(want);
}

}  // namespace

cudaError_t launch_dispatch(const DispatchLaunch &L, cudaStream_t stream)
{
    const int64_t n_pairs = L.T * L.k;
    if (n_pairs == 0)
        return cudaSuccess;
    int sort_launches;
    if (n_pairs <= kFusedMaxPairs && L.N <= kFusedMaxN) {
        const size_t smem = kFusedWarps * L.N * sizeof(int32_t) + n_pairs * sizeof(int16_t);
        static DeviceOnce attr_once;   // per device: function attributes are per device
        const cudaError_t err = device_once(attr_once, nullptr, [](int *) {
            return cudaFuncSetAttribute(
                dispatch_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                static_cast<int>(kFusedWarps * kFusedMaxN * sizeof(int32_t) +
                                 kFusedMaxPairs * sizeof(int16_t)));
        });
        if (err != cudaSuccess)
            return err;
        launch_k(dispatch_fused_kernel, 1, kFusedThreads, smem, stream, L.topk_idx, L.T, L.k,
                 L.slot_priority, L.N, L.capacity, L.fallback, L.counts, L.offsets, L.perm,
                 L.inv_row, L.drop, L.p_mean, L.f, L.aux_loss, L.aux_alpha, L.status);
        sort_launches = 1;
    } else {
        const int nblk = static_cast<int>((n_pairs + kDispChunk - 1) / kDispChunk);
        launch_k(dispatch_count_kernel, nblk, kThreads, L.N * sizeof(int32_t), stream,
                 L.topk_idx, L.T, L.k, L.slot_priority, L.N, L.block_base, L.status);
        launch_k(dispatch_scan_kernel, 1, 1024, 0, stream, nblk, L.N, n_pairs, L.capacity,
                 L.fallback, L.block_base, L.counts, L.offsets, L.p_mean, L.f, L.aux_loss,
                 L.aux_alpha);
        launch_k(dispatch_rank_kernel, nblk, kThreads, kWarps * L.N * sizeof(int32_t), stream,
                 L.topk_idx, L.T, L.k, L.slot_priority, L.N, L.capacity, L.fallback, L.block_base,
                 L.offsets, L.perm, L.inv_row, L.drop);
        sort_launches = 3;
    }
    if (L.x_perm == nullptr) {      // the caller builds the expert-ordered rows itself
        count_launches(sort_launches);
        return cudaGetLastError();
    }
    const int grid = gather_grid(n_pairs);
    const uint8_t *x = static_cast<const uint8_t *>(L.x);
    uint8_t *xp = static_cast<uint8_t *>(L.x_perm);
    if (L.dtype == MOE_F32)
        launch_k(dispatch_gather_kernel<false, false>, grid, kThreads, 0, stream, 
            x, L.d, L.k, L.perm, L.offsets + L.N + (L.fallback ? 1 : 0), xp, nullptr, nullptr);
    else if (!L.fp8)
        launch_k(dispatch_gather_kernel<true, false>, grid, kThreads, 0, stream, 
            x, L.d, L.k, L.perm, L.offsets + L.N + (L.fallback ? 1 : 0), xp, nullptr, nullptr);
    else
        launch_k(dispatch_gather_kernel<true, true>, grid, kThreads, 0, stream, 
            x, L.d, L.k, L.perm, L.offsets + L.N + (L.fallback ? 1 : 0), xp, L.x_scale,
            static_cast<__nv_bfloat16 *>(L.x_bf16_copy));
    count_launches(sort_launches + 1);
    return cudaGetLastError();
}

cudaError_t launch_quantize_scatter(const void *x, int64_t T, int32_t d, int32_t k,
                                    const int32_t *inv_row, void *out, float *out_scale,
                                    cudaStream_t stream)
{
    if (T == 0)
        return cudaSuccess;
    if (k < 1 || k > 8)
        return cudaErrorInvalidValue;
    const uint8_t *xs = static_cast<const uint8_t *>(x);
    uint8_t *o = static_cast<uint8_t *>(out);
    const int grid = gather_grid(T);
    const int cpl = (d / 8 + 31) / 32;   // 16-byte chunks of a row per lane
    // rows of 4097-8192 elements (the DeepSeek-V3 7168 among them): the first
    // pass's loads all in flight at once
    if (k > 2 && cpl > 16 && cpl <= 28)
        launch_k(quantize_scatter_wide_kernel<8, 28>, grid, kThreads, 0, stream, xs, T, d, k,
                 inv_row, o, out_scale);
    else if (k > 2 && cpl > 28 && cpl <= 32)
        launch_k(quantize_scatter_wide_kernel<8, 32>, grid, kThreads, 0, stream, xs, T, d, k,
                 inv_row, o, out_scale);
    else if (k <= 2)
        launch_k(quantize_scatter_kernel<2>, grid, kThreads, 0, stream, xs, T, d, k, inv_row, o,
                 out_scale);
    else
        launch_k(quantize_scatter_kernel<8>, grid, kThreads, 0, stream, xs, T, d, k, inv_row, o,
                 out_scale);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_fp8_to_bf16(const uint8_t *q, int64_t rows_cap, int32_t d,
                               const int32_t *offsets, int32_t N, void *out, cudaStream_t stream)
{
    if (rows_cap == 0)
        return cudaSuccess;
    launch_k(fp8_to_bf16_kernel, gather_grid(rows_cap), kThreads, 0, stream, 
        q, d, offsets + N, static_cast<__nv_bfloat16 *>(out));
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
