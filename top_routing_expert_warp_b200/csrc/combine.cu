// Combine: the gate-weighted un-permute.
//
//   y[t] = sum over kept slots j (in slot order) of g[t, j] * y_perm[inv_row[t k + j]]
//          (+ y_shared[t])
//
// "moe communication costs", Router design: the layer output is the sum over
// the selected experts of G(x)_i E_i(x); on one GPU the return all-to-all of
// "MoE: what it costs to train and serve" (Expert parallelism, step 3) becomes
// this gather.  A dropped slot (inv_row = -1, "moe communication costs",
// Capacity factor) contributes nothing.  The always-on shared expert's output,
// when present, is added with coefficient 1.  One warp per token, 16-byte
// accesses, fp32 accumulation in a fixed order.
#include "common.cuh"
#include "kernels.h"
#include "moe.h"

namespace moe {

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxK = 8;

// KM: bound on k (the loads of all slots are held in registers at once);
// U chunks per lane per pass (4 for k <= 2, else 2).
template <bool BF16, int KM>
__global__ void __launch_bounds__(kThreads)
    combine_kernel(const uint8_t *__restrict__ y_perm, const int32_t *__restrict__ inv_row,
                   const float *__restrict__ topk_w, const uint8_t *__restrict__ y_shared,
                   uint8_t *__restrict__ y, int64_t T, int d, int k, int64_t rows_cap,
                   uint32_t *status)
{
    grid_dep_wait();
    const int lane = threadIdx.x & 31;
    const int esz = BF16 ? 2 : 4;
    const int chunks = d * esz / 16;
    const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kWarps;
    for (int64_t t = static_cast<int64_t>(blockIdx.x) * kWarps + (threadIdx.x >> 5); t < T;
         t += nwarps) {
        int32_t row[KM];
        float g[KM];
        int32_t my_row = -1;
        float my_g = 0.0f;
        if (lane < k) {
            my_row = inv_row[t * k + lane];
            my_g = topk_w[t * k + lane];
            if (my_row >= rows_cap || my_row < -1) {
                set_status(status, DEV_BAD_ROW);
                my_row = -1;
            }
        }
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            row[j] = __shfl_sync(0xffffffffu, my_row, j);
            g[j] = __shfl_sync(0xffffffffu, my_g, j);
        }
        // U chunks per lane per pass; the loads of every slot are issued
        // before any is used (predicated, no branches), so k * U loads per
        // lane are in flight at once
        constexpr int U = KM >= 4 ? 2 : 4;
        constexpr int V = BF16 ? 8 : 4;
        for (int c0 = lane; c0 < chunks; c0 += 32 * U) {
            uint4 v[KM][U];
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    y_perm + static_cast<int64_t>(row[j] > 0 ? row[j] : 0) * d * esz);
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + 32 * u;
                    v[j][u] = (j < k && row[j] >= 0 && c < chunks) ? __ldg(src + c)
                                                                   : make_uint4(0, 0, 0, 0);
                }
            }
            float acc[U][V];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < V; ++i)
                    acc[u][i] = 0.0f;
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                if (j < k && row[j] >= 0) {
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const uint32_t w[4] = {v[j][u].x, v[j][u].y, v[j][u].z, v[j][u].w};
                        if (BF16) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                acc[u][2 * i] = fmaf(g[j], __uint_as_float(w[i] << 16), acc[u][2 * i]);
                                acc[u][2 * i + 1] =
                                    fmaf(g[j], __uint_as_float(w[i] & 0xFFFF0000u), acc[u][2 * i + 1]);
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                acc[u][i] = fmaf(g[j], __uint_as_float(w[i]), acc[u][i]);
                        }
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + 32 * u;
                if (c >= chunks)
                    continue;
                if (y_shared != nullptr) {
                    const uint4 v = __ldg(reinterpret_cast<const uint4 *>(
                                              y_shared + t * static_cast<int64_t>(d) * esz) + c);
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                    if (BF16) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            acc[u][2 * i] += __uint_as_float(w[i] << 16);
                            acc[u][2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            acc[u][i] += __uint_as_float(w[i]);
                    }
                }
                uint4 o;
                if (BF16) {
                    o.x = pack_bf16x2(acc[u][0], acc[u][1]);
                    o.y = pack_bf16x2(acc[u][2], acc[u][3]);
                    o.z = pack_bf16x2(acc[u][4], acc[u][5]);
                    o.w = pack_bf16x2(acc[u][6], acc[u][7]);
                } else {
                    o.x = __float_as_uint(acc[u][0]);
                    o.y = __float_as_uint(acc[u][1]);
                    o.z = __float_as_uint(acc[u][2]);
                    o.w = __float_as_uint(acc[u][3]);
                }
                reinterpret_cast<uint4 *>(y + t * static_cast<int64_t>(d) * esz)[c] = o;
            }
        }
    }
}

// Wide rows (d of 2048 bf16 or more): one block per token, each thread a
// few 16-byte chunks of every slot, all of a pass's loads issued before they
// are used.  Same arithmetic, in the same order, as combine_kernel.
constexpr int kTokThreads = 256;

template <bool BF16, int KM>
__global__ void __launch_bounds__(kTokThreads, 3)
    combine_token_kernel(const uint8_t *__restrict__ y_perm, const int32_t *__restrict__ inv_row,
                         const float *__restrict__ topk_w, const uint8_t *__restrict__ y_shared,
                         uint8_t *__restrict__ y, int64_t T, int d, int k, int64_t rows_cap,
                         uint32_t *status)
{
    grid_dep_wait();
    __shared__ int32_t s_row[KM];
    __shared__ float s_g[KM];
    const int esz = BF16 ? 2 : 4;
    const int chunks = d * esz / 16;
    constexpr int U = KM >= 8 ? 1 : (KM >= 4 ? 2 : 4);
    constexpr int V = BF16 ? 8 : 4;
    for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
        __syncthreads();   // the previous token's slots are no longer read
        if (threadIdx.x < KM) {
            const int j = threadIdx.x;
            int32_t row = -1;
            float g = 0.0f;
            if (j < k) {
                row = inv_row[t * k + j];
                g = topk_w[t * k + j];
                if (row >= rows_cap || row < -1) {
                    set_status(status, DEV_BAD_ROW);
                    row = -1;
                }
            }
            s_row[j] = row;
            s_g[j] = g;
        }
        __syncthreads();
        int32_t row[KM];
        float g[KM];
#pragma unroll
        for (int j = 0; j < KM; ++j) {
            row[j] = s_row[j];
            g[j] = s_g[j];
        }
        for (int c0 = threadIdx.x; c0 < chunks; c0 += kTokThreads * U) {
            uint4 v[KM][U];
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                const uint4 *src = reinterpret_cast<const uint4 *>(
                    y_perm + static_cast<int64_t>(row[j] > 0 ? row[j] : 0) * d * esz);
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const int c = c0 + kTokThreads * u;
                    v[j][u] = (j < k && row[j] >= 0 && c < chunks) ? __ldg(src + c)
                                                                   : make_uint4(0, 0, 0, 0);
                }
            }
            uint4 sh[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + kTokThreads * u;
                sh[u] = (y_shared != nullptr && c < chunks)
                            ? __ldg(reinterpret_cast<const uint4 *>(
                                        y_shared + t * static_cast<int64_t>(d) * esz) + c)
                            : make_uint4(0, 0, 0, 0);
            }
            float acc[U][V];
#pragma unroll
            for (int u = 0; u < U; ++u)
#pragma unroll
                for (int i = 0; i < V; ++i)
                    acc[u][i] = 0.0f;
#pragma unroll
            for (int j = 0; j < KM; ++j) {
                if (j < k && row[j] >= 0) {
#pragma unroll
                    for (int u = 0; u < U; ++u) {
                        const uint32_t w[4] = {v[j][u].x, v[j][u].y, v[j][u].z, v[j][u].w};
                        if (BF16) {
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                acc[u][2 * i] = fmaf(g[j], __uint_as_float(w[i] << 16), acc[u][2 * i]);
                                acc[u][2 * i + 1] =
                                    fmaf(g[j], __uint_as_float(w[i] & 0xFFFF0000u), acc[u][2 * i + 1]);
                            }
                        } else {
#pragma unroll
                            for (int i = 0; i < 4; ++i)
                                acc[u][i] = fmaf(g[j], __uint_as_float(w[i]), acc[u][i]);
                        }
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + kTokThreads * u;
                if (c >= chunks)
                    continue;
                if (y_shared != nullptr) {
                    const uint32_t w[4] = {sh[u].x, sh[u].y, sh[u].z, sh[u].w};
                    if (BF16) {
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            acc[u][2 * i] += __uint_as_float(w[i] << 16);
                            acc[u][2 * i + 1] += __uint_as_float(w[i] & 0xFFFF0000u);
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            acc[u][i] += __uint_as_float(w[i]);
                    }
                }
                uint4 o;
                if (BF16) {
                    o.x = pack_bf16x2(acc[u][0], acc[u][1]);
                    o.y = pack_bf16x2(acc[u][2], acc[u][3]);
                    o.z = pack_bf16x2(acc[u][4], acc[u][5]);
                    o.w = pack_bf16x2(acc[u][6], acc[u][7]);
                } else {
                    o.x = __float_as_uint(acc[u][0]);
                    o.y = __float_as_uint(acc[u][1]);
                    o.z = __float_as_uint(acc[u][2]);
                    o.w = __float_as_uint(acc[u][3]);
                }
                reinterpret_cast<uint4 *>(y + t * static_cast<int64_t>(d) * esz)[c] = o;
            }
        }
    }
}

}  // namespace

cudaError_t launch_combine(int dtype, const void *y_perm, const int32_t *inv_row,
                           const float *topk_w, const void *y_shared, void *y, int64_t T,
                           int32_t d, int32_t k, uint32_t *status, cudaStream_t stream)
{
    if (T == 0)
        return cudaSuccess;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t grid = (T + kWarps - 1) / kWarps;
    if (grid > static_cast<int64_t>(sms) * 8)
        grid = static_cast<int64_t>(sms) * 8;
    const int64_t rows_cap = T * k;
    const uint8_t *yp = static_cast<const uint8_t *>(y_perm);
    const uint8_t *ys = static_cast<const uint8_t *>(y_shared);
    uint8_t *yo = static_cast<uint8_t *>(y);
    const int g = static_cast<int>(grid);
    if (dtype == MOE_BF16 && d >= 2048 && k >= 4) {
        // wide rows and many slots: a block per token
        const int gt = static_cast<int>(T < static_cast<int64_t>(sms) * 8 ? T : sms * 8);
        if (k <= 2)
            launch_k(combine_token_kernel<true, 2>, gt, kTokThreads, 0, stream, yp, inv_row,
                     topk_w, ys, yo, T, d, k, rows_cap, status);
        else if (k <= 4)
            launch_k(combine_token_kernel<true, 4>, gt, kTokThreads, 0, stream, yp, inv_row,
                     topk_w, ys, yo, T, d, k, rows_cap, status);
        else
            launch_k(combine_token_kernel<true, kMaxK>, gt, kTokThreads, 0, stream, yp, inv_row,
                     topk_w, ys, yo, T, d, k, rows_cap, status);
        count_launches(1);
        return cudaGetLastError();
    }
    if (dtype == MOE_BF16) {
        if (k <= 1)
            launch_k(combine_kernel<true, 1>, g, kThreads, 0, stream, yp, inv_row, topk_w, ys, yo,
                     T, d, k, rows_cap, status);
        else if (k <= 2)
            launch_k(combine_kernel<true, 2>, g, kThreads, 0, stream, yp, inv_row, topk_w, ys, yo,
                     T, d, k, rows_cap, status);
        else if (k <= 4)
            launch_k(combine_kernel<true, 4>, g, kThreads, 0, stream, yp, inv_row, topk_w, ys, yo,
                     T, d, k, rows_cap, status);
        else
            launch_k(combine_kernel<true, kMaxK>, g, kThreads, 0, stream, yp, inv_row, topk_w, ys,
                     yo, T, d, k, rows_cap, status);
    } else {
        launch_k(combine_kernel<false, kMaxK>, g, kThreads, 0, stream, yp, inv_row, topk_w, ys, yo,
                 T, d, k, rows_cap, status);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
