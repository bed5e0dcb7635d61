// fp32 grouped GEMM on the CUDA cores, for fp32 layers (the tensor-core
// kernel takes bf16 operands; TF32 would not meet an fp32 parity bound).
//
//   out[r, n] = act( sum_k A[r, k] B[g n_out + n, k] )   (SwiGLU: silu(.) * (A B2^T))
//
// for the rows r of group g.  One block per row: the row of A is staged in
// shared memory and each thread produces output columns.  Sized for small
// fp32 layers, where launch latency rather than arithmetic bounds the time.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kThreads = 128;

template <int EPI>
__global__ void __launch_bounds__(kThreads)
    simt_gemm_f32_kernel(const float *__restrict__ A, int64_t rows_cap, int K,
                         const float *__restrict__ B, const float *__restrict__ B2, int n_out,
                         const int32_t *__restrict__ offsets, int G, int w_blocks,
                         int rows_single, float *__restrict__ out)
{
    grid_dep_wait();
    extern __shared__ float s_a[];
    int64_t R = offsets ? offsets[G] : rows_single;
    if (R > rows_cap)
        R = rows_cap;
    for (int64_t r = blockIdx.x; r < R; r += gridDim.x) {
        int g = 0;
        if (offsets) {
            int lo = 0, hi = G;  // largest g with offsets[g] <= r
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (offsets[mid] <= r)
                    lo = mid;
                else
                    hi = mid;
            }
            g = lo % w_blocks;   // the group's weight block
        }
        __syncthreads();
        for (int i = threadIdx.x; i < K; i += kThreads)
            s_a[i] = A[r * K + i];
        __syncthreads();
        for (int n = threadIdx.x; n < n_out; n += kThreads) {
            const float *b = B + (static_cast<int64_t>(g) * n_out + n) * K;
            float acc = 0.0f;
            for (int i = 0; i < K; ++i)
                acc = fmaf(s_a[i], b[i], acc);
            float v;
            if (EPI == EPI_SWIGLU) {
                const float *b2 = B2 + (static_cast<int64_t>(g) * n_out + n) * K;
                float acc2 = 0.0f;
                for (int i = 0; i < K; ++i)
                    acc2 = fmaf(s_a[i], b2[i], acc2);
                v = acc / (1.0f + expf(-acc)) * acc2;
            } else if (EPI == EPI_RELU) {
                v = fmaxf(acc, 0.0f);
            } else {
                v = acc;
            }
            out[r * n_out + n] = v;
        }
    }
}

}  // namespace

cudaError_t launch_simt_gemm_f32(int epi, const float *A, int64_t rows_cap, int32_t K,
                                 const float *B, const float *B2, int32_t n_out,
                                 const int32_t *offsets, int32_t G, int32_t w_blocks,
                                 int32_t rows_single, float *out, cudaStream_t stream)
{
    if (w_blocks <= 0)
        w_blocks = G;
    if (rows_cap == 0)
        return cudaSuccess;
    int sms = 148, dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t grid = rows_cap < static_cast<int64_t>(sms) * 8 ? rows_cap : static_cast<int64_t>(sms) * 8;
    const size_t smem = static_cast<size_t>(K) * sizeof(float);
    if (smem > 48 * 1024)
        return cudaErrorInvalidValue;
    if (epi == EPI_SWIGLU)
        launch_k(simt_gemm_f32_kernel<EPI_SWIGLU>, static_cast<int>(grid), kThreads, smem, stream, 
            A, rows_cap, K, B, B2, n_out, offsets, G, w_blocks, rows_single, out);
    else if (epi == EPI_RELU)
        launch_k(simt_gemm_f32_kernel<EPI_RELU>, static_cast<int>(grid), kThreads, smem, stream, 
            A, rows_cap, K, B, B2, n_out, offsets, G, w_blocks, rows_single, out);
    else
        launch_k(simt_gemm_f32_kernel<EPI_STORE>, static_cast<int>(grid), kThreads, smem, stream, 
            A, rows_cap, K, B, B2, n_out, offsets, G, w_blocks, rows_single, out);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace moe
