// Grouped GEMM on CTA pairs (tcgen05 cta_group::2), for compute-bound shapes.
//
// Same contract as gemm_tc.cu (rows of group g times B[g * n_out + n, :]^T,
// bf16 K-major operands, fp32 accumulation, ReLU / SwiGLU / plain epilogue),
// but a tile is 256 rows x 256 MMA columns computed by two CTAs of a cluster:
// each CTA stages its own 128 rows of A and its own half of B (128 rows), and
// one MMA issued by the first CTA of the pair reads both CTAs' shared memory.
// Per SM this halves the B bytes every k-block must bring into shared memory
// (32 KB instead of 48 KB for the same tensor work), which is what limits the
// one-CTA kernel on the Mixtral-shaped expert projections.
//
// Roles (192 threads per CTA):
//   warp 0: TMA producer of this CTA's A and B halves (both CTAs);
//   warp 1: TMEM allocation (collective over the pair); in the first CTA the
//           MMA issuer;
//   warps 2-5: epilogue of this CTA's 128 rows, which the MMA leaves in this
//           CTA's TMEM; the release of an accumulator is an arrive on the
//           first CTA's barrier (remote for the second CTA).
// A stage is "full" on the first CTA's barrier, which expects the bytes of
// both halves: the second CTA's TMA loads land in its own shared memory and
// count their bytes on that barrier (the pair form of the bulk tensor copy).
// Stage-free and accumulator-full signals are tcgen05.commit arrivals
// multicast to both CTAs.  No TMA multicast is used.  Every wait is bounded;
// a cluster barrier precedes the collective TMEM release.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int PBM = 256;                 // rows per pair tile
constexpr int HBM = 128;                 // rows per CTA
constexpr int BK = 64;
constexpr int BN = 256;                  // MMA N
constexpr int A_BYTES = HBM * BK * 2;    // 16 KB
constexpr int B_BYTES = 128 * BK * 2;    // 16 KB: this CTA's half of B
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int STAGES = 6;
constexpr int kThreads = 192;
constexpr int kMaxGroups = 1024;
constexpr int TMEM_COLS = 512;           // two 256-column accumulators
constexpr int AUX_BYTES = 8 * (2 * STAGES + 5) + 16 + 8 * (kMaxGroups + 2);
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + AUX_BYTES;

struct PairParams {
    const int32_t *offsets;
    int32_t rows_single;
    int32_t G;
    int32_t w_blocks;        // group g uses weight block g % w_blocks
    int32_t n_out;
    int32_t K;
    void *out;
    int64_t ld_out;
    const float *row_scale;
    int64_t rows_cap;
    uint32_t *status;
};

struct PairTile {
    int32_t g, row0, rows_valid, n0;
};

__device__ __forceinline__ PairTile pair_tile(int t, const int32_t *s_prefix,
                                              const int32_t *s_off, int G, int outn)
{
    int lo = 0, hi = G;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (s_prefix[mid] <= t)
            lo = mid;
        else
            hi = mid;
    }
    const int g = lo;
    const int rows_g = s_off[g + 1] - s_off[g];
    const int mt_g = (rows_g + PBM - 1) / PBM;
    const int local = t - s_prefix[g];
    const int n_tile = local / mt_g;
    const int m_tile = local - n_tile * mt_g;
    PairTile ti;
    ti.g = g;
    ti.row0 = s_off[g] + m_tile * PBM;
    ti.rows_valid = min(PBM, rows_g - m_tile * PBM);
    ti.n0 = n_tile * outn;
    return ti;
}

__device__ __forceinline__ float silu2(float a)
{
    return a / (1.0f + __expf(-a));
}

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc_pair(const __grid_constant__ CUtensorMap tmA,
                         const __grid_constant__ CUtensorMap tmB,
                         const __grid_constant__ CUtensorMap tmB2, PairParams p)
{
    grid_dep_wait();
    constexpr int OUTN = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *stage_base = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    uint64_t *full = bars;
    uint64_t *empty = bars + STAGES;
    uint64_t *acc_full = bars + 2 * STAGES;
    uint64_t *acc_empty = bars + 2 * STAGES + 2;
    uint64_t *drain = bars + 2 * STAGES + 4;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5);
    volatile int *s_abort = reinterpret_cast<volatile int *>(s_tmem + 1);
    int32_t *s_off = reinterpret_cast<int32_t *>(s_tmem + 4);
    int32_t *s_prefix = s_off + (kMaxGroups + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();      // 0: MMA leader, 1: peer
    const bool leader = rank == 0;
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    const int G = p.G;
    const int n_tiles = (p.n_out + OUTN - 1) / OUTN;
    const int KB = (p.K + BK - 1) / BK;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);   // the leader's expect-tx arrive (both halves' bytes)
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 2 * 4 * 32);   // both CTAs' epilogue threads
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (EPI == EPI_SWIGLU)
            tma_prefetch_desc(&tmB2);
    }
    if (warp == 1) {
        tmem_alloc_pair(s_tmem, TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (warp == 2) {
        const int per = (G + 32) / 32;
        for (int i = lane; i <= G; i += 32)
            s_off[i] = p.offsets ? p.offsets[i] : (i == 0 ? 0 : p.rows_single);
        __syncwarp();
        int base = lane * per, sum = 0;
        for (int i = 0; i < per; ++i) {
            const int g = base + i;
            if (g < G) {
                int rows = s_off[g + 1] - s_off[g];
                rows = rows > 0 ? rows : 0;
                sum += ((rows + PBM - 1) / PBM) * n_tiles;
            }
        }
        int incl = sum;
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += v;
        }
        int run = incl - sum;
        for (int i = 0; i < per; ++i) {
            const int g = base + i;
            if (g <= G) {
                s_prefix[g] = run;
                if (g < G) {
                    int rows = s_off[g + 1] - s_off[g];
                    rows = rows > 0 ? rows : 0;
                    run += ((rows + PBM - 1) / PBM) * n_tiles;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();      // the peer's barriers exist before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int total_tiles = s_prefix[G];

    if (warp == 0) {
        // ================= TMA producer (this CTA's halves) =================
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0, last_par = 0, used = 0;
            bool ok = true;
            const CUtensorMap *mapB = (EPI == EPI_SWIGLU && !leader) ? &tmB2 : &tmB;
            for (int t = pair; t < total_tiles && ok; t += npairs) {
                const PairTile ti = pair_tile(t, s_prefix, s_off, G, OUTN);
                const int arow = ti.row0 + static_cast<int>(rank) * HBM;
                const int brow = (ti.g % p.w_blocks) * p.n_out + ti.n0 +
                                 ((EPI == EPI_SWIGLU) ? 0 : static_cast<int>(rank) * 128);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded_cluster(&empty[s], ph ^ 1u, s_abort)) {
                        set_status(p.status, DEV_TIMEOUT_PRODUCER);
                        *s_abort = 1;
                        ok = false;
                        break;
                    }
                    uint8_t *sa = stage_base + s * STAGE_BYTES;
                    if (leader) {
                        mbar_arrive_expect_tx(&full[s], 2 * STAGE_BYTES);
                        tma_load_2d(sa, &tmA, &full[s], kb * BK, arow);
                        tma_load_2d(sa + A_BYTES, mapB, &full[s], kb * BK, brow);
                    } else {
                        const uint32_t lbar = mapa_shared(smem_u32(&full[s]), 0);
                        tma_load_2d_pairbar(sa, &tmA, lbar, kb * BK, arow);
                        tma_load_2d_pairbar(sa + A_BYTES, mapB, lbar, kb * BK, brow);
                    }
                    last_par = (last_par & ~(1u << s)) | (ph << s);
                    used |= 1u << s;
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // the leader's barriers count both halves: once they complete, no
            // copy of either CTA is still in flight
            for (int i = 0; i < STAGES && leader; ++i) {
                if ((used >> i) & 1u) {
                    volatile int never = 0;
                    if (!mbar_wait_bounded_cluster(&full[i], (last_par >> i) & 1u, &never))
                        set_status(p.status, DEV_TIMEOUT_DRAIN);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            // ================= MMA issuer (pair) =================
            constexpr uint32_t idesc = idesc_bf16_f32(PBM, BN);
            int s = 0;
            uint32_t ph = 0;
            int it = 0;
            bool ok = true;
            for (int t = pair; t < total_tiles && ok; t += npairs, ++it) {
                const int a = it & 1;
                const uint32_t aph = (it >> 1) & 1;
                if (!mbar_wait_bounded_cluster(&acc_empty[a], aph ^ 1u, s_abort)) {
                    set_status(p.status, DEV_TIMEOUT_MMA);
                    *s_abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + a * BN;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded_cluster(&full[s], ph, s_abort)) {
                        set_status(p.status, DEV_TIMEOUT_MMA);
                        *s_abort = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(stage_base + s * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        tc_mma_bf16_pair(d_tmem, sdesc_kmajor_sw128(sa + kk * 32),
                                         sdesc_kmajor_sw128(sb + kk * 32), idesc,
                                         (kb > 0 || kk > 0) ? 1u : 0u);
                    tc_commit_pair_mc(&empty[s], 0x3);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (ok)
                    tc_commit_pair_mc(&acc_full[a], 0x3);
            }
        }
    } else {
        // ================= epilogue (warps 2..5, this CTA's 128 rows) =================
        const int q = warp & 3;
        const int r_local = q * 32 + lane;
        const int r_in_tile = static_cast<int>(rank) * HBM + r_local;
        const uint32_t leader_acc_empty[2] = {mapa_shared(smem_u32(&acc_empty[0]), 0),
                                              mapa_shared(smem_u32(&acc_empty[1]), 0)};
        int it = 0;
        for (int t = pair; t < total_tiles; t += npairs, ++it) {
            const PairTile ti = pair_tile(t, s_prefix, s_off, G, OUTN);
            const int a = it & 1;
            const uint32_t aph = (it >> 1) & 1;
            const bool got = mbar_wait_bounded_cluster(&acc_full[a], aph, s_abort);
            if (!__all_sync(0xffffffffu, got)) {
                if (lane == 0) {
                    set_status(p.status, DEV_TIMEOUT_EPILOGUE);
                    *s_abort = 1;
                }
                break;
            }
            tc_fence_after();
            const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * BN;
            const int64_t row = static_cast<int64_t>(ti.row0) + r_in_tile;
            const bool row_ok = r_in_tile < ti.rows_valid && row >= 0 && row < p.rows_cap;
            float scale = 1.0f;
            if (p.row_scale != nullptr && row_ok)
                scale = p.row_scale[row];
#pragma unroll 1
            for (int c = 0; c < OUTN; c += 32) {
                uint32_t v[32];
                float o[32];
                tmem_ld32(tacc + c, v);
                if (EPI == EPI_SWIGLU) {
                    uint32_t u[32];
                    tmem_ld32(tacc + OUTN + c, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        o[i] = silu2(__uint_as_float(v[i]) * scale) * (__uint_as_float(u[i]) * scale);
                } else {
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        const float x = __uint_as_float(v[i]) * scale;
                        o[i] = (EPI == EPI_RELU) ? fmaxf(x, 0.0f) : x;
                    }
                }
                const int col0 = ti.n0 + c;
                if (row_ok) {
                    __nv_bfloat16 *dst =
                        reinterpret_cast<__nv_bfloat16 *>(p.out) + row * p.ld_out + col0;
                    if (col0 + 32 <= p.n_out) {
#pragma unroll
                        for (int i = 0; i < 32; i += 8) {
                            uint4 w;
                            w.x = pack_bf16x2(o[i], o[i + 1]);
                            w.y = pack_bf16x2(o[i + 2], o[i + 3]);
                            w.z = pack_bf16x2(o[i + 4], o[i + 5]);
                            w.w = pack_bf16x2(o[i + 6], o[i + 7]);
                            *reinterpret_cast<uint4 *>(dst + i) = w;
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            if (col0 + i < p.n_out)
                                dst[i] = __float2bfloat16_rn(o[i]);
                    }
                }
            }
            tc_fence_before();
            if (leader)
                mbar_arrive(&acc_empty[a]);
            else
                mbar_arrive_cluster(leader_acc_empty[a]);
        }
    }

    // ---- teardown: MMAs of the pair complete, then the pair releases TMEM
    __syncwarp();
    if (warp == 1 && lane == 0 && leader && *s_abort) {
        tc_commit_pair_mc(drain, 0x1);
        volatile int never = 0;
        if (!mbar_wait_bounded(drain, 0, &never))
            set_status(p.status, DEV_TIMEOUT_DRAIN);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    cluster_sync_all();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
}

typedef CUresult (*PFN_encodeTiled2)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                     const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                     const cuuint32_t *, CUtensorMapInterleave,
                                     CUtensorMapSwizzle, CUtensorMapL2promotion,
                                     CUtensorMapFloatOOBfill);

bool make_map(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int box_rows)
{
    static PFN_encodeTiled2 enc = nullptr;
    if (!enc) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        enc = reinterpret_cast<PFN_encodeTiled2>(ptr);
    }
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int EPI>
cudaError_t launch_pair_impl(const GemmLaunch &L, cudaStream_t stream)
{
    CUtensorMap mA, mB, mB2;
    if (!make_map(&mA, L.A, L.a_rows, L.K, HBM) || !make_map(&mB, L.B, L.b_rows, L.K, 128))
        return cudaErrorInvalidValue;
    if (EPI == EPI_SWIGLU) {
        if (!make_map(&mB2, L.B2, L.b_rows, L.K, 128))
            return cudaErrorInvalidValue;
    } else {
        mB2 = mB;
    }
    static DeviceOnce pair_once;   // per device: function attributes are per device
    int max_pairs = 0;
    cudaError_t e = device_once(pair_once, &max_pairs, [](int *v) {
        cudaError_t err = cudaFuncSetAttribute(grouped_gemm_tc_pair<EPI>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                                               SMEM_BYTES);
        if (err != cudaSuccess)
            return err;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2, 1, 1);
        cfg.blockDim = dim3(kThreads, 1, 1);
        cfg.dynamicSmemBytes = SMEM_BYTES;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        err = cudaOccupancyMaxActiveClusters(&n, grouped_gemm_tc_pair<EPI>, &cfg);
        if (err != cudaSuccess)
            return err;
        if (n <= 0)
            return cudaErrorInvalidConfiguration;
        *v = n;
        return cudaSuccess;
    });
    if (e != cudaSuccess)
        return e;
    PairParams p;
    p.offsets = L.offsets;
    p.rows_single = L.rows_single;
    p.G = L.G;
    p.w_blocks = L.w_blocks > 0 ? L.w_blocks : L.G;
    p.n_out = L.n_out;
    p.K = L.K;
    p.out = L.out;
    p.ld_out = L.ld_out;
    p.row_scale = L.row_scale;
    p.rows_cap = L.out_rows;
    p.status = L.status;
    const int outn = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
    const int64_t n_tiles = (L.n_out + outn - 1) / outn;
    const int64_t m_tiles_max = (L.a_rows + PBM - 1) / PBM + (L.offsets ? L.G : 0);
    int64_t pairs = n_tiles * m_tiles_max;
    if (pairs > max_pairs)
        pairs = max_pairs;
    if (pairs <= 0)
        return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // as launch_k
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, grouped_gemm_tc_pair<EPI>, mA, mB, mB2, p);
    count_launches(1);
    return e;
}

}  // namespace

cudaError_t launch_grouped_gemm_pair(const GemmLaunch &L, cudaStream_t stream)
{
    if (L.G > kMaxGroups || L.G < 1 || L.out_f32 || L.ksplit > 1)
        return cudaErrorInvalidValue;
    switch (L.epi) {
    case EPI_SWIGLU:
        return launch_pair_impl<EPI_SWIGLU>(L, stream);
    case EPI_RELU:
        return launch_pair_impl<EPI_RELU>(L, stream);
    default:
        return launch_pair_impl<EPI_STORE>(L, stream);
    }
}

}  // namespace moe
