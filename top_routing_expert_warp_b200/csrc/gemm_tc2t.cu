// Grouped GEMM on CTA pairs with the weights as the MMA's M ("transposed"
// pair tiles), for the HBM-bound expert projections: groups (experts) of few
// rows whose weights are streamed once per launch.
//
// Same contract as gemm_tc.cu (rows of group g times B[g * n_out + n, :]^T,
// bf16 K-major operands, fp32 accumulation, ReLU / SwiGLU / plain epilogue,
// an optional per-row scale), computed as D^T: a tile is up to 160 rows of
// one group (the MMA's N, split 80 + 80 between the two CTAs of a cluster)
// against 512 weight rows (two MMAs of M = 256 per K step, 128 weight rows of
// each in each CTA).  Each CTA therefore stages 32 KB of weights and at most
// 10 KB of rows per K step: five stages fit in shared memory, where the
// one-CTA kernel holds four stages of 32 KB weights + 16 KB rows (+ leftover
// rows).  On these layers the copy pipeline, not HBM, sets the pace (a stage
// waits for all of its row segments, each ~1-3 us away), so more weight
// bytes in flight per SM and fewer row segments per weight segment are the
// levers ("MoE: what it costs to train and serve", Expert parallelism step 2,
// run locally, for the expert FFNs).
//
// For SwiGLU the two MMAs of a K step are W1 and W3 of the same 256 features
// (128 in each CTA), so a TMEM lane holds both halves of its feature's gate:
// no exchange between the CTAs.  Otherwise the two MMAs are 512 consecutive
// weight rows.  A tile of at most 128 rows fits both MMAs' accumulators in
// one 256-column TMEM slot (two slots: the epilogue of one tile overlaps the
// MMAs of the next); a tile of 129-160 rows takes both slots.  A group of
// more than 160 rows is cut into equal chunks of at most 160 rows, each its
// own tile; chunks of a group are adjacent in the tile order, so pairs
// running side by side share the weight tiles through L2.
//
// Roles as in gemm_tc2.cu: warp 0 lane 0 of each CTA loads that CTA's weight
// blocks and row half (the second CTA's copies count their bytes on the
// first CTA's stage barrier); warp 1 allocates TMEM collectively and, in the
// first CTA, issues the pair MMAs and the multicast commits; warps 2-9 of
// each CTA drain that CTA's 128 TMEM lanes (its weight rows) for every row
// of the tile, two warps per lane quarter taking alternate 16-row steps (a
// tile of 129-160 rows holds both accumulator slots until its epilogue is
// done, so that epilogue is on the MMAs' path).  No TMA multicast.  Every
// wait is bounded; on expiry the kernel records a status bit, tells the
// other roles to stop, waits (bounded) for its copies and MMAs in flight and
// releases TMEM.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int BK = 64;                        // bf16 elements per 128-byte row
constexpr int WR = 128;                       // weight rows per CTA per MMA
constexpr int W_BLOCK = WR * BK * 2;          // 16 KB
constexpr int W_BYTES = 2 * W_BLOCK;          // two MMAs per K step
constexpr int TMAX = 160;                     // rows per tile (both CTAs)
constexpr int T_BYTES = (TMAX / 2) * BK * 2;  // 10 KB: this CTA's half of the rows
constexpr int STAGE_BYTES = W_BYTES + T_BYTES;
constexpr int STAGES = 5;
constexpr int kEpiWarps = 8;                  // two per TMEM lane quarter
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kMaxGroups = 1024;
constexpr int TMEM_COLS = 512;
constexpr int SLOT = 256;                     // columns of one accumulator slot
constexpr int AUX_BYTES = 8 * (2 * STAGES + 6) + 16 + 8 * (kMaxGroups + 2);
constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + AUX_BYTES;
static_assert(SMEM_BYTES <= 232448, "shared memory per block");
static_assert(STAGE_BYTES % 1024 == 0 && W_BLOCK % 1024 == 0,
              "stages and blocks keep the 1024-byte swizzle alignment");

struct PairTParams {
    const int32_t *offsets;  // [G+1]
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

struct TTile {
    int32_t g, row0, rows, ntok, f0;
    bool big;                // 129-160 rows: both accumulator slots
};

// Features per tile: 256 for SwiGLU (W1 and W3 of the same features), else
// the 512 weight rows of the two MMAs.
template <int EPI>
__host__ __device__ constexpr int feat_of() { return EPI == EPI_SWIGLU ? 2 * WR : 4 * WR; }

// Tiles (row chunks) of a group: one of up to TMAX rows; a longer group in
// chunks of at most 128 rows, which keep the TMEM double buffer (a chunk of
// 129-160 rows takes both accumulator slots and stalls the next tile's MMAs
// for its epilogue).
__host__ __device__ __forceinline__ int chunks_of(int rows)
{
    return rows <= 0 ? 0 : (rows <= TMAX ? 1 : (rows + 127) / 128);
}

// Tile t: group by binary search over the tile prefix, then (n tile, chunk)
// with the chunk fastest.
__device__ __forceinline__ TTile ttile(int t, const int32_t *s_prefix, const int32_t *s_off,
                                       int G, int feat)
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
    const int nc = chunks_of(rows_g);
    const int local = t - s_prefix[g];
    const int n_tile = local / nc;
    const int c = local - n_tile * nc;
    const int64_t r_lo = static_cast<int64_t>(c) * rows_g / nc;
    const int64_t r_hi = static_cast<int64_t>(c + 1) * rows_g / nc;
    TTile ti;
    ti.g = g;
    ti.row0 = s_off[g] + static_cast<int>(r_lo);
    ti.rows = static_cast<int>(r_hi - r_lo);
    ti.ntok = (ti.rows + 31) & ~31;   // each CTA's half a multiple of 16 rows
    ti.f0 = n_tile * feat;
    ti.big = ti.ntok > 128;
    return ti;
}

__device__ __forceinline__ float silu_t(float a)
{
    return a / (1.0f + __expf(-a));
}

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc_pairt(const __grid_constant__ CUtensorMap tmW,
                          const __grid_constant__ CUtensorMap tmW2,
                          const __grid_constant__ CUtensorMap tmT, PairTParams p)
{
    grid_dep_wait();
    constexpr int FEAT = feat_of<EPI>();
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *stage_base = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    uint64_t *full = bars;                    // first CTA: both CTAs' bytes of a stage
    uint64_t *empty = bars + STAGES;          // both CTAs: the pair's MMAs read the stage
    uint64_t *acc_full = bars + 2 * STAGES;
    uint64_t *acc_empty = bars + 2 * STAGES + 2;   // first CTA: both CTAs' epilogues
    uint64_t *drain = bars + 2 * STAGES + 4;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 6);
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
    const int n_tiles = (p.n_out + FEAT - 1) / FEAT;
    const int KB = (p.K + BK - 1) / BK;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);   // the leader's expect-tx arrive (both halves' bytes)
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 2 * kEpiWarps * 32);   // both CTAs' epilogue threads
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmT);
        if (EPI == EPI_SWIGLU)
            tma_prefetch_desc(&tmW2);
    }
    if (warp == 1) {
        tmem_alloc_pair(s_tmem, TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (warp == 2) {
        const int per = (G + 32) / 32;
        for (int i = lane; i <= G; i += 32)
            s_off[i] = p.offsets[i];
        __syncwarp();
        int base = lane * per, sum = 0;
        for (int i = 0; i < per; ++i) {
            const int g = base + i;
            if (g < G)
                sum += chunks_of(s_off[g + 1] - s_off[g]) * n_tiles;
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
                if (g < G)
                    run += chunks_of(s_off[g + 1] - s_off[g]) * n_tiles;
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
        // ================= TMA producer (this CTA's weight blocks and row half) =================
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0, last_par = 0, used = 0;
            bool ok = true;
            const CUtensorMap *mapW1 = (EPI == EPI_SWIGLU) ? &tmW2 : &tmW;   // second MMA's block
            for (int t = pair; t < total_tiles && ok; t += npairs) {
                const TTile ti = ttile(t, s_prefix, s_off, G, FEAT);
                const int half = ti.ntok / 2;
                const int trow = ti.row0 + static_cast<int>(rank) * half;
                const int wbase = (ti.g % p.w_blocks) * p.n_out + ti.f0 + static_cast<int>(rank) * WR;
                // SwiGLU: W1 and W3 rows of the same features; else the two
                // 256-row halves of the tile's 512 weight rows
                const int wrow0 = wbase;
                const int wrow1 = (EPI == EPI_SWIGLU) ? wbase : wbase + 2 * WR;
                const int boxes = half / 16;
                const uint32_t bytes = 2u * static_cast<uint32_t>(W_BYTES + boxes * 16 * BK * 2);
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded_cluster(&empty[s], ph ^ 1u, s_abort)) {
                        set_status(p.status, DEV_TIMEOUT_PRODUCER);
                        *s_abort = 1;
                        ok = false;
                        break;
                    }
                    uint8_t *sw = stage_base + s * STAGE_BYTES;
                    uint8_t *st = sw + W_BYTES;
                    // this CTA's copy of box (c0, c1) of map m into dst, counted
                    // on the leader's stage barrier (no L2 policy: evict-first
                    // weights and evict-last rows made this kernel 25 % slower)
                    const uint32_t lbar = mapa_shared(smem_u32(&full[s]), 0);
                    auto load = [&](uint8_t *dst, const CUtensorMap *m, int c0, int c1) {
                        if (leader)
                            tma_load_2d(dst, m, &full[s], c0, c1);
                        else
                            tma_load_2d_pairbar(dst, m, lbar, c0, c1);
                    };
                    if (leader)
                        mbar_arrive_expect_tx(&full[s], bytes);
                    load(sw, &tmW, kb * BK, wrow0);
                    load(sw + W_BLOCK, mapW1, kb * BK, wrow1);
                    for (int b = 0; b < boxes; ++b)
                        load(st + b * 16 * BK * 2, &tmT, kb * BK, trow + 16 * b);
                    last_par = (last_par & ~(1u << s)) | (ph << s);
                    used |= 1u << s;
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // the leader's barriers count both CTAs' bytes: once they complete,
            // no copy of either CTA is still in flight
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
            int s = 0;
            uint32_t ph = 0;
            int it = 0;
            bool ok = true;
            for (int t = pair; t < total_tiles && ok; t += npairs) {
                const TTile ti = ttile(t, s_prefix, s_off, G, FEAT);
                const int a = it & 1;
                const uint32_t aph = (it >> 1) & 1;
                const int a2 = (it + 1) & 1;
                const uint32_t aph2 = ((it + 1) >> 1) & 1;
                if (!mbar_wait_bounded_cluster(&acc_empty[a], aph ^ 1u, s_abort) ||
                    (ti.big && !mbar_wait_bounded_cluster(&acc_empty[a2], aph2 ^ 1u, s_abort))) {
                    set_status(p.status, DEV_TIMEOUT_MMA);
                    *s_abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t idesc = idesc_bf16_f32(2 * WR, ti.ntok);
                // first MMA's accumulator at the slot's start; the second's
                // after it, or in the other slot for a tile of > 128 rows
                const uint32_t d0 = tmem_base + a * SLOT;
                const uint32_t d1 = ti.big ? tmem_base + a2 * SLOT : d0 + ti.ntok;
                for (int kb = 0; kb < KB; ++kb) {
                    if (!mbar_wait_bounded_cluster(&full[s], ph, s_abort)) {
                        set_status(p.status, DEV_TIMEOUT_MMA);
                        *s_abort = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sw = smem_u32(stage_base + s * STAGE_BYTES);
                    const uint32_t st = sw + W_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
                        const uint64_t bdesc = sdesc_kmajor_sw128(st + kk * 32);
                        tc_mma_bf16_pair(d0, sdesc_kmajor_sw128(sw + kk * 32), bdesc, idesc, acc);
                        tc_mma_bf16_pair(d1, sdesc_kmajor_sw128(sw + W_BLOCK + kk * 32), bdesc,
                                         idesc, acc);
                    }
                    tc_commit_pair_mc(&empty[s], 0x3);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (ok) {
                    tc_commit_pair_mc(&acc_full[a], 0x3);
                    if (ti.big)
                        tc_commit_pair_mc(&acc_full[a2], 0x3);
                }
                it += ti.big ? 2 : 1;
            }
        }
    } else {
        // ================= epilogue (warps 2..9: this CTA's 128 weight rows) =================
        const int q = warp & 3;   // TMEM lane quarter: weight rows 32q .. 32q+31 of the block
        const int half = (warp - 2) >> 2;   // the two warps of a quarter take alternate 16-row steps
        const uint32_t leader_acc_empty[2] = {mapa_shared(smem_u32(&acc_empty[0]), 0),
                                              mapa_shared(smem_u32(&acc_empty[1]), 0)};
        const float *row_scale = p.row_scale;
        __nv_bfloat16 *out = reinterpret_cast<__nv_bfloat16 *>(p.out);
        int it = 0;
        for (int t = pair; t < total_tiles; t += npairs) {
            const TTile ti = ttile(t, s_prefix, s_off, G, FEAT);
            const int a = it & 1;
            const uint32_t aph = (it >> 1) & 1;
            const int a2 = (it + 1) & 1;
            const uint32_t aph2 = ((it + 1) >> 1) & 1;
            bool got = mbar_wait_bounded_cluster(&acc_full[a], aph, s_abort);
            if (ti.big)
                got = got && mbar_wait_bounded_cluster(&acc_full[a2], aph2, s_abort);
            if (!__all_sync(0xffffffffu, got)) {   // tcgen05.ld below needs the whole warp
                if (lane == 0) {
                    set_status(p.status, DEV_TIMEOUT_EPILOGUE);
                    *s_abort = 1;
                }
                break;
            }
            tc_fence_after();
            const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
            const uint32_t t0 = tmem_base + lane_off + a * SLOT;
            const uint32_t t1 = ti.big ? tmem_base + lane_off + a2 * SLOT : t0 + ti.ntok;
            // feature (output column) of this lane in the first / second MMA
            const int f_a = ti.f0 + static_cast<int>(rank) * WR + q * 32 + lane;
            const int f_b = (EPI == EPI_SWIGLU) ? f_a : f_a + 2 * WR;
            // release of accumulator slot b: an arrive on the first CTA's barrier
            auto release = [&](int b) {
                tc_fence_before();
                if (leader)
                    mbar_arrive(&acc_empty[b]);
                else
                    mbar_arrive_cluster(leader_acc_empty[b]);
            };
            // 16 rows (row0 + c0 ..) of feature f, lane = feature: the warp
            // writes 64 contiguous bytes of each output row
            auto put16 = [&](int c0, int f, const float (&o)[16]) {
                if (f >= p.n_out)
                    return;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int64_t row = static_cast<int64_t>(ti.row0) + c0 + i;
                    if (c0 + i < ti.rows && row < p.rows_cap)
                        out[row * p.ld_out + f] = __float2bfloat16_rn(o[i]);
                }
            };
            // the scales of rows row0 + c0 .. + 15 (1 past the tile's rows)
            auto scales = [&](int c0, float (&sc)[16]) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int64_t row = static_cast<int64_t>(ti.row0) + c0 + i;
                    sc[i] = (row_scale != nullptr && c0 + i < ti.rows && row < p.rows_cap)
                                ? row_scale[row] : 1.0f;
                }
            };
            if (EPI == EPI_SWIGLU) {
                // a lane's W1 and W3 values of one feature, 16 rows at a time
#pragma unroll 1
                for (int c0 = 16 * half; c0 < ti.ntok; c0 += 32) {
                    float sc[16], o[16];
                    scales(c0, sc);
                    uint32_t v[16], u[16];
                    tmem_ld16(t0 + c0, v);
                    tmem_ld16(t1 + c0, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        o[i] = silu_t(__uint_as_float(v[i]) * sc[i]) * (__uint_as_float(u[i]) * sc[i]);
                    put16(c0, f_a, o);
                }
                release(a);
                if (ti.big)
                    release(a2);
            } else {
                // the two MMAs' features one after the other; a tile of > 128
                // rows frees its first slot before draining the second
#pragma unroll 1
                for (int j = 0; j < 2; ++j) {
                    const uint32_t tb = j == 0 ? t0 : t1;
#pragma unroll 1
                    for (int c0 = 16 * half; c0 < ti.ntok; c0 += 32) {
                        float sc[16], o[16];
                        scales(c0, sc);
                        uint32_t v[16];
                        tmem_ld16(tb + c0, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const float x = __uint_as_float(v[i]) * sc[i];
                            o[i] = (EPI == EPI_RELU) ? fmaxf(x, 0.0f) : x;
                        }
                        put16(c0, j == 0 ? f_a : f_b, o);
                    }
                    if (j == 0 && ti.big)
                        release(a);
                }
                release(ti.big ? a2 : a);
            }
            it += ti.big ? 2 : 1;
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

typedef CUresult (*PFN_encodeTiledT)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                     const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                     const cuuint32_t *, CUtensorMapInterleave,
                                     CUtensorMapSwizzle, CUtensorMapL2promotion,
                                     CUtensorMapFloatOOBfill);

// 2-D bf16 map over [rows, cols] (cols contiguous), box box_rows x 64, 128-byte swizzle.
bool make_map_t(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int box_rows)
{
    static PFN_encodeTiledT enc = nullptr;
    if (!enc) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return false;
        enc = reinterpret_cast<PFN_encodeTiledT>(ptr);
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
cudaError_t launch_pairt_impl(const GemmLaunch &L, cudaStream_t stream)
{
    CUtensorMap mW, mW2, mT;
    if (!make_map_t(&mW, L.B, L.b_rows, L.K, WR) || !make_map_t(&mT, L.A, L.a_rows, L.K, 16))
        return cudaErrorInvalidValue;
    if (EPI == EPI_SWIGLU) {
        if (!make_map_t(&mW2, L.B2, L.b_rows, L.K, WR))
            return cudaErrorInvalidValue;
    } else {
        mW2 = mW;
    }
    static DeviceOnce pair_once;   // per device: function attributes are per device
    int max_pairs = 0;
    cudaError_t e = device_once(pair_once, &max_pairs, [](int *v) {
        cudaError_t err = cudaFuncSetAttribute(grouped_gemm_tc_pairt<EPI>,
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
        err = cudaOccupancyMaxActiveClusters(&n, grouped_gemm_tc_pairt<EPI>, &cfg);
        if (err != cudaSuccess)
            return err;
        if (n <= 0)
            return cudaErrorInvalidConfiguration;
        *v = n;
        return cudaSuccess;
    });
    if (e != cudaSuccess)
        return e;
    PairTParams p;
    p.offsets = L.offsets;
    p.G = L.G;
    p.w_blocks = L.w_blocks > 0 ? L.w_blocks : L.G;
    p.n_out = L.n_out;
    p.K = L.K;
    p.out = L.out;
    p.ld_out = L.ld_out;
    p.row_scale = L.row_scale;
    p.rows_cap = L.out_rows;
    p.status = L.status;
    const int64_t n_tiles = (L.n_out + feat_of<EPI>() - 1) / feat_of<EPI>();
    const int64_t chunks_max = L.a_rows / TMAX + L.G;   // >= sum over groups of their chunks
    int64_t pairs = n_tiles * chunks_max;
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
    e = cudaLaunchKernelEx(&cfg, grouped_gemm_tc_pairt<EPI>, mW, mW2, mT, p);
    count_launches(1);
    return e;
}

}  // namespace

cudaError_t launch_grouped_gemm_pairt(const GemmLaunch &L, cudaStream_t stream)
{
    if (L.G > kMaxGroups || L.G < 1 || L.out_f32 || L.ksplit > 1 || L.offsets == nullptr)
        return cudaErrorInvalidValue;
    switch (L.epi) {
    case EPI_SWIGLU:
        return launch_pairt_impl<EPI_SWIGLU>(L, stream);
    case EPI_RELU:
        return launch_pairt_impl<EPI_RELU>(L, stream);
    default:
        return launch_pairt_impl<EPI_STORE>(L, stream);
    }
}

}  // namespace moe
