// Grouped GEMM on the 5th-generation tensor cores (tcgen05 + TMEM + TMA).
//
// Computes, for every group g (an expert's row segment),
//   D[r, n] = epilogue( sum_k A[r, k] * B[g * n_out + n, k] )
// for rows r in [offsets[g], offsets[g+1]) and n in [0, n_out).  A and B are
// bf16, K-major (the reduction axis contiguous), accumulation is fp32 in TMEM.
//
// This one kernel serves every dense contraction of the MoE layer forward:
//   - the router logits x W_g^T (one group, fp32 output; "moe communication
//     costs", Router design),
//   - the expert up-projection with a fused ReLU or SwiGLU epilogue and the
//     down-projection ("MoE: what it costs to train and serve", Expert
//     parallelism step 2, run locally), and the shared expert.
//
// Design (sm_100a):
//   - persistent CTAs, one per SM, walking a static round-robin tile list;
//     the tile list is derived on the device from the group offsets, so no
//     host synchronisation is needed between dispatch and the GEMM;
//   - tile = 128 rows x BN columns of the MMA (BN <= 256), K step 64 (one
//     128-byte swizzle atom of bf16); for SwiGLU the BN = 256 MMA columns hold
//     128 columns of W1 next to the same 128 columns of W3, so one MMA feeds
//     both halves of the gated activation;
//   - warp 0: TMA producer (one thread); warp 1: TMEM allocator and MMA issuer
//     (one thread); warps 2-5: epilogue, one TMEM lane quarter each;
//   - an S-stage shared-memory ring (full/empty mbarriers) and two TMEM
//     accumulators, so the epilogue of one tile overlaps the MMAs of the next;
//   - tile order inside a group: m fastest, so CTAs running at the same time
//     share the weight tile through L2;
//   - a group that ends a few rows past a multiple of 128 (at most
//     kComboMaxRows) has those rows computed in the same tile as its last
//     128 rows ("combined" tile): one stage carries the weight block, the 128
//     rows and the leftover rows; one MMA covers the 128 rows, a transposed
//     MMA (weights as M, leftover rows as N) the rest, into the second TMEM
//     accumulator.  The weight block is then streamed once for both, where a
//     separate short tile would run at its own pace and read it again;
//   - every mbarrier wait is bounded in time; on expiry the kernel records a
//     status bit, tells the other roles to stop, waits (bounded) for its own
//     copies and MMAs in flight, frees TMEM and returns.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;                      // bf16 elements per 128-byte row
constexpr int A_STAGE_BYTES = BM * BK * 2;  // 16 KB
constexpr int kThreads = 192;
constexpr int kMaxGroups = 1024;

struct GemmParams {
    const int32_t *offsets;  // [G+1] row offsets of the groups in A, or null
    int32_t rows_single;     // rows of the only group when offsets is null
    int32_t G;
    int32_t w_blocks;        // group g uses weight block g % w_blocks
    int32_t n_out;           // output columns per group (= rows of B per group)
    int32_t K;
    void *out;
    int64_t ld_out;          // elements
    const float *row_scale;  // multiply each accumulator row by row_scale[r], or null
    int64_t rows_cap;        // rows allocated in out (and row_scale); rows beyond are never written
    int32_t ksplit;          // >1: split K; split s writes its partial sums at out + s*split_stride
    int64_t split_stride;    // elements
    uint32_t *status;
    // 1: the grouped problem's weights are streamed once (few rows per group):
    // load the weight tiles of groups of one or two m tiles evict-first from
    // L2, and the rows evict-last, since every n tile of a group reads them
    int32_t stream_hint;
};

// Leftover rows a combined tile takes (multiple of 16; 256-column tiles only).
constexpr int kComboMaxRows = 48;

template <int BN, int EPI>
struct Geometry {
    static constexpr int OUTN = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
    static constexpr int B_STAGE_BYTES = BN * BK * 2;
    static constexpr int AB_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
    static constexpr int REM_ROWS = (BN >= 256) ? kComboMaxRows : 0;   // combined tiles
    static constexpr int REM_BYTES = REM_ROWS * BK * 2;
    static constexpr int STAGE_BYTES = AB_BYTES + REM_BYTES;
    static constexpr int STAGES = (BN >= 256) ? 4 : ((BN >= 128) ? 6 : 8);
    static constexpr int TMEM_COLS = (2 * BN <= 32) ? 32 : (2 * BN <= 64 ? 64 : (2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512)));
    // shared memory: [1 KB align slack][stages][barriers + tables]
    static constexpr int AUX_BYTES = 8 * (2 * STAGES + 5) + 16 + 8 * (kMaxGroups + 2);
    static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + AUX_BYTES;
    static_assert(SMEM_BYTES <= 232448, "shared memory per block");
    static_assert(STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
};

// A partial tile of at most kSwapMaxRows rows runs "swapped": the weight rows
// are the MMA's M (128 per MMA) and the tile's rows, rounded up to a multiple
// of 16, its N, so the tensor cores do not pad the rows to 128.
constexpr int kSwapMaxRows = 112;

struct TileInfo {
    int32_t g, row0, rows_valid, n0;
    bool swap;
    int32_t ntok;   // swapped tiles: MMA N (rows_valid rounded up to 16)
    int32_t ks, kb0, kb1;   // K split index and its k-block range
    bool combo;             // combined tile: rows_valid = 128 plus rem_rows more
    int32_t rem_rows, rem_ntok;
    int32_t mtiles;         // m tiles of the tile's group
};

// m tiles of a group of `rows` rows when up to rem_max leftover rows ride
// in the last full tile (rem_max = 0: one tile per 128 rows or part of it).
__host__ __device__ __forceinline__ int m_tiles_of(int rows, int rem_max)
{
    if (rows <= 0)
        return 0;
    if (rows <= BM)
        return 1;
    const int q = rows / BM;
    const int rem = rows - q * BM;
    return (rem == 0 || rem <= rem_max) ? q : q + 1;
}

// Tile `local` of one group of `rows_g` rows starting at row `row_base`, in
// the order (K split, n tile, m tile) with m fastest, so CTAs running side by
// side share the weight tile through L2.
__device__ __forceinline__ TileInfo group_tile(int g, int local, int row_base, int rows_g,
                                               int n_tiles, int outn, int ksplit, int KB,
                                               int rem_max)
{
    const int mt_g = m_tiles_of(rows_g, rem_max);
    const int per_split = mt_g * n_tiles;
    const int ks = local / per_split;
    local -= ks * per_split;
    const int n_tile = local / mt_g;
    const int m_tile = local - n_tile * mt_g;
    TileInfo ti;
    ti.g = g;
    ti.row0 = row_base + m_tile * BM;
    ti.rows_valid = min(BM, rows_g - m_tile * BM);
    ti.n0 = n_tile * outn;
    const int rest = rows_g - (m_tile + 1) * BM;   // rows past this tile (last tile: <= rem_max)
    ti.combo = (m_tile == mt_g - 1) && rest > 0;
    ti.rem_rows = ti.combo ? rest : 0;
    ti.rem_ntok = (ti.rem_rows + 15) & ~15;
    ti.swap = !ti.combo && ti.rows_valid <= kSwapMaxRows;
    ti.ntok = (ti.rows_valid + 15) & ~15;
    ti.ks = ks;
    ti.kb0 = static_cast<int>((static_cast<int64_t>(ks) * KB) / ksplit);
    ti.kb1 = static_cast<int>((static_cast<int64_t>(ks + 1) * KB) / ksplit);
    ti.mtiles = mt_g;
    return ti;
}

// Locate tile t: prefix[g] <= t < prefix[g+1] finds the group.
__device__ __forceinline__ TileInfo tile_info(int t, const int32_t *s_prefix,
                                              const int32_t *s_off, int G, int n_tiles,
                                              int outn, int ksplit, int KB, int rem_max)
{
    int lo = 0, hi = G;  // find largest g with prefix[g] <= t
    while (hi - lo > 1) {
        int mid = (lo + hi) >> 1;
        if (s_prefix[mid] <= t)
            lo = mid;
        else
            hi = mid;
    }
    const int g = lo;
    return group_tile(g, t - s_prefix[g], s_off[g], s_off[g + 1] - s_off[g], n_tiles, outn,
                      ksplit, KB, rem_max);
}

__device__ __forceinline__ float silu_f(float a)
{
    return a / (1.0f + __expf(-a));
}

// 32 consecutive outputs of one row (columns col0 .. col0+31, masked at n_out).
template <bool OUT_F32>
__device__ __forceinline__ void store_row32(void *out, int64_t row_off, int col0, int n_out,
                                            const float (&o)[32])
{
    if (OUT_F32) {
        float *dst = reinterpret_cast<float *>(out) + row_off + col0;
        if (col0 + 32 <= n_out) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
                *reinterpret_cast<float4 *>(dst + i) = make_float4(o[i], o[i + 1], o[i + 2], o[i + 3]);
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)
                if (col0 + i < n_out)
                    dst[i] = o[i];
        }
    } else {
        __nv_bfloat16 *dst = reinterpret_cast<__nv_bfloat16 *>(out) + row_off + col0;
        if (col0 + 32 <= n_out) {
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
                if (col0 + i < n_out)
                    dst[i] = __float2bfloat16_rn(o[i]);
        }
    }
}

template <bool OUT_F32>
__device__ __forceinline__ void store_one(void *out, int64_t off, float v)
{
    if (OUT_F32)
        reinterpret_cast<float *>(out)[off] = v;
    else
        reinterpret_cast<__nv_bfloat16 *>(out)[off] = __float2bfloat16_rn(v);
}

template <int BN, int EPI, bool OUT_F32>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA16,
                    const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB2,
                    GemmParams p)
{
    grid_dep_wait();
    using Geo = Geometry<BN, EPI>;
    constexpr int STAGES = Geo::STAGES;
    constexpr int OUTN = Geo::OUTN;
    constexpr int HALVES = BN / 128;   // swapped tiles: one M=128 MMA per 128 weight rows

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    uint8_t *stage_base = smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * Geo::STAGE_BYTES);
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
    const int G = p.G;
    const int n_tiles = (p.n_out + OUTN - 1) / OUTN;
    const int KB = (p.K + BK - 1) / BK;

    // ---- barriers (warp 0), TMEM (warp 1), group table and tile prefix (warp 2)
    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4 * 32);
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmA16);
        tma_prefetch_desc(&tmB);
        if (EPI == EPI_SWIGLU)
            tma_prefetch_desc(&tmB2);
    }
    if (warp == 1) {
        tmem_alloc(s_tmem, Geo::TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 2) {
        const int per = (G + 32) / 32;  // G+1 entries of offsets
        for (int i = lane; i <= G; i += 32)
            s_off[i] = p.offsets ? p.offsets[i] : (i == 0 ? 0 : p.rows_single);
        __syncwarp();
        int base = lane * per, sum = 0;
        for (int i = 0; i < per; ++i) {
            int g = base + i;
            if (g < G) {
                int rows = s_off[g + 1] - s_off[g];
                rows = rows > 0 ? rows : 0;
                sum += m_tiles_of(rows, Geo::REM_ROWS) * n_tiles * p.ksplit;
            }
        }
        int incl = sum;
        for (int o = 1; o < 32; o <<= 1) {
            int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o)
                incl += v;
        }
        int run = incl - sum;
        for (int i = 0; i < per; ++i) {
            int g = base + i;
            if (g <= G) {
                s_prefix[g] = run;
                if (g < G) {
                    int rows = s_off[g + 1] - s_off[g];
                    rows = rows > 0 ? rows : 0;
                    run += m_tiles_of(rows, Geo::REM_ROWS) * n_tiles * p.ksplit;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *s_tmem;
    const int total_tiles = s_prefix[G];
    auto info = [&](int t) {
        return tile_info(t, s_prefix, s_off, G, n_tiles, OUTN, p.ksplit, KB, Geo::REM_ROWS);
    };

    if (warp == 0) {
        // ================= TMA producer =================
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t last_par = 0;  // bit s: parity of the last load issued to stage s
            uint32_t used = 0;
            bool ok = true;
            const uint64_t pol_first = l2_policy_evict_first();
            const uint64_t pol_last = l2_policy_evict_last();
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                const TileInfo ti = info(t);
                // weights of groups of one or two m tiles are read once or twice in a row
                const bool hint = p.stream_hint != 0 && ti.mtiles <= 2;
                const uint64_t pol_a = hint ? pol_last : 0;
                const CUtensorMap *mA = &tmA, *mA16 = &tmA16, *mB = &tmB, *mB2 = &tmB2;
                const int brow = (ti.g % p.w_blocks) * p.n_out + ti.n0;
                const int a_boxes = ti.ntok / 16;          // swapped tile: 16-row boxes
                const int r_boxes = ti.rem_ntok / 16;      // combined tile: leftover rows
                const uint32_t bytes =
                    ti.swap ? (a_boxes * 16 * BK * 2 + Geo::B_STAGE_BYTES)
                            : (Geo::AB_BYTES + r_boxes * 16 * BK * 2);
                auto load_a = [&](uint8_t *dst, const CUtensorMap *m, int c0, int c1) {
                    if (hint)
                        tma_load_2d_hint(dst, m, &full[s], c0, c1, pol_a);
                    else
                        tma_load_2d(dst, m, &full[s], c0, c1);
                };
                auto load_b = [&](uint8_t *dst, const CUtensorMap *m, int c0, int c1) {
                    if (hint)
                        tma_load_2d_hint(dst, m, &full[s], c0, c1, pol_first);
                    else
                        tma_load_2d(dst, m, &full[s], c0, c1);
                };
                for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
                    if (!mbar_wait_bounded(&empty[s], ph ^ 1u, s_abort)) {
                        set_status(p.status, DEV_TIMEOUT_PRODUCER);
                        *s_abort = 1;
                        ok = false;
                        break;
                    }
                    uint8_t *sa = stage_base + s * Geo::STAGE_BYTES;
                    uint8_t *sb = sa + A_STAGE_BYTES;
                    mbar_arrive_expect_tx(&full[s], bytes);
                    if (ti.swap) {
                        for (int b = 0; b < a_boxes; ++b)
                            load_a(sa + b * 16 * BK * 2, mA16, kb * BK, ti.row0 + 16 * b);
                    } else {
                        load_a(sa, mA, kb * BK, ti.row0);
                        for (int b = 0; b < r_boxes; ++b)   // leftover rows after the B block
                            load_a(sb + Geo::B_STAGE_BYTES + b * 16 * BK * 2, mA16, kb * BK,
                                   ti.row0 + BM + 16 * b);
                    }
                    load_b(sb, mB, kb * BK, brow);
                    if (EPI == EPI_SWIGLU)
                        load_b(sb + (BN / 2) * BK * 2, mB2, kb * BK, brow);
                    last_par = (last_par & ~(1u << s)) | (ph << s);
                    used |= 1u << s;
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            // copies still in flight land before the CTA may exit
            for (int i = 0; i < STAGES; ++i) {
                if ((used >> i) & 1u) {
                    volatile int never = 0;
                    if (!mbar_wait_bounded(&full[i], (last_par >> i) & 1u, &never))
                        set_status(p.status, DEV_TIMEOUT_DRAIN);
                }
            }
        }
    } else if (warp == 1) {
        // ================= MMA issuer =================
        if (lane == 0) {
            constexpr uint32_t idesc_n = idesc_bf16_f32(BM, BN);
            int s = 0;
            uint32_t ph = 0;
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                const TileInfo ti = info(t);
                const uint32_t idesc_s = idesc_bf16_f32(128, ti.ntok);
                const uint32_t idesc_r = idesc_bf16_f32(128, ti.rem_ntok > 0 ? ti.rem_ntok : 16);
                // accumulator(s): a combined tile takes the next two
                const int a = it & 1;
                const uint32_t aph = (it >> 1) & 1;
                const int a2 = (it + 1) & 1;
                const uint32_t aph2 = ((it + 1) >> 1) & 1;
                if (!mbar_wait_bounded(&acc_empty[a], aph ^ 1u, s_abort) ||
                    (ti.combo && !mbar_wait_bounded(&acc_empty[a2], aph2 ^ 1u, s_abort))) {
                    set_status(p.status, DEV_TIMEOUT_MMA);
                    *s_abort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + a * BN;
                const uint32_t d_rem = tmem_base + a2 * BN;
                for (int kb = ti.kb0; kb < ti.kb1; ++kb) {
                    if (!mbar_wait_bounded(&full[s], ph, s_abort)) {
                        set_status(p.status, DEV_TIMEOUT_MMA);
                        *s_abort = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(stage_base + s * Geo::STAGE_BYTES);
                    const uint32_t sb = sa + A_STAGE_BYTES;
                    const uint32_t sr = sb + Geo::B_STAGE_BYTES;
                    if (!ti.swap) {
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
                            tc_mma_bf16(d_tmem, sdesc_kmajor_sw128(sa + kk * 32),
                                        sdesc_kmajor_sw128(sb + kk * 32), idesc_n,
                                        (kb > ti.kb0 || kk > 0) ? 1u : 0u);
                        if (ti.combo) {
                            // leftover rows, transposed, into the second accumulator
#pragma unroll
                            for (int kk = 0; kk < BK / 16; ++kk)
#pragma unroll
                                for (int h = 0; h < HALVES; ++h)
                                    tc_mma_bf16(d_rem + h * 128,
                                                sdesc_kmajor_sw128(sb + h * 128 * BK * 2 + kk * 32),
                                                sdesc_kmajor_sw128(sr + kk * 32), idesc_r,
                                                (kb > ti.kb0 || kk > 0) ? 1u : 0u);
                        }
                    } else {
                        // D^T: weight rows are the MMA's M, the tile's tokens its N
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk)
#pragma unroll
                            for (int h = 0; h < HALVES; ++h)
                                tc_mma_bf16(d_tmem + h * 128,
                                            sdesc_kmajor_sw128(sb + h * 128 * BK * 2 + kk * 32),
                                            sdesc_kmajor_sw128(sa + kk * 32), idesc_s,
                                            (kb > ti.kb0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(&empty[s]);
                    if (++s == STAGES) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (ok) {
                    tc_commit(&acc_full[a]);
                    if (ti.combo)
                        tc_commit(&acc_full[a2]);
                }
                it += ti.combo ? 2 : 1;
            }
        }
    } else {
        // ================= epilogue (warps 2..5) =================
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        const int r_in_tile = q * 32 + lane;
        // one accumulator's worth: a plain or transposed tile (or part of a
        // combined one) from accumulator it & 1; false when its wait failed
        auto part = [&](const TileInfo &ti, int it) -> bool {
            const int a = it & 1;
            const uint32_t aph = (it >> 1) & 1;
            const bool got = mbar_wait_bounded(&acc_full[a], aph, s_abort);
            if (!__all_sync(0xffffffffu, got)) {   // tcgen05.ld below needs the whole warp
                if (lane == 0) {
                    set_status(p.status, DEV_TIMEOUT_EPILOGUE);
                    *s_abort = 1;
                }
                return false;
            }
            tc_fence_after();
            const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + a * BN;
            void *out = p.out;
            const int64_t ld_out = p.ld_out;
            const int n_out = p.n_out;
            const float *row_scale = p.row_scale;
            const int64_t rows_cap = p.rows_cap;
            const int64_t split_off = ti.ks * p.split_stride;
            if (!ti.swap) {
                // lane = output row, columns = output features
                const int64_t row = static_cast<int64_t>(ti.row0) + r_in_tile;
                const bool row_ok = r_in_tile < ti.rows_valid && row >= 0 && row < rows_cap;
                float scale = 1.0f;
                if (row_scale != nullptr && row_ok)
                    scale = row_scale[row];
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
                            o[i] = silu_f(__uint_as_float(v[i]) * scale) *
                                   (__uint_as_float(u[i]) * scale);
                    } else {
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            float x = __uint_as_float(v[i]) * scale;
                            o[i] = (EPI == EPI_RELU) ? fmaxf(x, 0.0f) : x;
                        }
                    }
                    if (row_ok)
                        store_row32<OUT_F32>(out, split_off + row * ld_out,
                                             ti.n0 + c, n_out, o);
                }
            } else {
                // swapped tile: lane = output feature, columns = tokens
#pragma unroll 1
                for (int c = 0; c < ti.ntok; c += 16) {
                    float sc[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int64_t row = static_cast<int64_t>(ti.row0) + c + i;
                        sc[i] = (row_scale != nullptr && c + i < ti.rows_valid && row < rows_cap)
                                    ? row_scale[row] : 1.0f;
                    }
                    if (EPI == EPI_SWIGLU) {
                        uint32_t v[16], u[16];
                        tmem_ld16(tacc + c, v);
                        tmem_ld16(tacc + 128 + c, u);
                        tmem_wait_ld();
                        const int col = ti.n0 + r_in_tile;
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int64_t row = static_cast<int64_t>(ti.row0) + c + i;
                            const float o = silu_f(__uint_as_float(v[i]) * sc[i]) *
                                            (__uint_as_float(u[i]) * sc[i]);
                            if (c + i < ti.rows_valid && row < rows_cap && col < n_out)
                                store_one<OUT_F32>(out, split_off + row * ld_out + col, o);
                        }
                    } else {
#pragma unroll
                        for (int h = 0; h < HALVES; ++h) {
                            uint32_t v[16];
                            tmem_ld16(tacc + h * 128 + c, v);
                            tmem_wait_ld();
                            const int col = ti.n0 + h * 128 + r_in_tile;
#pragma unroll
                            for (int i = 0; i < 16; ++i) {
                                const int64_t row = static_cast<int64_t>(ti.row0) + c + i;
                                float x = __uint_as_float(v[i]) * sc[i];
                                if (EPI == EPI_RELU)
                                    x = fmaxf(x, 0.0f);
                                if (c + i < ti.rows_valid && row < rows_cap && col < n_out)
                                    store_one<OUT_F32>(out, split_off + row * ld_out + col, x);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&acc_empty[a]);
            return true;
        };
        int it = 0;
        for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
            const TileInfo ti = info(t);
            if (!part(ti, it))
                break;
            if (ti.combo) {
                // the leftover rows of a combined tile, transposed, in the next accumulator
                TileInfo tr = ti;
                tr.row0 = ti.row0 + BM;
                tr.rows_valid = ti.rem_rows;
                tr.ntok = ti.rem_ntok;
                tr.swap = true;
                tr.combo = false;
                if (!part(tr, it + 1))
                    break;
            }
            it += ti.combo ? 2 : 1;
        }
    }

    // ---- teardown: MMAs complete, then TMEM is released by its owner warp.
    // On the normal path the epilogue has already seen the last accumulator
    // commit (which covers every MMA issued before it).  After an abort, one
    // more commit on a fresh barrier tells us when the MMAs in flight are done.
    __syncwarp();
    if (warp == 1 && lane == 0 && *s_abort) {
        tc_commit(drain);
        volatile int never = 0;
        if (!mbar_wait_bounded(drain, 0, &never))
            set_status(p.status, DEV_TIMEOUT_DRAIN);
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        tmem_dealloc(tmem_base, Geo::TMEM_COLS);
}

// ------------------------------------------------------------------ host
typedef CUresult (*PFN_encodeTiled)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                    const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                    const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

PFN_encodeTiled get_encode()
{
    static PFN_encodeTiled fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_encodeTiled>(ptr);
    }
    return fn;
}

// 2-D bf16 tensor map over a [rows, cols] row-major matrix (cols contiguous),
// box = box_rows x 64 columns, 128-byte swizzle, zero fill out of bounds.
bool make_map_bf16(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int box_rows)
{
    PFN_encodeTiled enc = get_encode();
    if (!enc)
        return false;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims,
                     strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// SMs of the current device.
int sm_count()
{
    static DeviceOnce once;
    int n = 0;
    if (device_once(once, &n, [](int *v) {
            int dev = 0;
            cudaError_t e = cudaGetDevice(&dev);
            if (e == cudaSuccess)
                e = cudaDeviceGetAttribute(v, cudaDevAttrMultiProcessorCount, dev);
            return e;
        }) != cudaSuccess || n <= 0)
        n = 148;
    return n;
}

template <int BN, int EPI, bool OUT_F32>
cudaError_t launch_impl(const GemmLaunch &L, cudaStream_t stream)
{
    using Geo = Geometry<BN, EPI>;
    CUtensorMap mA, mA16, mB, mB2;
    const int b_box = (EPI == EPI_SWIGLU) ? BN / 2 : BN;
    if (!make_map_bf16(&mA, L.A, L.a_rows, L.K, BM) ||
        !make_map_bf16(&mA16, L.A, L.a_rows, L.K, 16) ||
        !make_map_bf16(&mB, L.B, L.b_rows, L.K, b_box))
        return cudaErrorInvalidValue;
    if (EPI == EPI_SWIGLU) {
        if (!make_map_bf16(&mB2, L.B2, L.b_rows, L.K, b_box))
            return cudaErrorInvalidValue;
    } else {
        mB2 = mB;
    }
    static DeviceOnce attr_once;   // per device: function attributes are per device
    cudaError_t e = device_once(attr_once, nullptr, [](int *) {
        return cudaFuncSetAttribute(grouped_gemm_tc<BN, EPI, OUT_F32>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, Geo::SMEM_BYTES);
    });
    if (e != cudaSuccess)
        return e;
    GemmParams p;
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
    p.ksplit = L.ksplit > 1 ? L.ksplit : 1;
    p.split_stride = L.split_stride;
    p.status = L.status;
    p.stream_hint = L.stream_hint;
    const int outn = Geo::OUTN;
    const int64_t n_tiles = (L.n_out + outn - 1) / outn;
    const int64_t m_tiles_max = (L.a_rows + BM - 1) / BM + (L.offsets ? L.G : 0);
    int64_t tiles_max = n_tiles * m_tiles_max * p.ksplit;
    int grid = static_cast<int>(tiles_max < sm_count() ? tiles_max : sm_count());
    if (grid <= 0)
        return cudaSuccess;
    launch_k(grouped_gemm_tc<BN, EPI, OUT_F32>, grid, kThreads, Geo::SMEM_BYTES, stream, mA, mA16,
             mB, mB2, p);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace

int router_ksplit(int64_t T, int32_t N, int32_t d)
{
    const int64_t m_tiles = (T + BM - 1) / BM;
    const int64_t KB = (d + BK - 1) / BK;
    (void)N;  // one n tile (N <= 256)
    // as many slices as keep the tiles within one wave of the SMs
    int64_t ks = sm_count() / m_tiles;
    const int64_t cap = router_ksplit_cap(T, N);
    if (ks > cap)
        ks = cap;
    if (ks > KB)
        ks = KB;
    return ks < 1 ? 1 : static_cast<int>(ks);
}

cudaError_t launch_grouped_gemm(const GemmLaunch &L, cudaStream_t stream)
{
    if (L.G > kMaxGroups || L.G < 1)
        return cudaErrorInvalidValue;
    switch (L.epi) {
    case EPI_SWIGLU:
        return launch_impl<256, EPI_SWIGLU, false>(L, stream);
    case EPI_RELU:
        return launch_impl<256, EPI_RELU, false>(L, stream);
    case EPI_STORE:
    default:
        if (L.out_f32) {
            if (L.n_out <= 128)
                return launch_impl<128, EPI_STORE, true>(L, stream);
            return launch_impl<256, EPI_STORE, true>(L, stream);
        }
        return launch_impl<256, EPI_STORE, false>(L, stream);
    }
}

}  // namespace moe
