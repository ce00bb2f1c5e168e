// igemm_tcgen05.cu -- int8 x int8 -> int32 GEMM on the 5th-generation tensor
// cores with the dequantisation fused into the epilogue.
//
//   acc[m][n] = sum_k qa[m][k] * qb[n][k]                   (exact, int32)
//   y[m][n]   = bf16(acc * s_a[m] * (s_b[n] * alpha) + bias[n])   [optional GELU]
//
// The GEMM is the pages' "INT8 MMA" (MiniMax-H3-Rung-Omega README, "Technical
// Architecture Overview", item 2); the scales are the per-token activation
// scale and the "per-output F32 scales" of the weights ("MiniMax H3 - pruned
// INT8 ConvRot - input-major", section "Input-major checkpoint"); the output
// is bf16 because "the residual stream reaches 2.4e5, beyond fp16's range"
// ("HyperFlow H3 Flash MLX", section "How to run").
//
// Two kernels share the roles and the epilogue; both are persistent,
// warp-specialised, one CTA per SM:
//   warp 0      TMA producer into a shared-memory ring (mbarrier per stage,
//               128-byte swizzle)
//   warp 1      MMA issuer: one thread issues tcgen05.mma kind::i8 (K = 32
//               per instruction) into a TMEM accumulator; tcgen05.commit
//               frees each stage and, per tile, signals the epilogue
//   warps 2..    epilogue (4 warps, or 8 for CTA pairs: two per TMEM lane
//               quadrant): tcgen05.ld 32 columns at a time, scale + bias
//               (+ GELU), bf16, swizzled shared staging, TMA store
// Two 256-column accumulators (all 512 TMEM columns) let the epilogue of one
// tile overlap the main loop of the next.  Tiles run n-fastest so an A panel
// is read from HBM once and reused from L2 across N.
//
//   igemm_kernel       one CTA per 128 x 256 tile (M = 128, N = 256 MMAs),
//                      A 16 KB + B 32 KB per stage, 4 stages.
//   igemm_pair_kernel  a cluster of two CTAs per 256 x 256 tile
//                      (cta_group::2, M = 256, N = 256 MMAs issued by the
//                      pair's leader): each CTA stages 128 rows of A and half
//                      of B's 256 rows (32 KB per stage, 6 stages), so per
//                      output element the pair moves a third less operand data
//                      through shared memory and L2 than the single-CTA tile.
// No load uses cluster multicast (the pair's commits do, which is allowed).
#include <cuda_bf16.h>

#include "gemm_core.cuh"
#include "kernels.h"
#include "ptx.cuh"

#ifndef CONVROT_GEMM_PAIR
#define CONVROT_GEMM_PAIR 1  // 1: CTA-pair tiles, 0: single-CTA tiles
#endif

namespace convrot {

namespace {

using namespace gcore;

constexpr int kEpiWarps1 = 4;  // single-CTA tiles: one epilogue warp per TMEM lane quadrant
constexpr int kEpiWarpsP = 8;  // CTA pairs: two per quadrant, alternate 32-column chunks
constexpr int kThreads1 = (2 + kEpiWarps1) * 32;
constexpr int kThreadsP = (2 + kEpiWarpsP) * 32;

// single-CTA tiles
constexpr int BM1 = kGemmBM;  // 128
constexpr int kStages1 = 4;
constexpr int kEpiBufs1 = 2;
constexpr int kAStage1 = BM1 * BK;  // 16 KB
constexpr int kBStage1 = BN * BK;   // 32 KB
constexpr int kSmemRing1 = kStages1 * (kAStage1 + kBStage1);
constexpr int kSmemBars1 = 8 * (2 * kStages1 + 2 * kAccBufs) + 16;
constexpr int kSmemTotal1 = kSmemRing1 + epi_smem(kEpiWarps1, kEpiBufs1) + kSmemBars1 + 1024;
static_assert(kSmemTotal1 <= 227 * 1024, "shared memory budget");

// CTA-pair tiles
constexpr int BMP = 2 * kGemmBM;         // 256 rows per pair, 128 per CTA
constexpr int kAStageP = kGemmBM * BK;   // 16 KB: this CTA's 128 rows of A
constexpr int kBStageP = (BN / 2) * BK;  // 16 KB: this CTA's half of B
constexpr int kStagesP = 6;
constexpr int kEpiBufsP = 1;  // with eight epilogue warps one staging buffer each fits beside 6 stages
constexpr int kSmemRingP = kStagesP * (kAStageP + kBStageP);
constexpr int kSmemBarsP = 8 * (2 * kStagesP + 2 * kAccBufs) + 16;
constexpr int kSmemTotalP = kSmemRingP + epi_smem(kEpiWarpsP, kEpiBufsP) + kSmemBarsP + 1024;
static_assert(kSmemTotalP <= 227 * 1024, "shared memory budget");

// ============================================================================ single-CTA tiles

template <int EPI>
__global__ void __launch_bounds__(kThreads1, 1)
    igemm_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                 const __grid_constant__ CUtensorMap ymap, const GemmArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages1 * kAStage1;
    uint8_t* sEpi = smem + kSmemRing1;
    float* sCols = reinterpret_cast<float*>(sEpi + kEpiWarps1 * kEpiBufs1 * kEpiBufBytes);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(sCols + kEpiWarps1 * 2 * BN);
    uint64_t* empty_bar = full_bar + kStages1;
    uint64_t* accf_bar = empty_bar + kStages1;
    uint64_t* acce_bar = accf_bar + kAccBufs;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce_bar + kAccBufs);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tiles_m = (p.M + BM1 - 1) / BM1;
    const int tiles_n = (p.N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n * p.batch;
    const int k_blocks = (p.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&bmap);
        tma_prefetch_desc(&ymap);
        for (int s = 0; s < kStages1; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < kAccBufs; ++a) {
            mbar_init(&accf_bar[a], 1);
            mbar_init(&acce_bar[a], kEpiWarps1 * 32);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    // Everything above overlaps the previous kernel; from here on we read its output.
    pdl_wait_primary();

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------- producer
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                const TileCoord c = tile_coord(t, tiles_m, tiles_n, BM1, p.group_m);
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, p.limit_ns, kErrTimeoutEmpty, p.err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full_bar[stage], kAStage1 + kBStage1);
                    tma_load_3d(sA + stage * kAStage1, &amap, &full_bar[stage], kb * BK, c.m0, c.b);
                    tma_load_3d(sB + stage * kBStage1, &bmap, &full_bar[stage], kb * BK, c.n0, c.b);
                    if (++stage == kStages1) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (ok) drain_ring(empty_bar, kStages1, stage, phase, p.limit_ns, kErrTimeoutEmpty, p.err);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer
            constexpr uint32_t idesc = umma_idesc_i8(BM1, BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
                if (!mbar_wait_bounded(&acce_bar[acc], acc_phase ^ 1u, p.limit_ns, kErrTimeoutAccEmpty, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait_bounded(&full_bar[stage], phase, p.limit_ns, kErrTimeoutMmaFull, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_u32(sA + stage * kAStage1);
                    const uint32_t b_addr = smem_u32(sB + stage * kBStage1);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) {
                        mma_i8(d_tmem, umma_desc_sw128_kmajor(a_addr + k * 32),
                               umma_desc_sw128_kmajor(b_addr + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit(&empty_bar[stage]);
                    if (++stage == kStages1) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                mma_commit(&accf_bar[acc]);
                if (++acc == kAccBufs) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
        }
    } else {
        // -------------------------------------------------------------- epilogue
        const int ew = warp - 2;    // 0..3
        const int quad = warp & 3;  // TMEM lane quadrant this warp may read
        uint8_t* ebuf = sEpi + ew * kEpiBufs1 * kEpiBufBytes;
        float* sColScale = sCols + ew * 2 * BN;
        float* sColBias = sColScale + BN;
        int acc = 0;
        uint32_t acc_phase = 0;
        int nbuf = 0;
        TileScales next{};
        if (blockIdx.x < num_tiles) {
            const TileCoord c = tile_coord(blockIdx.x, tiles_m, tiles_n, BM1, p.group_m);
            fetch_tile_scales<EPI>(p, c, c.m0 + quad * 32 + lane, lane, next);
        }
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
            const TileCoord c = tile_coord(t, tiles_m, tiles_n, BM1, p.group_m);
            store_tile_columns<EPI>(next, p.alpha, sColScale, sColBias, lane);
            const float sa = next.row_scale;
            if (t + static_cast<int>(gridDim.x) < num_tiles) {
                const TileCoord cn = tile_coord(t + gridDim.x, tiles_m, tiles_n, BM1, p.group_m);
                fetch_tile_scales<EPI>(p, cn, cn.m0 + quad * 32 + lane, lane, next);
            }
            const bool ok = mbar_wait_bounded(&accf_bar[acc], acc_phase, p.limit_ns, kErrTimeoutAccFull, p.err);
            tc_fence_after_sync();
            const int row0 = c.m0 + quad * 32;
            if (ok && row0 < p.M)
                epilogue_slice<EPI, kEpiWarps1, kEpiBufs1>(p, &ymap, tmem_base, quad, static_cast<uint32_t>(acc * BN),
                                                           row0, c.n0, c.b, sa, sColScale, sColBias, ebuf, lane, 0, nbuf);
            tc_fence_before_sync();
            mbar_arrive(&acce_bar[acc]);
            if (!ok) break;
            if (++acc == kAccBufs) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0) bulk_wait_group<0>();
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc(tmem_base, kTmemCols);
}

// ============================================================================ CTA-pair tiles

template <int EPI>
__global__ void __launch_bounds__(kThreadsP, 1)
    igemm_pair_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                      const __grid_constant__ CUtensorMap ymap, const GemmArgs p) {
    extern __shared__ uint8_t smem_raw[];
    // The same layout in both CTAs: the pair's MMAs and commits address the
    // peer's shared memory at the same offsets as the leader's.
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStagesP * kAStageP;
    uint8_t* sEpi = smem + kSmemRingP;
    float* sCols = reinterpret_cast<float*>(sEpi + kEpiWarpsP * kEpiBufsP * kEpiBufBytes);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(sCols + kEpiWarpsP * 2 * BN);  // used in the leader
    uint64_t* empty_bar = full_bar + kStagesP;                                       // in both CTAs
    uint64_t* accf_bar = empty_bar + kStagesP;                                       // in both CTAs
    uint64_t* acce_bar = accf_bar + kAccBufs;                                        // used in the leader
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce_bar + kAccBufs);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();  // 0 = leader
    const int pair = blockIdx.x >> 1;
    const int num_pairs = gridDim.x >> 1;
    const int tiles_m = (p.M + BMP - 1) / BMP;
    const int tiles_n = (p.N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n * p.batch;
    const int k_blocks = (p.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&bmap);
        tma_prefetch_desc(&ymap);
        for (int s = 0; s < kStagesP; ++s) {
            mbar_init(&full_bar[s], 1);   // the leader's producer arrives; both CTAs' loads complete bytes
            mbar_init(&empty_bar[s], 1);  // the leader's commit arrives (multicast)
        }
        for (int a = 0; a < kAccBufs; ++a) {
            mbar_init(&accf_bar[a], 1);              // the leader's commit arrives (multicast)
            mbar_init(&acce_bar[a], 2 * kEpiWarpsP);  // every epilogue warp of both CTAs
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    cluster_sync();  // barriers initialised and TMEM allocated in both CTAs
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    pdl_wait_primary();

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------- producer (both CTAs)
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += num_pairs) {
                const TileCoord c = tile_coord(t, tiles_m, tiles_n, BMP, p.group_m);
                const int a_row = c.m0 + static_cast<int>(rank) * kGemmBM;
                const int b_row = c.n0 + static_cast<int>(rank) * (BN / 2);
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, p.limit_ns, kErrTimeoutEmpty, p.err)) {
                        ok = false;
                        break;
                    }
                    // The leader expects both CTAs' bytes on its own barrier.
                    if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * (kAStageP + kBStageP));
                    const uint32_t leader_full = mapa_shared(smem_u32(&full_bar[stage]), 0);
                    tma_load_3d_pair(sA + stage * kAStageP, &amap, leader_full, kb * BK, a_row, c.b);
                    tma_load_3d_pair(sB + stage * kBStageP, &bmap, leader_full, kb * BK, b_row, c.b);
                    if (++stage == kStagesP) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // the stage-releasing commits reach both CTAs' empty barriers
            if (ok) drain_ring(empty_bar, kStagesP, stage, phase, p.limit_ns, kErrTimeoutEmpty, p.err);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------------------------------------------------- MMA issuer (leader only)
            constexpr uint32_t idesc = umma_idesc_i8(BMP, BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += num_pairs) {
                if (!mbar_wait_bounded(&acce_bar[acc], acc_phase ^ 1u, p.limit_ns, kErrTimeoutAccEmpty, p.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait_bounded(&full_bar[stage], phase, p.limit_ns, kErrTimeoutMmaFull, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_addr = smem_u32(sA + stage * kAStageP);
                    const uint32_t b_addr = smem_u32(sB + stage * kBStageP);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) {
                        mma_i8_pair(d_tmem, umma_desc_sw128_kmajor(a_addr + k * 32),
                                    umma_desc_sw128_kmajor(b_addr + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair(&empty_bar[stage], 0x3);  // frees this stage in both CTAs
                    if (++stage == kStagesP) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                mma_commit_pair(&accf_bar[acc], 0x3);  // both CTAs' accumulators are ready
                if (++acc == kAccBufs) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
        }
    } else {
        // -------------------------------------------------------------- epilogue (both CTAs)
        const int ew = warp - 2;     // 0..7
        const int quad = warp & 3;   // TMEM lane quadrant this warp may read
        const int part = ew >> 2;    // which alternate 32-column chunks it drains
        uint8_t* ebuf = sEpi + ew * kEpiBufsP * kEpiBufBytes;
        float* sColScale = sCols + ew * 2 * BN;
        float* sColBias = sColScale + BN;
        const uint32_t leader_acce0 = mapa_shared(smem_u32(&acce_bar[0]), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        int nbuf = 0;
        const int row_off = static_cast<int>(rank) * kGemmBM + quad * 32;  // this warp's rows within the tile
        TileScales next{};
        if (pair < num_tiles) {
            const TileCoord c = tile_coord(pair, tiles_m, tiles_n, BMP, p.group_m);
            fetch_tile_scales<EPI>(p, c, c.m0 + row_off + lane, lane, next);
        }
        for (int t = pair; t < num_tiles; t += num_pairs) {
            const TileCoord c = tile_coord(t, tiles_m, tiles_n, BMP, p.group_m);
            store_tile_columns<EPI>(next, p.alpha, sColScale, sColBias, lane);
            const float sa = next.row_scale;
            if (t + num_pairs < num_tiles) {
                const TileCoord cn = tile_coord(t + num_pairs, tiles_m, tiles_n, BMP, p.group_m);
                fetch_tile_scales<EPI>(p, cn, cn.m0 + row_off + lane, lane, next);
            }
            const bool ok = mbar_wait_bounded(&accf_bar[acc], acc_phase, p.limit_ns, kErrTimeoutAccFull, p.err);
            tc_fence_after_sync();
            const int row0 = c.m0 + row_off;
            if (ok && row0 < p.M)
                epilogue_slice<EPI, kEpiWarpsP, kEpiBufsP>(p, &ymap, tmem_base, quad, static_cast<uint32_t>(acc * BN),
                                                          row0, c.n0, c.b, sa, sColScale, sColBias, ebuf, lane, part,
                                                          nbuf);
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_acce0 + static_cast<uint32_t>(acc * 8));
            if (!ok) break;
            if (++acc == kAccBufs) {
                acc = 0;
                acc_phase ^= 1u;
            }
        }
        if (lane == 0) bulk_wait_group<0>();
    }

    tc_fence_before_sync();
    cluster_sync();  // no CTA leaves while its peer may still signal it or read its TMEM
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

// ============================================================================ launchers

template <int EPI>
cudaError_t launch_single(const CUtensorMap& amap, const CUtensorMap& bmap, const CUtensorMap& ymap,
                          const GemmArgs& a, int num_sms, bool pdl, cudaStream_t stream) {
    auto kern = igemm_kernel<EPI>;
    int set = 0;
    cudaError_t e;
    if (!launch_figure_get(reinterpret_cast<const void*>(kern), kThreads1, kSmemTotal1, &set)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotal1);
        if (e != cudaSuccess) return e;
        launch_figure_put(reinterpret_cast<const void*>(kern), kThreads1, kSmemTotal1, 1);
    }
    const int64_t tiles = static_cast<int64_t>((a.M + BM1 - 1) / BM1) * ((a.N + BN - 1) / BN) * a.batch;
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads1);
    cfg.dynamicSmemBytes = kSmemTotal1;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, amap, bmap, ymap, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_pair(const CUtensorMap& amap, const CUtensorMap& bmap, const CUtensorMap& ymap,
                        const GemmArgs& a, int num_sms, bool pdl, cudaStream_t stream) {
    auto kern = igemm_pair_kernel<EPI>;
    cudaError_t e;
    const int64_t tiles = static_cast<int64_t>((a.M + BMP - 1) / BMP) * ((a.N + BN - 1) / BN) * a.batch;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreadsP);
    cfg.dynamicSmemBytes = kSmemTotalP;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    int max_clusters = 0;
    if (!launch_figure_get(reinterpret_cast<const void*>(kern), kThreadsP, kSmemTotalP, &max_clusters)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotalP);
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3(static_cast<unsigned>(2 * (num_sms / 2)));
        e = cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg);
        if (e != cudaSuccess) return e;
        if (max_clusters < 1) return cudaErrorInvalidConfiguration;
        launch_figure_put(reinterpret_cast<const void*>(kern), kThreadsP, kSmemTotalP, max_clusters);
    }
    const int64_t pairs = tiles < max_clusters ? tiles : max_clusters;
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    e = cudaLaunchKernelEx(&cfg, kern, amap, bmap, ymap, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_epi(const CUtensorMap& amap, const CUtensorMap& bmap, const CUtensorMap& ymap,
                       const GemmArgs& a, int num_sms, bool pdl, cudaStream_t stream) {
    if (gemm_uses_pair()) return launch_pair<EPI>(amap, bmap, ymap, a, num_sms, pdl, stream);
    return launch_single<EPI>(amap, bmap, ymap, a, num_sms, pdl, stream);
}

}  // namespace

bool gemm_uses_pair() { return CONVROT_GEMM_PAIR != 0; }

int gemm_b_box_rows() { return gemm_uses_pair() ? BN / 2 : BN; }

cudaError_t launch_igemm(const CUtensorMap& amap, const CUtensorMap& bmap, const CUtensorMap& ymap,
                         const GemmArgs& a, int epilogue, int num_sms, bool pdl, cudaStream_t stream) {
    switch (epilogue) {
        case kEpiBf16:
            return launch_epi<kEpiBf16>(amap, bmap, ymap, a, num_sms, pdl, stream);
        case kEpiBf16Gelu:
            return launch_epi<kEpiBf16Gelu>(amap, bmap, ymap, a, num_sms, pdl, stream);
        case kEpiS32:
            return launch_epi<kEpiS32>(amap, bmap, ymap, a, num_sms, pdl, stream);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace convrot
