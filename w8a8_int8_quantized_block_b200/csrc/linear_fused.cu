// linear_fused.cu -- the whole ConvRot W8A8 linear in one persistent kernel:
// rotate + quantise the activations while the tensor cores run the int8 GEMM
// on the rows that are already quantised.
//
// The steps are those of rotate_quant.cu (block-diagonal Hadamard rotation,
// rowwise int8: lehuy.net "Nen mo hinh video khuech tan 31B xuong 14B",
// section "Cach nen hoat dong"; MiniMax-H3-Rung-Omega README, "Technical
// Architecture Overview", item 2) and igemm_tcgen05.cu (int8 GEMM, per-token x
// per-output-channel dequantisation, bf16 out); the arithmetic and its order
// are identical, so the codes, scales and outputs equal the two-kernel path
// bit for bit.
//
// Why one kernel: the GEMM is tensor-bound and leaves most of the SM's issue
// slots and HBM bandwidth idle, while the quantiser is memory- and
// latency-bound.  Here each CTA of the CTA-pair GEMM (cta_group::2, 256 x 256
// tiles, see igemm_tcgen05.cu) also runs two quantiser groups of three warps.
// Rows are dealt round-robin to the groups of all CTAs; each group reads its
// next row straight from global memory into registers while it quantises the
// current one (no shared memory: the GEMM keeps its full 6-stage ring), writes
// the codes and scale to global memory and adds the row to its 256-row panel's
// ready count (release).  The GEMM producer of a tile acquires its panel's count before it
// loads A by TMA; the epilogue does the same before it reads the panel's
// scales.  Panels become ready in order, the tiles walk the panels in order,
// and every CTA is resident (the grid is sized to what fits), so every wait
// ends; each wait is bounded all the same.
//
// The codes live in a ring of panel slots (about 16.5 MB: 12 slots at K =
// 5376) rather than an [M][K] array: panel p goes to slot p % ring once every
// tile has loaded the panel that held the slot before (the MMA issuer counts
// a tile's panel as loaded when the last stage of its A has landed).  When
// the weights are small enough to stay in L2 beside it (N K <= 48 MB), the
// codes are stored and loaded with an L2 evict-last policy, so the ring stays
// in L2 next to the weights while x and y stream past (evict-first), and a
// slot is overwritten there rather than written back to HBM; with one slot
// per panel the codes made a ~390 MB round trip through HBM per 768p step.
// (Larger weights, as in a 4x MLP, need the L2 more; there the normal policy
// is kept.)  No wait forms a cycle: a
// quantiser waits on a panel `ring` panels earlier, whose tiles only need
// that panel's codes.
//
// Shared memory per CTA: the 6-stage GEMM ring (192 KB) and epilogue staging
// and column scales (24 KB), as in the GEMM alone.  (A 4-stage ring, which
// left room to stage input rows by TMA, ran the GEMM part 10% slower.)
#include <cuda_bf16.h>

#include "gemm_core.cuh"
#include "kernels.h"
#include "ptx.cuh"
#include "quant_core.cuh"

namespace convrot {

namespace {

using namespace gcore;
using qcore::kPairs;
using qcore::kPerThread;

constexpr int kQGroups = 2;                    // quantiser groups per CTA
constexpr int kQWarps = 3;                     // warps per group: one row of K <= 6144
constexpr int kQThreads = kQWarps * 32;
constexpr int kEpiWarpsF = 4;  // one epilogue warp per TMEM lane quadrant
constexpr int kEpiBufsF = 2;   // staging buffers per epilogue warp
constexpr int kFirstQWarp = 2 + kEpiWarpsF;
constexpr int kThreadsF = (kFirstQWarp + kQGroups * kQWarps) * 32;
constexpr int kPanelRows = 2 * kGemmBM;        // 256: the pair's tile height
// Quantisers stay at most this many panels ahead of the first panel the GEMM
// has not started, so the codes (1.4 MB per panel at K = 5376) are still in L2
// when the tensor cores read them instead of making a round trip to HBM.
// (With the 12-slot ring below, 10 panels ahead measured best: DRAM traffic
// per 768p step 846 MB, against 1025 MB for 20 slots / 16 ahead and 1210 MB
// with one slot per panel.)
constexpr int kPanelsAhead = 10;
constexpr int kStagesF = 6;
constexpr int kAStageF = kGemmBM * BK;
constexpr int kBStageF = (BN / 2) * BK;
constexpr int kSmemRingF = kStagesF * (kAStageF + kBStageF);
constexpr int kSmemBarsF = 8 * (2 * kStagesF + 2 * kAccBufs) + 16;
constexpr int kSmemRedF = kQGroups * 2 * kQWarps * 4 + kQGroups * 4;  // warp maxima, then one abort flag per group
constexpr int kSmemTotalF = kSmemRingF + epi_smem(kEpiWarpsF, kEpiBufsF) + kSmemBarsF + kSmemRedF + 1024;
static_assert(kSmemTotalF <= 227 * 1024, "shared memory budget");
static_assert(kQThreads * kPerThread >= kFusedMaxK, "a group must cover a row");

struct FusedArgs {
    GemmArgs g;             // the GEMM and its epilogue (s_a = the scales below)
    const uint16_t* x;      // [M][ldx] bf16 activations
    int64_t ldx;
    int8_t* q;              // [M][K] codes (workspace)
    float* s;               // [M] scales (workspace)
    unsigned int* ready;    // [ceil(M/256)] rows of each panel already quantised (zeroed)
    unsigned int* started;  // panels the GEMM has begun (a running max; zeroed)
    unsigned int* loaded;   // [ceil(M/256)] tiles of each panel whose codes have landed (zeroed)
    int ring;               // panel slots of the codes ring
    int l2_hint;            // mark the ring's lines evict-last in L2 (else the normal policy)
    int tpr;                // K / 64: threads of a group holding data
    int kind;               // the rotation (a RotKind; the kernel is instantiated for it)
};

__device__ __forceinline__ uint32_t panel_rows(int panel, int M) {
    const int r = M - panel * kPanelRows;
    return static_cast<uint32_t>(r < kPanelRows ? r : kPanelRows);
}

template <int EPI, int KIND>
__global__ void __launch_bounds__(kThreadsF, 1)
    linear_fused_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                        const __grid_constant__ CUtensorMap ymap, const FusedArgs f) {
    const GemmArgs& p = f.g;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStagesF * kAStageF;
    uint8_t* sEpi = smem + kSmemRingF;
    float* sCols = reinterpret_cast<float*>(sEpi + kEpiWarpsF * kEpiBufsF * kEpiBufBytes);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(sCols + kEpiWarpsF * 2 * BN);
    uint64_t* empty_bar = full_bar + kStagesF;
    uint64_t* accf_bar = empty_bar + kStagesF;
    uint64_t* acce_bar = accf_bar + kAccBufs;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce_bar + kAccBufs);
    float* red = reinterpret_cast<float*>(tmem_slot + 4);  // [group][2][warp]
    int* qabort = reinterpret_cast<int*>(red + kQGroups * 2 * kQWarps);  // [group]: a wait of the group gave up

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1;
    const int num_pairs = gridDim.x >> 1;
    const int tiles_m = (p.M + kPanelRows - 1) / kPanelRows;
    const int tiles_n = (p.N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n;
    const int k_blocks = (p.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&bmap);
        tma_prefetch_desc(&ymap);
        for (int s = 0; s < kStagesF; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < kAccBufs; ++a) {
            mbar_init(&accf_bar[a], 1);
            mbar_init(&acce_bar[a], 2 * kEpiWarpsF);
        }
        for (int gq = 0; gq < kQGroups; ++gq) qabort[gq] = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before_sync();
    cluster_sync();
    tc_fence_after_sync();
    const uint32_t tmem_base = *tmem_slot;

    pdl_wait_primary();

    if (warp >= kFirstQWarp) {
        // ================================================================ quantiser groups
        const int qg = (warp - kFirstQWarp) / kQWarps;
        const int qw = (warp - kFirstQWarp) % kQWarps;
        const int t = qw * 32 + lane;  // 0..95 within the group
        const bool holds = t < f.tpr;
        const int64_t stride = static_cast<int64_t>(gridDim.x) * kQGroups;
        const int64_t first = blockIdx.x + static_cast<int64_t>(gridDim.x) * qg;
        float* gred = red + qg * 2 * kQWarps;
        // the codes ring stays in L2 until it is reused
        const uint64_t keep_l2 = f.l2_hint ? l2_policy_evict_last() : l2_policy_evict_normal();
        uint32_t w[qcore::kRawWords];  // the next row's elements, loaded ahead
        if (holds && first < p.M) qcore::load_bf16_global(f.x + first * f.ldx, t, w);
        int it = 0;
        for (int64_t row = first; row < p.M; row += stride, ++it) {
            // Two waits before the row's codes may be written, both taken by
            // thread 0 of the group alone; the group barrier below hands the
            // outcome (and, through the barrier, the acquired counts) to all
            // 96 threads, which then go on or leave together.  A thread that
            // timed out on its own could otherwise leave the others stuck at
            // that barrier.
            //  - Keep within kPanelsAhead panels of the GEMM.  The GEMM starts
            //    panels in order and each group quantises its rows in order, so
            //    every panel inside the window gets finished and the window
            //    moves on.
            //  - The ring slot is free once every tile of its previous panel
            //    has loaded it.
            const int panel = static_cast<int>(row / kPanelRows);
            if (t == 0) {
                bool ok = panel < kPanelsAhead ||
                          wait_count_bounded(f.started, static_cast<uint32_t>(panel - kPanelsAhead + 1),
                                             p.limit_ns, kErrTimeoutPanel, p.err);
                ok = ok && (panel < f.ring || wait_count_bounded(f.loaded + (panel - f.ring),
                                                                 static_cast<uint32_t>(tiles_n), p.limit_ns,
                                                                 kErrTimeoutPanel, p.err));
                if (!ok) qabort[qg] = 1;  // the error word is set; the GEMM side times out the same way
            }
            const int64_t qrow = static_cast<int64_t>(panel % f.ring) * kPanelRows + (row - int64_t{panel} * kPanelRows);
            uint64_t P[kPairs];
            if (holds) {
                qcore::unpack_bf16_pairs(w, P);
                const int64_t rn = row + stride;
                if (rn < p.M) qcore::load_bf16_global(f.x + rn * f.ldx, t, w);  // prefetch
            } else {
#pragma unroll
                for (int j = 0; j < kPairs; ++j) P[j] = 0ull;
            }
            qcore::rotate_piece<KIND>(P, t);
            // amax is a non-negative, non-NaN float (fmaxf from +0 drops NaNs),
            // so its bits order like the values.
            float amax = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(qcore::piece_absmax(P))));
            if (lane == 0) gred[(it & 1) * kQWarps + qw] = amax;
            named_bar_sync(1 + qg, kQThreads);  // warp maxima and thread 0's wait outcome published
            if (qabort[qg]) break;              // the same value for every thread of the group
            amax = gred[(it & 1) * kQWarps];
            for (int i = 1; i < kQWarps; ++i) amax = fmaxf(amax, gred[(it & 1) * kQWarps + i]);
            if (holds) {
                const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
                qcore::quantize_store<true, true>(P, inv, f.q + qrow * p.K + static_cast<int64_t>(t) * kPerThread,
                                                  keep_l2);
                if (t == 0) f.s[row] = __fdiv_rn(amax, 127.0f);
            }
            __threadfence();                    // this thread's codes are visible device-wide
            named_bar_sync(1 + qg, kQThreads);  // ... and so are the whole group's
            if (t == 0) {
                fence_proxy_async_global();
                red_release_gpu_add(f.ready + row / kPanelRows, 1u);
            }
        }
    } else if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------- producer (both CTAs)
            const uint64_t keep_l2 = f.l2_hint ? l2_policy_evict_last() : l2_policy_evict_normal();
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int ready_panel = -1;
            for (int t = pair; t < num_tiles && ok; t += num_pairs) {
                const TileCoord c = tile_coord(t, tiles_m, tiles_n, kPanelRows, p.group_m);
                const int panel = c.m0 / kPanelRows;
                if (panel != ready_panel) {
                    if (!wait_count_bounded(f.ready + panel, panel_rows(panel, p.M), p.limit_ns, kErrTimeoutPanel,
                                            p.err)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_global();  // the TMA reads below see the quantised panel
                    ready_panel = panel;
                    atomicMax(f.started, static_cast<unsigned int>(panel + 1));  // lets the quantisers move on
                }
                const int a_row = (panel % f.ring) * kPanelRows + static_cast<int>(rank) * kGemmBM;
                const int b_row = c.n0 + static_cast<int>(rank) * (BN / 2);
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, p.limit_ns, kErrTimeoutEmpty, p.err)) {
                        ok = false;
                        break;
                    }
                    if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], 2 * (kAStageF + kBStageF));
                    const uint32_t leader_full = mapa_shared(smem_u32(&full_bar[stage]), 0);
                    tma_load_3d_pair_hint(sA + stage * kAStageF, &amap, leader_full, kb * BK, a_row, 0, keep_l2);
                    tma_load_3d_pair(sB + stage * kBStageF, &bmap, leader_full, kb * BK, b_row, 0);
                    if (++stage == kStagesF) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // the stage-releasing commits reach both CTAs' empty barriers
            if (ok) drain_ring(empty_bar, kStagesF, stage, phase, p.limit_ns, kErrTimeoutEmpty, p.err);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------------------------------------------------- MMA issuer (leader only)
            constexpr uint32_t idesc = umma_idesc_i8(kPanelRows, BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            bool ok = true;
            for (int t = pair; t < num_tiles && ok; t += num_pairs) {
                // the tile's row panel (its codes' ring slot gets one reader less below)
                const int tile_panel = tile_coord(t, tiles_m, tiles_n, kPanelRows, p.group_m).m0 / kPanelRows;
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
                    const uint32_t a_addr = smem_u32(sA + stage * kAStageF);
                    const uint32_t b_addr = smem_u32(sB + stage * kBStageF);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) {
                        mma_i8_pair(d_tmem, umma_desc_sw128_kmajor(a_addr + k * 32),
                                    umma_desc_sw128_kmajor(b_addr + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair(&empty_bar[stage], 0x3);
                    if (++stage == kStagesF) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                // Both CTAs' A stages of this tile have landed (each full barrier
                // counts both halves), so its reads of the panel's ring slot are
                // complete: the slot has one reader less.  (A plain reduction: the
                // reads finished before the barrier wait returned.)
                if (ok && f.ring < tiles_m) atomicAdd(f.loaded + tile_panel, 1u);
                mma_commit_pair(&accf_bar[acc], 0x3);
                if (++acc == kAccBufs) {
                    acc = 0;
                    acc_phase ^= 1u;
                }
            }
        }
    } else {
        // -------------------------------------------------------------- epilogue (both CTAs)
        const int ew = warp - 2;
        const int quad = warp & 3;
        uint8_t* ebuf = sEpi + ew * kEpiBufsF * kEpiBufBytes;
        float* sColScale = sCols + ew * 2 * BN;
        float* sColBias = sColScale + BN;
        const uint32_t leader_acce0 = mapa_shared(smem_u32(&acce_bar[0]), 0);
        int acc = 0;
        uint32_t acc_phase = 0;
        int nbuf = 0;
        for (int t = pair; t < num_tiles; t += num_pairs) {
            const TileCoord c = tile_coord(t, tiles_m, tiles_n, kPanelRows, p.group_m);
            load_tile_columns<EPI>(p, c, sColScale, sColBias, lane);
            bool ok = mbar_wait_bounded(&accf_bar[acc], acc_phase, p.limit_ns, kErrTimeoutAccFull, p.err);
            tc_fence_after_sync();
            // The accumulator is done, so the panel was ready; acquire it again
            // here so that this warp's reads of the panel's scales see them.
            const int panel = c.m0 / kPanelRows;
            if (ok && lane == 0)
                ok = wait_count_bounded(f.ready + panel, panel_rows(panel, p.M), p.limit_ns, kErrTimeoutPanel, p.err);
            ok = __shfl_sync(0xFFFFFFFFu, ok ? 1 : 0, 0) != 0;
            __syncwarp();  // orders lane 0's acquire before every lane's reads of the scales
            const int row0 = c.m0 + static_cast<int>(rank) * kGemmBM + quad * 32;
            float sa = 0.0f;
            if (ok && row0 + lane < p.M) sa = f.s[row0 + lane];
            if (ok && row0 < p.M)
                epilogue_slice<EPI, kEpiWarpsF, kEpiBufsF>(p, &ymap, tmem_base, quad, static_cast<uint32_t>(acc * BN),
                                                           row0, c.n0, 0, sa, sColScale, sColBias, ebuf, lane, 0, nbuf);
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
    cluster_sync();
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

template <int EPI, int KIND>
cudaError_t launch_fused_epi(const CUtensorMap& amap, const CUtensorMap& bmap, const CUtensorMap& ymap,
                             const FusedArgs& f, int num_sms, bool pdl, cudaStream_t stream) {
    auto kern = linear_fused_kernel<EPI, KIND>;
    cudaError_t e;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreadsF);
    cfg.dynamicSmemBytes = kSmemTotalF;
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
    if (!launch_figure_get(reinterpret_cast<const void*>(kern), kThreadsF, kSmemTotalF, &max_clusters)) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotalF);
        if (e != cudaSuccess) return e;
        cfg.gridDim = dim3(static_cast<unsigned>(2 * (num_sms / 2)));
        e = cudaOccupancyMaxActiveClusters(&max_clusters, kern, &cfg);
        if (e != cudaSuccess) return e;
        if (max_clusters < 1) return cudaErrorInvalidConfiguration;
        launch_figure_put(reinterpret_cast<const void*>(kern), kThreadsF, kSmemTotalF, max_clusters);
    }
    // Every CTA quantises rows other CTAs wait for, so all of them must be
    // resident at once: never launch more clusters than fit.  Launch all that
    // fit even when there are fewer tiles: the quantiser groups of CTAs without
    // a tile still share the rows (a 256-row problem of two tiles would
    // otherwise quantise its rows 32 at a time in each of 8 groups).
    cfg.gridDim = dim3(static_cast<unsigned>(2 * max_clusters));
    e = cudaLaunchKernelEx(&cfg, kern, amap, bmap, ymap, f);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_fused_kind(const CUtensorMap& amap, const CUtensorMap& bmap, const CUtensorMap& ymap,
                              const FusedArgs& f, int num_sms, bool pdl, cudaStream_t stream) {
    switch (f.kind) {
        case kRotNone: return launch_fused_epi<EPI, kRotNone>(amap, bmap, ymap, f, num_sms, pdl, stream);
        case kRotSyl64: return launch_fused_epi<EPI, kRotSyl64>(amap, bmap, ymap, f, num_sms, pdl, stream);
        case kRotSyl128: return launch_fused_epi<EPI, kRotSyl128>(amap, bmap, ymap, f, num_sms, pdl, stream);
        case kRotSyl256: return launch_fused_epi<EPI, kRotSyl256>(amap, bmap, ymap, f, num_sms, pdl, stream);
        case kRotReg16: return launch_fused_epi<EPI, kRotReg16>(amap, bmap, ymap, f, num_sms, pdl, stream);
        case kRotReg64: return launch_fused_epi<EPI, kRotReg64>(amap, bmap, ymap, f, num_sms, pdl, stream);
        case kRotReg256: return launch_fused_epi<EPI, kRotReg256>(amap, bmap, ymap, f, num_sms, pdl, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_linear_fused(const uint16_t* x, int64_t ldx, const CUtensorMap& amap, const CUtensorMap& bmap,
                                const CUtensorMap& ymap, const GemmArgs& g, int8_t* q, float* s,
                                unsigned int* ready, int kind, int epilogue, int num_sms, bool pdl,
                                cudaStream_t stream) {
    FusedArgs f;
    f.g = g;
    f.x = x;
    f.ldx = ldx;
    f.q = q;
    f.s = s;
    f.ready = ready;
    f.started = ready + (g.M + kPanelRows - 1) / kPanelRows;
    f.loaded = f.started + 1;
    f.ring = fused_ring_slots(g.M, g.K);
    f.l2_hint = fused_codes_l2_hint(g.K, g.N) ? 1 : 0;
    f.tpr = g.K / kPerThread;
    f.kind = kind;
    if (f.tpr > kQThreads || g.K % kPerThread != 0) return cudaErrorInvalidValue;
    switch (epilogue) {
        case kEpiBf16:
            return launch_fused_kind<kEpiBf16>(amap, bmap, ymap, f, num_sms, pdl, stream);
        case kEpiBf16Gelu:
            return launch_fused_kind<kEpiBf16Gelu>(amap, bmap, ymap, f, num_sms, pdl, stream);
        default:
            return cudaErrorInvalidValue;
    }
}

}  // namespace convrot
