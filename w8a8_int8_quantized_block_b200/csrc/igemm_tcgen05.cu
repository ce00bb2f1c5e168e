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
// Design (B200, one CTA per SM, persistent):
//   warp 0      TMA producer: 128x128-byte A and 256x128-byte B tiles, 128-byte
//               swizzle, into a 4-stage shared-memory ring (mbarrier per stage)
//   warp 1      MMA issuer: one thread issues tcgen05.mma kind::i8
//               (M=128, N=256, K=32) into a TMEM accumulator; tcgen05.commit
//               frees each stage and, per tile, signals the epilogue
//   warps 2..5  epilogue: tcgen05.ld 32 columns at a time, scale + bias
//               (+ GELU), bf16, swizzled shared staging, TMA store
// Two 256-column accumulators (all 512 TMEM columns) let the epilogue of one
// tile overlap the main loop of the next.  Tiles run n-fastest so the A panel
// of a 128-row block is read from HBM once and reused from L2 across N.
// No load uses cluster multicast.
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace convrot {

namespace {

constexpr int BM = kGemmBM, BN = kGemmBN, BK = kGemmBK;
constexpr int kStages = 4;
constexpr int kAccBufs = 2;
constexpr int kEpiWarps = 4;
constexpr int kThreads = (2 + kEpiWarps) * 32;
constexpr uint32_t kTmemCols = 512;
constexpr int kAStage = BM * BK;                 // 16 KB
constexpr int kBStage = BN * BK;                 // 32 KB
constexpr int kEpiBufBytes = 4096;               // per epilogue warp
constexpr int kSmemRing = kStages * (kAStage + kBStage);
constexpr int kSmemEpi = kEpiWarps * kEpiBufBytes;
constexpr int kSmemCols = kEpiWarps * 2 * BN * 4;  // per-warp column scale and bias
constexpr int kSmemBars = 8 * (2 * kStages + 2 * kAccBufs) + 16;
constexpr int kSmemTotal = kSmemRing + kSmemEpi + kSmemCols + kSmemBars + 1024;
static_assert(kSmemTotal <= 227 * 1024, "shared memory budget");

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float gelu_erf(float y) { return 0.5f * y * (1.0f + erff(y * 0.70710678118654752f)); }

struct TileCoord {
    int m0, n0, b;
};

__device__ __forceinline__ TileCoord tile_coord(int t, int tiles_m, int tiles_n) {
    const int per_batch = tiles_m * tiles_n;
    const int b = t / per_batch;
    const int r = t - b * per_batch;
    const int mb = r / tiles_n;
    return {mb * BM, (r - mb * tiles_n) * BN, b};
}

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    igemm_kernel(const __grid_constant__ CUtensorMap amap, const __grid_constant__ CUtensorMap bmap,
                 const __grid_constant__ CUtensorMap ymap, const GemmArgs p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* sA = smem;
    uint8_t* sB = smem + kStages * kAStage;
    uint8_t* sEpi = smem + kSmemRing;
    float* sCols = reinterpret_cast<float*>(sEpi + kSmemEpi);  // [warp][scale | bias][BN]
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(sCols + kEpiWarps * 2 * BN);
    uint64_t* empty_bar = full_bar + kStages;
    uint64_t* accf_bar = empty_bar + kStages;
    uint64_t* acce_bar = accf_bar + kAccBufs;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce_bar + kAccBufs);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int tiles_m = (p.M + BM - 1) / BM;
    const int tiles_n = (p.N + BN - 1) / BN;
    const int num_tiles = tiles_m * tiles_n * p.batch;
    const int k_blocks = (p.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&amap);
        tma_prefetch_desc(&bmap);
        tma_prefetch_desc(&ymap);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int a = 0; a < kAccBufs; ++a) {
            mbar_init(&accf_bar[a], 1);
            mbar_init(&acce_bar[a], kEpiWarps * 32);
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
                const TileCoord c = tile_coord(t, tiles_m, tiles_n);
                for (int kb = 0; kb < k_blocks; ++kb) {
                    if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u, p.limit_ns, kErrTimeoutEmpty, p.err)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full_bar[stage], kAStage + kBStage);
                    tma_load_3d(sA + stage * kAStage, &amap, &full_bar[stage], kb * BK, c.m0, c.b);
                    tma_load_3d(sB + stage * kBStage, &bmap, &full_bar[stage], kb * BK, c.n0, c.b);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer
            constexpr uint32_t idesc = umma_idesc_i8(BM, BN);
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
                    const uint32_t a_addr = smem_u32(sA + stage * kAStage);
                    const uint32_t b_addr = smem_u32(sB + stage * kBStage);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k) {
                        mma_i8(d_tmem, umma_desc_sw128_kmajor(a_addr + k * 32),
                               umma_desc_sw128_kmajor(b_addr + k * 32), idesc, (kb | k) != 0 ? 1u : 0u);
                    }
                    mma_commit(&empty_bar[stage]);
                    if (++stage == kStages) {
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
        // Each warp keeps its own copy of the tile's column scales, so the four
        // epilogue warps never wait on one another.
        const int ew = warp - 2;             // 0..3
        const int quad = warp & 3;           // TMEM lane quadrant this warp may read
        uint8_t* ebuf = sEpi + ew * kEpiBufBytes;
        float* sColScale = sCols + ew * 2 * BN;
        float* sColBias = sColScale + BN;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int t = blockIdx.x; t < num_tiles; t += gridDim.x) {
            const TileCoord c = tile_coord(t, tiles_m, tiles_n);
            if constexpr (EPI != kEpiS32) {
                __syncwarp();  // every lane is done with the previous tile's columns
                for (int i = lane; i < BN; i += 32) {
                    const int n = c.n0 + i;
                    const bool in = n < p.N;
                    sColScale[i] = in ? p.s_b[static_cast<int64_t>(c.b) * p.N + n] * p.alpha : 0.0f;
                    sColBias[i] = (in && p.bias != nullptr) ? p.bias[n] : 0.0f;
                }
                __syncwarp();
            }
            const bool ok = mbar_wait_bounded(&accf_bar[acc], acc_phase, p.limit_ns, kErrTimeoutAccFull, p.err);
            tc_fence_after_sync();
            const int row_in_tile = quad * 32 + lane;
            const int m = c.m0 + row_in_tile;
            float sa = 0.0f;
            if constexpr (EPI != kEpiS32) {
                if (m < p.M) sa = p.s_a[static_cast<int64_t>(c.b) * p.M + m];
            }
            const bool rows_in = c.m0 + quad * 32 < p.M;  // else this warp's rows are all past M
            if (ok && rows_in) {
                for (int cc = 0; cc < BN / 32; ++cc) {
                    if (c.n0 + cc * 32 >= p.N) break;  // whole chunk past the last column
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                                           static_cast<uint32_t>(acc * BN + cc * 32),
                                       r);
                    tmem_ld_wait();
                    if constexpr (EPI == kEpiS32) {
                        // 32 int32 = 128 bytes per row, 128-byte swizzle, single buffer
                        if (lane == 0) bulk_wait_group_read<0>();
                        __syncwarp();
                        uint8_t* rowp = ebuf + lane * 128;
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            *reinterpret_cast<uint4*>(rowp + ((j ^ (lane & 7)) << 4)) =
                                make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_3d(&ymap, ebuf, c.n0 + cc * 32, c.m0 + quad * 32, c.b);
                            bulk_commit_group();
                        }
                    } else {
                        // 32 bf16 = 64 bytes per row, 64-byte swizzle, two buffers
                        uint8_t* buf = ebuf + (cc & 1) * 2048;
                        if (lane == 0) bulk_wait_group_read<1>();
                        __syncwarp();
                        uint32_t w[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int i0 = cc * 32 + 2 * j;
                            float y0 = fmaf(static_cast<float>(static_cast<int32_t>(r[2 * j])),
                                            sa * sColScale[i0], sColBias[i0]);
                            float y1 = fmaf(static_cast<float>(static_cast<int32_t>(r[2 * j + 1])),
                                            sa * sColScale[i0 + 1], sColBias[i0 + 1]);
                            if constexpr (EPI == kEpiBf16Gelu) {
                                y0 = gelu_erf(y0);
                                y1 = gelu_erf(y1);
                            }
                            w[j] = pack_bf16x2(y0, y1);
                        }
                        uint8_t* rowp = buf + lane * 64;
                        const int sw = (lane >> 1) & 3;
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            *reinterpret_cast<uint4*>(rowp + ((j ^ sw) << 4)) =
                                make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_3d(&ymap, buf, c.n0 + cc * 32, c.m0 + quad * 32, c.b);
                            bulk_commit_group();
                        }
                    }
                }
            }
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

template <int EPI>
cudaError_t launch_epi(const CUtensorMap& amap, const CUtensorMap& bmap, const CUtensorMap& ymap,
                       const GemmArgs& a, int num_sms, bool pdl, cudaStream_t stream) {
    auto kern = igemm_kernel<EPI>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemTotal);
    if (e != cudaSuccess) return e;
    const int64_t tiles = static_cast<int64_t>((a.M + BM - 1) / BM) * ((a.N + BN - 1) / BN) * a.batch;
    const int grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = kSmemTotal;
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

}  // namespace

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
