// gemm_core.cuh -- pieces shared by the int8 GEMM kernels: tile
// coordinates, the per-warp column scales and the TMEM-draining epilogue
// (scale, bias, optional GELU, bf16 or raw int32, swizzled staging, TMA store).
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace convrot {
namespace gcore {

constexpr int BN = kGemmBN, BK = kGemmBK;
constexpr int kAccBufs = 2;
constexpr uint32_t kTmemCols = 512;
constexpr int kEpiRowBytes = 64;                  // one staged row: 32 bf16 or 16 int32
constexpr int kEpiBufBytes = 32 * kEpiRowBytes;   // one 32-row staging buffer (64-byte swizzle)

// Shared memory the epilogue of `ew` warps with `bufs` staging buffers each
// needs: the buffers and a private copy of the tile's column scales and
// biases per warp.
__host__ __device__ constexpr int epi_smem(int ew, int bufs) { return ew * (bufs * kEpiBufBytes + 2 * BN * 4); }

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

// f32 pairs in one 64-bit register: packed FMA / multiply on both halves.
__device__ __forceinline__ uint64_t pk2f(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk2f(uint64_t r, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t fma2f(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t mul2f(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float exp2_approx(float x) {
    float r;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// GELU(y) = y Phi(y) = 0.5 y erfc(-y / sqrt 2) (the exact-erf GELU), two
// values at a time.  With x = |y| / sqrt 2 and t = 1 / (1 + x / 2),
// erfc(x) = t 2^(g(t) - log2(e) x^2), g a degree-7 polynomial in t
// interpolated at Chebyshev nodes (log2(e) log(erfcx(x) / t), the form of the
// Chebyshev-fitted erfc in Numerical Recipes); fit_gelu_erfc.py in the package
// derives the coefficients and reports the error of this evaluation in f32:
// at most 1.5e-5 relative to GELU in float64, far below bf16's 2^-9.
// y >= 0 gives y - 0.5 y erfc(x); y < 0 gives 0.5 y erfc(x), so the negative
// tail keeps its relative accuracy.  No branch: both values take the same path.
__device__ __forceinline__ void gelu_pair(float& y0, float& y1) {
    const float a0 = fabsf(y0), a1 = fabsf(y1);
    const uint64_t t = pk2f(rcp_approx(fmaf(a0, 0.353553391f, 1.0f)), rcp_approx(fmaf(a1, 0.353553391f, 1.0f)));
    uint64_t g = fma2f(pk2f(-2.396635413e-01f, -2.396635413e-01f), t, pk2f(9.644635320e-01f, 9.644635320e-01f));
    g = fma2f(g, t, pk2f(-1.259334445e+00f, -1.259334445e+00f));
    g = fma2f(g, t, pk2f(3.582076728e-01f, 3.582076728e-01f));
    g = fma2f(g, t, pk2f(5.822304171e-03f, 5.822304171e-03f));
    g = fma2f(g, t, pk2f(5.541245341e-01f, 5.541245341e-01f));
    g = fma2f(g, t, pk2f(1.442124605e+00f, 1.442124605e+00f));
    g = fma2f(g, t, pk2f(-1.825744033e+00f, -1.825744033e+00f));
    const uint64_t a = pk2f(a0, a1);
    float e0, e1;
    upk2f(fma2f(mul2f(a, pk2f(-0.721347520f, -0.721347520f)), a, g), e0, e1);  // - log2(e) x^2 + g
    const uint64_t h = mul2f(mul2f(t, pk2f(exp2_approx(e0), exp2_approx(e1))),
                             mul2f(pk2f(y0, y1), pk2f(0.5f, 0.5f)));  // 0.5 y erfc(x)
    float h0, h1;
    upk2f(h, h0, h1);
    y0 = y0 >= 0.0f ? y0 - h0 : h0;
    y1 = y1 >= 0.0f ? y1 - h1 : h1;
}

struct TileCoord {
    int m0, n0, b;
};

// Tile t of a [batch][tiles_m][tiles_n] grid of bm x BN tiles.  Within a
// batch the row tiles go in groups of `group` (the last group may be
// shorter); inside a group the column tile changes slowest and the row tile
// fastest, so consecutive tiles (run at the same time by neighbouring CTA
// pairs) share their column tile.  group = 1: n fastest, one row tile after
// another.
__device__ __forceinline__ TileCoord tile_coord(int t, int tiles_m, int tiles_n, int bm, int group = 1) {
    const int per_batch = tiles_m * tiles_n;
    const int b = t / per_batch;
    const int r = t - b * per_batch;
    if (group == 1) {  // the plain order (the same tiles; two divisions fewer)
        const int mb = r / tiles_n;
        return {mb * bm, (r - mb * tiles_n) * BN, b};
    }
    const int per_group = group * tiles_n;
    const int g = r / per_group;
    const int rows = min(group, tiles_m - g * group);  // row tiles in this group
    const int w = r - g * per_group;
    const int n = w / rows;
    const int mb = g * group + (w - n * rows);
    return {mb * bm, n * BN, b};
}

// Column scale (s_b * alpha) and bias of one tile's BN columns into this
// warp's private copy (no cross-warp waits anywhere in the epilogue).
template <int EPI>
__device__ __forceinline__ void load_tile_columns(const GemmArgs& p, const TileCoord& c, float* sColScale,
                                                  float* sColBias, int lane) {
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
}

// A tile's column scales and biases (raw s_b, not yet times alpha) and this
// lane's row scale, fetched into registers one tile ahead so that the global
// loads' latency overlaps the previous tile's drain instead of preceding it.
struct TileScales {
    float col_scale[BN / 32];
    float col_bias[BN / 32];
    float row_scale;
};

template <int EPI>
__device__ __forceinline__ void fetch_tile_scales(const GemmArgs& p, const TileCoord& c, int row, int lane,
                                                  TileScales& ts) {
    if constexpr (EPI != kEpiS32) {
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) {
            const int n = c.n0 + lane + 32 * j;
            const bool in = n < p.N;
            ts.col_scale[j] = in ? p.s_b[static_cast<int64_t>(c.b) * p.N + n] : 0.0f;
            ts.col_bias[j] = (in && p.bias != nullptr) ? p.bias[n] : 0.0f;
        }
        ts.row_scale = row < p.M ? p.s_a[static_cast<int64_t>(c.b) * p.M + row] : 0.0f;
    }
}

// The prefetched column values into this warp's private shared-memory copy.
template <int EPI>
__device__ __forceinline__ void store_tile_columns(const TileScales& ts, float alpha, float* sColScale,
                                                   float* sColBias, int lane) {
    if constexpr (EPI != kEpiS32) {
        __syncwarp();  // every lane is done with the previous tile's columns
#pragma unroll
        for (int j = 0; j < BN / 32; ++j) {
            sColScale[lane + 32 * j] = ts.col_scale[j] * alpha;
            sColBias[lane + 32 * j] = ts.col_bias[j];
        }
        __syncwarp();
    }
}

// Drain a 32-row slice of the tile's accumulator (TMEM lane quadrant
// `quad`, columns from `tmem_col`) into y rows [row0, row0 + 32).  With EW
// epilogue warps, the EW/4 warps sharing a quadrant take every (EW/4)-th
// 32-column chunk starting at `part`.  Values are staged in 64-byte rows
// (64-byte swizzle, conflict-free 16-byte stores) and written by TMA; bf16
// stores are marked first-to-evict in L2 (y is written once and not read
// back here, so it should not displace the operands).  The raw int32 path
// stores each chunk as two 16-column halves.  The warp's NBUF staging
// buffers rotate through `nbuf`, which the caller keeps across tiles: a
// buffer is rewritten only after the store that last read it (NBUF stores
// ago) has finished reading, however many chunks a ragged tile had.
template <int EPI, int EW, int NBUF>
__device__ __forceinline__ void epilogue_slice(const GemmArgs& p, const CUtensorMap* ymap, uint32_t tmem_base,
                                               int quad, uint32_t tmem_col, int row0, int n0, int b, float sa,
                                               const float* sColScale, const float* sColBias, uint8_t* ebuf,
                                               int lane, int part, int& nbuf) {
    constexpr int kStep = EW / 4;
    static_assert(NBUF >= 1, "at least one staging buffer");
    const uint64_t policy = l2_policy_evict_first();
    const int sw = (lane >> 1) & 3;  // 64-byte swizzle: chunk j of row `lane` sits at j ^ sw
    for (int cc = part; cc < BN / 32; cc += kStep) {
        if (n0 + cc * 32 >= p.N) break;  // whole chunk past the last column
        uint32_t r[32];
        tmem_ld_32x32b_x32(
            tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + tmem_col + static_cast<uint32_t>(cc * 32), r);
        tmem_ld_wait();
        if constexpr (EPI == kEpiS32) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (n0 + cc * 32 + h * 16 >= p.N) break;
                uint8_t* buf = ebuf + nbuf * kEpiBufBytes;
                if (lane == 0) bulk_wait_group_read<NBUF - 1>();
                __syncwarp();
                uint8_t* rowp = buf + lane * kEpiRowBytes;
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    *reinterpret_cast<uint4*>(rowp + ((j ^ sw) << 4)) =
                        make_uint4(r[16 * h + 4 * j], r[16 * h + 4 * j + 1], r[16 * h + 4 * j + 2],
                                   r[16 * h + 4 * j + 3]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(ymap, buf, n0 + cc * 32 + h * 16, row0, b);
                    bulk_commit_group();
                }
                if (++nbuf == NBUF) nbuf = 0;
            }
        } else {
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int i0 = cc * 32 + 2 * j;
                float y0 =
                    fmaf(static_cast<float>(static_cast<int32_t>(r[2 * j])), sa * sColScale[i0], sColBias[i0]);
                float y1 = fmaf(static_cast<float>(static_cast<int32_t>(r[2 * j + 1])), sa * sColScale[i0 + 1],
                                sColBias[i0 + 1]);
                if constexpr (EPI == kEpiBf16Gelu) gelu_pair(y0, y1);
                w[j] = pack_bf16x2(y0, y1);
            }
            // The values are ready; now wait until the buffer is free again.
            uint8_t* buf = ebuf + nbuf * kEpiBufBytes;
            if (lane == 0) bulk_wait_group_read<NBUF - 1>();
            __syncwarp();
            uint8_t* rowp = buf + lane * kEpiRowBytes;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                *reinterpret_cast<uint4*>(rowp + ((j ^ sw) << 4)) =
                    make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_3d_hint(ymap, buf, n0 + cc * 32, row0, b, policy);
                bulk_commit_group();
            }
            if (++nbuf == NBUF) nbuf = 0;
        }
    }
}

}  // namespace gcore
}  // namespace convrot
