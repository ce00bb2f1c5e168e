// attention.cu -- int8 attention on the 5th-generation tensor cores, without
// materialising the score matrix.
//
// What it computes (the Rung-Omega engine's "sageattn_qk_int8_pv_fp16_cuda":
// int8 Q K^T and 16-bit P V -- MiniMax-H3-Rung-Omega README, "Technical
// Architecture Overview", item 2), for every head h and query row i:
//
//   S_ij = (q_i . k_j) * s_q[i] * s_k[j] * scale      q, k: int8 rows, per-row scales
//   O_i  = sum_j softmax_j(S_i.) v_j                   v: bf16, O: bf16
//
// with the online softmax (running row maximum m and sum l, the partial O
// rescaled by 2^(m_old - m_new) whenever m grows), so S only ever lives one
// 128 x 128 tile at a time in tensor memory.
//
// One CTA per (head, 128-query tile), 192 threads:
//   warp 0     TMA producer: the Q tile once, then for each 128-key tile its
//              K codes, the two halves of V^T and the 128 key scales into one
//              of two ring stages
//   warp 1     TMEM owner and MMA issuer (one thread):
//                S_b = Q K_j^T      kind::i8, M = N = 128, 4 MMAs of K = 32,
//                                   into S buffer b = j % 2 (TMEM columns 128 b)
//                O  += P_j V_j      kind::f16 (bf16 in, f32 accumulate),
//                                   8 MMAs of K = 16, into TMEM columns 256..383
//              QK_{j+1} is issued before P V_j, so the next scores are being
//              computed while the softmax works on this tile.
//   warps 2-5  softmax, one thread per query row (TMEM lane quadrant =
//              warp % 4): scores from TMEM into registers, scaled to log2
//              units, the row maximum, p = 2^(x - m) on the special-function
//              unit, p rounded to bf16 into the P buffer (128-byte swizzle,
//              the A operand's canonical K-major layout), the row sum; then,
//              once P V_{j-1} is done, O *= 2^(m_old - m_new) in TMEM (skipped
//              when no row of the warp changed its maximum); finally O / l,
//              bf16, to global memory.
// Every wait is bounded (a time-out records kErrTimeoutAttn and the CTA
// unwinds).  V arrives as V^T [h][d][key] (K-major for the P V product),
// written by transpose_kernel below.
#include <cuda_bf16.h>

#include "attention.h"
#include "gemm_core.cuh"
#include "ptx.cuh"
#include "ptx_attn.cuh"

namespace convrot {

namespace {

constexpr int kD = 128;        // head dimension
constexpr int kTile = 128;     // queries per CTA and keys per tile
constexpr int kThreadsA = 192;
constexpr int kQBytes = kTile * kD;           // int8 Q tile: 16 KB
constexpr int kKBytes = kTile * kD;           // int8 K tile: 16 KB
constexpr int kAtomBytes = 128 * 128;         // one 128-row x 128-byte swizzle column: 16 KB
constexpr int kVBytes = 2 * kAtomBytes;       // V^T tile (128 d x 128 keys bf16): 32 KB
constexpr int kPBytes = 2 * kAtomBytes;       // P tile (128 queries x 128 keys bf16): 32 KB
constexpr int kSkBytes = kTile * 4;           // the tile's key scales
constexpr int kStages = 2;
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQBytes;
constexpr int kOffV = kOffK + kStages * kKBytes;
constexpr int kOffP = kOffV + kStages * kVBytes;
constexpr int kOffSk = kOffP + 2 * kPBytes;
constexpr int kOffBar = kOffSk + kStages * kSkBytes;
constexpr int kNumBars = 1 + 2 * kStages + 2 + 2 + 2 + 2;
constexpr int kSmemA = kOffBar + kNumBars * 8 + 16 + 1024;  // + TMEM slot, + 1024-byte alignment slack
static_assert(kSmemA <= 227 * 1024, "shared memory budget");
constexpr uint32_t kTmemColsA = 512;          // S0, S1, O (384 used)
constexpr uint32_t kColO = 256;

struct AttnArgs {
    int H, Lq, Lk;
    const float* s_q;      // [H][Lq]
    const float* s_k;      // [H][Lk]
    float scale_log2;      // softmax scale * log2(e)
    uint16_t* o;           // [H][Lq][128] bf16
    uint64_t limit_ns;
    unsigned int* err;
};

__device__ __forceinline__ float int_to_float_exact(uint32_t s) {
    // |s| < 2^22 (|q . k| <= 127^2 * 128): adding 1.5 * 2^23 in the integer
    // domain puts s in the mantissa of a float near 2^23 + 2^22, exactly.
    return __uint_as_float(s + 0x4B400000u) - 12582912.0f;
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__global__ void __launch_bounds__(kThreadsA, 1)
    attention_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vtmap, const AttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = gcore::align1024(smem_raw);
    uint8_t* sQ = smem + kOffQ;
    uint8_t* sK = smem + kOffK;
    uint8_t* sV = smem + kOffV;
    uint8_t* sP = smem + kOffP;
    float* sSk = reinterpret_cast<float*>(smem + kOffSk);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* q_full = bars;
    uint64_t* kv_full = bars + 1;             // [2]
    uint64_t* kv_empty = kv_full + kStages;   // [2]
    uint64_t* s_full = kv_empty + kStages;    // [2]
    uint64_t* s_free = s_full + 2;            // [2]
    uint64_t* p_ready = s_free + 2;           // [2]
    uint64_t* pv_done = p_ready + 2;          // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int q_tiles = a.Lq / kTile;
    const int h = blockIdx.x / q_tiles;
    const int q0 = (blockIdx.x - h * q_tiles) * kTile;
    const int T = a.Lk / kTile;  // key tiles

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&qmap);
        tma_prefetch_desc(&kmap);
        tma_prefetch_desc(&vtmap);
        mbar_init(q_full, 1);
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&s_full[b], 1);
            mbar_init(&s_free[b], 4);   // one arrival per softmax warp
            mbar_init(&p_ready[b], 4);
            mbar_init(&pv_done[b], 1);
        }
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemColsA);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    pdl_wait_primary();  // Q, K, V^T and the scales may come from the previous kernels

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------------- producer
            bool ok = true;
            mbar_arrive_expect_tx(q_full, kQBytes);
            tma_load_3d(sQ, &qmap, q_full, 0, q0, h);
            for (int j = 0; j < T && ok; ++j) {
                const int st = j % kStages;
                if (!mbar_wait_bounded(&kv_empty[st], ((j / kStages) & 1) ^ 1u, a.limit_ns, kErrTimeoutAttn,
                                       a.err)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&kv_full[st], kKBytes + kVBytes + kSkBytes);
                tma_load_3d(sK + st * kKBytes, &kmap, &kv_full[st], 0, j * kTile, h);
                // V^T rows are the 128 d; each 64-key half is one 128-byte swizzle column
                tma_load_3d(sV + st * kVBytes, &vtmap, &kv_full[st], j * kTile, 0, h);
                tma_load_3d(sV + st * kVBytes + kAtomBytes, &vtmap, &kv_full[st], j * kTile + 64, 0, h);
                bulk_load_g2s(sSk + st * kTile, a.s_k + static_cast<int64_t>(h) * a.Lk + j * kTile, kSkBytes,
                              &kv_full[st]);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer
            constexpr uint32_t idesc_qk = umma_idesc_i8(kTile, kTile);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(kTile, kD);
            bool ok = mbar_wait_bounded(q_full, 0, a.limit_ns, kErrTimeoutAttn, a.err);
            const uint32_t q_addr = smem_u32(sQ);
            auto issue_pv = [&](int i) -> bool {
                const int pb = i & 1;
                if (!mbar_wait_bounded(&p_ready[pb], (i >> 1) & 1, a.limit_ns, kErrTimeoutAttn, a.err)) return false;
                tc_fence_after_sync();
                const uint32_t p_addr = smem_u32(sP + pb * kPBytes);
                const uint32_t v_addr = smem_u32(sV + (i % kStages) * kVBytes);
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {  // K = 16 keys per MMA
                    const uint32_t off = static_cast<uint32_t>((kk >> 2) * kAtomBytes + (kk & 3) * 32);
                    mma_bf16(tmem + kColO, umma_desc_sw128_kmajor(p_addr + off), umma_desc_sw128_kmajor(v_addr + off),
                             idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&pv_done[pb]);
                mma_commit(&kv_empty[i % kStages]);
                return true;
            };
            for (int j = 0; j < T && ok; ++j) {
                const int st = j % kStages;
                const int b = j & 1;
                if (!mbar_wait_bounded(&kv_full[st], (j / kStages) & 1, a.limit_ns, kErrTimeoutAttn, a.err)) {
                    ok = false;
                    break;
                }
                if (j >= 2 && !mbar_wait_bounded(&s_free[b], ((j - 2) >> 1) & 1, a.limit_ns, kErrTimeoutAttn, a.err)) {
                    ok = false;
                    break;
                }
                tc_fence_after_sync();
                const uint32_t k_addr = smem_u32(sK + st * kKBytes);
#pragma unroll
                for (int k = 0; k < kD / 32; ++k)  // K = 32 int8 per MMA
                    mma_i8(tmem + static_cast<uint32_t>(b * kTile), umma_desc_sw128_kmajor(q_addr + k * 32),
                           umma_desc_sw128_kmajor(k_addr + k * 32), idesc_qk, k > 0 ? 1u : 0u);
                mma_commit(&s_full[b]);
                if (j >= 1 && !issue_pv(j - 1)) {
                    ok = false;
                    break;
                }
            }
            if (ok) issue_pv(T - 1);
        }
    } else {
        // -------------------------------------------------------------- softmax (warps 2..5)
        const int quad = warp & 3;
        const int row = quad * 32 + lane;  // query row within the tile
        const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
        const float rs = a.s_q[static_cast<int64_t>(h) * a.Lq + q0 + row] * a.scale_log2;
        float m = -INFINITY, l = 0.0f;
        bool ok = true;
        for (int j = 0; j < T; ++j) {
            const int b = j & 1;
            const int st = j % kStages;
            // the stage's key scales (bulk copy) and the tile's scores
            ok = mbar_wait_bounded(&kv_full[st], (j / kStages) & 1, a.limit_ns, kErrTimeoutAttn, a.err) &&
                 mbar_wait_bounded(&s_full[b], (j >> 1) & 1, a.limit_ns, kErrTimeoutAttn, a.err);
            ok = __all_sync(0xFFFFFFFFu, ok);
            if (!ok) break;
            tc_fence_after_sync();
            // the tile's scores, scaled to log2 units: x = float(q.k) * s_k[c] * s_q * scale * log2(e)
            const float* cs = sSk + st * kTile;
            float x[kTile];
            float mx = -INFINITY;
#pragma unroll
            for (int c4 = 0; c4 < kTile / 32; ++c4) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + lane_base + static_cast<uint32_t>(b * kTile + c4 * 32), r);
                tmem_ld_wait();
#pragma unroll
                for (int t = 0; t < 32; ++t) {
                    const float v = int_to_float_exact(r[t]) * cs[c4 * 32 + t] * rs;
                    x[c4 * 32 + t] = v;
                    mx = fmaxf(mx, v);
                }
            }
            // S_b has been read: QK_{j+2} may overwrite it
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s_free[b]);

            const float m_new = fmaxf(m, mx);
            const float alpha = ex2_approx(m - m_new);  // 0 on the first tile (m = -inf)
            // P buffer b is free once P V_{j-2} is done
            if (j >= 2) {
                ok = mbar_wait_bounded(&pv_done[b], ((j - 2) >> 1) & 1, a.limit_ns, kErrTimeoutAttn, a.err);
                ok = __all_sync(0xFFFFFFFFu, ok);
                if (!ok) break;
            }
            uint8_t* prow = sP + b * kPBytes + row * 128;
            float sum = 0.0f;
#pragma unroll
            for (int c8 = 0; c8 < kTile / 8; ++c8) {  // 8 keys = one 16-byte chunk
                float p[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    p[e] = ex2_approx(x[c8 * 8 + e] - m_new);
                    sum += p[e];
                }
                const uint4 w = make_uint4(pack2_bf16(p[0], p[1]), pack2_bf16(p[2], p[3]), pack2_bf16(p[4], p[5]),
                                           pack2_bf16(p[6], p[7]));
                const int atom = c8 >> 3, chunk = c8 & 7;
                *reinterpret_cast<uint4*>(prow + atom * kAtomBytes + ((chunk ^ (row & 7)) << 4)) = w;
            }
            l = l * alpha + sum;
            m = m_new;
            // O *= alpha once P V_{j-1} is done (O holds nothing before P V_0)
            if (j >= 1) {
                ok = mbar_wait_bounded(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1, a.limit_ns, kErrTimeoutAttn, a.err);
                ok = __all_sync(0xFFFFFFFFu, ok);
                if (!ok) break;
                tc_fence_after_sync();
                if (__any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
#pragma unroll
                    for (int c4 = 0; c4 < kD / 32; ++c4) {
                        uint32_t r[32];
                        const uint32_t taddr = tmem + lane_base + kColO + static_cast<uint32_t>(c4 * 32);
                        tmem_ld_32x32b_x32(taddr, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int t = 0; t < 32; ++t) r[t] = __float_as_uint(__uint_as_float(r[t]) * alpha);
                        tmem_st_32x32b_x32(taddr, r);
                    }
                    tmem_st_wait();
                }
            }
            // P (generic-proxy stores) and O are ready for the tensor cores
            fence_proxy_async_smem();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_ready[b]);
        }
        // ------------------------------------------------------------- epilogue: O / l -> bf16
        if (ok) {
            ok = mbar_wait_bounded(&pv_done[(T - 1) & 1], ((T - 1) >> 1) & 1, a.limit_ns, kErrTimeoutAttn, a.err);
            ok = __all_sync(0xFFFFFFFFu, ok);
        }
        if (ok) {
            tc_fence_after_sync();
            const float inv = 1.0f / l;
            uint16_t* orow = a.o + (static_cast<int64_t>(h) * a.Lq + q0 + row) * kD;
#pragma unroll
            for (int c4 = 0; c4 < kD / 32; ++c4) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + lane_base + kColO + static_cast<uint32_t>(c4 * 32), r);
                tmem_ld_wait();
                uint32_t w[16];
#pragma unroll
                for (int t = 0; t < 16; ++t)
                    w[t] = pack2_bf16(__uint_as_float(r[2 * t]) * inv, __uint_as_float(r[2 * t + 1]) * inv);
#pragma unroll
                for (int v = 0; v < 2; ++v)
                    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(
                                     orow + c4 * 32 + v * 16),
                                 "r"(w[8 * v]), "r"(w[8 * v + 1]), "r"(w[8 * v + 2]), "r"(w[8 * v + 3]),
                                 "r"(w[8 * v + 4]), "r"(w[8 * v + 5]), "r"(w[8 * v + 6]), "r"(w[8 * v + 7])
                                 : "memory");
            }
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc(tmem, kTmemColsA);
}

// V [h][key][d] -> V^T [h][d][key], bf16, through 32 x 32 shared tiles.
__global__ void transpose_kernel(const uint16_t* __restrict__ v, uint16_t* __restrict__ vt, int L) {
    __shared__ uint16_t tile[32][33];
    const int h = blockIdx.z;
    const int key0 = blockIdx.x * 32, d0 = blockIdx.y * 32;
    const uint16_t* src = v + static_cast<int64_t>(h) * L * kD;
    uint16_t* dst = vt + static_cast<int64_t>(h) * kD * L;
    for (int r = threadIdx.y; r < 32; r += blockDim.y)
        tile[r][threadIdx.x] = src[static_cast<int64_t>(key0 + r) * kD + d0 + threadIdx.x];
    __syncthreads();
    for (int r = threadIdx.y; r < 32; r += blockDim.y)
        dst[static_cast<int64_t>(d0 + r) * L + key0 + threadIdx.x] = tile[threadIdx.x][r];
}

}  // namespace

cudaError_t launch_attention(const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vtmap, int H,
                             int Lq, int Lk, const float* s_q, const float* s_k, float scale_log2, uint16_t* o,
                             uint64_t limit_ns, unsigned int* err, bool pdl, cudaStream_t stream) {
    cudaError_t e = cudaFuncSetAttribute(attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemA);
    if (e != cudaSuccess) return e;
    AttnArgs a;
    a.H = H;
    a.Lq = Lq;
    a.Lk = Lk;
    a.s_q = s_q;
    a.s_k = s_k;
    a.scale_log2 = scale_log2;
    a.o = o;
    a.limit_ns = limit_ns;
    a.err = err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(H * (Lq / kTile)));
    cfg.blockDim = dim3(kThreadsA);
    cfg.dynamicSmemBytes = kSmemA;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, attention_kernel, qmap, kmap, vtmap, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_transpose_v(const uint16_t* v, uint16_t* vt, int H, int L, cudaStream_t stream) {
    transpose_kernel<<<dim3(static_cast<unsigned>(L / 32), kD / 32, static_cast<unsigned>(H)), dim3(32, 8), 0,
                       stream>>>(v, vt, L);
    return cudaGetLastError();
}

}  // namespace convrot
