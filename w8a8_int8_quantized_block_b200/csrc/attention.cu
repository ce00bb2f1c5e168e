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
// One CTA per (head, pair of 128-query tiles A and B), 352 threads:
//   warp 0     TMA producer of the keys: the two Q tiles once, then for each
//              128-key tile its K codes and its 128 key scales into one of
//              three ring stages (freed once both tiles' scores are computed
//              and their softmax has read the scales)
//   warp 10    TMA producer of the values: the two halves of V^T of each key
//              tile into one of two ring stages (freed by both tiles' P V).
//              With separate rings the next keys load while the current P V
//              still holds its values, so no load waits on the P V chain.
//   warp 1     TMEM owner and MMA issuer (one thread), per key tile j and
//              query tile t = A, B in turn:
//                O_t += P_t V_j       kind::f16 (bf16 in, f32 accumulate), 8
//                                     MMAs of K = 16, A (P_t) read from TMEM
//                S_t = Q_t K_{j+1}^T  kind::i8, M = N = 128, 4 MMAs of K = 32
//              TMEM holds S_A, O_A, S_B, O_B (128 columns each); P_t sits in
//              the first 64 columns of S_t (bf16 pairs).  The tensor pipe runs
//              one thread's MMAs in issue order, so the next scores overwrite
//              P_t only after P V has read it; the tensor cores work on one
//              query tile while the softmax works on the other.  (One issuer
//              serving both tiles in turn measured faster than one issuer per
//              tile: 1.90 vs 2.01 ms on 42 heads of 8192.)
//   warps 2-9  softmax, four warps per query tile, one thread per query row
//              (TMEM lane quadrant = warp % 4).  One sweep over the scores in
//              TMEM (16-column loads, each overlapped with the arithmetic on
//              the previous 16) gives, against the running maximum m,
//              p = 2^(x - m) on the special-function unit, rounded to bf16
//              (kept in registers) and summed.  The tile's row maximum is
//              only taken when some row's sum of p exceeds 2^8 (else every
//              p <= 2^8 and m stays), and the exponentials are redone only
//              when a row's maximum moved (see below).  p goes back into TMEM
//              over the scores just read (two 32-column stores), where P V
//              takes it as its A operand, so P never passes through shared
//              memory (which the MMAs' operand reads keep busy).  Then O *=
//              2^(m_old - m_new) in TMEM (the reference maximum moves only
//              when a row's scores exceed it by more than 8 in log2 units, and
//              the rescale is skipped when no row of the warp moved); finally
//              O / l, bf16, to global memory.
// Two softmax warps per SM sub-partition hide each other's latencies.
// Every wait is bounded (a time-out records kErrTimeoutAttn and the CTA
// unwinds).  V arrives as V^T [h][d][key] (K-major for the P V product),
// written by transpose_kernel below.
#include <cuda_bf16.h>

#include <type_traits>

#include "attention.h"
#include "gemm_core.cuh"
#include "ptx.cuh"
#include "ptx_attn.cuh"

namespace convrot {

namespace {

constexpr int kD = 128;        // head dimension
constexpr int kTile = 128;     // queries per tile and keys per tile
constexpr int kQTiles = 2;     // query tiles per CTA
constexpr int kThreadsA = (3 + 4 * kQTiles) * 32;  // key producer, MMA, softmax, value producer
constexpr int kWarpV = 2 + 4 * kQTiles;             // the value producer's warp
constexpr int kQBytes = kTile * kD;           // int8 Q tile: 16 KB
constexpr int kKBytes = kTile * kD;           // int8 K tile: 16 KB
constexpr int kAtomBytes = 128 * 128;         // one 128-row x 128-byte swizzle column: 16 KB
constexpr int kVBytes = 2 * kAtomBytes;       // V^T tile (128 d x 128 keys bf16): 32 KB
constexpr int kSkBytes = kTile * 4;           // the tile's key scales
constexpr int kKStages = 3;                   // K codes + key scales
constexpr int kVStages = 2;                   // V^T
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQTiles * kQBytes;
constexpr int kOffV = kOffK + kKStages * kKBytes;
constexpr int kOffSk = kOffV + kVStages * kVBytes;
constexpr int kOffBar = kOffSk + kKStages * kSkBytes;
constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 3 * kQTiles;
constexpr int kSmemA = kOffBar + kNumBars * 8 + 16 + 1024;  // + TMEM slot, + 1024-byte alignment slack
static_assert(kSmemA <= 227 * 1024, "shared memory budget");
constexpr uint32_t kTmemColsA = 512;          // per query tile: S (128 columns), O (128 columns)
constexpr float kRescaleLog2 = 8.0f;          // the running maximum moves only by more than this

struct AttnArgs {
    int H, Lq, Lk;
    const float* s_q;      // [H][Lq]
    const float* s_k;      // [H][Lk]
    float scale_log2;      // softmax scale * log2(e)
    uint16_t* o;           // [H][Lq][128] bf16
    uint64_t limit_ns;
    unsigned int* err;
    // Work split: CTA i takes unit unit0 + i / splits (a head and a pair of
    // query tiles) and the splits-th part (i % splits) of its key tiles.
    // With splits > 1 it writes its unnormalised O and (m, l) per row to
    // o_part / ml_part (slot i) for attention_combine_kernel instead of O.
    int unit0, splits;
    float* o_part;         // [slot][256][128] f32
    float2* ml_part;       // [slot][256] (m, l)
};

__device__ __forceinline__ uint64_t pk2(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk2(uint64_t r, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
// A 16-byte shared load the compiler must issue where it stands (so values
// read in a loop are not held in registers across its iterations).
__device__ __forceinline__ float4 lds128(const float4* p) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(smem_u32(p)));
    return v;
}

__device__ __forceinline__ float max3(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t col_s(int t) { return static_cast<uint32_t>(t * 2 * kTile); }
__device__ __forceinline__ uint32_t col_o(int t) { return static_cast<uint32_t>(t * 2 * kTile + kTile); }

__global__ void __launch_bounds__(kThreadsA, 1)
    attention_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vtmap, const AttnArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = gcore::align1024(smem_raw);
    uint8_t* sQ = smem + kOffQ;
    uint8_t* sK = smem + kOffK;
    uint8_t* sV = smem + kOffV;
    float* sSk = reinterpret_cast<float*>(smem + kOffSk);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint64_t* q_full = bars;
    uint64_t* k_full = bars + 1;              // [key stage]
    uint64_t* k_empty = k_full + kKStages;    // [key stage]
    uint64_t* v_full = k_empty + kKStages;    // [value stage]
    uint64_t* v_empty = v_full + kVStages;    // [value stage]
    uint64_t* s_full = v_empty + kVStages;    // [query tile]
    uint64_t* p_ready = s_full + kQTiles;     // [query tile]
    uint64_t* pv_done = p_ready + kQTiles;    // [query tile]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int pairs = (a.Lq / kTile + kQTiles - 1) / kQTiles;
    const int unit = a.unit0 + static_cast<int>(blockIdx.x) / a.splits;
    const int piece = static_cast<int>(blockIdx.x) % a.splits;
    const int h = unit / pairs;
    const int q0 = (unit - h * pairs) * kQTiles * kTile;
    const int nq = min(kQTiles, (a.Lq - q0) / kTile);  // 1 when Lq / 128 is odd and this is the last pair
    const int T_all = a.Lk / kTile;
    const int j0 = piece * T_all / a.splits;           // this CTA's key tiles: [j0, j0 + T)
    const int T = (piece + 1) * T_all / a.splits - j0;

    if (threadIdx.x == 0) {
        tma_prefetch_desc(&qmap);
        tma_prefetch_desc(&kmap);
        tma_prefetch_desc(&vtmap);
        mbar_init(q_full, 1);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(&k_full[s], 1);
            mbar_init(&k_empty[s], 5 * nq);  // per query tile: the scores' commit and 4 softmax warps
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(&v_full[s], 1);
            mbar_init(&v_empty[s], nq);  // one commit per query tile's P V
        }
        for (int t = 0; t < kQTiles; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&p_ready[t], 4);  // one arrival per softmax warp of the tile
            mbar_init(&pv_done[t], 1);
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
            mbar_arrive_expect_tx(q_full, nq * kQBytes);
            for (int t = 0; t < nq; ++t) tma_load_3d(sQ + t * kQBytes, &qmap, q_full, 0, q0 + t * kTile, h);
            for (int j = 0; j < T && ok; ++j) {
                const int st = j % kKStages;
                if (!mbar_wait_bounded(&k_empty[st], ((j / kKStages) & 1) ^ 1u, a.limit_ns, kErrTimeoutAttn,
                                       a.err)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&k_full[st], kKBytes + kSkBytes);
                tma_load_3d(sK + st * kKBytes, &kmap, &k_full[st], 0, (j0 + j) * kTile, h);
                bulk_load_g2s(sSk + st * kTile, a.s_k + static_cast<int64_t>(h) * a.Lk + (j0 + j) * kTile,
                              kSkBytes, &k_full[st]);
            }
            if (ok) drain_ring(k_empty, kKStages, T % kKStages, static_cast<uint32_t>(T / kKStages) & 1u, a.limit_ns,
                               kErrTimeoutAttn, a.err);
        }
    } else if (warp == kWarpV) {
        if (lane == 0) {
            // ---------------------------------------------------------- value producer
            bool ok = true;
            for (int j = 0; j < T; ++j) {
                const int st = j % kVStages;
                if (!mbar_wait_bounded(&v_empty[st], ((j / kVStages) & 1) ^ 1u, a.limit_ns, kErrTimeoutAttn,
                                       a.err)) {
                    ok = false;
                    break;
                }
                mbar_arrive_expect_tx(&v_full[st], kVBytes);
                // V^T rows are the 128 d; each 64-key half is one 128-byte swizzle column
                tma_load_3d(sV + st * kVBytes, &vtmap, &v_full[st], (j0 + j) * kTile, 0, h);
                tma_load_3d(sV + st * kVBytes + kAtomBytes, &vtmap, &v_full[st], (j0 + j) * kTile + 64, 0, h);
            }
            if (ok) drain_ring(v_empty, kVStages, T % kVStages, static_cast<uint32_t>(T / kVStages) & 1u, a.limit_ns,
                               kErrTimeoutAttn, a.err);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------------- MMA issuer (both tiles)
            constexpr uint32_t idesc_qk = umma_idesc_i8(kTile, kTile);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(kTile, kD);
            auto issue_qk = [&](int t, int j) {
                const uint64_t qd = umma_desc_sw128_kmajor(smem_u32(sQ + t * kQBytes));
                const uint64_t kd = umma_desc_sw128_kmajor(smem_u32(sK + (j % kKStages) * kKBytes));
#pragma unroll
                for (int k = 0; k < kD / 32; ++k)  // + 32 bytes along K: + 2 in the descriptor's address field
                    mma_i8(tmem + col_s(t), qd + static_cast<uint64_t>(k * 2), kd + static_cast<uint64_t>(k * 2),
                           idesc_qk, k > 0 ? 1u : 0u);
                mma_commit(&s_full[t]);
                mma_commit(&k_empty[j % kKStages]);
            };
            auto issue_pv = [&](int t, int j) {
                const uint64_t vd = umma_desc_sw128_kmajor(smem_u32(sV + (j % kVStages) * kVBytes));
#pragma unroll
                for (int kk = 0; kk < kTile / 16; ++kk) {
                    const uint32_t off = static_cast<uint32_t>((kk >> 2) * kAtomBytes + (kk & 3) * 32);
                    mma_bf16_ts(tmem + col_o(t), tmem + col_s(t) + static_cast<uint32_t>(kk * 8),
                                vd + static_cast<uint64_t>(off >> 4), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
                }
                mma_commit(&pv_done[t]);
                mma_commit(&v_empty[j % kVStages]);
            };
            bool ok = mbar_wait_bounded(q_full, 0, a.limit_ns, kErrTimeoutAttn, a.err) &&
                      mbar_wait_bounded(&k_full[0], 0, a.limit_ns, kErrTimeoutAttn, a.err);
            if (ok) {
                tc_fence_after_sync();
                for (int t = 0; t < nq; ++t) issue_qk(t, 0);
            }
            for (int j = 0; j < T && ok; ++j) {
                for (int t = 0; t < nq && ok; ++t) {
                    ok = mbar_wait_bounded(&p_ready[t], j & 1, a.limit_ns, kErrTimeoutAttn, a.err) &&
                         (t > 0 || mbar_wait_bounded(&v_full[j % kVStages], (j / kVStages) & 1, a.limit_ns,
                                                     kErrTimeoutAttn, a.err)) &&
                         (t > 0 || j + 1 >= T ||
                          mbar_wait_bounded(&k_full[(j + 1) % kKStages], ((j + 1) / kKStages) & 1, a.limit_ns,
                                            kErrTimeoutAttn, a.err));
                    if (!ok) break;
                    tc_fence_after_sync();
                    issue_pv(t, j);  // reads P_t from S_t's first 64 columns
                    if (j + 1 < T) issue_qk(t, j + 1);  // in the same in-order pipe: after P V has read P_t
                }
            }
        }
    } else {
        // -------------------------------------------------------------- softmax (warps 2..9)
        const int t = (warp - 2) >> 2;     // query tile
        const int quad = warp & 3;
        const int row = quad * 32 + lane;  // query row within the tile
        if (t < nq) {
            const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
            const uint32_t ts = tmem + lane_base + col_s(t);
            const uint32_t to = tmem + lane_base + col_o(t);
            const float rs = a.s_q[static_cast<int64_t>(h) * a.Lq + q0 + t * kTile + row] * a.scale_log2;
            const uint64_t rs2 = pk2(rs, rs);
            float m = -INFINITY, l = 0.0f;
            bool ok = true;
            for (int j = 0; j < T; ++j) {
                const int st = j % kKStages;
                // the stage's key scales (bulk copy) and the tile's scores
                ok = mbar_wait_bounded(&k_full[st], (j / kKStages) & 1, a.limit_ns, kErrTimeoutAttn, a.err) &&
                     mbar_wait_bounded(&s_full[t], j & 1, a.limit_ns, kErrTimeoutAttn, a.err);
                ok = __all_sync(0xFFFFFFFFu, ok);
                if (!ok) break;
                tc_fence_after_sync();
                const float4* cs4 = reinterpret_cast<const float4*>(sSk + st * kTile);
                // Passes over the tile's scores from TMEM: x = float(q . k) * s_k[c]
                // (the score in log2 units is x * rs, rs = s_q * scale * log2(e) >= 0)
                // and p = 2^(x rs - mref) as packed bf16 in registers with their sum.
                // The softmax is exact for any reference m (O / l cancels it); m
                // only has to keep 2^(x - m) in range.  So the exponentials are
                // taken against the running m right away, and m moves only when a
                // row's maximum exceeds it by more than 8 (p <= 2^8 otherwise, fine
                // in bf16 and f32).  A row whose p sum to at most 2^8 has every
                // p <= 2^8, so the maximum is taken (a second pass) only when some
                // row's sum exceeds that, and a third pass redoes the exponentials
                // only when some row's maximum moved.  The first tile (m = -inf)
                // takes its maximum first, then the exponentials.
                float m_new = m;
                uint64_t sum2 = pk2(0.0f, 0.0f);
                uint32_t pw[kTile / 2];
                // One pass: with do_exp, p = 2^(x rs - mref) into pw and sum2; with
                // do_max, the row maximum of x (returned, in log2 units).
                auto pass = [&](auto do_max, auto do_exp, float mref) -> float {
                    constexpr bool kMax = decltype(do_max)::value, kExp = decltype(do_exp)::value;
                    const uint64_t nm2 = pk2(-mref, -mref);
                    float mxa = -INFINITY, mxb = -INFINITY;
                    float4 cq;
                    sum2 = pk2(0.0f, 0.0f);
                    uint32_t rb[2][16];
                    tmem_ld_32x32b_x16(ts, rb[0]);
                    tmem_ld_wait_regs(rb[0]);
#pragma unroll
                    for (int c = 0; c < kTile / 16; ++c) {
                        if (c + 1 < kTile / 16)
                            tmem_ld_32x32b_x16(ts + static_cast<uint32_t>((c + 1) * 16), rb[(c + 1) & 1]);
                        const uint32_t(&r)[16] = rb[c & 1];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {  // column pairs (2 q, 2 q + 1) of the 16
                            const int pi = c * 8 + q;
                            if ((q & 1) == 0) cq = lds128(cs4 + (pi >> 1));
                            const uint64_t c2 = (q & 1) ? pk2(cq.z, cq.w) : pk2(cq.x, cq.y);
                            const uint64_t x2 = mul2(pk2(__int2float_rn(static_cast<int>(r[2 * q])),
                                                         __int2float_rn(static_cast<int>(r[2 * q + 1]))),
                                                     c2);
                            if constexpr (kMax) {
                                float x0, x1;
                                upk2(x2, x0, x1);
                                if (q & 1)
                                    mxb = max3(mxb, x0, x1);
                                else
                                    mxa = max3(mxa, x0, x1);
                            }
                            if constexpr (kExp) {
                                float y0, y1;
                                upk2(fma2(x2, rs2, nm2), y0, y1);
                                const float p0 = ex2_approx(y0), p1 = ex2_approx(y1);
                                sum2 = add2(sum2, pk2(p0, p1));
                                pw[pi] = pack2_bf16(p0, p1);
                            }
                        }
                        if (c + 1 < kTile / 16) tmem_ld_wait_regs(rb[(c + 1) & 1]);
                    }
                    return fmaxf(mxa, mxb) * rs;
                };
                using T_ = std::true_type;
                using F_ = std::false_type;
                if (m == -INFINITY) {
                    // the first key tile: the maximum first, then the exponentials against it
                    m_new = pass(T_{}, F_{}, 0.0f);
                    pass(F_{}, T_{}, m_new);
                } else {
                    // Against the running maximum m.  Every p <= 2^8 whenever the
                    // tile's sum of p is at most 2^8, and then m need not move; only
                    // a larger sum asks for the tile's maximum, and the exponentials
                    // are redone when some row's maximum exceeds m by more than 8.
                    pass(F_{}, T_{}, m);
                    float s0, s1;
                    upk2(sum2, s0, s1);
                    if (__any_sync(0xFFFFFFFFu, !(s0 + s1 <= 256.0f))) {
                        const float mx = pass(T_{}, F_{}, 0.0f);
                        m_new = (mx > m + kRescaleLog2) ? mx : m;
                        if (__any_sync(0xFFFFFFFFu, m_new != m)) pass(F_{}, T_{}, m_new);
                    }
                }
                __syncwarp();  // the warp is done with the stage's key scales
                if (lane == 0) mbar_arrive(&k_empty[st]);
                const float alpha = ex2_approx(m - m_new);  // 0 on the first tile (m = -inf), 1 when m stays
                // P over S_t's first 64 columns (S_t is read; P V of key tile
                // j - 1 completed before these scores were committed)
                tmem_st_32x32b_x32(ts, pw);
                tmem_st_32x32b_x32(ts + 32u, pw + 32);
                float s0, s1;
                upk2(sum2, s0, s1);
                l = l * alpha + (s0 + s1);
                m = m_new;
                // O *= alpha (O holds nothing before the first P V)
                if (j >= 1 && __any_sync(0xFFFFFFFFu, alpha != 1.0f)) {
#pragma unroll
                    for (int c4 = 0; c4 < kD / 32; ++c4) {
                        uint32_t r[32];
                        const uint32_t taddr = to + static_cast<uint32_t>(c4 * 32);
                        tmem_ld_32x32b_x32(taddr, r);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                        tmem_st_32x32b_x32(taddr, r);
                    }
                }
                tmem_st_wait();  // P and the rescaled O are in tensor memory
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_ready[t]);
            }
            // ------------------------------------------------------------- epilogue: O / l -> bf16
            if (ok) {
                ok = mbar_wait_bounded(&pv_done[t], (T - 1) & 1, a.limit_ns, kErrTimeoutAttn, a.err);
                ok = __all_sync(0xFFFFFFFFu, ok);
            }
            if (ok && a.splits > 1) {
                // a part of the keys: the unnormalised O rows and (m, l) for the combine
                tc_fence_after_sync();
                const int64_t slot_row = static_cast<int64_t>(blockIdx.x) * (kQTiles * kTile) + t * kTile + row;
                float* prow_o = a.o_part + slot_row * kD;  // 16-byte aligned (the entry's contract)
#pragma unroll 1
                for (int c4 = 0; c4 < kD / 32; ++c4) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(to + static_cast<uint32_t>(c4 * 32), r);
                    tmem_ld_wait();
#pragma unroll
                    for (int v = 0; v < 8; ++v)
                        reinterpret_cast<uint4*>(prow_o + c4 * 32)[v] =
                            make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
                }
                a.ml_part[slot_row] = make_float2(m, l);
            } else if (ok) {
                tc_fence_after_sync();
                const float inv = 1.0f / l;
                uint16_t* orow = a.o + (static_cast<int64_t>(h) * a.Lq + q0 + t * kTile + row) * kD;
#pragma unroll
                for (int c4 = 0; c4 < kD / 32; ++c4) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(to + static_cast<uint32_t>(c4 * 32), r);
                    tmem_ld_wait();
                    uint32_t w[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e)
                        w[e] = pack2_bf16(__uint_as_float(r[2 * e]) * inv, __uint_as_float(r[2 * e + 1]) * inv);
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
    }

    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    if (warp == 1) tmem_dealloc(tmem, kTmemColsA);
}

// O rows of the split units from their parts: with m_p, l_p and the
// unnormalised O_p of part p (each against its own reference m_p),
// O = sum_p 2^(m_p - M) O_p / sum_p 2^(m_p - M) l_p for M = max_p m_p.  One
// warp per row, four columns per lane.
constexpr int kCombineRows = 8;  // rows (warps) per CTA

__global__ void __launch_bounds__(kCombineRows * 32)
    attention_combine_kernel(const float* __restrict__ o_part, const float2* __restrict__ ml_part, int Lq,
                             int unit0, int splits, uint16_t* __restrict__ o) {
    pdl_wait_primary();  // the parts come from the previous kernel
    const int lane = threadIdx.x & 31;
    const int r = static_cast<int>(blockIdx.x) * kCombineRows + (threadIdx.x >> 5);  // row among the split units
    const int u = r / (kQTiles * kTile);     // split unit, 0-based
    const int rr = r - u * (kQTiles * kTile);  // row within the unit's query-tile pair
    const int pairs = (Lq / kTile + kQTiles - 1) / kQTiles;
    const int unit = unit0 + u;
    const int h = unit / pairs;
    const int q0 = (unit - h * pairs) * kQTiles * kTile;
    if (rr >= min(kQTiles, (Lq - q0) / kTile) * kTile) return;  // past the unit's last query tile
    const int q = q0 + rr;
    const int64_t slot0 = static_cast<int64_t>(u) * splits;
    float M = -INFINITY;
    for (int p = 0; p < splits; ++p) M = fmaxf(M, ml_part[(slot0 + p) * (kQTiles * kTile) + rr].x);
    float L = 0.0f;
    float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int p = 0; p < splits; ++p) {
        const int64_t sr = (slot0 + p) * (kQTiles * kTile) + rr;
        const float2 ml = ml_part[sr];
        const float w = ex2_approx(ml.x - M);
        L = fmaf(w, ml.y, L);
        const float4 v = reinterpret_cast<const float4*>(o_part + sr * kD)[lane];
        acc.x = fmaf(w, v.x, acc.x);
        acc.y = fmaf(w, v.y, acc.y);
        acc.z = fmaf(w, v.z, acc.z);
        acc.w = fmaf(w, v.w, acc.w);
    }
    const float inv = 1.0f / L;
    uint2 out;
    out.x = pack2_bf16(acc.x * inv, acc.y * inv);
    out.y = pack2_bf16(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(o + (static_cast<int64_t>(h) * Lq + q) * kD)[lane] = out;
}

// V [h][key][d] -> V^T [h][d][key], bf16.  Each thread moves one block of
// 8 keys x 8 d through registers: 8 16-byte loads (one per key row), 32 byte
// permutes, 8 16-byte stores (one per d row).  A warp covers 32 keys x 64 d:
// 8 lanes read 128 contiguous bytes of a key row and 4 lanes write 64
// contiguous bytes of a d row, so every access fills whole 32-byte sectors.
constexpr int kTransposeThreads = 256;

__global__ void __launch_bounds__(kTransposeThreads)
    transpose_kernel(const uint16_t* __restrict__ v, uint16_t* __restrict__ vt, int L) {
    const int h = blockIdx.y;
    const int w = (blockIdx.x * kTransposeThreads + threadIdx.x) >> 5;  // warp within the head
    const int lane = threadIdx.x & 31;
    const int key0 = (w >> 1) * 32 + (lane >> 3) * 8;
    const int d0 = (w & 1) * 64 + (lane & 7) * 8;
    if (key0 >= L) return;
    const uint4* src = reinterpret_cast<const uint4*>(v + (static_cast<int64_t>(h) * L + key0) * kD + d0);
    uint4 r[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) r[i] = __ldg(src + i * (kD / 8));
    auto word = [](const uint4& q, int k) { return k == 0 ? q.x : k == 1 ? q.y : k == 2 ? q.z : q.w; };
#pragma unroll
    for (int j = 0; j < 8; ++j) {  // d0 + j: keys key0 .. key0 + 7, pairs (2k, 2k + 1) per word
        const uint32_t sel = (j & 1) ? 0x7632u : 0x5410u;
        uint4 o;
        o.x = __byte_perm(word(r[0], j >> 1), word(r[1], j >> 1), sel);
        o.y = __byte_perm(word(r[2], j >> 1), word(r[3], j >> 1), sel);
        o.z = __byte_perm(word(r[4], j >> 1), word(r[5], j >> 1), sel);
        o.w = __byte_perm(word(r[6], j >> 1), word(r[7], j >> 1), sel);
        *reinterpret_cast<uint4*>(vt + (static_cast<int64_t>(h) * kD + d0 + j) * L + key0) = o;
    }
}

}  // namespace

AttnSplit attention_split_plan(int H, int Lq, int Lk, int num_sms) {
    AttnSplit sp;
    sp.units = H * ((Lq / kTile + kQTiles - 1) / kQTiles);
    sp.main = sp.units;
    if (num_sms <= 0) return sp;
    const int tail = sp.units % num_sms;
    const int s = min(num_sms / max(tail, 1), (Lk / kTile) / 2);  // at least two key tiles per part
    if (tail == 0 || s < 2) return sp;
    sp.main = sp.units - tail;
    sp.tail = tail;
    sp.splits = s;
    return sp;
}

size_t attention_split_bytes(int slots) {
    return static_cast<size_t>(slots) * (kQTiles * kTile) * (kD * sizeof(float) + sizeof(float2));
}

cudaError_t launch_attention(const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vtmap, int H,
                             int Lq, int Lk, const float* s_q, const float* s_k, float scale_log2, uint16_t* o,
                             uint64_t limit_ns, unsigned int* err, bool pdl, cudaStream_t stream,
                             const AttnSplit& sp, void* part) {
    cudaError_t e;
    int set = 0;
    if (!launch_figure_get(reinterpret_cast<const void*>(attention_kernel), kThreadsA, kSmemA, &set)) {
        e = cudaFuncSetAttribute(attention_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemA);
        if (e != cudaSuccess) return e;
        launch_figure_put(reinterpret_cast<const void*>(attention_kernel), kThreadsA, kSmemA, 1);
    }
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
    a.unit0 = 0;
    a.splits = 1;
    a.o_part = nullptr;
    a.ml_part = nullptr;
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(kThreadsA);
    cfg.dynamicSmemBytes = kSmemA;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    const bool split = sp.splits > 1 && part != nullptr;
    const int main_units = split ? sp.main : sp.units;
    if (main_units > 0) {
        cfg.gridDim = dim3(static_cast<unsigned>(main_units));
        e = cudaLaunchKernelEx(&cfg, attention_kernel, qmap, kmap, vtmap, a);
        if (e != cudaSuccess) return e;
    }
    if (split) {
        // the units of the last, partly filled wave: their keys spread over all SMs
        const int slots = sp.tail * sp.splits;
        a.unit0 = sp.main;
        a.splits = sp.splits;
        a.o_part = static_cast<float*>(part);
        a.ml_part = reinterpret_cast<float2*>(static_cast<uint8_t*>(part) +
                                              static_cast<size_t>(slots) * (kQTiles * kTile) * kD * sizeof(float));
        cfg.gridDim = dim3(static_cast<unsigned>(slots));
        cfg.numAttrs = (main_units > 0 || pdl) ? 1 : 0;  // after the main launch (or the producers of Q, K, V^T)
        e = cudaLaunchKernelEx(&cfg, attention_kernel, qmap, kmap, vtmap, a);
        if (e != cudaSuccess) return e;
        cudaLaunchConfig_t cc = {};
        cc.gridDim = dim3(static_cast<unsigned>(sp.tail * kQTiles * kTile / kCombineRows));
        cc.blockDim = dim3(kCombineRows * 32);
        cc.stream = stream;
        cc.attrs = attr;
        cc.numAttrs = 1;
        e = cudaLaunchKernelEx(&cc, attention_combine_kernel, static_cast<const float*>(a.o_part),
                               static_cast<const float2*>(a.ml_part), Lq, sp.main, sp.splits, o);
        if (e != cudaSuccess) return e;
    }
    return cudaGetLastError();
}

cudaError_t launch_transpose_v(const uint16_t* v, uint16_t* vt, int H, int L, cudaStream_t stream) {
    // two warps (one per 64-d half) per 32 keys
    const int warps = (L + 31) / 32 * 2;
    const int blocks = (warps * 32 + kTransposeThreads - 1) / kTransposeThreads;
    transpose_kernel<<<dim3(static_cast<unsigned>(blocks), static_cast<unsigned>(H)), kTransposeThreads, 0, stream>>>(
        v, vt, L);
    return cudaGetLastError();
}

}  // namespace convrot
