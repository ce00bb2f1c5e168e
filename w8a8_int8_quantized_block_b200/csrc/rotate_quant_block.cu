// rotate_quant_block.cu -- the activation quantiser with one whole Hadamard
// block per thread: the same rotation and rowwise int8 quantisation as
// rotate_quant.cu (block-diagonal Hadamard rotation: lehuy.net "Nen mo hinh
// video khuech tan 31B xuong 14B", section "Cach nen hoat dong"; "Rowwise
// INT8 Quantize": MiniMax-H3-Rung-Omega README, "Technical Architecture
// Overview", item 2), for bf16 rows with the 128-point Sylvester rotation or
// none:
//
//   z = blockdiag(H_128) x            (fp32 butterflies, stages 1, 2, ..., 64)
//   amax = max |z|;  s = amax / 127;  q = rne(z * (127 / amax))
//
// Why a second kernel.  The quantiser is issue-bound, not DRAM-bound: with 64
// elements per thread (half a block) the last butterfly stage crosses lanes,
// 64 shuffles and 32 packed FMAs per thread, and the per-row overhead (the
// division, addressing, the barrier) is spread over 64 elements only.  Here a
// thread owns all 128 elements of its block as 64 packed f32x2 pairs
// P[j] = (element j, element j + 64):
//   - stages h = 1 .. 32 are packed add/sub on pairs (j, j + h), both halves
//     of the block at once; stage h = 64 is inside each pair;
//   - no shuffle touches the data; the row maximum is reduced as in
//     rotate_quant.cu (shuffles for short rows; for rows longer than a warp,
//     rows packed back to back, a max-reduction per warp segment and one
//     tagged 64-bit shared atomicMax per segment);
//   - codes: packed multiply by 127/amax, then a packed fma(v, 1, 1.5*2^23)
//     that rounds v half-to-even to an integer whose low byte is the code,
//     byte permutes, four 32-byte stores.
// Every butterfly is the same IEEE single-precision operation on the same
// operands as in the canonical stage order, so codes and scales equal those
// of rotate_quant.cu bit for bit.
//
// Shared memory.  Rows arrive by TMA through a 4-D view of x,
// {64 elements, K/128 blocks, 2 halves, rows}, whose box puts the first
// halves of a row's blocks in consecutive 128-byte shared rows, then the
// second halves.  Thread t of a row reads 128-byte rows t and K/128 + t, so the
// eight threads of each 16-byte read phase see eight different rows and, with
// the 128-byte swizzle, eight different bank groups (blocks stored back to
// back would put a thread's two halves in rows 2t and 2t + 1 and make every
// read a two-way bank conflict).
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"
#include "quant_core.cuh"

namespace convrot {

namespace {

using qcore::add2;
using qcore::fma2;
using qcore::mul2;
using qcore::pk;
using qcore::prmt;
using qcore::sub2;
using qcore::upk;

constexpr int kPerB = 128;           // elements per thread: one Hadamard block
constexpr int kPairsB = kPerB / 2;   // P[j] = (element j, element j + 64)
constexpr int kMaxThreadsB = 384;    // 168 registers per thread: at most 390 threads per SM
constexpr int kMaxRowsB = 8;         // rows per group when rows span several warps
constexpr int kMaxStagesB = 3;
constexpr int kSmemBudgetB = 200 * 1024;
#ifndef CONVROT_RQB_MAXREG
#define CONVROT_RQB_MAXREG 168
#endif

__device__ __forceinline__ uint8_t* align1024b(uint8_t* p) {
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

// bf16 element i (0..7) of a 16-byte chunk, widened exactly to f32.
__device__ __forceinline__ float bf16_elem(const uint4& v, int i) {
    const uint32_t w = (i >> 1) == 0 ? v.x : (i >> 1) == 1 ? v.y : (i >> 1) == 2 ? v.z : v.w;
    return __uint_as_float((i & 1) ? (w & 0xFFFF0000u) : (w << 16));
}

// The thread's block from the slot: first halves at 128-byte shared row Ra,
// second halves at Rb (chunk c of row R sits at chunk position c ^ (R & 7)).
__device__ __forceinline__ void load_block(const uint8_t* slot, int Ra, int Rb, uint64_t (&P)[kPairsB]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 a = *reinterpret_cast<const uint4*>(slot + Ra * 128 + ((c ^ (Ra & 7)) << 4));
        const uint4 b = *reinterpret_cast<const uint4*>(slot + Rb * 128 + ((c ^ (Rb & 7)) << 4));
#pragma unroll
        for (int i = 0; i < 8; ++i) P[8 * c + i] = pk(bf16_elem(a, i), bf16_elem(b, i));
    }
}

// Sylvester H_128 in the canonical order: stages h = 1 .. 32 on pairs
// (j, j + h) (packed: the block's two halves at once), then h = 64 inside
// each pair.  Butterfly (u, w) -> (u + w, u - w), u the lower index.
__device__ __forceinline__ void fwht_block(uint64_t (&P)[kPairsB]) {
#pragma unroll
    for (int h = 1; h < kPairsB; h <<= 1) {
#pragma unroll
        for (int j = 0; j < kPairsB; ++j) {
            if ((j & h) == 0) {
                const uint64_t u = P[j], w = P[j + h];
                P[j] = add2(u, w);
                P[j + h] = sub2(u, w);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kPairsB; ++j) {
        float u, w;
        upk(P[j], u, w);
        P[j] = pk(__fadd_rn(u, w), __fsub_rn(u, w));
    }
}

__device__ __forceinline__ float block_absmax(const uint64_t (&P)[kPairsB]) {
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < kPairsB; ++j) {
        float a, b;
        upk(P[j], a, b);
        amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
    }
    return amax;
}

// The 128 codes of the block: v = f32(z * inv), then fma(v, 1, 1.5 * 2^23)
// rounds v half-to-even to an integer (the f32 spacing there is 1) whose low
// byte is the code; the multiply and the rounding stay two separate
// roundings (written as a plain add, the pair would be fused into one FMA).
// |v| <= 127 (1 + 2^-24) < 127.5, so no clamp can bind.  Word i < 16 holds
// elements 4i .. 4i + 3 (low halves of P[4i .. 4i + 3]), word 16 + i the
// elements 64 + 4i .. (the high halves); four 32-byte stores at dst.
__device__ __forceinline__ void quantize_store_block(const uint64_t (&P)[kPairsB], float inv, int8_t* dst) {
    const uint64_t inv2 = pk(inv, inv);
    const uint64_t one2 = pk(1.0f, 1.0f);
    const uint64_t magic2 = pk(12582912.0f, 12582912.0f);  // 1.5 * 2^23
    uint32_t word[kPerB / 4];
#pragma unroll
    for (int i = 0; i < kPairsB / 4; ++i) {
        uint32_t lo[4], hi[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float a, b;
            upk(fma2(mul2(P[4 * i + k], inv2), one2, magic2), a, b);
            lo[k] = __float_as_uint(a);
            hi[k] = __float_as_uint(b);
        }
        word[i] = prmt(prmt(lo[0], lo[1], 0x0040u), prmt(lo[2], lo[3], 0x0040u), 0x5410u);
        word[kPairsB / 4 + i] = prmt(prmt(hi[0], hi[1], 0x0040u), prmt(hi[2], hi[3], 0x0040u), 0x5410u);
    }
#pragma unroll
    for (int i = 0; i < kPerB / 32; ++i)
        asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + 32 * i),
                     "r"(word[8 * i]), "r"(word[8 * i + 1]), "r"(word[8 * i + 2]), "r"(word[8 * i + 3]),
                     "r"(word[8 * i + 4]), "r"(word[8 * i + 5]), "r"(word[8 * i + 6]), "r"(word[8 * i + 7])
                     : "memory");
}

template <int KIND>
__global__ void __maxnreg__(CONVROT_RQB_MAXREG)
    rotate_quant_block_kernel(const __grid_constant__ CUtensorMap xmap, int64_t M, int tpr, int tpr_pad,
                              int rows_per_cta, int nb, int nstage, int64_t num_groups, int8_t* __restrict__ q,
                              int64_t ldq, float* __restrict__ s, uint64_t limit_ns, unsigned int* err) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full[kMaxStagesB];
    // Row maxima of long rows: (iteration << 32) | bits of the max, double-buffered.
    __shared__ unsigned long long rowmax[2][kMaxRowsB];
    __shared__ int abort_flag;
    uint8_t* ring = align1024b(smem_raw);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int rloc = tid / tpr_pad;
    const int t = tid - rloc * tpr_pad;
    const bool active = rloc < rows_per_cta && t < tpr;
    const bool long_rows = tpr_pad > 32;
    const int rr = rloc < rows_per_cta ? rloc : rows_per_cta - 1;
    int split = 32;  // long rows: the first lane of the warp's second row segment (32: none)
    if (long_rows) {
        const int r0 = min((warp * 32) / tpr, rows_per_cta - 1);
        if (r0 < rows_per_cta - 1) split = min((r0 + 1) * tpr - warp * 32, 32);
    }
    const uint32_t lo_mask = split >= 32 ? 0xFFFFFFFFu : ((1u << split) - 1u);
    const uint32_t row_bytes = static_cast<uint32_t>(nb) * 256u;
    const uint32_t slot_bytes = row_bytes * static_cast<uint32_t>(rows_per_cta);  // what one group's load brings
    const uint32_t slot_stride = (slot_bytes + 1023u) & ~1023u;  // slots start on 1024-byte boundaries (swizzle)

    const uint64_t policy = l2_policy_evict_first();  // every input byte is read once
    auto issue = [&](int64_t g, int slot) {
        // Full boxes are credited even where they run past the tensor (zero fill).
        mbar_arrive_expect_tx(&full[slot], slot_bytes);
        tma_load_4d_hint(ring + static_cast<size_t>(slot) * slot_stride, &xmap, &full[slot], 0, 0, 0,
                         static_cast<int>(g * rows_per_cta), policy);
    };

    if (tid < 2 * kMaxRowsB) rowmax[tid / kMaxRowsB][tid % kMaxRowsB] = 0ull;
    if (tid == 0) {
        abort_flag = 0;
        for (int i = 0; i < nstage; ++i) mbar_init(&full[i], 1);
        fence_mbar_init();
        for (int i = 0; i < nstage; ++i) {
            const int64_t g = blockIdx.x + static_cast<int64_t>(i) * gridDim.x;
            if (g < num_groups) issue(g, i);
        }
    }
    __syncthreads();

    const int Ra = rloc * 2 * nb + t;  // the thread's first halves, then its second halves nb rows on
    const int Rb = Ra + nb;
    int it = 0;
    for (int64_t g = blockIdx.x; g < num_groups; g += gridDim.x, ++it) {
        const int slot = it % nstage;
        const uint32_t parity = static_cast<uint32_t>(it / nstage) & 1u;
        // Every thread waits for the slot itself; a time-out is acted on after
        // the next CTA barrier so that all threads leave the loop together.
        if (!mbar_wait_bounded(&full[slot], parity, limit_ns, kErrTimeoutLoad, err)) abort_flag = 1;

        uint64_t P[kPairsB];
        if (active) {
            load_block(ring + static_cast<size_t>(slot) * slot_stride, Ra, Rb, P);
            if constexpr (KIND == kRotSyl128) fwht_block(P);
        } else {
#pragma unroll
            for (int j = 0; j < kPairsB; ++j) P[j] = 0ull;
        }
        float amax = block_absmax(P);
        if (!long_rows) {
            for (int o = tpr_pad >> 1; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        } else {
            // amax is a non-negative, non-NaN float (fmaxf from +0 drops NaNs),
            // so its bits order like the values.
            const uint32_t bits = __float_as_uint(amax);
            uint32_t m;
            if (lane < split) m = __reduce_max_sync(lo_mask, bits);
            else m = __reduce_max_sync(~lo_mask, bits);
            if (lane == 0 || lane == split)
                atomicMax(&rowmax[it & 1][rr], (static_cast<unsigned long long>(it) << 32) | m);
        }
        // The one CTA barrier per group: every thread has read the slot (so it
        // can be refilled) and has published its share of the row maximum.
        __syncthreads();
        if (abort_flag) break;  // uniform across the CTA
        if (tid == 0) {
            const int64_t gn = g + static_cast<int64_t>(nstage) * gridDim.x;
            if (gn < num_groups) {
                fence_proxy_async_smem();
                issue(gn, slot);
            }
        }
        // Every row's first segment wrote with this iteration's tag, which
        // beats whatever an earlier group left in this buffer.
        if (long_rows) amax = __uint_as_float(static_cast<uint32_t>(rowmax[it & 1][rr]));

        const int64_t row = g * rows_per_cta + rloc;
        if (row < M && active) {
            const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
            quantize_store_block(P, inv, q + row * ldq + static_cast<int64_t>(t) * kPerB);
            if (t == 0) s[row] = __fdiv_rn(amax, 127.0f);
        }
    }
}

int next_pow2_b(int v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

}  // namespace

bool rqb_geometry(int64_t K, RqbGeometry* g) {
    if (K <= 0 || K % kPerB != 0 || K > 32768) return false;
    g->tpr = static_cast<int>(K / kPerB);
    g->nb = g->tpr;  // Hadamard blocks per row (box extent, at most 256)
    auto round32 = [](int v) { return (v + 31) / 32 * 32; };
    if (g->tpr <= 32) {
        // Short rows: a power-of-two lane group per row, 128 threads per CTA.
        g->tpr_pad = next_pow2_b(g->tpr);
        g->rows_per_cta = 128 / g->tpr_pad;
        g->threads = 128;
    } else {
        // Long rows packed back to back: the fewest rows (at most kMaxRowsB,
        // within kMaxThreadsB threads) that leave at most 2% of the threads
        // idle, else the least idle share.
        g->tpr_pad = g->tpr;
        int best = 0;
        for (int r = 1; r <= kMaxRowsB && round32(r * g->tpr) <= kMaxThreadsB; ++r) {
            const int thr = round32(r * g->tpr);
            const int idle = thr - r * g->tpr;
            if (best == 0) best = r;
            if (idle * 100 <= 2 * thr) {
                best = r;
                break;
            }
            const int bthr = round32(best * g->tpr);
            if (idle * bthr < (bthr - best * g->tpr) * thr) best = r;
        }
        if (best == 0) return false;  // a row needs more threads than a CTA may have
        g->rows_per_cta = best;
        g->threads = round32(best * g->tpr);
    }
    if (g->rows_per_cta > 256) return false;  // box extent
    const size_t slot = (static_cast<size_t>(g->rows_per_cta) * static_cast<size_t>(g->nb) * 256 + 1023) / 1024 * 1024;
    g->nstage = 2;
    if (slot * 3 + 1024 <= 96 * 1024) g->nstage = 3;  // small slots: one more group in flight
    g->smem_bytes = slot * g->nstage + 1024;  // slack for 1024-byte alignment
    return g->smem_bytes <= static_cast<size_t>(kSmemBudgetB);
}

cudaError_t launch_rotate_quant_block(const CUtensorMap& xmap, int kind, int64_t M, const RqbGeometry& g, int8_t* q,
                                      int64_t ldq, float* s, uint64_t limit_ns, unsigned int* err, int num_sms,
                                      cudaStream_t stream) {
    if (kind != kRotSyl128 && kind != kRotNone) return cudaErrorInvalidValue;
    auto kern = kind == kRotSyl128 ? rotate_quant_block_kernel<kRotSyl128> : rotate_quant_block_kernel<kRotNone>;
    int per_sm = 0;
    if (!launch_figure_get(reinterpret_cast<const void*>(kern), g.threads, g.smem_bytes, &per_sm)) {
        // the opt-in is the largest ring any geometry asks for, so it never shrinks
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBudgetB);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, g.threads, g.smem_bytes);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        launch_figure_put(reinterpret_cast<const void*>(kern), g.threads, g.smem_bytes, per_sm);
    }
    const int64_t groups = (M + g.rows_per_cta - 1) / g.rows_per_cta;
    const int64_t cap = static_cast<int64_t>(per_sm) * num_sms;
    const int64_t grid = groups < cap ? groups : cap;
    kern<<<static_cast<unsigned>(grid), g.threads, g.smem_bytes, stream>>>(xmap, M, g.tpr, g.tpr_pad, g.rows_per_cta,
                                                                           g.nb, g.nstage, groups, q, ldq, s,
                                                                           limit_ns, err);
    return cudaGetLastError();
}

}  // namespace convrot
