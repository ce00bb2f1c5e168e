// rotate_quant.cu -- block-diagonal Hadamard rotation + rowwise symmetric int8
// quantisation, one pass over HBM.
//
// What it computes (activations: "Rowwise INT8 Quantize" behind "ConvRot",
// MiniMax-H3-Rung-Omega README, "Technical Architecture Overview", item 2;
// the block-diagonal Hadamard rotation: lehuy.net "Nen mo hinh video khuech
// tan 31B xuong 14B", section "Cach nen hoat dong"; weights: "per-output F32
// scales", "MiniMax H3 - pruned INT8 ConvRot - input-major", section
// "Input-major checkpoint"):
//
//   z = blockdiag(H_128) x            (fp32 butterflies, stages 1, 2, ..., 64)
//   amax = max |z|;  s = amax / 127;  q = clamp(rne(z * (127 / amax)), +-127)
//
// Design (B200).  A persistent CTA walks over groups of rows; each group is
// brought into one slot of a two-slot shared-memory ring by TMA (128-byte
// swizzle, so the 16-byte reads below are bank-conflict free) while the
// previous group is computed.  Each thread owns 64 consecutive elements of a
// row (half a Hadamard block), held as 32 packed f32x2 register pairs
// (element j with element j+32):
//   - butterfly stages h = 1, 2, 4, 8, 16 are packed add/sub (two lanes of
//     work per instruction), stage h = 32 is inside each pair;
//   - stage h = 64 pairs lanes t and t^1: a shuffle brings the partner's
//     values and one packed FMA with a +-1 sign computes self + partner on
//     the lower side and partner - self on the upper side, each rounded once
//     exactly like the add or subtract it replaces;
//   - the row absmax is reduced with shuffles when a row fits in a warp;
//     longer rows are packed back to back (no padding threads between them,
//     so a 5376-element row takes 84 threads and three rows fill eight
//     warps): a max-reduction over each warp's segment of a row, then one
//     64-bit shared-memory atomicMax per segment, tagged with the group's
//     iteration so that no reset between groups is needed;
//   - codes: v = z * (127/amax) (packed multiply, rounded), then a packed
//     fma(v, 1, 1.5*2^23) rounds v half-to-even to an integer whose low byte
//     is the code (|v| <= 127*(1+2^-24) < 127.5, so no clamp can bind); byte
//     permutes pack four codes per word and two 32-byte stores write the
//     thread's 64 codes.  The product is rounded on its own before the
//     integer rounding, as the definition has it (see quantize_store).
// The arithmetic is therefore the same sequence of IEEE single-precision
// operations as the plain definition, in the same order.
#include <cuda_bf16.h>

#include <algorithm>

#include "kernels.h"
#include "ptx.cuh"
#include "quant_core.cuh"

namespace convrot {

namespace {

using namespace qcore;

constexpr int kMaxThreads = 512;
// 80 registers and two ring slots let eight 96-thread CTAs share an SM (the
// kernel is latency-bound; more rows in flight beat more registers per thread).
#ifndef CONVROT_RQ_MAXREG
#define CONVROT_RQ_MAXREG 80
#endif
// The activation prologues (erfc / exp per element next to 64 live values)
// need more registers than 80; they are compute-heavy, so fewer resident
// CTAs cost them little.
#ifndef CONVROT_RQ_MAXREG_ACT
#define CONVROT_RQ_MAXREG_ACT 128
#endif
#ifndef CONVROT_RQ_STAGES
#define CONVROT_RQ_STAGES 2  // ring slots (row groups in flight) per CTA
#endif
#ifndef CONVROT_RQ_MAX_IDLE_PCT
#define CONVROT_RQ_MAX_IDLE_PCT 2  // pack long rows until at most this share of threads is idle
#endif
constexpr int kMaxStages = 3;
constexpr int kRqSmemBudget = 200 * 1024;  // the largest ring of row slots a geometry may ask for
constexpr int kRqSmemOptIn = 226 * 1024;   // ring + an activation's table: the most any launch asks for
constexpr int kMaxLongRows = 8;  // rows per group when rows span several warps

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

template <typename Tin, int KIND, int ACT>
__global__ void __maxnreg__(ACT == kActNone ? CONVROT_RQ_MAXREG : CONVROT_RQ_MAXREG_ACT) rotate_quant_kernel(const __grid_constant__ CUtensorMap xmap, int64_t M,
                                                            int tpr, int tpr_pad, int rows_per_cta, int rows128,
                                                            int box1, int nbox, int nstage, int64_t num_groups,
                                                            int8_t* __restrict__ q, int64_t ldq,
                                                            float* __restrict__ s, uint64_t limit_ns,
                                                            unsigned int* err) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t full[kMaxStages];
    // Row maxima of long rows: (iteration << 32) | bits of the max, double-buffered.
    __shared__ unsigned long long rowmax[2][kMaxLongRows];
    __shared__ int abort_flag;
    uint8_t* ring = align1024(smem_raw);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int rloc = tid / tpr_pad;
    const int t = tid - rloc * tpr_pad;
    const bool active = rloc < rows_per_cta && t < tpr;  // long rows: threads past the last row idle
    // Long rows: the row this lane reduces into (idle lanes join the last
    // row) and the first lane of the warp's second row segment (32: none).
    const bool long_rows = tpr_pad > 32;
    const int rr = rloc < rows_per_cta ? rloc : rows_per_cta - 1;
    int split = 32;
    if (long_rows) {
        const int r0 = min((warp * 32) / tpr, rows_per_cta - 1);
        if (r0 < rows_per_cta - 1) split = min((r0 + 1) * tpr - warp * 32, 32);
    }
    const uint32_t lo_mask = split >= 32 ? 0xFFFFFFFFu : ((1u << split) - 1u);
    const uint32_t slot_bytes = static_cast<uint32_t>(nbox) * box1 * 128u * rows_per_cta;
    const int row_pitch = nbox * box1;  // 128-byte shared rows between consecutive input rows of a group
    (void)rows128;

    const uint64_t policy = l2_policy_evict_first();  // every input byte is read once
    auto issue = [&](int64_t g, int slot) {
        // Full boxes are credited even where they run past the tensor (zero fill).
        mbar_arrive_expect_tx(&full[slot], slot_bytes);
        uint8_t* dst = ring + static_cast<size_t>(slot) * slot_bytes;
        for (int b = 0; b < nbox; ++b)
            tma_load_3d_hint(dst + static_cast<size_t>(b) * box1 * 128, &xmap, &full[slot], 0, b * box1,
                             static_cast<int>(g * rows_per_cta), policy);
    };

    // The activation's table follows the ring (act_table_bytes(ACT) bytes).
    void* act_tab = ring + static_cast<size_t>(nstage) * slot_bytes;
    if constexpr (ACT != kActNone) act_table_fill<ACT>(act_tab, tid, blockDim.x);
    if (tid < 2 * kMaxLongRows) rowmax[tid / kMaxLongRows][tid % kMaxLongRows] = 0ull;
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

    int it = 0;
    for (int64_t g = blockIdx.x; g < num_groups; g += gridDim.x, ++it) {
        const int slot = it % nstage;
        const uint32_t parity = static_cast<uint32_t>(it / nstage) & 1u;
        // Every thread waits for the slot itself; a time-out is acted on after
        // the next CTA barrier so that all threads leave the loop together.
        if (!mbar_wait_bounded(&full[slot], parity, limit_ns, kErrTimeoutLoad, err)) abort_flag = 1;

        uint64_t P[kPairs];
        if (active) {
            const uint8_t* sl = ring + static_cast<size_t>(slot) * slot_bytes;
            load_pairs<Tin>(sl, rloc * row_pitch, t, P);
            if constexpr (ACT == kActGelu) gelu_pairs(P, static_cast<const float*>(act_tab));
            if constexpr (ACT == kActSwiglu)  // u: the row's second half
                swiglu_pairs(P, sl, rloc * row_pitch + tpr + t, static_cast<const double*>(act_tab));
        } else {
#pragma unroll
            for (int j = 0; j < kPairs; ++j) P[j] = 0ull;
        }

        rotate_piece<KIND>(P, t);
        float amax = piece_absmax(P);
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
            quantize_store<true>(P, inv, q + row * ldq + static_cast<int64_t>(t) * kPerThread);
            if (t == 0) s[row] = __fdiv_rn(amax, 127.0f);
        }
    }
}

template <typename Tin, int KIND, int ACT>
cudaError_t launch_typed(const CUtensorMap& xmap, int64_t M, const RqGeometry& g, int8_t* q, int64_t ldq,
                         float* s, uint64_t limit_ns, unsigned int* err, int num_sms, cudaStream_t stream) {
    auto kern = rotate_quant_kernel<Tin, KIND, ACT>;
    const size_t smem = g.smem_bytes + static_cast<size_t>(act_table_bytes(ACT));  // ring (+ the activation's table)
    if (smem > static_cast<size_t>(kRqSmemOptIn)) return cudaErrorInvalidValue;
    int per_sm = 0;
    if (!launch_figure_get(reinterpret_cast<const void*>(kern), g.threads, smem, &per_sm)) {
        // The opt-in is the most any geometry may ask for, so that it never
        // shrinks below what an earlier launch of this kernel needed.
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kRqSmemOptIn);
        if (e != cudaSuccess) return e;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, g.threads, smem);
        if (e != cudaSuccess) return e;
        if (per_sm < 1) return cudaErrorInvalidConfiguration;
        launch_figure_put(reinterpret_cast<const void*>(kern), g.threads, smem, per_sm);
    }
    const int64_t groups = (M + g.rows_per_cta - 1) / g.rows_per_cta;
    const int64_t cap = static_cast<int64_t>(per_sm) * num_sms;
    const int64_t grid = groups < cap ? groups : cap;
    kern<<<static_cast<unsigned>(grid), g.threads, smem, stream>>>(
        xmap, M, g.tpr, g.tpr_pad, g.rows_per_cta, g.rows128, g.box1, g.nbox, g.nstage, groups, q, ldq, s, limit_ns,
        err);
    return cudaGetLastError();
}

int next_pow2(int v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

}  // namespace

bool rq_geometry(int64_t K, int64_t row_elems, int in_elem_bytes, RqGeometry* g, int act) {
    if (K <= 0 || K % 64 != 0 || K > 32768) return false;
    if (row_elems != K && row_elems != 2 * K) return false;
    g->tpr = static_cast<int>(K / kPerThread);
    g->rows128 = static_cast<int>(row_elems * in_elem_bytes / 128);
    if (g->tpr <= 32) {
        // Short rows: a power-of-two lane group per row, 256 threads per CTA.
        g->tpr_pad = next_pow2(g->tpr);
        g->rows_per_cta = 256 / g->tpr_pad;
        g->nbox = 1;
        g->box1 = g->rows128;  // <= 32; the slot size is a multiple of 1024 bytes
        g->threads = g->tpr_pad * g->rows_per_cta;
    } else {
        // Long rows: packed back to back, tpr threads each (tpr is even, so
        // the lane pairs of the last butterfly stage never straddle rows);
        // boxes padded to 8 rows of 128 bytes so every box and slot starts on
        // a 1024-byte boundary.
        g->tpr_pad = g->tpr;
        g->nbox = (g->rows128 + 255) / 256;
        const int per = (g->rows128 + g->nbox - 1) / g->nbox;
        g->box1 = (per + 7) / 8 * 8;
        if (g->box1 > 256) return false;
        // Rows per group: one when a row needs several boxes (the slot holds
        // one row's boxes back to back), else the fewest rows that leave at
        // most CONVROT_RQ_MAX_IDLE_PCT of the CTA's threads idle (or, failing
        // that, the fewest idle threads).
        auto round32 = [](int v) { return (v + 31) / 32 * 32; };
        g->rows_per_cta = 1;
        if (g->nbox == 1) {
            int best = 1;
            for (int r = 1; r <= kMaxLongRows && round32(r * g->tpr) <= kMaxThreads; ++r) {
                const int thr = round32(r * g->tpr);
                const int idle = thr - r * g->tpr;
                if (idle * 100 <= CONVROT_RQ_MAX_IDLE_PCT * thr) {
                    best = r;
                    break;
                }
                const int bthr = round32(best * g->tpr);
                if (idle * bthr < (bthr - best * g->tpr) * thr) best = r;
            }
            g->rows_per_cta = best;
        }
        g->threads = round32(g->rows_per_cta * g->tpr);
    }
    const size_t slot = static_cast<size_t>(g->nbox) * g->box1 * 128 * g->rows_per_cta;
    if (slot % 1024 != 0) return false;  // slots must stay 1024-byte aligned for the swizzle
    // the ring's share: an activation kernel also keeps its table in shared memory
    const size_t budget = std::min<size_t>(kRqSmemBudget, kRqSmemOptIn - act_table_bytes(act));
    g->nstage = CONVROT_RQ_STAGES;
    while (g->nstage > 1 && slot * g->nstage + 1024 > budget) --g->nstage;
    if (g->nstage > 2 && slot * g->nstage > 96 * 1024) g->nstage = 2;  // leave room for a second CTA
    g->smem_bytes = slot * g->nstage + 1024;  // slack for 1024-byte alignment
    return g->smem_bytes <= budget;
}

template <typename Tin, int ACT>
cudaError_t launch_kind(const CUtensorMap& xmap, int kind, int64_t M, const RqGeometry& g, int8_t* q, int64_t ldq,
                        float* s, uint64_t limit_ns, unsigned int* err, int num_sms, cudaStream_t stream) {
    switch (kind) {
        case kRotNone: return launch_typed<Tin, kRotNone, ACT>(xmap, M, g, q, ldq, s, limit_ns, err, num_sms, stream);
        case kRotSyl64: return launch_typed<Tin, kRotSyl64, ACT>(xmap, M, g, q, ldq, s, limit_ns, err, num_sms, stream);
        case kRotSyl128: return launch_typed<Tin, kRotSyl128, ACT>(xmap, M, g, q, ldq, s, limit_ns, err, num_sms, stream);
        case kRotSyl256: return launch_typed<Tin, kRotSyl256, ACT>(xmap, M, g, q, ldq, s, limit_ns, err, num_sms, stream);
        case kRotReg16: return launch_typed<Tin, kRotReg16, ACT>(xmap, M, g, q, ldq, s, limit_ns, err, num_sms, stream);
        case kRotReg64: return launch_typed<Tin, kRotReg64, ACT>(xmap, M, g, q, ldq, s, limit_ns, err, num_sms, stream);
        case kRotReg256: return launch_typed<Tin, kRotReg256, ACT>(xmap, M, g, q, ldq, s, limit_ns, err, num_sms, stream);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_rotate_quant(const CUtensorMap& xmap, int in_elem_bytes, int kind, int act, int64_t M, int64_t K,
                                const RqGeometry& g, int8_t* q, int64_t ldq, float* s, uint64_t limit_ns,
                                unsigned int* err, int num_sms, cudaStream_t stream) {
    (void)K;
    if (in_elem_bytes == 2) {
        switch (act) {
            case kActNone:
                return launch_kind<__nv_bfloat16, kActNone>(xmap, kind, M, g, q, ldq, s, limit_ns, err, num_sms, stream);
            case kActGelu:
                return launch_kind<__nv_bfloat16, kActGelu>(xmap, kind, M, g, q, ldq, s, limit_ns, err, num_sms, stream);
            case kActSwiglu:
                return launch_kind<__nv_bfloat16, kActSwiglu>(xmap, kind, M, g, q, ldq, s, limit_ns, err, num_sms,
                                                              stream);
            default:
                return cudaErrorInvalidValue;
        }
    }
    if (act != kActNone) return cudaErrorInvalidValue;  // weights take no activation
    return launch_kind<float, kActNone>(xmap, kind, M, g, q, ldq, s, limit_ns, err, num_sms, stream);
}

namespace {
__global__ void wait_selftest_kernel(uint64_t limit_ns, unsigned int* err) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        // Nothing ever arrives: the bounded wait has to give up.
        (void)mbar_wait_bounded(&bar, 0, limit_ns, kErrTimeoutSelfTest, err);
    }
}
}  // namespace

cudaError_t launch_wait_selftest(uint64_t limit_ns, unsigned int* err, cudaStream_t stream) {
    wait_selftest_kernel<<<1, 32, 0, stream>>>(limit_ns, err);
    return cudaGetLastError();
}

}  // namespace convrot
