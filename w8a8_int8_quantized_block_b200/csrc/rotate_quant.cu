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
// Design (B200): one CTA owns `rows_per_cta` rows.  A single TMA load brings
// the rows into shared memory with 128-byte swizzling, so every thread's
// 16-byte reads are bank-conflict free.  Each thread holds 32 consecutive
// elements in registers: the first five butterfly stages (h = 1..16) run in
// registers and the last two (h = 32, 64) by shuffles with lanes t^1 and t^2.
// The row's absmax is reduced by shuffles (and shared memory when a row spans
// several warps), then each thread writes its 32 codes as one 32-byte store.
#include <cuda_bf16.h>

#include "kernels.h"
#include "ptx.cuh"

namespace convrot {

namespace {

constexpr int kPerThread = 32;  // elements each thread owns

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
    const uint32_t a = smem_u32(p);
    return p + ((1024u - (a & 1023u)) & 1023u);
}

// Load this thread's 32 elements from the swizzled stage into registers.
// `R0` is the index of the 128-byte shared row holding element 0 of the
// thread's input row.
template <typename Tin>
__device__ __forceinline__ void load_row_piece(const uint8_t* stage, int R0, int t, float (&v)[kPerThread]) {
    if constexpr (sizeof(Tin) == 2) {
        // 32 bf16 = 64 bytes = half of a 128-byte row: row t/2, chunks 4*(t&1) .. +3
        const int R = R0 + (t >> 1);
        const int c0 = (t & 1) * 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint4 w = *reinterpret_cast<const uint4*>(stage + R * 128 + (((c0 + j) ^ (R & 7)) << 4));
            const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                v[8 * j + 2 * i] = __uint_as_float(u[i] << 16);
                v[8 * j + 2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
            }
        }
    } else {
        // 32 f32 = one whole 128-byte row: row t, chunks 0..7
        const int R = R0 + t;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 w = *reinterpret_cast<const float4*>(stage + R * 128 + ((j ^ (R & 7)) << 4));
            v[4 * j + 0] = w.x;
            v[4 * j + 1] = w.y;
            v[4 * j + 2] = w.z;
            v[4 * j + 3] = w.w;
        }
    }
}

// Stages h = 1, 2, 4, 8, 16 of the 128-point transform, on the thread's
// 32 consecutive elements.  Each butterfly (u, w) -> (u + w, u - w).
__device__ __forceinline__ void fwht_in_registers(float (&v)[kPerThread]) {
#pragma unroll
    for (int h = 1; h < kPerThread; h <<= 1) {
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) {
            if ((e & h) == 0) {
                const float u = v[e];
                const float w = v[e + h];
                v[e] = __fadd_rn(u, w);
                v[e + h] = __fsub_rn(u, w);
            }
        }
    }
}

// Stage across lanes: the partner lane (lane ^ sh) holds the elements `sh*32`
// positions away.  The lower-index side keeps u + w, the upper side u - w,
// where u is always the lower-index element.
__device__ __forceinline__ void fwht_across_lanes(float (&v)[kPerThread], int sh, bool upper) {
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) {
        const float p = __shfl_xor_sync(0xFFFFFFFFu, v[e], sh);
        v[e] = upper ? __fsub_rn(p, v[e]) : __fadd_rn(v[e], p);
    }
}

template <typename Tin, int BLOCK>
__global__ void __launch_bounds__(1024) rotate_quant_kernel(const __grid_constant__ CUtensorMap xmap, int64_t M,
                                                            int K, int tpr, int tpr_pad, int rows_per_cta,
                                                            int rows128, int box1, int nbox, int8_t* __restrict__ q,
                                                            int64_t ldq, float* __restrict__ s,
                                                            uint64_t limit_ns, unsigned int* err) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ uint64_t bar;
    __shared__ float red[32];
    __shared__ int abort_flag;
    uint8_t* stage = align1024(smem_raw);

    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int64_t row0 = static_cast<int64_t>(blockIdx.x) * rows_per_cta;
    const int rloc = tid / tpr_pad;
    const int t = tid - rloc * tpr_pad;

    if (tid == 0) {
        abort_flag = 0;
        mbar_init(&bar, 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (tid == 0) {
        // Full boxes are credited even where they run past the tensor (zero fill).
        const uint32_t bytes = static_cast<uint32_t>(nbox) * box1 * 128u * rows_per_cta;
        mbar_arrive_expect_tx(&bar, bytes);
        for (int b = 0; b < nbox; ++b)
            tma_load_3d(stage + static_cast<size_t>(b) * box1 * 128, &xmap, &bar, 0, b * box1,
                        static_cast<int>(row0));
        if (!mbar_wait_bounded(&bar, 0, limit_ns, kErrTimeoutLoad, err)) abort_flag = 1;
    }
    __syncthreads();
    if (abort_flag) return;  // uniform across the CTA

    float v[kPerThread];
    if (t < tpr) {
        load_row_piece<Tin>(stage, rloc * rows128, t, v);
    } else {
#pragma unroll
        for (int e = 0; e < kPerThread; ++e) v[e] = 0.0f;
    }

    if constexpr (BLOCK == 128) {
        fwht_in_registers(v);
        fwht_across_lanes(v, 1, (t & 1) != 0);  // h = 32
        fwht_across_lanes(v, 2, (t & 2) != 0);  // h = 64
    }

    float amax = 0.0f;
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) amax = fmaxf(amax, fabsf(v[e]));

    if (tpr_pad <= 32) {
        for (int o = tpr_pad >> 1; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    } else {
        // one row per CTA: warp maxima through shared memory
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        if (lane == 0) red[warp] = amax;
        __syncthreads();
        const int nw = tpr_pad >> 5;
        amax = red[0];
        for (int i = 1; i < nw; ++i) amax = fmaxf(amax, red[i]);
    }

    const int64_t row = row0 + rloc;
    if (row >= M || t >= tpr) return;

    const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    uint32_t packed[8];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
        uint32_t word = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            int c = __float2int_rn(__fmul_rn(v[4 * w + b], inv));
            c = max(-127, min(127, c));
            word |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * b);
        }
        packed[w] = word;
    }
    int8_t* dst = q + row * ldq + static_cast<int64_t>(t) * kPerThread;
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(packed[0]),
                 "r"(packed[1]), "r"(packed[2]), "r"(packed[3]), "r"(packed[4]), "r"(packed[5]), "r"(packed[6]),
                 "r"(packed[7])
                 : "memory");
    if (t == 0) s[row] = __fdiv_rn(amax, 127.0f);
}

template <typename Tin, int BLOCK>
cudaError_t launch_typed(const CUtensorMap& xmap, int64_t M, int64_t K, const RqGeometry& g, int8_t* q,
                         int64_t ldq, float* s, uint64_t limit_ns, unsigned int* err, cudaStream_t stream) {
    auto kern = rotate_quant_kernel<Tin, BLOCK>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(g.smem_bytes));
    if (e != cudaSuccess) return e;
    const int64_t grid = (M + g.rows_per_cta - 1) / g.rows_per_cta;
    kern<<<static_cast<unsigned>(grid), g.threads, g.smem_bytes, stream>>>(
        xmap, M, static_cast<int>(K), g.tpr, g.tpr_pad, g.rows_per_cta, g.rows128, g.box1, g.nbox, q, ldq, s,
        limit_ns, err);
    return cudaGetLastError();
}

int next_pow2(int v) {
    int p = 1;
    while (p < v) p <<= 1;
    return p;
}

}  // namespace

bool rq_geometry(int64_t K, int in_elem_bytes, RqGeometry* g) {
    if (K <= 0 || K % 64 != 0 || K > 32768) return false;
    if ((K * in_elem_bytes) % 128 != 0) return false;
    g->tpr = static_cast<int>(K / kPerThread);
    if (g->tpr <= 32) {
        g->tpr_pad = next_pow2(g->tpr);
        g->rows_per_cta = 256 / g->tpr_pad;
    } else {
        g->tpr_pad = (g->tpr + 31) / 32 * 32;
        g->rows_per_cta = 1;
    }
    g->threads = g->tpr_pad * g->rows_per_cta;
    g->rows128 = static_cast<int>(K * in_elem_bytes / 128);
    if (g->rows_per_cta > 1) {
        g->nbox = 1;
        g->box1 = g->rows128;  // <= 32 here
    } else {
        g->nbox = (g->rows128 + 255) / 256;
        int per = (g->rows128 + g->nbox - 1) / g->nbox;
        g->box1 = (per + 7) / 8 * 8;  // keep every box 1024-byte aligned
        if (g->box1 > 256) return false;
    }
    const size_t stage = static_cast<size_t>(g->nbox) * g->box1 * 128 * g->rows_per_cta;
    g->smem_bytes = stage + 1024;  // slack for 1024-byte alignment
    return g->smem_bytes <= 200 * 1024;
}

cudaError_t launch_rotate_quant(const CUtensorMap& xmap, int in_elem_bytes, int block, int64_t M, int64_t K,
                                const RqGeometry& g, int8_t* q, int64_t ldq, float* s, uint64_t limit_ns,
                                unsigned int* err, cudaStream_t stream) {
    const bool rot = block == 128;
    if (in_elem_bytes == 2)
        return rot ? launch_typed<__nv_bfloat16, 128>(xmap, M, K, g, q, ldq, s, limit_ns, err, stream)
                   : launch_typed<__nv_bfloat16, 0>(xmap, M, K, g, q, ldq, s, limit_ns, err, stream);
    return rot ? launch_typed<float, 128>(xmap, M, K, g, q, ldq, s, limit_ns, err, stream)
               : launch_typed<float, 0>(xmap, M, K, g, q, ldq, s, limit_ns, err, stream);
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
