// kernels.h -- host-side launchers of the sm_100a kernels (internal to the
// library; the public surface is include/convrot.h).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace convrot {

// ---------------------------------------------------------------- launch set-up cache
//
// A kernel's launch set-up depends only on the kernel and the device: its
// dynamic shared-memory opt-in and how many CTAs (or CTA clusters) of a given
// block size and shared memory fit.  Asking the runtime for them costs tens of
// microseconds of host time per call, which a small problem would spend
// waiting, so each figure is found on its first use on a device and kept.
// Key: the kernel's address, the current device, block size, dynamic shared
// memory.  Thread-safe.
bool launch_figure_get(const void* kernel, int threads, size_t smem, int* figure);
void launch_figure_put(const void* kernel, int threads, size_t smem, int figure);

// ---------------------------------------------------------------- rotate + quantise

// Launch geometry of the rotate+quantise kernel for one row length.
struct RqGeometry {
    int tpr;           // threads holding data in one row (K / 32)
    int tpr_pad;       // threads per row including idle ones (long rows: = tpr, packed back to back)
    int rows_per_cta;  // rows one CTA handles
    int threads;       // CTA size
    int rows128;       // 128-byte shared-memory rows per input row (all row_elems)
    int box1;          // TMA box extent along the 128-byte-row dimension
    int nbox;          // TMA boxes per input row
    int nstage;        // shared-memory ring slots (row groups in flight per CTA)
    size_t smem_bytes; // dynamic shared memory requested
};

// K: elements quantised per row; row_elems: elements loaded per row (K, or
// 2K for the SwiGLU prologue); in_elem_bytes: 2 for bf16 activations, 4 for
// f32 weights.
// act: the ActKind the kernel applies first (its table takes shared memory).
bool rq_geometry(int64_t K, int64_t row_elems, int in_elem_bytes, RqGeometry* g, int act = 0);

// The rotations a row can get: none, Sylvester H_b (b = 64, 128, 256) or the
// regular H_4^(x)k (b = 16, 64, 256).
enum RotKind : int {
    kRotNone = 0,
    kRotSyl64 = 1,
    kRotSyl128 = 2,
    kRotSyl256 = 3,
    kRotReg16 = 4,
    kRotReg64 = 5,
    kRotReg256 = 6,
};

// The activation applied before the rotation (the down projection's input):
// none, x = gelu(h), or x = silu(g) * u with [g | u] the halves of h's row.
enum ActKind : int { kActNone = 0, kActGelu = 1, kActSwiglu = 2 };

// x: bf16 (bits) or f32 rows, described by `xmap` (3D: 128-byte inner rows,
// rows128, M) with 128-byte swizzling.  kind: a RotKind; act: an ActKind
// (bf16 rows only; with kActSwiglu each row holds 2K elements).
cudaError_t launch_rotate_quant(const CUtensorMap& xmap, int in_elem_bytes, int kind, int act, int64_t M, int64_t K,
                                const RqGeometry& g, int8_t* q, int64_t ldq, float* s, uint64_t limit_ns,
                                unsigned int* err, int num_sms, cudaStream_t stream);

// Launch geometry of the one-block-per-thread quantiser (rotate_quant_block.cu).
struct RqbGeometry {
    int tpr;           // threads holding data in one row (K / 128, one Hadamard block each)
    int tpr_pad;       // threads per row including idle ones (long rows: = tpr, packed back to back)
    int rows_per_cta;  // rows one CTA handles per group
    int threads;       // CTA size
    int nb;            // Hadamard blocks per row (the 4-D view's block extent)
    int nstage;        // shared-memory ring slots
    size_t smem_bytes; // dynamic shared memory requested
};

// Geometry for bf16 rows of K elements (K % 128 == 0, K <= 32768); false when
// the rows do not fit this kernel.
bool rqb_geometry(int64_t K, RqbGeometry* g);

// The quantiser with one whole 128-element block per thread, for bf16 rows
// rotated by the Sylvester H_128 (kind kRotSyl128) or not at all (kRotNone).
// `xmap`: 4-D view {64 elements, K/128 blocks, 2 halves, M rows} with byte
// strides {256, 128, row stride}, box {64, K/128, 2, rows_per_cta}, 128-byte
// swizzle.  Same codes and scales as launch_rotate_quant.
cudaError_t launch_rotate_quant_block(const CUtensorMap& xmap, int kind, int64_t M, const RqbGeometry& g, int8_t* q,
                                      int64_t ldq, float* s, uint64_t limit_ns, unsigned int* err, int num_sms,
                                      cudaStream_t stream);

// One CTA waits on an mbarrier that nothing arrives on, so its bounded wait
// must give up after `limit_ns` and record kErrTimeoutSelfTest.
cudaError_t launch_wait_selftest(uint64_t limit_ns, unsigned int* err, cudaStream_t stream);

// ---------------------------------------------------------------- int8 GEMM

enum EpilogueKind : int {
    kEpiBf16 = 0,      // y = acc * s_a[m] * s_b[n] * alpha + bias[n] -> bf16
    kEpiBf16Gelu = 1,  // same, then exact-erf GELU
    kEpiS32 = 2,       // raw int32 accumulators
};

struct GemmArgs {
    int M, N, K, batch;
    const float* s_a;   // [batch * M] (bf16 epilogues)
    const float* s_b;   // [batch * N] (bf16 epilogues)
    const float* bias;  // [N] or null
    float alpha;        // 1/b for a rotated pair, else 1
    uint64_t limit_ns;  // bound on every wait
    unsigned int* err;  // device error word
    int group_m = 1;    // row panels that share each column tile in turn (tile order; 1 = n fastest)
};

// Row panels a GEMM walks together, column tile by column tile.  Weights of
// N x K bytes that do not stay in L2 would otherwise stream from HBM once per
// row panel (every panel walks all column tiles); with G panels per column
// tile, G CTA pairs read each weight tile while it is in L2.  About sqrt(74)
// panels balance the row panels and weight tiles that 74 concurrent tiles
// touch; small weights keep the plain order (G = 1).  Measured on the 768p
// MLP (115.6 MB of weights each way): the down projection's GEMM 2239 ->
// 2170 us with G = 8 (G = 2 and 4 in between).
inline int gemm_group_m(int64_t N, int64_t K) { return N * K > (int64_t{48} << 20) ? 8 : 1; }

// amap: int8 [batch][M][K]; bmap: int8 [batch][N][K]; ymap: output
// [batch][M][N] (bf16, or int32 for kEpiS32).  `pdl` lets the kernel start
// while the previous kernel on the stream drains.
cudaError_t launch_igemm(const CUtensorMap& amap, const CUtensorMap& bmap, const CUtensorMap& ymap,
                         const GemmArgs& a, int epilogue, int num_sms, bool pdl, cudaStream_t stream);

// Whether the GEMM runs as CTA pairs (256 x 256 tiles, cta_group::2).
bool gemm_uses_pair();
// Rows of B one CTA loads per stage: BN for single-CTA tiles, BN/2 for pairs.
int gemm_b_box_rows();

// Box sizes the GEMM's tensor maps must use.
constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmBK = 128;     // bytes of K per stage (= int8 elements)
constexpr int kEpiColsBf16 = 32;  // output columns per epilogue store (bf16: 64-byte rows)
constexpr int kEpiColsS32 = 16;   // output columns per epilogue store (int32: 64-byte rows)
constexpr int kEpiRows = 32;      // rows per epilogue store (one warp)

// ---------------------------------------------------------------- fused linear (one kernel)

// Largest K the one-kernel linear handles (one 96-thread group per row).
constexpr int kFusedMaxK = 6144;

// The one-kernel linear keeps the codes of a few 256-row panels at a time (a
// ring of slots, reused once every tile has loaded the panel in it), so that
// they stay in L2 between the quantiser that writes them and the tensor cores
// that read them, and are overwritten there instead of written back: about
// 16.5 MB of slots (12 panels at K = 5376), at least 4 and at most 12.
constexpr int kFusedRingPanels = 12;
constexpr int64_t kFusedRingBytes = int64_t{12} * 256 * 5376;

// Slots of the ring for M rows of K: every panel its own slot when they fit.
inline int fused_ring_slots(int64_t M, int64_t K) {
    const int64_t panels = (M + 2 * kGemmBM - 1) / (2 * kGemmBM);
    int64_t slots = kFusedRingBytes / (2 * kGemmBM * K);
    slots = slots < 4 ? 4 : (slots > kFusedRingPanels ? kFusedRingPanels : slots);
    return static_cast<int>(panels < slots ? panels : slots);
}

// Whether the ring's lines are marked evict-last in L2: only while the weights
// (N x K bytes, re-read for every panel) fit beside it with room to spare;
// larger weights need the L2 more than the codes do.
inline bool fused_codes_l2_hint(int64_t K, int64_t N) { return K * N <= (int64_t{48} << 20); }

// Rotate + quantise + GEMM + epilogue in one persistent CTA-pair kernel.
// x: bf16 rows [M][ldx] (16-byte aligned rows); amap/bmap/ymap as for
// launch_igemm with batch 1, amap over q's fused_ring_slots(M, K) * 256 rows
// (M rows when the panels all fit).  q: the ring of codes; s: the scales
// [M]; ready: 2 ceil(M/256) + 1 zeroed counters (per-panel ready rows, the
// panels the GEMM has started, per-panel tiles whose codes are loaded).
// kind: a RotKind.
cudaError_t launch_linear_fused(const uint16_t* x, int64_t ldx, const CUtensorMap& amap, const CUtensorMap& bmap,
                                const CUtensorMap& ymap, const GemmArgs& g, int8_t* q, float* s,
                                unsigned int* ready, int kind, int epilogue, int num_sms, bool pdl,
                                cudaStream_t stream);

}  // namespace convrot
