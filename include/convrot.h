/*
 * convrot.h -- C ABI of libconvrot.so, the B200 (sm_100a) ConvRot W8A8 INT8
 * linear projection.
 *
 * The operation (the pages' "int8_convrot" linear):
 *   1. rotate: z = blockdiag(H_b) x for every token, H_b the Sylvester Hadamard
 *      matrix H[i][j] = (-1)^popcount(i & j), b = 128 (other blocks and the
 *      regular H_4^(x)k: see "Block values" below) ("180 linear layers
 *      quantized to INT8 behind a block-diagonal Hadamard rotation" -- lehuy.net,
 *      "Nen mo hinh video khuech tan 31B xuong 14B chi voi 6 buoc", section
 *      "Cach nen hoat dong");
 *   2. quantise each token row to symmetric int8 with one F32 scale
 *      ("Rowwise INT8 Quantize" -- MiniMax-H3-Rung-Omega README, "Technical
 *      Architecture Overview", item 2, Floor 1):
 *      s = amax/127, q = clamp(rne(z * (127/amax)), -127, 127);
 *   3. multiply with int8 weights that were rotated the same way and quantised
 *      per output channel offline ("per-output F32 scales", "ConvRot metadata",
 *      [output, input] storage -- "MiniMax H3 - pruned INT8 ConvRot -
 *      input-major", section "Input-major checkpoint"), accumulating in int32;
 *   4. dequantise: y = acc * s_x[m] * s_w[n] / b + bias[n], stored as bf16
 *      (bf16, not fp16: "the residual stream reaches 2.4e5" -- "HyperFlow H3
 *      Flash MLX", section "How to run").
 * The 1/b folds the 1/sqrt(b) of both orthonormal rotations into one exact
 * power-of-two factor.
 *
 * Block values (the `block` argument and convrot_wdesc.block):
 *   0 or 1                      no rotation (b = 1);
 *   64, 128, 256                Sylvester H_b, fp32 butterflies in stage order
 *                               h = 1, 2, ..., b/2 (128 is the pages' ConvRot
 *                               block; 64 is their "ConvRot64", MiniMax-H3-
 *                               Rung-Omega README, "Technical Architecture
 *                               Overview", item 2);
 *   CONVROT_HADAMARD_REGULAR | b, b = 16, 64, 256
 *                               the regular H_4^(x)k with H_4 = J - 2I, every
 *                               row summing to sqrt(b) (the "DC-balanced
 *                               regular orthogonal Hadamard matrix
 *                               H_256 = H_4^(x)4", same README, item 1); fp32
 *                               radix-4 stages in digit strides 1, 4, 16, 64,
 *                               each group (x0..x3) -> t - 2 x_i with
 *                               t = (x0 + x1) + (x2 + x3).
 * Both kinds satisfy H_b H_b^T = b I, so the dequantisation divides by b.
 * Any other value is CONVROT_EUNSUPPORTED; K must be a multiple of b.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, except
 *     where a name ends in `_host`.  The library never allocates or frees.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream) on the current device, which must be sm_100 (B200).
 *   - Argument errors are detected on the host and returned before anything is
 *     launched: CONVROT_EINVAL (null pointer, non-positive or oversized size,
 *     bad stride, pointer not 16-byte aligned), CONVROT_EUNSUPPORTED (block
 *     size, device), CONVROT_ELAYOUT (weight descriptor mismatch).
 *     CONVROT_ECUDA reports a failed CUDA call (launch, attribute, copy).
 *   - Every device-side wait is bounded; a wait that gives up records a code
 *     in the library's device error word, which convrot_last_device_status()
 *     reports as CONVROT_ETIMEOUT.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Row-major everywhere: element (r, c) of a matrix with leading dimension
 *     ld is at offset r*ld + c.
 */
#ifndef CONVROT_H
#define CONVROT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum convrot_status {
    CONVROT_OK = 0,
    CONVROT_EINVAL = 1,
    CONVROT_EUNSUPPORTED = 2,
    CONVROT_ELAYOUT = 3,
    CONVROT_ECUDA = 4,
    CONVROT_ETIMEOUT = 5,
    CONVROT_ETOOLARGE = 6  /* exceeds the fixed scratch of convrot_linear_fused_noalloc */
} convrot_status;

/* Packed-weight descriptor.  Plays the role of the pages' "versioned layout
 * marker" that is validated before the pipeline is built ("MiniMax H3 -
 * pruned INT8 ConvRot - input-major", section "Input-major checkpoint"). */
#define CONVROT_WDESC_MAGIC 0x52564E43u   /* "CNVR" */
#define CONVROT_WDESC_VERSION 1u
#define CONVROT_LAYOUT_OUTPUT_MAJOR 1u    /* int8 [N][K], K contiguous */

typedef struct convrot_wdesc {
    uint32_t magic;    /* CONVROT_WDESC_MAGIC */
    uint32_t version;  /* CONVROT_WDESC_VERSION */
    uint32_t layout;   /* CONVROT_LAYOUT_OUTPUT_MAJOR */
    int32_t block;     /* block value used when packing (see above); 0 = none */
    int64_t N;         /* output channels */
    int64_t K;         /* input channels */
} convrot_wdesc;

/* Flag on a block value selecting the regular H_4^(x)k rotation. */
#define CONVROT_HADAMARD_REGULAR 0x10000

/* Epilogue selector of the linear entry points. */
#define CONVROT_EPI_NONE 0  /* y = acc*s_x*s_w/b + bias */
#define CONVROT_EPI_GELU 1  /* then exact-erf GELU: 0.5*y*(1 + erf(y/sqrt(2))) */

/* Human-readable name of a status code (static string, never NULL). */
const char* convrot_status_string(int status);

/* ABI version of this header/library pair (currently 1). */
int convrot_abi_version(void);

/* Offline weight packing (step 3's weights).
 * w: f32 [N][K] row-major.  block: a block value (see above).
 * Writes q: int8 [N][K] (K contiguous, "output-major") and s_w: f32 [N], and
 * fills *desc (HOST pointer) synchronously.  Requires K % 64 == 0,
 * K % b == 0, K <= 32768, N <= 2^31-1, w 16-byte aligned, q 32-byte
 * aligned (the codes are written in 32-byte stores), s_w 4-byte aligned.  Weights
 * must be finite: a row holding inf or NaN is outside the contract (its codes
 * and scale are unspecified; nothing checks them on the device). */
convrot_status convrot_pack_weight(const float* w, int64_t N, int64_t K, int32_t block, int8_t* q,
                                   float* s_w, convrot_wdesc* desc, void* stream);

/* Steps 1-2: x: bf16 [M][K] with row stride ldx (elements) ->
 * q: int8 [M][K] (contiguous) and s_x: f32 [M].  block: a block value.
 * Requires K % 64 == 0, K % b == 0, K <= 32768, ldx >= K, ldx % 8 == 0,
 * 0 < M <= 2^31-1, x 16-byte aligned, q 32-byte aligned, s_x 4-byte
 * aligned.  A row of zeros gives s_x = 0 and zero codes.  Inputs
 * must be finite: a row holding inf or NaN is outside the contract (its codes
 * and scale are unspecified; nothing checks them on the device).  The same
 * holds for every entry point that quantises activations. */
convrot_status convrot_quantize_act(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int32_t block,
                                    int8_t* q, float* s_x, void* stream);

/* Steps 3-4 on already quantised activations.
 * qx: int8 [M][K], s_x: f32 [M]; qw/s_w/desc from convrot_pack_weight;
 * bias: f32 [N] or NULL; epilogue: CONVROT_EPI_*; y: bf16 [M][N] with row
 * stride ldy (ldy >= N, ldy % 8 == 0).  K is desc->K (K % 16 == 0). */
convrot_status convrot_w8a8_linear(const int8_t* qx, const float* s_x, const int8_t* qw, const float* s_w,
                                   const convrot_wdesc* desc, const float* bias, int32_t epilogue, int64_t M,
                                   uint16_t* y, int64_t ldy, void* stream);

/* Workspace of the linear entry points (convrot_linear_fused, _act, _host).
 * Layout, each region starting on a 256-byte boundary:
 *   scales    f32 [M]                                        at byte 0
 *   counters  uint32 [2 ceil(M/256) + 1] (one-kernel path)   after the scales
 *   codes     int8, last: the whole [M][K] array on the two-kernel path, or
 *             a ring of min(M, R * 256) rows on the one-kernel path (R = 12
 *             panel slots at K = 5376; R * 256 * K is about 16.5 MB, 4 <= R
 *             <= 12), reused as the tensor cores finish each panel.
 * convrot_workspace_bytes: enough for either path (the whole codes array).
 * convrot_fused_workspace_bytes: enough for the one-kernel path alone, which
 * convrot_linear_fused takes when K % 128 == 0, 128 <= K <= 6144, x is
 * 32-byte aligned and ldx % 16 == 0 (about 17 MB instead of 208 MB at
 * M = 38656, K = 5376); for other K it equals convrot_workspace_bytes.
 * Both return 0 for M <= 0 or K <= 0. */
size_t convrot_workspace_bytes(int64_t M, int64_t K);
size_t convrot_fused_workspace_bytes(int64_t M, int64_t K);

/* The whole linear, steps 1-4, on `stream`: one kernel (quantiser warps run
 * ahead of the tensor cores in the same CTAs) when K % 128 == 0, 128 <= K <=
 * 6144, x is 32-byte aligned and ldx % 16 == 0; otherwise two kernels (the
 * GEMM starts while the quantiser drains).  x: bf16 [M][K] (row stride ldx);
 * the codes and scales go to `workspace` (256-byte aligned, caller-owned,
 * must not be shared by calls that overlap) of at least the size of the path
 * taken: convrot_fused_workspace_bytes(M, K) on the one-kernel path,
 * convrot_workspace_bytes(M, K) on the two-kernel path (CONVROT_EINVAL with
 * less).  The one-kernel path keeps only a ring of row panels' codes, so
 * after the call the workspace holds the scales of every row but not every
 * row's codes. */
convrot_status convrot_linear_fused(const uint16_t* x, int64_t M, int64_t ldx, const int8_t* qw,
                                    const float* s_w, const convrot_wdesc* desc, const float* bias,
                                    int32_t epilogue, void* workspace, size_t ws_bytes, uint16_t* y, int64_t ldy,
                                    void* stream);

/* Activation prologue of a down projection: the rotation and quantisation
 * of act(h), where h is the up projection's bf16 output ("SwiGLU + ConvRot64
 * + Rowwise INT8 Quantize" fused in MLP.fc2 -- MiniMax-H3-Rung-Omega README,
 * "Technical Architecture Overview", item 2).  The pages print no formula;
 * the reading here:
 *   CONVROT_ACT_GELU    x = gelu(h) = h * Phi(h), h: bf16 [M][K];
 *   CONVROT_ACT_SWIGLU  x = silu(g) * u, silu(g) = g / (1 + e^-g), where each
 *                       row of h holds 2K bf16: g = h[m][0..K), u = h[m][K..2K).
 * x is computed in f32 and goes straight into the rotation and quantiser of
 * convrot_quantize_act (same block values, same q / s_x); it is never stored.
 * Requires ldh >= K (GELU) or 2K (SwiGLU), ldh % 8 == 0, K % 64 == 0,
 * K % b == 0, K <= 32768, h 16-byte aligned, q 32-byte aligned.  Any other
 * act is CONVROT_EINVAL. */
#define CONVROT_ACT_NONE 0
#define CONVROT_ACT_GELU 1
#define CONVROT_ACT_SWIGLU 2
convrot_status convrot_act_quantize(const uint16_t* h, int64_t M, int64_t K, int64_t ldh, int32_t act,
                                    int32_t block, int8_t* q, float* s_x, void* stream);

/* The down projection with the activation prologue: convrot_act_quantize of
 * h into `workspace` (laid out as above, the whole codes array: at least
 * convrot_workspace_bytes(M, desc->K) bytes), then steps 3-4 with the packed
 * weights (K = desc->K).  Two kernels on `stream`; the GEMM starts while the
 * prologue drains. */
convrot_status convrot_linear_act(const uint16_t* h, int64_t M, int64_t ldh, int32_t act, const int8_t* qw,
                                  const float* s_w, const convrot_wdesc* desc, const float* bias, int32_t epilogue,
                                  void* workspace, size_t ws_bytes, uint16_t* y, int64_t ldy, void* stream);

/* int8 attention without materialising the scores ("sageattn_qk_int8_pv_fp16_cuda"
 * in the Rung-Omega engine's Floor 1 -- MiniMax-H3-Rung-Omega README,
 * "Technical Architecture Overview", item 2: int8 Q K^T, 16-bit P V).  The
 * pages give no formula; the reading here, per head h and query row i:
 *   S_ij = (q_i . k_j) * s_q[i] * s_k[j] * scale,  O_i = sum_j softmax_j(S_i.) v_j
 * with q, k the rows of Q and K quantised by the rowwise int8 quantiser (no
 * rotation), v the bf16 rows of V, P rounded to bf16 for the P V product,
 * f32 accumulation, O stored as bf16.  No mask.  Head dimension 128.
 *
 * convrot_attention: q [H][Lq][128], k and v [H][Lk][128], bf16, contiguous;
 * o [H][Lq][128] bf16 (32-byte aligned).  Lq and Lk multiples of 128, scale > 0
 * (1/sqrt(128) for the usual softmax scale).  `workspace` (256-byte aligned,
 * >= convrot_attention_workspace_bytes(H, Lq, Lk)) receives the Q and K codes
 * and scales, V^T and the split parts (see convrot_attention_int8).  Four to
 * six kernels on `stream`. */
size_t convrot_attention_workspace_bytes(int64_t H, int64_t Lq, int64_t Lk);
convrot_status convrot_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t H, int64_t Lq,
                                 int64_t Lk, float scale, void* workspace, size_t ws_bytes, uint16_t* o,
                                 void* stream);

/* The attention kernel alone, on quantised inputs: qx int8 [H][Lq][128] and
 * s_q f32 [H][Lq]; kx int8 [H][Lk][128] and s_k f32 [H][Lk] (16-byte
 * aligned); vt = V^T, bf16 [H][128][Lk]; o as above.
 *
 * The work runs as one CTA per SM for each head and pair of query tiles.
 * When the last wave of those units would leave most SMs idle, the keys of
 * its units are split over all SMs and a small kernel combines the parts
 * (O = sum_p 2^(m_p - M) O_p / sum_p 2^(m_p - M) l_p).  That needs
 * `split_ws`, a caller-owned device buffer (16-byte aligned) of
 * convrot_attention_split_bytes(H, Lq, Lk) bytes; pass NULL (or fewer bytes)
 * to run every unit whole.  The split has no counterpart on the pages; it
 * only changes the order of the f32 sums.  The size depends on the current
 * device's SM count (0 when nothing would be split). */
size_t convrot_attention_split_bytes(int64_t H, int64_t Lq, int64_t Lk);
convrot_status convrot_attention_int8(const int8_t* qx, const float* s_q, const int8_t* kx, const float* s_k,
                                      const uint16_t* vt, int64_t H, int64_t Lq, int64_t Lk, float scale,
                                      void* split_ws, size_t split_bytes, uint16_t* o, void* stream);

/* End-to-end form of convrot_linear_fused for callers whose activations live
 * in host memory: copies x_host (bf16 [M][K], contiguous; pinned for overlap)
 * into the caller's device buffer x_dev, runs the fused linear into y_dev
 * (bf16 [M][N], contiguous) and copies it back to y_host.  The workspace is
 * that of convrot_linear_fused for the largest chunk of rows it is called on
 * (convrot_workspace_bytes(M, K) is always enough).  Rows of
 * more than ~32 MiB of input run in chunks whose copy in, compute and copy
 * out overlap: the copies go on two streams the library owns (one per
 * direction and device), ordered by events, and `stream` waits for the last
 * copy out, so the call is ordered on `stream` as one operation.  The host
 * buffers must stay valid until the stream reaches the end of the call. */
convrot_status convrot_linear_fused_host(const uint16_t* x_host, int64_t M, const int8_t* qw, const float* s_w,
                                         const convrot_wdesc* desc, const float* bias, int32_t epilogue,
                                         uint16_t* x_dev, void* workspace, size_t ws_bytes, uint16_t* y_dev,
                                         uint16_t* y_host, void* stream);

/* Allocation-free form of convrot_linear_fused, for callers that cannot call
 * cudaMalloc: a plugin or embedded runtime whose host owns every device
 * allocation (a pre-planned pool, an ABI that hands out no allocator), or a
 * per-batch loop that cannot afford cudaMalloc's latency and implicit
 * device-wide synchronisation.  (The pages have no counterpart; this is a
 * property of this library's interface, not of the method.)
 * The caller still passes x and y exactly as for convrot_linear_fused; the
 * int8 codes and scales go to a scratch array built into the library instead
 * of a caller workspace.  That array is 32 MiB per device, held by every GPU
 * that loads the library until the process exits: the call accepts problems
 * whose workspace on the path convrot_linear_fused would take fits in
 * 33554432 bytes (convrot_fused_workspace_bytes on the one-kernel path: M up
 * to about 4.2 million rows at K = 5376; convrot_workspace_bytes on the
 * two-kernel path: M <= 6236 at K = 5376, M <= 1560 at K = 21504) and returns
 * CONVROT_ETOOLARGE, launching nothing, beyond that.
 * The first call on each device looks up the array's device address (with
 * that device current); make that first call before any stream capture.
 * All calls share the one array and it keeps the previous call's contents
 * (every byte a call reads was written earlier in the same call, so nothing
 * needs clearing); calls whose kernels overlap on the GPU (different streams,
 * or different host threads) race on it and must be serialised by the caller.
 * Allocates nothing, on the host or the device. */
convrot_status convrot_linear_fused_noalloc(const uint16_t* x, int64_t M, int64_t ldx, const int8_t* qw,
                                            const float* s_w, const convrot_wdesc* desc, const float* bias,
                                            int32_t epilogue, uint16_t* y, int64_t ldy, void* stream);

/* Batched int8 GEMM with per-row scales on both operands and no rotation:
 * y[b][m][n] = bf16(sum_k qa[b][m][k]*qb[b][n][k] * sa[b*M+m] * sb[b*N+n]).
 * Shapes like attention's Q K^T over heads.  All contiguous; K % 16 == 0. */
convrot_status convrot_w8a8_bmm(const int8_t* qa, const float* sa, const int8_t* qb, const float* sb,
                                int64_t batch, int64_t M, int64_t N, int64_t K, uint16_t* y, void* stream);

/* Test hook: raw int32 accumulators acc[b][m][n] = sum_k qa[b][m][k]*qb[b][n][k]
 * from the same tensor-core main loop (N % 4 == 0, K % 16 == 0). */
convrot_status convrot_igemm_s32(const int8_t* qa, const int8_t* qb, int64_t batch, int64_t M, int64_t N,
                                 int64_t K, int32_t* acc, void* stream);

/* Synchronises `stream`, then reads and clears the device error word of the
 * current device: CONVROT_ETIMEOUT if any bounded wait gave up since the last
 * call, CONVROT_ECUDA if the synchronisation failed, else CONVROT_OK.
 * *code (may be NULL) receives the raw site code (0 = none). */
convrot_status convrot_last_device_status(void* stream, uint32_t* code);

/* Bound, in nanoseconds, on every device-side wait of later launches
 * (default 2e9; 0 restores the default). */
void convrot_set_wait_limit_ns(uint64_t ns);

/* Test hook for the failure path: launches one CTA whose wait can never be
 * satisfied, bounded by limit_ns; afterwards convrot_last_device_status()
 * must report CONVROT_ETIMEOUT with code 6.  Faults nothing. */
convrot_status convrot_selftest_wait_timeout(uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* CONVROT_H */
