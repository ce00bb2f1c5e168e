// api.cu -- the C ABI of libconvrot.so: argument validation, TMA descriptor
// encoding and kernel launches.  The library owns no memory apart from one
// 4-byte device error word per device.
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "convrot.h"
#include "attention.h"
#include "kernels.h"

namespace convrot {

__device__ unsigned int g_device_error = 0;

namespace {

constexpr int kMaxDevices = 64;
constexpr uint64_t kDefaultLimitNs = 2000000000ull;

std::atomic<uint64_t> g_limit_ns{kDefaultLimitNs};

struct DeviceInfo {
    bool ready = false;
    bool supported = false;
    int num_sms = 0;
    unsigned int* err = nullptr;
};

DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mutex;

struct LaunchFigure {
    const void* kernel;
    int dev;
    int threads;
    size_t smem;
    int figure;
};
constexpr int kMaxLaunchFigures = 1024;
LaunchFigure g_figures[kMaxLaunchFigures];
int g_num_figures = 0;
std::mutex g_figure_mutex;

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

const DeviceInfo* device_info() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceInfo& d = g_dev[dev];
    if (!d.ready) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return nullptr;
        if (cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) return nullptr;
        if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return nullptr;
        d.supported = (major == 10 && minor == 0);
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        d.err = static_cast<unsigned int*>(p);
        d.ready = true;
    }
    return &d;
}

bool encoder_ready() {
    std::call_once(g_encode_once, [] {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    });
    return g_encode != nullptr;
}

// 3D tiled tensor map: dims {d0 (contiguous), d1, d2}, byte strides of dims 1
// and 2, box {b0, b1, b2}.
bool encode_3d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
               uint64_t stride1, uint64_t stride2, uint32_t b0, uint32_t b1, uint32_t b2, CUtensorMapSwizzle sw) {
    if (!encoder_ready()) return false;
    cuuint64_t dims[3] = {d0, d1, d2};
    cuuint64_t strides[2] = {stride1, stride2};
    cuuint32_t box[3] = {b0, b1, b2};
    cuuint32_t estr[3] = {1, 1, 1};
    std::memset(map, 0, sizeof(*map));
    CUresult r = g_encode(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 4D tiled tensor map: dims {d0 (contiguous), d1, d2, d3}, byte strides of
// dims 1-3 (any order: a view may visit memory out of its natural order), box
// {b0, b1, b2, b3}.
bool encode_4d(CUtensorMap* map, CUtensorMapDataType dt, const void* base, const uint64_t (&dims)[4],
               const uint64_t (&strides)[3], const uint32_t (&box)[4], CUtensorMapSwizzle sw) {
    if (!encoder_ready()) return false;
    cuuint64_t d[4] = {dims[0], dims[1], dims[2], dims[3]};
    cuuint64_t st[3] = {strides[0], strides[1], strides[2]};
    cuuint32_t b[4] = {box[0], box[1], box[2], box[3]};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    std::memset(map, 0, sizeof(*map));
    CUresult r = g_encode(map, dt, 4, const_cast<void*>(base), d, st, b, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t round256(size_t v) { return (v + 255) / 256 * 256; }
constexpr int64_t kMaxI32 = 2147483647;

convrot_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CONVROT_OK : CONVROT_ECUDA; }

// The ABI's block value: 0 or 1 = no rotation; 64, 128, 256 = Sylvester H_b;
// CONVROT_HADAMARD_REGULAR | 16, 64, 256 = the regular H_4^(x)k.  Sets the
// block length b (1 when there is no rotation) and the kernels' RotKind.
bool decode_block(int32_t block, int* b, int* kind) {
    const bool regular = (block & CONVROT_HADAMARD_REGULAR) != 0;
    const int32_t n = block & ~CONVROT_HADAMARD_REGULAR;
    int k = -1;
    if (!regular) {
        if (n == 0 || n == 1) k = kRotNone;
        else if (n == 64) k = kRotSyl64;
        else if (n == 128) k = kRotSyl128;
        else if (n == 256) k = kRotSyl256;
    } else {
        if (n == 16) k = kRotReg16;
        else if (n == 64) k = kRotReg64;
        else if (n == 256) k = kRotReg256;
    }
    if (k < 0) return false;
    *b = n > 1 ? n : 1;
    *kind = k;
    return true;
}

// Shared by activations (bf16, optionally behind an activation prologue)
// and weights (f32).  act: CONVROT_ACT_*; with SwiGLU each row of x holds
// 2K elements (gate, then up).
convrot_status rotate_quant(const void* x, int in_elem_bytes, int64_t M, int64_t K, int64_t ldx, int32_t block,
                            int8_t* q, float* s, cudaStream_t stream, int32_t act = CONVROT_ACT_NONE) {
    if (!x || !q || !s) return CONVROT_EINVAL;
    if (M <= 0 || M > kMaxI32 || K <= 0) return CONVROT_EINVAL;
    int b = 1, kind = kRotNone;
    if (!decode_block(block, &b, &kind)) return CONVROT_EUNSUPPORTED;
    if (act != CONVROT_ACT_NONE && act != CONVROT_ACT_GELU && act != CONVROT_ACT_SWIGLU) return CONVROT_EINVAL;
    if (act != CONVROT_ACT_NONE && in_elem_bytes != 2) return CONVROT_EINVAL;
    const int64_t row_elems = act == CONVROT_ACT_SWIGLU ? 2 * K : K;
    if (K % 64 != 0 || K > 32768 || K % b != 0) return CONVROT_EINVAL;
    if (ldx < row_elems || (ldx * in_elem_bytes) % 16 != 0) return CONVROT_EINVAL;
    // the codes go out in 32-byte stores (each thread's 64 or 128 codes of a row)
    if (!aligned16(x) || (reinterpret_cast<uintptr_t>(q) & 31u) != 0 || (reinterpret_cast<uintptr_t>(s) & 3u) != 0)
        return CONVROT_EINVAL;
    const DeviceInfo* d = device_info();
    if (!d) return CONVROT_ECUDA;
    if (!d->supported) return CONVROT_EUNSUPPORTED;
    // bf16 rows with the 128-point Sylvester rotation (or none), 256 <= K <= 8192
    // and K % 128 == 0: one whole Hadamard block per thread (fewer instructions
    // per element).  Measured against the 64-element kernel, back to back on
    // 38656 rows: K = 5376 117 vs 123 us, K = 2048 equal; longer rows (K =
    // 21504: 526 vs 508 us, one 352-thread CTA per SM) and K = 128 (24.6 vs
    // 23.5 us on 344064 rows) keep the 64-element kernel.
    RqbGeometry gb;
    if (in_elem_bytes == 2 && act == CONVROT_ACT_NONE && (kind == kRotSyl128 || kind == kRotNone) &&
        K >= 256 && K <= 8192 && rqb_geometry(K, &gb)) {
        CUtensorMap xmap4;
        const uint64_t nb = static_cast<uint64_t>(K / 128);
        // {64 elements, K/128 blocks, 2 halves, M rows}: the first halves of a
        // row's blocks land in consecutive shared rows, then the second halves
        if (!encode_4d(&xmap4, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, {64, nb, 2, static_cast<uint64_t>(M)},
                       {256, 128, static_cast<uint64_t>(ldx) * 2},
                       {64, static_cast<uint32_t>(nb), 2, static_cast<uint32_t>(gb.rows_per_cta)},
                       CU_TENSOR_MAP_SWIZZLE_128B))
            return CONVROT_ECUDA;
        return cuda_status(launch_rotate_quant_block(xmap4, kind, M, gb, q, K, s, g_limit_ns.load(), d->err,
                                                     d->num_sms, stream));
    }
    const int ak = act == CONVROT_ACT_GELU ? kActGelu : act == CONVROT_ACT_SWIGLU ? kActSwiglu : kActNone;
    RqGeometry g;
    if (!rq_geometry(K, row_elems, in_elem_bytes, &g, ak)) return CONVROT_EINVAL;
    CUtensorMap xmap;
    const uint32_t inner = 128u / static_cast<uint32_t>(in_elem_bytes);
    const CUtensorMapDataType dt =
        in_elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    if (!encode_3d(&xmap, dt, x, inner, static_cast<uint64_t>(g.rows128), static_cast<uint64_t>(M), 128,
                   static_cast<uint64_t>(ldx) * in_elem_bytes, inner, static_cast<uint32_t>(g.box1),
                   static_cast<uint32_t>(g.rows_per_cta), CU_TENSOR_MAP_SWIZZLE_128B))
        return CONVROT_ECUDA;
    return cuda_status(launch_rotate_quant(xmap, in_elem_bytes, kind, ak, M, K, g, q, K, s, g_limit_ns.load(),
                                           d->err, d->num_sms, stream));
}

convrot_status check_desc(const convrot_wdesc* desc) {
    if (!desc) return CONVROT_EINVAL;
    if (desc->magic != CONVROT_WDESC_MAGIC || desc->version != CONVROT_WDESC_VERSION ||
        desc->layout != CONVROT_LAYOUT_OUTPUT_MAJOR)
        return CONVROT_ELAYOUT;
    if (desc->N <= 0 || desc->N > kMaxI32 || desc->K <= 0 || desc->K % 16 != 0 || desc->K > kMaxI32)
        return CONVROT_ELAYOUT;
    int b = 1, kind = kRotNone;
    if (!decode_block(desc->block, &b, &kind) || desc->K % b != 0) return CONVROT_ELAYOUT;
    return CONVROT_OK;
}

// GEMM + epilogue over [batch][M][K] x [batch][N][K] -> [batch][M][N].
convrot_status gemm(const int8_t* qa, const int8_t* qb, const float* sa, const float* sb, const float* bias,
                    float alpha, int epi, int64_t batch, int64_t M, int64_t N, int64_t K, void* y, int64_t ldy,
                    bool pdl, cudaStream_t stream) {
    const DeviceInfo* d = device_info();
    if (!d) return CONVROT_ECUDA;
    if (!d->supported) return CONVROT_EUNSUPPORTED;
    const bool s32 = epi == kEpiS32;
    const int ebytes = s32 ? 4 : 2;
    CUtensorMap amap, bmap, ymap;
    if (!encode_3d(&amap, CU_TENSOR_MAP_DATA_TYPE_UINT8, qa, static_cast<uint64_t>(K), static_cast<uint64_t>(M),
                   static_cast<uint64_t>(batch), static_cast<uint64_t>(K), static_cast<uint64_t>(M * K), kGemmBK,
                   kGemmBM, 1, CU_TENSOR_MAP_SWIZZLE_128B))
        return CONVROT_ECUDA;
    if (!encode_3d(&bmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, qb, static_cast<uint64_t>(K), static_cast<uint64_t>(N),
                   static_cast<uint64_t>(batch), static_cast<uint64_t>(K), static_cast<uint64_t>(N * K), kGemmBK,
                   static_cast<uint32_t>(gemm_b_box_rows()), 1, CU_TENSOR_MAP_SWIZZLE_128B))
        return CONVROT_ECUDA;
    if (!encode_3d(&ymap, s32 ? CU_TENSOR_MAP_DATA_TYPE_INT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y,
                   static_cast<uint64_t>(N), static_cast<uint64_t>(M), static_cast<uint64_t>(batch),
                   static_cast<uint64_t>(ldy) * ebytes, static_cast<uint64_t>(M * ldy) * ebytes,
                   s32 ? kEpiColsS32 : kEpiColsBf16, kEpiRows, 1, CU_TENSOR_MAP_SWIZZLE_64B))
        return CONVROT_ECUDA;
    GemmArgs a;
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.batch = static_cast<int>(batch);
    a.s_a = sa;
    a.s_b = sb;
    a.bias = bias;
    a.alpha = alpha;
    a.limit_ns = g_limit_ns.load();
    a.err = d->err;
    a.group_m = gemm_group_m(N, K);
    return cuda_status(launch_igemm(amap, bmap, ymap, a, epi, d->num_sms, pdl, stream));
}

// H_b H_b^T = b I for both kinds, so a rotated pair of operands carries a
// factor b that the epilogue removes (1/b is a power of two: exact).
float alpha_for_block(int32_t block) {
    int b = 1, kind = kRotNone;
    if (!decode_block(block, &b, &kind)) return 1.0f;
    return 1.0f / static_cast<float>(b);
}

int kind_for_block(int32_t block) {
    int b = 1, kind = kRotNone;
    return decode_block(block, &b, &kind) ? kind : kRotNone;
}

bool tiles_fit_int(int64_t batch, int64_t M, int64_t N) {
    const int64_t tiles = ((M + kGemmBM - 1) / kGemmBM) * ((N + kGemmBN - 1) / kGemmBN) * batch;
    return tiles <= kMaxI32;
}

convrot_status linear_checks(const int8_t* qw, const float* s_w, const convrot_wdesc* desc, int32_t epilogue,
                             int64_t M, const void* y, int64_t ldy, const float* bias) {
    convrot_status st = check_desc(desc);
    if (st != CONVROT_OK) return st;
    if (!qw || !s_w || !y) return CONVROT_EINVAL;
    if (epilogue != CONVROT_EPI_NONE && epilogue != CONVROT_EPI_GELU) return CONVROT_EINVAL;
    if (M <= 0 || M > kMaxI32 || !tiles_fit_int(1, M, desc->N)) return CONVROT_EINVAL;
    if (ldy < desc->N || ldy % 8 != 0) return CONVROT_EINVAL;
    if (!aligned16(qw) || !aligned16(y) || (reinterpret_cast<uintptr_t>(s_w) & 3u) != 0) return CONVROT_EINVAL;
    if (bias && (reinterpret_cast<uintptr_t>(bias) & 3u) != 0) return CONVROT_EINVAL;
    return CONVROT_OK;
}

// The one-kernel linear covers every rotation kind for rows whose length
// fits one quantiser group (the descriptor check has already tied the block
// to K).
bool fused_eligible(int64_t K, int32_t block) {
    int b = 1, kind = kRotNone;
    return decode_block(block, &b, &kind) && K % 128 == 0 && K >= 128 && K <= kFusedMaxK;
}

// Workspace of the linear entry points.  Every region starts on a 256-byte
// boundary:
//   scales    f32 [M]                                         at 0
//   counters  u32 [2 ceil(M/256) + 1] of the one-kernel path  after the scales
//   codes     int8: the whole [M][K] array (two-kernel path), or the ring of
//             min(M, fused_ring_slots(M, K) * 256) rows (one-kernel path)
// The codes come last, so the two paths differ only in the workspace's length.
struct WsLayout {
    size_t counters;  // byte offset of the counters
    size_t codes;     // byte offset of the codes
    size_t full;      // bytes with the whole [M][K] codes array
    size_t ring;      // bytes with the one-kernel path's ring of codes
};

WsLayout ws_layout(int64_t M, int64_t K) {
    WsLayout l;
    const size_t panels = static_cast<size_t>((M + 2 * kGemmBM - 1) / (2 * kGemmBM));
    l.counters = round256(static_cast<size_t>(M) * 4);
    l.codes = l.counters + round256((2 * panels + 1) * 4);
    l.full = l.codes + round256(static_cast<size_t>(M) * static_cast<size_t>(K));
    const int64_t ring_rows = std::min<int64_t>(M, int64_t{fused_ring_slots(M, K)} * 2 * kGemmBM);
    l.ring = l.codes + round256(static_cast<size_t>(ring_rows) * static_cast<size_t>(K));
    return l;
}

// Whether convrot_linear_fused takes the one-kernel path for these rows.
bool takes_one_kernel(const void* x, int64_t ldx, const convrot_wdesc* desc) {
    return fused_eligible(desc->K, desc->block) && (reinterpret_cast<uintptr_t>(x) & 31u) == 0 && ldx % 16 == 0;
}

// Workspace bytes convrot_linear_fused needs on the path it takes.
size_t linear_ws_needed(const void* x, int64_t M, int64_t ldx, const convrot_wdesc* desc) {
    const WsLayout l = ws_layout(M, desc->K);
    return takes_one_kernel(x, ldx, desc) ? l.ring : l.full;
}

convrot_status linear_one_kernel(const uint16_t* x, int64_t M, int64_t ldx, const int8_t* qw, const float* s_w,
                                 const convrot_wdesc* desc, const float* bias, int epi, int8_t* qx, float* sx,
                                 unsigned int* ready, uint16_t* y, int64_t ldy, cudaStream_t stream) {
    const DeviceInfo* d = device_info();
    if (!d) return CONVROT_ECUDA;
    if (!d->supported) return CONVROT_EUNSUPPORTED;
    const int64_t K = desc->K, N = desc->N;
    CUtensorMap amap, bmap, ymap;
    const size_t panels = static_cast<size_t>((M + 2 * kGemmBM - 1) / (2 * kGemmBM));
    // the codes ring: every panel its own slot when they fit (then rows past M
    // read as zeros), else kFusedRingPanels full slots
    const int64_t qrows = static_cast<int64_t>(fused_ring_slots(M, K)) < static_cast<int64_t>(panels)
                              ? int64_t{fused_ring_slots(M, K)} * 2 * kGemmBM
                              : M;
    if (!encode_3d(&amap, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx, static_cast<uint64_t>(K), static_cast<uint64_t>(qrows),
                   1, static_cast<uint64_t>(K), static_cast<uint64_t>(qrows * K), kGemmBK, kGemmBM, 1,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return CONVROT_ECUDA;
    if (!encode_3d(&bmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, qw, static_cast<uint64_t>(K), static_cast<uint64_t>(N), 1,
                   static_cast<uint64_t>(K), static_cast<uint64_t>(N * K), kGemmBK, kGemmBN / 2, 1,
                   CU_TENSOR_MAP_SWIZZLE_128B))
        return CONVROT_ECUDA;
    if (!encode_3d(&ymap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, y, static_cast<uint64_t>(N), static_cast<uint64_t>(M), 1,
                   static_cast<uint64_t>(ldy) * 2, static_cast<uint64_t>(M * ldy) * 2, kEpiColsBf16, kEpiRows, 1,
                   CU_TENSOR_MAP_SWIZZLE_64B))
        return CONVROT_ECUDA;
    if (cudaMemsetAsync(ready, 0, (2 * panels + 1) * 4, stream) != cudaSuccess) return CONVROT_ECUDA;
    GemmArgs a;
    a.M = static_cast<int>(M);
    a.N = static_cast<int>(N);
    a.K = static_cast<int>(K);
    a.batch = 1;
    a.s_a = sx;
    a.s_b = s_w;
    a.bias = bias;
    a.alpha = alpha_for_block(desc->block);
    a.limit_ns = g_limit_ns.load();
    a.err = d->err;
    // At most half the codes ring's slots of panels per group.  A group holds
    // the slots of its panels until its last column tile, so with at most the
    // ring's slots no group waits on itself, and with half of them the next
    // group's panels are quantised while the current group runs (the 768p MLP's
    // up projection, 12 slots: 3787 us with G = 1, 3557 us with G = 8, 3490 us
    // with G = 6).
    a.group_m = std::max(1, std::min(gemm_group_m(N, K), fused_ring_slots(M, K) / 2));
    return cuda_status(launch_linear_fused(x, ldx, amap, bmap, ymap, a, qx, sx, ready, kind_for_block(desc->block),
                                           epi, d->num_sms, true, stream));
}

// Rows per chunk of convrot_linear_fused_host's copy/compute pipeline: about
// 32 MiB of input per chunk, a multiple of the 256-row panel (measured at the
// 768p projection: 4, 8, 16, 32, 64, 128 MiB chunks gave 11.8, 10.3, 9.7, 9.5,
// 9.8, 10.7 ms per step).
int64_t host_chunk_rows(int64_t M, int64_t K) {
    const int64_t rows = ((int64_t{32} << 20) / (K * 2) + 255) / 256 * 256;
    return std::max<int64_t>(rows, 256) >= M ? M : std::max<int64_t>(rows, 256);
}

// The library's copy streams and events of the host-buffer pipeline, one set
// per device, created on first use with that device current.
struct HostPipe {
    static constexpr int kEvents = 4;
    std::mutex mutex;  // one call at a time enqueues on this device's set
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, end = nullptr, in[kEvents] = {}, out[kEvents] = {};
    bool ready = false;
};
HostPipe g_host_pipe[kMaxDevices];

HostPipe* host_pipe() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    HostPipe& hp = g_host_pipe[dev];
    if (!hp.ready) {
        bool good = cudaStreamCreateWithFlags(&hp.h2d, cudaStreamNonBlocking) == cudaSuccess &&
                    cudaStreamCreateWithFlags(&hp.d2h, cudaStreamNonBlocking) == cudaSuccess &&
                    cudaEventCreateWithFlags(&hp.start, cudaEventDisableTiming) == cudaSuccess &&
                    cudaEventCreateWithFlags(&hp.end, cudaEventDisableTiming) == cudaSuccess;
        for (int i = 0; good && i < HostPipe::kEvents; ++i)
            good = cudaEventCreateWithFlags(&hp.in[i], cudaEventDisableTiming) == cudaSuccess &&
                   cudaEventCreateWithFlags(&hp.out[i], cudaEventDisableTiming) == cudaSuccess;
        if (!good) return nullptr;  // the caller falls back to the one-piece form
        hp.ready = true;
    }
    return &hp;
}

}  // namespace

bool launch_figure_get(const void* kernel, int threads, size_t smem, int* figure) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    std::lock_guard<std::mutex> lock(g_figure_mutex);
    for (int i = 0; i < g_num_figures; ++i) {
        const LaunchFigure& f = g_figures[i];
        if (f.kernel == kernel && f.dev == dev && f.threads == threads && f.smem == smem) {
            *figure = f.figure;
            return true;
        }
    }
    return false;
}

void launch_figure_put(const void* kernel, int threads, size_t smem, int figure) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return;
    std::lock_guard<std::mutex> lock(g_figure_mutex);
    if (g_num_figures < kMaxLaunchFigures) g_figures[g_num_figures++] = LaunchFigure{kernel, dev, threads, smem, figure};
}

}  // namespace convrot

using namespace convrot;

extern "C" {

const char* convrot_status_string(int status) {
    switch (status) {
        case CONVROT_OK: return "ok";
        case CONVROT_EINVAL: return "invalid argument";
        case CONVROT_EUNSUPPORTED: return "unsupported (block size or device)";
        case CONVROT_ELAYOUT: return "weight descriptor does not match this library's layout";
        case CONVROT_ECUDA: return "CUDA call failed";
        case CONVROT_ETIMEOUT: return "a device-side wait timed out";
        case CONVROT_ETOOLARGE: return "problem exceeds the fixed scratch of the allocation-free entry point";
        default: return "unknown status";
    }
}

int convrot_abi_version(void) { return 1; }

void convrot_set_wait_limit_ns(uint64_t ns) { g_limit_ns.store(ns == 0 ? kDefaultLimitNs : ns); }

convrot_status convrot_pack_weight(const float* w, int64_t N, int64_t K, int32_t block, int8_t* q, float* s_w,
                                   convrot_wdesc* desc, void* stream) {
    if (!desc) return CONVROT_EINVAL;
    convrot_status st = rotate_quant(w, 4, N, K, K, block, q, s_w, static_cast<cudaStream_t>(stream));
    if (st != CONVROT_OK) return st;
    desc->magic = CONVROT_WDESC_MAGIC;
    desc->version = CONVROT_WDESC_VERSION;
    desc->layout = CONVROT_LAYOUT_OUTPUT_MAJOR;
    desc->block = block > 1 ? block : 0;
    desc->N = N;
    desc->K = K;
    return CONVROT_OK;
}

convrot_status convrot_quantize_act(const uint16_t* x, int64_t M, int64_t K, int64_t ldx, int32_t block,
                                    int8_t* q, float* s_x, void* stream) {
    return rotate_quant(x, 2, M, K, ldx, block, q, s_x, static_cast<cudaStream_t>(stream));
}

convrot_status convrot_w8a8_linear(const int8_t* qx, const float* s_x, const int8_t* qw, const float* s_w,
                                   const convrot_wdesc* desc, const float* bias, int32_t epilogue, int64_t M,
                                   uint16_t* y, int64_t ldy, void* stream) {
    convrot_status st = linear_checks(qw, s_w, desc, epilogue, M, y, ldy, bias);
    if (st != CONVROT_OK) return st;
    if (!qx || !s_x || !aligned16(qx) || (reinterpret_cast<uintptr_t>(s_x) & 3u) != 0) return CONVROT_EINVAL;
    return gemm(qx, qw, s_x, s_w, bias, alpha_for_block(desc->block),
                epilogue == CONVROT_EPI_GELU ? kEpiBf16Gelu : kEpiBf16, 1, M, desc->N, desc->K, y, ldy, false,
                static_cast<cudaStream_t>(stream));
}

size_t convrot_workspace_bytes(int64_t M, int64_t K) {
    if (M <= 0 || K <= 0) return 0;
    return ws_layout(M, K).full;
}

size_t convrot_fused_workspace_bytes(int64_t M, int64_t K) {
    if (M <= 0 || K <= 0) return 0;
    const WsLayout l = ws_layout(M, K);
    return (K % 128 == 0 && K >= 128 && K <= kFusedMaxK) ? l.ring : l.full;
}

convrot_status convrot_linear_fused(const uint16_t* x, int64_t M, int64_t ldx, const int8_t* qw, const float* s_w,
                                    const convrot_wdesc* desc, const float* bias, int32_t epilogue,
                                    void* workspace, size_t ws_bytes, uint16_t* y, int64_t ldy, void* stream) {
    convrot_status st = linear_checks(qw, s_w, desc, epilogue, M, y, ldy, bias);
    if (st != CONVROT_OK) return st;
    if (!x || !aligned16(x) || ldx < desc->K || ldx % 8 != 0) return CONVROT_EINVAL;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return CONVROT_EINVAL;
    if (ws_bytes < linear_ws_needed(x, M, ldx, desc)) return CONVROT_EINVAL;
    const WsLayout l = ws_layout(M, desc->K);
    uint8_t* w = static_cast<uint8_t*>(workspace);
    float* sx = reinterpret_cast<float*>(w);
    unsigned int* ready = reinterpret_cast<unsigned int*>(w + l.counters);
    int8_t* qx = reinterpret_cast<int8_t*>(w + l.codes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int epi = epilogue == CONVROT_EPI_GELU ? kEpiBf16Gelu : kEpiBf16;
    // One kernel (the quantiser warps run ahead of the tensor cores) when the
    // rows suit its 32-byte loads; otherwise the two-kernel path below.
    if (takes_one_kernel(x, ldx, desc))
        return linear_one_kernel(x, M, ldx, qw, s_w, desc, bias, epi, qx, sx, ready, y, ldy, s);
    st = rotate_quant(x, 2, M, desc->K, ldx, desc->block, qx, sx, s);
    if (st != CONVROT_OK) return st;
    return gemm(qx, qw, sx, s_w, bias, alpha_for_block(desc->block), epi, 1, M, desc->N, desc->K, y, ldy, true, s);
}

convrot_status convrot_act_quantize(const uint16_t* h, int64_t M, int64_t K, int64_t ldh, int32_t act,
                                    int32_t block, int8_t* q, float* s_x, void* stream) {
    if (act != CONVROT_ACT_GELU && act != CONVROT_ACT_SWIGLU) return CONVROT_EINVAL;
    return rotate_quant(h, 2, M, K, ldh, block, q, s_x, static_cast<cudaStream_t>(stream), act);
}

convrot_status convrot_linear_act(const uint16_t* h, int64_t M, int64_t ldh, int32_t act, const int8_t* qw,
                                  const float* s_w, const convrot_wdesc* desc, const float* bias, int32_t epilogue,
                                  void* workspace, size_t ws_bytes, uint16_t* y, int64_t ldy, void* stream) {
    convrot_status st = linear_checks(qw, s_w, desc, epilogue, M, y, ldy, bias);
    if (st != CONVROT_OK) return st;
    if (act != CONVROT_ACT_GELU && act != CONVROT_ACT_SWIGLU) return CONVROT_EINVAL;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return CONVROT_EINVAL;
    const WsLayout l = ws_layout(M, desc->K);
    if (ws_bytes < l.full) return CONVROT_EINVAL;
    float* sx = static_cast<float*>(workspace);
    int8_t* qx = reinterpret_cast<int8_t*>(static_cast<uint8_t*>(workspace) + l.codes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    st = rotate_quant(h, 2, M, desc->K, ldh, desc->block, qx, sx, s, act);
    if (st != CONVROT_OK) return st;
    const int epi = epilogue == CONVROT_EPI_GELU ? kEpiBf16Gelu : kEpiBf16;
    return gemm(qx, qw, sx, s_w, bias, alpha_for_block(desc->block), epi, 1, M, desc->N, desc->K, y, ldy, true, s);
}

size_t convrot_attention_split_bytes(int64_t H, int64_t Lq, int64_t Lk) {
    if (H <= 0 || Lq <= 0 || Lk <= 0 || Lq % 128 != 0 || Lk % 128 != 0) return 0;
    if (H * Lq > kMaxI32 || H * Lk > kMaxI32) return 0;
    const DeviceInfo* d = device_info();
    if (!d) return 0;
    const AttnSplit sp = attention_split_plan(static_cast<int>(H), static_cast<int>(Lq), static_cast<int>(Lk),
                                              d->num_sms);
    return sp.splits > 1 ? attention_split_bytes(sp.tail * sp.splits) : 0;
}

size_t convrot_attention_workspace_bytes(int64_t H, int64_t Lq, int64_t Lk) {
    if (H <= 0 || Lq <= 0 || Lk <= 0) return 0;
    const size_t hq = static_cast<size_t>(H) * static_cast<size_t>(Lq);
    const size_t hk = static_cast<size_t>(H) * static_cast<size_t>(Lk);
    return round256(hq * 128) + round256(hq * 4) + round256(hk * 128) + round256(hk * 4) + round256(hk * 128 * 2) +
           round256(convrot_attention_split_bytes(H, Lq, Lk));
}

convrot_status convrot_attention_int8(const int8_t* qx, const float* s_q, const int8_t* kx, const float* s_k,
                                      const uint16_t* vt, int64_t H, int64_t Lq, int64_t Lk, float scale,
                                      void* split_ws, size_t split_bytes, uint16_t* o, void* stream) {
    if (!qx || !s_q || !kx || !s_k || !vt || !o) return CONVROT_EINVAL;
    if (H <= 0 || Lq <= 0 || Lk <= 0 || Lq % 128 != 0 || Lk % 128 != 0) return CONVROT_EINVAL;
    if (H * Lq > kMaxI32 || H * Lk > kMaxI32 || Lk > (int64_t{1} << 24)) return CONVROT_EINVAL;
    if (!(scale > 0.0f) || !(scale < 3.0e38f)) return CONVROT_EINVAL;
    if (!aligned16(qx) || !aligned16(kx) || !aligned16(vt) || !aligned16(s_k)) return CONVROT_EINVAL;
    if ((reinterpret_cast<uintptr_t>(s_q) & 3u) != 0 || (reinterpret_cast<uintptr_t>(o) & 31u) != 0)
        return CONVROT_EINVAL;
    if (split_ws != nullptr && !aligned16(split_ws)) return CONVROT_EINVAL;
    const DeviceInfo* d = device_info();
    if (!d) return CONVROT_ECUDA;
    if (!d->supported) return CONVROT_EUNSUPPORTED;
    const AttnSplit plan = attention_split_plan(static_cast<int>(H), static_cast<int>(Lq), static_cast<int>(Lk),
                                                d->num_sms);
    void* part = nullptr;  // without room for the parts every unit runs whole
    if (split_ws != nullptr && plan.splits > 1 && split_bytes >= attention_split_bytes(plan.tail * plan.splits))
        part = split_ws;
    CUtensorMap qmap, kmap, vtmap;
    if (!encode_3d(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, qx, 128, static_cast<uint64_t>(Lq), static_cast<uint64_t>(H),
                   128, static_cast<uint64_t>(Lq) * 128, 128, 128, 1, CU_TENSOR_MAP_SWIZZLE_128B))
        return CONVROT_ECUDA;
    if (!encode_3d(&kmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, kx, 128, static_cast<uint64_t>(Lk), static_cast<uint64_t>(H),
                   128, static_cast<uint64_t>(Lk) * 128, 128, 128, 1, CU_TENSOR_MAP_SWIZZLE_128B))
        return CONVROT_ECUDA;
    if (!encode_3d(&vtmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, vt, static_cast<uint64_t>(Lk), 128,
                   static_cast<uint64_t>(H), static_cast<uint64_t>(Lk) * 2, static_cast<uint64_t>(Lk) * 128 * 2, 64,
                   128, 1, CU_TENSOR_MAP_SWIZZLE_128B))
        return CONVROT_ECUDA;
    const float scale_log2 = scale * 1.4426950408889634f;
    return cuda_status(launch_attention(qmap, kmap, vtmap, static_cast<int>(H), static_cast<int>(Lq),
                                        static_cast<int>(Lk), s_q, s_k, scale_log2, o, g_limit_ns.load(), d->err, true,
                                        static_cast<cudaStream_t>(stream), plan, part));
}

convrot_status convrot_attention(const uint16_t* q, const uint16_t* k, const uint16_t* v, int64_t H, int64_t Lq,
                                 int64_t Lk, float scale, void* workspace, size_t ws_bytes, uint16_t* o,
                                 void* stream) {
    if (!q || !k || !v || !o || !workspace) return CONVROT_EINVAL;
    if (H <= 0 || Lq <= 0 || Lk <= 0 || Lq % 128 != 0 || Lk % 128 != 0) return CONVROT_EINVAL;
    if (H * Lq > kMaxI32 || H * Lk > kMaxI32) return CONVROT_EINVAL;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return CONVROT_EINVAL;
    if (ws_bytes < convrot_attention_workspace_bytes(H, Lq, Lk)) return CONVROT_EINVAL;
    if (!aligned16(v)) return CONVROT_EINVAL;
    const size_t hq = static_cast<size_t>(H) * static_cast<size_t>(Lq);
    const size_t hk = static_cast<size_t>(H) * static_cast<size_t>(Lk);
    uint8_t* w = static_cast<uint8_t*>(workspace);
    int8_t* qx = reinterpret_cast<int8_t*>(w);
    w += round256(hq * 128);
    float* sq = reinterpret_cast<float*>(w);
    w += round256(hq * 4);
    int8_t* kx = reinterpret_cast<int8_t*>(w);
    w += round256(hk * 128);
    float* sk = reinterpret_cast<float*>(w);
    w += round256(hk * 4);
    uint16_t* vt = reinterpret_cast<uint16_t*>(w);
    w += round256(hk * 128 * 2);
    void* part = w;  // the parts of split units (convrot_attention_split_bytes)
    const size_t part_bytes = convrot_attention_split_bytes(H, Lq, Lk);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Q and K: the rowwise int8 quantiser without rotation, one row per token
    convrot_status st = rotate_quant(q, 2, static_cast<int64_t>(hq), 128, 128, 0, qx, sq, s);
    if (st != CONVROT_OK) return st;
    st = rotate_quant(k, 2, static_cast<int64_t>(hk), 128, 128, 0, kx, sk, s);
    if (st != CONVROT_OK) return st;
    st = cuda_status(launch_transpose_v(v, vt, static_cast<int>(H), static_cast<int>(Lk), s));
    if (st != CONVROT_OK) return st;
    return convrot_attention_int8(qx, sq, kx, sk, vt, H, Lq, Lk, scale, part_bytes ? part : nullptr, part_bytes, o,
                                  stream);
}

convrot_status convrot_linear_fused_host(const uint16_t* x_host, int64_t M, const int8_t* qw, const float* s_w,
                                         const convrot_wdesc* desc, const float* bias, int32_t epilogue,
                                         uint16_t* x_dev, void* workspace, size_t ws_bytes, uint16_t* y_dev,
                                         uint16_t* y_host, void* stream) {
    convrot_status st = linear_checks(qw, s_w, desc, epilogue, M, y_dev, desc ? desc->N : 0, bias);
    if (st != CONVROT_OK) return st;
    if (!x_host || !y_host || !x_dev || !aligned16(x_dev)) return CONVROT_EINVAL;
    if (desc->N % 8 != 0) return CONVROT_EINVAL;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return CONVROT_EINVAL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t K = desc->K, N = desc->N;
    const int64_t chunk = host_chunk_rows(M, K);
    // every chunk's call runs on the first (largest) chunk's workspace
    if (ws_bytes < linear_ws_needed(x_dev, chunk, K, desc)) return CONVROT_EINVAL;
    HostPipe* hp = chunk < M ? host_pipe() : nullptr;
    if (hp == nullptr && ws_bytes < linear_ws_needed(x_dev, M, K, desc)) return CONVROT_EINVAL;
    if (hp == nullptr) {  // one piece: copy in, compute, copy out, all on the caller's stream
        if (cudaMemcpyAsync(x_dev, x_host, static_cast<size_t>(M * K) * 2, cudaMemcpyHostToDevice, s) !=
            cudaSuccess)
            return CONVROT_ECUDA;
        st = convrot_linear_fused(x_dev, M, K, qw, s_w, desc, bias, epilogue, workspace, ws_bytes, y_dev, N,
                                  stream);
        if (st != CONVROT_OK) return st;
        if (cudaMemcpyAsync(y_host, y_dev, static_cast<size_t>(M * N) * 2, cudaMemcpyDeviceToHost, s) !=
            cudaSuccess)
            return CONVROT_ECUDA;
        return CONVROT_OK;
    }
    // Row chunks in a pipeline: chunk i's rows go in on the library's
    // host-to-device stream while chunk i - 1 computes on the caller's stream
    // and chunk i - 2's results come out on the device-to-host stream (the two
    // copy directions run on separate copy engines).  Events order each
    // chunk's three steps; the caller's stream waits for the last copy out, so
    // the call stays ordered on `stream` like the one-piece form.
    std::lock_guard<std::mutex> lock(hp->mutex);
    auto ok = [](cudaError_t e) { return e == cudaSuccess; };
    if (!ok(cudaEventRecord(hp->start, s)) || !ok(cudaStreamWaitEvent(hp->h2d, hp->start, 0)) ||
        !ok(cudaStreamWaitEvent(hp->d2h, hp->start, 0)))
        return CONVROT_ECUDA;
    int i = 0;
    for (int64_t r0 = 0; r0 < M; r0 += chunk, ++i) {
        const int64_t rows = std::min(chunk, M - r0);
        cudaEvent_t in = hp->in[i % HostPipe::kEvents], out = hp->out[i % HostPipe::kEvents];
        if (!ok(cudaMemcpyAsync(x_dev + r0 * K, x_host + r0 * K, static_cast<size_t>(rows * K) * 2,
                                cudaMemcpyHostToDevice, hp->h2d)) ||
            !ok(cudaEventRecord(in, hp->h2d)) || !ok(cudaStreamWaitEvent(s, in, 0)))
            return CONVROT_ECUDA;
        st = convrot_linear_fused(x_dev + r0 * K, rows, K, qw, s_w, desc, bias, epilogue, workspace, ws_bytes,
                                  y_dev + r0 * N, N, stream);
        if (st != CONVROT_OK) return st;
        if (!ok(cudaEventRecord(out, s)) || !ok(cudaStreamWaitEvent(hp->d2h, out, 0)) ||
            !ok(cudaMemcpyAsync(y_host + r0 * N, y_dev + r0 * N, static_cast<size_t>(rows * N) * 2,
                                cudaMemcpyDeviceToHost, hp->d2h)))
            return CONVROT_ECUDA;
    }
    if (!ok(cudaEventRecord(hp->end, hp->d2h)) || !ok(cudaStreamWaitEvent(s, hp->end, 0))) return CONVROT_ECUDA;
    return CONVROT_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- allocation-free fused linear
//
// For callers that cannot allocate device memory (see the header): the codes
// and scales that convrot_linear_fused keeps in the caller's workspace live in
// this fixed array instead.  Host code must not hand `g_noalloc_scratch`
// itself to a kernel -- on the host that name is only a stand-in for the
// device symbol -- so its device address is looked up once per device.
namespace convrot {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call per device, with that device current), or null on failure.
void* noalloc_scratch() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    if (g_noalloc_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
        g_noalloc_ptr[dev] = p;
    }
    return g_noalloc_ptr[dev];
}

}  // namespace
}  // namespace convrot

extern "C" {

convrot_status convrot_linear_fused_noalloc(const uint16_t* x, int64_t M, int64_t ldx, const int8_t* qw,
                                            const float* s_w, const convrot_wdesc* desc, const float* bias,
                                            int32_t epilogue, uint16_t* y, int64_t ldy, void* stream) {
    convrot_status st = linear_checks(qw, s_w, desc, epilogue, M, y, ldy, bias);
    if (st != CONVROT_OK) return st;
    if (!x || !aligned16(x) || ldx < desc->K || ldx % 8 != 0) return CONVROT_EINVAL;
    if (linear_ws_needed(x, M, ldx, desc) > kNoAllocScratchBytes) return CONVROT_ETOOLARGE;
    void* scratch = noalloc_scratch();
    if (scratch == nullptr) return CONVROT_ECUDA;
    return convrot_linear_fused(x, M, ldx, qw, s_w, desc, bias, epilogue, scratch, kNoAllocScratchBytes, y, ldy,
                                stream);
}

convrot_status convrot_w8a8_bmm(const int8_t* qa, const float* sa, const int8_t* qb, const float* sb,
                                int64_t batch, int64_t M, int64_t N, int64_t K, uint16_t* y, void* stream) {
    if (!qa || !sa || !qb || !sb || !y) return CONVROT_EINVAL;
    if (batch <= 0 || M <= 0 || N <= 0 || K <= 0 || K % 16 != 0 || N % 8 != 0) return CONVROT_EINVAL;
    if (batch > kMaxI32 || M > kMaxI32 || N > kMaxI32 || K > kMaxI32 || !tiles_fit_int(batch, M, N))
        return CONVROT_EINVAL;
    if (!aligned16(qa) || !aligned16(qb) || !aligned16(y)) return CONVROT_EINVAL;
    if ((reinterpret_cast<uintptr_t>(sa) & 3u) != 0 || (reinterpret_cast<uintptr_t>(sb) & 3u) != 0)
        return CONVROT_EINVAL;
    return gemm(qa, qb, sa, sb, nullptr, 1.0f, kEpiBf16, batch, M, N, K, y, N, false,
                static_cast<cudaStream_t>(stream));
}

convrot_status convrot_igemm_s32(const int8_t* qa, const int8_t* qb, int64_t batch, int64_t M, int64_t N, int64_t K,
                                 int32_t* acc, void* stream) {
    if (!qa || !qb || !acc) return CONVROT_EINVAL;
    if (batch <= 0 || M <= 0 || N <= 0 || K <= 0 || K % 16 != 0 || N % 4 != 0) return CONVROT_EINVAL;
    if (batch > kMaxI32 || M > kMaxI32 || N > kMaxI32 || K > kMaxI32 || !tiles_fit_int(batch, M, N))
        return CONVROT_EINVAL;
    if (!aligned16(qa) || !aligned16(qb) || !aligned16(acc)) return CONVROT_EINVAL;
    return gemm(qa, qb, nullptr, nullptr, nullptr, 1.0f, kEpiS32, batch, M, N, K, acc, N, false,
                static_cast<cudaStream_t>(stream));
}

convrot_status convrot_last_device_status(void* stream, uint32_t* code) {
    if (code) *code = 0;
    const DeviceInfo* d = device_info();
    if (!d) return CONVROT_ECUDA;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return CONVROT_ECUDA;
    unsigned int v = 0;
    if (cudaMemcpy(&v, d->err, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return CONVROT_ECUDA;
    if (v != 0) {
        const unsigned int zero = 0;
        if (cudaMemcpy(d->err, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return CONVROT_ECUDA;
    }
    if (code) *code = v;
    return v ? CONVROT_ETIMEOUT : CONVROT_OK;
}

convrot_status convrot_selftest_wait_timeout(uint64_t limit_ns, void* stream) {
    const DeviceInfo* d = device_info();
    if (!d) return CONVROT_ECUDA;
    if (!d->supported) return CONVROT_EUNSUPPORTED;
    if (limit_ns == 0 || limit_ns > 10000000000ull) return CONVROT_EINVAL;
    return cuda_status(launch_wait_selftest(limit_ns, d->err, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
