// attention.h -- host-side launchers of the int8 attention kernels (attention.cu).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace convrot {

// O [H][Lq][128] bf16 = softmax((q . k) s_q s_k scale) V per head, q/k int8
// codes described by qmap / kmap (3D {128, L, H}, 128 x 128 boxes, 128-byte
// swizzle), V^T [H][128][Lk] bf16 by vtmap ({Lk, 128, H}, 64 x 128 boxes).
// Lq, Lk multiples of 128; s_k 16-byte aligned; o 32-byte aligned.
cudaError_t launch_attention(const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vtmap, int H,
                             int Lq, int Lk, const float* s_q, const float* s_k, float scale_log2, uint16_t* o,
                             uint64_t limit_ns, unsigned int* err, bool pdl, cudaStream_t stream);

// V [H][L][128] -> V^T [H][128][L], bf16; L a multiple of 32.
cudaError_t launch_transpose_v(const uint16_t* v, uint16_t* vt, int H, int L, cudaStream_t stream);

}  // namespace convrot
