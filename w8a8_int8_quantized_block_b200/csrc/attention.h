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
//
// Work split: the kernel's units (a head and a pair of 128-query tiles) run
// one CTA per SM.  When the last wave is only partly filled (units % SMs =
// tail), its tail units get their key tiles split into `splits` parts on
// separate CTAs (tail * splits <= SMs), which write partial results to `part`
// (attention_split_bytes(tail * splits) bytes, 16-byte aligned), and a small
// kernel combines them.  Without `part` (or with splits = 1) every unit runs
// whole.
struct AttnSplit {
    int units = 0;   // heads x query-tile pairs
    int main = 0;    // units run whole
    int tail = 0;    // units split over their keys
    int splits = 1;  // parts per tail unit
};
AttnSplit attention_split_plan(int H, int Lq, int Lk, int num_sms);
size_t attention_split_bytes(int slots);

cudaError_t launch_attention(const CUtensorMap& qmap, const CUtensorMap& kmap, const CUtensorMap& vtmap, int H,
                             int Lq, int Lk, const float* s_q, const float* s_k, float scale_log2, uint16_t* o,
                             uint64_t limit_ns, unsigned int* err, bool pdl, cudaStream_t stream,
                             const AttnSplit& split, void* part);

// V [H][L][128] -> V^T [H][128][L], bf16; L a multiple of 32.
cudaError_t launch_transpose_v(const uint16_t* v, uint16_t* vt, int H, int L, cudaStream_t stream);

}  // namespace convrot
