// quant_core.cuh -- the per-thread pieces of the rotate + quantise pipeline,
// shared by the standalone quantiser and the fused quantise-ahead linear.
//
// A thread owns kPerThread = 64 consecutive elements of a row, held as
// packed f32x2 register pairs P[j] = (element j, element j + 32).  All
// arithmetic is IEEE single precision with round-to-nearest-even, in the
// canonical order of each rotation:
//   Sylvester H_b (b = 64, 128, 256): the textbook in-place fast
//     Walsh-Hadamard transform, stages h = 1, 2, ..., b/2, butterfly
//     (u, w) -> (u + w, u - w); blocks wider than 64 span 2 or 4 lanes.
//   regular H_4^(x)k (b = 16, 64, 256), H_4 = J - 2I: radix-4 stages with
//     digit strides 1, 4, 16, 64; a group (x0, x1, x2, x3) becomes t - 2 x_i
//     with t = (x0 + x1) + (x2 + x3) (2 x_i is exact, so t - 2 x_i is one
//     rounding, done as fma(-2, x_i, t)); the order-256 block spans 4 lanes.
#pragma once

#include <cstdint>

#include "kernels.h"
#include "ptx.cuh"

namespace convrot {
namespace qcore {

constexpr int kPerThread = 64;            // elements each thread owns
constexpr int kPairs = kPerThread / 2;    // P[j] = (element j, element j + kPairs)

// ---- packed single-precision pairs (one 64-bit register pair)

__device__ __forceinline__ uint64_t pk(float a, float b) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
    return r;
}
__device__ __forceinline__ void upk(uint64_t r, float& a, float& b) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Load this thread's kPerThread consecutive elements from the swizzled slot
// into pairs P[j] = (element j, element j + kPairs).  `R0` is the 128-byte
// shared row holding element 0 of the thread's input row.  A 16-byte chunk c
// of 128-byte row R sits at chunk position c ^ (R & 7) (128-byte swizzle).
constexpr int kRawWords = kPerThread / 2;  // 32-bit words of one thread's bf16 elements

// bf16 words (word k holds elements 2k in its low half and 2k+1 in its high
// half; widening to f32 is exact) into pairs P[j] = (element j, element j + kPairs).
__device__ __forceinline__ void unpack_bf16_pairs(const uint32_t (&w)[kRawWords], uint64_t (&P)[kPairs]) {
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
        const uint32_t lo = w[j >> 1], hi = w[(j + kPairs) >> 1];
        const float a = __uint_as_float((j & 1) ? (lo & 0xFFFF0000u) : (lo << 16));
        const float b = __uint_as_float((j & 1) ? (hi & 0xFFFF0000u) : (hi << 16));
        P[j] = pk(a, b);
    }
}

// This thread's kPerThread bf16 elements of a row, straight from global
// memory: 32-byte read-only loads at `row + t*kPerThread` (32-byte aligned),
// marked first-to-evict in L2 (each input byte is read exactly once, so it
// should not displace the codes and weights the tensor cores are about to use).
__device__ __forceinline__ void load_bf16_global(const uint16_t* row, int t, uint32_t (&w)[kRawWords]) {
    const uint16_t* src = row + static_cast<int64_t>(t) * kPerThread;
#pragma unroll
    for (int c = 0; c < kRawWords / 8; ++c) {
        asm volatile(
            "ld.global.nc.L1::no_allocate.L2::evict_first.v8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
            : "=r"(w[8 * c]), "=r"(w[8 * c + 1]), "=r"(w[8 * c + 2]), "=r"(w[8 * c + 3]), "=r"(w[8 * c + 4]),
              "=r"(w[8 * c + 5]), "=r"(w[8 * c + 6]), "=r"(w[8 * c + 7])
            : "l"(src + 16 * c));
    }
}

// Load this thread's kPerThread consecutive elements from a swizzled
// shared-memory slot into pairs.  `R0` is the 128-byte shared row holding
// element 0 of the thread's input row.  A 16-byte chunk c of 128-byte row R
// sits at chunk position c ^ (R & 7) (128-byte swizzle).
template <typename Tin>
__device__ __forceinline__ void load_pairs(const uint8_t* slot, int R0, int t, uint64_t (&P)[kPairs]) {
    constexpr int kBytes = kPerThread * static_cast<int>(sizeof(Tin));
    constexpr int kChunks = kBytes / 16;
    const int off = t * kBytes;  // byte offset of the thread's span in its row
    uint32_t w[kBytes / 4];
#pragma unroll
    for (int c = 0; c < kChunks; ++c) {
        const int cc = (off >> 4) + c;  // chunk index counted from the row start
        const int R = R0 + (cc >> 3);
        const uint4 v = *reinterpret_cast<const uint4*>(slot + R * 128 + (((cc & 7) ^ (R & 7)) << 4));
        w[4 * c] = v.x;
        w[4 * c + 1] = v.y;
        w[4 * c + 2] = v.z;
        w[4 * c + 3] = v.w;
    }
    if constexpr (sizeof(Tin) == 2) {
        unpack_bf16_pairs(w, P);
    } else {
#pragma unroll
        for (int j = 0; j < kPairs; ++j) P[j] = pk(__uint_as_float(w[j]), __uint_as_float(w[j + kPairs]));
    }
}

// ---- the activation prologue of the down projection
//
// The activation is evaluated in double precision and rounded once to f32,
// operation by operation as the plain definition reads: the input (a bf16
// value) is exact in double, the double erfc / exp are within a few units in
// the 53-bit last place of the true value, so the f32 result is the correctly
// rounded activation unless the exact value lies within about 2^-28 of an f32
// rounding boundary.  (An f32 evaluation with erfcf / expf is off by several
// f32 ulp, and in GELU's negative tail by far more, because rounding the
// argument of erfc is amplified there; those errors moved codes across
// rounding ties.)

// gelu(x) = x Phi(x) = 0.5 x erfc(-x / sqrt 2) (the erfc form has no
// cancellation for negative x).  0.5 x is exact; the quotient by the double
// nearest sqrt 2 and the product are IEEE-rounded double operations.
__device__ __forceinline__ float gelu_prologue(float x) {
    const double v = static_cast<double>(x);
    const double t = __ddiv_rn(-v, 1.4142135623730951);  // the double nearest sqrt(2)
    return __double2float_rn(__dmul_rn(0.5 * v, erfc(t)));
}


// silu(g) = g / (1 + e^-g) in double (IEEE sum and division).
__device__ __forceinline__ double silu_double(float g) {
    const double gd = static_cast<double>(g);
    return __ddiv_rn(gd, __dadd_rn(1.0, exp(-gd)));
}

// Tables of the activation for the common inputs.  The input h (or the gate
// g) is a bf16 value, so its double-precision activation depends on 16 bits
// only: a CTA evaluates it once for every bf16 value of a range of binades,
// with the same double operations as above, into shared memory, and each
// element then costs one shared-memory read.  Inputs outside the range (zero,
// tiny or huge values, a few per million in activations) take the direct
// evaluation, so every element gets the value the direct evaluation gives
// it.  Entry of a bf16 bit pattern b: sign, then the binade
// e - E0 (e the biased exponent), then the 7 mantissa bits.
template <int E0, int BINADES>
struct ActTable {
    static constexpr int kEntries = 2 * BINADES * 128;
    // The entry of bf16 bit pattern b, or -1 outside [2^(E0-127), 2^(E0-127+BINADES)).
    __device__ static __forceinline__ int index(uint32_t b) {
        const uint32_t d = ((b >> 7) & 0xFFu) - static_cast<uint32_t>(E0);
        return d < static_cast<uint32_t>(BINADES)
                   ? static_cast<int>((b >> 15) * (BINADES * 128) + d * 128 + (b & 0x7Fu))
                   : -1;
    }
    // The bf16 value of entry i, widened to f32.
    __device__ static __forceinline__ float value(int i) {
        const int sgn = i / (BINADES * 128), r = i - sgn * (BINADES * 128);
        return __uint_as_float(static_cast<uint32_t>((sgn << 15) | ((E0 + (r >> 7)) << 7) | (r & 127)) << 16);
    }
};
using GeluTable = ActTable<107, 32>;  // |h| in [2^-20, 2^12): f32 entries, 32 KB
using SiluTable = ActTable<111, 24>;  // |g| in [2^-16, 2^8): double entries (silu(g) before the product), 48 KB

// Shared-memory bytes of the table an activation kernel keeps (0: none).
constexpr int act_table_bytes(int act) {
    return act == kActGelu ? GeluTable::kEntries * 4 : act == kActSwiglu ? SiluTable::kEntries * 8 : 0;
}

// Fill the table (all threads of the CTA; the caller synchronises after).
template <int ACT>
__device__ __forceinline__ void act_table_fill(void* tab, int tid, int nthreads) {
    if constexpr (ACT == kActGelu) {
        float* t = static_cast<float*>(tab);
        for (int i = tid; i < GeluTable::kEntries; i += nthreads) t[i] = gelu_prologue(GeluTable::value(i));
    } else if constexpr (ACT == kActSwiglu) {
        double* t = static_cast<double*>(tab);
        for (int i = tid; i < SiluTable::kEntries; i += nthreads) t[i] = silu_double(SiluTable::value(i));
    }
}

__device__ __forceinline__ float gelu_lookup(float h, const float* tab) {
    const int i = GeluTable::index(__float_as_uint(h) >> 16);
    return i >= 0 ? tab[i] : gelu_prologue(h);
}

__device__ __forceinline__ void gelu_pairs(uint64_t (&P)[kPairs], const float* tab) {
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
        float a, b;
        upk(P[j], a, b);
        P[j] = pk(gelu_lookup(a, tab), gelu_lookup(b, tab));
    }
}

// silu(g) * u = g / (1 + e^-g) * u: the product in double (IEEE), rounded
// once to f32; silu(g) from the table when g is in its range.
__device__ __forceinline__ float swiglu_lookup(float g, float u, const double* tab) {
    const int i = SiluTable::index(__float_as_uint(g) >> 16);
    const double sg = i >= 0 ? tab[i] : silu_double(g);
    return __double2float_rn(__dmul_rn(sg, static_cast<double>(u)));
}

// x = silu(g) * u for this thread's 64 elements: P holds g; the matching u
// are the thread's 64 bf16 of the row's second half, one 128-byte shared row
// at 128-byte row `Ru` of the swizzled slot, read one 16-byte chunk (eight
// elements) at a time.
__device__ __forceinline__ void swiglu_pairs(uint64_t (&P)[kPairs], const uint8_t* slot, int Ru, const double* tab) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(slot + Ru * 128 + ((c ^ (Ru & 7)) << 4));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int e = 8 * c + i;  // element of the thread's piece
            const float u = __uint_as_float((i & 1) ? (w[i >> 1] & 0xFFFF0000u) : (w[i >> 1] << 16));
            const int j = e & (kPairs - 1);
            float a, b;
            upk(P[j], a, b);
            if (e < kPairs) a = swiglu_lookup(a, u, tab);
            else b = swiglu_lookup(b, u, tab);
            P[j] = pk(a, b);
        }
    }
}

// Stages h = 1, 2, ..., kPairs/2 (packed, both halves at once) then
// h = kPairs (inside each pair).  Butterfly (u, w) -> (u + w, u - w), u the
// lower index.
__device__ __forceinline__ void fwht_in_registers(uint64_t (&P)[kPairs]) {
#pragma unroll
    for (int h = 1; h < kPairs; h <<= 1) {
#pragma unroll
        for (int j = 0; j < kPairs; ++j) {
            if ((j & h) == 0) {
                const uint64_t u = P[j], w = P[j + h];
                P[j] = add2(u, w);
                P[j + h] = sub2(u, w);
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
        float u, w;
        upk(P[j], u, w);
        P[j] = pk(__fadd_rn(u, w), __fsub_rn(u, w));
    }
}

// Stage across lanes: the partner (lane ^ sh) holds the elements
// sh*kPerThread positions away.  sign = +1 on the lower side (self + partner), -1 on the
// upper side (partner - self); fma(sign, self, partner) rounds once, exactly
// like that add or subtract.
__device__ __forceinline__ void fwht_across_lanes(uint64_t (&P)[kPairs], int sh, bool upper) {
    const float sg = upper ? -1.0f : 1.0f;
    const uint64_t S = pk(sg, sg);
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
        float a, b;
        upk(P[j], a, b);
        const float pa = __shfl_xor_sync(0xFFFFFFFFu, a, sh);
        const float pb = __shfl_xor_sync(0xFFFFFFFFu, b, sh);
        P[j] = fma2(S, P[j], pk(pa, pb));
    }
}

// Round and store this thread's codes: v = z * inv rounded to f32 (packed
// multiply), then rounded half-to-even to an integer (|v| <= 127*(1+2^-24) <
// 127.5, so no clamp can bind); byte permutes pack four codes per word; two
// 32-byte stores write the thread's 64 codes at `dst` (32-byte aligned).
//
// Two ways to round v to an integer:
//   kMagicAdd = false: cvt.rni to int32, one conversion per element.
//   kMagicAdd = true:  a packed fma(v, 1, 1.5 * 2^23), half an instruction
//     per element and no conversion unit.  Near 1.5 * 2^23 the f32 spacing is
//     exactly 1, so the fma (v * 1 is exact, so it is the plain add) rounds v
//     half-to-even to an integer, and the low byte of the sum's bits is the
//     code in two's complement.  The multiply and this add must stay two
//     separate roundings: fused into one FMA they would round the exact
//     product instead, which moves values that sit within half an ulp of a
//     tie.  Written as a plain packed add (add.rn.f32x2), ptxas fused it with
//     the packed multiply even with -fmad=false; as fma(v, 1, c) there is no
//     multiply-add pair to fuse.  Crafted rows whose f32 product is exactly
//     k + 1/2 while the exact product is not check this on the GPU.
template <bool kMagicAdd, bool kL2Hint = false>
__device__ __forceinline__ void quantize_store(const uint64_t (&P)[kPairs], float inv, int8_t* dst,
                                               uint64_t l2_policy = 0) {
    const uint64_t inv2 = pk(inv, inv);
    const uint64_t one2 = pk(1.0f, 1.0f);
    const uint64_t magic2 = pk(12582912.0f, 12582912.0f);  // 1.5 * 2^23
    // Pairs 4i..4i+3 hold elements 4i..4i+3 (low halves) and kPairs+4i..+3
    // (high halves): each group of four pairs completes word i and word
    // kPairs/4 + i, so the codes are packed as soon as they exist.
    uint32_t word[kPerThread / 4];
#pragma unroll
    for (int i = 0; i < kPairs / 4; ++i) {
        uint32_t lo[4], hi[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float a, b;
            if constexpr (kMagicAdd) {
                upk(fma2(mul2(P[4 * i + k], inv2), one2, magic2), a, b);
                lo[k] = __float_as_uint(a);
                hi[k] = __float_as_uint(b);
            } else {
                upk(mul2(P[4 * i + k], inv2), a, b);
                lo[k] = static_cast<uint32_t>(__float2int_rn(a));
                hi[k] = static_cast<uint32_t>(__float2int_rn(b));
            }
        }
        word[i] = prmt(prmt(lo[0], lo[1], 0x0040u), prmt(lo[2], lo[3], 0x0040u), 0x5410u);
        word[kPairs / 4 + i] = prmt(prmt(hi[0], hi[1], 0x0040u), prmt(hi[2], hi[3], 0x0040u), 0x5410u);
    }
#pragma unroll
    for (int i = 0; i < kPerThread / 32; ++i) {
        if constexpr (kL2Hint)
            asm volatile("st.global.L2::cache_hint.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8}, %9;" ::"l"(
                             dst + 32 * i),
                         "r"(word[8 * i]), "r"(word[8 * i + 1]), "r"(word[8 * i + 2]), "r"(word[8 * i + 3]),
                         "r"(word[8 * i + 4]), "r"(word[8 * i + 5]), "r"(word[8 * i + 6]), "r"(word[8 * i + 7]),
                         "l"(l2_policy)
                         : "memory");
        else
            asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst + 32 * i),
                         "r"(word[8 * i]), "r"(word[8 * i + 1]), "r"(word[8 * i + 2]), "r"(word[8 * i + 3]),
                         "r"(word[8 * i + 4]), "r"(word[8 * i + 5]), "r"(word[8 * i + 6]), "r"(word[8 * i + 7])
                         : "memory");
    }
}

// ---- regular H_4^(x)k stages

// One radix-4 group of packed pairs: (X0, X1, X2, X3) -> T - 2 X_i with
// T = (X0 + X1) + (X2 + X3), both halves of every pair at once.
__device__ __forceinline__ void reg_group(uint64_t& X0, uint64_t& X1, uint64_t& X2, uint64_t& X3) {
    const uint64_t m2 = pk(-2.0f, -2.0f);
    const uint64_t T = add2(add2(X0, X1), add2(X2, X3));
    X0 = fma2(m2, X0, T);
    X1 = fma2(m2, X1, T);
    X2 = fma2(m2, X2, T);
    X3 = fma2(m2, X3, T);
}

// Digit stride ST (1 or 4) inside each half: the group (e, e+ST, e+2ST,
// e+3ST) of elements is the same group of pair indices, in both halves.
template <int ST>
__device__ __forceinline__ void reg_stage_pairs(uint64_t (&P)[kPairs]) {
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
        if ((j / ST) % 4 == 0) reg_group(P[j], P[j + ST], P[j + 2 * ST], P[j + 3 * ST]);
    }
}

// Digit stride 16: the group (e, e+16, e+32, e+48) is
// (P[e].lo, P[e+16].lo, P[e].hi, P[e+16].hi); t = (x0 + x1) + (x2 + x3) is
// the packed sum of the two pairs followed by the sum of its halves.
__device__ __forceinline__ void reg_stage16(uint64_t (&P)[kPairs]) {
    const uint64_t m2 = pk(-2.0f, -2.0f);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        float s01, s23;
        upk(add2(P[e], P[e + 16]), s01, s23);
        const float t = __fadd_rn(s01, s23);
        const uint64_t T = pk(t, t);
        P[e] = fma2(m2, P[e], T);
        P[e + 16] = fma2(m2, P[e + 16], T);
    }
}

// Digit stride 64: the four 64-element pieces of an order-256 block sit in
// lanes t, t^1, t^2, t^3 (t & 3 = piece).  First u = own + partner(^1), i.e.
// x0 + x1 or x2 + x3 (addition commutes, so both partners round alike), then
// t = u + partner(^2)'s u = (x0 + x1) + (x2 + x3) in every lane.
__device__ __forceinline__ void reg_stage_lanes(uint64_t (&P)[kPairs]) {
    const uint64_t m2 = pk(-2.0f, -2.0f);
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
        float a, b;
        upk(P[j], a, b);
        const uint64_t U = add2(P[j], pk(__shfl_xor_sync(0xFFFFFFFFu, a, 1), __shfl_xor_sync(0xFFFFFFFFu, b, 1)));
        float u0, u1;
        upk(U, u0, u1);
        const uint64_t T = add2(U, pk(__shfl_xor_sync(0xFFFFFFFFu, u0, 2), __shfl_xor_sync(0xFFFFFFFFu, u1, 2)));
        P[j] = fma2(m2, P[j], T);
    }
}

// ---- the rotation kinds

// The whole block transform of this thread's piece; t is the thread's index
// within its row (lanes sharing a block are t ^ 1 and, for 256, t ^ 2, t ^ 3).
template <int KIND>
__device__ __forceinline__ void rotate_piece(uint64_t (&P)[kPairs], int t) {
    if constexpr (KIND == kRotSyl64 || KIND == kRotSyl128 || KIND == kRotSyl256) {
        fwht_in_registers(P);  // h = 1 .. 32
        if constexpr (KIND != kRotSyl64) fwht_across_lanes(P, 1, (t & 1) != 0);  // h = 64
        if constexpr (KIND == kRotSyl256) fwht_across_lanes(P, 2, (t & 2) != 0);  // h = 128
    } else if constexpr (KIND == kRotReg16 || KIND == kRotReg64 || KIND == kRotReg256) {
        reg_stage_pairs<1>(P);
        reg_stage_pairs<4>(P);
        if constexpr (KIND != kRotReg16) reg_stage16(P);
        if constexpr (KIND == kRotReg256) reg_stage_lanes(P);
    }
    (void)t;
}

// Largest |z| over this thread's piece.
__device__ __forceinline__ float piece_absmax(const uint64_t (&P)[kPairs]) {
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < kPairs; ++j) {
        float a, b;
        upk(P[j], a, b);
        amax = fmaxf(amax, fmaxf(fabsf(a), fabsf(b)));
    }
    return amax;
}

}  // namespace qcore
}  // namespace convrot
