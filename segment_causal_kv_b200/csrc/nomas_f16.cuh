// FP16 operands of the INT8-cache attention forms, shared by the RoPE prep
// kernel, the window dequantisation and the in-shared-memory conversion.
//
// The model card ("Single-GPU Low-Memory Inference") stores K/V in INT8 and
// computes attention in 16-bit floating point. FP16 carries 11 significant
// bits against BF16's 8, but only 5 exponent bits, so every FP16 operand here
// is a power-of-two rescaling of the true value, with the exponent kept beside
// it in fp32:
//   Q row i           Q^_i = RN16(Q~_i * 2^-a_i),   max |Q^_i| in [2^14, 2^15)
//   current K tile T  K^_j = RN16(K~_j * 2^-b_T),   max over the tile in [2^14, 2^15)
//   cache K tile T    K^_j = RN16(code_j * r_j),    r_j = RN16(s_j * 2^-b_T),
//                                                   max_j s_j * 2^-b_T in [2^7, 2^8)
//   cache V tile T    the same with the V scales and exponent c_T
// so |operand| <= 2^15 and the fp32 products of a 128-term dot product stay
// far inside fp32's range. Scaling by a power of two is exact, so the only
// roundings are the FP16 ones. Exponents are clamped to [-100, 100]: values
// beyond 2^±100 are outside what this path supports.
#pragma once

#include <stdint.h>

namespace nomas {

constexpr int kTopFloat = 14; // Q rows and current K tiles: max in [2^14, 2^15)
constexpr int kTopCode = 7;   // INT8 scales: max scale * 2^-e in [2^7, 2^8), codes <= 127

// e such that m * 2^-e lies in [2^top, 2^(top+1)) for a normal m > 0; 0 for
// m == 0 (an all-zero row or tile) or NaN; clamped to [-100, 100].
__device__ __forceinline__ int pow2_exponent(float m, int top) {
    if (!(m > 0.0f)) return 0;
    const int e = ((__float_as_int(m) >> 23) & 0xFF) - 127 - top;
    return e < -100 ? -100 : (e > 100 ? 100 : e);
}

// 2^e for e in [-126, 127], exactly.
__device__ __forceinline__ float exp2_int(int e) { return __int_as_float((e + 127) << 23); }

// Per-tile record read by the attention kernel: (2^b, 2^-b, c, 2^-c) with b
// the tile's K exponent and c its V exponent (0 for current-segment tiles,
// whose V is the caller's BF16 tensor).
__device__ __forceinline__ float4 tile_record(int b, int c) {
    return make_float4(exp2_int(b), exp2_int(-b), static_cast<float>(c), exp2_int(-c));
}

// FP16 bits of RN16(x), twice (both halves of a packed pair).
__device__ __forceinline__ uint32_t f16x2_splat(float x) {
    uint32_t r;
    asm("cvt.rn.f16x2.f32 %0, %1, %1;" : "=r"(r) : "f"(x));
    return r;
}

// 8 INT8 codes times a per-row factor r (a packed FP16 pair r|r) -> 8 FP16
// values RN16(code * r). A code c is read exactly as the FP16 number 1152 + c:
// the byte of c ^ 0x80 (= c + 128) placed in the mantissa of 1024 (ulp 1 on
// [1024, 2048)); the subtraction of 1152 (0x6480) is exact, then one rounded
// product.
__device__ __forceinline__ uint4 codes_to_f16(uint2 w, uint32_t r2) {
    const uint32_t w0 = w.x ^ 0x80808080u, w1 = w.y ^ 0x80808080u;
    uint32_t out[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t src = q < 2 ? w0 : w1;
        uint32_t h = __byte_perm(src, 0x64646464u, (q & 1) ? 0x5342u : 0x5140u);
        asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(h) : "r"(h), "r"(0x64806480u));
        asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(h) : "r"(h), "r"(r2));
        out[q] = h;
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

} // namespace nomas
