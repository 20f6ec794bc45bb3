// RN(x / 127) in fp32 without a division instruction, shared by the commit
// kernel (the INT8 row scale is absmax / 127, correctly rounded) and by the
// device self-test that checks it against the IEEE division for every
// non-negative fp32 input.
#pragma once

namespace nomas {

// RN(x / 127) for a finite x >= 0, by Markstein's division (P. Markstein,
// "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Dev. 34(1), 1990): with r = RN(1/127) and
// q0 = RN(x * r) within an ulp of x / 127, the remainder e = x - 127 q0 is
// exact in one fma and q1 = RN(q0 + e * r) is the correctly rounded quotient
// while nothing underflows. Below 2^-100, and for a non-finite x, the IEEE
// division is used instead. nomas_selftest_div127 compares this function with
// the IEEE division for all 2^31 non-negative fp32 bit patterns.
__device__ __forceinline__ float div127_rn(float x) {
    if (!(x >= 7.8886090522101181e-31f && x <= 3.4028234663852886e38f)) return __fdiv_rn(x, 127.0f); // 2^-100
    constexpr float r = 1.0f / 127.0f;                            // RN(1/127), folded at compile time
    const float q0 = __fmul_rn(x, r);
    const float e = __fmaf_rn(-q0, 127.0f, x);
    return __fmaf_rn(e, r, q0);
}

} // namespace nomas
