// fp_div.cuh -- correctly rounded division of many dividends by one shared
// divisor, for the block quantizer (the 16 elements of a block all divide by
// the block's decode scale d = fl32(s * g)).
//
// Method: with r = RN(1/d) computed once (CUDA's correctly rounded
// reciprocal), each quotient is
//     q = RN(x * r),  e = x - d*q  (exact, one fused multiply-add),
//     y = RN(q + e*r)              (one fused multiply-add),
// the final correction step of P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Develop.
// 34(1), 1990: when r is the correctly rounded reciprocal and q is within one
// ulp of x/d, y is the correctly rounded quotient, provided nothing leaves the
// normal range.  div_shared_ok() checks the divisor once per block; outside
// that range the caller uses the plain IEEE division.  With d >= 2^-80 the
// remainder e is exact whenever |x| >= 2^-103, so every quotient of magnitude
// >= 2^-20 is the IEEE one; smaller quotients (from dividends near the bottom
// of the fp32 range) may differ in their last bits but stay far below 0.25,
// where every one of them encodes to the same E2M1 code, +-0 by the sign of x.
// tests/test_division_gpu.py compares this routine with __fdiv_rn over every
// pair of bf16 and fp32 significands and over the whole accepted range.
#pragma once

#include <cstdint>

namespace nvfp4 {

// d is normal and far from both ends of the exponent range, and every
// |x| <= bound keeps x / d below 2^100.
__device__ __forceinline__ bool div_shared_ok(float d, float bound)
{
    return d >= 0x1p-80f && d <= 0x1p100f && bound <= __fmul_rn(d, 0x1p100f);
}

__device__ __forceinline__ float div_shared(float x, float d, float r)
{
    // e' = d*q - x = -e.  Written this way round, x = -0 gives q = -0,
    // e' = (-0) + (+0) = +0 and y = (-0) + (-0) = -0: the IEEE sign of zero
    // comes out of the arithmetic without a separate sign fix-up.
    const float q = __fmul_rn(x, r);
    const float en = __fmaf_rn(d, q, -x);
    return __fmaf_rn(-en, r, q);
}

// div_shared on the two bf16 values packed in w (low half first), with the
// packed two-lane fp32 instructions of sm_100 (mul/fma .rn.f32x2): one
// instruction per step for both quotients.  nr = -RN(1/d).  The steps run on
// the negated dividends -x and the negated reciprocal, which gives the same
// products, remainders and sums as div_shared (every negation is exact and
// each fused operation sees the same operand values and signs), so the
// results are bit-identical to it, signed zeros included.
__device__ __forceinline__ void div_shared_x2(uint32_t w, float d, float nr, float &y_lo, float &y_hi)
{
    const uint32_t wn = w ^ 0x80008000u;  // -x, both halves
    const float nx_lo = __uint_as_float(wn << 16);
    const float nx_hi = __uint_as_float(wn & 0xFFFF0000u);
    asm("{\n\t.reg .b64 x, q, e, dd, rr;\n\t"
        "mov.b64 x, {%2, %3};\n\t"
        "mov.b64 dd, {%4, %4};\n\t"
        "mov.b64 rr, {%5, %5};\n\t"
        "mul.rn.f32x2 q, x, rr;\n\t"      // q = (-x)(-r) = RN(x r)
        "fma.rn.f32x2 e, dd, q, x;\n\t"   // e = RN(d q - x)
        "fma.rn.f32x2 q, e, rr, q;\n\t"   // y = RN(q - e r)
        "mov.b64 {%0, %1}, q;\n\t}"
        : "=f"(y_lo), "=f"(y_hi)
        : "f"(nx_lo), "f"(nx_hi), "f"(d), "f"(nr));
}

// The negated quotients -(x/d) of the two bf16 values packed in w, computed
// from x itself (no negation of the inputs): with nr = -RN(1/d),
//     q = RN(x nr),  e = RN(d q + x),  -y = RN(e nr + q).
// Each step is the exact negation of the matching div_shared step: rounding
// to nearest is symmetric, and where a sum is exactly zero the two forms may
// differ only in the sign of that zero, which reaches the result only for
// x = +-0, where it gives the negated signed zero as well (x = -0 yields
// +0 = -(-0)).  So the results are bit-identical to -div_shared(x, d, RN(1/d)).  The quantizer
// encodes -y and flips the sign bit of every code afterwards, one XOR per
// eight codes instead of one per two inputs.
__device__ __forceinline__ void div_shared_neg_x2(uint32_t w, float d, float nr, float &n_lo, float &n_hi)
{
    asm("{\n\t.reg .b32 l, h;\n\t.reg .b64 x, q, e, dd, rr;\n\t"
        "shl.b32 l, %2, 16;\n\t"
        "and.b32 h, %2, 0xFFFF0000;\n\t"
        "mov.b64 x, {l, h};\n\t"
        "mov.b64 dd, {%3, %3};\n\t"
        "mov.b64 rr, {%4, %4};\n\t"
        "mul.rn.f32x2 q, x, rr;\n\t"     // q = RN(x nr) = -RN(x r)
        "fma.rn.f32x2 e, dd, q, x;\n\t"  // e = RN(x - d RN(x r))
        "fma.rn.f32x2 q, e, rr, q;\n\t"  // -y = RN(-(RN(x r) + e r))
        "mov.b64 {%0, %1}, q;\n\t}"
        : "=f"(n_lo), "=f"(n_hi)
        : "r"(w), "f"(d), "f"(nr));
}

}  // namespace nvfp4
