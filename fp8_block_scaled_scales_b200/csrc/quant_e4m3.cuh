// BF16 -> E4M3 conversion shared by the block quantizer and the GEMM that
// quantizes its activations itself (2kiu.com/news/5461879 §2.1 block-wise scaling,
// §3.3 FP32 scales).  Bit-exact contract, for every element x of a block:
//   s = fl32(amax / 448) (1 if amax == 0);  q = E4M3_rn_satfinite(fl32(x / s)).
//
// Division: fl32(x/s) is needed only through its E4M3 rounding.  The code forms
// y = x * r with r = 1/s correctly rounded (__frcp_rn).  Two roundings of relative
// size <= 2^-24 each put y within 2 FP32 ulps of x/s, and fl32(x/s) is within half
// an ulp of it; so unless an E4M3 rounding boundary lies within 3 ulps of y, y and
// fl32(x/s) round to the same E4M3 code.  Near a boundary (see quantize8) or when
// r is not finite, the IEEE division x / s is used instead.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace dg {

// Four floats -> four E4M3 codes (round to nearest even, saturating at +-448), the
// first in the lowest byte.  cvt...e4m3x2 puts its first source operand in the
// high byte of the 16-bit result.
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
    uint32_t out;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(out)
        : "f"(a), "f"(b), "f"(c), "f"(d));
    return out;
}

// The largest |x| of eight BF16 (one 16-byte group), folded into `m2`: two 16-bit
// magnitude maxima side by side.  For non-NaN BF16 the order of |x| is the order
// of (bits & 0x7fff).
__device__ __forceinline__ uint32_t amax_fold8(uint32_t m2, uint4 v) {
    m2 = __vmaxu2(m2, v.x & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v.y & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v.z & 0x7FFF7FFFu);
    m2 = __vmaxu2(m2, v.w & 0x7FFF7FFFu);
    return m2;
}

// The BF16 magnitude bits of a folded maximum.
__device__ __forceinline__ uint32_t amax_bits_of(uint32_t m2) { return max(m2 & 0xFFFFu, m2 >> 16); }

// Block scale from the block's BF16 amax bits, with what the conversion needs.
struct BlockScale {
    float s;       // fl32(amax / 448), 1 for an all-zero block
    float2 r2;     // (1/s, 1/s) correctly rounded
    bool fast_ok;  // 1/s is finite
};

__device__ __forceinline__ BlockScale block_scale(uint32_t amax_bits) {
    BlockScale b;
    const float amax = __uint_as_float(amax_bits << 16);
    b.s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
    const float r = __frcp_rn(b.s);
    b.fast_ok = isfinite(r);
    b.r2 = make_float2(r, r);
    return b;
}

// Eight BF16 (one 16-byte group) -> eight E4M3 codes.
//
// y = x * r is within 3 FP32 ulps of fl32(x / s), so the two round to the same E4M3
// code unless an E4M3 rounding boundary lies within 3 ulps of y.  Two screens find
// every such y, branch-free, over the eight values:
//   - normal range (|y| >= 2^-6): the boundaries are the FP32 values whose mantissa
//     is ...1000...0 below the three kept bits, i.e. bits[19:0] == 0x80000; y is
//     within 6 ulps of one iff (bits + 0x80006) & 0xFFFFF <= 12;
//   - below 2^-6 (E4M3 subnormals, quantum 2^-9): the boundaries are the odd
//     multiples of 2^-10, i.e. 1024 y an odd integer.  With M = 1.5 * 2^23,
//     rr = fl32(1024 y + M) holds the nearest integer n to 1024 y in its last bits
//     (its lowest bit is n's parity), and d = 1024 y - n is exact; 3 ulps of y
//     below 2^-6 are at most 3 * 2^-20 in these units, so the test is |d| <= 2^-18
//     with n odd.  Values that are exact E4M3 numbers (n even), zero included, never
//     fire.
// Only when a screen fires -- about once in 10^5 values -- are the eight quotients
// recomputed with IEEE division.  (A screen that sent every |y| < 2^-6 to the
// division fired in most warps: measured, half the quantizer's time.)
__device__ __forceinline__ uint2 quantize8(uint4 v, const BlockScale &b) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    const float2 k1024 = make_float2(1024.0f, 1024.0f);
    const float2 magic = make_float2(0x1.8p23f, 0x1.8p23f);
    const float2 neg_magic = make_float2(-0x1.8p23f, -0x1.8p23f);
    float2 x[4], y[4];
    uint32_t dmin = 0xFFFFFFFFu, sub = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        x[j] = make_float2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xFFFF0000u));
        y[j] = __fmul2_rn(x[j], b.r2);
        dmin = min(dmin, (__float_as_uint(y[j].x) + 0x80006u) & 0xFFFFFu);
        dmin = min(dmin, (__float_as_uint(y[j].y) + 0x80006u) & 0xFFFFFu);
        const float2 rr = __ffma2_rn(y[j], k1024, magic);
        const float2 n = __fadd2_rn(rr, neg_magic);
        const float2 d = __ffma2_rn(y[j], k1024, make_float2(-n.x, -n.y));
        sub |= (fabsf(d.x) <= 0x1p-18f) ? (__float_as_uint(rr.x) & 1u) : 0u;
        sub |= (fabsf(d.y) <= 0x1p-18f) ? (__float_as_uint(rr.y) & 1u) : 0u;
    }
    if (__builtin_expect(dmin <= 12u || sub != 0u || !b.fast_ok, 0)) {
#pragma unroll
        for (int j = 0; j < 4; ++j) y[j] = make_float2(__fdiv_rn(x[j].x, b.s), __fdiv_rn(x[j].y, b.s));
    }
    uint2 out;
    out.x = e4m3x4(y[0].x, y[0].y, y[1].x, y[1].y);
    out.y = e4m3x4(y[2].x, y[2].y, y[3].x, y[3].y);
    return out;
}

}  // namespace dg
