// BF16 -> E4M3 conversion shared by the block quantizer and the GEMM that
// quantizes its activations itself (2kiu.com/news/5461879 §2.1 block-wise scaling,
// §3.3 FP32 scales).  Bit-exact contract, for every element x of a block:
//   s = fl32(amax / 448) (1 if amax == 0);  q = E4M3_rn_satfinite(fl32(x / s)).
//
// Division: fl32(x/s) is needed only through its E4M3 rounding, so the code is
// decided from two products that bracket it (quantize8) and the IEEE division
// x / s is used only when the bracket straddles an E4M3 rounding boundary or when
// 1/s is not finite.
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
    float s;        // fl32(amax / 448), 1 for an all-zero block
    float2 rlo2;    // 1/s nudged down and up by a relative 2^-21 (see quantize8)
    float2 rhi2;
    bool fast_ok;   // 1/s is finite
};

__device__ __forceinline__ BlockScale block_scale(uint32_t amax_bits) {
    BlockScale b;
    const float amax = __uint_as_float(amax_bits << 16);
    b.s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
    const float r = __frcp_rn(b.s);
    b.fast_ok = isfinite(r);
    const float rlo = __fmul_rn(r, 1.0f - 0x1p-21f), rhi = __fmul_rn(r, 1.0f + 0x1p-21f);
    b.rlo2 = make_float2(rlo, rlo);
    b.rhi2 = make_float2(rhi, rhi);
    return b;
}

// Eight BF16 (one 16-byte group) -> eight E4M3 codes.
//
// The code wanted is E4M3(t), t = fl32(x / s).  With rlo, rhi = 1/s (correctly
// rounded) times 1 -+ 2^-21 (rounded), ylo = fl32(x rlo) and yhi = fl32(x rhi)
// bracket t strictly: three roundings of relative size at most 2^-24 each put
// |ylo| below |x/s| (1 - 2^-21)(1 + 2^-24)^3 < |x/s| (1 - 2^-24) <= |t|, and |yhi|
// above |t| likewise (FP32 underflow aside, where every candidate is far below the
// E4M3 range and gets the code of zero).  Rounding to E4M3 is monotone, so when
// ylo and yhi get the same code, t gets it too.  They differ only when a rounding
// boundary falls inside the bracket -- for data with an arbitrary amax about once
// in 10^5 values; more often when x / s lands exactly on a boundary, as it can when
// s is a power of two -- and then the eight quotients are recomputed with IEEE
// division.  Per value this costs two multiplies and two conversions, no bit tests.
// (Checked exhaustively on the CPU for every BF16 x and every block amax.)
__device__ __forceinline__ uint2 quantize8(uint4 v, const BlockScale &b) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float2 x[4], lo[4], hi[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        x[j] = make_float2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xFFFF0000u));
        lo[j] = __fmul2_rn(x[j], b.rlo2);
        hi[j] = __fmul2_rn(x[j], b.rhi2);
    }
    uint2 out;
    out.x = e4m3x4(hi[0].x, hi[0].y, hi[1].x, hi[1].y);
    out.y = e4m3x4(hi[2].x, hi[2].y, hi[3].x, hi[3].y);
    const uint32_t lx = e4m3x4(lo[0].x, lo[0].y, lo[1].x, lo[1].y);
    const uint32_t ly = e4m3x4(lo[2].x, lo[2].y, lo[3].x, lo[3].y);
    if (__builtin_expect(((out.x ^ lx) | (out.y ^ ly)) != 0u || !b.fast_ok, 0)) {
        float2 y[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) y[j] = make_float2(__fdiv_rn(x[j].x, b.s), __fdiv_rn(x[j].y, b.s));
        out.x = e4m3x4(y[0].x, y[0].y, y[1].x, y[1].y);
        out.y = e4m3x4(y[2].x, y[2].y, y[3].x, y[3].y);
    }
    return out;
}

}  // namespace dg
