// BF16 -> E4M3 block quantizer with one FP32 scale per 128x128 block
// (2kiu.com/news/5461879 §2.1 block-wise scaling, §3.3 FP32 scales; the scale
// comes from the block's value range, §5 dynamic activation scales).
//
// Definition (bit-exact contract):
//   amax = max |x| over the block's elements; s = fl32(amax / 448), 1 if amax == 0;
//   q    = E4M3_rn_satfinite( fl32(x / s) ).
//
// One CTA of 256 threads per block.  Each thread loads 8 rows x 16 bytes (8 BF16)
// with 16-byte coalesced loads (a warp covers two 256-byte row segments), keeps
// them in registers through the block max-reduction, then writes 8-byte groups
// of codes.  HBM-bound: 3 bytes of traffic per element.
//
// Division: fl32(x/s) is needed only through its E4M3 rounding.  The kernel forms
// y = x * r with r = 1/s correctly rounded (__frcp_rn).  Two roundings of relative
// size <= 2^-24 each put y within 2 FP32 ulps of x/s, and fl32(x/s) is within half
// an ulp of it; so unless y lies within a few ulps of an E4M3 rounding midpoint
// (mantissa pattern ...1000...0 at the 4th bit), y and fl32(x/s) round to the same
// E4M3 code.  Near a midpoint, below the E4M3 normal range (where the midpoints
// sit at other bit positions) or when r is not finite, the kernel falls back to the
// IEEE division x / s.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "dg_device.cuh"
#include "dg_internal.h"

namespace dg {

constexpr int kQuantThreads = 256;

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

// Eight BF16 (one 16-byte group) -> eight E4M3 codes.
//
// y = x * r (r = 1/s correctly rounded) decides the same E4M3 code as fl32(x / s)
// unless y lies within a few FP32 ulps of an E4M3 rounding midpoint (mantissa bit
// 19 set and bits 0-18 clear: bits[19:0] in [0x7FFFA, 0x80006]) or below 2^-6,
// where E4M3 is subnormal and its midpoints sit at other bit positions.  Both
// conditions are tracked branch-free as running minima over the eight values
// (distance to the midpoint pattern, and |y|); only when one fires -- rarely --
// are the eight quotients recomputed with IEEE division.
__device__ __forceinline__ uint2 quantize8(uint4 v, float s, float2 r2, bool fast_ok) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float2 x[4], y[4];
    uint32_t dmin = 0xFFFFFFFFu;
    float ymin = 1.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        x[j] = make_float2(__uint_as_float(w[j] << 16), __uint_as_float(w[j] & 0xFFFF0000u));
        y[j] = __fmul2_rn(x[j], r2);
        dmin = min(dmin, (__float_as_uint(y[j].x) + 0x80006u) & 0xFFFFFu);
        dmin = min(dmin, (__float_as_uint(y[j].y) + 0x80006u) & 0xFFFFFu);
        ymin = fminf(ymin, fminf(fabsf(y[j].x), fabsf(y[j].y)));
    }
    if (__builtin_expect(dmin <= 12u || ymin < 0x1p-6f || !fast_ok, 0)) {
#pragma unroll
        for (int j = 0; j < 4; ++j) y[j] = make_float2(__fdiv_rn(x[j].x, s), __fdiv_rn(x[j].y, s));
    }
    uint2 out;
    out.x = e4m3x4(y[0].x, y[0].y, y[1].x, y[1].y);
    out.y = e4m3x4(y[2].x, y[2].y, y[3].x, y[3].y);
    return out;
}

__global__ void __launch_bounds__(kQuantThreads)
    quantize_kernel(const uint16_t *__restrict__ X, int64_t R, int64_t C, int64_t Cb, uint8_t *__restrict__ Q,
                    float *__restrict__ S) {
    __shared__ uint32_t red[kQuantThreads / 32];
    const int64_t blk = blockIdx.x;
    const int64_t br = blk / Cb, bc = blk - br * Cb;
    const int tid = static_cast<int>(threadIdx.x);
    const int chunk = tid & 15;  // 8-element column group
    const int sub = tid >> 4;    // 0..15
    const int64_t col = bc * 128 + chunk * 8;
    const bool col_ok = col < C;  // C % 16 == 0, so a group is whole or absent

    uint4 v[8];
    uint32_t m2 = 0;  // two 16-bit magnitude maxima side by side
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t row = br * 128 + sub + 16 * i;
        if (col_ok && row < R) {
            v[i] = __ldg(reinterpret_cast<const uint4 *>(X + row * C + col));
        } else {
            v[i] = make_uint4(0, 0, 0, 0);
        }
    }
    // |x| ordering equals the ordering of (bits & 0x7fff) for non-NaN BF16
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        m2 = __vmaxu2(m2, v[i].x & 0x7FFF7FFFu);
        m2 = __vmaxu2(m2, v[i].y & 0x7FFF7FFFu);
        m2 = __vmaxu2(m2, v[i].z & 0x7FFF7FFFu);
        m2 = __vmaxu2(m2, v[i].w & 0x7FFF7FFFu);
    }
    uint32_t amax_bits = max(m2 & 0xFFFFu, m2 >> 16);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax_bits = max(amax_bits, __shfl_xor_sync(0xFFFFFFFFu, amax_bits, o));
    if ((tid & 31) == 0) red[tid >> 5] = amax_bits;
    __syncthreads();
    uint32_t m = red[0];
#pragma unroll
    for (int i = 1; i < kQuantThreads / 32; ++i) m = max(m, red[i]);
    const float amax = __uint_as_float(m << 16);
    const float s = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 448.0f);
    const float r = __frcp_rn(s);
    const bool fast_ok = isfinite(r);
    const float2 r2 = make_float2(r, r);
    if (tid == 0) S[br * Cb + bc] = s;

    if (!col_ok) return;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t row = br * 128 + sub + 16 * i;
        if (row >= R) break;
        *reinterpret_cast<uint2 *>(Q + row * C + col) = quantize8(v[i], s, r2, fast_ok);
    }
}

dg_status_t launch_quantize(const void *X, int64_t rows, int64_t cols, uint8_t *Q, float *S,
                            const DeviceInfo &dev, cudaStream_t stream) {
    (void)dev;
    const int64_t Rb = (rows + 127) / 128, Cb = (cols + 127) / 128;
    const int64_t blocks = Rb * Cb;
    if (blocks > 0x7FFFFFFFLL) return DG_ERR_SHAPE;
    quantize_kernel<<<static_cast<unsigned>(blocks), kQuantThreads, 0, stream>>>(
        static_cast<const uint16_t *>(X), rows, cols, Cb, Q, S);
    return cudaGetLastError() == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

}  // namespace dg
