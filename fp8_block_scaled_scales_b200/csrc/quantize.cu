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

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// True when y = x * r might not round to the same E4M3 code as fl32(x / s): y is
// within 6 FP32 ulps of an E4M3 rounding midpoint (bit 19 set, bits 0-18 clear,
// i.e. bits[19:0] in [0x7FFFA, 0x80006]) or below 2^-6, where E4M3 is subnormal
// and its midpoints sit at other bit positions.
__device__ __forceinline__ bool needs_exact(float y) {
    const uint32_t b = __float_as_uint(y);
    const bool near_mid = ((b + 0x80006u) & 0xFFFFFu) <= 12u;
    return near_mid || (fabsf(y) < 0x1p-6f);
}

__device__ __forceinline__ uint32_t to_e4m3x4(float2 a, float2 b) {
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(a, __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(b, __NV_SATFINITE, __NV_E4M3);
    return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// Eight BF16 (one 16-byte group) -> eight E4M3 codes.
__device__ __forceinline__ uint2 quantize8(uint4 v, float s, float2 r2, bool fast_ok) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float2 x[4], y[4];
    bool slow = !fast_ok;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        x[j] = make_float2(bf16_lo(w[j]), bf16_hi(w[j]));
        y[j] = __fmul2_rn(x[j], r2);
        slow |= needs_exact(y[j].x) | needs_exact(y[j].y);
    }
    if (__builtin_expect(slow, 0)) {
#pragma unroll
        for (int j = 0; j < 4; ++j) y[j] = make_float2(__fdiv_rn(x[j].x, s), __fdiv_rn(x[j].y, s));
    }
    uint2 out;
    out.x = to_e4m3x4(y[0], y[1]);
    out.y = to_e4m3x4(y[2], y[3]);
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
