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

// fl32(x / s) as far as its E4M3 rounding can tell (see the file comment).
__device__ __forceinline__ float scaled(float x, float s, float r, bool fast_ok) {
    float y = x * r;
    const uint32_t bits = __float_as_uint(y);
    const uint32_t mag = bits & 0x7FFFFFFFu;
    const int d = static_cast<int>(bits & 0xFFFFFu) - 0x80000;
    const bool near_mid = (d <= 6) && (d >= -6);
    // below 2^-6 (biased exponent 121) E4M3 values are subnormal: other midpoints
    if (!fast_ok || near_mid || mag < (121u << 23)) y = __fdiv_rn(x, s);
    return y;
}

__device__ __forceinline__ uint32_t to_e4m3x4(float a, float b, float c, float d) {
    const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
    return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
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
    uint32_t amax_bits = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t row = br * 128 + sub + 16 * i;
        if (col_ok && row < R) {
            v[i] = __ldg(reinterpret_cast<const uint4 *>(X + row * C + col));
        } else {
            v[i] = make_uint4(0, 0, 0, 0);
        }
        // |x| ordering equals the ordering of (bits & 0x7fff) for non-NaN BF16
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            amax_bits = max(amax_bits, w[j] & 0x7FFFu);
            amax_bits = max(amax_bits, (w[j] >> 16) & 0x7FFFu);
        }
    }
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
    if (tid == 0) S[br * Cb + bc] = s;

    if (!col_ok) return;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t row = br * 128 + sub + 16 * i;
        if (row >= R) break;
        const uint32_t w[4] = {v[i].x, v[i].y, v[i].z, v[i].w};
        float f[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            f[2 * j] = scaled(bf16_lo(w[j]), s, r, fast_ok);
            f[2 * j + 1] = scaled(bf16_hi(w[j]), s, r, fast_ok);
        }
        uint2 out;
        out.x = to_e4m3x4(f[0], f[1], f[2], f[3]);
        out.y = to_e4m3x4(f[4], f[5], f[6], f[7]);
        *reinterpret_cast<uint2 *>(Q + row * C + col) = out;
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
