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
// of codes.  Its traffic is 3 bytes per element, but measured it is bound by
// instruction issue (the exact conversion) more than by HBM bandwidth.
//
// The conversion itself (and why x * (1/s) may stand in for x / s) lives in
// quant_e4m3.cuh, shared with the GEMM that quantizes its own activations.
#include <cuda_bf16.h>
#include <cuda_fp8.h>

#include "dg_device.cuh"
#include "dg_internal.h"
#include "quant_e4m3.cuh"

namespace dg {

constexpr int kQuantThreads = 256;
// Masked layout: CTAs per slab and column block, each taking every kMaskedRowCtas-th
// token-holding row block.  Measured on 8 x 6912-row slabs for 16384 tokens: 4 ->
// 71 us, 8 -> 54, 16 -> 47-49, 24 -> 49, 32 -> 51; one CTA per block 66.
constexpr int64_t kMaskedRowCtas = 16;

// One 128x128 block: rows lb*128 .. of the matrix Xs (R rows in all, of which `rows`
// hold data), column block bc; scale into *Sp.  red: one word per warp, unused by
// this CTA since the barrier before its previous block.
__device__ __forceinline__ void quantize_block(const uint16_t *__restrict__ Xs, uint8_t *__restrict__ Qs,
                                               float *__restrict__ Sp, int64_t C, int64_t rows, int64_t lb,
                                               int64_t bc, uint32_t *red) {
    const int tid = static_cast<int>(threadIdx.x);
    const int chunk = tid & 15;  // 8-element column group
    const int sub = tid >> 4;    // 0..15
    const int64_t col = bc * 128 + chunk * 8;
    const bool col_ok = col < C;  // C % 16 == 0, so a group is whole or absent
    const int64_t row0 = lb * 128 + sub;
    // rows of this thread's 8 (row0 + 16 i) inside the matrix; the loads and stores
    // step through them by pointer (64-bit row * C products for each of the 8 spilled
    // registers and cost 6 %: 147.5 vs 139.3 us on 36608 x 7168, measured)
    const int nr = col_ok ? static_cast<int>(min(max((rows - row0 + 15) / 16, int64_t(0)), int64_t(8))) : 0;
    const int64_t step = 16 * C;
    const uint16_t *xp = Xs + row0 * C + col;

    uint4 v[8];
    uint32_t m2 = 0;  // two 16-bit magnitude maxima side by side
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        v[i] = i < nr ? __ldg(reinterpret_cast<const uint4 *>(xp + i * step)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) m2 = amax_fold8(m2, v[i]);
    uint32_t amax_bits = amax_bits_of(m2);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax_bits = max(amax_bits, __shfl_xor_sync(0xFFFFFFFFu, amax_bits, o));
    if ((tid & 31) == 0) red[tid >> 5] = amax_bits;
    __syncthreads();
    uint32_t m = red[0];
#pragma unroll
    for (int i = 1; i < kQuantThreads / 32; ++i) m = max(m, red[i]);
    const BlockScale bs = block_scale(m);
    if (tid == 0) *Sp = bs.s;

    uint8_t *qp = Qs + row0 * C + col;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        if (i >= nr) break;
        *reinterpret_cast<uint2 *>(qp + i * step) = quantize8(v[i], bs);
    }
}

// One CTA per block; four CTAs per SM (at most 64 registers): measured 8 % faster
// than three on the 262 M-element MoE activations (147.5 vs 160.1 us), the extra warps
// hiding load latency.
__global__ void __launch_bounds__(kQuantThreads, 4)
    quantize_kernel(const uint16_t *__restrict__ X, int64_t R, int64_t C, int64_t Cb, uint8_t *__restrict__ Q,
                    float *__restrict__ S) {
    __shared__ uint32_t red[kQuantThreads / 32];
    // The GEMM that follows may start its set-up (and its weight prefetch into L2)
    // at once: it still waits for this grid to complete before reading Q and S.
    // Measured 5 % shorter for a quantize + skinny GEMM step at M = 16.
    grid_dep_launch_dependents();
    grid_dep_wait();  // X may come from the previous kernel
    const int64_t blk = blockIdx.x;
    const int64_t lb = blk / Cb, bc = blk - lb * Cb;
    quantize_block(X, Q, S + blk, C, R, lb, bc, red);
}

// The masked MoE layout: X is G slabs of R rows each; slab g holds masked_m[g] tokens
// (clamped to [0, R]) in its first rows and is quantized as the matrix of those rows
// alone: the last token block's amax covers its tokens only, rows past the count are
// neither read nor written, and the blocks past the last token are skipped (their Q
// and S are left as they are).  Block (g, lb, bc) writes scale S[(g * Rb + lb) * Cb +
// bc].  CTA (g, y, bc) takes the slab's row blocks y, y + Ry, ... that hold tokens, so
// mostly empty slabs cost few CTAs (one CTA per block: 9700 of 13800 CTAs exited at
// once on 8 x 6912-row slabs for 16384 tokens).
__global__ void __launch_bounds__(kQuantThreads, 4)
    quantize_masked_kernel(const uint16_t *__restrict__ X, int64_t R, int64_t C, int64_t Cb,
                           uint8_t *__restrict__ Q, float *__restrict__ S, const int32_t *__restrict__ masked_m,
                           int64_t Rb, int64_t Ry) {
    __shared__ uint32_t red[2][kQuantThreads / 32];
    grid_dep_launch_dependents();  // as in quantize_kernel
    grid_dep_wait();               // X and masked_m may come from the previous kernel
    const int64_t blk = blockIdx.x;
    const int64_t gy = blk / Cb, bc = blk - gy * Cb;
    const int64_t g = gy / Ry, y = gy - g * Ry;
    const int64_t rows = min(max(static_cast<int64_t>(__ldg(masked_m + g)), int64_t(0)), R);
    const uint16_t *Xs = X + g * R * C;
    uint8_t *Qs = Q + g * R * C;
    int par = 0;
    for (int64_t lb = y; lb * 128 < rows; lb += Ry) {
        quantize_block(Xs, Qs, S + (g * Rb + lb) * Cb + bc, C, rows, lb, bc, red[par]);
        par ^= 1;
    }
}

// One scale per row and 128-column group ("per-group, 128 elements a group",
// demingchina.com/news/60142 §5.2): the same conversion with the group as the
// block.  Sixteen lanes own a group (16 bytes = 8 BF16 each; a row's group is 256
// contiguous bytes), so the amax needs only shuffles.  A CTA takes one 128-column
// group of kGroupRows consecutive rows, each team of 16 lanes every 16th of them, so
// a thread has four 16-byte loads in flight, and the scales of a CTA go out to
// consecutive addresses of the K-block-major St[kb][row], the layout in which the
// GEMM's epilogue reads one per row with coalesced loads.  Measured at 4096^2: one
// group per thread 22.5 us (latency-bound), this form 20.5 us; working each scale
// out once per team and broadcasting it cut the instructions issued by a fifth but
// was no faster.
constexpr int kGroupRows = 64;

__global__ void __launch_bounds__(kQuantThreads)
    quantize_groups_kernel(const uint16_t *__restrict__ X, int64_t R, int64_t C, int64_t Cb,
                           uint8_t *__restrict__ Q, float *__restrict__ St) {
    grid_dep_launch_dependents();  // as in quantize_kernel
    grid_dep_wait();               // X may come from the previous kernel
    const int tid = static_cast<int>(threadIdx.x);
    const int64_t rt = blockIdx.x / Cb;  // row tile
    const int64_t kb = blockIdx.x - rt * Cb;
    const int64_t col = kb * 128 + (tid & 15) * 8;
    const bool col_ok = col < C;  // C % 16 == 0: an 8-column piece is whole or absent
    const int64_t row0 = rt * kGroupRows + (tid >> 4);
    constexpr int kPer = kGroupRows / 16;  // rows of each team
    const int nr = static_cast<int>(min(max((R - row0 + 15) / 16, int64_t(0)), int64_t(kPer)));
    const int64_t step = 16 * C;
    const uint16_t *xp = X + row0 * C + col;
    uint8_t *qp = Q + row0 * C + col;
    uint4 v[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j)
        v[j] = (col_ok && j < nr) ? __ldg(reinterpret_cast<const uint4 *>(xp + j * step)) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        uint32_t amax_bits = amax_bits_of(amax_fold8(0u, v[j]));
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) amax_bits = max(amax_bits, __shfl_xor_sync(0xFFFFFFFFu, amax_bits, o));
        const BlockScale bs = block_scale(amax_bits);
        if (j < nr) {
            if (col_ok) *reinterpret_cast<uint2 *>(qp + j * step) = quantize8(v[j], bs);
            if ((tid & 15) == 0) St[kb * R + row0 + 16 * j] = bs.s;
        }
    }
}

dg_status_t launch_quantize_groups(const void *X, int64_t rows, int64_t cols, uint8_t *Q, float *St,
                                   const DeviceInfo &dev, cudaStream_t stream) {
    (void)dev;
    const int64_t Cb = (cols + 127) / 128;
    const int64_t blocks = (rows + kGroupRows - 1) / kGroupRows * Cb;
    if (blocks > 0x7FFFFFFFLL) return DG_ERR_SHAPE;
    if (blocks == 0) return DG_OK;
    return launch_pdl(quantize_groups_kernel, static_cast<int>(blocks), kQuantThreads, 0, stream,
                      static_cast<const uint16_t *>(X), rows, cols, Cb, Q, St);
}

dg_status_t launch_quantize_masked(const void *X, int64_t slabs, int64_t rows, int64_t cols,
                                   const int32_t *masked_m, uint8_t *Q, float *S, const DeviceInfo &dev,
                                   cudaStream_t stream);

dg_status_t launch_quantize(const void *X, int64_t rows, int64_t cols, uint8_t *Q, float *S,
                            const DeviceInfo &dev, cudaStream_t stream) {
    return launch_quantize_masked(X, 1, rows, cols, nullptr, Q, S, dev, stream);
}

dg_status_t launch_quantize_masked(const void *X, int64_t slabs, int64_t rows, int64_t cols,
                                   const int32_t *masked_m, uint8_t *Q, float *S, const DeviceInfo &dev,
                                   cudaStream_t stream) {
    (void)dev;
    const int64_t Rb = (rows + 127) / 128, Cb = (cols + 127) / 128;
    const int64_t blocks = slabs * Rb * Cb;
    if (blocks > 0x7FFFFFFFLL) return DG_ERR_SHAPE;
    if (masked_m == nullptr) {
        if (slabs != 1) return DG_ERR_INVALID_ARG;
        return launch_pdl(quantize_kernel, static_cast<int>(blocks), kQuantThreads, 0, stream,
                          static_cast<const uint16_t *>(X), rows, cols, Cb, Q, S);
    }
    const int64_t Ry = min(Rb, kMaskedRowCtas);
    return launch_pdl(quantize_masked_kernel, static_cast<int>(slabs * Ry * Cb), kQuantThreads, 0, stream,
                      static_cast<const uint16_t *>(X), rows, cols, Cb, Q, S, masked_m, Rb, Ry);
}

}  // namespace dg
