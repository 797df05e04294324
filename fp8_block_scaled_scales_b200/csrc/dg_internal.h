// Host-side internals shared by the translation units of libdg.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dg.h"

namespace dg {

// Per-device facts the dispatch needs (filled once per device).
struct DeviceInfo {
    int ok;          // compute capability 10.0
    int num_sms;
    int max_smem_optin;
};

// Returns DG_OK and fills *info for the current device, or an error status.
dg_status_t current_device(DeviceInfo *info, int *device);

// Encodes a 2-D tiled tensor map (row-major [rows][cols] of elem_bytes each)
// with a box of box_cols x box_rows and the given swizzle.  make_tmap_2d serves
// repeated keys from a small per-thread cache; encode_tmap_2d always encodes.
dg_status_t make_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes,
                         uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                         CUtensorMapSwizzle swizzle);
dg_status_t encode_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes,
                           uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                           CUtensorMapSwizzle swizzle);

// Time limit for every bounded wait inside the kernels, and test-only switches.
struct KernelControl {
    uint64_t timeout_ns;
    int debug_flags;  // bit 0: the tile kernel's producer skips its first stage
    int *status;      // device address of the status word on the current device
};
// Valid after current_device() succeeded on the calling thread's device.
KernelControl kernel_control();

// Launches `kernel` on `stream` with programmatic stream serialisation (the kernel
// may start its set-up while the previous kernel of the stream finishes; it calls
// griddepcontrol.wait before touching memory).  The launch's own return code is the
// status: an error left pending by earlier, unrelated work is neither reported as
// this library's nor cleared.
template <typename... KArgs, typename... Args>
dg_status_t launch_pdl(void (*kernel)(KArgs...), int grid, int block, size_t smem, cudaStream_t stream,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
    cfg.blockDim = dim3(static_cast<unsigned>(block), 1, 1);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...) == cudaSuccess ? DG_OK : DG_ERR_CUDA;
}

// --- launchers (validated arguments only) ----------------------------------
struct GemmArgs {
    const uint8_t *A;
    const float *sA;
    const uint8_t *B;
    const float *sB;
    void *C;
    const int32_t *offsets;  // grouped only
    int64_t M;               // dense: M, grouped: M_total_capacity, masked: G * M_max
    int64_t N;
    int64_t K;
    int G;                   // grouped only
    const int32_t *masked_m = nullptr;  // masked only: tokens per expert (device)
    int64_t m_max = 0;                  // masked only: rows per expert slab
    bool row_scales = false;            // dense only: sA is [ceil(K/128)][M], one scale per row
};

// group: 0 dense, 1 grouped-contiguous, 2 masked
dg_status_t launch_tile_gemm(const GemmArgs &a, int group, const DeviceInfo &dev, cudaStream_t stream);
dg_status_t launch_pair_gemm(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream);
dg_status_t launch_pair_gemm_n128(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream);
dg_status_t launch_skinny_gemm(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream);
// M <= kFusedMaxM with BF16 A quantized inside the GEMM; a.A and a.sA are unused.
// Chosen explicitly (DG_KERNEL_SKINNY_FUSED): in a graph of back-to-back steps
// (N = K = 4096) the quantizer + GEMM pair, whose GEMM starts its weight prefetch
// while the quantizer runs, is as fast or faster (6.65 vs 6.9-7.0 us at M = 1-2;
// 7.1 vs 10.3 us at M = 16), so the automatic dispatch never picks it.
constexpr int64_t kFusedMaxM = 16;
dg_status_t launch_skinny_gemm_fused(const GemmArgs &a, const void *A_bf16, uint8_t *qa_out, float *sa_out,
                                     const DeviceInfo &dev, cudaStream_t stream);
// one scale per row and 128-column group, written K-block-major: St[ceil(cols/128)][rows]
dg_status_t launch_quantize_groups(const void *X, int64_t rows, int64_t cols, uint8_t *Q, float *St,
                                   const DeviceInfo &dev, cudaStream_t stream);
dg_status_t launch_quantize(const void *X, int64_t rows, int64_t cols, uint8_t *Q, float *S,
                            const DeviceInfo &dev, cudaStream_t stream);

}  // namespace dg
