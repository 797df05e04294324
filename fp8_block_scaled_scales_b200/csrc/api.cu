// C ABI of libdg.so: argument validation, device checks, tensor-map encoding,
// kernel dispatch and the device status word.  See include/dg.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>

#include <mutex>

#include "dg_device.cuh"
#include "dg_internal.h"

namespace dg {

// quantize.cu: `slabs` slabs of `rows` rows each, quantized slab by slab; with masked_m
// (device, [slabs]) the row blocks of slab g at or past ceil(masked_m[g] / 128) are skipped.
dg_status_t launch_quantize_masked(const void *X, int64_t slabs, int64_t rows, int64_t cols,
                                   const int32_t *masked_m, uint8_t *Q, float *S, const DeviceInfo &dev,
                                   cudaStream_t stream);

// The device status word: [0] status of the first failure since the last read,
// [1] role, [2] block, [3] step; [4..7] the snapshot the last read took.  One per
// device (a module global).
__device__ int g_status[8];

// Takes the status word: swaps [0] with zero atomically (a failure recorded
// concurrently is kept for the next read) and copies it with its details to [4..7].
__global__ void status_take_kernel() {
    const int st = atomicExch(&g_status[0], 0);
    g_status[4] = st;
    g_status[5] = g_status[1];
    g_status[6] = g_status[2];
    g_status[7] = g_status[3];
}

namespace {

constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
int *g_status_addr[kMaxDevices];
bool g_dev_ready[kMaxDevices];
std::mutex g_mu;

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

dg_status_t load_encoder() {
    if (g_encode) return DG_OK;
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
        return DG_ERR_CUDA;
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    return DG_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

uint64_t g_timeout_ns = 2000000000ull;
int g_debug_flags = 0;

}  // namespace

KernelControl kernel_control() {
    int dev = 0;
    cudaGetDevice(&dev);
    KernelControl c;
    c.timeout_ns = g_timeout_ns;
    c.debug_flags = g_debug_flags;
    c.status = (dev >= 0 && dev < kMaxDevices) ? g_status_addr[dev] : nullptr;
    return c;
}

dg_status_t current_device(DeviceInfo *info, int *device) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return DG_ERR_UNSUPPORTED_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_dev_ready[dev]) {
        int major = 0, minor = 0, sms = 0, smem = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return DG_ERR_CUDA;
        g_dev[dev].ok = (major == 10 && minor == 0);
        g_dev[dev].num_sms = sms;
        g_dev[dev].max_smem_optin = smem;
        if (load_encoder() != DG_OK) return DG_ERR_CUDA;
        void *addr = nullptr;
        if (g_dev[dev].ok) {
            if (cudaGetSymbolAddress(&addr, g_status) != cudaSuccess) return DG_ERR_CUDA;
        }
        g_status_addr[dev] = static_cast<int *>(addr);
        g_dev_ready[dev] = true;
    }
    *info = g_dev[dev];
    if (device) *device = dev;
    return info->ok ? DG_OK : DG_ERR_UNSUPPORTED_DEVICE;
}

namespace {
// Encoded tensor maps of recent calls, per host thread.  A map depends only on the
// address, shape, box and swizzle (no device state), so an entry with the same key
// is the same map; a decode loop that reuses its buffers skips the encoding.
struct TmapEntry {
    const void *base;
    uint64_t rows, cols;
    uint32_t box_rows, box_cols;
    int dtype, elem_bytes, swizzle;
    CUtensorMap map;
};
constexpr int kTmapCache = 32;
thread_local TmapEntry t_tmaps[kTmapCache];
thread_local int t_tmap_used = 0, t_tmap_next = 0;
}  // namespace

dg_status_t make_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes,
                         uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                         CUtensorMapSwizzle swizzle) {
    for (int i = 0; i < t_tmap_used; ++i) {
        const TmapEntry &e = t_tmaps[i];
        if (e.base == base && e.rows == rows && e.cols == cols && e.box_rows == box_rows &&
            e.box_cols == box_cols && e.dtype == static_cast<int>(dtype) && e.elem_bytes == elem_bytes &&
            e.swizzle == static_cast<int>(swizzle)) {
            *map = e.map;
            return DG_OK;
        }
    }
    const dg_status_t st = encode_tmap_2d(map, base, dtype, elem_bytes, rows, cols, box_rows, box_cols, swizzle);
    if (st != DG_OK) return st;
    TmapEntry &e = t_tmaps[t_tmap_next];
    e = TmapEntry{base, rows, cols, box_rows, box_cols, static_cast<int>(dtype), elem_bytes,
                  static_cast<int>(swizzle), *map};
    t_tmap_next = (t_tmap_next + 1) % kTmapCache;
    if (t_tmap_used < kTmapCache) ++t_tmap_used;
    return DG_OK;
}

dg_status_t encode_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, int elem_bytes,
                           uint64_t rows, uint64_t cols, uint32_t box_rows, uint32_t box_cols,
                           CUtensorMapSwizzle swizzle) {
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * static_cast<uint64_t>(elem_bytes)};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t elem_strides[2] = {1, 1};
    const CUresult r = g_encode(map, dtype, 2, const_cast<void *>(base), dims, strides, box, elem_strides,
                                CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

}  // namespace dg

using namespace dg;

extern "C" {

int dg_version(void) { return 105; }

const char *dg_status_string(dg_status_t s) {
    switch (s) {
        case DG_OK: return "DG_OK";
        case DG_ERR_INVALID_ARG: return "DG_ERR_INVALID_ARG: null pointer or bad argument";
        case DG_ERR_SHAPE: return "DG_ERR_SHAPE: size outside the shape contract";
        case DG_ERR_ALIGNMENT: return "DG_ERR_ALIGNMENT: pointer not aligned as required";
        case DG_ERR_UNSUPPORTED_DEVICE: return "DG_ERR_UNSUPPORTED_DEVICE: needs compute capability 10.0 (sm_100a)";
        case DG_ERR_CUDA: return "DG_ERR_CUDA: a CUDA call failed";
        case DG_ERR_TIMEOUT: return "DG_ERR_TIMEOUT: a device pipeline wait ran past its limit";
        case DG_ERR_GROUP_OFFSETS: return "DG_ERR_GROUP_OFFSETS: group_offsets broke its contract; nothing was computed";
    }
    return "unknown dg_status_t";
}

dg_status_t dg_get_last_device_status(cudaStream_t stream) {
    DeviceInfo dev;
    const dg_status_t st = current_device(&dev, nullptr);
    if (st != DG_OK) return st;
    if (cudaLaunchKernel(reinterpret_cast<const void *>(status_take_kernel), dim3(1), dim3(1), nullptr, 0,
                         stream) != cudaSuccess)
        return DG_ERR_CUDA;
    int h[4] = {0, 0, 0, 0};
    if (cudaMemcpyFromSymbolAsync(h, g_status, sizeof(h), 4 * sizeof(int), cudaMemcpyDeviceToHost, stream) !=
            cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
        return DG_ERR_CUDA;
    return static_cast<dg_status_t>(h[0]);
}

// Test hook (declared in the test-only section of include/dg.h): sets the time
// limit of the kernels' bounded waits and the debug switches for later launches.
void dg_test_set_kernel_control(uint64_t timeout_ns, int debug_flags) {
    g_timeout_ns = timeout_ns ? timeout_ns : 2000000000ull;
    g_debug_flags = debug_flags;
}

dg_status_t dg_quantize_blockwise(const void *X_bf16, int64_t rows, int64_t cols, uint8_t *Q, float *S,
                                  cudaStream_t stream) {
    if (rows < 0 || cols < 0 || cols % 16 != 0) return DG_ERR_SHAPE;
    if (rows == 0 || cols == 0) return DG_OK;
    if (!X_bf16 || !Q || !S) return DG_ERR_INVALID_ARG;
    if (!aligned(X_bf16, 16) || !aligned(Q, 16) || !aligned(S, 4)) return DG_ERR_ALIGNMENT;
    DeviceInfo dev;
    dg_status_t st = current_device(&dev, nullptr);
    if (st != DG_OK) return st;
    return launch_quantize(X_bf16, rows, cols, Q, S, dev, stream);
}

dg_status_t dg_quantize_blockwise_masked(const void *X_bf16, int G, int64_t M_max, int64_t cols,
                                         const int32_t *masked_m, uint8_t *Q, float *S, cudaStream_t stream) {
    if (G < 1 || G > 1024 || M_max < 0 || cols < 0 || cols % 16 != 0) return DG_ERR_SHAPE;
    if (M_max == 0 || cols == 0) return DG_OK;
    if (!X_bf16 || !masked_m || !Q || !S) return DG_ERR_INVALID_ARG;
    if (!aligned(X_bf16, 16) || !aligned(Q, 16) || !aligned(S, 4) || !aligned(masked_m, 4)) return DG_ERR_ALIGNMENT;
    DeviceInfo dev;
    dg_status_t st = current_device(&dev, nullptr);
    if (st != DG_OK) return st;
    return launch_quantize_masked(X_bf16, G, M_max, cols, masked_m, Q, S, dev, stream);
}

dg_status_t dg_quantize_1x128(const void *X_bf16, int64_t rows, int64_t cols, uint8_t *Q, float *S_t,
                              cudaStream_t stream) {
    if (rows < 0 || cols < 0 || cols % 16 != 0) return DG_ERR_SHAPE;
    if (rows == 0 || cols == 0) return DG_OK;
    if (!X_bf16 || !Q || !S_t) return DG_ERR_INVALID_ARG;
    if (!aligned(X_bf16, 16) || !aligned(Q, 16) || !aligned(S_t, 4)) return DG_ERR_ALIGNMENT;
    DeviceInfo dev;
    dg_status_t st = current_device(&dev, nullptr);
    if (st != DG_OK) return st;
    return launch_quantize_groups(X_bf16, rows, cols, Q, S_t, dev, stream);
}

static dg_status_t check_gemm_common(const uint8_t *A, const float *sA, const uint8_t *B, const float *sB,
                                     const void *C) {
    if (!A || !sA || !B || !sB || !C) return DG_ERR_INVALID_ARG;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(C, 16) || !aligned(sA, 4) || !aligned(sB, 4))
        return DG_ERR_ALIGNMENT;
    return DG_OK;
}

dg_status_t dg_fp8_gemm_blockscaled_select(const uint8_t *A, const float *sA, const uint8_t *B, const float *sB,
                                           void *C_bf16, int64_t M, int64_t N, int64_t K, dg_kernel_t kernel,
                                           cudaStream_t stream) {
    if (M < 0 || N < 0 || K <= 0 || K % 16 != 0 || N % 16 != 0) return DG_ERR_SHAPE;
    // TMA coordinates are 32-bit signed
    if (M > 0x7FFFFFFFLL || N > 0x7FFFFFFFLL || K > 0x7FFFFFFFLL) return DG_ERR_SHAPE;
    if (kernel != DG_KERNEL_AUTO && kernel != DG_KERNEL_TILE && kernel != DG_KERNEL_SKINNY &&
        kernel != DG_KERNEL_PAIR)
        return DG_ERR_INVALID_ARG;
    if (kernel == DG_KERNEL_SKINNY && M > 128) return DG_ERR_SHAPE;
    if (M == 0 || N == 0) return DG_OK;
    dg_status_t st = check_gemm_common(A, sA, B, sB, C_bf16);
    if (st != DG_OK) return st;
    DeviceInfo dev;
    st = current_device(&dev, nullptr);
    if (st != DG_OK) return st;
    GemmArgs a = {A, sA, B, sB, C_bf16, nullptr, M, N, K, 0};
    if (kernel == DG_KERNEL_AUTO) kernel = M <= 128 ? DG_KERNEL_SKINNY : DG_KERNEL_TILE;
    if (kernel == DG_KERNEL_SKINNY) return launch_skinny_gemm(a, dev, stream);
    if (kernel == DG_KERNEL_TILE) return launch_tile_gemm(a, 0, dev, stream);
    return N <= 128 ? launch_pair_gemm_n128(a, dev, stream) : launch_pair_gemm(a, dev, stream);
}

dg_status_t dg_fp8_gemm_blockscaled(const uint8_t *A, const float *sA, const uint8_t *B, const float *sB,
                                    void *C_bf16, int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
    return dg_fp8_gemm_blockscaled_select(A, sA, B, sB, C_bf16, M, N, K, DG_KERNEL_AUTO, stream);
}

dg_status_t dg_fp8_gemm_1x128_select(const uint8_t *A, const float *sA_t, const uint8_t *B, const float *sB,
                                     void *C_bf16, int64_t M, int64_t N, int64_t K, dg_kernel_t kernel,
                                     cudaStream_t stream) {
    if (M < 0 || N < 0 || K <= 0 || K % 16 != 0 || N % 16 != 0) return DG_ERR_SHAPE;
    if (M > 0x7FFFFFFFLL || N > 0x7FFFFFFFLL || K > 0x7FFFFFFFLL) return DG_ERR_SHAPE;
    if (kernel != DG_KERNEL_AUTO && kernel != DG_KERNEL_TILE && kernel != DG_KERNEL_PAIR) return DG_ERR_INVALID_ARG;
    if (M == 0 || N == 0) return DG_OK;
    dg_status_t st = check_gemm_common(A, sA_t, B, sB, C_bf16);
    if (st != DG_OK) return st;
    DeviceInfo dev;
    st = current_device(&dev, nullptr);
    if (st != DG_OK) return st;
    GemmArgs a = {A, sA_t, B, sB, C_bf16, nullptr, M, N, K, 0};
    a.row_scales = true;
    if (kernel == DG_KERNEL_AUTO) kernel = DG_KERNEL_TILE;
    if (kernel == DG_KERNEL_TILE) return launch_tile_gemm(a, 0, dev, stream);
    return N <= 128 ? launch_pair_gemm_n128(a, dev, stream) : launch_pair_gemm(a, dev, stream);
}

dg_status_t dg_fp8_gemm_1x128(const uint8_t *A, const float *sA_t, const uint8_t *B, const float *sB, void *C_bf16,
                              int64_t M, int64_t N, int64_t K, cudaStream_t stream) {
    return dg_fp8_gemm_1x128_select(A, sA_t, B, sB, C_bf16, M, N, K, DG_KERNEL_AUTO, stream);
}

dg_status_t dg_fp8_gemm_blockscaled_bf16a_select(const void *A_bf16, const uint8_t *B, const float *sB,
                                                 void *C_bf16, uint8_t *QA, float *sA, int64_t M, int64_t N,
                                                 int64_t K, dg_kernel_t kernel, cudaStream_t stream) {
    if (M < 0 || N < 0 || K <= 0 || K % 16 != 0 || N % 16 != 0) return DG_ERR_SHAPE;
    if (M > 0x7FFFFFFFLL || N > 0x7FFFFFFFLL || K > 0x7FFFFFFFLL) return DG_ERR_SHAPE;
    if (kernel != DG_KERNEL_AUTO && kernel != DG_KERNEL_TILE && kernel != DG_KERNEL_SKINNY &&
        kernel != DG_KERNEL_PAIR && kernel != DG_KERNEL_SKINNY_FUSED)
        return DG_ERR_INVALID_ARG;
    if ((kernel == DG_KERNEL_SKINNY && M > 128) || (kernel == DG_KERNEL_SKINNY_FUSED && M > kFusedMaxM))
        return DG_ERR_SHAPE;
    if (M == 0 || N == 0) return DG_OK;
    if (!A_bf16) return DG_ERR_INVALID_ARG;
    dg_status_t st = check_gemm_common(QA, sA, B, sB, C_bf16);
    if (st != DG_OK) return st;
    if (!aligned(A_bf16, 16)) return DG_ERR_ALIGNMENT;
    DeviceInfo dev;
    st = current_device(&dev, nullptr);
    if (st != DG_OK) return st;
    if (kernel == DG_KERNEL_SKINNY_FUSED) {
        // one launch: the skinny kernel quantizes A itself and writes QA, sA on the way
        GemmArgs a = {QA, sA, B, sB, C_bf16, nullptr, M, N, K, 0};
        return launch_skinny_gemm_fused(a, A_bf16, QA, sA, dev, stream);
    }
    st = launch_quantize(A_bf16, M, K, QA, sA, dev, stream);
    if (st != DG_OK) return st;
    return dg_fp8_gemm_blockscaled_select(QA, sA, B, sB, C_bf16, M, N, K, kernel, stream);
}

dg_status_t dg_fp8_gemm_blockscaled_bf16a(const void *A_bf16, const uint8_t *B, const float *sB, void *C_bf16,
                                          uint8_t *QA, float *sA, int64_t M, int64_t N, int64_t K,
                                          cudaStream_t stream) {
    return dg_fp8_gemm_blockscaled_bf16a_select(A_bf16, B, sB, C_bf16, QA, sA, M, N, K, DG_KERNEL_AUTO, stream);
}

dg_status_t dg_fp8_grouped_gemm_masked(const uint8_t *A, const float *sA, const uint8_t *B, const float *sB,
                                       void *C_bf16, const int32_t *masked_m, int G, int64_t M_max, int64_t N,
                                       int64_t K, cudaStream_t stream) {
    if (G < 1 || G > 256 || M_max < 0 || N < 0 || N % 128 != 0 || K <= 0 || K % 16 != 0) return DG_ERR_SHAPE;
    if (static_cast<int64_t>(G) * M_max > 0x7FFFFFFFLL || static_cast<int64_t>(G) * N > 0x7FFFFFFFLL ||
        K > 0x7FFFFFFFLL)
        return DG_ERR_SHAPE;
    if (M_max == 0 || N == 0) return DG_OK;
    if (!masked_m) return DG_ERR_INVALID_ARG;
    if (!aligned(masked_m, 4)) return DG_ERR_ALIGNMENT;
    dg_status_t st = check_gemm_common(A, sA, B, sB, C_bf16);
    if (st != DG_OK) return st;
    DeviceInfo dev;
    st = current_device(&dev, nullptr);
    if (st != DG_OK) return st;
    GemmArgs a = {A, sA, B, sB, C_bf16, nullptr, static_cast<int64_t>(G) * M_max, N, K, G};
    a.masked_m = masked_m;
    a.m_max = M_max;
    return launch_tile_gemm(a, 2, dev, stream);
}

dg_status_t dg_fp8_grouped_gemm_contiguous(const uint8_t *A, const float *sA, const uint8_t *B, const float *sB,
                                           void *C_bf16, const int32_t *group_offsets, int64_t M_total_capacity,
                                           int G, int64_t N, int64_t K, cudaStream_t stream) {
    if (M_total_capacity < 0 || M_total_capacity % 128 != 0 || N < 0 || N % 128 != 0 || K <= 0 ||
        K % 16 != 0 || G < 1 || G > 1024)
        return DG_ERR_SHAPE;
    if (M_total_capacity > 0x7FFFFFFFLL || static_cast<int64_t>(G) * N > 0x7FFFFFFFLL || K > 0x7FFFFFFFLL)
        return DG_ERR_SHAPE;
    if (M_total_capacity == 0 || N == 0) return DG_OK;
    if (!group_offsets) return DG_ERR_INVALID_ARG;
    if (!aligned(group_offsets, 4)) return DG_ERR_ALIGNMENT;
    dg_status_t st = check_gemm_common(A, sA, B, sB, C_bf16);
    if (st != DG_OK) return st;
    DeviceInfo dev;
    st = current_device(&dev, nullptr);
    if (st != DG_OK) return st;
    GemmArgs a = {A, sA, B, sB, C_bf16, group_offsets, M_total_capacity, N, K, G};
    return launch_tile_gemm(a, 1, dev, stream);
}

}  // extern "C"
