// Skinny-M (M <= 128) FP8 block-scaled GEMM for sm_100a: the decode-style shape
// where the weight matrix B dominates the bytes and HBM bandwidth bounds the time
// (2kiu.com/news/5461879 §6: at M=16, N=K=4096 launch overhead and bandwidth
// dominate).
//
// Same formula as the tile kernel, computed as C^T = B * A^T ("swap AB"): a
// 128-row slab of B is the MMA's M=128 operand and the M tokens, padded to MP
// (a multiple of 16, rows beyond M zero-filled by TMA), are the MMA's N.  Each
// K block's partial sits in TMEM (lane = output column n, column = token m); the
// epilogue warps promote it with sB[n/128][kb] * sA[0][kb] into registers.
//
// Split-K without global scratch: a thread-block cluster of S CTAs shares one
// 128-column block of C and splits its K blocks S ways.  Each CTA leaves its
// FP32 partial tile in shared memory; after a cluster barrier, CTA r adds the S
// partials of its 128/S columns in rank order 0..S-1 through distributed shared
// memory and writes them as BF16.  The order is fixed, so the result is
// deterministic (no float atomics; demingchina.com/news/60142 §6.4).
#include <cuda_bf16.h>

#include "dg_device.cuh"
#include "dg_internal.h"

namespace dg {

struct SkinnyParams {
    const float *sA;
    const float *sB;
    __nv_bfloat16 *C;
    int M, N, Kb;
    int splits;
    uint64_t timeout_ns;
    int *status;  // device status word
};

constexpr int kSkinnyThreads = 256;

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_addr), "r"(rank));
    return out;
}

__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}

// 16 consecutive FP32 TMEM columns of this warp's 32 lanes, waited on.
__device__ __forceinline__ void tmem_load16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

template <int MP, int STAGES>
struct SkinnySmem {
    static constexpr uint32_t kWBytes = 128 * 128;  // weight slab: 128 rows of B x 128 K
    static constexpr uint32_t kXBytes = MP * 128;   // token slab: MP rows of A x 128 K
    static constexpr uint32_t kOffW = 0;
    static constexpr uint32_t kOffX = kOffW + STAGES * kWBytes;
    static constexpr uint32_t kStageEnd = kOffX + STAGES * kXBytes;
    static constexpr uint32_t kRedBytes = MP * 128 * 4;  // FP32 partial, [MP][128]
    static constexpr uint32_t kDataBytes = kStageEnd > kRedBytes ? kStageEnd : kRedBytes;
    static constexpr uint32_t kOffBar = kDataBytes;
    static constexpr uint32_t kOffMisc = kOffBar + 8 * (2 * STAGES + 4);
    static constexpr uint32_t kBytes = kOffMisc + 16;
    static constexpr uint32_t kDynamicBytes = kBytes + 1024;
};

template <int MP, int STAGES>
__global__ void __launch_bounds__(kSkinnyThreads, 1)
    skinny_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const SkinnyParams p) {
    using L = SkinnySmem<MP, STAGES>;
    constexpr uint32_t kTmemCols = (2 * MP < 32) ? 32 : 2 * MP;
    constexpr uint32_t kIdesc = idesc_e4m3_f32(128, MP);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
    float *red = reinterpret_cast<float *>(smem);  // reuses the stage memory after the K loop

    const int warp = static_cast<int>(threadIdx.x >> 5);
    const int lane = lane_id();
    const int S = p.splits;
    const int rank = static_cast<int>(cluster_rank());
    const int nb = static_cast<int>(blockIdx.x) / S;
    const int kb0 = static_cast<int>((static_cast<int64_t>(p.Kb) * rank) / S);
    const int kb1 = static_cast<int>((static_cast<int64_t>(p.Kb) * (rank + 1)) / S);
    const int nkb = kb1 - kb0;

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmW);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0 && lane == 0) {
        // -------------------------------------------------------------- producer
        uint32_t issued = 0, parity_bits = 0;
        for (int i = 0; i < nkb; ++i) {
            const int s = i % STAGES;
            const uint32_t u = static_cast<uint32_t>(i / STAGES);
            if (!mbar_wait(&empty[s], (u & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
                record_failure(p.status, kStatusTimeout, 10, i);
                *abort_flag = 1;
                break;
            }
            const int kb = kb0 + i;
            mbar_arrive_expect_tx(&full[s], L::kWBytes + L::kXBytes);
            tma_load_2d(smem + L::kOffW + s * L::kWBytes, &tmW, &full[s], kb * 128, nb * 128);
            tma_load_2d(smem + L::kOffX + s * L::kXBytes, &tmX, &full[s], kb * 128, 0);
            issued |= 1u << s;
            parity_bits = (parity_bits & ~(1u << s)) | ((u & 1u) << s);
        }
        const int never = 0;
        for (int s = 0; s < STAGES; ++s)
            if (issued & (1u << s))
                if (!mbar_wait(&full[s], (parity_bits >> s) & 1u, &never, p.timeout_ns))
                    record_failure(p.status, kStatusTimeout, 10, -1 - s);
    } else if (warp == 1 && lane == 0) {
        // ------------------------------------------------------------------- MMA
        const uint32_t w0 = smem_u32(smem + L::kOffW);
        const uint32_t x0 = smem_u32(smem + L::kOffX);
        int done = 0;
        for (int i = 0; i < nkb; ++i) {
            const int s = i % STAGES;
            const uint32_t u = static_cast<uint32_t>(i / STAGES);
            const int buf = i & 1;
            const uint32_t v = static_cast<uint32_t>(i >> 1);
            if (!mbar_wait(&tempty[buf], (v & 1u) ^ 1u, abort_flag, p.timeout_ns) ||
                !mbar_wait(&full[s], u & 1u, abort_flag, p.timeout_ns)) {
                record_failure(p.status, kStatusTimeout, 11, i);
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint64_t wdesc = sdesc_kmajor_sw128(w0 + s * L::kWBytes);
            const uint64_t xdesc = sdesc_kmajor_sw128(x0 + s * L::kXBytes);
            const uint32_t d = tmem_base + static_cast<uint32_t>(buf * MP);
#pragma unroll
            for (int k = 0; k < 4; ++k) umma_e4m3(d, wdesc + 2u * k, xdesc + 2u * k, kIdesc, k > 0 ? 1u : 0u);
            umma_commit(&empty[s]);
            umma_commit(&tfull[buf]);
            done = i + 1;
        }
        if (done > 0) {
            const int never = 0;
            const int last = done - 1;
            if (!mbar_wait(&tfull[last & 1], static_cast<uint32_t>(last >> 1) & 1u, &never, p.timeout_ns))
                record_failure(p.status, kStatusTimeout, 11, -1);
        }
    } else if (warp >= 4) {
        // -------------------------------------------------------------- epilogue
        const int quarter = warp & 3;
        const int row = quarter * 32 + lane;  // output column n = nb*128 + row
        float acc[MP];
#pragma unroll
        for (int j = 0; j < MP; ++j) acc[j] = 0.0f;
        ScaleStream scales;
        scales.start(p.sA, p.sB + static_cast<int64_t>(nb) * p.Kb, kb0, kb1);
        bool ok = true;
        for (int i = 0; i < nkb; ++i) {
            const int buf = i & 1;
            const uint32_t v = static_cast<uint32_t>(i >> 1);
            const int kb = kb0 + i;
            const float scale = scales.scale(kb, i);
            if (!mbar_wait(&tfull[buf], v & 1u, abort_flag, p.timeout_ns)) {
                record_failure(p.status, kStatusTimeout, 12, i);
                *abort_flag = 1;
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(buf * MP);
            if constexpr (MP == 16) {
                float part[16];
                tmem_load16(taddr, part);
#pragma unroll
                for (int j = 0; j < 16; ++j) acc[j] = fmaf(scale, part[j], acc[j]);
            } else {
#pragma unroll
                for (int c = 0; c < MP / 32; ++c) {
                    float part[32];
                    tmem_load32(taddr + c * 32, part);
#pragma unroll
                    for (int j = 0; j < 32; ++j) acc[c * 32 + j] = fmaf(scale, part[j], acc[c * 32 + j]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[buf]);
        }
        // Every MMA of this CTA must be complete before the stage memory is reused
        // for the partial tile: the MMA warp's last commit arrives on tfull.
        if (ok && nkb > 0) {
            const int last = nkb - 1;
            const int never = 0;
            mbar_wait(&tfull[last & 1], static_cast<uint32_t>(last >> 1) & 1u, &never, p.timeout_ns);
        }
        // partial tile, [MP][128]: consecutive threads write consecutive words
#pragma unroll
        for (int j = 0; j < MP; ++j) red[j * 128 + row] = acc[j];
    }

    // ---------------------------------------------- split-K reduction over the cluster
    __syncwarp();
    cluster_sync_all();
    {
        const int W = 128 / S;            // columns of the block this CTA finishes
        const int groups = W / 4;         // 4 columns per item
        const int items = p.M * groups;
        const uint32_t red0 = smem_u32(red);
        for (int it = static_cast<int>(threadIdx.x); it < items; it += kSkinnyThreads) {
            const int m = it / groups;
            const int nl = rank * W + (it - m * groups) * 4;
            const uint32_t off = static_cast<uint32_t>((m * 128 + nl) * 4);
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int r = 0; r < S; ++r) {  // fixed order: deterministic
                const float4 v = ld_cluster_f4(map_to_rank(red0 + off, static_cast<uint32_t>(r)));
                sum.x += v.x;
                sum.y += v.y;
                sum.z += v.z;
                sum.w += v.w;
            }
            const int n = nb * 128 + nl;
            if (n < p.N) {
                uint2 w;
                w.x = pack_bf16x2(sum.x, sum.y);
                w.y = pack_bf16x2(sum.z, sum.w);
                *reinterpret_cast<uint2 *>(p.C + static_cast<int64_t>(m) * p.N + n) = w;
            }
        }
    }
    // no CTA may leave while its peers still read its shared memory
    __syncwarp();
    cluster_sync_all();

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

template <int MP, int STAGES>
static dg_status_t launch_skinny_impl(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream) {
    using L = SkinnySmem<MP, STAGES>;
    static_assert(L::kDynamicBytes <= 232448, "shared memory budget");
    CUtensorMap tmW, tmX;
    dg_status_t st = make_tmap_2d(&tmW, a.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.N, a.K, 128, 128,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DG_OK) return st;
    st = make_tmap_2d(&tmX, a.A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.M, a.K, MP, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DG_OK) return st;

    auto kernel = skinny_gemm_kernel<MP, STAGES>;
    static thread_local int configured_device = -1;
    int device = 0;
    cudaGetDevice(&device);
    if (configured_device != device) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(L::kDynamicBytes)) != cudaSuccess ||
            cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0) != cudaSuccess)
            return DG_ERR_CUDA;
        configured_device = device;
    }

    const int Kb = static_cast<int>(a.K / 128);
    const int Nt = static_cast<int>((a.N + 127) / 128);
    // Split K so that the clusters cover the SMs about once: S in {1,2,4,8}, S <= Kb.
    int S = 1;
    while (S < 8 && 2 * S <= Kb && static_cast<int64_t>(Nt) * 2 * S <= dev.num_sms) S *= 2;

    SkinnyParams p;
    p.sA = a.sA;
    p.sB = a.sB;
    p.C = static_cast<__nv_bfloat16 *>(a.C);
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.Kb = Kb;
    p.splits = S;
    p.timeout_ns = kernel_control().timeout_ns;
    p.status = kernel_control().status;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(Nt * S), 1, 1);
    cfg.blockDim = dim3(kSkinnyThreads, 1, 1);
    cfg.dynamicSmemBytes = L::kDynamicBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(S);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, tmW, tmX, p) != cudaSuccess) return DG_ERR_CUDA;
    return DG_OK;
}

dg_status_t launch_skinny_gemm(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream) {
    if (a.M <= 16) return launch_skinny_impl<16, 8>(a, dev, stream);
    if (a.M <= 32) return launch_skinny_impl<32, 8>(a, dev, stream);
    if (a.M <= 64) return launch_skinny_impl<64, 8>(a, dev, stream);
    return launch_skinny_impl<128, 6>(a, dev, stream);
}

}  // namespace dg
