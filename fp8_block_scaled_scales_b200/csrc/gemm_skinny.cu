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
//
// Fused activation quantization (FUSED): A arrives as BF16 and four more warps
// quantize it per 128x128 block (for M <= 16 the block of K block kb is rows
// 0..M-1 x its 128 columns) straight into the MMA's shared-memory stage, in the
// 128-byte-swizzled K-major layout TMA would have written, with exactly the
// arithmetic of the block quantizer (quant_e4m3.cuh).  The step before the GEMM
// thus needs no launch of its own (2kiu.com/news/5461879 §5: activation scales
// are recomputed on every call).  Each warp owns every fourth K block: it loads
// the block's M x 128 values from global memory, reduces amax with shuffles and
// converts, so four K blocks are quantized at once and no block waits on a
// CTA-wide barrier; the weight stream does not wait for the quantizer.  The CTAs
// of the first N block also write the codes and scales out, so the caller gets
// the same Q, S as from the quantizer.  Every N block's CTAs repeat the
// quantization of their K range (M x K values, small next to the weights).
#include <cuda_bf16.h>

#include "dg_device.cuh"
#include "dg_internal.h"
#include "quant_e4m3.cuh"

namespace dg {

struct SkinnyParams {
    const float *sA;  // null when FUSED (the kernel derives the scales)
    const float *sB;
    __nv_bfloat16 *C;
    int M, N, Kb;
    int splits;
    uint64_t timeout_ns;
    int *status;  // device status word
    int debug_flags;  // bit 0 (tests): the producer never fills stage 0, so a wait must time out
    // FUSED only: BF16 A [M][K], and the codes / scales written by the first N block
    const uint4 *Xa;
    int K;
    uint8_t *qa_out;
    float *sa_out;
};

// Epilogue warps: four (one per TMEM lane quarter), or for 128-row token slabs eight,
// two per quarter each taking half the slab's columns, which halves the per-K-block
// TMEM read and promotion (measured: M = 128 step 13.36 -> 13.13 us; at M = 64 the
// extra warps cost more than they save, 9.60 -> 9.76 us).
template <int MP, bool FUSED>
constexpr int skinny_epi_warps() { return (!FUSED && MP == 128) ? 8 : 4; }
template <int MP, bool FUSED>
constexpr int skinny_threads() { return (FUSED || skinny_epi_warps<MP, FUSED>() == 8) ? 384 : 256; }

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

template <int MP, int STAGES, int NBUF>
struct SkinnySmem {
    static constexpr uint32_t kWBytes = 128 * 128;  // weight slab: 128 rows of B x 128 K
    static constexpr uint32_t kXBytes = MP * 128;   // token slab: MP rows of A x 128 K
    static constexpr uint32_t kOffW = 0;
    static constexpr uint32_t kOffX = kOffW + STAGES * kWBytes;
    static constexpr uint32_t kStageEnd = kOffX + STAGES * kXBytes;
    static constexpr uint32_t kRedBytes = MP * 128 * 4;  // FP32 partial, [MP][128]
    static constexpr uint32_t kDataBytes = kStageEnd > kRedBytes ? kStageEnd : kRedBytes;
    static constexpr uint32_t kOffBar = kDataBytes;
    static constexpr uint32_t kOffMisc = kOffBar + 8 * (2 * STAGES + 2 * NBUF + 2);
    // misc: TMEM address (0), abort flag (4)
    static constexpr uint32_t kOffScaleA = kOffMisc + 16;  // FUSED: A scale of each stage
    static constexpr uint32_t kBytes = kOffScaleA + 4 * STAGES;
    static constexpr uint32_t kDynamicBytes = kBytes + 1024;
};

// All threads of the cluster; the arrival does not order earlier memory accesses
// (used where every shared-memory read the peers depend on has already returned).
__device__ __forceinline__ void cluster_sync_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}

template <int MP, int STAGES, int NBUF, bool FUSED>
__global__ void __launch_bounds__(skinny_threads<MP, FUSED>(), 1)
    skinny_gemm_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const SkinnyParams p) {
    constexpr int kThreads = skinny_threads<MP, FUSED>();
    constexpr int kEpiWarps = skinny_epi_warps<MP, FUSED>();
    constexpr int kEpiCols = MP * 4 / kEpiWarps;  // token columns per epilogue warp
    using L = SkinnySmem<MP, STAGES, NBUF>;
    static_assert(STAGES % 2 == 0 && NBUF % 2 == 0, "each MMA thread must own its stages and buffers");
    constexpr uint32_t kTmemCols = tmem_cols_for(NBUF * MP);
    constexpr uint32_t kIdesc = idesc_e4m3_f32(128, MP);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + NBUF;
    uint64_t *mdone = tempty + NBUF;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
    float *red = reinterpret_cast<float *>(smem);  // reuses the stage memory after the K loop
    float *sa_stage = reinterpret_cast<float *>(smem + L::kOffScaleA);

    const int warp = static_cast<int>(threadIdx.x >> 5);
    const int lane = lane_id();
    const int S = p.splits;
    const int rank = static_cast<int>(cluster_rank());
    const int nb = static_cast<int>(blockIdx.x) / S;
    const int kb0 = static_cast<int>((static_cast<int64_t>(p.Kb) * rank) / S);
    const int kb1 = static_cast<int>((static_cast<int64_t>(p.Kb) * (rank + 1)) / S);
    const int nkb = kb1 - kb0;

    // The weight slabs do not depend on the previous kernel in a decode loop, but
    // they may; an L2 prefetch is safe either way, so it starts the weight stream
    // before the dependency wait, overlapping the tail of the previous kernel.
    if (warp == 2 && lane == 0)
        for (int kb = kb0; kb < kb1; ++kb) tma_prefetch_l2_2d(&tmW, kb * 128, nb * 128);

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            // FUSED: a stage is full once the weight slab landed and the quantizer
            // warps wrote the token slab; it is empty once every epilogue warp has
            // read the stage's A scale
            mbar_init(&full[s], FUSED ? 2 : 1);
            mbar_init(&empty[s], FUSED ? 4 : 1);
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], kEpiWarps);
        }
        for (int q = 0; q < 2; ++q) mbar_init(&mdone[q], 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmW);
        if (!FUSED) tma_prefetch_desc(&tmX);
    }
    if (warp == 3) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    grid_dep_wait();  // inputs and outputs are touched only from here on
    grid_dep_launch_dependents();

    if ((warp == 0 || warp == 3) && lane == 0) {
        // ------------------------------------------------------------- producers
        // Two threads, one per parity of the K block (one thread's issue of a stage
        // takes ~600 cycles, measured; the whole K range is issued up front, so this
        // halves the time to the last copy).
        const int np = 2;
        const int pr = warp == 0 ? 0 : 1;
        uint32_t issued = 0, parity_bits = 0;
        for (int i = pr; i < nkb; i += np) {
            const int s = i % STAGES;
            const uint32_t u = static_cast<uint32_t>(i / STAGES);
            const int kb = kb0 + i;
            if (!mbar_wait(&empty[s], (u & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
                record_failure(p.status, kStatusTimeout, 10, i);
                *abort_flag = 1;
                break;
            }
            if ((p.debug_flags & 1) && i == 0) continue;  // test hook: stage 0 never filled
            mbar_arrive_expect_tx(&full[s], FUSED ? L::kWBytes : L::kWBytes + L::kXBytes);
            tma_load_2d(smem + L::kOffW + s * L::kWBytes, &tmW, &full[s], kb * 128, nb * 128);
            if (!FUSED) tma_load_2d(smem + L::kOffX + s * L::kXBytes, &tmX, &full[s], kb * 128, 0);
            issued |= 1u << s;
            parity_bits = (parity_bits & ~(1u << s)) | ((u & 1u) << s);
        }
        const int never = 0;
        for (int s = 0; s < STAGES; ++s)
            if (issued & (1u << s))
                if (!mbar_wait(&full[s], (parity_bits >> s) & 1u, &never, p.timeout_ns))
                    record_failure(p.status, kStatusTimeout, 10, -1 - s);
    } else if ((warp == 1 || warp == 2) && lane == 0) {
        // -------------------------------------------------- MMA (two threads)
        // Thread q issues K blocks i with i % 2 == q; with STAGES and NBUF even
        // each stage and buffer belongs to one thread (in-order parity waits).
        const int q = warp - 1;
        const uint32_t w0 = smem_u32(smem + L::kOffW);
        const uint32_t x0 = smem_u32(smem + L::kOffX);
        int last = -1;
        for (int i = q; i < nkb; i += 2) {
            const int s = i % STAGES;
            const uint32_t u = static_cast<uint32_t>(i / STAGES);
            const int buf = i % NBUF;
            const uint32_t v = static_cast<uint32_t>(i / NBUF);
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
            // unfused: the stage is free once these MMAs have read it (fused, the
            // epilogue frees it after reading the stage's A scale)
            if (!FUSED) umma_commit(&empty[s]);
            umma_commit(&tfull[buf]);
            last = i;
        }
        if (last >= 0) {
            const int never = 0;
            umma_commit(&mdone[q]);
            if (!mbar_wait(&mdone[q], 0, &never, p.timeout_ns)) record_failure(p.status, kStatusTimeout, 11, -1);
        }
    } else if (FUSED && warp >= 8) {
        // ------------------------------------------ activation quantizer (FUSED)
        // Warp qw quantizes K blocks qw, qw + 4, ...: item (row r, 8-column group g)
        // = lane + 32 t holds A[r][kb*128 + 8g .. +7]; rows past M and columns past K
        // are zero and quantize to +0.  The codes go where TMA would have put them in
        // the 128-byte-swizzled K-major stage: row r's 16-byte group j at byte
        // r*128 + ((j ^ (r % 8)) * 16).
        // The loads of the warp's next K block are issued before the current one is
        // converted, so one load latency is exposed per warp, not one per K block.
        const int qw = warp - 8;
        constexpr int kItems = MP * 16 / 32;
        auto load_block = [&](int i, uint4(&v)[kItems]) {
            const int64_t colbase = static_cast<int64_t>(kb0 + i) * 128;
#pragma unroll
            for (int t = 0; t < kItems; ++t) {
                const int item = lane + 32 * t;
                const int r = item >> 4;
                const int64_t col = colbase + (item & 15) * 8;
                v[t] = make_uint4(0, 0, 0, 0);
                if (i < nkb && r < p.M && col < p.K)  // K % 16 == 0: a group is whole or absent
                    v[t] = p.Xa[(static_cast<int64_t>(r) * p.K + col) >> 3];
            }
        };
        uint4 v[kItems], vn[kItems];
        load_block(qw, v);
        for (int i = qw; i < nkb; i += 4) {
            const int s = i % STAGES;
            const uint32_t u = static_cast<uint32_t>(i / STAGES);
            const int64_t colbase = static_cast<int64_t>(kb0 + i) * 128;
            load_block(i + 4, vn);
            uint32_t m2 = 0;
#pragma unroll
            for (int t = 0; t < kItems; ++t) m2 = amax_fold8(m2, v[t]);
            uint32_t ab = amax_bits_of(m2);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ab = max(ab, __shfl_xor_sync(0xFFFFFFFFu, ab, o));
            const BlockScale bs = block_scale(ab);
            // the stage's previous K block has been consumed by its MMAs and its A
            // scale read by the epilogue
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&empty[s], (u & 1u) ^ 1u, abort_flag, p.timeout_ns) ? 1 : 0;
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) {
                if (lane == 0) {
                    record_failure(p.status, kStatusTimeout, 13, i);
                    *abort_flag = 1;
                }
                break;
            }
            uint8_t *xs = smem + L::kOffX + s * L::kXBytes;
            uint2 codes[kItems];
#pragma unroll
            for (int t = 0; t < kItems; ++t) {
                const int item = lane + 32 * t;
                const int r = item >> 4, g = item & 15;
                codes[t] = make_uint2(0, 0);
                if (r < p.M && colbase + g * 8 < p.K) codes[t] = quantize8(v[t], bs);
                *reinterpret_cast<uint2 *>(xs + r * 128 + (((g >> 1) ^ (r & 7)) << 4) + (g & 1) * 8) = codes[t];
            }
            if (lane == 0) sa_stage[s] = bs.s;
            fence_async_smem();  // the codes are read by the tensor cores (async proxy)
            __syncwarp();
            if (lane == 0) mbar_arrive(&full[s]);
            if (nb == 0) {  // the caller's copy, off the MMA's path
#pragma unroll
                for (int t = 0; t < kItems; ++t) {
                    const int item = lane + 32 * t;
                    const int r = item >> 4;
                    const int64_t col = colbase + (item & 15) * 8;
                    if (r < p.M && col < p.K)
                        *reinterpret_cast<uint2 *>(p.qa_out + static_cast<int64_t>(r) * p.K + col) = codes[t];
                }
                if (lane == 0) p.sa_out[kb0 + i] = bs.s;
            }
#pragma unroll
            for (int t = 0; t < kItems; ++t) v[t] = vn[t];
        }
    } else if (warp >= 4 && warp < 4 + kEpiWarps) {
        // -------------------------------------------------------------- epilogue
        const int quarter = warp & 3;
        const int col0 = ((warp - 4) >> 2) * kEpiCols;  // this warp's first token column
        const int row = quarter * 32 + lane;  // output column n = nb*128 + row
        float2 acc[kEpiCols / 2];
#pragma unroll
        for (int j = 0; j < kEpiCols / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
        ScaleStream scales;
        scales.start(p.sA, p.sB + static_cast<int64_t>(nb) * p.Kb, kb0, kb1);
        for (int i = 0; i < nkb; ++i) {
            const int buf = i % NBUF;
            const uint32_t v = static_cast<uint32_t>(i / NBUF);
            const int kb = kb0 + i;
            float scale = scales.scale(kb, i);
            if (!mbar_wait(&tfull[buf], v & 1u, abort_flag, p.timeout_ns)) {
                record_failure(p.status, kStatusTimeout, 12, i);
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            if (FUSED) {
                // the MMAs of this K block are done: the stage may be refilled once
                // every epilogue warp has read its A scale
                // the stage's A scale, published with the stage's full phase (which
                // is complete, and cannot advance before this warp's empty arrival)
                const int s = i % STAGES;
                if (!mbar_wait(&full[s], static_cast<uint32_t>(i / STAGES) & 1u, abort_flag, p.timeout_ns)) {
                    record_failure(p.status, kStatusTimeout, 12, i);
                    *abort_flag = 1;
                    break;
                }
                scale = scale * sa_stage[s];  // = fl32(sA * sB), as in the unfused path
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            const float2 s2 = make_float2(scale, scale);
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                   static_cast<uint32_t>(buf * MP + col0);
            constexpr int kChunks = kEpiCols / 16;
            uint32_t r0[16], r1[16];
            tmem_load16_async(taddr, r0);
            tmem_wait16(r0);
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                uint32_t(&cur)[16] = (c & 1) ? r1 : r0;
                uint32_t(&nxt)[16] = (c & 1) ? r0 : r1;
                if (c + 1 < kChunks) {
                    tmem_load16_async(taddr + (c + 1) * 16, nxt);
                } else {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tempty[buf]);
                }
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    acc[c * 8 + j] = __ffma2_rn(make_float2(__uint_as_float(cur[2 * j]), __uint_as_float(cur[2 * j + 1])),
                                                s2, acc[c * 8 + j]);
                if (c + 1 < kChunks) tmem_wait16(nxt);
            }
        }
        // every MMA of this CTA has completed once the epilogue saw its last tfull
        // (or the MMA threads drained after a failure), so the stage memory may now
        // hold the partial tile, [MP][128]: consecutive threads write consecutive words
        bar_named_sync(1, 32 * kEpiWarps);  // every epilogue warp: all TMEM reads done
#pragma unroll
        for (int j = 0; j < kEpiCols / 2; ++j) {
            red[(col0 + 2 * j) * 128 + row] = acc[j].x;
            red[(col0 + 2 * j + 1) * 128 + row] = acc[j].y;
        }
    }

    // ---------------------------------------------- split-K reduction over the cluster
    __syncwarp();
    cluster_sync_all();
    {
        const int W = 128 / S;            // columns of the block this CTA finishes
        const int groups = W / 4;         // 4 columns per item
        const int items = p.M * groups;
        const uint32_t red0 = smem_u32(red);
        for (int it = static_cast<int>(threadIdx.x); it < items; it += kThreads) {
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
    // no CTA may leave while its peers still read its shared memory; every read a
    // peer depends on has returned by the time it arrives
    __syncwarp();
    cluster_sync_relaxed();

    tc_fence_before();
    __syncthreads();
    if (warp == 3) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

template <int MP, int STAGES, int NBUF, bool FUSED>
static dg_status_t launch_skinny_impl(const GemmArgs &a, const uint16_t *Xa, uint8_t *qa_out, float *sa_out,
                                      const DeviceInfo &dev, cudaStream_t stream) {
    using L = SkinnySmem<MP, STAGES, NBUF>;
    static_assert(L::kDynamicBytes <= 232448, "shared memory budget");
    CUtensorMap tmW, tmX;
    dg_status_t st = make_tmap_2d(&tmW, a.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.N, a.K, 128, 128,
                                  CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DG_OK) return st;
    if (FUSED) {
        tmX = tmW;  // unused: the quantizer warps read A from global memory
    } else {
        st = make_tmap_2d(&tmX, a.A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.M, a.K, MP, 128, CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != DG_OK) return st;
    }

    auto kernel = skinny_gemm_kernel<MP, STAGES, NBUF, FUSED>;
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

    const int Kb = static_cast<int>((a.K + 127) / 128);
    const int Nt = static_cast<int>((a.N + 127) / 128);
    // Split K so that the clusters cover the SMs about once: S in {1,2,4,8}, S <= Kb.
    int S = 1;
    while (S < 8 && 2 * S <= Kb && static_cast<int64_t>(Nt) * 2 * S <= dev.num_sms) S *= 2;

    SkinnyParams p;
    p.sA = FUSED ? nullptr : a.sA;
    p.sB = a.sB;
    p.C = static_cast<__nv_bfloat16 *>(a.C);
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.Kb = Kb;
    p.splits = S;
    p.timeout_ns = kernel_control().timeout_ns;
    p.status = kernel_control().status;
    p.debug_flags = kernel_control().debug_flags;
    p.Xa = reinterpret_cast<const uint4 *>(Xa);
    p.K = static_cast<int>(a.K);
    p.qa_out = qa_out;
    p.sa_out = sa_out;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(Nt * S), 1, 1);
    cfg.blockDim = dim3(static_cast<unsigned>(skinny_threads<MP, FUSED>()), 1, 1);
    cfg.dynamicSmemBytes = L::kDynamicBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(S);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, kernel, tmW, tmX, p) != cudaSuccess) return DG_ERR_CUDA;
    return DG_OK;
}

dg_status_t launch_skinny_gemm(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream) {
    if (a.M <= 16) return launch_skinny_impl<16, 8, 8, false>(a, nullptr, nullptr, nullptr, dev, stream);
    if (a.M <= 32) return launch_skinny_impl<32, 8, 8, false>(a, nullptr, nullptr, nullptr, dev, stream);
    if (a.M <= 64) return launch_skinny_impl<64, 8, 8, false>(a, nullptr, nullptr, nullptr, dev, stream);
    return launch_skinny_impl<128, 6, 4, false>(a, nullptr, nullptr, nullptr, dev, stream);
}

dg_status_t launch_skinny_gemm_fused(const GemmArgs &a, const void *A_bf16, uint8_t *qa_out, float *sa_out,
                                     const DeviceInfo &dev, cudaStream_t stream) {
    const uint16_t *x = static_cast<const uint16_t *>(A_bf16);
    static_assert(kFusedMaxM <= 16, "one token slab of 16 rows");
    if (a.M <= kFusedMaxM) return launch_skinny_impl<16, 8, 8, true>(a, x, qa_out, sa_out, dev, stream);
    return DG_ERR_SHAPE;
}

}  // namespace dg
