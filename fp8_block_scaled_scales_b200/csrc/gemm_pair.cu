// CTA-pair (cta_group::2) FP8 block-scaled GEMM tile kernel for sm_100a, dense form,
// with 128x128 A scales or (ROWS) one A scale per row and K block.
//
// Same method and roles as the single-CTA tile kernel (gemm_tile.cu): per 128-wide
// K block the tensor cores produce P_kb in FP32 in tensor memory and the epilogue
// warps promote it, acc += sA[m/128][kb] * sB[n/128][kb] * P_kb, in ascending kb
// (2kiu.com/news/5461879 §2.1, §3.3).  What changes is the MMA shape: the two CTAs
// of a cluster pair compute one 256 x BN output tile together.  Each CTA loads its
// own 128 rows of A and its own half (BN/2 rows) of the B tile; the even CTA's MMA
// warp issues tcgen05.mma.cta_group::2 with M = 256, which reads the A halves from
// both CTAs' shared memory, shares the two B halves across the pair and writes
// each CTA's 128 rows x BN columns into that CTA's tensor memory.
//
// Per CTA and K block this moves 16 KB of A plus BN/2 x 128 bytes of B through
// shared memory instead of 16 KB + BN x 128 bytes, so the same shared memory holds
// a deeper ring (6 stages of 32 KB for BN = 256), and every B tile is fetched from
// L2 once per pair.  The pages' cluster sharing of B tiles between neighbouring
// CTAs (demingchina.com/news/60142 §3.4) is done here by the pair MMA itself, with
// no multicast copy.
//
// Synchronisation across the pair:
//   full[s]    even CTA only: its producer posts the byte count of both CTAs' loads,
//              both producers' TMA loads complete on it.
//   empty[s]   in both CTAs: the MMA thread's commit (multicast) arrives on both once
//              the pair's MMAs that read the stage are done, however far behind
//              the epilogue runs.
//   tfull[b]   in both CTAs: the MMA commit (multicast) arrives on both.
// Two threads of the even CTA issue the MMAs, alternating K blocks.
//   tempty[b]  even CTA only: all 16 epilogue warps of the pair arrive on it.
// All waits are CTA-scope polls of the waiting CTA's own barrier.  The remote
// arrivals only hand back tensor memory, whose reads are ordered by tcgen05
// fences, not generic memory, so they use the default CTA-scope semantics (a
// cluster-scope release fenced every arrival and halved the throughput).
#include <cuda_bf16.h>

#include "dg_device.cuh"
#include "dg_internal.h"

namespace dg {

struct PairParams {
    const float *sA;
    const float *sB;
    int num_m;        // m-blocks: ceil(M / 128)
    int num_n_tiles;  // ceil(N / BN)
    int M, N;
    int Nb;           // ceil(N / 128)
    int Kb;           // ceil(K / 128); the last K block may be partial
    int tiles_wide;   // tiles [0, tiles_wide) run 256 x BN; each later tile runs as two 256 x BN/2 halves
    int num_units;    // tiles_wide + 2 * (tiles - tiles_wide)
    uint64_t timeout_ns;
    int *status;
    int debug_flags;
};

constexpr int kPairThreads = 384;
constexpr int kPairRegsLaunch = 168;
template <int BN> __host__ __device__ constexpr int pair_regs_producer() { return BN == 256 ? 56 : 64; }
template <int BN> __host__ __device__ constexpr int pair_regs_epilogue() { return BN == 256 ? 224 : 216; }
static_assert(128 * pair_regs_producer<256>() + 256 * pair_regs_epilogue<256>() <= kPairThreads * kPairRegsLaunch &&
                  128 * pair_regs_producer<128>() + 256 * pair_regs_epilogue<128>() <= kPairThreads * kPairRegsLaunch,
              "setmaxnreg split exceeds the registers the block is launched with");
constexpr int kPairRasterM = 4;  // m-pairs per raster group

__device__ __forceinline__ void pair_tile_coords(int t, int num_mp, int num_n, int &mp, int &nb) {
    const int group = t / (kPairRasterM * num_n);
    const int first = group * kPairRasterM;
    const int gm = min(kPairRasterM, num_mp - first);
    const int local = t - group * kPairRasterM * num_n;
    mp = first + local % gm;
    nb = local / gm;
}

// A unit of work: a whole 256 x BN tile, or (in the last round, see the launcher)
// one 256 x BN/2 half of one.  Column n0 is the unit's first output column.
struct PairUnit {
    int mp;     // m-pair: rows 256 mp .. 256 mp + 255
    int n0;     // first column
    bool narrow;
};

template <int BN>
__device__ __forceinline__ PairUnit pair_unit(const PairParams &p, int num_mp, int u) {
    PairUnit w;
    int t = u, h = 0;
    w.narrow = u >= p.tiles_wide;
    if (w.narrow) {
        t = p.tiles_wide + (u - p.tiles_wide) / 2;
        h = (u - p.tiles_wide) & 1;
    }
    int nb;
    pair_tile_coords(t, num_mp, p.num_n_tiles, w.mp, nb);
    w.n0 = nb * BN + h * (BN / 2);
    return w;
}

template <int BN, int STAGES, int NBUF>
struct PairSmem {
    static constexpr uint32_t kABytes = 128 * 128;
    static constexpr uint32_t kBBytes = (BN / 2) * 128;
    static constexpr uint32_t kCBoxBytes = 32 * 64 * 2;
    static constexpr uint32_t kOffA = 0;
    static constexpr uint32_t kOffB = kOffA + STAGES * kABytes;
    static constexpr uint32_t kOffC = kOffB + STAGES * kBBytes;
    static constexpr uint32_t kOffBar = kOffC + 8 * kCBoxBytes;
    static constexpr uint32_t kNumBars = 2 * STAGES + 2 * NBUF + 2;
    static constexpr uint32_t kOffMisc = kOffBar + 8 * kNumBars;
    // misc: TMEM address (0), abort flag (4); then per stage the last iteration this
    // CTA's producer issued loads for (the leader: posted the byte count for)
    static constexpr uint32_t kOffIssued = kOffMisc + 16;
    static constexpr uint32_t kBytes = kOffIssued + 4 * STAGES;
    static constexpr uint32_t kDynamicBytes = kBytes + 1024;
};

__device__ __forceinline__ void mbar_complete_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.complete_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// ROWS: sA holds one scale per row of A and K block, K-block-major (sA[kb][m]);
// each epilogue thread promotes its row with its own scale.
template <int BN, int STAGES, int NBUF, bool ROWS>
__global__ void __launch_bounds__(kPairThreads, 1)
    pair_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmBn, const __grid_constant__ CUtensorMap tmC,
                     const PairParams p) {
    using L = PairSmem<BN, STAGES, NBUF>;
    constexpr int kColsPerWarp = BN / 2;
    constexpr uint32_t kTmemCols = tmem_cols_for(NBUF * BN);
    constexpr uint32_t kIdesc = idesc_e4m3_f32(256, BN);
    constexpr uint32_t kIdescNarrow = idesc_e4m3_f32(256, BN / 2);
    // bytes one CTA's loads bring per K block: A + its half of the B tile
    constexpr uint32_t kCtaBytes = L::kABytes + L::kBBytes;
    constexpr uint32_t kCtaBytesNarrow = L::kABytes + L::kBBytes / 2;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + NBUF;
    uint64_t *mdone = tempty + NBUF;  // one per MMA thread: all its MMAs complete
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
    int *issued = reinterpret_cast<int *>(smem + L::kOffIssued);

    const int warp = static_cast<int>(threadIdx.x >> 5);
    const int lane = lane_id();
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int num_pairs = static_cast<int>(gridDim.x >> 1);
    const int num_mp = (p.num_m + 1) / 2;
    const int Kb = p.Kb;
    // the units of this pair: pair, pair + num_pairs, ...
    const int my_units = pair < p.num_units ? (p.num_units - 1 - pair) / num_pairs + 1 : 0;
    auto unit_bytes = [&](int it) {  // one CTA's bytes in iteration `it`
        return (pair + (it / Kb) * num_pairs) >= p.tiles_wide ? kCtaBytesNarrow : kCtaBytes;
    };

    // L2 prefetch of this CTA's first B slabs, before the dependency wait (a cache
    // fill only, so it cannot observe stale data)
    if (warp == 3 && lane == 0 && my_units > 0) {
        const PairUnit w = pair_unit<BN>(p, num_mp, pair);
        const int rows = w.narrow ? BN / 4 : BN / 2;
        for (int kb = 0; kb < Kb && kb < 2 * STAGES; ++kb)
            tma_prefetch_l2_2d(w.narrow ? &tmBn : &tmB, kb * 128, w.n0 + static_cast<int>(rank) * rows);
    }

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            issued[s] = -1;
        }
        for (int q = 0; q < 2; ++q) mbar_init(&mdone[q], 1);
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 16);
        }
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmBn);
        tma_prefetch_desc(&tmC);
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, kTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    grid_dep_wait();  // inputs and outputs are touched only from here on
    grid_dep_launch_dependents();

    if (warp < 4) {
        regs_dealloc<pair_regs_producer<BN>()>();
        if ((warp == 0 || warp == 3) && lane == 0) {
            // --------------------------------------------- producers (both CTAs)
            // Two threads per CTA, one per parity of the iteration (one thread's
            // issue of a stage takes longer than the K block's MMAs, measured); with
            // STAGES even each stage belongs to one thread.
            const int pr = warp == 0 ? 0 : 1;
            const uint32_t full0 = mapa_shared(smem_u32(&full[0]), 0);  // the even CTA's full[0]
            int it = 0;
            bool ok = true;
            for (int i = 0; i < my_units && ok; ++i) {
                const PairUnit w = pair_unit<BN>(p, num_mp, pair + i * num_pairs);
                const int a_row = (2 * w.mp + static_cast<int>(rank)) * 128;
                const int b_row = w.n0 + static_cast<int>(rank) * (w.narrow ? BN / 4 : BN / 2);
                for (int kb = 0; kb < Kb; ++kb, ++it) {
                    if ((it & 1) != pr) continue;  // the other producer's stage
                    const int s = it % STAGES;
                    const uint32_t u = static_cast<uint32_t>(it / STAGES);
                    if (!mbar_wait(&empty[s], (u & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
                        record_failure(p.status, kStatusTimeout, 20 + static_cast<int>(rank), it);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                    if ((p.debug_flags & 1) && it == 0 && leader) continue;  // test hook: stage 0 never posted
                    if (leader) mbar_arrive_expect_tx(&full[s], 2 * (w.narrow ? kCtaBytesNarrow : kCtaBytes));
                    issued[s] = it;
                    tma_load_2d_pair(smem + L::kOffA + s * L::kABytes, &tmA, full0 + 8u * s, kb * 128, a_row);
                    tma_load_2d_pair(smem + L::kOffB + s * L::kBBytes, w.narrow ? &tmBn : &tmB, full0 + 8u * s,
                                     kb * 128, b_row);
                }
            }
        } else if ((warp == 1 || warp == 2) && lane == 0 && leader) {
            // ----------------------------------- MMA (even CTA only, two threads)
            // Thread q issues the K blocks kc with kc % 2 == q (independent partials,
            // each in its own TMEM buffer; with STAGES and NBUF even each stage and
            // buffer belongs to one thread, so its parity waits stay in order); one
            // multicast commit per K block.
            const int q = warp - 1;
            const int total = my_units * Kb;
            const uint32_t a0 = smem_u32(smem + L::kOffA);
            const uint32_t b0 = smem_u32(smem + L::kOffB);
            int last = -1;
            int unit = 0, kb = q;  // kc = unit * Kb + kb
            while (kb >= Kb) kb -= Kb, ++unit;
            for (int kc = q; kc < total; kc += 2) {
                const int s = kc % STAGES;
                const uint32_t u = static_cast<uint32_t>(kc / STAGES);
                const int buf = kc % NBUF;
                const uint32_t v = static_cast<uint32_t>(kc / NBUF);
                const bool narrow = pair + unit * num_pairs >= p.tiles_wide;
                if (!mbar_wait(&tempty[buf], (v & 1u) ^ 1u, abort_flag, p.timeout_ns) ||
                    !mbar_wait(&full[s], u & 1u, abort_flag, p.timeout_ns)) {
                    record_failure(p.status, kStatusTimeout, 22, kc);
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
                const uint64_t adesc = sdesc_kmajor_sw128(a0 + s * L::kABytes);
                const uint64_t bdesc = sdesc_kmajor_sw128(b0 + s * L::kBBytes);
                const uint32_t d = tmem_base + static_cast<uint32_t>(buf * BN);
                const uint32_t idesc = narrow ? kIdescNarrow : kIdesc;
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    umma_e4m3_pair(d, adesc + 2u * k, bdesc + 2u * k, idesc, k > 0 ? 1u : 0u);
                umma_commit_pair(&empty[s], 0x3);  // both CTAs' stage s is free once these MMAs have read it
                umma_commit_pair(&tfull[buf], 0x3);
                last = kc;
                kb += 2;
                while (kb >= Kb) kb -= Kb, ++unit;
            }
            if (last >= 0) {
                const int never = 0;
                umma_commit_pair(&mdone[q], 0x1);  // this CTA's barrier only
                if (!mbar_wait(&mdone[q], 0, &never, p.timeout_ns)) record_failure(p.status, kStatusTimeout, 22, -1);
            }
        }
    } else {
        regs_alloc<pair_regs_epilogue<BN>()>();
        // -------------------------------------------------- epilogue (both CTAs)
        const int ew = warp - 4;
        const int quarter = warp & 3;
        const int half = ew >> 2;
        uint8_t *cstage = smem + L::kOffC + ew * L::kCBoxBytes;
        const uint32_t tempty0 = mapa_shared(smem_u32(&tempty[0]), 0);  // the even CTA's tempty[0]
        float2 acc[kColsPerWarp / 2];
        int kc = 0;
        bool ok = true;
        for (int i = 0; i < my_units && ok; ++i) {
            const PairUnit w = pair_unit<BN>(p, num_mp, pair + i * num_pairs);
            // this warp's columns: BN/2 of a whole tile, BN/4 of a half tile
            const int ncols = (BN == 256 && w.narrow) ? kColsPerWarp / 2 : kColsPerWarp;
            const int mb = 2 * w.mp + static_cast<int>(rank);
            const int col0 = w.n0 + half * ncols;
            const int nb128 = col0 / 128;
            const bool valid = nb128 < p.Nb && mb < p.num_m;
            ScaleStream scales;
            scales.start(ROWS ? nullptr : p.sA + static_cast<int64_t>(valid ? mb : 0) * Kb,
                         p.sB + static_cast<int64_t>(valid ? nb128 : 0) * Kb, 0, valid ? Kb : 0);
            // ROWS: this thread's row scales, loaded two K blocks ahead
            const int my_row = mb * 128 + quarter * 32 + lane;
            const bool row_ok = ROWS && valid && my_row < p.M;
            float sa_next = row_ok ? __ldg(p.sA + my_row) : 0.0f;
            float sa_next2 = (row_ok && Kb > 1) ? __ldg(p.sA + p.M + my_row) : 0.0f;
#pragma unroll
            for (int j = 0; j < kColsPerWarp / 2; ++j) acc[j] = make_float2(0.0f, 0.0f);
            for (int kb = 0; kb < Kb; ++kb, ++kc) {
                const int buf = kc % NBUF;
                const uint32_t v = static_cast<uint32_t>(kc / NBUF);
                float scale = scales.scale(kb, kb);
                if (ROWS) {
                    const float sa = sa_next;
                    sa_next = sa_next2;
                    sa_next2 = (row_ok && kb + 2 < Kb) ? __ldg(p.sA + static_cast<int64_t>(kb + 2) * p.M + my_row) : 0.0f;
                    scale = sa * scale;  // fl32(sA[row][kb] * sB[n/128][kb])
                }
                const float2 s2 = make_float2(scale, scale);
                if (!mbar_wait(&tfull[buf], v & 1u, abort_flag, p.timeout_ns)) {
                    record_failure(p.status, kStatusTimeout, 24 + static_cast<int>(rank), kc);
                    *abort_flag = 1;
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                                       static_cast<uint32_t>(buf * BN + half * ncols);
                promote_kblock<kColsPerWarp, kPromoChunk>(taddr, s2, acc, ncols / kPromoChunk, [&] {
                    // this warp's columns of the buffer are in registers: hand it back
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(tempty0 + 8u * buf);
                });
            }
            if (!ok) break;
            const int row0 = mb * 128 + quarter * 32;
#pragma unroll
            for (int j = 0; j < kColsPerWarp / 64; ++j) {
                if (j * 64 >= ncols) break;
                if (lane == 0) bulk_wait_read0();
                __syncwarp();
                uint8_t *rowp = cstage + lane * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float2 *x = acc + j * 32 + c * 4;
                    uint4 q4;
                    q4.x = pack_bf16x2(x[0].x, x[0].y);
                    q4.y = pack_bf16x2(x[1].x, x[1].y);
                    q4.z = pack_bf16x2(x[2].x, x[2].y);
                    q4.w = pack_bf16x2(x[3].x, x[3].y);
                    *reinterpret_cast<uint4 *>(rowp + ((c ^ (lane & 7)) << 4)) = q4;
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0 && col0 + j * 64 < p.N && row0 < p.M) {
                    tma_store_2d(&tmC, cstage, col0 + j * 64, row0);
                    bulk_commit();
                }
            }
        }
        if (lane == 0) bulk_wait_all0();
    }

    // Neither CTA may leave while a load it issued can still land in its shared
    // memory or signal a barrier.  Every load completes on the even CTA's full[s],
    // whose phase for iteration `it` counts both CTAs' bytes once the even CTA has
    // posted them.  After a normal run every posted phase has completed (the MMAs
    // consumed them); after a timeout the even CTA drains each stage: the odd CTA's
    // last load on a stage is either in the phase the even CTA posted last, or one
    // phase later (it cannot run further ahead: its stage must first be freed by an
    // MMA that waited for that phase).  Bytes that were posted but will never be sent
    // (the odd CTA stopped first) are completed by hand; bytes sent for a phase
    // never posted are posted now.  Every wait is bounded.
    tc_fence_before();
    __syncwarp();
    cluster_sync();
    if (leader && warp == 0 && lane == 0) {
        const uint32_t peer_issued = mapa_shared(smem_u32(issued), 1);
        const int never = 0;
        for (int s = 0; s < STAGES; ++s) {
            const int mine = issued[s];
            int peer;
            asm volatile("ld.shared::cluster.b32 %0, [%1];" : "=r"(peer) : "r"(peer_issued + 4u * s) : "memory");
            int it = mine;
            if (peer > mine) {
                mbar_arrive_expect_tx(&full[s], unit_bytes(peer));  // the odd CTA's loads alone
                it = peer;
            } else if (mine >= 0 && peer < mine) {
                mbar_complete_tx(&full[s], unit_bytes(mine));  // the odd CTA's share that never came
            }
            if (it >= 0 && !mbar_wait(&full[s], static_cast<uint32_t>(it / STAGES) & 1u, &never, p.timeout_ns))
                record_failure(p.status, kStatusTimeout, 26, -1 - s);
        }
    }
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kTmemCols);
    }
}

template <int BN, int STAGES, int NBUF, bool ROWS>
static dg_status_t launch_pair_impl(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream) {
    using L = PairSmem<BN, STAGES, NBUF>;
    static_assert(L::kDynamicBytes <= 232448, "shared memory budget");
    static_assert(STAGES % 2 == 0 && NBUF % 2 == 0, "each MMA thread must own its stages and buffers");
    CUtensorMap tmA, tmB, tmBn, tmC;
    dg_status_t st;
    st = make_tmap_2d(&tmA, a.A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.M, a.K, 128, 128, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DG_OK) return st;
    st = make_tmap_2d(&tmB, a.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.N, a.K, BN / 2, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DG_OK) return st;
    st = make_tmap_2d(&tmBn, a.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.N, a.K, BN / 4, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DG_OK) return st;
    st = make_tmap_2d(&tmC, a.C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.M, a.N, 32, 64, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DG_OK) return st;

    const KernelControl ctl = kernel_control();
    PairParams p;
    p.sA = a.sA;
    p.sB = a.sB;
    p.num_m = static_cast<int>((a.M + 127) / 128);
    p.num_n_tiles = static_cast<int>((a.N + BN - 1) / BN);
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.Nb = static_cast<int>((a.N + 127) / 128);
    p.Kb = static_cast<int>((a.K + 127) / 128);
    p.timeout_ns = ctl.timeout_ns;
    p.status = ctl.status;
    p.debug_flags = ctl.debug_flags;

    auto kernel = pair_gemm_kernel<BN, STAGES, NBUF, ROWS>;
    static thread_local int configured_device = -1;
    static thread_local int max_pairs = 0;
    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess) return DG_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(kPairThreads, 1, 1);
    cfg.dynamicSmemBytes = L::kDynamicBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (configured_device != device) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(L::kDynamicBytes)) != cudaSuccess)
            return DG_ERR_CUDA;
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return DG_ERR_CUDA;
        if (128 * pair_regs_producer<BN>() + 256 * pair_regs_epilogue<BN>() > kPairThreads * fa.numRegs) return DG_ERR_CUDA;
        cfg.gridDim = dim3(static_cast<unsigned>(dev.num_sms & ~1), 1, 1);
        int clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &cfg) != cudaSuccess || clusters < 1)
            return DG_ERR_CUDA;
        max_pairs = clusters;
        configured_device = device;
    }
    // Tiles go round-robin to the pairs.  When the last round would keep at most half
    // of the pairs busy (4096^3: 256 tiles on 74 pairs leave 34 for the fourth round),
    // its tiles run as two 256 x BN/2 halves each, so that round takes about half a
    // tile's time; the halves are the last units, one per pair.
    const int64_t tiles = static_cast<int64_t>((p.num_m + 1) / 2) * p.num_n_tiles;
    if (tiles > 0x3FFFFFFFLL) return DG_ERR_SHAPE;
    const int64_t last_round = tiles - ((tiles - 1) / max_pairs) * max_pairs;  // 1 .. max_pairs tiles
    const bool split = BN == 256 && 2 * last_round <= max_pairs;
    p.tiles_wide = static_cast<int>(split ? tiles - last_round : tiles);
    p.num_units = static_cast<int>(split ? tiles + last_round : tiles);
    const int pairs = static_cast<int>(p.num_units < max_pairs ? p.num_units : max_pairs);
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs), 1, 1);
    cfg.numAttrs = 2;  // the occupancy query above ran with the cluster shape alone
    if (cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, tmBn, tmC, p) != cudaSuccess) return DG_ERR_CUDA;
    return DG_OK;
}

dg_status_t launch_pair_gemm(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream) {
    return a.row_scales ? launch_pair_impl<256, 6, 2, true>(a, dev, stream)
                        : launch_pair_impl<256, 6, 2, false>(a, dev, stream);
}

dg_status_t launch_pair_gemm_n128(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream) {
    return a.row_scales ? launch_pair_impl<128, 8, 4, true>(a, dev, stream)
                        : launch_pair_impl<128, 8, 4, false>(a, dev, stream);
}

}  // namespace dg
