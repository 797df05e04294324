// Persistent, warp-specialised FP8 (E4M3) block-scaled GEMM tile kernel for
// sm_100a: dense, MoE grouped-contiguous and MoE masked forms, with 128x128 A
// scales or (ROWS, dense) one A scale per row and K block.
//
// Method (2kiu.com/news/5461879 §2.1, §3.3; demingchina.com/news/60142 §3.1):
//   C[m][n] = bf16( sum_kb sA[m/128][kb] * sB[n/128][kb] * P_kb[m][n] ),
//   P_kb[m][n] = sum over the 128-wide K block kb of A[m][k] * B[n][k].
// The tensor cores produce each P_kb in FP32 in tensor memory; the epilogue warps
// multiply it by the block-scale product and add it to an FP32 accumulator held in
// registers ("segmented accumulation", 2kiu.com/news/5461879 §3.3), in ascending kb.
//
// Roles (one CTA per SM, 12 warps; warpgroup 0 gives registers to the two
// epilogue warpgroups with setmaxnreg (128 x 56 + 256 x 224 = 384 x 168, the
// registers the block is launched with, for 256-column tiles) -- a split above
// them would make setmaxnreg.inc wait forever; the launcher checks the count):
//   warps 0, 3  TMA producers (one thread each, alternate K blocks): 128-K slabs of
//               A (128 rows) and B (BN rows) into a STAGES-deep ring of
//               128-byte-swizzled shared-memory stages (demingchina.com/news/60142
//               §3.3 producer/consumer split, §4.2 swizzle, §4.3 multi-stage ring).
//   warps 1-2   MMA issuers: one thread each, alternating K blocks; per K block
//               four tcgen05.mma (K = 32 each) into that K block's TMEM partial
//               buffer, then a commit to the stage's "empty" barrier (the stage
//               is free once the MMAs have read it) and one to the buffer's "full".
//               (kMasked: warp 3 first builds the m-block prefix table.)
//   warps 4-11  epilogue: per kb, tcgen05.ld the
//               partial kPromoChunk columns at a time (promote_kblock), release
//               the TMEM buffer as soon as the last load has landed, and
//               acc += s * P_kb with packed FP32 FMAs (ROWS: s is the thread's
//               row scale, loaded two K blocks ahead, times the B scale); after
//               the last kb, round to
//               BF16, stage in swizzled shared memory and TMA-store.  Warp w reads
//               TMEM lanes 32*(w%4).. (the lane quarter its warp id allows) and
//               columns half (w-4)/4 of the tile.
// While the epilogue works on buffer b the MMA threads fill the next buffer, so
// the tensor cores run ahead by NBUF - 1 K blocks; at a tile boundary they run into the
// next tile while the epilogue writes the previous tile's output.
//
// Grouped forms (GMODE): B is addressed as rows g*N + n of a [G*N][K] matrix.
//   kContiguous: m-blocks run over the padded concatenation of the experts' rows;
//     the expert of m-block i is the g with off[g] <= 128 i < off[g+1] (the pages'
//     "experts stored contiguously by expert id", nxmr.cn/news/132300 §2.2).
//   kMasked: expert g owns a slab of M_max rows of A and C and uses its first
//     masked_m[g] (a device count; only M varies between experts and it changes
//     from call to call, 2kiu.com/news/5461879 §2.2).  Each CTA turns the counts
//     into a prefix of m-blocks in shared memory and walks only the m-blocks that
//     hold tokens; rows at or past masked_m[g] are never written.
#include <cuda_bf16.h>

#include "dg_device.cuh"
#include "dg_internal.h"

namespace dg {

enum GroupMode { kDense = 0, kContiguous = 1, kMasked = 2 };
constexpr int kMaskedMaxG = 256;  // prefix table in shared memory

struct TileParams {
    const float *sA;
    const float *sB;
    const int32_t *offsets;   // kContiguous: off[G+1]
    const int32_t *masked_m;  // kMasked: tokens per expert
    int m_max;                // kMasked: rows per expert slab
    int mb_max;               // kMasked: ceil(m_max / 128), sA rows per expert
    __nv_bfloat16 *C;         // kMasked: rows stored one by one at an expert's last block
    int G;
    int num_m_cap;    // m-blocks of the allocation (dense: ceil(M/128))
    int num_n_tiles;  // ceil(N / BN)
    int M;            // rows of A and C (dense: M, grouped: capacity)
    int N;
    int Nb;           // ceil(N / 128)
    int Kb;           // ceil(K / 128); the last K block may be partial
    uint64_t timeout_ns;
    int *status;  // device status word
    int debug_flags;
};

constexpr int kTileThreads = 384;
constexpr int kRegsLaunch = 168;    // 65536 / 384 rounded down to a multiple of 8
// setmaxnreg split: warpgroup 0 (TMA producer, two MMA issuers, an idle warp) and the two
// epilogue warpgroups; the 256-column epilogue needs the larger share.
template <int BN> __host__ __device__ constexpr int regs_producer() { return BN == 256 ? 56 : 64; }
template <int BN> __host__ __device__ constexpr int regs_epilogue() { return BN == 256 ? 224 : 216; }
static_assert(128 * regs_producer<256>() + 256 * regs_epilogue<256>() <= kTileThreads * kRegsLaunch &&
                  128 * regs_producer<128>() + 256 * regs_epilogue<128>() <= kTileThreads * kRegsLaunch,
              "setmaxnreg split exceeds the registers the block is launched with");
// Tiles run m-block-fastest through raster groups of kRasterM m-blocks x all n-tiles,
// so a group's B tiles are read from L2 by its m-blocks.  Dense: 32 (measured at
// 8192^3: 432 us, against 437 with 16, 446-455 with 8 and 465 with 64; at 4096^3,
// a single group, up to 3 % faster than 16); grouped: 8 (16 was about 1 % slower on
// the 64-expert MoE GEMM).
template <int GMODE>
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int &mb, int &nb) {
    constexpr int kRasterM = GMODE == kDense ? 32 : 8;
    const int group = t / (kRasterM * num_n);
    const int first_m = group * kRasterM;
    const int gm = min(kRasterM, num_m - first_m);
    const int local = t - group * kRasterM * num_n;
    mb = first_m + local % gm;
    nb = local / gm;
}

// Expert owning padded row `row` (off[g] <= row < off[g+1]); requires row < off[G].
__device__ __forceinline__ int expert_of_row(const int32_t *off, int G, int row) {
    int lo = 0, hi = G;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (__ldg(off + mid) <= row) lo = mid; else hi = mid;
    }
    return lo;
}

template <int BN, int STAGES, int NBUF, int GMODE>
struct TileSmem {
    static constexpr uint32_t kABytes = 128 * 128;
    static constexpr uint32_t kBBytes = BN * 128;
    static constexpr uint32_t kCBoxBytes = 32 * 64 * 2;  // one 32-row x 64-column BF16 box
    static constexpr uint32_t kOffA = 0;
    static constexpr uint32_t kOffB = kOffA + STAGES * kABytes;
    static constexpr uint32_t kOffC = kOffB + STAGES * kBBytes;
    static constexpr uint32_t kOffBar = kOffC + 8 * kCBoxBytes;
    static constexpr uint32_t kNumBars = 2 * STAGES + 2 * NBUF + 2;
    static constexpr uint32_t kOffMisc = kOffBar + 8 * kNumBars;
    static constexpr uint32_t kOffPrefix = kOffMisc + 16;  // kMasked: m-block prefix, G + 1 ints
    static constexpr uint32_t kBytes = kOffPrefix + (GMODE == kMasked ? 4 * (kMaskedMaxG + 4) : 0);
    static constexpr uint32_t kDynamicBytes = kBytes + 1024;  // slack for 1024-byte alignment
};

// Where tile t's operands and output live.
struct TileInfo {
    int a_row;   // TMA row of A (and C) where the tile's 128 rows start
    int b_row;   // TMA row of B
    int sa_row;  // row of sA
    int sb_row;  // row of sB for the tile's first 128 columns
    int rows;    // rows of the tile that hold output (kMasked: up to masked_m; else 128)
};

// Number of m-blocks; kMasked also fills the prefix table (all threads call it
// after the table is built, so they agree).
template <int GMODE>
__device__ __forceinline__ int count_m_blocks(const TileParams &p, const int *prefix) {
    if (GMODE == kMasked) return prefix[p.G];
    if (GMODE == kContiguous) return min(p.num_m_cap, __ldg(p.offsets + p.G) / 128);
    return p.num_m_cap;
}

__device__ __forceinline__ int masked_count(const TileParams &p, int g) {
    return min(max(__ldg(p.masked_m + g), 0), p.m_max);  // counts outside [0, M_max] are clamped
}

template <int BN, int GMODE>
__device__ __forceinline__ TileInfo resolve_tile(const TileParams &p, const int *prefix, int t, int num_m,
                                                 int &nb) {
    int mb;
    tile_coords<GMODE>(t, num_m, p.num_n_tiles, mb, nb);
    TileInfo ti;
    if (GMODE == kMasked) {
        int lo = 0, hi = p.G;  // the g with prefix[g] <= mb < prefix[g+1]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (prefix[mid] <= mb) lo = mid; else hi = mid;
        }
        const int local = mb - prefix[lo];
        ti.a_row = lo * p.m_max + local * 128;
        ti.b_row = lo * p.N + nb * BN;
        ti.sa_row = lo * p.mb_max + local;
        ti.sb_row = lo * p.Nb;
        ti.rows = min(128, masked_count(p, lo) - local * 128);
    } else {
        const int g = GMODE == kContiguous ? expert_of_row(p.offsets, p.G, mb * 128) : 0;
        ti.a_row = mb * 128;
        ti.b_row = g * p.N + nb * BN;
        ti.sa_row = mb;
        ti.sb_row = g * p.Nb;
        ti.rows = 128;
    }
    return ti;
}

// ROWS (dense only): sA holds one scale per row of A and K block, K-block-major
// (sA[kb][m]); each epilogue thread promotes its row with its own scale.
template <int BN, int GMODE, int STAGES, int NBUF, bool ROWS>
__global__ void __launch_bounds__(kTileThreads, 1)
    tile_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmBn, const __grid_constant__ CUtensorMap tmC,
                     const TileParams p) {
    using L = TileSmem<BN, STAGES, NBUF, GMODE>;
        constexpr int kColsPerWarp = BN / 2;
    constexpr uint32_t kTmemCols = tmem_cols_for(NBUF * BN);
    constexpr uint32_t kIdesc = idesc_e4m3_f32(128, BN);
    constexpr uint32_t kIdescNarrow = idesc_e4m3_f32(128, BN / 2);

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::kOffBar);
    uint64_t *empty = full + STAGES;
    uint64_t *tfull = empty + STAGES;
    uint64_t *tempty = tfull + NBUF;
    uint64_t *mdone = tempty + NBUF;  // one per MMA thread: all its MMAs complete
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kOffMisc);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 4);
    volatile int *groups_bad = reinterpret_cast<volatile int *>(smem + L::kOffMisc + 8);
    int *prefix = reinterpret_cast<int *>(smem + L::kOffPrefix);  // kMasked only

    const int warp = static_cast<int>(threadIdx.x >> 5);
    const int lane = lane_id();

    // dense: L2 prefetch of the first tile's first B slabs before the dependency
    // wait (a cache fill only, so it cannot observe stale data); the grouped forms
    // need the routing, an input, to know their first tile
    if (GMODE == kDense && warp == 3 && lane == 0 && static_cast<int>(blockIdx.x) < p.num_m_cap * p.num_n_tiles) {
        int mb, nb;
        tile_coords<GMODE>(static_cast<int>(blockIdx.x), p.num_m_cap, p.num_n_tiles, mb, nb);
        for (int kb = 0; kb < p.Kb && kb < 2 * STAGES; ++kb) tma_prefetch_l2_2d(&tmB, kb * 128, nb * BN);
    }

    if (warp == 0 && lane == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int q = 0; q < 2; ++q) mbar_init(&mdone[q], 1);
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(&tfull[b], 1);
            mbar_init(&tempty[b], 8);
        }
        *abort_flag = 0;
        *groups_bad = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmBn);
        tma_prefetch_desc(&tmC);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    grid_dep_wait();  // inputs and outputs are touched only from here on
    grid_dep_launch_dependents();
    if (GMODE == kContiguous && warp == 3) {
        // group_offsets must start at 0, not decrease, hold multiples of 128 and end
        // within the rows allocated; otherwise nothing is computed and the status
        // word says why (memory stays safe either way: TMA clips every box)
        const int cap = p.num_m_cap * 128;
        bool bad = false;
        for (int g = lane; g <= p.G; g += 32) {
            const int o = __ldg(p.offsets + g);
            const int prev = g > 0 ? __ldg(p.offsets + g - 1) : 0;
            bad |= (o & 127) != 0 || o < prev || o > cap || (g == 0 && o != 0);
        }
        bad = __any_sync(0xFFFFFFFFu, bad);
        if (lane == 0 && bad) {
            *groups_bad = 1;
            if (blockIdx.x == 0) record_failure(p.status, kStatusBadGroups, 3, -1);
        }
    }
    if (GMODE == kMasked && warp == 3) {
        // prefix[g] = sum over h < g of ceil(count_h / 128): lane l takes experts
        // 8l .. 8l+7, then an exclusive scan of the lane sums
        constexpr int kPer = kMaskedMaxG / 32;
        int blocks[kPer];
        int sum = 0;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int g = lane * kPer + i;
            blocks[i] = g < p.G ? (masked_count(p, g) + 127) / 128 : 0;
            sum += blocks[i];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xFFFFFFFFu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - sum;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int g = lane * kPer + i;
            if (g < p.G) prefix[g] = run;
            run += blocks[i];
        }
        if (lane == 31) prefix[p.G] = incl;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    const int num_m = (GMODE == kContiguous && *groups_bad) ? 0 : count_m_blocks<GMODE>(p, prefix);
    const int num_tiles = num_m * p.num_n_tiles;
    const int Kb = p.Kb;
    // Tiles go round-robin to the CTAs.  When the last round would keep at most half
    // of them busy, its tiles run as two 128 x BN/2 halves each (two units), so that
    // round takes about half a tile's time.  Decided here because the grouped forms
    // only know their tile count on the device; every CTA computes the same split.
    const int grid = static_cast<int>(gridDim.x);
    int tiles_wide = num_tiles, num_units = num_tiles;
    if (BN == 256 && num_tiles > 0) {
        const int last_round = num_tiles - ((num_tiles - 1) / grid) * grid;
        if (2 * last_round <= grid) {
            tiles_wide = num_tiles - last_round;
            num_units = num_tiles + last_round;
        }
    }
    // unit u: tile u below tiles_wide, else half (u - tiles_wide) % 2 of tile
    // tiles_wide + (u - tiles_wide) / 2
    auto unit_tile = [&](int u, int &t, int &h) {
        if (u < tiles_wide) {
            t = u;
            h = -1;
        } else {
            t = tiles_wide + (u - tiles_wide) / 2;
            h = (u - tiles_wide) & 1;
        }
    };
    const int my_units = static_cast<int>(blockIdx.x) < num_units
                             ? (num_units - 1 - static_cast<int>(blockIdx.x)) / grid + 1
                             : 0;

    if (warp < 4) {
        regs_dealloc<regs_producer<BN>()>();
        if ((warp == 0 || warp == 3) && lane == 0) {
            // ----------------------------------------------------------- producers
            // Two threads, one per parity of the iteration: a thread's issue of one
            // stage (barrier wait, byte count, two tile copies) takes ~600 cycles,
            // measured, more than the K block's MMAs, and two threads double the
            // rate.  With STAGES even each stage belongs to one thread, whose parity
            // waits then stay in order.
            const int pr = warp == 0 ? 0 : 1;
            uint32_t issued = 0, parity_bits = 0;
            int it = 0;
            bool ok = true;
            for (int i = 0; i < my_units && ok; ++i) {
                int t, h, nb;
                unit_tile(static_cast<int>(blockIdx.x) + i * grid, t, h);
                const TileInfo ti = resolve_tile<BN, GMODE>(p, prefix, t, num_m, nb);
                const bool narrow = h >= 0;
                const int b_row = ti.b_row + (narrow ? h * (BN / 2) : 0);
                for (int kb = 0; kb < Kb; ++kb, ++it) {
                    if ((it & 1) != pr) continue;  // the other producer's stage
                    const int s = it % STAGES;
                    const uint32_t u = static_cast<uint32_t>(it / STAGES);
                    if (!mbar_wait(&empty[s], (u & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
                        record_failure(p.status, kStatusTimeout, 0, it);
                        *abort_flag = 1;
                        ok = false;
                        break;
                    }
                    if ((p.debug_flags & 1) && it == 0) continue;  // test hook: never fill stage 0
                    mbar_arrive_expect_tx(&full[s], L::kABytes + (narrow ? L::kBBytes / 2 : L::kBBytes));
                    tma_load_2d(smem + L::kOffA + s * L::kABytes, &tmA, &full[s], kb * 128, ti.a_row);
                    tma_load_2d(smem + L::kOffB + s * L::kBBytes, narrow ? &tmBn : &tmB, &full[s], kb * 128, b_row);
                    issued |= 1u << s;
                    parity_bits = (parity_bits & ~(1u << s)) | ((u & 1u) << s);
                }
            }
            // every load issued must land before the CTA may exit
            const int never = 0;
            for (int s = 0; s < STAGES; ++s)
                if (issued & (1u << s))
                    if (!mbar_wait(&full[s], (parity_bits >> s) & 1u, &never, p.timeout_ns))
                        record_failure(p.status, kStatusTimeout, 0, -1 - s);
        } else if ((warp == 1 || warp == 2) && lane == 0) {
            // ------------------------------------------------------- MMA (two threads)
            // Thread q issues the K blocks kc with kc % 2 == q.  Every K block's
            // partial starts from zero in its own TMEM buffer, so the two streams are
            // independent, and each issuer's barrier waits and commits hide behind the
            // other's MMAs.  With STAGES and NBUF even, every stage and every buffer
            // belongs to one thread, which therefore waits on each barrier's phases in
            // order -- a parity wait is only sound one phase ahead.  Two commits per K
            // block: one frees the shared-memory stage as soon as the MMAs have read it
            // (so the producer can refill it however far behind the epilogue runs),
            // one marks the TMEM buffer full for the epilogue.
            const int q = warp - 1;
            const int total = my_units * Kb;
            const uint32_t a0 = smem_u32(smem + L::kOffA);
            const uint32_t b0 = smem_u32(smem + L::kOffB);
            int last = -1;
            int unit = 0, kbi = q;  // kc = unit * Kb + kbi
            while (kbi >= Kb) kbi -= Kb, ++unit;
            for (int kc = q; kc < total; kc += 2) {
                const bool narrow = static_cast<int>(blockIdx.x) + unit * grid >= tiles_wide;
                const int s = kc % STAGES;
                const uint32_t u = static_cast<uint32_t>(kc / STAGES);
                const int buf = kc % NBUF;
                const uint32_t v = static_cast<uint32_t>(kc / NBUF);
                const uint64_t adesc = sdesc_kmajor_sw128(a0 + s * L::kABytes);
                const uint64_t bdesc = sdesc_kmajor_sw128(b0 + s * L::kBBytes);
                const uint32_t d = tmem_base + static_cast<uint32_t>(buf * BN);
                const uint32_t idesc = narrow ? kIdescNarrow : kIdesc;
                // The stage has almost always landed long before the buffer comes back
                // from the epilogue: waiting on it first keeps its (successful) wait
                // off the path from the hand-back to the first MMA.
                if (!mbar_wait(&full[s], u & 1u, abort_flag, p.timeout_ns) ||
                    !mbar_wait(&tempty[buf], (v & 1u) ^ 1u, abort_flag, p.timeout_ns)) {
                    record_failure(p.status, kStatusTimeout, 1, kc);
                    *abort_flag = 1;
                    break;
                }
                tc_fence_after();
#pragma unroll
                for (int k = 0; k < 4; ++k)  // 32 bytes of K per instruction = +2 in the address field
                    umma_e4m3(d, adesc + 2u * k, bdesc + 2u * k, idesc, k > 0 ? 1u : 0u);
                umma_commit(&empty[s]);  // the stage is free once these MMAs have read it
                umma_commit(&tfull[buf]);
                last = kc;
                kbi += 2;
                while (kbi >= Kb) kbi -= Kb, ++unit;
            }
            // the tensor memory may only be released once every MMA issued is done
            if (last >= 0) {
                const int never = 0;
                umma_commit(&mdone[q]);
                if (!mbar_wait(&mdone[q], 0, &never, p.timeout_ns)) record_failure(p.status, kStatusTimeout, 1, -1);
            }
        }
    } else {
        regs_alloc<regs_epilogue<BN>()>();
        // -------------------------------------------------------------- epilogue
        const int ew = warp - 4;
        const int quarter = warp & 3;
        const int half = ew >> 2;
        uint8_t *cstage = smem + L::kOffC + ew * L::kCBoxBytes;
        float2 acc[kColsPerWarp / 2];
        int kc = 0;
        bool ok = true;
        for (int i = 0; i < my_units && ok; ++i) {
            int t, h, nb;
            unit_tile(static_cast<int>(blockIdx.x) + i * grid, t, h);
            const TileInfo ti = resolve_tile<BN, GMODE>(p, prefix, t, num_m, nb);
            // this warp's columns: BN/2 of a whole tile, BN/4 of a half tile
            const int ncols = h >= 0 ? kColsPerWarp / 2 : kColsPerWarp;
            const int col0 = nb * BN + (h >= 0 ? h * (BN / 2) : 0) + half * ncols;
            const int nb128 = col0 / 128;
            const bool n_valid = nb128 < p.Nb;
            const int sb_row = ti.sb_row + nb128;
            ScaleStream scales;
            scales.start(ROWS ? nullptr : p.sA + static_cast<int64_t>(ti.sa_row) * Kb,
                         p.sB + static_cast<int64_t>(sb_row) * Kb, 0, n_valid ? Kb : 0);
            // ROWS: this thread's row scales, loaded two K blocks ahead through a pointer that
            // advances by M floats a K block (recomputing the 64-bit address each K block
            // spilled registers and cost 15 %: 80.9 vs 68.5 us at 4096^3, measured)
            const int my_row = ti.a_row + quarter * 32 + lane;
            const bool row_ok = ROWS && my_row < p.M;
            const float *sa_ptr = p.sA + (row_ok ? my_row : 0);  // advances one K block (M floats) per load
            float sa_next = row_ok ? __ldg(sa_ptr) : 0.0f;
            sa_ptr += p.M;
            float sa_next2 = (row_ok && Kb > 1) ? __ldg(sa_ptr) : 0.0f;
            sa_ptr += p.M;
#pragma unroll
            for (int i = 0; i < kColsPerWarp / 2; ++i) acc[i] = make_float2(0.0f, 0.0f);
            for (int kb = 0; kb < Kb; ++kb, ++kc) {
                const int buf = kc % NBUF;
                const uint32_t v = static_cast<uint32_t>(kc / NBUF);
                float scale = scales.scale(kb, kb);
                if (ROWS) {
                    const float sa = sa_next;
                    sa_next = sa_next2;
                    sa_next2 = (row_ok && kb + 2 < Kb) ? __ldg(sa_ptr) : 0.0f;
                    sa_ptr += p.M;
                    scale = sa * scale;  // fl32(sA[row][kb] * sB[n/128][kb])
                }
                const float2 s2 = make_float2(scale, scale);
                if (!mbar_wait(&tfull[buf], v & 1u, abort_flag, p.timeout_ns)) {
                    record_failure(p.status, kStatusTimeout, 2, kc);
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
                    if (lane == 0) mbar_arrive(&tempty[buf]);
                });
            }
            if (!ok) break;
            // BF16 output: rows a_row + 32*quarter + lane, columns col0 .. col0 + ncols
            const int row0 = ti.a_row + quarter * 32;
            const int vrows = ti.rows - quarter * 32;  // rows of this warp's box that hold output
#pragma unroll
            for (int j = 0; j < kColsPerWarp / 64; ++j) {
                if (j * 64 >= ncols) break;
                if (GMODE == kMasked && vrows < 32) {
                    // the box runs past the expert's tokens: each row that holds
                    // output stores itself, the rest of the slab is left untouched
                    if (lane < vrows && col0 + j * 64 < p.N) {
                        uint4 *dst = reinterpret_cast<uint4 *>(p.C + static_cast<int64_t>(row0 + lane) * p.N + col0 + j * 64);
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const float2 *x = acc + j * 32 + c * 4;
                            dst[c] = make_uint4(pack_bf16x2(x[0].x, x[0].y), pack_bf16x2(x[1].x, x[1].y),
                                                pack_bf16x2(x[2].x, x[2].y), pack_bf16x2(x[3].x, x[3].y));
                        }
                    }
                    continue;
                }
                if (lane == 0) bulk_wait_read0();  // the previous store has finished reading cstage
                __syncwarp();
                uint8_t *rowp = cstage + lane * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float2 *x = acc + j * 32 + c * 4;
                    uint4 w;
                    w.x = pack_bf16x2(x[0].x, x[0].y);
                    w.y = pack_bf16x2(x[1].x, x[1].y);
                    w.z = pack_bf16x2(x[2].x, x[2].y);
                    w.w = pack_bf16x2(x[3].x, x[3].y);
                    *reinterpret_cast<uint4 *>(rowp + ((c ^ (lane & 7)) << 4)) = w;
                }
                fence_async_smem();
                __syncwarp();
                // a box that starts past the matrix edge is skipped, not clipped
                if (lane == 0 && col0 + j * 64 < p.N && row0 < p.M) {
                    tma_store_2d(&tmC, cstage, col0 + j * 64, row0);
                    bulk_commit();
                }
            }
        }
        if (lane == 0) bulk_wait_all0();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

template <int BN, int GMODE, int STAGES, int NBUF, bool ROWS = false>
static dg_status_t launch_tile_impl(const GemmArgs &a, const DeviceInfo &dev, cudaStream_t stream) {
    using L = TileSmem<BN, STAGES, NBUF, GMODE>;
    static_assert(L::kDynamicBytes <= 232448, "shared memory budget");
    static_assert(STAGES % 2 == 0 && NBUF % 2 == 0, "each MMA thread must own its stages and buffers");
    CUtensorMap tmA, tmB, tmBn, tmC;
    const uint64_t b_rows = GMODE != kDense ? static_cast<uint64_t>(a.G) * a.N : static_cast<uint64_t>(a.N);
    dg_status_t st;
    st = make_tmap_2d(&tmA, a.A, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, a.M, a.K, 128, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DG_OK) return st;
    st = make_tmap_2d(&tmB, a.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, b_rows, a.K, BN, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DG_OK) return st;
    st = make_tmap_2d(&tmBn, a.B, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, b_rows, a.K, BN / 2, 128,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DG_OK) return st;
    st = make_tmap_2d(&tmC, a.C, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.M, a.N, 32, 64,
                      CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DG_OK) return st;

    const KernelControl ctl = kernel_control();
    TileParams p;
    p.sA = a.sA;
    p.sB = a.sB;
    p.offsets = a.offsets;
    p.masked_m = a.masked_m;
    p.m_max = static_cast<int>(a.m_max);
    p.mb_max = static_cast<int>((a.m_max + 127) / 128);
    p.C = static_cast<__nv_bfloat16 *>(a.C);
    p.G = a.G;
    p.num_m_cap = static_cast<int>((a.M + 127) / 128);
    p.num_n_tiles = static_cast<int>((a.N + BN - 1) / BN);
    p.M = static_cast<int>(a.M);
    p.N = static_cast<int>(a.N);
    p.Nb = static_cast<int>((a.N + 127) / 128);
    p.Kb = static_cast<int>((a.K + 127) / 128);
    p.timeout_ns = ctl.timeout_ns;
    p.status = ctl.status;
    p.debug_flags = ctl.debug_flags;

    auto kernel = tile_gemm_kernel<BN, GMODE, STAGES, NBUF, ROWS>;
    static thread_local int configured_device = -1;
    int device = 0;
    cudaGetDevice(&device);
    if (configured_device != device) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(L::kDynamicBytes)) != cudaSuccess)
            return DG_ERR_CUDA;
        // the register split inside the kernel must fit what a launch provides
        cudaFuncAttributes fa;
        if (cudaFuncGetAttributes(&fa, kernel) != cudaSuccess) return DG_ERR_CUDA;
        if (128 * regs_producer<BN>() + 256 * regs_epilogue<BN>() > kTileThreads * fa.numRegs) return DG_ERR_CUDA;
        configured_device = device;
    }
    // kMasked: the counts live on the device, so size the grid for full slabs
    const int64_t m_blocks = GMODE == kMasked ? static_cast<int64_t>(a.G) * p.mb_max : p.num_m_cap;
    const int64_t tiles = m_blocks * p.num_n_tiles;
    if (tiles > 0x3FFFFFFFLL) return DG_ERR_SHAPE;
    // up to twice the tiles: a single partial round may run as half tiles (see the kernel)
    const int64_t want = BN == 256 ? 2 * tiles : tiles;
    const int grid = static_cast<int>(want < dev.num_sms ? want : dev.num_sms);
    return launch_pdl(kernel, grid, kTileThreads, L::kDynamicBytes, stream, tmA, tmB, tmBn, tmC, p);
}

dg_status_t launch_tile_gemm(const GemmArgs &a, int group, const DeviceInfo &dev, cudaStream_t stream) {
    // BN = 256 columns per tile unless the matrix is narrower (fewer idle columns).
    const bool narrow = a.N <= 128;
    if (group == kContiguous)
        return narrow ? launch_tile_impl<128, kContiguous, 6, 4>(a, dev, stream)
                      : launch_tile_impl<256, kContiguous, 4, 2>(a, dev, stream);
    if (group == kMasked)
        return narrow ? launch_tile_impl<128, kMasked, 6, 4>(a, dev, stream)
                      : launch_tile_impl<256, kMasked, 4, 2>(a, dev, stream);
    if (a.row_scales)
        return narrow ? launch_tile_impl<128, kDense, 6, 4, true>(a, dev, stream)
                      : launch_tile_impl<256, kDense, 4, 2, true>(a, dev, stream);
    return narrow ? launch_tile_impl<128, kDense, 6, 4>(a, dev, stream) : launch_tile_impl<256, kDense, 4, 2>(a, dev, stream);
}

}  // namespace dg
