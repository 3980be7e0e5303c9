// FP8 block-scaled GEMM on tcgen05 tensor cores (sm_100a), CTA-pair version.
//
//   C[i, j] = sum_t  s_a(t, i) * s_b(t, j) * P_t[i, j],
//   P_t[i, j] = sum_{k in slab t} A[i, k] * B[j, k]      (E4M3 codes)
//
// with 128-wide contraction slabs t.  This is the promotion scheme of the
// DeepSeek-V3 FP8 recipe that the Puro-2B tech report's related-work section
// (part 7/7, section 5) cites: every slab's partial sum leaves the tensor
// core in FP32 and is scaled before it joins the running FP32 accumulator.
// The result is either rounded to BF16 and stored, or (main-gradient mode)
// added in FP32 to the FP32 array already in memory (vector reductions
// straight from the registers, round-to-nearest-even; a subnormal sum may
// be flushed to zero), or added the same way into the data-parallel owners'
// shards of that array (the reduce-scatter of a weight gradient).
//
// Work schedule (template parameter SPLIT): whole 256 x 256 tiles
// round-robin over the CTA pairs, or, for long GEMMs whose last wave of
// tiles would leave pairs idle, whole tiles for all waves but the last two
// and then equal ranges of (tile, slab) units per pair, with FP32 partial
// sums handed over through a workspace (see segment()).
//
// Structure: clusters of two CTAs (one per SM) compute 256 x 256 output
// tiles; persistent, 384 threads (3 warpgroups) per CTA.
//   warp 0      operand producer (both CTAs): TMA loads of this CTA's 128
//               rows of A and 128 rows of B per slab into a 4-deep ring of
//               128-byte-swizzled stages, counted on the leader CTA's
//               barrier (plain loads; no multicast anywhere).
//   warp 2      scale producer (both CTAs): the scale vectors of 8 slabs at
//               a time into a CTA-local 2-slot ring by bulk copy (in row-block
//               mode it also writes the tile's two weight-block scales of
//               each slab into the slot), paced by the promotion warps (one
//               wait and one arrive per 8 slabs).  Both producers sleep
//               between polls.
//   warps 1, 3  MMA issuers (leader CTA only), warp 1 for even slabs and warp
//               3 for odd slabs: 4 x tcgen05.mma.cta_group::2 (M=256, N=256,
//               K=32, E4M3 -> F32) per slab into the slab's 256-column TMEM
//               buffer (two, alternating), fresh every slab; each CTA's TMEM
//               receives its 128 rows.  Commits free both CTAs' smem stage
//               and publish the TMEM buffer to both CTAs' promotion warps.
//   warps 4..11 promotion + epilogue (both CTAs): each thread owns one output
//               row (TMEM lane) and 128 columns.  Per slab it loads the
//               partials with tcgen05.ld into two 32-column register sets
//               (the next chunk is loaded into a set as soon as its FMAs have
//               read it), hands the TMEM buffer back to the leader once the
//               last chunk has landed, and does acc = fma(c, P, acc) in
//               registers with packed FP32x2 FMAs.  After the last slab it
//               writes the tile through a per-warp 128-byte-swizzled staging
//               buffer and a TMA store (BF16), or adds it to the FP32 array
//               with vector reductions.
// Why this shape: the MMA of slab t+2 reuses the buffer of slab t, so each
// slab's hand-off (commit -> wake -> loads -> release -> issue, about 1 us
// measured on B200) must fit in the time of two slabs' MMAs.  A 256-column
// tile gives the most MMA work per hand-off that two buffers of tensor
// memory can hold; narrower tiles with more buffers, or a whole slab staged
// in registers by more promotion warps, measured slower (the operand feed of
// narrower tiles is slower, and more waiters per barrier wake later).
// Scale modes:
//   kScaleRowBlock (fprop, dgrad): s_a is per output row (1x128 activation
//     groups), s_b per 128-column block of the weight (128x128 blocks), so
//     the coefficient is one number per thread per slab.
//   kScaleOuter (wgrad): both operands are grouped along tokens, so the
//     coefficient is the outer product s_a(t, i) * s_b(t, j).
// Every mbarrier wait is bounded in time (see mbar_wait); on a time-out the
// CTA stops issuing work, drains the copies and MMAs it has in flight (each
// drain wait bounded by max(limit, 100 ms)), meets its partner at the closing
// cluster barrier, frees its tensor memory and exits.  The closing cluster
// barrier itself has no time limit: both CTAs of a pair reach it, because
// everything before it is bounded.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"

namespace fp8blk {
namespace gemm {

constexpr int BM = 128;              // output rows per CTA (256 per pair)
constexpr int BN = 256;              // output columns per pair tile
constexpr int BK = 128;              // one quantization slab
constexpr int UMMA_K = 32;           // K of one kind::f8f6f4 MMA
constexpr int STAGES = 4;
constexpr int SCHUNK = 8;            // slabs of scales per ring slot
constexpr int SSLOTS = 2;            // scale ring slots
constexpr int A_BYTES = BM * BK;             // this CTA's 128 rows of A
constexpr int B_BYTES = (BN / 2) * BK;       // this CTA's 128 rows of B
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int PAIR_STAGE_BYTES = 2 * STAGE_BYTES;
constexpr int EPI_WARPS = 8;
constexpr int EPI_WARP0 = 4;         // first epilogue warp (warpgroups 1 and 2)
constexpr int THREADS = (EPI_WARP0 + EPI_WARPS) * 32;
// Register split: launched at 168 per thread (384 x 168 = 64512).  Row-block
// mode: warpgroup 0 drops to 72 and the two epilogue warpgroups rise to 216
// (128 x 72 + 256 x 216 = 64512); at 40 the producer roles spill.  Outer mode
// needs more in the epilogue (the per-column scale products): 40 / 232.
constexpr int REGS_LAUNCH = 168;
template <int SCALE> struct RegSplit;
template <> struct RegSplit<0> { static constexpr int producer = 72, epilogue = 216; };
template <> struct RegSplit<1> { static constexpr int producer = 40, epilogue = 232; };
static_assert(128 * RegSplit<0>::producer + 256 * RegSplit<0>::epilogue <= THREADS * REGS_LAUNCH,
              "register split exceeds the launch allocation");
static_assert(128 * RegSplit<1>::producer + 256 * RegSplit<1>::epilogue <= THREADS * REGS_LAUNCH,
              "register split exceeds the launch allocation");
constexpr int TMEM_COLS = 2 * BN;
constexpr int SCALE_SLOT_BYTES = SCHUNK * (BM + BN) * 4;   // s_a then s_b, slab-major
constexpr int OUT_WARP_BYTES = 32 * 128 * 2;     // 32 rows x 128 BF16 per epilogue warp

constexpr int OFF_SCALES = STAGES * STAGE_BYTES;
constexpr int OFF_OUT = OFF_SCALES + SSLOTS * SCALE_SLOT_BYTES;
constexpr int OFF_BARS = OFF_OUT + EPI_WARPS * OUT_WARP_BYTES;
constexpr int NUM_BARS = 2 * STAGES + 2 + 2 + 2 * SSLOTS + 1;
constexpr int OFF_TMEM_SLOT = OFF_BARS + NUM_BARS * 8;
constexpr int OFF_ABORT = OFF_TMEM_SLOT + 4;
constexpr int SMEM_BYTES = OFF_ABORT + 4 + 1024;   // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
static_assert(OFF_OUT % 1024 == 0, "swizzled staging must be 1024-byte aligned");
static_assert(STAGE_BYTES % 1024 == 0 && A_BYTES % 1024 == 0, "swizzled stages must be 1024-byte aligned");

constexpr uint32_t IDESC = idesc_e4m3_f32(2 * BM, BN);

enum ScaleMode : int { kScaleRowBlock = 0, kScaleOuter = 1 };
// kOutAccF32Shards: like kOutAccF32, but row r of the output is added to
// the shard that owns it (rows [q * shard_rows, (q + 1) * shard_rows) in
// shard q, each a row-major [shard_rows, N] FP32 array, possibly in another
// GPU's memory mapped into this process): the data-parallel reduce-scatter
// of a weight gradient done by the epilogue's vector reductions.
enum OutMode : int { kOutBf16 = 0, kOutAccF32 = 1, kOutAccF32Shards = 2 };
constexpr int kMaxShards = 8;

// Sleep between polls (ns) of the waits that are not on the hand-off's
// critical path: the operand producer runs STAGES slabs ahead and the scale
// producer a chunk of 8 slabs ahead.
constexpr uint32_t kProducerSleepNs = 128;
constexpr uint32_t kScaleSleepNs = 256;
constexpr uint32_t kIssuerSleepNs = 0;

struct Params {
    const float* sa;        // s_a(t, i) = sa[t * sa_ld + i]
    int64_t sa_ld;
    const float* sb;        // row-block: s_b(nb, t) = sb[nb * sb_sn + t * sb_sk]
    int64_t sb_sn, sb_sk;   // outer:     s_b(t, j)  = sb[t * sb_ld + j]
    int64_t sb_ld;
    int M, N, K;            // output rows, output columns, contraction
    int tiles_m, tiles_n;   // pair tiles: 256-row by 256-column
    uint64_t wait_ns;
    uint32_t stall_tx;      // test only: extra bytes the first stage's barrier expects (0 normally)
    float* out_f32;         // main-gradient mode: the FP32 array [M, N] added to
    // Split schedule (see Schedule): tiles [0, dp_tiles) whole, the rest as
    // contiguous ranges of (tile, slab) units, partial sums through
    // ws_partial [pairs][2][EPI_WARPS][32][32 lanes][4] f32 and ws_flags
    // [pairs][2][EPI_WARPS][32 lanes] (zero between calls).  dp_tiles == total tiles
    // means no split (the workspace is then unused and may be null).
    int dp_tiles;
    float* ws_partial;
    int* ws_flags;
    float* shards[kMaxShards];  // kOutAccF32Shards: the owners' arrays
    int64_t shard_rows;
};

// The work of one CTA pair: first its share of whole tiles (tile = pair,
// pair + npairs, ... below dp_tiles), then one contiguous range of units
// (unit = tile * num_kb + slab) over the remaining tiles, cut evenly across
// the pairs so that the last wave has no idle pairs.  A range cuts tiles into
// segments of slabs: a segment that starts inside a tile leaves its FP32
// partial sums to the pair whose segment holds the tile's first slab, which
// adds them before the epilogue.  Every partial segment is the first segment
// of its pair's range, so a pair never waits for a partial before it has
// written its own, and no wait can be circular.
struct Seg {
    int tile, kb0, kb1;
};

// First unit (relative to the split part, which starts at unit
// dp_tiles * num_kb) of pair q's range.
__host__ __device__ __forceinline__ int64_t split_range_begin(const Params& p, int q, int npairs) {
    const int64_t units = static_cast<int64_t>(p.tiles_m * p.tiles_n - p.dp_tiles) * (p.K / BK);
    return units * q / npairs;
}

// Segment `idx` of pair `pair`'s work, or false past the last one.  It is
// computed from the launch parameters and idx alone: the roles carry only
// the index from one segment to the next, so the schedule adds no live
// registers to the promotion warps' slab loop (whose accumulators leave
// almost none spare).  SPLIT == false is the plain round-robin of whole tiles.
template <bool SPLIT>
__host__ __device__ __forceinline__ bool segment(const Params& p, int pair, int npairs, int idx, Seg& sg) {
    const int num_kb = p.K / BK;
    if (!SPLIT) {
        sg.tile = pair + idx * npairs;
        sg.kb0 = 0;
        sg.kb1 = num_kb;
        return sg.tile < p.tiles_m * p.tiles_n;
    }
    const int n_dp = pair < p.dp_tiles ? (p.dp_tiles - 1 - pair) / npairs + 1 : 0;
    if (idx < n_dp) {
        sg.tile = pair + idx * npairs;
        sg.kb0 = 0;
        sg.kb1 = num_kb;
        return true;
    }
    const int64_t base = static_cast<int64_t>(p.dp_tiles) * num_kb;
    const int64_t b = base + split_range_begin(p, pair, npairs);
    const int64_t e = base + split_range_begin(p, pair + 1, npairs);
    const int64_t j = idx - n_dp;
    // the first segment starts where the range does, later ones at tile starts
    const int64_t start = (j == 0) ? b : (b / num_kb + j) * num_kb;
    if (start >= e) return false;
    sg.tile = static_cast<int>(start / num_kb);
    const int64_t tile_u = static_cast<int64_t>(sg.tile) * num_kb;
    sg.kb0 = static_cast<int>(start - tile_u);
    sg.kb1 = static_cast<int>(e - tile_u < num_kb ? e - tile_u : num_kb);
    return true;
}

// Release / acquire flag accesses for the partial-sum hand-over between pairs.
__device__ __forceinline__ void st_release_gpu(int* addr, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_gpu(const int* addr) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
    return v;
}

struct Bars {
    uint32_t full, empty, tfull, tempty, sfull, sempty, drain;
    __device__ __forceinline__ uint32_t full_(int s) const { return full + 8 * s; }
    __device__ __forceinline__ uint32_t empty_(int s) const { return empty + 8 * s; }
    __device__ __forceinline__ uint32_t tfull_(int b) const { return tfull + 8 * b; }
    __device__ __forceinline__ uint32_t tempty_(int b) const { return tempty + 8 * b; }
    __device__ __forceinline__ uint32_t sfull_(int s) const { return sfull + 8 * s; }
    __device__ __forceinline__ uint32_t sempty_(int s) const { return sempty + 8 * s; }
};

// tmA: A codes [M, K] (box 128 x 128), tmB: B codes [N, K] (box 128 x 128),
// tmC: BF16 output [M, N], box 64 x 32, 128-byte swizzled (kOutBf16; in
// main-gradient mode p.out_f32 is written instead).
template <int SCALE, int OUT, bool SPLIT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmC, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();            // 0 = leader of the pair
    const int pair = blockIdx.x >> 1;
    const int npairs = gridDim.x >> 1;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_ABORT);

    Bars bars;
    bars.full = sbase + OFF_BARS;
    bars.empty = bars.full + 8 * STAGES;
    bars.tfull = bars.empty + 8 * STAGES;
    bars.tempty = bars.tfull + 16;
    bars.sfull = bars.tempty + 16;
    bars.sempty = bars.sfull + 8 * SSLOTS;
    bars.drain = bars.sempty + 8 * SSLOTS;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bars.full_(s), 1);      // leader: its producer's arrive + both CTAs' bytes
            mbar_init(bars.empty_(s), 1);     // one multicast commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(bars.tfull_(b), 1);
            mbar_init(bars.tempty_(b), 2 * EPI_WARPS);   // leader: both CTAs' epilogue warps
        }
        for (int s = 0; s < SSLOTS; ++s) {
            mbar_init(bars.sfull_(s), 1);
            mbar_init(bars.sempty_(s), EPI_WARPS);
        }
        mbar_init(bars.drain, 2);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_pair(sbase + OFF_TMEM_SLOT, TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
        prefetch_tensormap(&tmC);
    }
    tc_fence_before();
    __syncwarp();
    cluster_sync();                                      // barriers and TMEM ready in both CTAs
    tc_fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM_SLOT);
    griddep_wait();                                      // inputs of the preceding kernel are complete

    if (warp < EPI_WARP0) {
      asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(RegSplit<SCALE>::producer));
      if (warp == 0) {
        // ---------------------------------------------------- operand producer
        if (lane == 0) {
            const uint32_t full_leader = map_to_cta(bars.full, 0);
            int it = 0;    // slabs whose operand tiles were requested
            bool ok = true;
            Seg sg;
            for (int seg = 0; ok && segment<SPLIT>(p, pair, npairs, seg, sg); ++seg) {
                const int m_own = (sg.tile / p.tiles_n) * (2 * BM) + static_cast<int>(rank) * BM;
                const int n0 = (sg.tile % p.tiles_n) * BN;
                for (int kb = sg.kb0; kb < sg.kb1; ++kb) {
                    const int s = it % STAGES;
                    if (!mbar_wait(bars.empty_(s), ((it / STAGES) & 1) ^ 1, abort_flag, p.wait_ns, kErrTimeout,
                                   kProducerSleepNs)) {
                        ok = false;
                        break;
                    }
                    const uint32_t a_dst = sbase + s * STAGE_BYTES;
                    if (rank == 0) mbar_arrive_expect_tx(bars.full_(s), PAIR_STAGE_BYTES + (it == 0 ? p.stall_tx : 0u));
                    tma_load_2d_pair(a_dst, &tmA, kb * BK, m_own, full_leader + 8 * s);
                    tma_load_2d_pair(a_dst + A_BYTES, &tmB, kb * BK, n0 + static_cast<int>(rank) * (BN / 2),
                                     full_leader + 8 * s);
                    ++it;
                }
            }
            if (!ok && rank == 0) {
                // Let every copy already requested land before the pair
                // exits.  Both CTAs' copies complete on the leader's full
                // barriers, so the leader's drain covers rank 1's too, and
                // rank 1 leaves only after the closing cluster barrier.
                for (int j = max(0, it - STAGES); j < it; ++j)
                    drain_wait(bars.full_(j % STAGES), (j / STAGES) & 1, p.wait_ns);
            }
        }
      } else if (warp == 2) {
        // ------------------------------------------------------ scale producer
        // Lane 0 issues the bulk copies of s_a (and, in outer mode, s_b).  In
        // row-block mode lanes 0..15 also fetch the chunk's weight-block
        // scales (two blocks per 256-column tile; strided in dgrad, so not a
        // bulk copy) and store them into the slot before lane 0 arrives.
        int ic = 0;    // scale chunks requested
        bool ok = true;
        Seg sg;
        for (int seg = 0; ok && segment<SPLIT>(p, pair, npairs, seg, sg); ++seg) {
            const int m_own = (sg.tile / p.tiles_n) * (2 * BM) + static_cast<int>(rank) * BM;
            const int n0 = (sg.tile % p.tiles_n) * BN;
            const uint32_t sa_bytes = (m_own < p.M) ? BM * 4u : 0u;
            const uint32_t sb_bytes =
                (SCALE == kScaleOuter) ? static_cast<uint32_t>(min(BN, p.N - n0)) * 4u : 0u;
            for (int kb0 = sg.kb0; kb0 < sg.kb1; kb0 += SCHUNK) {
                const int nslab = min(SCHUNK, sg.kb1 - kb0);
                const int sl = ic % SSLOTS;
                const bool got = mbar_wait(bars.sempty_(sl), ((ic / SSLOTS) & 1) ^ 1, abort_flag, p.wait_ns,
                                           kErrTimeout, kScaleSleepNs);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                const uint32_t slot = sbase + OFF_SCALES + sl * SCALE_SLOT_BYTES;
                if (SCALE == kScaleRowBlock) {
                    const int j = lane >> 1, h = lane & 1;
                    const int nb = n0 / 128 + h;
                    if (j < nslab) {
                        float* dst = reinterpret_cast<float*>(smem + OFF_SCALES + sl * SCALE_SLOT_BYTES) +
                                     SCHUNK * BM + 2 * j + h;
                        *dst = (nb < p.N / 128) ? __ldg(p.sb + static_cast<int64_t>(nb) * p.sb_sn +
                                                        static_cast<int64_t>(kb0 + j) * p.sb_sk)
                                                : 0.0f;
                    }
                    __syncwarp();
                }
                if (lane == 0) {
                    mbar_arrive_expect_tx(bars.sfull_(sl), nslab * (sa_bytes + sb_bytes));
                    for (int j = 0; j < nslab; ++j) {
                        const int64_t kb = kb0 + j;
                        if (sa_bytes)
                            bulk_load(slot + j * BM * 4, p.sa + kb * p.sa_ld + m_own, sa_bytes, bars.sfull_(sl));
                        if (SCALE == kScaleOuter)
                            bulk_load(slot + SCHUNK * BM * 4 + j * BN * 4, p.sb + kb * p.sb_ld + n0, sb_bytes,
                                      bars.sfull_(sl));
                    }
                }
                ++ic;
            }
        }
        if (!ok && lane == 0) {
            for (int j = max(0, ic - SSLOTS); j < ic; ++j)
                drain_wait(bars.sfull_(j % SSLOTS), (j / SSLOTS) & 1, p.wait_ns);
        }
        __syncwarp();
      } else if (warp == 1 || warp == 3) {
        // -------------------------------------------------- MMA issuer (leader)
        if (lane == 0 && rank == 0) {
            const int sel = (warp == 1) ? 0 : 1;
            int it = 0;
            bool ok = true;
            Seg sg;
            for (int seg = 0; ok && segment<SPLIT>(p, pair, npairs, seg, sg); ++seg) {
                const int nslab = sg.kb1 - sg.kb0;
                for (int j = 0; j < nslab; ++j, ++it) {
                    if ((it & 1) != sel) continue;
                    const int buf = it & 1;
                    if (!mbar_wait(bars.tempty_(buf), ((it >> 1) & 1) ^ 1, abort_flag, p.wait_ns, kErrTimeout,
                                   kIssuerSleepNs)) {
                        ok = false;
                        break;
                    }
                    const int s = it % STAGES;
                    if (!mbar_wait(bars.full_(s), (it / STAGES) & 1, abort_flag, p.wait_ns, kErrTimeout)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = sbase + s * STAGE_BYTES;
                    const uint64_t a_desc = smem_desc_k128_sw128(a_addr);
                    const uint64_t b_desc = smem_desc_k128_sw128(a_addr + A_BYTES);
                    const uint32_t d_tmem = tmem_base + buf * BN;
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        // +32 bytes along K inside the swizzled 128-byte row
                        const uint64_t adv = static_cast<uint64_t>((k * UMMA_K) >> 4);
                        mma_f8_pair(d_tmem, a_desc + adv, b_desc + adv, IDESC, k > 0 ? 1u : 0u);
                    }
                    mma_commit_pair(bars.empty_(s), 0x3);
                    mma_commit_pair(bars.tfull_(buf), 0x3);
                }
            }
            // All MMAs of both issuers done before the pair may free TMEM.
            mma_commit_pair(bars.drain, 0x1);
            drain_wait(bars.drain, 0, p.wait_ns);
        }
        __syncwarp();
      }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(RegSplit<SCALE>::epilogue));
        // ----------------------------------------------- promotion + epilogue
        const int ew = warp - EPI_WARP0;
        const int quarter = warp & 3;          // TMEM lanes this warp may read
        const int half = ew >> 2;              // which 128 of the 256 columns
        const int row_in_tile = quarter * 32 + lane;
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16);
        const uint32_t tempty_leader = map_to_cta(bars.tempty, 0);

        float acc[128];
        bool pending = false;   // split only: this lane's partial-sum flag is still to be released
        int it = 0;
        int ic = 0;        // scale chunks consumed
        bool ok = true;
        for (int seg = 0; ok; ++seg) {
            Seg sg;
            if (!segment<SPLIT>(p, pair, npairs, seg, sg)) break;
            const int nslab = sg.kb1 - sg.kb0;
#pragma unroll
            for (int j = 0; j < 128; ++j) acc[j] = 0.0f;

            for (int js = 0; js < nslab; ++js, ++it) {
                const int buf = it & 1;
                const int sl = ic % SSLOTS;
                const int j_in_chunk = js % SCHUNK;
                bool got = true;
                if (j_in_chunk == 0)
                    got = mbar_wait(bars.sfull_(sl), (ic / SSLOTS) & 1, abort_flag, p.wait_ns, kErrTimeout);
                got = got && mbar_wait(bars.tfull_(buf), (it >> 1) & 1, abort_flag, p.wait_ns, kErrTimeout);
                if (!__all_sync(0xffffffffu, got)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const float* slot =
                    reinterpret_cast<const float*>(smem + OFF_SCALES + sl * SCALE_SLOT_BYTES);
                const float sa = slot[j_in_chunk * BM + row_in_tile];
                const uint32_t taddr = lane_base + buf * BN + half * 128;
                float2 cpair = make_float2(0.0f, 0.0f);
                if (SCALE == kScaleRowBlock) {
                    const float c = sa * slot[SCHUNK * BM + 2 * j_in_chunk + half];
                    cpair = make_float2(c, c);
                }
                const float* sbv = slot + SCHUNK * BM + j_in_chunk * BN + half * 128;
                // Promote 32 columns held in r (columns c0 .. c0+31 of this half)
                // with packed FP32x2 FMAs: acc = c * partial + acc, two
                // columns per instruction.
                auto promote = [&](const uint32_t (&r)[32], int c0) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const int a = c0 + j;
                        float2 p01 = make_float2(__uint_as_float(r[j + 0]), __uint_as_float(r[j + 1]));
                        float2 p23 = make_float2(__uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
                        float2 c01 = cpair, c23 = cpair;
                        if (SCALE == kScaleOuter) {
                            // column scales into the partials, then the row scale
                            const float4 b4 = *reinterpret_cast<const float4*>(sbv + a);
                            p01 = __fmul2_rn(make_float2(b4.x, b4.y), p01);
                            p23 = __fmul2_rn(make_float2(b4.z, b4.w), p23);
                            c01 = c23 = make_float2(sa, sa);
                        }
                        const float2 v01 = __ffma2_rn(c01, p01, make_float2(acc[a + 0], acc[a + 1]));
                        const float2 v23 = __ffma2_rn(c23, p23, make_float2(acc[a + 2], acc[a + 3]));
                        acc[a + 0] = v01.x;
                        acc[a + 1] = v01.y;
                        acc[a + 2] = v23.x;
                        acc[a + 3] = v23.y;
                    }
                };
                // Two 32-column register sets: chunks 0 and 1 land, chunk 2
                // and 3 loads are issued into a set as soon as its FMAs have
                // read it, and the buffer goes back to the MMA issuer once
                // chunks 2 and 3 have landed (two waits per slab).
                uint32_t ra[32], rb[32];
                tmem_ld_32x32b_x32(taddr, ra);
                tmem_ld_32x32b_x32(taddr + 32, rb);
                tmem_ld_wait();
                promote(ra, 0);
                tmem_ld_32x32b_x32(taddr + 64, ra);
                promote(rb, 32);
                tmem_ld_32x32b_x32(taddr + 96, rb);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    if (rank == 0)
                        mbar_arrive(bars.tempty_(buf));
                    else
                        mbar_arrive_remote(tempty_leader + 8 * buf);
                }
                promote(ra, 64);
                promote(rb, 96);
                if (SPLIT && pending) {
                    st_release_gpu(p.ws_flags + ((pair * 2 + static_cast<int>(rank)) * EPI_WARPS + ew) * 32 + lane, 1);
                    pending = false;
                }
                if (j_in_chunk == SCHUNK - 1 || js == nslab - 1) {
                    // last slab of this scale chunk: the slot may be refilled
                    __syncwarp();
                    if (lane == 0) mbar_arrive(bars.sempty_(sl));
                    ++ic;
                }
            }
            if (!ok) break;
            if (SPLIT) {
                // The segment again, from its index alone (the opaque move
                // keeps the compiler from carrying the first lookup's values
                // across the slab loop).
                asm volatile("" : "+r"(seg));
                segment<true>(p, pair, npairs, seg, sg);
                if (sg.kb0 > 0) {
                    // A later part of a split tile: leave the partial sums to
                    // the pair that holds the tile's first slab.  16-byte
                    // vectors, lane-fastest, so each store of the warp covers
                    // 512 contiguous bytes.  Each lane releases its own flag
                    // one slab later (or when the pair's work ends): the
                    // release orders the lane's stores before it, they have
                    // landed by then, and the finalizing pair needs them only
                    // at the end of its own range.
                    const int64_t slot = (static_cast<int64_t>(pair) * 2 + rank) * EPI_WARPS + ew;
                    float4* dst = reinterpret_cast<float4*>(p.ws_partial) + slot * (32 * 32) + lane;
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        __stcg(dst + j * 32, make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]));
                    pending = true;
                    continue;
                }
                const int num_kb = p.K / BK;
                if (sg.kb1 < num_kb) {
                    // The first part of a split tile: add the partial sums of
                    // the pairs holding the rest, in pair order, then the
                    // epilogue.  (A pair with an empty range holds nothing.)
                    const int64_t tile_end =
                        static_cast<int64_t>(sg.tile + 1) * num_kb - static_cast<int64_t>(p.dp_tiles) * num_kb;
                    for (int q = pair + 1; q < npairs && split_range_begin(p, q, npairs) < tile_end; ++q) {
                        if (split_range_begin(p, q, npairs) == split_range_begin(p, q + 1, npairs)) continue;
                        const int64_t slot = (static_cast<int64_t>(q) * 2 + rank) * EPI_WARPS + ew;
                        int* flag = p.ws_flags + slot * 32 + lane;
                        const uint64_t t0 = globaltimer_ns();
                        bool got = true;
                        while (ld_acquire_gpu(flag) == 0) {
                            if (*abort_flag || globaltimer_ns() - t0 > p.wait_ns) {
                                if (!*abort_flag) {
                                    record_error(kErrTimeout);
                                    *abort_flag = 1;
                                }
                                got = false;
                                break;
                            }
                        }
                        if (!__all_sync(0xffffffffu, got)) {
                            ok = false;
                            break;
                        }
                        const float4* src = reinterpret_cast<const float4*>(p.ws_partial) + slot * (32 * 32) + lane;
#pragma unroll
                        for (int j = 0; j < 32; ++j) {
                            const float4 v = __ldcg(src + j * 32);
                            acc[4 * j] += v.x;
                            acc[4 * j + 1] += v.y;
                            acc[4 * j + 2] += v.z;
                            acc[4 * j + 3] += v.w;
                        }
                        *const_cast<volatile int*>(flag) = 0;       // zero again for the next call
                    }
                    if (!ok) break;
                }
            }

            // BF16 round-to-nearest-even into this warp's staging buffer (two
            // 32 x 64 boxes, 128-byte rows, 16-byte chunk j of row r at
            // position j ^ (r % 8)), then TMA stores of the two boxes.
            const int m_own = (sg.tile / p.tiles_n) * (2 * BM) + static_cast<int>(rank) * BM;
            const int col0 = (sg.tile % p.tiles_n) * BN + half * 128;
            if ((OUT == kOutAccF32 || OUT == kOutAccF32Shards) && col0 < p.N && m_own < p.M) {
                // FP32 added to the array in memory straight from the
                // registers: one vector reduction per 4 columns, so each
                // element receives exactly one addition per call (per
                // rank, when the shards gather several ranks' products)
                const int64_t row = m_own + quarter * 32 + lane;
                float* dst;
                if (OUT == kOutAccF32Shards) {
                    const int64_t owner = row / p.shard_rows;
                    dst = p.shards[owner] + (row - owner * p.shard_rows) * p.N + col0;
                } else {
                    dst = p.out_f32 + row * p.N + col0;
                }
#pragma unroll
                for (int j = 0; j < 128; j += 4)
                    red_add_v4_f32(dst + j, acc[j + 0], acc[j + 1], acc[j + 2], acc[j + 3]);
            } else if (OUT == kOutBf16 && col0 < p.N && m_own < p.M) {
                // The row's staging address and swizzle key come out of an
                // opaque move, so that the compiler computes the 16 chunk
                // addresses here instead of keeping them live across the slab loop.
                uint32_t row_addr, key;
                asm volatile("mov.u32 %0, %1;" : "=r"(row_addr) : "r"(smem_u32(smem + OFF_OUT + ew * OUT_WARP_BYTES) + lane * 128));
                asm volatile("mov.u32 %0, %1;" : "=r"(key) : "r"((lane & 7) << 4));
                if (lane == 0) bulk_wait_group_read0();     // previous tile's store has read the buffer
                __syncwarp();
#pragma unroll
                for (int j = 0; j < 128; j += 8) {
                    uint4 o;
                    __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[j + 0], acc[j + 1]);
                    __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[j + 2], acc[j + 3]);
                    __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[j + 4], acc[j + 5]);
                    __nv_bfloat162 h3 = __floats2bfloat162_rn(acc[j + 6], acc[j + 7]);
                    o.x = *reinterpret_cast<uint32_t*>(&h0);
                    o.y = *reinterpret_cast<uint32_t*>(&h1);
                    o.z = *reinterpret_cast<uint32_t*>(&h2);
                    o.w = *reinterpret_cast<uint32_t*>(&h3);
                    const int box = j >> 6;                 // which 64-column box
                    const int chunk = (j & 63) >> 3;        // 16-byte chunk in the 128-byte row
                    st_shared_v4(row_addr + box * 4096 + ((static_cast<uint32_t>(chunk) << 4) ^ key), o);
                }
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                    const uint32_t src = smem_u32(smem + OFF_OUT + ew * OUT_WARP_BYTES);
                    tma_store_2d(&tmC, src, col0, m_own + quarter * 32);
                    tma_store_2d(&tmC, src + 4096, col0 + 64, m_own + quarter * 32);
                    bulk_commit_group();
                }
            }
        }
        if (SPLIT && pending)
            st_release_gpu(p.ws_flags + ((pair * 2 + static_cast<int>(rank)) * EPI_WARPS + ew) * 32 + lane, 1);
        if (lane == 0) bulk_wait_group0();                 // output stores complete
    }

    griddep_launch_dependents();
    tc_fence_before();
    __syncwarp();
    cluster_sync();                                      // partner done with our smem and barriers
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

}  // namespace gemm
}  // namespace fp8blk
