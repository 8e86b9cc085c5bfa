// hessian.cuh -- calibration Hessian H = X^T X / n on the 5th-generation
// tensor cores (blog "Opt.Gear-QAT", section 2 "Hessian-based scale
// initialize": layer sensitivity from calibration activations, the
// second-order output-reconstruction view).
//
// X is bf16 [n, C] row-major, so in D[i][j] = sum_t X[t][i] X[t][j] the
// reduction index t is X's row index and both operands are MN-major.  Only the
// upper-triangle 256x256 output tiles (I <= J) are computed; each is stored
// with its mirror, so H comes out bitwise symmetric.
//
// Pair-CTA tiles.  A tile is computed by a cluster of two CTAs on an SM pair
// with tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16): CTA r holds rows
// 128r..128r+127 of the tile's A operand and columns 128r..128r+127 of its B
// operand in its own shared memory, so each SM fetches a quarter of the
// tile's operand bytes -- half the L2->SM traffic of one-SM 128x128 tiles.
// CTA r's TMEM receives rows 128r..128r+127 of D (all 256 columns).  On a
// diagonal tile the A and B halves of a CTA are the same columns of X and
// are loaded once.  No load is multicast.
//
// Warps of each CTA:
//   warp 0      TMA producer: 128-row x 64-column boxes of X, 128-byte
//               swizzle, into a 3-stage ring of 128-row stages; the peer
//               CTA's copies complete on the leader's full barrier, which the
//               leader arms with the bytes of both CTAs;
//   warp 1      allocates the pair's 512 TMEM columns; in the leader CTA one
//               thread issues the MMAs; each commit frees the ring slot in
//               both CTAs;
//   warps 2..5  epilogue over TMEM lanes 32*(w%4)..+31 (= the CTA's rows).
// A stage holds 128 rows of X: eight K = 16 MMAs per stage between two
// barrier hand-offs.  (With 64-row stages, four MMAs per wait-and-commit, the
// tensor pipe idled about a quarter of its cycles at the stage boundaries; at
// 128 rows it runs at the rate of MMAs issued with no hand-off at all.)
// Chunked promotion: the tensor core accumulates kPChunkKB stages (16384 rows)
// into TMEM columns [0,256); the epilogue adds each finished chunk into a
// float32 master copy in columns [256,512) with IEEE round-to-nearest adds
// (the tensor core's own accumulation over 262144 rows drifts by more than
// 1e-3), then releases the accumulator to the MMA.
//
// Split of n: a unit is one CTA pair computing one tile over a part of the
// calibration rows.  With T <= 74 upper tiles, every tile's rows are cut into
// S = max(1, min(74 / T, kblocks / 16)) equal parts.  With more tiles, the
// tiles run one per unit in waves of 74 pairs; when the last wave would be
// partly empty (r = T mod 74 tiles), those r tiles -- the last ones, launched
// last -- are cut into S_t = min(74 / r, kblocks / 16) parts so that the last
// wave is full and 1/S_t as long (C = 8192: 528 tiles, 7.14 waves instead of
// 8).  Units with the same part index walk the same calibration rows at the
// same time, so X stays shared through L2.  The plan is a function of (n, C)
// only, so the result does not depend on the device.  A tile in one part is
// scaled by 1/n and stored with its mirror directly; a tile in several parts
// stores its fp32 partials into the workspace (at most 74 of them) and
// hessian_reduce_kernel adds them in fixed order, scales and stores the tile
// -- deterministic.
//
// Every mbarrier wait is bounded (device_common.cuh); on a timeout a CTA stops
// issuing work, waits (bounded) for its own copies and MMAs in flight, frees
// its TMEM and exits, leaving QAT4_DEV_ERR_TIMEOUT in the error word.
#pragma once

#include "device_common.cuh"

namespace qat4 {

constexpr int kPTile = 256;                   // tile rows = tile columns
constexpr int kPHalf = 128;                   // rows (A) / columns (B) held by one CTA
constexpr int kPBK = 128;                     // X rows per pipeline stage
constexpr int kPStages = 3;
constexpr int kPThreads = 192;
constexpr int kPChunkKB = 128;                // stages per promotion chunk (16384 rows)
constexpr int kPPairsPerGpu = 74;             // SM pairs of a B200; fixes the split of n
constexpr uint32_t kPBoxBytes = 64 * kPBK * 2;          // one 64-column x 128-row bf16 box = 16 KB
constexpr uint32_t kPOperandBytes = 2 * kPBoxBytes;     // 128 columns = 32 KB
constexpr uint32_t kPStageBytes = 2 * kPOperandBytes;   // A half + B half = 64 KB
constexpr uint32_t kPSmemBytes = kPStages * kPStageBytes + 1024;
constexpr uint32_t kPTmemCols = 512;                    // [0,256) accumulator, [256,512) master

// Instruction descriptor, kind::f16: D fp32, A/B bf16, A and B MN-major,
// N = 256, M = 256 (pair).
constexpr uint32_t kPIdesc = (1u << 4)            // D format: F32
                           | (1u << 7)            // A format: BF16
                           | (1u << 10)           // B format: BF16
                           | (1u << 15)           // A major: MN
                           | (1u << 16)           // B major: MN
                           | ((256u >> 3) << 17)  // N >> 3
                           | ((256u >> 4) << 24); // M >> 4

// Shared-memory matrix descriptor for one 128-column operand half laid out as
// [2 column blocks of 64][128 rows][128 B], 128-byte swizzle: leading byte
// offset = distance between the two 64-column blocks (16 KB), stride byte
// offset = distance between 8-row groups (1 KB).
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((kPBoxBytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((1024u >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;   // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2) << 61;   // SWIZZLE_128B
    return d;
}

// Upper-triangle tile t -> (I, J), I <= J.  Tiles are numbered in bands of
// kPBand tile rows: within a band column by column (J ascending), and within a
// column down the band's rows (I <= J).  74 consecutive tiles -- one wave of
// SM pairs, which walk the calibration rows together -- then touch about 18
// column strips of X instead of all of them, so each wave reads less of X from
// HBM (C = 14336: 56 strips; row-by-row numbering re-read all of X in every
// wave, 81 GB per Hessian of 131072 rows).
constexpr int kPBand = 8;
__host__ __device__ inline void hess_tile_coords(int t, int nb, int& I, int& J) {
    for (int i0 = 0; i0 < nb; i0 += kPBand) {
        const int i1 = i0 + kPBand < nb ? i0 + kPBand : nb;   // band rows [i0, i1)
        for (int j = i0; j < nb; ++j) {
            const int cnt = (i1 < j + 1 ? i1 : j + 1) - i0;   // rows i0 .. min(i1, j + 1) - 1
            if (t < cnt) {
                I = i0 + t;
                J = j;
                return;
            }
            t -= cnt;
        }
    }
    I = J = 0;   // not reached for t < nb (nb + 1) / 2
}

struct HessPlan {
    int nb;        // ceil(C / 256)
    int tiles;     // T = nb (nb + 1) / 2
    int kblocks;   // ceil(n / 128): pipeline stages over the calibration rows
    int split0;    // first tile cut into parts (T when none is)
    int split;     // parts of the tiles from split0 on (1 when none is cut)
    int units;     // CTA pairs: (split0 whole tiles) + (T - split0) * split
};

__host__ __device__ inline HessPlan hess_plan(int64_t n, int64_t C) {
    HessPlan p;
    p.nb = static_cast<int>((C + kPTile - 1) / kPTile);
    p.tiles = p.nb * (p.nb + 1) / 2;
    p.kblocks = static_cast<int>((n + kPBK - 1) / kPBK);
    const int cap = p.kblocks / 16;                       // a part holds at least 16 stages
    const int r = p.tiles <= kPPairsPerGpu ? p.tiles : p.tiles % kPPairsPerGpu;   // tiles of the last wave
    int s = r > 0 ? kPPairsPerGpu / r : 1;
    if (s > cap) s = cap;
    if (s < 2 || r == 0) {
        p.split0 = p.tiles;
        p.split = 1;
    } else {
        p.split0 = p.tiles - r;
        p.split = s;
    }
    p.units = p.split0 + (p.tiles - p.split0) * p.split;
    return p;
}

// Unit u -> (tile, part); the partial's workspace slot is u - split0 (units with one part have none).
__host__ __device__ __forceinline__ void hess_unit(const HessPlan& p, int u, int& tile, int& part) {
    if (u < p.split0) {
        tile = u;
        part = 0;
    } else {
        const int v = u - p.split0;
        tile = p.split0 + v / p.split;
        part = v % p.split;
    }
}

struct HessParams {
    int64_t n;
    int C;
    HessPlan plan;
    float inv_n;
    uint64_t limit_ns;   // bounded-wait limit
};


__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPThreads, 1)
hessian_pair_kernel(const __grid_constant__ CUtensorMap tmap, const HessParams p,
                    float* __restrict__ H, float* __restrict__ ws) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kPStages];    // used in the leader
    __shared__ __align__(8) uint64_t empty_bar[kPStages];
    __shared__ __align__(8) uint64_t tmem_full_bar;
    __shared__ __align__(8) uint64_t tmem_empty_bar;        // used in the leader
    __shared__ __align__(8) uint64_t mma_done_bar;          // used in the leader
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    const int unit = static_cast<int>(blockIdx.x >> 1);
    int tile, part;
    hess_unit(p.plan, unit, tile, part);
    const int nparts = tile < p.plan.split0 ? 1 : p.plan.split;
    int I, J;
    hess_tile_coords(tile, p.plan.nb, I, J);
    const bool diag = (I == J);
    const int kb0 = static_cast<int>(static_cast<int64_t>(part) * p.plan.kblocks / nparts);
    const int kb1 = static_cast<int>(static_cast<int64_t>(part + 1) * p.plan.kblocks / nparts);
    const int nk = kb1 - kb0;
    const int nchunks = (nk + kPChunkKB - 1) / kPChunkKB;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kPStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        mbar_init(&tmem_full_bar, 1);
        mbar_init(&tmem_empty_bar, 8);   // 4 epilogue warps in each CTA of the pair
        mbar_init(&mma_done_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap);
    }
    if (warp == 1) {
        tmem_alloc_pair(&tmem_slot, kPTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();      // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    volatile int* abort = &abort_flag;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs)
            const uint32_t cta_bytes = diag ? kPOperandBytes : kPStageBytes;
            const int xa = I * kPTile + static_cast<int>(rank) * kPHalf;   // this CTA's A columns of X
            const int xb = J * kPTile + static_cast<int>(rank) * kPHalf;   // this CTA's B columns of X
            int issued = 0;
            for (int i = 0; i < nk; ++i) {
                const int s = i % kPStages;
                const uint32_t ph = static_cast<uint32_t>(i / kPStages) & 1u;
                if (!mbar_wait(&empty_bar[s], ph ^ 1u, abort, p.limit_ns)) break;
                uint8_t* sa = smem + s * kPStageBytes;
                uint8_t* sb = sa + kPOperandBytes;
                const uint32_t fb = cluster_map(&full_bar[s], 0);
                if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], 2 * cta_bytes);
                const int y = (kb0 + i) * kPBK;
                tma_load_2d_pair(sa, &tmap, fb, xa, y);
                tma_load_2d_pair(sa + kPBoxBytes, &tmap, fb, xa + 64, y);
                if (!diag) {
                    tma_load_2d_pair(sb, &tmap, fb, xb, y);
                    tma_load_2d_pair(sb + kPBoxBytes, &tmap, fb, xb + 64, y);
                }
                issued = i + 1;
            }
            // no copy may still be landing in shared memory when the CTA exits:
            // the leader waits for its full barriers; the peer's copies complete
            // on the leader's barriers, so the peer waits until the MMAs that
            // read its slots have freed them
            for (int i = (issued > kPStages ? issued - kPStages : 0); i < issued; ++i) {
                if (rank == 0)
                    mbar_wait_cluster(&full_bar[i % kPStages], static_cast<uint32_t>(i / kPStages) & 1u,
                                      nullptr, kDrainLimitNs);
                else
                    mbar_wait(&empty_bar[i % kPStages], static_cast<uint32_t>(i / kPStages) & 1u,
                              nullptr, kDrainLimitNs);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------- MMA issuer (leader CTA only)
            for (int i = 0; i < nk; ++i) {
                const int chunk = i / kPChunkKB;
                const bool first = (i % kPChunkKB) == 0;
                const bool last = (i % kPChunkKB) == kPChunkKB - 1 || i == nk - 1;
                if (first && chunk >= 1) {
                    // both epilogues have folded the previous chunk into the master copy
                    if (!mbar_wait_cluster(&tmem_empty_bar, static_cast<uint32_t>(chunk - 1) & 1u, abort,
                                           p.limit_ns)) break;
                    tc_fence_after();
                }
                const int s = i % kPStages;
                const uint32_t ph = static_cast<uint32_t>(i / kPStages) & 1u;
                if (!mbar_wait_cluster(&full_bar[s], ph, abort, p.limit_ns)) break;
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + s * kPStageBytes);
                const uint32_t sb = diag ? sa : sa + kPOperandBytes;
#pragma unroll
                for (int kk = 0; kk < kPBK / 16; ++kk) {
                    // K = 16 rows of X = two 8-row swizzle groups = 2 KB further on
                    tc_mma_f16_pair(tmem_base, smem_desc_mn_sw128(sa + kk * 2048u),
                                    smem_desc_mn_sw128(sb + kk * 2048u), kPIdesc,
                                    (!first || kk > 0) ? 1u : 0u);
                }
                tc_commit_pair_mc(&empty_bar[s], 0x3);
                if (last) tc_commit_pair_mc(&tmem_full_bar, 0x3);
            }
            // every MMA must have retired before TMEM is released
            tc_commit_pair(&mma_done_bar);
            mbar_wait(&mma_done_bar, 0, nullptr, kDrainLimitNs);
        }
    } else {
        // ---------------- epilogue: warps 2..5 of both CTAs
        const int q = warp & 3;                              // TMEM lanes 32q..32q+31
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
        const uint32_t empty_leader = cluster_map(&tmem_empty_bar, 0);
        const int C = p.C;
        const int row_in_tile = static_cast<int>(rank) * kPHalf + q * 32 + lane;
        const int gi = I * kPTile + row_in_tile;             // this thread's row of H
        for (int chunk = 0; chunk < nchunks; ++chunk) {
            bool got = mbar_wait(&tmem_full_bar, static_cast<uint32_t>(chunk) & 1u, abort, p.limit_ns);
            got = __all_sync(0xffffffffu, got);
            if (!got) break;
            tc_fence_after();
            const bool final_chunk = (chunk == nchunks - 1);
#pragma unroll 1
            for (int blk = 0; blk < kPTile / 32; ++blk) {
                uint32_t a[32];
                tmem_ld_32x32b_x32(lane_base + blk * 32, a);
                if (chunk > 0) {
                    uint32_t m[32];
                    tmem_ld_32x32b_x32(lane_base + kPTile + blk * 32, m);
                    tmem_ld_wait();
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj)
                        a[jj] = __float_as_uint(__fadd_rn(__uint_as_float(m[jj]), __uint_as_float(a[jj])));
                } else {
                    tmem_ld_wait();
                }
                if (!final_chunk) {
                    tmem_st_32x32b_x32(lane_base + kPTile + blk * 32, a);
                    continue;
                }
                // ---- final values of columns gj0 .. gj0+31 of row gi
                const int gj0 = J * kPTile + blk * 32;
                if (nparts > 1) {
                    // partial of this part: workspace [slot][column 256][row 256]
                    float* dst = ws + static_cast<int64_t>(unit - p.plan.split0) * kPTile * kPTile +
                                 static_cast<int64_t>(blk * 32) * kPTile + row_in_tile;
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) dst[jj * kPTile] = __uint_as_float(a[jj]);
                    continue;
                }
                if (gi >= C || (diag && gj0 + 31 < gi)) continue;   // nothing of this block is stored
                float v[32];
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) v[jj] = __uint_as_float(a[jj]) * p.inv_n;
                float* hrow = H + static_cast<int64_t>(gi) * C;
                if (gj0 + 32 <= C && (!diag || gj0 >= gi)) {
                    float4* d4 = reinterpret_cast<float4*>(hrow + gj0);
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        d4[x] = make_float4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
                } else {
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) {
                        const int gj = gj0 + jj;
                        if (gj < C && (!diag || gi <= gj)) hrow[gj] = v[jj];
                    }
                }
                // mirror: for a fixed column the 32 lanes write 32 consecutive floats
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) {
                    const int gj = gj0 + jj;
                    if (gj < C && (!diag || gi <= gj)) H[static_cast<int64_t>(gj) * C + gi] = v[jj];
                }
            }
            if (!final_chunk) {
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_remote(empty_leader);
            }
        }
    }

    tc_fence_before();
    cluster_sync_all();      // no CTA leaves while its peer may still signal its barriers
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kPTmemCols);
    }
}

// Adds the S partials of every tile cut into parts in fixed order, scales by
// 1/n and stores the tile's upper part and its mirror.  One 32x32 block of a
// tile per CTA of 32x8 threads (blockIdx.x counts the cut tiles from split0);
// the row-major store goes through a shared transpose so both stores are
// coalesced.
__global__ void __launch_bounds__(256)
hessian_reduce_kernel(const float* __restrict__ ws, const HessParams p, float* __restrict__ H) {
    __shared__ float blk[32][33];
    const int tile = p.plan.split0 + static_cast<int>(blockIdx.x);
    const int slot0 = static_cast<int>(blockIdx.x) * p.plan.split;
    const int bi = blockIdx.y >> 3;     // 8 x 8 blocks of 32 in a 256 tile
    const int bj = blockIdx.y & 7;
    int I, J;
    hess_tile_coords(tile, p.plan.nb, I, J);
    const bool diag = (I == J);
    if (diag && bj < bi) return;        // entirely below the diagonal
    const int C = p.C;
    const int S = p.plan.split;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    // read: lanes along rows i
    for (int jj = ty; jj < 32; jj += 8) {
        const int i = bi * 32 + tx, j = bj * 32 + jj;
        float s = 0.0f;
        for (int part = 0; part < S; ++part)
            s = __fadd_rn(s, ws[static_cast<int64_t>(slot0 + part) * kPTile * kPTile +
                                static_cast<int64_t>(j) * kPTile + i]);
        s *= p.inv_n;
        blk[tx][jj] = s;
        const int gi = I * kPTile + i, gj = J * kPTile + j;
        if (gi < C && gj < C && (!diag || gi <= gj)) H[static_cast<int64_t>(gj) * C + gi] = s;  // mirror
    }
    __syncthreads();
    // write: lanes along columns j
    for (int ii = ty; ii < 32; ii += 8) {
        const int i = bi * 32 + ii, j = bj * 32 + tx;
        const int gi = I * kPTile + i, gj = J * kPTile + j;
        if (gi < C && gj < C && (!diag || gi <= gj)) H[static_cast<int64_t>(gi) * C + gj] = blk[ii][tx];
    }
}

}  // namespace qat4
