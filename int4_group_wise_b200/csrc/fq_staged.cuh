// fq_staged.cuh -- the fake-quant forward product of a QAT step in two
// kernels (blog "Opt.Gear-QAT", section 3 "LSQ-based QAT": the forward pass
// runs on the weights projected onto the deployment INT4 grid):
//     Qb = bf16(Q_Delta(W))          (fq_quantize_kernel, HBM-bound)
//     Y  = X * Qb^T                  (gemm_bf16_pair_kernel, tensor cores)
// The quantizer is the one of the fused kernel (fq_half_group: the LSQ
// forward's code decision, Delta * q in binary32, bf16 round-to-nearest-even),
// so Y is the same product; Qb (R x C bf16, 33.5 MB for an 8192 x 2048 layer)
// lives in a caller workspace and mostly in L2 by the time the GEMM reads it.
// Splitting the work lets the GEMM run as a plain bf16 mainloop: the fused
// kernel's float32 W tiles doubled the operand bytes of every MMA step and its
// quantizer warps had to keep pace with the tensor core.
//
// GEMM.  Persistent: one CTA pair per SM pair walks output tiles of 256 rows
// of X (tokens) x 256 rows of Qb, cta_group::2 (M = 256, N = 256, K = 16),
// both operands K-major in the 128-byte swizzle (CTA r holds rows
// 128r..128r+127 of each operand's tile).  128-deep K stages (eight MMAs per
// barrier hand-off), three stages of 64 KB.  Two 256-column TMEM accumulators
// alternate between tiles, so the epilogue of one tile (tcgen05.ld, float32
// stores) runs while the tensor core computes the next.  No load is multicast.
//
// Warps of each CTA: warp 0 TMA producer (both CTAs; the peer's copies complete
// on the leader's barrier), warp 1 TMEM allocation and, in the leader, the MMA
// issuer, warps 2..5 epilogue over TMEM lanes 32*(w%4)..+31.
//
// Every mbarrier wait is bounded (device_common.cuh); on a timeout a CTA stops
// issuing work, waits (bounded) for its copies and MMAs in flight, frees its
// TMEM and exits, leaving QAT4_DEV_ERR_TIMEOUT in the error word.
#pragma once

#include <cuda.h>

#include "device_common.cuh"
#include "fq_gemm.cuh"

namespace qat4 {

// ---------------------------------------------------------------- quantize
// Thread i converts weights 16i..16i+15 of the row-major W (half of group i/2).
constexpr int kFqQuantBlock = 256;
__global__ void __launch_bounds__(kFqQuantBlock)
fq_quantize_kernel(const float* __restrict__ W, const float* __restrict__ delta, int64_t nhalf,
                   uint16_t* __restrict__ Qb) {
    pdl_launch_dependents();      // the GEMM may set up while the last blocks convert
    const int64_t i = static_cast<int64_t>(blockIdx.x) * kFqQuantBlock + threadIdx.x;
    if (i >= nhalf) return;
    const float4* w4 = reinterpret_cast<const float4*>(W) + 4 * i;
    const float4 wv[4] = {__ldcs(w4), __ldcs(w4 + 1), __ldcs(w4 + 2), __ldcs(w4 + 3)};
    uint4 out[2];
    fq_half_group(wv, __ldg(delta + (i >> 1)), out);
    uint4* q = reinterpret_cast<uint4*>(Qb) + 2 * i;
    q[0] = out[0];
    q[1] = out[1];
}

// -------------------------------------------------------------------- GEMM
constexpr int kGTile = 256;                             // tile rows of A (tokens) = tile rows of B
constexpr int kGHalf = 128;                             // per CTA
constexpr int kGBK = 128;                               // K per stage
constexpr int kGStages = 3;
constexpr int kGThreads = 192;
constexpr int kGPairsPerGpu = 74;
constexpr uint32_t kGBoxBytes = kGHalf * 64 * 2;        // 128 rows x 64 K bf16 (one 128-byte swizzle row each)
constexpr uint32_t kGOperandBytes = 2 * kGBoxBytes;     // 128 rows x 128 K = 32 KB
constexpr uint32_t kGStageBytes = 2 * kGOperandBytes;   // A + B = 64 KB
constexpr uint32_t kGStoreBytes = 32 * 32 * 4;          // one 32 x 32 float32 block of Y (4 KB)
constexpr uint32_t kGEpiBytes = 4 * 2 * kGStoreBytes;    // two staging blocks per epilogue warp
constexpr uint32_t kGSmemBytes = kGStages * kGStageBytes + kGEpiBytes + 1024;
constexpr uint32_t kGTmemCols = 512;                    // two 256-column accumulators

// kind::f16: D float32, A and B bf16, both K-major, N = 256, M = 256 (pair).
constexpr uint32_t kGIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((256u >> 3) << 17) | ((256u >> 4) << 24);

struct GemmParams {
    float* Y;            // [T, R] row-major
    int T, R, C;
    int tma_store;       // Y's rows are 16-byte aligned (R % 4 == 0): blocks leave by bulk-tensor stores
    int tiles_m;         // ceil(T / 256)
    int tiles;           // tiles_m * ceil(R / 256)
    int ksteps;          // ceil(C / 128)
    uint64_t limit_ns;
};

// Bulk-tensor store of one staged block (shared -> global), tracked as a bulk group of this thread.
__device__ __forceinline__ void tma_store_2d(const void* tmap, uint32_t src, int32_t c0, int32_t c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];"
                 :: "l"(tmap), "r"(c0), "r"(c1), "r"(src) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Waits until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read %0;" :: "n"(N) : "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kGThreads, 1)
gemm_bf16_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                      const __grid_constant__ CUtensorMap tmap_y, const GemmParams p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kGStages];    // leader: both CTAs' bytes
    __shared__ __align__(8) uint64_t empty_bar[kGStages];   // MMA commit, both CTAs
    __shared__ __align__(8) uint64_t tfull_bar[2];          // accumulator b holds a finished tile (both CTAs)
    __shared__ __align__(8) uint64_t tempty_bar[2];         // leader: both epilogues have read accumulator b
    __shared__ __align__(8) uint64_t mma_done_bar;          // leader
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int pair = static_cast<int>(blockIdx.x >> 1);
    const int npairs = static_cast<int>(gridDim.x >> 1);
    const int nk = p.ksteps;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], 8);   // 4 epilogue warps in each CTA of the pair
        }
        mbar_init(&mma_done_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
        if (p.tma_store) prefetch_tmap(&tmap_y);
    }
    if (warp == 1) {
        tmem_alloc_pair(&tmem_slot, kGTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();      // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    volatile int* abort = &abort_flag;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs), all of this pair's tiles
            pdl_wait();           // Qb is written by the quantizer launched just before
            int it = 0, issued = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < p.tiles; tile += npairs) {
                const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
                const int ya = tm * kGTile + static_cast<int>(rank) * kGHalf;   // this CTA's rows of X
                const int yb = tn * kGTile + static_cast<int>(rank) * kGHalf;   // this CTA's rows of Qb
                for (int k = 0; k < nk; ++k, ++it) {
                    const int s = it % kGStages;
                    const uint32_t ph = static_cast<uint32_t>(it / kGStages) & 1u;
                    if (!mbar_wait(&empty_bar[s], ph ^ 1u, abort, p.limit_ns)) { ok = false; break; }
                    uint8_t* sa = smem + s * kGStageBytes;
                    uint8_t* sb = sa + kGOperandBytes;
                    const uint32_t fb = cluster_map(&full_bar[s], 0);
                    if (rank == 0) mbar_arrive_expect_tx(&full_bar[s], 2 * kGStageBytes);
                    const int x = k * kGBK;
                    tma_load_2d_pair(sa, &tmap_a, fb, x, ya);
                    tma_load_2d_pair(sa + kGBoxBytes, &tmap_a, fb, x + 64, ya);
                    tma_load_2d_pair(sb, &tmap_b, fb, x, yb);
                    tma_load_2d_pair(sb + kGBoxBytes, &tmap_b, fb, x + 64, yb);
                    issued = it + 1;
                }
            }
            // no copy may still be landing in shared memory when the CTA exits (as in the Hessian)
            for (int i = (issued > kGStages ? issued - kGStages : 0); i < issued; ++i) {
                if (rank == 0)
                    mbar_wait_cluster(&full_bar[i % kGStages], static_cast<uint32_t>(i / kGStages) & 1u,
                                      nullptr, kDrainLimitNs);
                else
                    mbar_wait(&empty_bar[i % kGStages], static_cast<uint32_t>(i / kGStages) & 1u,
                              nullptr, kDrainLimitNs);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------- MMA issuer (leader CTA only)
            int it = 0, j = 0;
            bool ok = true;
            for (int tile = pair; ok && tile < p.tiles; tile += npairs, ++j) {
                const int b = j & 1;
                if (j >= 2) {   // both epilogues have read accumulator b (tile j - 2)
                    if (!mbar_wait_cluster(&tempty_bar[b], static_cast<uint32_t>((j >> 1) - 1) & 1u, abort,
                                           p.limit_ns)) break;
                    tc_fence_after();
                }
                const uint32_t d = tmem_base + static_cast<uint32_t>(b) * 256u;
                for (int k = 0; k < nk; ++k, ++it) {
                    const int s = it % kGStages;
                    const uint32_t ph = static_cast<uint32_t>(it / kGStages) & 1u;
                    if (!mbar_wait_cluster(&full_bar[s], ph, abort, p.limit_ns)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(smem + s * kGStageBytes);
                    const uint32_t sb = sa + kGOperandBytes;
#pragma unroll
                    for (int kk = 0; kk < kGBK / 16; ++kk) {
                        // K = 16 columns = 32 bytes along a 128-byte swizzle row; the second box holds K 64..127
                        const uint32_t off = static_cast<uint32_t>(kk & 3) * 32u + static_cast<uint32_t>(kk >> 2) * kGBoxBytes;
                        tc_mma_f16_pair(d, smem_desc_k_sw128(sa + off), smem_desc_k_sw128(sb + off), kGIdesc,
                                        (k > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit_pair_mc(&empty_bar[s], 0x3);
                }
                if (!ok) break;
                tc_commit_pair_mc(&tfull_bar[b], 0x3);
            }
            // every MMA must have retired before TMEM is released
            tc_commit_pair(&mma_done_bar);
            mbar_wait(&mma_done_bar, 0, nullptr, kDrainLimitNs);
        }
    } else {
        // ---------------- epilogue: warps 2..5 of both CTAs
        // Each warp moves its 32 rows of the tile in 32 x 32 blocks: with 16-byte aligned rows of Y,
        // a block is written into one of the warp's two shared staging buffers (128-byte swizzle)
        // and leaves by a bulk-tensor store, so Y is written in whole lines; otherwise each thread
        // stores its own row's 32 values.
        const int q = warp & 3;                                  // TMEM lanes 32q..32q+31
        const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
        const uint32_t empty_leader0 = cluster_map(&tempty_bar[0], 0);
        const uint32_t empty_leader1 = cluster_map(&tempty_bar[1], 0);
        const uint32_t stage0 = smem_u32(smem + kGStages * kGStageBytes) + static_cast<uint32_t>(q) * 2 * kGStoreBytes;
        const uint32_t swz = static_cast<uint32_t>(lane) & 7u;
        int j = 0, nstore = 0;
        for (int tile = pair; tile < p.tiles; tile += npairs, ++j) {
            const int b = j & 1;
            bool got = mbar_wait(&tfull_bar[b], static_cast<uint32_t>(j >> 1) & 1u, abort, p.limit_ns);
            got = __all_sync(0xffffffffu, got);
            if (!got) break;
            tc_fence_after();
            const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
            const int row0 = tm * kGTile + static_cast<int>(rank) * kGHalf + q * 32;   // the warp's first row of Y
            const int t = row0 + lane;                                                 // this thread's row
            float* yrow = p.Y + static_cast<int64_t>(t) * p.R;
#pragma unroll 1
            for (int blk = 0; blk < kGTile / 32; ++blk) {
                uint32_t a[32];
                tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(b) * 256u + blk * 32, a);
                tmem_ld_wait();
                const int c0 = tn * kGTile + blk * 32;
                if (row0 >= p.T || c0 >= p.R) continue;
                if (p.tma_store) {
                    // the buffer used two blocks ago must have been read by its store
                    const uint32_t buf = stage0 + static_cast<uint32_t>(nstore & 1) * kGStoreBytes;
                    if (lane == 0) bulk_wait_read<1>();
                    __syncwarp();
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                     :: "r"(buf + static_cast<uint32_t>(lane) * 128u + ((static_cast<uint32_t>(c) ^ swz) << 4)),
                                        "r"(a[4 * c]), "r"(a[4 * c + 1]), "r"(a[4 * c + 2]), "r"(a[4 * c + 3])
                                     : "memory");
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmap_y, buf, c0, row0);    // rows past T and columns past R are clipped
                        bulk_commit();
                    }
                    ++nstore;
                    continue;
                }
                if (t >= p.T) continue;
                if (c0 + 32 <= p.R && (p.R & 3) == 0) {
                    float4* d4 = reinterpret_cast<float4*>(yrow + c0);
#pragma unroll
                    for (int x = 0; x < 8; ++x)
                        __stcs(d4 + x, make_float4(__uint_as_float(a[4 * x]), __uint_as_float(a[4 * x + 1]),
                                                   __uint_as_float(a[4 * x + 2]), __uint_as_float(a[4 * x + 3])));
                } else {
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj)
                        if (c0 + jj < p.R) __stcs(yrow + c0 + jj, __uint_as_float(a[jj]));
                }
            }
            // accumulator b may take tile j + 2
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(b ? empty_leader1 : empty_leader0);
        }
        // the staging buffers must outlive the stores that read them
        if (lane == 0) bulk_wait_all();
        __syncwarp();
    }

    tc_fence_before();
    cluster_sync_all();      // no CTA leaves while its peer may still signal its barriers
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kGTmemCols);
    }
}

}  // namespace qat4
