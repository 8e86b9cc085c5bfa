// hessian.cuh -- calibration Hessian H = X^T X / n on the 5th-generation
// tensor cores (blog "Opt.Gear-QAT", section 2 "Hessian-based scale
// initialize": layer sensitivity from calibration activations, the
// second-order output-reconstruction view).
//
// X is bf16 [n, C] row-major, so in the product D[i][j] = sum_t X[t][i] X[t][j]
// the reduction index t is X's row index and both operands are "MN-major"
// (M resp. N contiguous in memory).  Only upper-triangle 128x128 output tiles
// (I <= J) are computed; each is written together with its mirror, so H comes
// out bitwise symmetric.
//
// One CTA per upper tile, 6 warps:
//   warp 0      TMA producer: 64-row x 128-column boxes of X (two 64x64 boxes
//               per operand, 128-byte swizzle) into a 6-stage shared ring;
//               diagonal tiles load one operand and use it twice;
//   warp 1      allocates 2 x 128 TMEM columns and issues tcgen05.mma
//               (kind::f16, M=128, N=128, K=16, both operands MN-major,
//               fp32 accumulators in TMEM); tcgen05.commit frees ring slots;
//   warps 2..5  epilogue: warp w owns TMEM lanes 32*(w%4)..+31 (= tile rows).
// Chunked promotion: the tensor core accumulates kHChunkKB stages (1024 rows
// of X) into one of two TMEM buffers; the epilogue warps add each finished
// chunk into a float32 register accumulator (128 values per thread, IEEE
// round-to-nearest adds) while the MMA fills the other buffer.  This bounds
// the error of the tensor core's internal accumulation to 1024-term sums; a
// single accumulator over n = 262144 rows drifts by more than 1e-3.  At the
// end the epilogue scales by 1/n and stores the tile and its transpose.
// All CTAs walk the reduction dimension in the same order and at the same
// rate, so each 64-row slab of X is fetched from HBM about once and then
// served to every tile from L2.
//
// Every mbarrier wait is bounded (device_common.cuh); on a timeout the CTA
// stops issuing work, waits (bounded) for its own copies and MMAs in flight,
// frees its TMEM and exits, leaving QAT4_DEV_ERR_TIMEOUT in the error word.
#pragma once

#include "device_common.cuh"

namespace qat4 {

constexpr int kHBM = 128;                    // tile rows (M) = tile cols (N)
constexpr int kHBK = 64;                     // X rows per pipeline stage
constexpr int kHStages = 6;
constexpr int kHThreads = 192;
constexpr uint32_t kHBoxBytes = 64 * kHBK * 2;          // one 64x64 bf16 box = 8 KB
constexpr uint32_t kHOperandBytes = 2 * kHBoxBytes;     // 128 columns = 16 KB
constexpr uint32_t kHStageBytes = 2 * kHOperandBytes;   // A + B = 32 KB
constexpr uint32_t kHSmemBytes = kHStages * kHStageBytes + 1024;  // + alignment slack
constexpr uint32_t kHTmemCols = 256;          // two 128-column accumulators
constexpr int kHChunkKB = 16;                 // stages per promotion chunk (1024 rows)

// Instruction descriptor, kind::f16: D fp32, A/B bf16, A and B MN-major,
// N = 128, M = 128.
constexpr uint32_t kHIdesc = (1u << 4)            // D format: F32
                           | (1u << 7)            // A format: BF16
                           | (1u << 10)           // B format: BF16
                           | (1u << 15)           // A major: MN
                           | (1u << 16)           // B major: MN
                           | ((128u >> 3) << 17)  // N >> 3
                           | ((128u >> 4) << 24); // M >> 4

// Shared-memory matrix descriptor for one operand tile laid out as
// [2 column halves][64 rows][128 B] with the 128-byte swizzle:
// leading byte offset = distance between the two 64-column halves (8 KB),
// stride byte offset = distance between 8-row groups (1 KB).
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t saddr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((kHBoxBytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((1024u >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;   // descriptor version (sm_100)
    d |= static_cast<uint64_t>(2) << 61;   // SWIZZLE_128B
    return d;
}

// Upper-triangle tile t -> (I, J), I <= J, enumerated row by row.
__device__ __forceinline__ void hess_tile_coords(int t, int nb, int& I, int& J) {
    int i = 0;
    int rowlen = nb;
    while (t >= rowlen) { t -= rowlen; ++i; --rowlen; }
    I = i;
    J = i + t;
}

struct HessParams {
    int64_t n;
    int C;
    int nb;              // ceil(C / 128)
    int kblocks;         // ceil(n / 64)
    float inv_n;
    uint64_t limit_ns;   // bounded-wait limit
};

constexpr uint64_t kDrainLimitNs = 1000000000ull;   // bounded drain on the error path

__global__ void __launch_bounds__(kHThreads, 1)
hessian_tc_kernel(const __grid_constant__ CUtensorMap tmap, const HessParams p, float* __restrict__ H) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_bar[kHStages];
    __shared__ __align__(8) uint64_t empty_bar[kHStages];
    __shared__ __align__(8) uint64_t tmem_full_bar[2];
    __shared__ __align__(8) uint64_t tmem_empty_bar[2];
    __shared__ __align__(8) uint64_t mma_done_bar;
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // the 128-byte swizzle pattern is anchored at 1024-byte boundaries
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

    int I, J;
    hess_tile_coords(static_cast<int>(blockIdx.x), p.nb, I, J);
    const bool diag = (I == J);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kHStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tmem_full_bar[b], 1);
            mbar_init(&tmem_empty_bar[b], 4);   // one arrive per epilogue warp
        }
        mbar_init(&mma_done_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap);
    }
    if (warp == 1) {
        tmem_alloc(&tmem_slot, kHTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    volatile int* abort = &abort_flag;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            const uint32_t tx = diag ? kHOperandBytes : kHStageBytes;
            int issued = 0;
            for (int kb = 0; kb < p.kblocks; ++kb) {
                const int s = kb % kHStages;
                const uint32_t ph = static_cast<uint32_t>(kb / kHStages) & 1u;
                if (!mbar_wait(&empty_bar[s], ph ^ 1u, abort, p.limit_ns)) break;
                uint8_t* sa = smem + s * kHStageBytes;
                uint8_t* sb = sa + kHOperandBytes;
                const int y = kb * kHBK;
                mbar_arrive_expect_tx(&full_bar[s], tx);
                tma_load_2d(sa, &tmap, &full_bar[s], I * kHBM, y);
                tma_load_2d(sa + kHBoxBytes, &tmap, &full_bar[s], I * kHBM + 64, y);
                if (!diag) {
                    tma_load_2d(sb, &tmap, &full_bar[s], J * kHBM, y);
                    tma_load_2d(sb + kHBoxBytes, &tmap, &full_bar[s], J * kHBM + 64, y);
                }
                issued = kb + 1;
            }
            // no copy may still be landing in shared memory when the CTA exits
            for (int kb = (issued > kHStages ? issued - kHStages : 0); kb < issued; ++kb)
                mbar_wait(&full_bar[kb % kHStages], static_cast<uint32_t>(kb / kHStages) & 1u,
                          nullptr, kDrainLimitNs);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            bool ok = true;
            for (int kb = 0; kb < p.kblocks && ok; ++kb) {
                const int chunk = kb / kHChunkKB;
                const int buf = chunk & 1;
                const bool first = (kb % kHChunkKB) == 0;
                const bool last = (kb % kHChunkKB) == kHChunkKB - 1 || kb == p.kblocks - 1;
                if (first && chunk >= 2) {
                    // the epilogue must have drained this buffer (chunk - 2)
                    if (!mbar_wait(&tmem_empty_bar[buf], static_cast<uint32_t>((chunk >> 1) - 1) & 1u, abort,
                                   p.limit_ns)) { ok = false; break; }
                    tc_fence_after();
                }
                const int s = kb % kHStages;
                const uint32_t ph = static_cast<uint32_t>(kb / kHStages) & 1u;
                if (!mbar_wait(&full_bar[s], ph, abort, p.limit_ns)) { ok = false; break; }
                tc_fence_after();
                const uint32_t sa = smem_u32(smem + s * kHStageBytes);
                const uint32_t sb = diag ? sa : sa + kHOperandBytes;
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kHBM);
#pragma unroll
                for (int kk = 0; kk < kHBK / 16; ++kk) {
                    // K = 16 rows of X = two 8-row swizzle groups = 2 KB further on
                    tc_mma_f16(d_tmem, smem_desc_mn_sw128(sa + kk * 2048u),
                               smem_desc_mn_sw128(sb + kk * 2048u), kHIdesc,
                               (!first || kk > 0) ? 1u : 0u);
                }
                tc_commit(&empty_bar[s]);
                if (last) tc_commit(&tmem_full_bar[buf]);
            }
            // every MMA must have retired before TMEM is released
            tc_commit(&mma_done_bar);
            mbar_wait(&mma_done_bar, 0, nullptr, kDrainLimitNs);
        }
    } else {
        // ---------------- epilogue: warps 2..5
        const int q = warp & 3;                       // TMEM lanes 32q..32q+31
        const int nchunks = (p.kblocks + kHChunkKB - 1) / kHChunkKB;
        float acc[kHBM];
#pragma unroll
        for (int j = 0; j < kHBM; ++j) acc[j] = 0.0f;
        bool ok = true;
        for (int chunk = 0; chunk < nchunks; ++chunk) {
            const int buf = chunk & 1;
            bool got = mbar_wait(&tmem_full_bar[buf], static_cast<uint32_t>(chunk >> 1) & 1u, abort, p.limit_ns);
            got = __all_sync(0xffffffffu, got);
            if (!got) { ok = false; break; }
            tc_fence_after();
            const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(buf * kHBM);
#pragma unroll
            for (int c = 0; c < kHBM / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(taddr + c * 32, r);
                tmem_ld_wait();
#pragma unroll
                for (int jj = 0; jj < 32; ++jj) acc[c * 32 + jj] = __fadd_rn(acc[c * 32 + jj], __uint_as_float(r[jj]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty_bar[buf]);
        }
        if (ok) {
            const int C = p.C;
            const int gi = I * kHBM + q * 32 + lane;  // this thread's row of H
            if (gi < C) {
                float* hrow = H + static_cast<int64_t>(gi) * C;
#pragma unroll
                for (int c = 0; c < kHBM / 32; ++c) {
                    float v[32];
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) v[jj] = acc[c * 32 + jj] * p.inv_n;
                    const int gj0 = J * kHBM + c * 32;
                    if (gj0 + 32 <= C && (!diag || gj0 >= gi)) {
                        float4* dst = reinterpret_cast<float4*>(hrow + gj0);
#pragma unroll
                        for (int x = 0; x < 8; ++x)
                            dst[x] = make_float4(v[4 * x], v[4 * x + 1], v[4 * x + 2], v[4 * x + 3]);
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
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem_base, kHTmemCols);
    }
}

}  // namespace qat4
