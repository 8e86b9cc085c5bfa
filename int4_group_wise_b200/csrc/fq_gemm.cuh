// fq_gemm.cuh -- the fake-quant forward product of a QAT step,
//     Y = X * bf16(Q_Delta(W))^T,   Q_Delta(w) = Delta * clamp(rint(w / Delta), -8, 7)
// (blog "Opt.Gear-QAT", section 3 "LSQ-based QAT": the forward pass runs on the
// weights projected onto the INT4 grid that deployment uses), with the
// quantizer inside the producer of a 5th-generation tensor-core GEMM: W stays
// float32 in HBM, each CTA turns its tile of W into bf16 codes-times-scale in
// shared memory, and the tensor core multiplies them with bf16 X, accumulating
// in float32.  Q_Delta is computed exactly as the LSQ forward computes it (the
// same code decision), then rounded to bf16 to nearest even.
//
// X is bf16 [T, C] and W float32 [R, C], both row-major, so both operands are
// K-major.  A 256 x 256 output tile (256 tokens x 256 rows of W) belongs to a
// cluster of two CTAs on an SM pair, tcgen05.mma.cta_group::2 (M = 256,
// N = 256, K = 16): CTA r holds tokens 128r..128r+127 of the A operand and
// rows 128r..128r+127 of the B operand, so each SM quantizes half of the
// tile's weights.  Operands use the canonical K-major 128-byte swizzle (row of
// 64 bf16 = 128 B; 8-row atoms of 1 KB; 16-byte chunk c of row n at
// n*128 + (c ^ (n & 7)) * 16).
//
// A pair computes two token tiles (512 tokens) against the same W tile, so
// every quantized B serves two M = 256 MMAs (two 256-column TMEM
// accumulators): half the quantization per tensor-core flop.
//
// Warps of each CTA (576 threads):
//   warp 0      producer: per 64-column step, two 32x128 float32 boxes of W into
//               a 2-slot W ring (complete on this CTA's barrier) and two
//               64x128 bf16 boxes of X (the CTA's 128 tokens of each token
//               tile; pair form: they complete on the leader's barrier, never
//               multicast) into a 3-stage A/B ring;
//   warp 1      allocates the pair's 512 TMEM columns; in the leader CTA one
//               thread issues the MMAs and commits each stage to both CTAs;
//               in the peer CTA, one thread of warp 1 forwards "B written" to
//               the leader: one cluster-scope release per step;
//   warps 2..17 quantizers: thread (row n, quarter k) turns 16 weights (half
//               of group 2*step + k/2) of row n into 16 bf16 values of B,
//               fences them for the tensor core's proxy, and each warp frees
//               the W slot and marks B written on this CTA's barriers.  After
//               the main loop the same warps are the epilogue (TMEM lanes
//               32*(warp%4).., column quarter (warp-2)/4), storing float32 Y
//               through a shared transpose.
//
// Every mbarrier wait is bounded (device_common.cuh); on a timeout a CTA stops
// issuing work, waits (bounded) for its own copies and MMAs in flight, frees
// its TMEM and exits, leaving QAT4_DEV_ERR_TIMEOUT in the error word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "device_common.cuh"

namespace qat4 {

constexpr int kFqTile = 256;                  // tokens x W rows per pair tile
constexpr int kFqHalf = 128;                  // per CTA
constexpr int kFqMTiles = 2;                  // token tiles per pair sharing one quantized B
constexpr int kFqBK = 64;                     // columns of X / W per stage
constexpr int kFqStages = 3;                  // A/B ring
constexpr int kFqWStages = 2;                 // W ring
constexpr int kFqQuantWarps = 16;
constexpr int kFqThreads = 64 + 32 * kFqQuantWarps;            // 576
constexpr uint32_t kFqABytes = kFqHalf * kFqBK * 2;             // 16 KB bf16 X box (one token tile)
constexpr uint32_t kFqWBoxBytes = kFqHalf * 32 * 4;             // 16 KB float32 W box (32 columns)
constexpr uint32_t kFqWBytes = 2 * kFqWBoxBytes;                // 32 KB
constexpr uint32_t kFqBBytes = kFqHalf * kFqBK * 2;             // 16 KB bf16 B
constexpr uint32_t kFqABStageBytes = kFqMTiles * kFqABytes + kFqBBytes;   // 48 KB
constexpr uint32_t kFqWRingBytes = kFqWStages * kFqWBytes;                // 64 KB
constexpr uint32_t kFqSmemBytes = kFqWRingBytes + kFqStages * kFqABStageBytes + 1024;
constexpr uint32_t kFqTmemCols = 256 * kFqMTiles;

// Instruction descriptor, kind::f16: D fp32, A/B bf16, both K-major, N = 256, M = 256 (pair).
constexpr uint32_t kFqIdesc = (1u << 4)            // D format: F32
                            | (1u << 7)            // A format: BF16
                            | (1u << 10)           // B format: BF16
                            | ((256u >> 3) << 17)  // N >> 3
                            | ((256u >> 4) << 24); // M >> 4

struct FqParams {
    const float* delta;   // [R, C/32]
    float* Y;             // [T, R]
    int T, R, C, G;       // G = C / 32
    int tiles_r;          // ceil(R / 256)
    int ksteps;           // ceil(C / 64)
    uint64_t limit_ns;
};

__device__ __forceinline__ float4 fq_lds128(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a));
    return v;
}
__device__ __forceinline__ void fq_sts128(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" :: "r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}
__device__ __forceinline__ void fq_sts32(uint32_t a, float v) {
    asm volatile("st.shared.f32 [%0], %1;" :: "r"(a), "f"(v) : "memory");
}
__device__ __forceinline__ float fq_lds32(uint32_t a) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(a) : "memory");
    return v;
}
// One thread's 16 weights (half a group) -> 16 bf16 values of Q_Delta, as 2 x uint4 (element 2i
// in the low half of word i).  The code is rint(w * (1/Delta)) clamped to [-8, 7]; it equals the
// code of the IEEE quotient w / Delta unless a product lands within 2^-18 of a half-integer
// (w * rcp is within 3 ulp of the quotient), or 1/Delta is not finite: then the IEEE division is
// redone for the 16 weights.  Delta == 0 (all-zero group) gives 0.
__device__ __forceinline__ void fq_half_group(const float4 (&wv)[4], float d, uint4 (&out)[2]) {
    constexpr float kM = 12582912.0f;                       // 1.5 * 2^23
    constexpr float kWin = 0.5f - 3.814697265625e-06f;      // 0.5 - 2^-18
    const float rc = __frcp_rn(d);
    float2 qf[8];
    float m = 0.0f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const float4& v = wv[e >> 1];
        const float2 w = (e & 1) ? make_float2(v.z, v.w) : make_float2(v.x, v.y);
        float2 r = __fmul2_rn(w, make_float2(rc, rc));
        r.x = fminf(fmaxf(r.x, kQmin), kQmax);
        r.y = fminf(fmaxf(r.y, kQmin), kQmax);
        qf[e] = __fadd2_rn(__fadd2_rn(r, make_float2(kM, kM)), make_float2(-kM, -kM));   // rint
        const float2 f = __fadd2_rn(r, make_float2(-qf[e].x, -qf[e].y));                  // r - q
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
    if (!(m <= kWin) || !(fabsf(rc) <= 3.4028234663852886e38f)) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float4& v = wv[e >> 1];
            qf[e].x = code_of(scaled_exact((e & 1) ? v.z : v.x, d));
            qf[e].y = code_of(scaled_exact((e & 1) ? v.w : v.y, d));
        }
    }
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        uint32_t o[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const float2 q = __fmul2_rn(qf[4 * j + e], make_float2(d, d));   // Q = fl(Delta * q)
            const __nv_bfloat162 hq = __float22bfloat162_rn(q);             // .x -> low half
            o[e] = *reinterpret_cast<const uint32_t*>(&hq);
        }
        out[j] = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kFqThreads, 1)
fq_gemm_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_w,
               const FqParams p) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t full_a[kFqStages];     // leader: both CTAs' X bytes
    __shared__ __align__(8) uint64_t bdone[kFqStages];      // this CTA's 8 quantizer warps wrote B
    __shared__ __align__(8) uint64_t bready[kFqStages];     // leader: the peer's B is written
    __shared__ __align__(8) uint64_t ab_empty[kFqStages];   // MMA commit, both CTAs
    __shared__ __align__(8) uint64_t full_w[kFqWStages];    // this CTA's W bytes
    __shared__ __align__(8) uint64_t w_empty[kFqWStages];   // the quantizer warps are done with the W slot
    __shared__ __align__(8) uint64_t tmem_full_bar;
    __shared__ __align__(8) uint64_t mma_done_bar;          // leader
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    // 1 KB-aligned base of the dynamic shared memory, as a shared-window address and a pointer
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
    uint8_t* smem = smem_raw + pad;
    const uint32_t sbase = raw + pad;
    const uint32_t w_ring = sbase;                           // [kFqWStages][2 boxes][128 rows][128 B]
    const uint32_t ab_ring = sbase + kFqWRingBytes;          // [kFqStages][A tile 0, A tile 1, B]

    const int pair_tile = static_cast<int>(blockIdx.x >> 1);
    const int tm = pair_tile / p.tiles_r, tr = pair_tile - tm * p.tiles_r;
    const int r0 = tr * kFqTile + static_cast<int>(rank) * kFqHalf;    // this CTA's first W row
    const int nk = p.ksteps;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kFqStages; ++s) {
            mbar_init(&full_a[s], 1);
            mbar_init(&bdone[s], kFqQuantWarps);
            mbar_init(&bready[s], 1);
            mbar_init(&ab_empty[s], 1);
        }
        for (int s = 0; s < kFqWStages; ++s) {
            mbar_init(&full_w[s], 1);
            mbar_init(&w_empty[s], kFqQuantWarps);
        }
        mbar_init(&tmem_full_bar, 1);
        mbar_init(&mma_done_bar, 1);
        abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmap_x);
        prefetch_tmap(&tmap_w);
    }
    if (warp == 1) {
        tmem_alloc_pair(&tmem_slot, kFqTmemCols);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    cluster_sync_all();      // barriers of both CTAs initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem_base = tmem_slot;
    volatile int* abort = &abort_flag;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- producer (both CTAs)
            int issued_w = 0, issued_a = 0;
            for (int i = 0; i < nk; ++i) {
                const int k0 = i * kFqBK;                           // multiple of 64 columns
                const int sw = i % kFqWStages;
                const uint32_t phw = static_cast<uint32_t>(i / kFqWStages) & 1u;
                if (!mbar_wait(&w_empty[sw], phw ^ 1u, abort, p.limit_ns)) break;
                uint8_t* wdst = smem + sw * kFqWBytes;
                mbar_arrive_expect_tx(&full_w[sw], kFqWBytes);
                tma_load_2d(wdst, &tmap_w, &full_w[sw], k0, r0);
                tma_load_2d(wdst + kFqWBoxBytes, &tmap_w, &full_w[sw], k0 + 32, r0);
                issued_w = i + 1;
                const int s = i % kFqStages;
                const uint32_t ph = static_cast<uint32_t>(i / kFqStages) & 1u;
                if (!mbar_wait(&ab_empty[s], ph ^ 1u, abort, p.limit_ns)) break;
                uint8_t* adst = smem + kFqWRingBytes + s * kFqABStageBytes;
                const uint32_t fa = cluster_map(&full_a[s], 0);
                if (rank == 0) mbar_arrive_expect_tx(&full_a[s], 2 * kFqMTiles * kFqABytes);
#pragma unroll
                for (int mt = 0; mt < kFqMTiles; ++mt)
                    tma_load_2d_pair(adst + mt * kFqABytes, &tmap_x, fa, k0,
                                     (tm * kFqMTiles + mt) * kFqTile + static_cast<int>(rank) * kFqHalf);
                issued_a = i + 1;
            }
            // no copy may still be landing when the CTA exits: W copies complete here; X copies
            // complete on the leader, so the peer waits until the MMAs that read them are done
            for (int i = (issued_w > kFqWStages ? issued_w - kFqWStages : 0); i < issued_w; ++i)
                mbar_wait(&full_w[i % kFqWStages], static_cast<uint32_t>(i / kFqWStages) & 1u, nullptr,
                          kDrainLimitNs);
            for (int i = (issued_a > kFqStages ? issued_a - kFqStages : 0); i < issued_a; ++i) {
                const uint32_t ph = static_cast<uint32_t>(i / kFqStages) & 1u;
                if (rank == 0)
                    mbar_wait_cluster(&full_a[i % kFqStages], ph, nullptr, kDrainLimitNs);
                else
                    mbar_wait(&ab_empty[i % kFqStages], ph, nullptr, kDrainLimitNs);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------- MMA issuer (leader CTA only)
            for (int i = 0; i < nk; ++i) {
                const int s = i % kFqStages;
                const uint32_t ph = static_cast<uint32_t>(i / kFqStages) & 1u;
                if (!mbar_wait_cluster(&full_a[s], ph, abort, p.limit_ns)) break;
                if (!mbar_wait(&bdone[s], ph, abort, p.limit_ns)) break;
                if (!mbar_wait_cluster(&bready[s], ph, abort, p.limit_ns)) break;
                tc_fence_after();
                const uint32_t sa = ab_ring + s * kFqABStageBytes;
                const uint32_t sb = sa + kFqMTiles * kFqABytes;
#pragma unroll
                for (int kk = 0; kk < kFqBK / 16; ++kk) {
                    // K = 16 bf16 = 32 bytes further along the swizzled 128-byte row
                    const uint64_t bdesc = smem_desc_k_sw128(sb + kk * 32u);
#pragma unroll
                    for (int mt = 0; mt < kFqMTiles; ++mt)
                        tc_mma_f16_pair(tmem_base + mt * 256u, smem_desc_k_sw128(sa + mt * kFqABytes + kk * 32u), bdesc,
                                        kFqIdesc, (i > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit_pair_mc(&ab_empty[s], 0x3);
                if (i == nk - 1) tc_commit_pair_mc(&tmem_full_bar, 0x3);
            }
            // every MMA must have retired before TMEM is released
            tc_commit_pair(&mma_done_bar);
            mbar_wait(&mma_done_bar, 0, nullptr, kDrainLimitNs);
        } else if (lane == 0) {
            // ---------------- peer CTA: forward "B written" to the leader, one cluster-scope
            // release per step
            const uint32_t bready_leader = cluster_map(&bready[0], 0);
            for (int i = 0; i < nk; ++i) {
                const int s = i % kFqStages;
                if (!mbar_wait(&bdone[s], static_cast<uint32_t>(i / kFqStages) & 1u, abort, p.limit_ns)) break;
                mbar_arrive_remote(bready_leader + static_cast<uint32_t>(s) * 8u);
            }
        }
    } else {
        // ---------------- quantizers, then epilogue: warps 2..9 of both CTAs
        const int qt = threadIdx.x - 64;             // 0..511
        const int qw = qt >> 5;
        const int n = (qw & 3) * 32 + lane;          // row of this CTA's B half
        const int part = qw >> 2;                    // which 16 columns of the 64-column step
        const int h = part >> 1;                     // which 32-column W box / group of the step
        const uint32_t c0 = static_cast<uint32_t>(part & 1) * 4u;   // first 16-byte chunk in the W box
        const int row = r0 + n;                      // row of W
        const uint32_t sw7 = static_cast<uint32_t>(n & 7);
        const uint32_t w_off = static_cast<uint32_t>(h) * kFqWBoxBytes + static_cast<uint32_t>(n) * 128u;
        const uint32_t b_off = kFqMTiles * kFqABytes + static_cast<uint32_t>(n) * 128u;
        const float* drow = p.delta + static_cast<int64_t>(row < p.R ? row : 0) * p.G;
        // scales two steps ahead
        float d0 = (row < p.R && h < p.G) ? __ldg(drow + h) : 0.0f;
        float d1 = (nk > 1 && row < p.R && 2 + h < p.G) ? __ldg(drow + 2 + h) : 0.0f;
        bool ok = true;
        for (int i = 0; i < nk; ++i) {
            const int s = i % kFqStages, sw = i % kFqWStages;
            const uint32_t ph = static_cast<uint32_t>(i / kFqStages) & 1u;
            const uint32_t phw = static_cast<uint32_t>(i / kFqWStages) & 1u;
            const float d = d0;
            d0 = d1;
            {
                const int g = 2 * (i + 2) + h;
                d1 = (i + 2 < nk && row < p.R && g < p.G) ? __ldg(drow + g) : 0.0f;
            }
            // W of this step has landed, and the MMA that last read this B slot is done
            bool got = mbar_wait(&full_w[sw], phw, abort, p.limit_ns) &&
                       mbar_wait(&ab_empty[s], ph ^ 1u, abort, p.limit_ns);
            got = __all_sync(0xffffffffu, got);
            if (!got) { ok = false; break; }
            const uint32_t wrow = w_ring + sw * kFqWBytes + w_off;
            const uint32_t brow = ab_ring + s * kFqABStageBytes + b_off;
            // all four loads first (the shared accesses keep their source order)
            float4 wv[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) wv[c] = fq_lds128(wrow + (((c0 + c) ^ sw7) << 4));
            uint4 out[2];
            fq_half_group(wv, d, out);
            // columns 16 part + 8j .. +7 -> B chunk 2 part + j
#pragma unroll
            for (int j = 0; j < 2; ++j)
                fq_sts128(brow + (((2u * static_cast<uint32_t>(part) + j) ^ sw7) << 4), out[j]);
            // the tensor core reads B through the async proxy
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
            // the W values are consumed (B is computed from them), so the slot may be refilled: a
            // release issued while a shared load is still in flight does not keep the next bulk
            // copy from overwriting the slot under it
            if (lane == 0) {
                mbar_arrive(&w_empty[sw]);
                mbar_arrive(&bdone[s]);
            }
        }

        // ---------------- epilogue
        bool got = ok && mbar_wait(&tmem_full_bar, 0, abort, p.limit_ns);
        got = __all_sync(0xffffffffu, got);
        if (got) {
            tc_fence_after();
            const int q = warp & 3;                               // TMEM lanes 32q..32q+31
            const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
            // a 32 x 33 float transpose buffer per warp in the (now idle) rings
            const uint32_t tbuf = sbase + static_cast<uint32_t>(qw) * (32u * 33u * 4u);
#pragma unroll 1
            for (int mt = 0; mt < kFqMTiles; ++mt) {
                const int tok0 = (tm * kFqMTiles + mt) * kFqTile + static_cast<int>(rank) * kFqHalf + q * 32;
#pragma unroll 1
                for (int blk = 0; blk < 2; ++blk) {
                    const int col = part * 64 + blk * 32;         // column of the pair tile
                    uint32_t a[32];
                    tmem_ld_32x32b_x32(lane_base + mt * 256u + col, a);
                    tmem_ld_wait();
#pragma unroll
                    for (int jj = 0; jj < 32; ++jj) fq_sts32(tbuf + (lane * 33u + jj) * 4u, __uint_as_float(a[jj]));
                    __syncwarp();
                    // lane -> column, loop over the 32 rows: 128 contiguous bytes per store
                    const int rcol = tr * kFqTile + col + lane;
#pragma unroll 4
                    for (int rr = 0; rr < 32; ++rr) {
                        const int tok = tok0 + rr;
                        const float v = fq_lds32(tbuf + (rr * 33u + lane) * 4u);
                        if (tok < p.T && rcol < p.R) p.Y[static_cast<int64_t>(tok) * p.R + rcol] = v;
                    }
                    __syncwarp();
                }
            }
        }
    }

    tc_fence_before();
    cluster_sync_all();      // no CTA leaves while its peer may still signal its barriers
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, kFqTmemCols);
    }
}

}  // namespace qat4
