// w4a16_gemv.cuh -- the inference product on the W4A16 export (model card
// "Opt.Gear-1B-qat-int4-per-channel-unquantized", section "Quantization
// Configuration": INT4 weights with 16-bit activations; "QAT Highlights": the
// learned grid survives export).  For a decode batch of MT <= 8 tokens:
//     y[m, r] = sum_c x[m, c] * (scale[r, c / group] * code[r, c])
// with x in bf16, the codes and binary16 scales of the packed export (element
// 2j in the low nibble of byte j), products exact and float32 sums.  The
// kernel reads the 0.5 B of codes and 2/group B of scale of every weight once:
// it is HBM-bound, so its inner products go to the tensor cores only to take
// the multiply-adds off the issue slots that the decoding needs.
//
// Tensor cores.  mma.sync m16n8k16 (bf16 x bf16 -> f32): A = 16 rows of W by
// 16 columns of codes (exact small integers in bf16), B = 16 columns of x by 8
// tokens (tokens past MT are zero), D in registers.  Two MMAs cover one
// 32-column group; their D is scaled by the group's scale into a float32
// accumulator.  The 16 columns of one MMA are a permutation of the group's
// columns, the same for A and B: lane (g, t) takes word t of the group (its 8
// nibbles, columns 8t..8t+7) for rows g and g+8, and the MMA's column pairs
// (2t, 2t+1) and (2t+8, 2t+9) are nibbles (0, 4) and (1, 5) in the first MMA,
// (2, 6) and (3, 7) in the second.  x is staged with every 8-column word in
// the order (0, 4, 1, 5, 2, 6, 3, 7), so one 16-byte load gives a lane both
// MMAs' B registers.
//
// Decoding.  One three-input logic op turns the nibbles at bits 0..3 and
// 16..19 of a word (shifted right by 0, 4, 8 or 12) into two bf16 values
// 128 + (code + 8) -- the nibble with its top bit flipped, under the exponent
// of 128 -- and one packed bf16 subtraction of 136 leaves the two codes,
// exactly.
//
// Data movement.  A persistent grid walks the list of stages (block of 16 rows)
// x (chunk of 2048 columns), cut into equal contiguous ranges of at least one
// row block, one per CTA.  A producer warp streams each stage's codes as eight
// 16-row x 128-byte boxes (2-D bulk-tensor copies, 128-byte swizzle, no
// multicast) into a ring of shared-memory slots; eight consumer warps take 8
// groups each, so a lane reads its 4-byte words of 8 rows from 8 different
// bank groups.  At the end of a row block the warps' partial tiles are summed
// in shared memory in a fixed order.  A row block cut between two CTAs gets one
// partial sum from each, added atomically into y (zeroed by the host): with at
// most two contributions, fl(0 + a + b) does not depend on their order.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include "device_common.cuh"

namespace qat4 {

constexpr int kGmWarps = 8;                                 // consumer warps
constexpr int kGmThreads = 32 * (kGmWarps + 1);             // + one producer warp
constexpr int kGmRows = 16;                                 // rows per block (one MMA tile)
constexpr int kGmChunkCols = 2048;                          // columns per stage
constexpr int kGmBoxBytes = kGmRows * 128;                  // 16 rows x 256 columns of codes
constexpr int kGmStageBytes = 8 * kGmBoxBytes;              // 16 KB
constexpr int kGmMaxStages = 12;
constexpr int kGmQuads = kGmChunkCols / 32 / kGmWarps;      // groups per warp and stage (8)
constexpr int kGmMaxTokens = 8;
constexpr uint64_t kGmDrainLimitNs = 1000000000ull;

struct GemvParams {
    const uint16_t* x;       // bf16 bits [MT, C], row stride C
    const uint16_t* scales;  // binary16 bits [R, C / group]
    float* y;                // [MT, R], zeroed by the host
    int R, C, group, G;      // G = C / group
    int MT;                  // tokens of this pass, 1..8
    int nblocks, nchunks;    // blocks of 16 rows, chunks of 2048 columns
    int stages;              // ring slots
    int xstride;             // bytes per staged token row
    uint64_t limit_ns;
    // mask and exponent-and-flip pattern of the decode, filled by the host so that they stay
    // register operands of one three-input logic op
    uint32_t dmask, dbits;
};

// Bytes per staged token row of x: the columns rounded up to whole chunks, 8 bf16 per 16 bytes,
// plus 64 bytes so that consecutive tokens start in different bank groups.
__host__ __device__ constexpr int gemv_xstride(int C) {
    return ((C + kGmChunkCols - 1) / kGmChunkCols) * kGmChunkCols * 2 + 64;
}

// Shared-memory bytes of the kernel for MT tokens, C columns and `stages` ring slots.
__host__ __device__ constexpr size_t gemv_smem_bytes(int MT, int C, int stages) {
    return 1024 + static_cast<size_t>(stages) * kGmStageBytes + static_cast<size_t>(MT) * gemv_xstride(C) +
           static_cast<size_t>(kGmWarps) * 32 * 4 * 4 + static_cast<size_t>(2 * kGmMaxStages) * 8 + 16;
}

// (a & m) ^ c as one three-input logic op.
__device__ __forceinline__ uint32_t gm_and_xor(uint32_t a, uint32_t m, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(m), "r"(c));
    return d;
}

// Codes of the nibbles at bits 0..3 and 16..19 of v, as a bf16 pair (low half first).
__device__ __forceinline__ uint32_t gm_pair(uint32_t v, uint32_t m, uint32_t c) {
    __nv_bfloat162 h;
    *reinterpret_cast<uint32_t*>(&h) = gm_and_xor(v, m, c);                 // 128 + (code + 8)
    const __nv_bfloat162 r = __hsub2(h, __floats2bfloat162_rn(136.0f, 136.0f));
    return *reinterpret_cast<const uint32_t*>(&r);
}

__device__ __forceinline__ void gm_mma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t gm_lds32(uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(a));
    return v;
}
__device__ __forceinline__ uint4 gm_lds128(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
    return v;
}

// Scales of rows (g, g+8) of block b for the kGmQuads groups of warp `warp` in chunk ch, in the
// order (row g, row g+8) per group; 0 past the matrix.  The group-32 export reads the 8 scales of
// a row with one 16-byte load (no division), the per-row export one scale per row.
struct GmScaleCtx {
    const uint16_t* scales;
    int R, C, G, group, warp, g;
    bool fast32;             // group 32 and G % 8 == 0
};
__device__ __forceinline__ float gm_half(uint32_t v, int hi) {
    return __half2float(__ushort_as_half(static_cast<unsigned short>(hi ? v >> 16 : v & 0xFFFFu)));
}
__device__ __forceinline__ void gm_scales(const GmScaleCtx& x, int b, int ch, float (&s)[2 * kGmQuads]) {
    const int ra = b * kGmRows + x.g, rb = ra + 8;
    const int q0 = ch * (kGmChunkCols / 32) + kGmQuads * x.warp;   // this warp's first group of 32 columns
    if (x.fast32 && q0 + kGmQuads <= x.G) {
        uint4 va = make_uint4(0u, 0u, 0u, 0u), vb = make_uint4(0u, 0u, 0u, 0u);
        if (ra < x.R) va = __ldg(reinterpret_cast<const uint4*>(x.scales + static_cast<int64_t>(ra) * x.G + q0));
        if (rb < x.R) vb = __ldg(reinterpret_cast<const uint4*>(x.scales + static_cast<int64_t>(rb) * x.G + q0));
        const uint32_t a4[4] = {va.x, va.y, va.z, va.w}, b4[4] = {vb.x, vb.y, vb.z, vb.w};
#pragma unroll
        for (int j = 0; j < kGmQuads; ++j) {
            s[2 * j] = gm_half(a4[j >> 1], j & 1);
            s[2 * j + 1] = gm_half(b4[j >> 1], j & 1);
        }
        return;
    }
    if (x.G == 1) {
        const float sa = ra < x.R ? __half2float(__ushort_as_half(__ldg(x.scales + ra))) : 0.0f;
        const float sb = rb < x.R ? __half2float(__ushort_as_half(__ldg(x.scales + rb))) : 0.0f;
#pragma unroll
        for (int j = 0; j < kGmQuads; ++j) { s[2 * j] = sa; s[2 * j + 1] = sb; }
        return;
    }
#pragma unroll
    for (int j = 0; j < kGmQuads; ++j) {
        const int c = (q0 + j) * 32;
        const bool in = c < x.C;
        const int gi = in ? c / x.group : 0;
        s[2 * j] = (in && ra < x.R)
                       ? __half2float(__ushort_as_half(__ldg(x.scales + static_cast<int64_t>(ra) * x.G + gi))) : 0.0f;
        s[2 * j + 1] = (in && rb < x.R)
                           ? __half2float(__ushort_as_half(__ldg(x.scales + static_cast<int64_t>(rb) * x.G + gi))) : 0.0f;
    }
}

// Programmatic dependent launch (pdl_launch_dependents / pdl_wait in
// device_common.cuh).  Calls of the product on one stream are launched so that
// the next kernel may start while this one finishes: the next call's CTAs
// become resident as this one's retire and start streaming their (constant)
// codes, and wait for this kernel's completion only before they read x or
// touch y.

// Zeroes y (the row blocks cut between two CTAs get two atomic partials), in
// order: it may start early, but writes y only after the previous kernel of
// the stream -- which may still be reading or adding into the same buffer --
// has completed.
__global__ void __launch_bounds__(256)
gemv_zero_kernel(float* __restrict__ y, int64_t n) {
    pdl_launch_dependents();
    pdl_wait();
    const int64_t n4 = n >> 2;
    float4* y4 = reinterpret_cast<float4*>(y);
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        y4[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
    for (int64_t i = (n4 << 2) + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x)
        y[i] = 0.0f;
}

__global__ void __launch_bounds__(kGmThreads)
w4a16_gemv_kernel(const __grid_constant__ CUtensorMap tmap, const GemvParams p) {
    pdl_launch_dependents();
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;          // the swizzle needs 1 KB alignment
    uint8_t* smem = smem_raw + pad;
    const uint32_t ring = raw + pad;
    const uint32_t xs = ring + p.stages * kGmStageBytes;
    float* red = reinterpret_cast<float*>(smem + p.stages * kGmStageBytes + p.MT * p.xstride);
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(red + kGmWarps * 32 * 4);
    uint64_t* empty_bar = full_bar + kGmMaxStages;
    int* abort_flag = reinterpret_cast<int*>(empty_bar + kGmMaxStages);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nchunks = p.nchunks, stages = p.stages;
    // this CTA's contiguous range of stages, at least one row block long
    const int64_t total = static_cast<int64_t>(p.nblocks) * nchunks;
    const int t0 = static_cast<int>(total * blockIdx.x / gridDim.x);
    const int t1 = static_cast<int>(total * (blockIdx.x + 1) / gridDim.x);
    const int b0 = t0 / nchunks, ch0 = t0 - b0 * nchunks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kGmWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    volatile int* abort = abort_flag;

    if (warp == kGmWarps) {
        // ---------------------------------------------------------- producer
        // lane 0 streams the codes; lanes 0..15 also pull into L2 the scales of the stage's rows
        if (lane == 0) prefetch_tmap(&tmap);
        int issued = 0, s = 0, b = b0, ch = ch0;
        uint32_t ph = 0;
        for (int t = t0; t < t1; ++t) {
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&empty_bar[s], ph ^ 1u, abort, p.limit_ns) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            const int r = b * kGmRows + lane;
            if (lane < kGmRows && r < p.R) {
                const int g0 = ch * kGmChunkCols / p.group;
                const int g1 = min(p.G, (ch * kGmChunkCols + kGmChunkCols - 1) / p.group + 1);
                const uint16_t* a = p.scales + static_cast<int64_t>(r) * p.G;
                asm volatile("prefetch.global.L2 [%0];" :: "l"(a + g0));
                asm volatile("prefetch.global.L2 [%0];" :: "l"(a + g1 - 1));
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&full_bar[s], kGmStageBytes);
                uint8_t* dst = smem + s * kGmStageBytes;
#pragma unroll
                for (int bx = 0; bx < 8; ++bx)   // x = (8 ch + bx) * 32 words: a multiple of 128 bytes
                    tma_load_2d(dst + bx * kGmBoxBytes, &tmap, &full_bar[s], (8 * ch + bx) * 32, b * kGmRows);
            }
            issued = t - t0 + 1;
            if (++s == stages) { s = 0; ph ^= 1u; }
            if (++ch == nchunks) { ch = 0; ++b; }
        }
        // no copy may still be landing when the CTA exits
        if (lane == 0)
            for (int i = (issued > stages ? issued - stages : 0); i < issued; ++i)
                mbar_wait(&full_bar[i % stages], static_cast<uint32_t>(i / stages) & 1u, nullptr, kGmDrainLimitNs);
        return;
    }

    // -------------------------------------------------------------- consumers
    // x (and y) belong to the stream's order: wait for the kernel before this one
    pdl_wait();
    // stage x once: token m's word w (columns 8w..8w+7) in the order 0,4,1,5,2,6,3,7; columns
    // past C are zero
    {
        const int words = (p.xstride - 64) / 16;
        for (int u = threadIdx.x; u < p.MT * words; u += 32 * kGmWarps) {
            const int m = u / words, w = u - m * words;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (w * 8 < p.C) v = __ldg(reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(m) * p.C + w * 8));
            const uint4 o = make_uint4(__byte_perm(v.x, v.z, 0x5410), __byte_perm(v.x, v.z, 0x7632),
                                       __byte_perm(v.y, v.w, 0x5410), __byte_perm(v.y, v.w, 0x7632));
            *reinterpret_cast<uint4*>(smem + (xs - ring) + m * p.xstride + w * 16) = o;
        }
        asm volatile("bar.sync 1, %0;" :: "n"(32 * kGmWarps) : "memory");
    }

    const int g = lane >> 2, t = lane & 3;
    const uint32_t dm = p.dmask, dc = p.dbits;
    GmScaleCtx sc;
    sc.scales = p.scales;
    sc.R = p.R;
    sc.C = p.C;
    sc.G = p.G;
    sc.group = p.group;
    sc.warp = warp;
    sc.g = g;
    sc.fast32 = p.group == 32 && (p.G & 7) == 0;
    const int R = p.R, MT = p.MT;
    float* const y = p.y;
    const bool xtok = g < p.MT;
    const uint32_t xrow = xs + static_cast<uint32_t>(xtok ? g : 0) * p.xstride + 16u * t;
    // this lane's word in the codes of rows g and g+8 (the 128-byte swizzle puts chunk k of row r
    // at (k ^ (r & 7)) * 16; rows g and g+8 share r & 7)
    uint32_t aoff[kGmQuads];
#pragma unroll
    for (int j = 0; j < kGmQuads; ++j) {
        const int q = kGmQuads * warp + j, bx = q >> 3, qq = q & 7;
        aoff[j] = bx * kGmBoxBytes + g * 128 + ((qq ^ g) << 4) + 4 * t;
    }

    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    float s_cur[2 * kGmQuads], s_next[2 * kGmQuads];
    int s = 0, b = b0, ch = ch0;
    uint32_t ph = 0;
    bool dead = false;   // a bounded wait gave up: skip the work, keep every warp on the same barriers
    if (t0 < t1) gm_scales(sc, b, ch, s_next);
    for (int it = t0; it < t1; ++it) {
#pragma unroll
        for (int j = 0; j < 2 * kGmQuads; ++j) s_cur[j] = s_next[j];
        dead = dead || !mbar_wait(&full_bar[s], ph, abort, p.limit_ns);
        const bool live = !dead;
        const uint32_t sb = ring + s * kGmStageBytes;
        uint32_t wa[kGmQuads], wb[kGmQuads];
#pragma unroll
        for (int j = 0; j < kGmQuads; ++j) {
            wa[j] = live ? gm_lds32(sb + aoff[j]) : 0u;
            wb[j] = live ? gm_lds32(sb + aoff[j] + 8 * 128) : 0u;
        }
        const int bn = ch + 1 == nchunks ? b + 1 : b, chn = ch + 1 == nchunks ? 0 : ch + 1;
        if (it + 1 < t1) gm_scales(sc, bn, chn, s_next);
#pragma unroll
        for (int j = 0; live && j < kGmQuads; ++j) {
            const int q = ch * (kGmChunkCols / 32) + kGmQuads * warp + j;   // group of 32 in the row
            uint4 xv = make_uint4(0u, 0u, 0u, 0u);
            if (xtok) xv = gm_lds128(xrow + q * 64);
            float d[4] = {0.0f, 0.0f, 0.0f, 0.0f};
            gm_mma(d, gm_pair(wa[j], dm, dc), gm_pair(wb[j], dm, dc), gm_pair(wa[j] >> 4, dm, dc),
                   gm_pair(wb[j] >> 4, dm, dc), xv.x, xv.y);
            gm_mma(d, gm_pair(wa[j] >> 8, dm, dc), gm_pair(wb[j] >> 8, dm, dc), gm_pair(wa[j] >> 12, dm, dc),
                   gm_pair(wb[j] >> 12, dm, dc), xv.z, xv.w);
            acc[0] = fmaf(s_cur[2 * j], d[0], acc[0]);
            acc[1] = fmaf(s_cur[2 * j], d[1], acc[1]);
            acc[2] = fmaf(s_cur[2 * j + 1], d[2], acc[2]);
            acc[3] = fmaf(s_cur[2 * j + 1], d[3], acc[3]);
        }
        // the slot is released only once the codes loaded from it have been used: a release
        // issued while a shared load is still in flight does not keep the next bulk copy from
        // overwriting the slot under it
        __syncwarp();
        if (lane == 0 && live) mbar_arrive(&empty_bar[s]);

        if (ch == nchunks - 1 || it == t1 - 1) {
            // the eight warps' partial tiles, summed in warp order
#pragma unroll
            for (int c = 0; c < 4; ++c) red[(warp * 32 + lane) * 4 + c] = acc[c];
            asm volatile("bar.sync 1, %0;" :: "n"(32 * kGmWarps) : "memory");
            if (threadIdx.x < 128) {
                const int ol = threadIdx.x >> 2, oc = threadIdx.x & 3;      // output of lane ol, entry oc
                float v = 0.0f;
#pragma unroll
                for (int w = 0; w < kGmWarps; ++w) v += red[(w * 32 + ol) * 4 + oc];
                const int row = b * kGmRows + (ol >> 2) + (oc >= 2 ? 8 : 0);
                const int tok = 2 * (ol & 3) + (oc & 1);
                if (row < R && tok < MT && !*abort) atomicAdd(y + static_cast<int64_t>(tok) * R + row, v);
            }
            asm volatile("bar.sync 1, %0;" :: "n"(32 * kGmWarps) : "memory");
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[c] = 0.0f;
        }
        if (++s == stages) {
            s = 0;
            ph ^= 1u;
        }
        b = bn;
        ch = chn;
    }
}

}  // namespace qat4
