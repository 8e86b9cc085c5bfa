// w4a16_gemv.cuh -- the inference product on the W4A16 export (model card
// "Opt.Gear-1B-qat-int4-per-channel-unquantized", section "Quantization
// Configuration": INT4 weights with 16-bit activations; "QAT Highlights": the
// learned grid survives export).  For a decode batch of MT <= 4 tokens:
//     y[m, r] = sum_c x[m, c] * (scale[r, c / group] * code[r, c])
// with x in bf16, the codes and binary16 scales of the packed export (element
// 2j in the low nibble of byte j), and float32 accumulation.  The kernel reads
// the 0.5 B of codes and 2/group B of scale of every weight once: HBM-bound.
//
// Data movement.  A persistent grid (one CTA per SM) walks the list of
// "stages" (row block) x (column chunk of 1024 columns), cut into equal
// contiguous ranges, one per CTA.  A producer warp streams each stage's codes
// (512 B per row) into a ring of shared-memory slots with 2-D bulk-tensor
// copies (no multicast); sixteen consumer warps take RPW rows each (4, or 2
// above two tokens), so a row block is 64 or 32 rows.
// The CTA's x (all MT tokens, all C columns) is staged in shared memory once:
// converted to float32 when it fits (MT <= 2), else kept as bf16; the 16-byte
// slots of every 32-column quad are XOR-swizzled by the quad index, so that
// the 32 lanes of a warp (lane l on quad l of the chunk) read x without bank
// conflicts.  Each x load serves the warp's RPW rows.
//
// Decoding without int -> float conversions.  Nibble k of a 32-bit word,
// masked in place with its top bit flipped (code + 8) and placed into the bit
// pattern of 2^(23 - 4k), is the float 2^(23-4k) + code + 8 exactly (the
// mantissa unit at that exponent is 2^-4k); subtracting 2^(23-4k) + 8 leaves
// the code.  Mask, flip and exponent are one three-input logic op.  Nibbles 0..4 use the word itself, nibbles
// 5..7 the word shifted right by 16 (back at bits 4..15).  Products x * code
// are exact; they are summed with packed FP32x2 FMAs over the 32 weights of a
// quad, then scaled by the group's scale.
//
// Partial rows.  A row block cut between two CTAs gets one partial sum from
// each; both are added atomically into y, which the host zeroes first.  The
// ranges are at least one row block long, so no row has more than two
// contributions, and fl(0 + a + b) does not depend on their order: the result
// is deterministic.
#pragma once

#include <cuda.h>

#include "device_common.cuh"

namespace qat4 {

constexpr int kGvConsumerWarps = 16;
constexpr int kGvThreads = 32 * (kGvConsumerWarps + 1);            // + one producer warp
constexpr int kGvChunkCols = 1024;                                  // columns per stage
constexpr int kGvRowBytes = kGvChunkCols / 2;                       // 512 B of codes per row and stage
constexpr int kGvMaxStages = 12;
constexpr uint64_t kGvDrainLimitNs = 1000000000ull;

// Rows per consumer warp (the reuse of each x load) for MT tokens: 4, or 2 when MT > 2 so that
// the accumulators of 16 warps fit the register file.
__host__ __device__ constexpr int gemv_rows_per_warp(int MT) { return MT <= 2 ? 4 : 2; }
__host__ __device__ constexpr int gemv_row_block(int MT) { return kGvConsumerWarps * gemv_rows_per_warp(MT); }
__host__ __device__ constexpr int gemv_stage_bytes(int MT) { return gemv_row_block(MT) * kGvRowBytes; }


struct GemvParams {
    const uint16_t* x;       // bf16 bits [MT, C], row stride C
    const uint16_t* scales;  // binary16 bits [R, C / group]
    float* y;                // [MT, R], zeroed by the host
    int R, C, group, G;      // G = C / group
    int nblocks, nchunks;    // row blocks of gemv_row_block(MT) rows, column chunks of 1024
    int stages;              // ring slots
    uint64_t limit_ns;
    // nibble masks and exponent-and-flip patterns of the decode, filled by the host so that
    // they stay register operands of one three-input logic op each
    uint32_t dmask[5], dbits[5];
};

// Bytes of x in shared memory per column: float32 (converted once while staging) or bf16.
__host__ __device__ constexpr int gemv_x_bytes(bool xf32) { return xf32 ? 4 : 2; }

// Shared-memory bytes of the kernel for MT tokens, C columns and `stages` ring slots.
__host__ __device__ constexpr size_t gemv_smem_bytes(int MT, bool xf32, int C, int stages) {
    return static_cast<size_t>(stages) * gemv_stage_bytes(MT) + static_cast<size_t>(MT) * C * gemv_x_bytes(xf32) +
           static_cast<size_t>(2 * kGvMaxStages) * 8 + 128;
}

// Byte offset, in one token's row of x, of 16-byte slot j of the 32-column quad q: 8 slots of
// 4 floats (float32 x) or 4 slots of 8 bf16, XOR-swizzled by the quad index so that 32 lanes
// on 32 consecutive quads hit distinct banks.
__host__ __device__ constexpr uint32_t gv_xslot_f32(uint32_t q, uint32_t j) { return q * 128u + 16u * (j ^ (q & 7u)); }
__host__ __device__ constexpr uint32_t gv_xslot_bf16(uint32_t q, uint32_t j) {
    return q * 64u + 16u * (j ^ ((q >> 1) & 3u));
}

// (a & m) ^ c as one three-input logic op.
__device__ __forceinline__ uint32_t gv_and_xor(uint32_t a, uint32_t m, uint32_t c) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0x6A;" : "=r"(d) : "r"(a), "r"(m), "r"(c));
    return d;
}

// The 8 codes of one word as 4 float pairs (nibbles 0,1 | 2,3 | 4,5 | 6,7).  Nibbles 0..4 are
// taken from the word, nibbles 5..7 from the word shifted right by 16 (back at bits 4..15).
struct GvDec { uint32_t m[5], c[5]; };
__device__ __forceinline__ void gv_decode(uint32_t w, const GvDec& d, float2 (&v)[4]) {
    const uint32_t hi = w >> 16;
    const float2 f01 = make_float2(__uint_as_float(gv_and_xor(w, d.m[0], d.c[0])),
                                   __uint_as_float(gv_and_xor(w, d.m[1], d.c[1])));
    const float2 f23 = make_float2(__uint_as_float(gv_and_xor(w, d.m[2], d.c[2])),
                                   __uint_as_float(gv_and_xor(w, d.m[3], d.c[3])));
    const float2 f45 = make_float2(__uint_as_float(gv_and_xor(w, d.m[4], d.c[4])),
                                   __uint_as_float(gv_and_xor(hi, d.m[1], d.c[1])));
    const float2 f67 = make_float2(__uint_as_float(gv_and_xor(hi, d.m[2], d.c[2])),
                                   __uint_as_float(gv_and_xor(hi, d.m[3], d.c[3])));
    // 2^23 + 8, 2^19 + 8, 2^15 + 8, 2^11 + 8, 2^7 + 8
    v[0] = __fadd2_rn(f01, make_float2(-8388616.0f, -524296.0f));
    v[1] = __fadd2_rn(f23, make_float2(-32776.0f, -2056.0f));
    v[2] = __fadd2_rn(f45, make_float2(-136.0f, -524296.0f));
    v[3] = __fadd2_rn(f67, make_float2(-32776.0f, -2056.0f));
}

// Scales of the warp's RPW rows for the quad of `lane` in stage (b, ch); 0 past the matrix.
template <int RPW>
__device__ __forceinline__ void gv_scales(const uint16_t* __restrict__ scales, int R, int G, int C, int group,
                                          int b, int ch, int row0, int lane, float (&s)[RPW]) {
    const int q = ch * (kGvChunkCols / 32) + lane;
    const bool in = q < (C >> 5);
    const int g = group == 32 ? q : (q * 32) / group;
#pragma unroll
    for (int i = 0; i < RPW; ++i) {
        const int r = b * kGvConsumerWarps * RPW + row0 + i;
        s[i] = (r < R && in) ? __half2float(__ushort_as_half(__ldg(scales + static_cast<int64_t>(r) * G + g)))
                             : 0.0f;
    }
}

template <int MT, bool XF32>
__global__ void __launch_bounds__(kGvThreads, 1)
w4a16_gemv_kernel(const __grid_constant__ CUtensorMap tmap, const GemvParams p) {
    constexpr int RPW = gemv_rows_per_warp(MT);
    constexpr int RB = gemv_row_block(MT);
    constexpr int SB = gemv_stage_bytes(MT);
    constexpr int XB = gemv_x_bytes(XF32);
    extern __shared__ __align__(128) uint8_t smem[];
    const int R = p.R, C = p.C, G = p.G, group = p.group, nchunks = p.nchunks, stages = p.stages;
    uint8_t* ring = smem;
    uint8_t* xs = smem + static_cast<size_t>(stages) * SB;
    uint64_t* full_bar = reinterpret_cast<uint64_t*>(xs + static_cast<size_t>(MT) * C * XB);
    uint64_t* empty_bar = full_bar + kGvMaxStages;
    int* abort_flag = reinterpret_cast<int*>(empty_bar + kGvMaxStages);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // this CTA's contiguous range of stages, at least one row block long
    const int64_t total = static_cast<int64_t>(p.nblocks) * nchunks;
    const int t0 = static_cast<int>(total * blockIdx.x / gridDim.x);
    const int t1 = static_cast<int>(total * (blockIdx.x + 1) / gridDim.x);
    const int b0 = t0 / nchunks, ch0 = t0 - b0 * nchunks;

    if (threadIdx.x == 0) {
        for (int s = 0; s < stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kGvConsumerWarps);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    volatile int* abort = abort_flag;

    if (warp == kGvConsumerWarps) {
        // ---------------------------------------------------------- producer
        // lane 0 streams the codes; the lanes also pull into L2 the scales of the stage's rows,
        // a ring's length before the consumers read them
        if (lane == 0) prefetch_tmap(&tmap);
        int issued = 0, s = 0, b = b0, ch = ch0;
        uint32_t ph = 0;
        for (int t = t0; t < t1; ++t) {
            int ok = 1;
            if (lane == 0) ok = mbar_wait(&empty_bar[s], ph ^ 1u, abort, p.limit_ns) ? 1 : 0;
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            const int g0 = ch * kGvChunkCols / group;
            const int g1 = min(G, (ch * kGvChunkCols + kGvChunkCols - 1) / group + 1);
#pragma unroll
            for (int k = 0; k < RB / 32; ++k) {
                const int r = b * RB + 32 * k + lane;
                if (r < R) {
                    const uint16_t* a = p.scales + static_cast<int64_t>(r) * G;
                    asm volatile("prefetch.global.L2 [%0];" :: "l"(a + g0));
                    asm volatile("prefetch.global.L2 [%0];" :: "l"(a + g1 - 1));
                }
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&full_bar[s], SB);
                // x = ch * 128 words: a multiple of 512 bytes
                tma_load_2d(ring + static_cast<size_t>(s) * SB, &tmap, &full_bar[s], ch * (kGvRowBytes / 4), b * RB);
            }
            issued = t - t0 + 1;
            if (++s == stages) { s = 0; ph ^= 1u; }
            if (++ch == nchunks) { ch = 0; ++b; }
        }
        // no copy may still be landing when the CTA exits
        if (lane == 0)
            for (int i = (issued > stages ? issued - stages : 0); i < issued; ++i)
                mbar_wait(&full_bar[i % stages], static_cast<uint32_t>(i / stages) & 1u, nullptr, kGvDrainLimitNs);
        return;
    }

    // -------------------------------------------------------------- consumers
    // stage x once, token-major, into swizzled 16-byte slots
    if (XF32) {
        const int per_tok = C >> 2;                  // 4 columns per unit
        for (int u = threadIdx.x; u < MT * per_tok; u += 32 * kGvConsumerWarps) {
            const int m = u / per_tok, c = (u - m * per_tok) << 2;
            const uint2 v = __ldg(reinterpret_cast<const uint2*>(p.x + static_cast<int64_t>(m) * C + c));
            const float4 f = make_float4(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xFFFF0000u),
                                         __uint_as_float(v.y << 16), __uint_as_float(v.y & 0xFFFF0000u));
            *reinterpret_cast<float4*>(xs + static_cast<size_t>(m) * C * 4 + gv_xslot_f32(c >> 5, (c >> 2) & 7)) = f;
        }
    } else {
        const int per_tok = C >> 3;                  // 8 columns per unit
        for (int u = threadIdx.x; u < MT * per_tok; u += 32 * kGvConsumerWarps) {
            const int m = u / per_tok, c = (u - m * per_tok) << 3;
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(m) * C + c));
            *reinterpret_cast<uint4*>(xs + static_cast<size_t>(m) * C * 2 + gv_xslot_bf16(c >> 5, (c >> 3) & 3)) = v;
        }
    }
    asm volatile("bar.sync 1, %0;" :: "n"(32 * kGvConsumerWarps) : "memory");

    GvDec dec;
#pragma unroll
    for (int k = 0; k < 5; ++k) {
        dec.m[k] = p.dmask[k];
        dec.c[k] = p.dbits[k];
    }
    const int nquads = C >> 5;
    const int row0 = warp * RPW;                     // first row of this warp in a block
    const size_t xrow = static_cast<size_t>(C) * XB;
    // x slots of this lane's quad, relative to the chunk's first quad (a multiple of 32)
    constexpr int NSLOT = XF32 ? 8 : 4;
    uint32_t xoff[NSLOT];
#pragma unroll
    for (int j = 0; j < NSLOT; ++j) xoff[j] = XF32 ? gv_xslot_f32(lane, j) : gv_xslot_bf16(lane, j);
    const uint8_t* st_lane = ring + static_cast<size_t>(row0) * kGvRowBytes + 16 * lane;

    float acc[RPW][MT];
    float s_cur[RPW], s_next[RPW];
    int s = 0, b = b0, ch = ch0;
    uint32_t ph = 0;
    if (t0 < t1) gv_scales<RPW>(p.scales, R, G, C, group, b, ch, row0, lane, s_next);
    for (int t = t0; t < t1; ++t) {
        if (ch == 0 || t == t0) {
#pragma unroll
            for (int r = 0; r < RPW; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[r][m] = 0.0f;
        }
#pragma unroll
        for (int r = 0; r < RPW; ++r) s_cur[r] = s_next[r];
        if (!mbar_wait(&full_bar[s], ph, abort, p.limit_ns)) break;
        const uint8_t* st = st_lane + static_cast<size_t>(s) * SB;
        uint4 wq[RPW];
#pragma unroll
        for (int r = 0; r < RPW; ++r) wq[r] = *reinterpret_cast<const uint4*>(st + r * kGvRowBytes);
        const int bn = ch + 1 == nchunks ? b + 1 : b, chn = ch + 1 == nchunks ? 0 : ch + 1;
        if (t + 1 < t1) gv_scales<RPW>(p.scales, R, G, C, group, bn, chn, row0, lane, s_next);

        if (ch * (kGvChunkCols / 32) + lane < nquads) {
            // the chunk's first quad is 32 * ch: swizzle bits of the lane's quad are the lane's
            const uint8_t* xq = xs + static_cast<size_t>(ch) * 32 * (32 * XB);
            float2 part[RPW][MT];
#pragma unroll
            for (int r = 0; r < RPW; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) part[r][m] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int wd = 0; wd < 4; ++wd) {
                float2 xv[MT][4];               // x of the word's 8 columns, as 4 pairs
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    if (XF32) {
                        const float4 a = *reinterpret_cast<const float4*>(xq + m * xrow + xoff[2 * wd]);
                        const float4 c = *reinterpret_cast<const float4*>(xq + m * xrow + xoff[(2 * wd + 1) % NSLOT]);
                        xv[m][0] = make_float2(a.x, a.y);
                        xv[m][1] = make_float2(a.z, a.w);
                        xv[m][2] = make_float2(c.x, c.y);
                        xv[m][3] = make_float2(c.z, c.w);
                    } else {
                        const uint4 xr = *reinterpret_cast<const uint4*>(xq + m * xrow + xoff[wd % NSLOT]);
                        xv[m][0] = make_float2(__uint_as_float(xr.x << 16), __uint_as_float(xr.x & 0xFFFF0000u));
                        xv[m][1] = make_float2(__uint_as_float(xr.y << 16), __uint_as_float(xr.y & 0xFFFF0000u));
                        xv[m][2] = make_float2(__uint_as_float(xr.z << 16), __uint_as_float(xr.z & 0xFFFF0000u));
                        xv[m][3] = make_float2(__uint_as_float(xr.w << 16), __uint_as_float(xr.w & 0xFFFF0000u));
                    }
                }
#pragma unroll
                for (int r = 0; r < RPW; ++r) {
                    const uint32_t word = wd == 0 ? wq[r].x : wd == 1 ? wq[r].y : wd == 2 ? wq[r].z : wq[r].w;
                    float2 v[4];
                    gv_decode(word, dec, v);
#pragma unroll
                    for (int m = 0; m < MT; ++m) {
                        part[r][m] = __ffma2_rn(xv[m][0], v[0], part[r][m]);
                        part[r][m] = __ffma2_rn(xv[m][1], v[1], part[r][m]);
                        part[r][m] = __ffma2_rn(xv[m][2], v[2], part[r][m]);
                        part[r][m] = __ffma2_rn(xv[m][3], v[3], part[r][m]);
                    }
                }
            }
#pragma unroll
            for (int r = 0; r < RPW; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) acc[r][m] = fmaf(s_cur[r], part[r][m].x + part[r][m].y, acc[r][m]);
        }
        // the slot is released only once the codes loaded from it have been used: a release
        // issued while a shared load is still in flight does not keep the next bulk copy from
        // overwriting the slot under it
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[s]);

        if (ch == nchunks - 1 || t == t1 - 1) {
#pragma unroll
            for (int r = 0; r < RPW; ++r)
#pragma unroll
                for (int m = 0; m < MT; ++m) {
                    float v = acc[r][m];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                    acc[r][m] = v;
                }
            if (lane == 0) {
#pragma unroll
                for (int r = 0; r < RPW; ++r) {
                    const int row = b * RB + row0 + r;
                    if (row < R) {
#pragma unroll
                        for (int m = 0; m < MT; ++m) atomicAdd(p.y + static_cast<int64_t>(m) * R + row, acc[r][m]);
                    }
                }
            }
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
