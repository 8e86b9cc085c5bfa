// lsq_pack.cuh -- HBM-streaming kernels: LSQ fake-quant forward, LSQ backward
// (straight-through weight gradient + learned step-size gradient), the fused
// forward+backward pass, and the W4A16 export.
//
// Layout: W, G, Q, grad_W are flat [R*C] arrays; since C % 32 == 0 the group
// of flat element e is e / 32 and the per-group arrays are flat [R*C/32].
//
// Mapping: a warp streams 128 consecutive elements per load; lane l owns the
// float4 at elements 4l..4l+3, so 8 lanes cover one group of 32 and the warp
// covers 4 groups.  Loads and stores are 128-bit and fully coalesced; the
// per-group step-gradient sum is a 3-level xor butterfly inside each 8-lane
// segment.
#pragma once

#include "device_common.cuh"

namespace qat4 {

struct Bf16x4 { uint32_t lo, hi; };

__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xFFFF0000u); }

template <typename GT>
__device__ __forceinline__ float4 load_g4(const GT* G, int64_t quad);

template <>
__device__ __forceinline__ float4 load_g4<float>(const float* G, int64_t quad) {
    return __ldcs(reinterpret_cast<const float4*>(G) + quad);
}
template <>
__device__ __forceinline__ float4 load_g4<uint16_t>(const uint16_t* G, int64_t quad) {
    const uint2 u = __ldcs(reinterpret_cast<const uint2*>(G) + quad);
    return make_float4(bf16lo(u.x), bf16hi(u.x), bf16lo(u.y), bf16hi(u.y));
}

// Per element: forward value, STE weight gradient and dQ/dDelta (LSQ).
struct LsqElem { float q, gw, dq; };

__device__ __forceinline__ LsqElem lsq_elem(float w, float d, float g) {
    const float v = scaled_exact(w, d);
    const float r = rintf(v);
    LsqElem o;
    o.q = __fmul_rn(d, fminf(fmaxf(r, kQmin), kQmax));
    const bool inside = (v >= kQmin) && (v <= kQmax);
    o.gw = inside ? g : 0.0f;
    o.dq = (v <= kQmin) ? kQmin : ((v >= kQmax) ? kQmax : __fsub_rn(r, v));
    return o;
}

// FWD: write Q.  BWD: write grad_W and grad_delta.  A 128-thread block takes
// 128 * U consecutive quads (thread t: quads base + u * 128 + t, so 8
// consecutive lanes hold one group for the butterfly), issues all of its loads,
// then computes and stores; no thread runs a second iteration.  Blocks are
// short-lived and plentiful: the block scheduler starts a new one as soon as
// one finishes, so every SM keeps its loads in flight from the first wave to
// the last (a grid-stride loop over a fixed grid measured 7% slower: its last
// round of iterations leaves warps idle).
constexpr int kLsqBlock = 128;
template <typename GT, bool FWD, bool BWD, int U>
__global__ void __launch_bounds__(kLsqBlock)
lsq_blocks_kernel(const float* __restrict__ W, const float* __restrict__ delta,
                  const GT* __restrict__ G, int64_t nquads, float grad_scale,
                  float* __restrict__ Q, float* __restrict__ grad_W, float* __restrict__ grad_delta) {
    const int lane = threadIdx.x & 31;
    const int64_t base = static_cast<int64_t>(blockIdx.x) * (kLsqBlock * U) + threadIdx.x;
    float4 w[U], g[U];
    float d[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t quad = base + u * kLsqBlock;
        if (quad < nquads) {
            w[u] = __ldcs(reinterpret_cast<const float4*>(W) + quad);
            d[u] = __ldg(delta + (quad >> 3));
            if (BWD) g[u] = load_g4<GT>(G, quad);
        } else {
            w[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            d[u] = 0.f;
            g[u] = w[u];
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t quad = base + u * kLsqBlock;
        const bool valid = quad < nquads;
        const LsqElem e0 = lsq_elem(w[u].x, d[u], BWD ? g[u].x : 0.f);
        const LsqElem e1 = lsq_elem(w[u].y, d[u], BWD ? g[u].y : 0.f);
        const LsqElem e2 = lsq_elem(w[u].z, d[u], BWD ? g[u].z : 0.f);
        const LsqElem e3 = lsq_elem(w[u].w, d[u], BWD ? g[u].w : 0.f);
        if (FWD && valid) __stcs(reinterpret_cast<float4*>(Q) + quad, make_float4(e0.q, e1.q, e2.q, e3.q));
        if (BWD) {
            if (valid) __stcs(reinterpret_cast<float4*>(grad_W) + quad, make_float4(e0.gw, e1.gw, e2.gw, e3.gw));
            float acc = g[u].x * e0.dq;
            acc = fmaf(g[u].y, e1.dq, acc);
            acc = fmaf(g[u].z, e2.dq, acc);
            acc = fmaf(g[u].w, e3.dq, acc);
            acc += __shfl_xor_sync(0xffffffffu, acc, 4);
            acc += __shfl_xor_sync(0xffffffffu, acc, 2);
            acc += __shfl_xor_sync(0xffffffffu, acc, 1);
            if (valid && (lane & 7) == 0) grad_delta[quad >> 3] = grad_scale * acc;
        }
    }
}

// Eight codes of one group as the low nibbles of 1.5*2^23 + q, packed into a
// 32-bit word (element 0 in the lowest nibble).
// q = clamp(rint(w / d), -8, 7) is formed from r = w * (1/d): with both
// roundings r lies within 3 ulp of the IEEE quotient, so clamping r to
// [-8, 7] and rounding it (x + 1.5*2^23, which rounds to an integer in the
// last place) gives the same integer unless r lands within 2^-18 of a
// half-integer; then -- or when 1/d is not finite -- the IEEE division is
// redone for the eight elements.  For -8 <= q <= 7 the bit pattern of
// 1.5*2^23 + q is 0x4B400000 + q, whose low nibble is q in 4-bit two's
// complement.  The arithmetic runs on packed FP32x2 pairs.
__device__ __forceinline__ uint32_t pack8(float4 a, float4 b, float d) {
    constexpr float kM = 12582912.0f;                       // 1.5 * 2^23
    constexpr float kWin = 0.5f - 3.814697265625e-06f;      // 0.5 - 2^-18
    const float rc = __frcp_rn(d);
    bool slow = !(fabsf(rc) <= 3.4028234663852886e38f);
    const float2 rc2 = make_float2(rc, rc);
    const float2 M2 = make_float2(kM, kM);
    const float2 negM2 = make_float2(-kM, -kM);
    const float2 neg1 = make_float2(-1.0f, -1.0f);
    const float2 w[4] = {make_float2(a.x, a.y), make_float2(a.z, a.w), make_float2(b.x, b.y), make_float2(b.z, b.w)};
    float2 t[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float2 r = __fmul2_rn(w[e], rc2);
        r.x = fminf(fmaxf(r.x, kQmin), kQmax);
        r.y = fminf(fmaxf(r.y, kQmin), kQmax);
        t[e] = __fadd2_rn(r, M2);
        const float2 f = __ffma2_rn(__fadd2_rn(t[e], negM2), neg1, r);   // r - q
        slow |= !(fabsf(f.x) <= kWin) || !(fabsf(f.y) <= kWin);
    }
    if (slow) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            t[e].x = __fadd_rn(code_of(scaled_exact(w[e].x, d)), kM);
            t[e].y = __fadd_rn(code_of(scaled_exact(w[e].y, d)), kM);
        }
    }
    uint32_t out = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        out |= (__float_as_uint(t[e].x) & 0xFu) << (8 * e);
        out |= (__float_as_uint(t[e].y) & 0xFu) << (8 * e + 4);
    }
    return out;
}

// W4A16 export as many short blocks: a 128-thread block converts 128 * U
// consecutive octets (thread t: octets base + u * 128 + t, u < U, so each warp
// load covers 1 KB contiguous), issuing all of its loads before converting any.
// Blocks are short-lived and plentiful; the block scheduler starts a new one as
// soon as one finishes, so the loads in flight per SM stay high from the first
// wave to the last and no thread runs a second iteration.
//
// ROW selects the per-channel export (one scale per row of `row_oct` octets):
// the row of an octet is found by a binary64 multiply with 1/row_oct and a
// one-step correction (exact for any octet index below 2^52), and the first
// octet of a row writes the row's scale.  Otherwise the scale index is the
// group, octet / 4.
constexpr int kPackBlock = 128;
template <int U, bool ROW>
__global__ void __launch_bounds__(kPackBlock)
pack_w4a16_blocks_kernel(const float* __restrict__ W, const float* __restrict__ delta, int64_t noct,
                         int64_t row_oct, double inv_row_oct,
                         uint32_t* __restrict__ packed32, uint16_t* __restrict__ scales) {
    const int64_t base = static_cast<int64_t>(blockIdx.x) * (kPackBlock * U) + threadIdx.x;
    float4 a[U], b[U];
    float d[U];
    int64_t si[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t o = base + u * kPackBlock;
        if (ROW) {
            int64_t r = __double2ll_rz(__ll2double_rn(o) * inv_row_oct);
            if (r * row_oct > o) --r;
            else if ((r + 1) * row_oct <= o) ++r;
            si[u] = r;
        } else {
            si[u] = o >> 2;
        }
        if (o < noct) {
            a[u] = __ldcs(reinterpret_cast<const float4*>(W) + 2 * o);
            b[u] = __ldcs(reinterpret_cast<const float4*>(W) + 2 * o + 1);
            d[u] = __ldg(delta + si[u]);
        }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int64_t o = base + u * kPackBlock;
        if (o < noct) {
            __stcs(packed32 + o, pack8(a[u], b[u], d[u]));
            const bool first = ROW ? (o == si[u] * row_oct) : ((o & 3) == 0);
            if (first) scales[si[u]] = __half_as_ushort(__float2half_rn(d[u]));
        }
    }
}

}  // namespace qat4
