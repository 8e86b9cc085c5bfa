// lsq_pack.cuh -- HBM-streaming kernels: LSQ fake-quant forward, LSQ backward
// (straight-through weight gradient + learned step-size gradient), the fused
// forward+backward pass, and the W4A16 export.
//
// Layout: W, G, Q, grad_W are flat [R*C] arrays; since C % 32 == 0 the group
// of flat element e is e / 32 and the per-group arrays are flat [R*C/32].
//
// Mapping: a warp streams 128 consecutive elements per step; lane l owns the
// float4 at elements 4l..4l+3, so 8 lanes cover one group of 32 and the warp
// covers 4 groups.  Loads and stores are 128-bit and fully coalesced; the
// per-group step-gradient sum is a 3-level xor butterfly inside each 8-lane
// segment.  Each warp processes kUnroll steps per loop iteration with all of
// their loads issued first, to keep enough bytes in flight for HBM3e.
#pragma once

#include "device_common.cuh"

namespace qat4 {

constexpr int kStreamThreads = 256;
constexpr int kUnroll = 2;

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

// FWD: write Q.  BWD: write grad_W and grad_delta.  U steps in flight per warp.
template <typename GT, bool FWD, bool BWD, int U = kUnroll>
__global__ void __launch_bounds__(kStreamThreads)
lsq_kernel(const float* __restrict__ W, const float* __restrict__ delta,
           const GT* __restrict__ G, int64_t nquads, float grad_scale,
           float* __restrict__ Q, float* __restrict__ grad_W, float* __restrict__ grad_delta) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kStreamThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kStreamThreads) >> 5;
    const int64_t nsteps = nquads >> 5;  // nquads is a multiple of 8; handle tail below
    const int64_t nsteps_ceil = (nquads + 31) >> 5;
    (void)nsteps;

    for (int64_t s0 = warp * U; s0 < nsteps_ceil; s0 += nwarps * U) {
        float4 w[U], g[U];
        float d[U];
        bool valid[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t quad = (s0 + u) * 32 + lane;
            valid[u] = quad < nquads;
            if (valid[u]) {
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
            const int64_t quad = (s0 + u) * 32 + lane;
            const LsqElem e0 = lsq_elem(w[u].x, d[u], BWD ? g[u].x : 0.f);
            const LsqElem e1 = lsq_elem(w[u].y, d[u], BWD ? g[u].y : 0.f);
            const LsqElem e2 = lsq_elem(w[u].z, d[u], BWD ? g[u].z : 0.f);
            const LsqElem e3 = lsq_elem(w[u].w, d[u], BWD ? g[u].w : 0.f);
            if (FWD && valid[u])
                __stcs(reinterpret_cast<float4*>(Q) + quad, make_float4(e0.q, e1.q, e2.q, e3.q));
            if (BWD) {
                if (valid[u])
                    __stcs(reinterpret_cast<float4*>(grad_W) + quad,
                           make_float4(e0.gw, e1.gw, e2.gw, e3.gw));
                float acc = g[u].x * e0.dq;
                acc = fmaf(g[u].y, e1.dq, acc);
                acc = fmaf(g[u].z, e2.dq, acc);
                acc = fmaf(g[u].w, e3.dq, acc);
                acc += __shfl_xor_sync(0xffffffffu, acc, 4);
                acc += __shfl_xor_sync(0xffffffffu, acc, 2);
                acc += __shfl_xor_sync(0xffffffffu, acc, 1);
                if (valid[u] && (lane & 7) == 0) grad_delta[quad >> 3] = grad_scale * acc;
            }
        }
    }
}

// Four codes of one group as the low nibbles of 1.5*2^23 + q.
// q = clamp(rint(w / d), -8, 7) is formed from r = w * (1/d): with both
// roundings r lies within 3 ulp of the IEEE quotient, so clamping r to
// [-8, 7] and rounding it (x + 1.5*2^23, which rounds to an integer in the
// last place) gives the same integer unless r lands within 2^-18 of a
// half-integer; then -- or when 1/d is not finite -- the IEEE division is
// redone for the four elements.  For -8 <= q <= 7 the bit pattern of
// 1.5*2^23 + q is 0x4B400000 + q, whose low nibble is q in 4-bit two's
// complement.
__device__ __forceinline__ uint32_t pack4(float4 w, float d) {
    constexpr float kM = 12582912.0f;                       // 1.5 * 2^23
    constexpr float kWin = 0.5f - 3.814697265625e-06f;      // 0.5 - 2^-18
    const float rc = __frcp_rn(d);
    bool slow = !(fabsf(rc) <= 3.4028234663852886e38f);
    float t[4];
    const float wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float r = fminf(fmaxf(__fmul_rn(wv[e], rc), kQmin), kQmax);
        t[e] = __fadd_rn(r, kM);
        slow |= !(fabsf(__fsub_rn(r, __fsub_rn(t[e], kM))) <= kWin);
    }
    if (slow) {
#pragma unroll
        for (int e = 0; e < 4; ++e) t[e] = __fadd_rn(code_of(scaled_exact(wv[e], d)), kM);
    }
    return (__float_as_uint(t[0]) & 0xFu) | ((__float_as_uint(t[1]) & 0xFu) << 4) |
           ((__float_as_uint(t[2]) & 0xFu) << 8) | ((__float_as_uint(t[3]) & 0xFu) << 12);
}

// W4A16 export.  Lane l converts the float4 at elements 4l..4l+3 of a
// 128-element step into two bytes (one coalesced 2-byte store); lanes 0, 8,
// 16, 24 also write their group's binary16 scale.
template <int U = 4>
__global__ void __launch_bounds__(kStreamThreads)
pack_w4a16_kernel(const float* __restrict__ W, const float* __restrict__ delta, int64_t nquads,
                  uint16_t* __restrict__ packed16, uint16_t* __restrict__ scales) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kStreamThreads + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kStreamThreads) >> 5;
    const int64_t nsteps_ceil = (nquads + 31) >> 5;
    for (int64_t s0 = warp * U; s0 < nsteps_ceil; s0 += nwarps * U) {
        float4 w[U];
        float d[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t quad = (s0 + u) * 32 + lane;
            if (quad < nquads) {
                w[u] = __ldcs(reinterpret_cast<const float4*>(W) + quad);
                d[u] = __ldg(delta + (quad >> 3));
            } else {
                w[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                d[u] = 0.f;
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t quad = (s0 + u) * 32 + lane;
            if (quad < nquads) {
                packed16[quad] = static_cast<uint16_t>(pack4(w[u], d[u]));
                if ((lane & 7) == 0) scales[quad >> 3] = __half_as_ushort(__float2half_rn(d[u]));
            }
        }
    }
}

}  // namespace qat4
