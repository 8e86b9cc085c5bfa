// rowwise.cuh -- the per-channel variant: one scale per output row (model card
// "Opt.Gear-1B-qat-int4-per-channel-unquantized": the same symmetric INT4 grid
// with channel-wise scales).  LSQ forward / backward and the W4A16 export with
// the group widened to the whole row; the step gradient of a row sums all C
// weights and is normalised by the caller's grad_scale (1/sqrt(C * 7)).
//
// Mapping: one CTA of 256 threads per row.  The row streams through as float4
// with 128-bit coalesced accesses; the row's step-gradient sum is a
// warp-shuffle tree followed by a shared-memory sum over the 8 warps.  The
// per-channel export is the short-block pack of lsq_pack.cuh in its row mode.
#pragma once

#include "device_common.cuh"
#include "lsq_pack.cuh"

namespace qat4 {

constexpr int kRowThreads = 256;

template <typename GT, bool FWD, bool BWD>
__global__ void __launch_bounds__(kRowThreads)
lsq_rowwise_kernel(const float* __restrict__ W, const float* __restrict__ delta, const GT* __restrict__ G,
                   int C, float grad_scale, float* __restrict__ Q, float* __restrict__ grad_W,
                   float* __restrict__ grad_delta) {
    __shared__ float part[kRowThreads / 32];
    const int64_t r = blockIdx.x;
    const float d = __ldg(delta + r);
    const int nq = C >> 2;
    const int64_t q0 = r * nq;
    float acc = 0.0f;
    for (int i = threadIdx.x; i < nq; i += kRowThreads) {
        const int64_t quad = q0 + i;
        const float4 w = __ldcs(reinterpret_cast<const float4*>(W) + quad);
        float4 g = make_float4(0.f, 0.f, 0.f, 0.f);
        if (BWD) g = load_g4<GT>(G, quad);
        const LsqElem e0 = lsq_elem(w.x, d, g.x);
        const LsqElem e1 = lsq_elem(w.y, d, g.y);
        const LsqElem e2 = lsq_elem(w.z, d, g.z);
        const LsqElem e3 = lsq_elem(w.w, d, g.w);
        if (FWD) __stcs(reinterpret_cast<float4*>(Q) + quad, make_float4(e0.q, e1.q, e2.q, e3.q));
        if (BWD) {
            __stcs(reinterpret_cast<float4*>(grad_W) + quad, make_float4(e0.gw, e1.gw, e2.gw, e3.gw));
            acc = fmaf(g.x, e0.dq, acc);
            acc = fmaf(g.y, e1.dq, acc);
            acc = fmaf(g.z, e2.dq, acc);
            acc = fmaf(g.w, e3.dq, acc);
        }
    }
    if (BWD) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
        __syncthreads();
        if (threadIdx.x == 0) {
            float s = 0.0f;
#pragma unroll
            for (int w8 = 0; w8 < kRowThreads / 32; ++w8) s += part[w8];
            grad_delta[r] = grad_scale * s;
        }
    }
}

}  // namespace qat4
