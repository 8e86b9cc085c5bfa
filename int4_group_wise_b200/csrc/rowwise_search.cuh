// rowwise_search.cuh -- per-channel Hessian-weighted scale search (model card
// "Opt.Gear-1B-qat-int4-per-channel-unquantized": channel-wise scales chosen by
// the output-reconstruction objective Delta* = argmin ||W X - Q_Delta(W) X||_F^2
// of section "Quantization Configuration", one scale per row).
//
// For row w (length C) and candidate Delta_k = fl(alpha_k * fl(max|w| / 7)) the
// objective is E_k = e^T H e with e = w - Q, Q = fl(Delta_k q) the binary32
// quantized weights and q the codes.  Writing Q = Delta_k q + rho (rho the
// rounding residual of each product, exact through an FMA) and h = H w,
// t = H q:
//     E_k = w.h - 2 Q.h + Delta_k^2 q.t + 2 Delta_k rho.t + rho^T H rho,
// all in binary64.  The last term is below 1e-14 of w.h and is dropped; every
// other term is exact up to binary64 rounding.  Between consecutive candidates
// only a few codes change (about 30 of 2048 for a Gaussian row on the default
// grid), so t is updated incrementally: t += dq_i * H[i, :] for each changed
// code i -- C fused multiply-adds and one row of H per change instead of C^2
// per candidate.  The sweep visits the candidates in the caller's order; any
// order is correct, a sorted grid is fastest.
//
// Phase 0 (rowwise_base_kernel): base = fl(max|w| / 7) per row.
// H must be symmetric (every Hessian from qat4_hessian is bitwise symmetric):
// the cross terms use w^T H Q = Q^T H w.
// Phase 1 (rowwise_hq_kernel): h = H w and t_0 = H q_0 for a 64-row tile at a
//   time (binary64 accumulation of exact binary32 products, H read once per
//   tile), into the caller's workspace.
// Phase 2 (rowwise_sweep_kernel): one CTA per row walks the candidates; the
//   codes of its C weights are recomputed exactly (w * (1/Delta) with the IEEE
//   division near a rounding boundary), changed codes are gathered in shared
//   memory, and t, q.t, Q.h, rho.t are updated and reduced over the CTA.
//   The smallest k reaching the minimum wins.
#pragma once

#include "device_common.cuh"

namespace qat4 {

constexpr int kRsThreads = 256;       // threads of the sweep CTA
constexpr int kRsMaxC = 8192;         // per-row state limit (EPT <= 32)
constexpr int kHqTile = 64;           // rows x columns of a phase-1 tile
constexpr int kHqK = 16;              // reduction chunk of phase 1

// base = fl(max|w| / 7), one warp per row.
__global__ void __launch_bounds__(256)
rowwise_base_kernel(const float* __restrict__ W, int R, int C, float* __restrict__ base) {
    const int warp = (blockIdx.x * 256 + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= R) return;
    const float* w = W + static_cast<int64_t>(warp) * C;
    float m = 0.0f;
    for (int c = lane; c < C; c += 32) m = fmaxf(m, fabsf(w[c]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) base[warp] = __fdiv_rn(m, 7.0f);
}

// h = H w, t0 = H q0 (q0: codes at Delta_0 = fl(alpha_0 * base)), binary64.
// CTA: 64 rows x 64 columns of both outputs; 16 x 16 threads, 4 x 4 each.
__global__ void __launch_bounds__(256)
rowwise_hq_kernel(const float* __restrict__ W, int R, int C, const float* __restrict__ H, int64_t ldh,
                  const float* __restrict__ base, const float* __restrict__ alpha, double* __restrict__ hout,
                  double* __restrict__ t0out) {
    const float alpha0 = __ldg(alpha);
    __shared__ double sw[kHqTile][kHqK + 1];
    __shared__ double sq[kHqTile][kHqK + 1];
    __shared__ double sh[kHqK][kHqTile + 1];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int r0 = blockIdx.y * kHqTile, c0 = blockIdx.x * kHqTile;
    double acc_h[4][4], acc_t[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) { acc_h[a][b] = 0.0; acc_t[a][b] = 0.0; }
    for (int k0 = 0; k0 < C; k0 += kHqK) {
        for (int x = threadIdx.x; x < kHqTile * kHqK; x += 256) {
            const int rr = x / kHqK, kk = x % kHqK;
            const int r = r0 + rr, k = k0 + kk;
            float wv = 0.0f, qv = 0.0f;
            if (r < R && k < C) {
                wv = W[static_cast<int64_t>(r) * C + k];
                qv = code_of(scaled_exact(wv, __fmul_rn(alpha0, base[r])));
            }
            sw[rr][kk] = static_cast<double>(wv);
            sq[rr][kk] = static_cast<double>(qv);
        }
        for (int x = threadIdx.x; x < kHqK * kHqTile; x += 256) {
            const int kk = x / kHqTile, cc = x % kHqTile;
            const int k = k0 + kk, c = c0 + cc;
            // H is symmetric: (H w)_c = sum_k H[c][k] w_k = sum_k H[k][c] w_k
            sh[kk][cc] = (k < C && c < C) ? static_cast<double>(H[static_cast<int64_t>(k) * ldh + c]) : 0.0;
        }
        __syncthreads();
#pragma unroll 4
        for (int kk = 0; kk < kHqK; ++kk) {
            double wa[4], qa[4], hb[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) { wa[a] = sw[ty * 4 + a][kk]; qa[a] = sq[ty * 4 + a][kk]; }
#pragma unroll
            for (int b = 0; b < 4; ++b) hb[b] = sh[kk][tx * 4 + b];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) {
                    acc_h[a][b] = fma(wa[a], hb[b], acc_h[a][b]);
                    acc_t[a][b] = fma(qa[a], hb[b], acc_t[a][b]);
                }
        }
        __syncthreads();
    }
#pragma unroll
    for (int a = 0; a < 4; ++a) {
        const int r = r0 + ty * 4 + a;
        if (r >= R) continue;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
            const int c = c0 + tx * 4 + b;
            if (c < C) {
                hout[static_cast<int64_t>(r) * C + c] = acc_h[a][b];
                t0out[static_cast<int64_t>(r) * C + c] = acc_t[a][b];
            }
        }
    }
}

// Exact code of one element (see the file comment).
__device__ __forceinline__ float rowwise_code(float w, float dk, float rc) {
    constexpr float kM = 12582912.0f;                       // 1.5 * 2^23
    constexpr float kWin = 0.5f - 3.814697265625e-06f;      // 0.5 - 2^-18
    const float r = fminf(fmaxf(__fmul_rn(w, rc), kQmin), kQmax);
    const float q = __fsub_rn(__fadd_rn(r, kM), kM);
    if (!(fabsf(__fsub_rn(r, q)) <= kWin) || !(fabsf(rc) <= 3.4028234663852886e38f))
        return code_of(scaled_exact(w, dk));
    return q;
}

// Block-wide sum of three doubles; every thread gets the result.
__device__ __forceinline__ void block_sum3(double& a, double& b, double& c, double (*red)[3]) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        a += __shfl_xor_sync(0xffffffffu, a, o);
        b += __shfl_xor_sync(0xffffffffu, b, o);
        c += __shfl_xor_sync(0xffffffffu, c, o);
    }
    const int warp = threadIdx.x >> 5;
    if ((threadIdx.x & 31) == 0) { red[warp][0] = a; red[warp][1] = b; red[warp][2] = c; }
    __syncthreads();
    a = b = c = 0.0;
#pragma unroll
    for (int x = 0; x < kRsThreads / 32; ++x) { a += red[x][0]; b += red[x][1]; c += red[x][2]; }
}

template <int EPT>
__global__ void __launch_bounds__(kRsThreads, 1)
rowwise_sweep_kernel(const float* __restrict__ W, int C, const float* __restrict__ H, int64_t ldh,
                     const float* __restrict__ alpha, int K, const float* __restrict__ base,
                     const double* __restrict__ hin, const double* __restrict__ t0in,
                     float* __restrict__ delta_out, int* __restrict__ idx_out, float* __restrict__ err_out) {
    extern __shared__ __align__(16) uint8_t rs_smem[];
    double* sh = reinterpret_cast<double*>(rs_smem);                         // h, C doubles
    uint32_t* changes = reinterpret_cast<uint32_t*>(sh + C);                 // (index << 5) | (dq + 16)
    __shared__ double red[kRsThreads / 32][3];
    __shared__ int nchange;
    const int64_t r = blockIdx.x;
    const int tid = threadIdx.x;
    const float bs = base[r];
    const float* w_row = W + r * C;

    float w[EPT];
    float q[EPT];
    double t[EPT];
    double a_part = 0.0;
    const float d0 = __fmul_rn(__ldg(alpha), bs);
#pragma unroll
    for (int m = 0; m < EPT; ++m) {
        const int j = tid + kRsThreads * m;
        if (j < C) {
            w[m] = w_row[j];
            const double hj = hin[r * C + j];
            sh[j] = hj;
            t[m] = t0in[r * C + j];
            q[m] = code_of(scaled_exact(w[m], d0));     // the same codes phase 1 used
            a_part = fma(static_cast<double>(w[m]), hj, a_part);
        } else {
            w[m] = 0.0f; q[m] = 0.0f; t[m] = 0.0;
        }
    }
    if (tid == 0) nchange = 0;
    double dummy1 = 0.0, dummy2 = 0.0;
    block_sum3(a_part, dummy1, dummy2, red);       // a = w.h (includes a __syncthreads)
    const double a_total = a_part;
    __syncthreads();                               // red[] is reused below

    double best = 0.0;
    int best_k = -1;
    for (int k = 0; k < K; ++k) {
        const float dk = __fmul_rn(__ldg(alpha + k), bs);
        if (k > 0) {
            // codes that change at this candidate
            const float rc = __frcp_rn(dk);
#pragma unroll
            for (int m = 0; m < EPT; ++m) {
                const int j = tid + kRsThreads * m;
                if (j < C) {
                    const float qn = rowwise_code(w[m], dk, rc);
                    if (qn != q[m]) {
                        const int dq = static_cast<int>(qn - q[m]);
                        const int slot = atomicAdd(&nchange, 1);
                        changes[slot] = (static_cast<uint32_t>(j) << 5) | static_cast<uint32_t>(dq + 16);
                        q[m] = qn;
                    }
                }
            }
            __syncthreads();
            const int n = nchange;
            for (int x = 0; x < n; ++x) {
                const uint32_t e = changes[x];
                const int i = static_cast<int>(e >> 5);
                const double dq = static_cast<double>(static_cast<int>(e & 31u) - 16);
                const float* hrow = H + static_cast<int64_t>(i) * ldh;     // row i = column i
#pragma unroll
                for (int m = 0; m < EPT; ++m) {
                    const int j = tid + kRsThreads * m;
                    if (j < C) t[m] = fma(dq, static_cast<double>(__ldg(hrow + j)), t[m]);
                }
            }
            __syncthreads();
            if (tid == 0) nchange = 0;
        }
        // Q.h, q.t, rho.t for this candidate
        double qh = 0.0, qt = 0.0, rt = 0.0;
#pragma unroll
        for (int m = 0; m < EPT; ++m) {
            const int j = tid + kRsThreads * m;
            if (j < C) {
                const float Qj = __fmul_rn(dk, q[m]);
                const float rho = -__fmaf_rn(dk, q[m], -Qj);               // Q - dk*q, exact
                qh = fma(static_cast<double>(Qj), sh[j], qh);
                qt = fma(static_cast<double>(q[m]), t[m], qt);
                rt = fma(static_cast<double>(rho), t[m], rt);
            }
        }
        block_sum3(qh, qt, rt, red);
        const double D = static_cast<double>(dk);
        const double E = a_total - 2.0 * qh + D * D * qt + 2.0 * D * rt;
        if (best_k < 0 || E < best) { best = E; best_k = k; }
        __syncthreads();     // red[] is reused by the next reduction
    }
    if (tid == 0) {
        delta_out[r] = __fmul_rn(__ldg(alpha + best_k), bs);
        idx_out[r] = best_k;
        if (err_out) err_out[r] = static_cast<float>(best);
    }
}

}  // namespace qat4
