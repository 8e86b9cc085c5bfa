// refine.cuh -- full-objective refinement of the group scales (model card
// "Opt.Gear-1B-qat-int4-per-channel-unquantized", section "Quantization
// Configuration": the objective is written over the whole layer,
// Delta* = argmin ||W X - Q_Delta(W) X||_F^2, i.e. per row of W the quadratic
// form e H e^T of e = w - Q_Delta(w) over all C columns).  The scale search
// keeps only the diagonal 32x32 blocks of H; this refinement starts from its
// candidate indices and runs sweeps of coordinate descent: the groups of a row
// in order, each moved to the candidate of its own grid (Delta_k = alpha_k *
// fl(m/7)) that minimises the full objective with the other groups held; ties
// go to the smallest k.
//
// With v = H e (the whole row), changing group g from e_g to e'_g changes the
// objective by  e'_g H_gg e'_g^T + 2 e'_g . u_g  minus the same at e_g, where
// u_g = v_g - H_gg e_g^T (H symmetric).  So
//   refine_err_kernel   e = w - fl(Delta q) for the starting indices, binary64
//                       (exact: difference of two binary32 values);
//   refine_v_kernel     V = E H, a tiled binary64 product (H read once per
//                       64-row tile), into the caller's workspace;
//   refine_sweep_kernel one warp per row walks the groups: u_g from v and the
//                       group's block of H; every candidate's
//                       e' H_gg e'^T + 2 e'.u_g in binary64 (lanes take
//                       candidates k = lane, lane + 32, ...; H_gg folded into
//                       its upper triangle in shared memory); the warp's
//                       argmin; when the group moves, v += H[:, g] (e'_g - e_g).
// The codes are exact: w * (1/Delta) is rounded unless it lands within 2^-18
// of a half-integer (or 1/Delta is not finite), then the IEEE quotient is used.
#pragma once

#include "device_common.cuh"

namespace qat4 {

constexpr int kRfTile = 64;          // refine_v_kernel output tile (rows x columns)
constexpr int kRfK = 16;             // its reduction chunk
constexpr int kRfWarps = 8;          // rows (warps) per sweep CTA
constexpr int kRfPacked = 528;       // 32 * 33 / 2 entries of a folded 32x32 block

// Exact code of w at step dk with rc = 1/dk (see the file comment).
__device__ __forceinline__ float refine_code(float w, float dk, float rc, bool rc_ok) {
    constexpr float kWin = 0.5f - 3.814697265625e-06f;      // 0.5 - 2^-18
    const float r = fminf(fmaxf(w * rc, kQmin), kQmax);
    const float q = rintf(r);
    if (!rc_ok || !(fabsf(r - q) <= kWin)) return code_of(scaled_exact(w, dk));
    return q;
}

// base = fl(max|w| / 7) of the group held by the warp (lane i holds w_i).
__device__ __forceinline__ float refine_base(float w) {
    float m = fabsf(w);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    return __fdiv_rn(m, 7.0f);
}

// e = w - fl(Delta q) of the starting indices, binary64; one warp per group.
__global__ void __launch_bounds__(256)
refine_err_kernel(const float* __restrict__ W, int64_t ngroups, const float* __restrict__ alpha, int K,
                  const int32_t* __restrict__ idx, double* __restrict__ E) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
    for (int64_t u = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; u < ngroups; u += warps) {
        const float w = W[u * 32 + lane];
        const int k = min(max(idx[u], 0), K - 1);        // indices outside the grid are clamped
        const float dk = __ldg(alpha + k) * refine_base(w);
        const float q = code_of(scaled_exact(w, dk));
        E[u * 32 + lane] = static_cast<double>(w) - static_cast<double>(dk * q);
    }
}

// V[r, :] = E[r, :] H (H symmetric), binary64 accumulation of exact products; 64 x 64 tiles.
__global__ void __launch_bounds__(256)
refine_v_kernel(const double* __restrict__ E, int R, int C, const float* __restrict__ H, int64_t ldh,
                double* __restrict__ V) {
    __shared__ double se[kRfTile][kRfK + 1];
    __shared__ double sh[kRfK][kRfTile + 1];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int r0 = blockIdx.y * kRfTile, c0 = blockIdx.x * kRfTile;
    double acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
    for (int k0 = 0; k0 < C; k0 += kRfK) {
        for (int x = threadIdx.x; x < kRfTile * kRfK; x += 256) {
            const int rr = x / kRfK, kk = x % kRfK;
            const int r = r0 + rr, k = k0 + kk;
            se[rr][kk] = (r < R && k < C) ? E[static_cast<int64_t>(r) * C + k] : 0.0;
        }
        for (int x = threadIdx.x; x < kRfK * kRfTile; x += 256) {
            const int kk = x / kRfTile, cc = x % kRfTile;
            const int k = k0 + kk, c = c0 + cc;
            sh[kk][cc] = (k < C && c < C) ? static_cast<double>(H[static_cast<int64_t>(k) * ldh + c]) : 0.0;
        }
        __syncthreads();
#pragma unroll 4
        for (int kk = 0; kk < kRfK; ++kk) {
            double ea[4], hb[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) ea[a] = se[ty * 4 + a][kk];
#pragma unroll
            for (int b = 0; b < 4; ++b) hb[b] = sh[kk][tx * 4 + b];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = fma(ea[a], hb[b], acc[a][b]);
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
            if (c < C) V[static_cast<int64_t>(r) * C + c] = acc[a][b];
        }
    }
}

struct RefineWarpSmem {
    double hp[kRfPacked];    // H_gg folded: H_ii, then 2 H_ij for j > i, row by row
    double u[32];            // u_g = v_g - H_gg e_g
    double delta[32];        // e'_g - e_g of a move
    float w[32];             // the group's weights
};

// Row i of a folded 32x32 block starts at i*32 - i*(i-1)/2 and holds columns i..31.
__host__ __device__ constexpr int refine_tri(int i) { return i * 32 - i * (i - 1) / 2; }

__global__ void __launch_bounds__(32 * kRfWarps)
refine_sweep_kernel(const float* __restrict__ W, int R, int C, const float* __restrict__ H, int64_t ldh,
                    const float* __restrict__ alpha, int K, int sweeps, int32_t* __restrict__ idx,
                    float* __restrict__ delta_out, double* __restrict__ obj_out, double* __restrict__ V) {
    __shared__ RefineWarpSmem sm[kRfWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.x * kRfWarps + warp;
    if (r >= R) return;                          // no block-wide synchronisation below
    RefineWarpSmem& s = sm[warp];
    const int G = C >> 5;
    const float* wrow = W + static_cast<int64_t>(r) * C;
    double* v = V + static_cast<int64_t>(r) * C;
    int32_t* irow = idx + static_cast<int64_t>(r) * G;

    for (int sw = 0; sw < sweeps; ++sw) {
        for (int g = 0; g < G; ++g) {
            const int c0 = g * 32;
            const float wi = wrow[c0 + lane];
            const float base = refine_base(wi);
            s.w[lane] = wi;
            // lane i: row i of H_gg, folded into the upper triangle
            const float* hrow = H + static_cast<int64_t>(c0 + lane) * ldh + c0;
            float hr[32];
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 t = *reinterpret_cast<const float4*>(hrow + j);
                hr[j] = t.x; hr[j + 1] = t.y; hr[j + 2] = t.z; hr[j + 3] = t.w;
            }
            const int cur = min(max(irow[g], 0), K - 1);
            const float dcur = __ldg(alpha + cur) * base;
            const float qcur = code_of(scaled_exact(wi, dcur));
            const double ecur = static_cast<double>(wi) - static_cast<double>(dcur * qcur);
            // u_i = v_i - sum_j H_ij e_j (e_j from lane j)
            double hu = 0.0;
#pragma unroll
            for (int j = 0; j < 32; ++j) hu = fma(static_cast<double>(hr[j]), __shfl_sync(0xffffffffu, ecur, j), hu);
            s.u[lane] = v[c0 + lane] - hu;
            {
                const int t0 = refine_tri(lane);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (j >= lane) s.hp[t0 + j - lane] = (j == lane ? 1.0 : 2.0) * static_cast<double>(hr[j]);
            }
            __syncwarp();
            // candidates k = lane, lane + 32, ...: e' H_gg e'^T + 2 e'.u
            double best = 0.0;
            int best_k = -1;
            for (int k = lane; k < K; k += 32) {
                const float dk = __ldg(alpha + k) * base;
                const float rc = __frcp_rn(dk);
                const bool rc_ok = fabsf(rc) <= 3.4028234663852886e38f;
                double e[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const float wv = s.w[i];
                    e[i] = static_cast<double>(wv) - static_cast<double>(dk * refine_code(wv, dk, rc, rc_ok));
                }
                double Ek = 0.0;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    double row = 2.0 * s.u[i];
#pragma unroll
                    for (int j = i; j < 32; ++j) row = fma(s.hp[refine_tri(i) + j - i], e[j], row);
                    Ek = fma(e[i], row, Ek);
                }
                if (best_k < 0 || Ek < best) {
                    best = Ek;
                    best_k = k;
                }
            }
            // warp argmin, ties to the smallest k (lanes without a candidate carry +inf)
            if (best_k < 0) best = __longlong_as_double(0x7FF0000000000000ll);
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const double ob = __shfl_xor_sync(0xffffffffu, best, o);
                const int ok = __shfl_xor_sync(0xffffffffu, best_k, o);
                if (ob < best || (ob == best && ok >= 0 && (best_k < 0 || ok < best_k))) {
                    best = ob;
                    best_k = ok;
                }
            }
            if (best_k != cur) {
                const float dnew = __ldg(alpha + best_k) * base;
                const float qnew = code_of(scaled_exact(wi, dnew));
                s.delta[lane] = (static_cast<double>(wi) - static_cast<double>(dnew * qnew)) - ecur;
                __syncwarp();
                // v_j += sum_i H[c0 + i][j] delta_i (H symmetric), lanes along j
                for (int j = lane; j < C; j += 32) {
                    double a = 0.0;
#pragma unroll 8
                    for (int i = 0; i < 32; ++i)
                        a = fma(static_cast<double>(__ldg(H + static_cast<int64_t>(c0 + i) * ldh + j)), s.delta[i], a);
                    v[j] += a;
                }
                if (lane == 0) irow[g] = best_k;
            }
            __syncwarp();
        }
    }
    // outputs: Delta of every group and the final objective e . v
    double obj = 0.0;
    for (int g = 0; g < G; ++g) {
        const float wi = wrow[g * 32 + lane];
        const float base = refine_base(wi);
        const float dk = __ldg(alpha + min(max(irow[g], 0), K - 1)) * base;
        const float q = code_of(scaled_exact(wi, dk));
        obj = fma(static_cast<double>(wi) - static_cast<double>(dk * q), v[g * 32 + lane], obj);
        if (lane == 0) delta_out[static_cast<int64_t>(r) * G + g] = dk;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) obj += __shfl_xor_sync(0xffffffffu, obj, o);
    if (lane == 0 && obj_out != nullptr) obj_out[r] = obj;
}

}  // namespace qat4
