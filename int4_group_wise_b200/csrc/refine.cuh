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
//                       128-row tile of E), into the caller's workspace;
//   refine_sweep_kernel one warp per row, the CTA's rows walking the groups in
//                       lockstep: u_g from v and the group's block of H (staged
//                       once per CTA); every candidate's
//                       e' H_gg e'^T + 2 e'.u_g in binary64 (lanes take
//                       candidates k = lane, lane + 32, ...; H_gg folded into
//                       its upper triangle in shared memory); the warp's
//                       argmin; for the rows whose group moved,
//                       v += H[:, g] (e'_g - e_g), with each of the group's 32
//                       rows of H read once for the whole CTA.
// The codes are exact: w * (1/Delta) is rounded unless it lands within 2^-18
// of a half-integer (or 1/Delta is not finite), then the IEEE quotient is used.
#pragma once

#include "device_common.cuh"

namespace qat4 {

constexpr int kRfTileR = 128;        // refine_v_kernel output tile: rows
constexpr int kRfTileC = 64;         //                              columns
constexpr int kRfK = 16;             // its reduction chunk
constexpr int kRfWarps = 8;          // rows (warps) per sweep CTA, walking the groups in lockstep
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

// V[r, :] = E[r, :] H (H symmetric), binary64: one accumulator per output, k ascending.  A
// 256-thread CTA computes a 128 x 64 tile, each thread 8 rows x 4 columns; 16-deep chunks of E
// (stored transposed, rows padded to 130 doubles so that the transposing stores spread over the
// banks and every thread's 8 rows are two aligned 16-byte pairs) and of H (converted to binary64
// once) go through shared memory, the next chunk's global loads held in registers meanwhile.
__global__ void __launch_bounds__(256, 2)
refine_v_kernel(const double* __restrict__ E, int R, int C, const float* __restrict__ H, int64_t ldh,
                double* __restrict__ V) {
    constexpr int kEPad = kRfTileR + 2;
    __shared__ __align__(16) double se[kRfK][kEPad];
    __shared__ __align__(16) double sh[kRfK][kRfTileC];
    const int tid = threadIdx.x;
    const int tx = tid & 15, ty = tid >> 4;
    const int r0 = blockIdx.y * kRfTileR, c0 = blockIdx.x * kRfTileC;
    double acc[8][4];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = 0.0;
    // this thread's share of a chunk: E elements x = tid + 256 i (row x / 16, k x % 16: a row's 16
    // values are 128 contiguous bytes), H elements y = tid + 256 i (k y / 64, column y % 64)
    double pe[8];
    float ph[4];
    auto load = [&](int k0) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int x = tid + 256 * i, r = r0 + (x >> 4);
            pe[i] = r < R ? E[static_cast<int64_t>(r) * C + k0 + (x & 15)] : 0.0;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int y = tid + 256 * i, c = c0 + (y & 63);
            ph[i] = c < C ? H[static_cast<int64_t>(k0 + (y >> 6)) * ldh + c] : 0.0f;
        }
    };
    auto stash = [&]() {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int x = tid + 256 * i;
            se[x & 15][x >> 4] = pe[i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int y = tid + 256 * i;
            sh[y >> 6][y & 63] = static_cast<double>(ph[i]);
        }
    };
    load(0);
    stash();
    __syncthreads();
    for (int k0 = 0; k0 < C; k0 += kRfK) {
        const bool more = k0 + kRfK < C;
        if (more) load(k0 + kRfK);
#pragma unroll
        for (int kk = 0; kk < kRfK; ++kk) {
            double ea[8], hb[4];
            const double2* e2 = reinterpret_cast<const double2*>(&se[kk][ty * 8]);
            const double2* h2 = reinterpret_cast<const double2*>(&sh[kk][tx * 4]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const double2 t = e2[q];
                ea[2 * q] = t.x;
                ea[2 * q + 1] = t.y;
            }
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const double2 t = h2[q];
                hb[2 * q] = t.x;
                hb[2 * q + 1] = t.y;
            }
#pragma unroll
            for (int a = 0; a < 8; ++a)
#pragma unroll
                for (int b = 0; b < 4; ++b) acc[a][b] = fma(ea[a], hb[b], acc[a][b]);
        }
        __syncthreads();
        if (more) {
            stash();
            __syncthreads();
        }
    }
#pragma unroll
    for (int a = 0; a < 8; ++a) {
        const int r = r0 + ty * 8 + a;
        const int c = c0 + tx * 4;
        if (r >= R || c >= C) continue;                  // C % 32 == 0: a thread's 4 columns are all in or all out
        double2* dst = reinterpret_cast<double2*>(V + static_cast<int64_t>(r) * C + c);
        dst[0] = make_double2(acc[a][0], acc[a][1]);
        dst[1] = make_double2(acc[a][2], acc[a][3]);
    }
}

struct RefineRowSmem {
    double u[32];            // u_g = v_g - H_gg e_g
    double delta[32];        // e'_g - e_g of a move
    float w[32];             // the group's weights
};

// Row i of a folded 32x32 block starts at i*32 - i*(i-1)/2 and holds columns i..31.
__host__ __device__ constexpr int refine_tri(int i) { return i * 32 - i * (i - 1) / 2; }

// The rows of a CTA (one warp each) walk the groups in lockstep, so that each group's block of H
// is staged once per CTA and each group's 32 rows of H are read once per CTA for all of the
// CTA's rows that move: (1) the CTA stages H_gg, full (binary32) and folded (binary64); (2) every
// warp takes its row's decision; (3) the CTA adds H[c0.., :]^T (e'_g - e_g) into v of every row
// that moved.  Each row's arithmetic is the same sequence as one warp alone would run.
__global__ void __launch_bounds__(32 * kRfWarps)
refine_sweep_kernel(const float* __restrict__ W, int R, int C, const float* __restrict__ H, int64_t ldh,
                    const float* __restrict__ alpha, int K, int sweeps, int32_t* __restrict__ idx,
                    float* __restrict__ delta_out, double* __restrict__ obj_out, double* __restrict__ V) {
    __shared__ double hp[kRfPacked];         // H_gg folded: H_ii, then 2 H_ij for j > i, row by row
    __shared__ float hf[32][33];             // H_gg as it is (row i: column j)
    __shared__ RefineRowSmem rs[kRfWarps];
    __shared__ unsigned moved;               // bit m: row m of the CTA moved at this group
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int r0 = blockIdx.x * kRfWarps;
    const int r = r0 + warp;
    const bool live = r < R;                 // every thread takes part in the CTA barriers
    RefineRowSmem& s = rs[warp];
    const int G = C >> 5;
    const float* wrow = W + static_cast<int64_t>(live ? r : 0) * C;
    double* v = V + static_cast<int64_t>(live ? r : 0) * C;
    int32_t* irow = idx + static_cast<int64_t>(live ? r : 0) * G;

    for (int sw = 0; sw < sweeps; ++sw) {
        for (int g = 0; g < G; ++g) {
            const int c0 = g * 32;
            // (1) H_gg into shared memory
            for (int x = tid; x < 32 * 32; x += 32 * kRfWarps) {
                const int i = x >> 5, j = x & 31;
                const float h = H[static_cast<int64_t>(c0 + i) * ldh + c0 + j];
                hf[i][j] = h;
                if (j >= i) hp[refine_tri(i) + j - i] = (j == i ? 1.0 : 2.0) * static_cast<double>(h);
            }
            if (tid == 0) moved = 0u;
            __syncthreads();
            // (2) this warp's row
            if (live) {
                const float wi = wrow[c0 + lane];
                const float base = refine_base(wi);
                s.w[lane] = wi;
                const int cur = min(max(irow[g], 0), K - 1);
                const float dcur = __ldg(alpha + cur) * base;
                const float qcur = code_of(scaled_exact(wi, dcur));
                const double ecur = static_cast<double>(wi) - static_cast<double>(dcur * qcur);
                // u_i = v_i - sum_j H_ij e_j (e_j from lane j)
                double hu = 0.0;
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    hu = fma(static_cast<double>(hf[lane][j]), __shfl_sync(0xffffffffu, ecur, j), hu);
                s.u[lane] = v[c0 + lane] - hu;
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
                        for (int j = i; j < 32; ++j) row = fma(hp[refine_tri(i) + j - i], e[j], row);
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
                    if (lane == 0) {
                        irow[g] = best_k;
                        atomicOr(&moved, 1u << warp);
                    }
                }
            }
            __syncthreads();
            // (3) v_j += sum_i H[c0 + i][j] delta_i (H symmetric) for every row that moved; threads
            // along j, so each of the group's 32 rows of H is read once for the whole CTA
            const unsigned mm = moved;
            if (mm != 0u) {
                for (int j = tid; j < C; j += 32 * kRfWarps) {
                    float hc[32];
#pragma unroll
                    for (int i = 0; i < 32; ++i) hc[i] = __ldg(H + static_cast<int64_t>(c0 + i) * ldh + j);
                    for (unsigned left = mm; left != 0u; left &= left - 1u) {
                        const int m = __ffs(left) - 1;
                        double a = 0.0;
#pragma unroll
                        for (int i = 0; i < 32; ++i) a = fma(static_cast<double>(hc[i]), rs[m].delta[i], a);
                        V[static_cast<int64_t>(r0 + m) * C + j] += a;
                    }
                }
            }
            __syncthreads();
        }
    }
    if (!live) return;
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
