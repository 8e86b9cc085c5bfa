// scale_search.cuh -- Hessian-weighted per-group scale search.
//
// Model card "Opt.Gear-1B-qat-int4-per-channel-unquantized", section
// "Quantization Configuration": the scale of every quantization group is
// initialised by minimising the layer-output reconstruction error
// ||W X - Q_Delta(W) X||^2.  Read block-diagonally, group (r, g) minimises
// E(Delta) = e H_gg e^T with e = w_g - Q_Delta(w_g) and H_gg the 32x32 diagonal
// block of H, over the candidates Delta_k = fl(alpha_k * fl(max|w_g| / 7)).
//
// The error vector is the exact difference e = w - Q_Delta(w) of the binary32
// weights and their binary32 quantized values.
//
// Mapping: one CTA = one column group g x 128 rows; thread t owns row
// r0 + t and keeps its 32 weights in registers.  H_gg is staged once per CTA
// in shared memory as the upper triangle of H'_{ij} = H_ij + H_ji (j > i),
// H'_ii = H_ii (528 floats, stored twice and read as broadcast float4), so
// that E = sum_i e_i * (sum_{j >= i} H'_ij e_j): 528 + 32 FMA per candidate.
// Each thread evaluates two candidates per pass with packed FP32x2
// instructions (one FFMA2 = one FMA of each candidate); the quantization
// steps are packed the same way.
//
// Exactness: the codes are exact (rint of the IEEE quotient w / Delta_k; the
// quotient is formed as w * (1/Delta_k) and the IEEE division is redone for
// the group whenever that product lands within 2^-18 of a rounding boundary,
// which a 3-ulp error analysis shows is the only place the two can differ).
// E is screened in float32 together with a rigorous bound
//     |E32 - E| <= 80 u kappa S^2,   S = sum_i |e_i| sqrt|H_ii|,  u = 2^-24,
// kappa = max(1, max_{i != j} |H_ij| / sqrt|H_ii H_jj|)  (= 1 for a PSD H)
// which covers the <= 33-term FMA sums (about 66u), the rounding of H' and of
// the float32 difference fl(w - Q) used by the screen (about 3u).  Every candidate
// whose interval [E32 - b, E32 + b] can still contain the minimum is
// re-scored in float64 (the top four lower bounds are kept; if four or more
// are undecided, all K candidates are re-scored), and the float64 minimum
// wins, smallest k on ties.
#pragma once

#include <cstddef>
#include <utility>

#include "device_common.cuh"

namespace qat4 {

constexpr int kSearchThreads = 128;
constexpr int kTri = 528;          // entries of the upper triangle of a 32x32 block
constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23: x + M - M = rint(x) for |x| < 2^22
constexpr float kTieWindow = 0.5f - 3.814697265625e-06f;  // 0.5 - 2^-18
constexpr float kBoundC = 80.0f * 5.9604644775390625e-08f;  // 80 * 2^-24

// Row / column of entry p of the row-major upper triangle (j >= i) of a 32x32 matrix.
__host__ __device__ constexpr int tri_row(int p) {
    int i = 0;
    while (p >= 32 - i) { p -= 32 - i; ++i; }
    return i;
}
__host__ __device__ constexpr int tri_col(int p) {
    int i = 0;
    while (p >= 32 - i) { p -= 32 - i; ++i; }
    return i + p;
}
static_assert(tri_row(527) == 31 && tri_col(527) == 31 && tri_col(31) == 31 && tri_row(32) == 1, "tri");

constexpr int kSlot = 36;          // floats per thread slot (144 B: float4-aligned, few bank conflicts)

struct SearchSmem {
    float4 h32[kTri / 2];   // H' upper triangle, float32, each entry twice: (h_p, h_p, h_p+1, h_p+1)
    double h64[kTri];       // same, float64 (H_ij + H_ji exact)
    float4 sqrt_diag[8];    // sqrt(|H_ii|), rounded up
    float hfull[32][33];    // staging copy of H_gg (padded)
    unsigned kappa_bits;    // kappa as float bits (non-negative: int order == float order)
    // per-thread copies of the 32 weights and of an error vector, used only by
    // the exact (IEEE division) path so that it stays out of the unrolled loop
    alignas(16) float wslot[kSearchThreads * kSlot];
    alignas(16) float eslot[kSearchThreads * kSlot];
};
// every float4 access below needs these offsets to be multiples of 16 bytes
static_assert(sizeof(float4) * (kTri / 2) == 2 * kTri * sizeof(float) && offsetof(SearchSmem, h32) % 16 == 0 && offsetof(SearchSmem, sqrt_diag) % 16 == 0 &&
              offsetof(SearchSmem, h64) % 8 == 0 && offsetof(SearchSmem, wslot) % 16 == 0 &&
              offsetof(SearchSmem, eslot) % 16 == 0 && (kSlot * 4) % 16 == 0, "SearchSmem alignment");

// Exact error vector of one candidate from the weights parked in shared
// memory: q = clamp(rint(w / dk), -8, 7) with the IEEE division, in a rolled
// loop (taken only near a rounding boundary or when 1/dk is not finite).
__device__ __noinline__ void group_error_exact(const float* wslot, float dk, float* eslot) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
        const float wi = wslot[i];
        const float q = code_of(scaled_exact(wi, dk));
        eslot[i] = __fsub_rn(wi, __fmul_rn(dk, q));
    }
}

// e_i = fl(w_i - fl(dk * q_i)), q_i = clamp(rint(fl(w_i / dk)), -8, 7).
// wslot / eslot: this thread's shared-memory slots (wslot holds w).
__device__ __forceinline__ void group_error(const float (&w)[32], float dk, float (&e)[32],
                                            const float* wslot, float* eslot) {
    const float rc = __frcp_rn(dk);
    bool slow = !(fabsf(rc) <= 3.4028234663852886e38f);   // dk == 0 or 1/dk overflows
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float r = fminf(fmaxf(__fmul_rn(w[i], rc), kQmin), kQmax);
        const float q = __fsub_rn(__fadd_rn(r, kMagic), kMagic);
        slow |= !(fabsf(__fsub_rn(r, q)) <= kTieWindow);
        e[i] = __fsub_rn(w[i], __fmul_rn(dk, q));
    }
    if (slow) {
        group_error_exact(wslot, dk, eslot);
        const float4* e4 = reinterpret_cast<const float4*>(eslot);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const float4 x = e4[v];
            e[4 * v] = x.x; e[4 * v + 1] = x.y; e[4 * v + 2] = x.z; e[4 * v + 3] = x.w;
        }
    }
}

// Two candidates at once: element j of the pair register holds (e0_j, e1_j);
// one packed FMA (FFMA2) advances both candidates' row sums.  Each row sum is
// split into NCH interleaved chains (j - i mod NCH) so consecutive FFMA2s do
// not wait on each other; the chains are added at the end of the row.  (The
// screening bound holds for any summation order of these <= 33-term sums.)
template <int NCH, int P>
__device__ __forceinline__ void tri_ffma2(float2 h, const float2 (&e)[32], float2 (&t)[NCH], float2& E) {
    constexpr int i = tri_row(P);
    constexpr int j = tri_col(P);
    constexpr int c = (j - i) % NCH;
    t[c] = __ffma2_rn(h, e[j], t[c]);
    if constexpr (j == 31) {
        float2 r = t[0];
#pragma unroll
        for (int x = 1; x < NCH; ++x) r = __fadd2_rn(r, t[x]);
        E = __ffma2_rn(e[i], r, E);
#pragma unroll
        for (int x = 0; x < NCH; ++x) t[x] = make_float2(0.0f, 0.0f);
    }
}

template <int NCH, int Q2>
__device__ __forceinline__ void tri_pair2(const float4* h32, const float2 (&e)[32], float2 (&t)[NCH], float2& E) {
    const float4 h = h32[Q2];                     // (h_p, h_p, h_p+1, h_p+1)
    tri_ffma2<NCH, 2 * Q2 + 0>(make_float2(h.x, h.y), e, t, E);
    tri_ffma2<NCH, 2 * Q2 + 1>(make_float2(h.z, h.w), e, t, E);
}

template <int NCH, int... Q2s>
__device__ __forceinline__ float2 quad_form_pair_impl(std::integer_sequence<int, Q2s...>, const float4* h32,
                                                      const float2 (&e)[32]) {
    float2 t[NCH];
#pragma unroll
    for (int x = 0; x < NCH; ++x) t[x] = make_float2(0.0f, 0.0f);
    float2 E = make_float2(0.0f, 0.0f);
    (tri_pair2<NCH, Q2s>(h32, e, t, E), ...);
    return E;
}

// float32 screening values of two candidates, E.x and E.y.
template <int NCH>
__device__ __forceinline__ float2 quad_form_pair(const float4* h32, const float2 (&e)[32]) {
    return quad_form_pair_impl<NCH>(std::make_integer_sequence<int, kTri / 2>{}, h32, e);
}

// Error vectors of two candidates (dk.x, dk.y) in packed form; every
// component goes through exactly the operations of group_error, so the
// values are bit-identical to it.
__device__ __forceinline__ void group_error_pair(const float2 (&w2)[32], float2 dk, float2 (&e)[32],
                                                 const float* wslot, float* eslot) {
    const float2 rc = make_float2(__frcp_rn(dk.x), __frcp_rn(dk.y));
    bool slow = !(fabsf(rc.x) <= 3.4028234663852886e38f) || !(fabsf(rc.y) <= 3.4028234663852886e38f);
    const float2 M = make_float2(kMagic, kMagic);
    const float2 negM = make_float2(-kMagic, -kMagic);
    const float2 neg1 = make_float2(-1.0f, -1.0f);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        float2 r = __fmul2_rn(w2[i], rc);
        r.x = fminf(fmaxf(r.x, kQmin), kQmax);
        r.y = fminf(fmaxf(r.y, kQmin), kQmax);
        const float2 q = __fadd2_rn(__fadd2_rn(r, M), negM);     // rint, exact for |r| <= 8
        const float2 f = __ffma2_rn(q, neg1, r);                  // r - q
        slow |= !(fabsf(f.x) <= kTieWindow) || !(fabsf(f.y) <= kTieWindow);
        e[i] = __ffma2_rn(__fmul2_rn(dk, q), neg1, w2[i]);       // w - fl(dk * q)
    }
    if (slow) {
        const float4* e4 = reinterpret_cast<const float4*>(eslot);
        group_error_exact(wslot, dk.x, eslot);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const float4 x = e4[v];
            e[4 * v].x = x.x; e[4 * v + 1].x = x.y; e[4 * v + 2].x = x.z; e[4 * v + 3].x = x.w;
        }
        group_error_exact(wslot, dk.y, eslot);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const float4 x = e4[v];
            e[4 * v].y = x.x; e[4 * v + 1].y = x.y; e[4 * v + 2].y = x.z; e[4 * v + 3].y = x.w;
        }
    }
}

// float64 value of one candidate (the re-score): codes with the IEEE
// division, Q = fl(dk * q), and the exact difference e = w - Q (exact in
// binary64), summed in binary64.
__device__ __forceinline__ double quad_form64(const double* h64, const float (&w)[32], float dk) {
    double ed[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float q = code_of(scaled_exact(w[i], dk));
        ed[i] = static_cast<double>(w[i]) - static_cast<double>(__fmul_rn(dk, q));
    }
    double E = 0.0;
    int p = 0;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        double t = 0.0;
#pragma unroll
        for (int j = i; j < 32; ++j) t = fma(h64[p++], ed[j], t);
        E = fma(ed[i], t, E);
    }
    return E;
}

struct TopK4 {
    float L[4];
    int k[4];
    __device__ __forceinline__ void init() {
#pragma unroll
        for (int a = 0; a < 4; ++a) { L[a] = __int_as_float(0x7f800000); k[a] = -1; }
    }
    // keeps the four smallest lower bounds, ascending
    __device__ __forceinline__ void insert(float l, int kk) {
        if (!(l < L[3])) return;
        if (l < L[2]) {
            L[3] = L[2]; k[3] = k[2];
            if (l < L[1]) {
                L[2] = L[1]; k[2] = k[1];
                if (l < L[0]) { L[1] = L[0]; k[1] = k[0]; L[0] = l; k[0] = kk; }
                else { L[1] = l; k[1] = kk; }
            } else { L[2] = l; k[2] = kk; }
        } else { L[3] = l; k[3] = kk; }
    }
};

template <int MINB, int NCH>
__global__ void __launch_bounds__(kSearchThreads, MINB)
scale_search_kernel(const float* __restrict__ W, int R, int C,
                    const float* __restrict__ H, int64_t ldh,
                    const float* __restrict__ alpha, int K,
                    float* __restrict__ delta_out, int* __restrict__ idx_out,
                    float* __restrict__ err_out) {
    extern __shared__ __align__(16) uint8_t search_smem_raw[];
    SearchSmem& sm = *reinterpret_cast<SearchSmem*>(search_smem_raw);
    const int g = blockIdx.y;
    const int G = C / kGroup;
    const int tid = threadIdx.x;

    // ---- stage H_gg and its derived tables
    const float* Hg = H + static_cast<int64_t>(g) * kGroup * ldh + static_cast<int64_t>(g) * kGroup;
    for (int x = tid; x < 32 * 32; x += kSearchThreads) {
        const int i = x >> 5, j = x & 31;
        sm.hfull[i][j] = Hg[static_cast<int64_t>(i) * ldh + j];
    }
    if (tid == 0) sm.kappa_bits = __float_as_uint(1.0f);
    __syncthreads();
    float* h32f = reinterpret_cast<float*>(sm.h32);
    float kap = 0.0f;
    for (int p = tid; p < kTri; p += kSearchThreads) {
        const int i = tri_row(p), j = tri_col(p);
        const float a = sm.hfull[i][j], b = sm.hfull[j][i];
        if (i == j) {
            h32f[2 * p] = a;
            h32f[2 * p + 1] = a;
            sm.h64[p] = static_cast<double>(a);
        } else {
            const float hp = __fadd_rn(a, b);
            h32f[2 * p] = hp;
            h32f[2 * p + 1] = hp;
            sm.h64[p] = static_cast<double>(a) + static_cast<double>(b);
            const double m = fmax(fabs(static_cast<double>(a)), fabs(static_cast<double>(b)));
            if (m != 0.0) {
                const double den = sqrt(fabs(static_cast<double>(sm.hfull[i][i])) *
                                        fabs(static_cast<double>(sm.hfull[j][j])));
                const double ratio = den > 0.0 ? m / den : 1e300;
                kap = fmaxf(kap, ratio > 3.0e38 ? __int_as_float(0x7f800000)
                                                : __double2float_ru(ratio));
            }
        }
    }
    if (tid < 32) reinterpret_cast<float*>(sm.sqrt_diag)[tid] = __fsqrt_ru(fabsf(sm.hfull[tid][tid]));
    atomicMax(&sm.kappa_bits, __float_as_uint(kap));
    __syncthreads();

    const int r = blockIdx.x * kSearchThreads + tid;
    if (r >= R) return;
    const float kappa = __uint_as_float(sm.kappa_bits);
    const float bound_c = kBoundC * kappa;

    float w[32];
    const float4* wp = reinterpret_cast<const float4*>(W + static_cast<int64_t>(r) * C + g * kGroup);
#pragma unroll
    for (int v = 0; v < 8; ++v) {
        const float4 x = __ldg(wp + v);
        w[4 * v] = x.x; w[4 * v + 1] = x.y; w[4 * v + 2] = x.z; w[4 * v + 3] = x.w;
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(w[i]));
    const int64_t out = static_cast<int64_t>(r) * G + g;
    if (m == 0.0f) {   // all-zero group: every candidate has zero error
        delta_out[out] = 0.0f;
        idx_out[out] = 0;
        if (err_out) err_out[out] = 0.0f;
        return;
    }
    const float base = __fdiv_rn(m, 7.0f);
    float* wslot = sm.wslot + tid * kSlot;
    float* eslot = sm.eslot + tid * kSlot;
    {
        float4* w4 = reinterpret_cast<float4*>(wslot);
#pragma unroll
        for (int v = 0; v < 8; ++v) w4[v] = make_float4(w[4 * v], w[4 * v + 1], w[4 * v + 2], w[4 * v + 3]);
    }

    TopK4 top;
    top.init();
    float upper = __int_as_float(0x7f800000);
    float2 w2[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) w2[i] = make_float2(w[i], w[i]);
    for (int k = 0; k < K; k += 2) {
        const int k1 = (k + 1 < K) ? k + 1 : k;
        const float2 dk = make_float2(__fmul_rn(__ldg(alpha + k), base), __fmul_rn(__ldg(alpha + k1), base));
        float2 e[32];
        group_error_pair(w2, dk, e, wslot, eslot);
        const float2 E = quad_form_pair<NCH>(sm.h32, e);
        float S0 = 0.0f, S1 = 0.0f;
#pragma unroll
        for (int v = 0; v < 8; ++v) {
            const float4 s4 = sm.sqrt_diag[v];
            S0 = fmaf(fabsf(e[4 * v + 0].x), s4.x, S0);
            S1 = fmaf(fabsf(e[4 * v + 0].y), s4.x, S1);
            S0 = fmaf(fabsf(e[4 * v + 1].x), s4.y, S0);
            S1 = fmaf(fabsf(e[4 * v + 1].y), s4.y, S1);
            S0 = fmaf(fabsf(e[4 * v + 2].x), s4.z, S0);
            S1 = fmaf(fabsf(e[4 * v + 2].y), s4.z, S1);
            S0 = fmaf(fabsf(e[4 * v + 3].x), s4.w, S0);
            S1 = fmaf(fabsf(e[4 * v + 3].y), s4.w, S1);
        }
        const float b0 = bound_c * S0 * S0;
        upper = fminf(upper, E.x + b0);
        top.insert(E.x - b0, k);
        if (k1 != k) {
            const float b1 = bound_c * S1 * S1;
            upper = fminf(upper, E.y + b1);
            top.insert(E.y - b1, k1);
        }
    }

    // ---- float64 re-score of every candidate the screening could not exclude
    int nfin = 0;
#pragma unroll
    for (int a = 0; a < 4; ++a) nfin += (top.k[a] >= 0 && top.L[a] <= upper) ? 1 : 0;
    const bool overflow = (nfin == 4 && K > 4) || nfin == 0;
    double best = 0.0;
    int best_k = -1;
    const int count = overflow ? K : nfin;
    for (int a = 0; a < count; ++a) {
        const int kk = overflow ? a : (a == 0 ? top.k[0] : a == 1 ? top.k[1] : a == 2 ? top.k[2] : top.k[3]);
        const double E = quad_form64(sm.h64, w, __fmul_rn(__ldg(alpha + kk), base));
        if (best_k < 0 || E < best || (E == best && kk < best_k)) { best = E; best_k = kk; }
    }
    delta_out[out] = __fmul_rn(__ldg(alpha + best_k), base);
    idx_out[out] = best_k;
    if (err_out) err_out[out] = static_cast<float>(best);
}

}  // namespace qat4
