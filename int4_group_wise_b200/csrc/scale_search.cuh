// scale_search.cuh -- the Hessian-weighted per-group scale search with the
// quadratic forms on the 5th-generation tensor cores.
//
// Model card "Opt.Gear-1B-qat-int4-per-channel-unquantized", section
// "Quantization Configuration": the scale of every group minimises the
// layer-output error ||W X - Q_Delta(W) X||^2; read block-diagonally, group
// (r, g) minimises E_k = e H_gg e^T over the candidates
// Delta_k = fl(alpha_k * fl(max|w_g| / 7)), with e = w - fl(Delta_k q) the
// exact difference of the binary32 weights and their quantized values.
//
// Mapping: one CTA = one column group g x 128 rows (thread = row = TMEM lane =
// row of the MMA's M = 128 tile).  For every candidate k the 128 threads
// quantize their 32 weights (exact codes, see tc_quantize) and write
// the error vector e as binary16 e_hi into the A operand in shared memory; one
// thread issues tcgen05.mma.kind::f16 (M = 128, N = 32, K = 16):
//     P = e_hi * (H_hi + H_lo)        (float32 accumulate in TMEM)
// where H_hi + H_lo is the symmetrised block (H + H^T)/2, scaled by a power of
// two into binary16 range and split into two binary16 parts.  Each thread then
// reads its row of P back and forms E = P . v, v = e + e_lo = 2e - e_hi: since
// e = e_hi + e_lo exactly and H is symmetric,
//     e H e = e_hi H (e + e_lo) + e_lo H e_lo,
// so one binary16 A operand gives E to about 2^-22 relative (the dropped
// e_lo H e_lo term is <= 2^-22 of the form's scale).  Weights are scaled by
// a power of two per row (2^13 <= max|w| sigma < 2^14) so that e fits binary16
// without overflow; scaling by powers of two leaves the codes and the argmin
// unchanged.
//
// Equilibration: when the binary16 split of the block would lose too much
// (its split-error ratio kappa_d above 2^-17 -- channels whose scales differ
// by a few hundred put the small entries below binary16's normal range, and
// every candidate of such a block would then be re-scored), the block is
// first scaled to H' = D^-1 H D^-1 with d_i a power of two near sqrt|H_ii|,
// and the error vectors to e' = D e, so that e' H' e' = e H e exactly; the
// bound below is then taken for (H', e').
//
// Two-stage pipeline: while the tensor core multiplies candidate k, the
// threads quantize candidate k + 1.  Each thread parks its v of a candidate in
// TMEM next to that candidate's P (columns 64s..64s+31 hold P of stage s,
// 64s+32..64s+63 hold v), so the pipeline costs no registers and four CTAs
// fit on an SM; the two stages' A operands share each 128-byte row (bytes
// 64s..64s+63).  One CTA barrier per candidate hands the A stage to the
// tensor core; the issuing thread rotates over the four warps.
//
// The screened value carries a rigorous bound
//     |E_screen - E| <= c * Sa^2 + c_f * T * Sa,
//     Sa = (1 + 2^-9)(S + 2^-14 T),  S = sum_i |v_i| sd_i,  T = sum_i sd_i,
//     sd_i = sqrt|H_ii| (scaled, rounded up),
//     c = (kappa + kappa_d)(tau + 2^-19 + 2^-22) + kappa_d + kappa (2^-20 + 2^-23),
// with kappa = max(1, max_{i != j} |H_ij| / (sd_i sd_j)), kappa_d the same ratio
// for the error of the binary16 split of H (computed exactly per CTA), tau =
// 2^-17 covering 64 float32 accumulation steps of the tensor core at one unit
// in the last place each (products of binary16 values are exact in float32),
// and c_f = 2^-12 (kappa + kappa_d) covering a tensor core that would flush
// binary16 subnormal inputs (e_hi < 2^-14) to zero.  Candidates whose
// interval can still hold the minimum are re-scored in float64
// (tc_quad_form64), so the returned index is the float64 argmin.
#pragma once

#include <cuda_fp16.h>

#include "device_common.cuh"

namespace qat4 {

constexpr int kTri = 528;          // entries of the upper triangle of a 32x32 block

template <bool B>
struct BoolTag {
    static constexpr bool value = B;
};
constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23: x + M - M = rint(x) for |x| < 2^22
constexpr float kTieWindow = 0.5f - 3.814697265625e-06f;  // 0.5 - 2^-18

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

constexpr int kTcRows = 128;
constexpr int kTcSlot = 36;                      // floats per exact-path slot
// kind::f16 instruction descriptor: D float32, A and B binary16, both K-major, N = 32, M = 128.
constexpr uint32_t kTcIdesc = (1u << 4) | ((32u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kTcStageCols = 64;            // TMEM columns per stage: P (32) then v (32)
constexpr uint32_t kTcTmemCols = 2 * kTcStageCols;

struct SearchTcSmem {
    // A: row m holds thread m's e_hi (binary16) of stage 0 in bytes 0..63 and of
    // stage 1 in bytes 64..127 (K-major, 128-byte swizzle)
    uint8_t a[kTcRows * 128];
    uint8_t bhi[32 * 128];        // row n: column n of the scaled symmetrised block, hi part (k < 32)
    uint8_t blo[32 * 128];        //        the lo part
    double h64[kTri];             // H'_ij = H_ij + H_ji (j > i), H'_ii = H_ii, binary64, unscaled
    union {
        float hfull[32][33];                       // set-up: staging copy of H_gg
        float eslot[kTcRows * kTcSlot];            // main loop: exact-path error vectors
    } u;
    uint64_t mbar[2];
    uint32_t tmem_base;
    unsigned kappa_bits;          // kappa (non-negative float bits)
    unsigned kappa_d_bits;        // kappa_d
    unsigned hmax_bits;           // max |H_sym| (unscaled)
    int exact_block;              // the split cannot represent this block: re-score every candidate
    int abort;
    float coef, coef_f, tsum;
    alignas(16) float sd[32];     // sqrt(sigma_H |H'_ii|), rounded up
    float isd[32];                // reciprocals rounded up (set-up only)
    alignas(16) float dsc[32];    // equilibration d_i (powers of two; all 1 unless equilibrated)
    float idsc[32];               // 1 / d_i
    int eq;                       // the block is equilibrated: H' = D^-1 H D^-1, e' = D e
};
constexpr size_t kTcSmemBytes = sizeof(SearchTcSmem) + 1024;   // + alignment of the operand tiles
static_assert(offsetof(SearchTcSmem, a) == 0 && offsetof(SearchTcSmem, bhi) % 1024 == 0 &&
              offsetof(SearchTcSmem, blo) % 1024 == 0 && offsetof(SearchTcSmem, u) % 16 == 0 &&
              offsetof(SearchTcSmem, mbar) % 8 == 0 && offsetof(SearchTcSmem, sd) % 16 == 0,
              "SearchTcSmem layout");

// Byte offset of logical 16-byte chunk c of row n in a K-major 128-byte-swizzled tile.
__host__ __device__ constexpr uint32_t sw128_off(uint32_t n, uint32_t c) {
    return n * 128u + ((c ^ (n & 7u)) << 4);
}

// Round-up helper for the bound (non-negative inputs).
__device__ __forceinline__ float up(double x) { return __double2float_ru(x); }

// Exact error vector of one candidate, scaled: e_i = sigma * fl(w_i - fl(dk * q_i)),
// q_i = clamp(rint(fl(w_i / dk)), -8, 7) with the IEEE division; w read from global
// memory (rolled loop, taken only near a rounding boundary or when 1/dk is not finite).
__device__ __noinline__ void tc_error_exact(const float* __restrict__ wrow, float dk, float sigma, float* eslot) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i) {
        const float wi = wrow[i];
        const float q = code_of(scaled_exact(wi, dk));
        eslot[i] = __fmul_rn(__fsub_rn(wi, __fmul_rn(dk, q)), sigma);
    }
}

// Start of row i of the row-major upper triangle (j >= i) of a 32x32 matrix.
__host__ __device__ constexpr int tri_start(int i) { return 32 * i - (i * (i - 1)) / 2; }

// float64 value of one candidate (the re-score; out of line, so that its 32 binary64
// differences do not add to the candidate loop's registers): the exact codes (w * (1/dk),
// with the IEEE division redone for the group near a rounding boundary or when
// 1/dk is not finite, as in the screen), Q = fl(dk * q), the exact difference
// e = w - Q (exact in binary64), and e H' e summed in binary64 over the upper
// triangle H' (H'_ij = H_ij + H_ji, H'_ii = H_ii).  Four rows at a time, each
// row's sum split in two, so eight independent FMA chains are in flight.
__device__ __noinline__ double tc_quad_form64(const double* h64, const float (&w)[32], float dk) {
    double ed[32];
    const float rc = __frcp_rn(dk);
    float fmax_abs = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float x = fminf(fmaxf(__fmul_rn(w[i], rc), kQmin), kQmax);
        const float q = __fsub_rn(__fadd_rn(x, kMagic), kMagic);
        fmax_abs = fmaxf(fmax_abs, fabsf(__fsub_rn(x, q)));
        ed[i] = static_cast<double>(w[i]) - static_cast<double>(__fmul_rn(dk, q));
    }
    if (!(fmax_abs <= kTieWindow && fabsf(rc) <= 3.4028234663852886e38f)) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const float q = code_of(scaled_exact(w[i], dk));
            ed[i] = static_cast<double>(w[i]) - static_cast<double>(__fmul_rn(dk, q));
        }
    }
    double E[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
        double t[8] = {0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0, 0.0};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            const double* row = h64 + tri_start(i + r);     // row i + r: j = i + r..31
#pragma unroll
            for (int j = i + r; j < 32; ++j) t[2 * r + ((j - i - r) & 1)] = fma(row[j - i - r], ed[j], t[2 * r + ((j - i - r) & 1)]);
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) E[r] = fma(ed[i + r], t[2 * r] + t[2 * r + 1], E[r]);
    }
    return (E[0] + E[1]) + (E[2] + E[3]);
}

// Quantizes one candidate for this thread's row: writes e_hi into the stage's
// half of its A row, parks v = 2e - e_hi in the stage's TMEM columns (this
// thread's lane) and returns S = sum |v_i| sd_i.  For an equilibrated block e
// is first scaled to D e.
template <bool EQ>
__device__ __forceinline__ float tc_quantize(const float2 (&ws)[16], float dk, float sig, bool screen,
                                             const float* __restrict__ wrow, float* eslot, const float* sd,
                                             const float* dsc,
                                             uint32_t a_row, uint32_t swz, uint32_t stage, uint32_t tv) {
    const float ds = __fmul_rn(dk, sig);                              // scaled (exact power of two)
    const float rc = __frcp_rn(ds);
    const float2 d2 = make_float2(ds, ds);
    const float2 rc2 = make_float2(rc, rc);
    const float2 M2 = make_float2(kMagic, kMagic);
    const float2 negM2 = make_float2(-kMagic, -kMagic);
    const float2 neg1 = make_float2(-1.0f, -1.0f);
    float2 v[16];
    float fmax_abs = 0.0f;                                            // max_i |x_i - q_i|
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        float2 x = __fmul2_rn(ws[j], rc2);
        x.x = fminf(fmaxf(x.x, kQmin), kQmax);
        x.y = fminf(fmaxf(x.y, kQmin), kQmax);
        const float2 q = __fadd2_rn(__fadd2_rn(x, M2), negM2);       // rint, exact for |x| <= 8
        const float2 f = __ffma2_rn(q, neg1, x);                      // x - q
        fmax_abs = fmaxf(fmax_abs, fmaxf(fabsf(f.x), fabsf(f.y)));
        v[j] = __ffma2_rn(__fmul2_rn(d2, q), neg1, ws[j]);           // e = w - fl(d q), scaled
    }
    // near a rounding boundary (or 1/ds not finite) redo the codes with the IEEE division
    if (screen && !(fmax_abs <= kTieWindow && fabsf(rc) <= 3.4028234663852886e38f)) {
        tc_error_exact(wrow, dk, sig, eslot);
        const float4* e4 = reinterpret_cast<const float4*>(eslot);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 x = e4[c];
            v[2 * c] = make_float2(x.x, x.y);
            v[2 * c + 1] = make_float2(x.z, x.w);
        }
    }
    if (EQ) {            // equilibrated block: e' = D e (powers of two, exact)
        const float4* d4 = reinterpret_cast<const float4*>(dsc);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 dd = d4[c];
            v[2 * c] = __fmul2_rn(v[2 * c], make_float2(dd.x, dd.y));
            v[2 * c + 1] = __fmul2_rn(v[2 * c + 1], make_float2(dd.z, dd.w));
        }
    }
    const float2 two = make_float2(2.0f, 2.0f);
    float S0 = 0.0f, S1 = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        uint32_t hw[4];
        const float4 sa = reinterpret_cast<const float4*>(sd)[2 * c];
        const float4 sb = reinterpret_cast<const float4*>(sd)[2 * c + 1];
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int j = 4 * c + t;
            const __half2 h = __float22half2_rn(v[j]);
            const float2 hf = __half22float2(h);
            v[j] = __ffma2_rn(v[j], two, make_float2(-hf.x, -hf.y));   // v = e + e_lo = 2e - e_hi
            hw[t] = *reinterpret_cast<const uint32_t*>(&h);
        }
        S0 = fmaf(fabsf(v[4 * c].x), sa.x, S0);
        S1 = fmaf(fabsf(v[4 * c].y), sa.y, S1);
        S0 = fmaf(fabsf(v[4 * c + 1].x), sa.z, S0);
        S1 = fmaf(fabsf(v[4 * c + 1].y), sa.w, S1);
        S0 = fmaf(fabsf(v[4 * c + 2].x), sb.x, S0);
        S1 = fmaf(fabsf(v[4 * c + 2].y), sb.y, S1);
        S0 = fmaf(fabsf(v[4 * c + 3].x), sb.z, S0);
        S1 = fmaf(fabsf(v[4 * c + 3].y), sb.w, S1);
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                     :: "r"(a_row + (((4u * stage + static_cast<uint32_t>(c)) ^ swz) << 4)),
                        "r"(hw[0]), "r"(hw[1]), "r"(hw[2]), "r"(hw[3]) : "memory");
    }
    uint32_t vb[32];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        vb[2 * j] = __float_as_uint(v[j].x);
        vb[2 * j + 1] = __float_as_uint(v[j].y);
    }
    tmem_st_32x32b_x32(tv, vb);
    return S0 + S1;
}

// The MMAs of one candidate (issued by one thread): P = e_hi (H_hi + H_lo) into
// the stage's TMEM columns 0..31.
__device__ __forceinline__ void tc_issue(uint32_t tmem_stage, uint32_t a_stage, uint32_t bh, uint32_t bl,
                                         uint64_t* bar) {
    tc_fence_after();
#pragma unroll
    for (uint32_t kk = 0; kk < 2; ++kk)
        tc_mma_f16(tmem_stage, smem_desc_k_sw128(a_stage + 32u * kk), smem_desc_k_sw128(bh + 32u * kk),
                   kTcIdesc, kk > 0 ? 1u : 0u);
#pragma unroll
    for (uint32_t kk = 0; kk < 2; ++kk)
        tc_mma_f16(tmem_stage, smem_desc_k_sw128(a_stage + 32u * kk), smem_desc_k_sw128(bl + 32u * kk),
                   kTcIdesc, 1u);
    tc_commit(bar);
}

struct TcBound {
    float coef, coef_f, tsum;
};

// Reads candidate k's P row and v from TMEM, forms E = P . v and its bound, and
// records them.  Returns false if the wait for the MMAs gave up.
__device__ __forceinline__ bool tc_consume(int k, uint32_t tst, uint64_t* bar, volatile int* abort,
                                           uint64_t limit_ns, float S, const TcBound& tb,
                                           TopK4& top, float& upper) {
    if (!mbar_wait_parked(bar, static_cast<uint32_t>((k >> 1) & 1), abort, limit_ns)) return false;
    tc_fence_after();
    float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t P[16], V[16];
        tmem_ld_32x32b_x16(tst + 16u * h, P);
        tmem_ld_32x32b_x16(tst + 32u + 16u * h, V);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j)
            acc[j & 3] = fmaf(__uint_as_float(P[j]), __uint_as_float(V[j]), acc[j & 3]);
    }
    const float E = (acc[0] + acc[1]) + (acc[2] + acc[3]);
    const float Sa = __fmul_ru(1.001953125f, __fmaf_ru(6.103515625e-05f, tb.tsum, S));     // (1+2^-9)(S + 2^-14 T)
    const float b = __fmaf_ru(tb.coef, __fmul_ru(Sa, Sa), __fmul_ru(tb.coef_f, __fmul_ru(tb.tsum, Sa)));
    upper = fminf(upper, E + b);
    top.insert(E - b, k);
    return true;
}

template <int MINB>
__global__ void __launch_bounds__(kTcRows, MINB)
scale_search_kernel(const float* __restrict__ W, int R, int C,
                       const float* __restrict__ H, int64_t ldh,
                       const float* __restrict__ alpha, int K,
                       float* __restrict__ delta_out, int* __restrict__ idx_out,
                       float* __restrict__ err_out, uint64_t limit_ns) {
    extern __shared__ __align__(16) uint8_t tc_smem_raw[];
    const uint32_t raw = smem_u32(tc_smem_raw);
    SearchTcSmem& sm = *reinterpret_cast<SearchTcSmem*>(tc_smem_raw + ((1024u - (raw & 1023u)) & 1023u));
    const int g = blockIdx.y;
    const int G = C / kGroup;
    const int tid = threadIdx.x;
    const int warp = tid >> 5;

    // ---- set-up: barriers, TMEM, H_gg and its derived tables
    if (tid == 0) {
        mbar_init(&sm.mbar[0], 1);
        mbar_init(&sm.mbar[1], 1);
        fence_mbar_init();
        sm.kappa_bits = __float_as_uint(1.0f);
        sm.kappa_d_bits = 0u;
        sm.hmax_bits = 0u;
        sm.exact_block = 0;
        sm.abort = 0;
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, kTcTmemCols);
        tmem_relinquish();
        tc_fence_before();
    }
    const float* Hg = H + static_cast<int64_t>(g) * kGroup * ldh + static_cast<int64_t>(g) * kGroup;
    for (int x = tid; x < 32 * 32; x += kTcRows) {
        const int i = x >> 5, j = x & 31;
        sm.u.hfull[i][j] = Hg[static_cast<int64_t>(i) * ldh + j];
    }
    // zero the B tiles (columns k >= 32 of each row are never written below)
    for (int x = tid; x < (2 * 32 * 128) / 16; x += kTcRows)
        reinterpret_cast<uint4*>(sm.bhi)[x] = make_uint4(0u, 0u, 0u, 0u);    // bhi and blo are contiguous
    __syncthreads();

    // float64 table of the block for the re-score: H'_ij = H_ij + H_ji (j > i), H'_ii = H_ii (unscaled)
    for (int x = tid; x < 32 * 32; x += kTcRows) {
        const int i = x >> 5, j = x & 31;
        if (j == i)
            sm.h64[tri_start(i)] = static_cast<double>(sm.u.hfull[i][j]);
        else if (j > i)
            sm.h64[tri_start(i) + (j - i)] =
                static_cast<double>(sm.u.hfull[i][j]) + static_cast<double>(sm.u.hfull[j][i]);
    }
    // The binary16 split and its bound, first for the block as it is (pass 0), then -- only if
    // that split's error ratio kappa_d exceeds 2^-17 -- for the equilibrated block
    // D^-1 H D^-1 (pass 1).  Every quantity below is of the block of the pass: entries
    // a' = a / (d_i d_j), exact in binary64 since the d_i are powers of two.
    for (int pass = 0; pass < 2; ++pass) {
        if (tid < 32) {
            float d = 1.0f;
            if (pass == 1) {   // a power of two near sqrt|H_ii|: H_ii / d^2 in [1, 4)
                const float h = fabsf(sm.u.hfull[tid][tid]);
                if (h >= 1.1754943508222875e-38f && h <= 3.4028234663852886e38f) {
                    const int e = static_cast<int>((__float_as_uint(h) >> 23) & 0xFF) - 127;
                    d = __uint_as_float(static_cast<uint32_t>(127 + (e >> 1)) << 23);
                }
            }
            sm.dsc[tid] = d;
            sm.idsc[tid] = 1.0f / d;     // exact: d is a power of two
        }
        if (tid == 0) {
            sm.kappa_bits = __float_as_uint(1.0f);
            sm.kappa_d_bits = 0u;
            sm.hmax_bits = 0u;
            sm.eq = pass;
        }
        __syncthreads();

        // 1/sqrt|H'_ii| rounded up (for kappa): an upper bound of the true reciprocal
        if (tid < 32) {
            const double hd = static_cast<double>(sm.u.hfull[tid][tid]) *
                              (static_cast<double>(sm.idsc[tid]) * static_cast<double>(sm.idsc[tid]));
            sm.isd[tid] = __fdiv_ru(1.0f, __fsqrt_rd(__double2float_rd(fabs(hd))));
        }
        __syncthreads();

        // kappa and the largest |(H'_ij + H'_ji)/2|
        float kap = 0.0f, hmax = 0.0f;
        for (int x = tid; x < 32 * 32; x += kTcRows) {
            const int i = x >> 5, j = x & 31;
            const double dij = static_cast<double>(sm.idsc[i]) * static_cast<double>(sm.idsc[j]);   // exact
            const double a = static_cast<double>(sm.u.hfull[i][j]) * dij, b = static_cast<double>(sm.u.hfull[j][i]) * dij;
            const float hs = up(fabs(0.5 * (a + b)));
            hmax = fmaxf(hmax, (hs <= 3.4028234663852886e38f) ? hs : __int_as_float(0x7f800000));
            if (j > i) {
                const float mm = up(fmax(fabs(a), fabs(b)));
                if (mm != 0.0f) {
                    const float ratio = __fmul_ru(__fmul_ru(mm, sm.isd[i]), sm.isd[j]);
                    kap = fmaxf(kap, (ratio <= 3.4028234663852886e38f) ? ratio : __int_as_float(0x7f800000));
                }
            }
        }
        {   // non-negative floats order like their bit patterns: one shared atomic per warp
            const unsigned kb = __reduce_max_sync(0xffffffffu, __float_as_uint(kap));
            const unsigned hb = __reduce_max_sync(0xffffffffu, __float_as_uint(hmax));
            if ((tid & 31) == 0) {
                atomicMax(&sm.kappa_bits, kb);
                atomicMax(&sm.hmax_bits, hb);
            }
        }
        __syncthreads();

        // scale of the block: 2^13 <= hmax * sigma_H < 2^14
        const float hmx = __uint_as_float(sm.hmax_bits);
        const bool hbad = !(hmx >= 1.0e-30f) || !(hmx <= 1.0e30f);
        const int eh = hbad ? 0 : static_cast<int>((__float_as_uint(hmx) >> 23) & 0xFF) - 127;
        const double sigH = static_cast<double>(__uint_as_float(static_cast<uint32_t>(127 + 13 - eh) << 23));
        if (tid < 32) {
            const double hd = static_cast<double>(sm.u.hfull[tid][tid]) *
                              (static_cast<double>(sm.idsc[tid]) * static_cast<double>(sm.idsc[tid]));
            const float sd = hbad ? 0.0f : __fsqrt_ru(up(fabs(hd) * sigH));
            sm.sd[tid] = sd;
            sm.isd[tid] = __fdiv_ru(1.0f, sd);          // for kappa_d (inf when sd = 0)
        }
        __syncthreads();

        // binary16 split of the scaled symmetrised block; entry (k, n) goes to row n, column k of B
        float kapd = 0.0f;
        for (int x = tid; x < 32 * 32; x += kTcRows) {
            const int k = x >> 5, n = x & 31;
            const double dkn = static_cast<double>(sm.idsc[k]) * static_cast<double>(sm.idsc[n]);   // exact
            const double s = 0.5 * (static_cast<double>(sm.u.hfull[k][n]) + static_cast<double>(sm.u.hfull[n][k])) *
                             dkn * sigH;
            __half hi = __float2half_rn(static_cast<float>(s));
            if (!(fabsf(__half2float(hi)) >= 6.103515625e-05f)) hi = __float2half_rn(0.0f);   // no subnormal parts
            const double r1 = s - static_cast<double>(__half2float(hi));
            __half lo = __float2half_rn(static_cast<float>(r1));
            if (!(fabsf(__half2float(lo)) >= 6.103515625e-05f)) lo = __float2half_rn(0.0f);
            const float dlt = up(fabs(r1 - static_cast<double>(__half2float(lo))));
            if (dlt != 0.0f) {
                const float ratio = __fmul_ru(__fmul_ru(dlt, sm.isd[k]), sm.isd[n]);
                kapd = fmaxf(kapd, (ratio <= 3.4028234663852886e38f) ? ratio : __int_as_float(0x7f800000));
            }
            const uint32_t off = sw128_off(static_cast<uint32_t>(n), static_cast<uint32_t>(k >> 3)) + (k & 7) * 2;
            *reinterpret_cast<__half*>(sm.bhi + off) = hi;
            *reinterpret_cast<__half*>(sm.blo + off) = lo;
        }
        {
            const unsigned db = __reduce_max_sync(0xffffffffu, __float_as_uint(kapd));
            if ((tid & 31) == 0) atomicMax(&sm.kappa_d_bits, db);
        }
        __syncthreads();
        if (tid == 0) {
            const double kp = static_cast<double>(__uint_as_float(sm.kappa_bits));
            const double kd = static_cast<double>(__uint_as_float(sm.kappa_d_bits));
            double ts = 0.0;
            for (int i = 0; i < 32; ++i) ts += static_cast<double>(sm.sd[i]);
            const double tau = 7.62939453125e-06;                         // 2^-17
            const double c = (kp + kd) * (tau + 1.9073486328125e-06 + 2.384185791015625e-07) + kd +
                             kp * (9.5367431640625e-07 + 1.1920928955078125e-07);
            sm.coef = up(c * 1.02);
            sm.coef_f = up((kp + kd) * 2.44140625e-04 * 1.02);            // 2^-12
            sm.tsum = up(ts * (1.0 + 1e-6));
            sm.exact_block = (hbad || !(sm.coef <= 1.0e30f) || !(sm.coef_f <= 1.0e30f)) ? 1 : 0;
        }
        __syncthreads();
        // keep this pass unless its split is poor and the block can be equilibrated
        if (pass == 1 || hbad || !(__uint_as_float(sm.kappa_d_bits) > 7.62939453125e-06f)) break;
        __syncthreads();
    }
    fence_proxy_async_smem();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    const TcBound tb{sm.coef, sm.coef_f, sm.tsum};
    const bool exact_block = sm.exact_block != 0;

    // ---- this thread's row
    const int r = blockIdx.x * kTcRows + tid;
    const bool valid = r < R;
    const float* wrow = W + static_cast<int64_t>(valid ? r : 0) * C + g * kGroup;
    float2 ws[16];
    if (valid) {
        const float4* wp = reinterpret_cast<const float4*>(wrow);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 x = __ldg(wp + c);
            ws[2 * c] = make_float2(x.x, x.y);
            ws[2 * c + 1] = make_float2(x.z, x.w);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) ws[j] = make_float2(0.0f, 0.0f);
    }
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 16; ++j) m = fmaxf(m, fmaxf(fabsf(ws[j].x), fabsf(ws[j].y)));
    const bool zero = (m == 0.0f);
    const float base = __fdiv_rn(m, 7.0f);
    const bool eq = sm.eq != 0;
    float md = m;        // the largest |w_i| d_i: m unless the block is equilibrated
    if (eq) {
        md = 0.0f;
        const float4* d4 = reinterpret_cast<const float4*>(sm.dsc);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const float4 dd = d4[c];
            md = fmaxf(md, fmaxf(fabsf(ws[2 * c].x) * dd.x, fabsf(ws[2 * c].y) * dd.y));
            md = fmaxf(md, fmaxf(fabsf(ws[2 * c + 1].x) * dd.z, fabsf(ws[2 * c + 1].y) * dd.w));
        }
    }
    // exact_row: the power-of-two row scale would leave binary32 range; re-score every candidate
    const bool exact_row = exact_block || !(m >= 7.888609052210118e-31f) ||      // 2^-100
                           !(md >= 7.888609052210118e-31f) || !(md <= 1.2676506002282294e30f);   // 2^100
    // row scale: 2^13 <= max_i |w_i| d_i sigma < 2^14, so every |e_i d_i| sigma < 2^14
    const int em = exact_row ? 0 : static_cast<int>((__float_as_uint(md) >> 23) & 0xFF) - 127;
    const float sig = __uint_as_float(static_cast<uint32_t>(127 + 13 - em) << 23);
    const bool screen = valid && !zero && !exact_row;
#pragma unroll
    for (int j = 0; j < 16; ++j)
        ws[j] = screen ? make_float2(__fmul_rn(ws[j].x, sig), __fmul_rn(ws[j].y, sig)) : make_float2(0.0f, 0.0f);
    float* eslot = sm.u.eslot + tid * kTcSlot;
    const uint32_t swz = static_cast<uint32_t>(tid) & 7u;
    const uint32_t a0 = smem_u32(sm.a);
    const uint32_t a_row = a0 + static_cast<uint32_t>(tid) * 128u;
    const uint32_t bh = smem_u32(sm.bhi), bl = smem_u32(sm.blo);
    const uint32_t tlane = tmem + (static_cast<uint32_t>(warp * 32) << 16);   // this warp's lanes
    const bool lane0 = (tid & 31) == 0;

    TopK4 top;
    top.init();
    float upper = __int_as_float(0x7f800000);
    bool ok = true;

    float S0 = 0.0f, S1 = 0.0f;
    // the candidate loop, compiled once for plain and once for equilibrated blocks
    auto candidate_loop = [&](auto eq_tag) {
        constexpr bool EQ = decltype(eq_tag)::value;
        // prologue: candidate 0 into stage 0
        S0 = tc_quantize<EQ>(ws, __fmul_rn(__ldg(alpha), base), sig, screen, wrow, eslot, sm.sd, sm.dsc, a_row,
                             swz, 0u, tlane + 32u);
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) tc_issue(tmem, a0, bh, bl, &sm.mbar[0]);

        // steady state, two candidates per trip so the stages alternate statically: quantize
        // candidate k + 1 into the other stage, hand it to the tensor core, then consume k
        for (int k = 0; k < K; k += 2) {
            if (k + 1 < K) {
                S1 = tc_quantize<EQ>(ws, __fmul_rn(__ldg(alpha + k + 1), base), sig, screen, wrow, eslot, sm.sd,
                                     sm.dsc, a_row, swz, 1u, tlane + kTcStageCols + 32u);
                tmem_st_wait();
                fence_proxy_async_smem();
                tc_fence_before();
                if (__syncthreads_or(!ok)) { ok = false; break; }
                if (lane0 && warp == ((k + 1) & 3)) tc_issue(tmem + kTcStageCols, a0 + 64u, bh, bl, &sm.mbar[1]);
            }
            if (ok) ok = tc_consume(k, tlane, &sm.mbar[0], &sm.abort, limit_ns, S0, tb, top, upper);
            if (k + 1 >= K) break;
            if (k + 2 < K) {
                S0 = tc_quantize<EQ>(ws, __fmul_rn(__ldg(alpha + k + 2), base), sig, screen, wrow, eslot, sm.sd,
                                     sm.dsc, a_row, swz, 0u, tlane + 32u);
                tmem_st_wait();
                fence_proxy_async_smem();
                tc_fence_before();
                if (__syncthreads_or(!ok)) { ok = false; break; }
                if (lane0 && warp == ((k + 2) & 3)) tc_issue(tmem, a0, bh, bl, &sm.mbar[0]);
            }
            if (ok) ok = tc_consume(k + 1, tlane + kTcStageCols, &sm.mbar[1], &sm.abort, limit_ns, S1, tb, top, upper);
        }
    };
    if (eq) candidate_loop(BoolTag<true>{});
    else candidate_loop(BoolTag<false>{});
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, kTcTmemCols);
    if (!ok) return;

    // ---- float64 re-score of every candidate the screening could not exclude
    int nfin = 0;
#pragma unroll
    for (int a = 0; a < 4; ++a) nfin += (top.k[a] >= 0 && top.L[a] <= upper) ? 1 : 0;
    // a row whose four smallest lower bounds all reach the upper bound is re-scored over every
    // candidate, by the whole warp (one row at a time, candidates spread over the lanes)
    const bool overflow = valid && !zero && (!screen || (nfin == 4 && K > 4) || nfin == 0);
    const int lane = tid & 31;
    double best = 0.0;
    int best_k = -1;
    unsigned pending = __ballot_sync(0xffffffffu, overflow);
    while (pending) {
        const int src = __ffs(pending) - 1;
        pending &= pending - 1;
        const float* wsrc = W + static_cast<int64_t>(blockIdx.x * kTcRows + warp * 32 + src) * C + g * kGroup;
        const float bsrc = __shfl_sync(0xffffffffu, base, src);
        float wv[32];
        {
            const float4* wp = reinterpret_cast<const float4*>(wsrc);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 x = __ldg(wp + c);
                wv[4 * c] = x.x; wv[4 * c + 1] = x.y; wv[4 * c + 2] = x.z; wv[4 * c + 3] = x.w;
            }
        }
        double lb = 0.0;
        int lk = -1;
        for (int kk = lane; kk < K; kk += 32) {
            const double E = tc_quad_form64(sm.h64, wv, __fmul_rn(__ldg(alpha + kk), bsrc));
            if (lk < 0 || E < lb) { lb = E; lk = kk; }            // kk ascending: ties keep the smaller
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {                          // argmin, smallest k on ties
            const double ob = __shfl_xor_sync(0xffffffffu, lb, o);
            const int ok2 = __shfl_xor_sync(0xffffffffu, lk, o);
            if (ok2 >= 0 && (lk < 0 || ob < lb || (ob == lb && ok2 < lk))) { lb = ob; lk = ok2; }
        }
        if (lane == src) { best = lb; best_k = lk; }
    }
    if (!valid) return;
    const int64_t out = static_cast<int64_t>(r) * G + g;
    if (zero) {   // all-zero group: every candidate has zero error
        delta_out[out] = 0.0f;
        idx_out[out] = 0;
        if (err_out) err_out[out] = 0.0f;
        return;
    }
    if (!overflow) {
        float wv[32];
        {
            const float4* wp = reinterpret_cast<const float4*>(wrow);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 x = __ldg(wp + c);
                wv[4 * c] = x.x; wv[4 * c + 1] = x.y; wv[4 * c + 2] = x.z; wv[4 * c + 3] = x.w;
            }
        }
        for (int a = 0; a < nfin; ++a) {
            const int kk = a == 0 ? top.k[0] : a == 1 ? top.k[1] : a == 2 ? top.k[2] : top.k[3];
            const double E = tc_quad_form64(sm.h64, wv, __fmul_rn(__ldg(alpha + kk), base));
            if (best_k < 0 || E < best || (E == best && kk < best_k)) { best = E; best_k = kk; }
        }
    }
    delta_out[out] = __fmul_rn(__ldg(alpha + best_k), base);
    idx_out[out] = best_k;
    if (err_out) err_out[out] = static_cast<float>(best);
}

}  // namespace qat4
