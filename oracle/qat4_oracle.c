/*
 * qat4_oracle.c -- plain CPU reference of the group-32 symmetric INT4 weight
 * quantizer (calibration Hessian, Hessian-weighted scale search, LSQ forward /
 * backward, W4A16 packing), and the products either side of it (the W4A16
 * inference GEMV on the export, the fake-quant forward GEMM of a QAT step).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or helper with the
 * CUDA kernels.
 *
 * Build: gcc -O2 -std=c11 -ffp-contract=off -fno-fast-math -fopenmp -fPIC
 *        -shared  (x86-64 SSE arithmetic: every float operation below is one
 *        IEEE binary32 operation in round-to-nearest-even, every double
 *        operation one binary64 operation; no contraction into FMA).
 *
 * Sources (web pages on the method):
 *  [card]  model card "Opt.Gear-1B-qat-int4-per-channel-unquantized",
 *          section "Quantization Configuration" (symmetric, zero-point 0;
 *          the per-group objective  Delta* = argmin ||W X - Q_Delta(W) X||_F^2)
 *          and "QAT Highlights" (group size 32, same grid at init/QAT/export).
 *  [blog]  "Opt.Gear-QAT: Preserving On-Device Performance with QAT",
 *          section "Quantization parameters of Opt.Gear-1B" (group size 32,
 *          symmetric), section 1 "Quantization scale is important" (uniform
 *          projection onto a limited integer grid with step Delta), section 2
 *          "Hessian-based scale initialize" (layer sensitivity from
 *          calibration inputs, second-order output reconstruction), section 3
 *          "LSQ-based QAT" (forward emulates the deployment INT4 grid; STE for
 *          round; step-size gradient normalised by the group's element count
 *          and the number of positive levels).
 *  The printed formulas of [blog] sections 1-3 were lost; where a step is not
 *  fixed by the surviving text the plainest reading is taken:
 *    Q_Delta(w) = Delta * clamp(rint(w / Delta), -8, 7), rint = half-to-even;
 *    H = X^T X / n;  Delta_k = alpha_k * (max|w_g| / 7);
 *    objective per group = e H_gg e^T with e = w_g - Q(w_g) exactly
 *    (block-diagonal reading of the objective, other groups held at zero
 *    error);
 *    LSQ (Esser et al., "Learned Step Size Quantization", ICLR 2020) step
 *    gradient with scale s = 1/sqrt(32 * 7).
 *
 * Pins: none of these functions can be pinned to a number printed on the
 * pages (they print no worked example of the quantizer).  Each is pinned by
 * mathematics instead -- closed forms, invariants, special cases and brute
 * force on tiny inputs -- in the CPU test-suite.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define GROUP 32
#define QMIN (-8.0f)
#define QMAX (7.0f)

/* ---------------------------------------------------------------- helpers */

int oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
    return omp_get_max_threads();
#else
    (void)n;
    return 1;
#endif
}

/* bf16 bit pattern -> float: the 16 bits are the top half of a binary32. */
static float bf16_to_float(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* v = w / Delta as one IEEE binary32 division ([blog] section 1).
 * Delta == 0 only happens for an all-zero group; v is then taken as 0. */
static float scaled(float w, float delta)
{
    if (delta == 0.0f) return 0.0f;
    return w / delta;
}

/* q = clamp(round(v), -8, 7), round = round-half-to-even ([card]
 * "Symmetric (zero-point fixed at 0)"; INT4 two's-complement range). */
static float code_of(float v)
{
    float q = rintf(v);
    if (q < QMIN) q = QMIN;
    if (q > QMAX) q = QMAX;
    return q;
}

/* Q_Delta(w) = Delta * q, one binary32 multiply. */
static float fake_quant(float w, float delta)
{
    float q = code_of(scaled(w, delta));
    return delta * q;
}

/* ----------------------------------------------------- (a) Hessian H=X^TX/n
 * [blog] section 2: layer sensitivity estimated from calibration inputs; the
 * second-order output-reconstruction Hessian of ||W X - Q X||^2 is X^T X
 * (up to the 1/n normalisation).  Products of bf16 values are exact in
 * double; the sum over the n calibration rows is taken in double.
 * X: bf16 bits, row-major [n, C].  H: double, row-major [C, C] (full). */
void oracle_hessian(const uint16_t *X, int64_t n, int64_t C, double *H)
{
    /* Row i of H is one accumulator per column j; the calibration rows t are
     * visited in order, so every entry is the sum over t = 0, 1, ..., n-1
     * taken left to right, starting from 0. */
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < C; ++i) {
        double *s = H + i * C;
        for (int64_t j = 0; j < C; ++j) s[j] = 0.0;
        for (int64_t t = 0; t < n; ++t) {
            const uint16_t *xt = X + t * C;
            const double xi = (double)bf16_to_float(xt[i]);
            for (int64_t j = 0; j < C; ++j)
                s[j] += xi * (double)bf16_to_float(xt[j]);
        }
        for (int64_t j = 0; j < C; ++j) s[j] = s[j] / (double)n;
    }
}

/* Selected entries H[ii[m], jj[m]] only (for sampled checks of large X). */
void oracle_hessian_entries(const uint16_t *X, int64_t n, int64_t C,
                            const int64_t *ii, const int64_t *jj, int64_t count,
                            double *out)
{
    #pragma omp parallel for schedule(dynamic, 16)
    for (int64_t m = 0; m < count; ++m) {
        int64_t i = ii[m], j = jj[m];
        double s = 0.0;
        for (int64_t t = 0; t < n; ++t) {
            double xi = (double)bf16_to_float(X[t * C + i]);
            double xj = (double)bf16_to_float(X[t * C + j]);
            s += xi * xj;
        }
        out[m] = s / (double)n;
    }
}

/* One block H[r0:r0+nr, c0:c0+nc] into out (row-major [nr, nc]), computed by
 * the calling thread: for every calibration row t in order, every entry of the
 * block adds x[t][r0+a] * x[t][c0+b].  Same sums, same order as
 * oracle_hessian. */
static void hessian_block_serial(const uint16_t *X, int64_t n, int64_t C,
                                 int64_t r0, int64_t nr, int64_t c0, int64_t nc, double *out)
{
    double xb[256];                       /* x[t][c0 .. c0+nc-1], nc <= 256 */
    for (int64_t m = 0; m < nr * nc; ++m) out[m] = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        const uint16_t *xt = X + t * C;
        for (int64_t b = 0; b < nc; ++b) xb[b] = (double)bf16_to_float(xt[c0 + b]);
        for (int64_t a = 0; a < nr; ++a) {
            const double xa = (double)bf16_to_float(xt[r0 + a]);
            double *s = out + a * nc;
            for (int64_t b = 0; b < nc; ++b)
                s[b] += xa * xb[b];
        }
    }
    for (int64_t m = 0; m < nr * nc; ++m) out[m] = out[m] / (double)n;
}

/* A dense block H[r0:r0+nr, c0:c0+nc] (row-major [nr, nc] in out). */
void oracle_hessian_block(const uint16_t *X, int64_t n, int64_t C,
                          int64_t r0, int64_t nr, int64_t c0, int64_t nc, double *out)
{
    /* one strip of 8 rows by up to 256 columns of the block per thread */
    const int64_t strips = (nr + 7) / 8, panels = (nc + 255) / 256;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t sp = 0; sp < strips * panels; ++sp) {
        const int64_t a = (sp / panels) * 8, b = (sp % panels) * 256;
        const int64_t rows = (nr - a < 8) ? nr - a : 8;
        const int64_t cols = (nc - b < 256) ? nc - b : 256;
        double tmp[8 * 256];
        hessian_block_serial(X, n, C, r0 + a, rows, c0 + b, cols, tmp);
        for (int64_t i = 0; i < rows; ++i)
            for (int64_t j = 0; j < cols; ++j) out[(a + i) * nc + b + j] = tmp[i * cols + j];
    }
}

/* Many b x b blocks (b <= 256): block m is H[r0[m]:r0[m]+b, c0[m]:c0[m]+b],
 * written to out + m*b*b (row-major).  One block per thread. */
void oracle_hessian_blocks(const uint16_t *X, int64_t n, int64_t C,
                           const int64_t *r0, const int64_t *c0, int64_t count, int64_t b,
                           double *out)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t m = 0; m < count; ++m)
        hessian_block_serial(X, n, C, r0[m], b, c0[m], b, out + m * b * b);
}

/* ------------------------------------------ (b) Hessian-weighted scale search
 * [card] "Quantization Configuration": for each quantization group the scale
 * is initialised as Delta* = argmin_Delta ||W X - Q_Delta(W) X||_F^2, searched
 * here over the finite grid Delta_k = alpha_k * (max|w_g| / 7).  For one
 * group g of row r the objective is the quadratic form e H_gg e^T with
 * e = w_g - Q_{Delta_k}(w_g), the exact difference of the binary32 weights and
 * their binary32 quantized values (exact in binary64), and H_gg the 32x32
 * diagonal block of H.  Every candidate is evaluated; the smallest index
 * reaching the minimum wins.
 *
 * W: float [R, C] row-major; H: float, row stride ldh (only the diagonal
 * 32x32 blocks are read); alpha: float [K].
 * Outputs per (r, g), row-major [R, C/32]: delta (float), idx (int32),
 * best_err (double).  all_err (nullable): double [R, C/32, K]. */
void oracle_scale_search(const float *W, int64_t R, int64_t C,
                         const float *H, int64_t ldh,
                         const float *alpha, int32_t K,
                         float *delta_out, int32_t *idx_out, double *best_err,
                         double *all_err)
{
    const int64_t G = C / GROUP;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t g = 0; g < G; ++g) {
            const float *w = W + r * C + g * GROUP;
            const float *Hg = H + (g * GROUP) * ldh + g * GROUP;
            float m = 0.0f;
            for (int i = 0; i < GROUP; ++i) {
                float a = fabsf(w[i]);
                if (a > m) m = a;
            }
            float base = m / 7.0f;
            int32_t best_k = -1;
            double best = 0.0;
            float best_delta = 0.0f;
            for (int32_t k = 0; k < K; ++k) {
                float dk = alpha[k] * base;
                double e[GROUP];
                for (int i = 0; i < GROUP; ++i) {
                    float qw = fake_quant(w[i], dk);
                    e[i] = (double)w[i] - (double)qw;   /* exact in binary64 */
                }
                double E = 0.0;
                for (int i = 0; i < GROUP; ++i)
                    for (int j = 0; j < GROUP; ++j)
                        E += e[i] * (double)Hg[i * ldh + j] * e[j];
                if (all_err) all_err[(r * G + g) * K + k] = E;
                if (best_k < 0 || E < best) {
                    best = E;
                    best_k = k;
                    best_delta = dk;
                }
            }
            delta_out[r * G + g] = best_delta;
            idx_out[r * G + g] = best_k;
            best_err[r * G + g] = best;
        }
    }
}

/* ----------------------------------------------------------- (c) LSQ forward
 * [blog] section 3: the forward pass emulates the deployment INT4 grid,
 * Q = Delta * clamp(round(w / Delta), -8, 7), each group with its own Delta.
 * W, Q: float [R, C]; delta: float [R, C/32]. */
void oracle_lsq_fwd(const float *W, const float *delta, int64_t R, int64_t C, float *Q)
{
    const int64_t G = C / GROUP;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < C; ++c)
            Q[r * C + c] = fake_quant(W[r * C + c], delta[r * G + c / GROUP]);
}

/* ---------------------------------------------------------- (c) LSQ backward
 * [blog] section 3: round is passed straight through (STE) to the weights;
 * LSQ carries the task gradient to the step size, normalised by the group's
 * element count and the number of positive levels (s = 1/sqrt(32*7) is
 * passed in as grad_scale).  With v = w / Delta (the same binary32 value as
 * the forward):
 *   grad_W = G            if -8 <= v <= 7, else 0
 *   dQ/dDelta = rint(v) - v  if -8 < v < 7;  -8 if v <= -8;  7 if v >= 7
 *   grad_Delta[r, g] = s * sum_{i in g} G_i * dQ_i/dDelta   (sum in double)
 * G: float [R, C] when g_is_bf16 == 0, else bf16 bits [R, C].
 * grad_W: float [R, C]; grad_delta: double [R, C/32]. */
void oracle_lsq_bwd(const float *W, const float *delta, const void *Gp, int g_is_bf16,
                    int64_t R, int64_t C, float grad_scale,
                    float *grad_W, double *grad_delta)
{
    const int64_t G = C / GROUP;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t g = 0; g < G; ++g) {
            float dl = delta[r * G + g];
            double acc = 0.0;
            for (int i = 0; i < GROUP; ++i) {
                int64_t idx = r * C + g * GROUP + i;
                float gi = g_is_bf16 ? bf16_to_float(((const uint16_t *)Gp)[idx])
                                     : ((const float *)Gp)[idx];
                float v = scaled(W[idx], dl);
                int inside = (v >= QMIN) && (v <= QMAX);
                grad_W[idx] = inside ? gi : 0.0f;
                float d;
                if (v <= QMIN)      d = QMIN;
                else if (v >= QMAX) d = QMAX;
                else                d = rintf(v) - v;
                acc += (double)gi * (double)d;
            }
            grad_delta[r * G + g] = (double)grad_scale * acc;
        }
    }
}

/* ------------------------------------------------------------ (c) W4A16 pack
 * [card] "QAT Highlights": the same INT4 grid is used at initialisation, QAT
 * and export, so the exported codes are the forward codes
 * q = clamp(rint(w / Delta), -8, 7) with the binary32 Delta.  Element 2j goes
 * to the low nibble of byte j and element 2j+1 to the high nibble (4-bit
 * two's complement); the per-group scale is exported as IEEE binary16,
 * round-to-nearest-even.
 * packed: uint8 [R, C/2]; scale16: binary16 bits [R, C/32]. */
void oracle_pack_w4a16(const float *W, const float *delta, int64_t R, int64_t C,
                       uint8_t *packed, uint16_t *scale16)
{
    const int64_t G = C / GROUP;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t j = 0; j < C / 2; ++j) {
            int64_t c0 = 2 * j, c1 = 2 * j + 1;
            int lo = (int)code_of(scaled(W[r * C + c0], delta[r * G + c0 / GROUP]));
            int hi = (int)code_of(scaled(W[r * C + c1], delta[r * G + c1 / GROUP]));
            packed[r * (C / 2) + j] = (uint8_t)((lo & 0xF) | ((hi & 0xF) << 4));
        }
        for (int64_t g = 0; g < G; ++g) {
            _Float16 h = (_Float16)delta[r * G + g];
            uint16_t bits;
            memcpy(&bits, &h, sizeof bits);
            scale16[r * G + g] = bits;
        }
    }
}

/* Codes only (int8), for unpack checks. */
void oracle_codes(const float *W, const float *delta, int64_t R, int64_t C, int8_t *codes)
{
    const int64_t G = C / GROUP;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < C; ++c)
            codes[r * C + c] = (int8_t)code_of(scaled(W[r * C + c], delta[r * G + c / GROUP]));
}

/* ------------------------------------------------ per-channel (one scale per row)
 * Model card "Opt.Gear-1B-qat-int4-per-channel-unquantized": the same
 * symmetric INT4 grid with one scale per output channel (row), W4A16 export
 * with learned channel-wise scales.  The quantizer, the straight-through
 * weight gradient and the step gradient are those of the group-32 functions
 * above with the group widened to the whole row; the step-gradient
 * normalisation uses the row's element count, s = 1/sqrt(C * 7), passed in.
 * delta, grad_delta, scale16: one value per row [R]. */
void oracle_lsq_fwd_rowwise(const float *W, const float *delta, int64_t R, int64_t C, float *Q)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < C; ++c)
            Q[r * C + c] = fake_quant(W[r * C + c], delta[r]);
}

void oracle_lsq_bwd_rowwise(const float *W, const float *delta, const void *Gp, int g_is_bf16,
                            int64_t R, int64_t C, float grad_scale,
                            float *grad_W, double *grad_delta)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        float dl = delta[r];
        double acc = 0.0;
        for (int64_t c = 0; c < C; ++c) {
            int64_t idx = r * C + c;
            float gi = g_is_bf16 ? bf16_to_float(((const uint16_t *)Gp)[idx])
                                 : ((const float *)Gp)[idx];
            float v = scaled(W[idx], dl);
            int inside = (v >= QMIN) && (v <= QMAX);
            grad_W[idx] = inside ? gi : 0.0f;
            float d;
            if (v <= QMIN)      d = QMIN;
            else if (v >= QMAX) d = QMAX;
            else                d = rintf(v) - v;
            acc += (double)gi * (double)d;
        }
        grad_delta[r] = (double)grad_scale * acc;
    }
}

void oracle_pack_w4a16_rowwise(const float *W, const float *delta, int64_t R, int64_t C,
                               uint8_t *packed, uint16_t *scale16)
{
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t j = 0; j < C / 2; ++j) {
            int lo = (int)code_of(scaled(W[r * C + 2 * j], delta[r]));
            int hi = (int)code_of(scaled(W[r * C + 2 * j + 1], delta[r]));
            packed[r * (C / 2) + j] = (uint8_t)((lo & 0xF) | ((hi & 0xF) << 4));
        }
        _Float16 h = (_Float16)delta[r];
        uint16_t bits;
        memcpy(&bits, &h, sizeof bits);
        scale16[r] = bits;
    }
}

/* Per-channel scale search: the model card's objective
 * Delta* = argmin ||W X - Q_Delta(W) X||_F^2 with one scale per row r, over the
 * grid Delta_k = alpha_k * (max_c |w_rc| / 7).  The row's objective is the
 * full quadratic form e H e^T, e = w_r - Q_{Delta_k}(w_r) (exact difference),
 * summed in binary64 over all C x C entries of H (row stride ldh).
 * Outputs per row [R]: delta, idx (smallest k on ties), best_err; all_err
 * (nullable) [R, K]. */
void oracle_scale_search_rowwise(const float *W, int64_t R, int64_t C,
                                 const float *H, int64_t ldh,
                                 const float *alpha, int32_t K,
                                 float *delta_out, int32_t *idx_out, double *best_err,
                                 double *all_err)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        const float *w = W + r * C;
        float m = 0.0f;
        for (int64_t i = 0; i < C; ++i) {
            float a = fabsf(w[i]);
            if (a > m) m = a;
        }
        float base = m / 7.0f;
        double *e = (double *)__builtin_alloca((size_t)C * sizeof(double));
        int32_t best_k = -1;
        double best = 0.0;
        float best_delta = 0.0f;
        for (int32_t k = 0; k < K; ++k) {
            float dk = alpha[k] * base;
            for (int64_t i = 0; i < C; ++i) e[i] = (double)w[i] - (double)fake_quant(w[i], dk);
            double E = 0.0;
            for (int64_t i = 0; i < C; ++i)
                for (int64_t j = 0; j < C; ++j)
                    E += e[i] * (double)H[i * ldh + j] * e[j];
            if (all_err) all_err[r * K + k] = E;
            if (best_k < 0 || E < best) {
                best = E;
                best_k = k;
                best_delta = dk;
            }
        }
        delta_out[r] = best_delta;
        idx_out[r] = best_k;
        best_err[r] = best;
    }
}

/* ------------------------------------------------------ W4A16 inference GEMV
 * The consumer of the export ([card] "Quantization Configuration": W4A16,
 * INT4 weights with 16-bit activations; "QAT Highlights": the same grid at
 * export): y[m, r] = sum_c x[m, c] * (scale[r, c / group] * code[r, c]), with
 * the binary16 scale and the 4-bit code of the packed layout (element 2j in the
 * low nibble of byte j), x in bf16, products and sums in binary64.
 * x: bf16 bits [M, C]; packed: uint8 [R, C/2]; scales: binary16 bits
 * [R, C/group]; y: double [M, R]. */
void oracle_w4a16_gemv(const uint16_t *x, const uint8_t *packed, const uint16_t *scales,
                       int64_t M, int64_t R, int64_t C, int64_t group, double *y)
{
    const int64_t G = C / group;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r) {
        for (int64_t m = 0; m < M; ++m) {
            double s = 0.0;
            for (int64_t c = 0; c < C; ++c) {
                uint8_t byte = packed[r * (C / 2) + c / 2];
                int nib = (c % 2 == 0) ? (byte & 0xF) : (byte >> 4);
                int code = nib >= 8 ? nib - 16 : nib;
                _Float16 h;
                uint16_t hb = scales[r * G + c / group];
                memcpy(&h, &hb, sizeof h);
                double w = (double)(float)h * (double)code;
                s += (double)bf16_to_float(x[m * C + c]) * w;
            }
            y[m * R + r] = s;
        }
    }
}

/* --------------------------------------------- fake-quant forward GEMM (QAT)
 * The forward of a quantized linear layer in a QAT step ([blog] section 3
 * "LSQ-based QAT": the forward pass runs on the weights projected onto the
 * INT4 grid that deployment uses): Y = X * Qb^T with Q = Q_Delta(W) in binary32
 * (as oracle_lsq_fwd) and Qb = Q rounded to bf16, round-to-nearest-even -- the
 * operand precision of a bf16 matrix multiply, which the pages leave implicit
 * (plainest reading: the usual bf16 mixed-precision forward).  Products and
 * sums in binary64.
 * X: bf16 bits [T, C]; W: float [R, C]; delta: float [R, C/32]; Y: double [T, R]. */

/* float -> bf16 bits, round to nearest, ties to even (finite inputs only). */
static uint16_t float_to_bf16_rne(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

static double fq_operand(const float *W, const float *delta, int64_t C, int64_t r, int64_t c)
{
    float q = fake_quant(W[r * C + c], delta[r * (C / GROUP) + c / GROUP]);
    return (double)bf16_to_float(float_to_bf16_rne(q));
}

void oracle_fq_gemm(const uint16_t *X, const float *W, const float *delta,
                    int64_t T, int64_t R, int64_t C, double *Y)
{
    double *Qb = (double *)malloc((size_t)(R * C) * sizeof(double));
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < R; ++r)
        for (int64_t c = 0; c < C; ++c) Qb[r * C + c] = fq_operand(W, delta, C, r, c);
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        for (int64_t r = 0; r < R; ++r) {
            double s = 0.0;
            for (int64_t c = 0; c < C; ++c) s += (double)bf16_to_float(X[t * C + c]) * Qb[r * C + c];
            Y[t * R + r] = s;
        }
    }
    free(Qb);
}

/* Selected entries Y[tt[m], rr[m]] of the same product (for sampled checks of
 * full-size outputs); out[m] in binary64. */
void oracle_fq_gemm_entries(const uint16_t *X, const float *W, const float *delta, int64_t C,
                            int64_t nsel, const int64_t *tt, const int64_t *rr, double *out)
{
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < nsel; ++m) {
        double s = 0.0;
        for (int64_t c = 0; c < C; ++c)
            s += (double)bf16_to_float(X[tt[m] * C + c]) * fq_operand(W, delta, C, rr[m], c);
        out[m] = s;
    }
}

/* -------------------------------------------- full-objective refinement
 * The model card ("Quantization Configuration") writes the objective over the
 * whole layer, Delta* = argmin ||W X - Q_Delta(W) X||_F^2, i.e. per row of W
 * the quadratic form e H e^T of e = w - Q_Delta(w) over all C columns.  The
 * search above keeps only the diagonal 32x32 blocks of H (each group on its
 * own).  This refinement starts from given candidate indices (the search's)
 * and runs `sweeps` passes of coordinate descent: groups in order g = 0..G-1,
 * each set to the candidate of its own grid (Delta_k = alpha_k * fl(m/7), as in
 * the search) that minimises the full objective with every other group held
 * at its current scale; ties go to the smallest k.  Every candidate's
 * objective is evaluated in full (all C x C terms, binary64, e exact).
 * W: float [R, C]; H: float, row stride ldh; alpha [K];
 * idx_io: int32 [R, C/32], start indices in, refined indices out;
 * delta_out: float [R, C/32]; obj_out: double [R], final objective. */
static double full_objective(const double *e, const float *H, int64_t ldh, int64_t C)
{
    double E = 0.0;
    for (int64_t i = 0; i < C; ++i) {
        double row = 0.0;
        for (int64_t j = 0; j < C; ++j) row += (double)H[i * ldh + j] * e[j];
        E += e[i] * row;
    }
    return E;
}

static void group_error(const float *w, float dk, double *e)
{
    for (int i = 0; i < GROUP; ++i) e[i] = (double)w[i] - (double)fake_quant(w[i], dk);
}

static float group_base(const float *w)
{
    float m = 0.0f;
    for (int i = 0; i < GROUP; ++i) {
        float a = fabsf(w[i]);
        if (a > m) m = a;
    }
    return m / 7.0f;
}

void oracle_refine(const float *W, int64_t R, int64_t C, const float *H, int64_t ldh,
                   const float *alpha, int32_t K, int32_t sweeps,
                   int32_t *idx_io, float *delta_out, double *obj_out)
{
    const int64_t G = C / GROUP;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        const float *w = W + r * C;
        int32_t *idx = idx_io + r * G;
        double *e = (double *)malloc((size_t)C * sizeof(double));
        for (int64_t g = 0; g < G; ++g)
            group_error(w + g * GROUP, alpha[idx[g]] * group_base(w + g * GROUP), e + g * GROUP);
        for (int32_t s = 0; s < sweeps; ++s) {
            for (int64_t g = 0; g < G; ++g) {
                const float base = group_base(w + g * GROUP);
                int32_t best_k = -1;
                double best = 0.0;
                for (int32_t k = 0; k < K; ++k) {
                    group_error(w + g * GROUP, alpha[k] * base, e + g * GROUP);
                    const double E = full_objective(e, H, ldh, C);
                    if (best_k < 0 || E < best) {
                        best = E;
                        best_k = k;
                    }
                }
                idx[g] = best_k;
                group_error(w + g * GROUP, alpha[best_k] * base, e + g * GROUP);
            }
        }
        for (int64_t g = 0; g < G; ++g) delta_out[r * G + g] = alpha[idx[g]] * group_base(w + g * GROUP);
        obj_out[r] = full_objective(e, H, ldh, C);
        free(e);
    }
}

/* One sweep replayed with given choices, for checking another implementation's
 * sweep: start from idx_start and, for g = 0..G-1 in order, evaluate every
 * candidate of group g in full (other groups: idx_pick for groups < g,
 * idx_start for groups > g), report the minimum (emin) and the objective at
 * idx_pick[g] (epick), then move group g to idx_pick[g].  Outputs [R, C/32]. */
void oracle_refine_replay(const float *W, int64_t R, int64_t C, const float *H, int64_t ldh,
                          const float *alpha, int32_t K, const int32_t *idx_start,
                          const int32_t *idx_pick, double *emin, double *epick)
{
    const int64_t G = C / GROUP;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < R; ++r) {
        const float *w = W + r * C;
        double *e = (double *)malloc((size_t)C * sizeof(double));
        for (int64_t g = 0; g < G; ++g)
            group_error(w + g * GROUP, alpha[idx_start[r * G + g]] * group_base(w + g * GROUP), e + g * GROUP);
        for (int64_t g = 0; g < G; ++g) {
            const float base = group_base(w + g * GROUP);
            const int32_t pick = idx_pick[r * G + g];
            double best = 0.0, at_pick = 0.0;
            for (int32_t k = 0; k < K; ++k) {
                group_error(w + g * GROUP, alpha[k] * base, e + g * GROUP);
                const double E = full_objective(e, H, ldh, C);
                if (k == 0 || E < best) best = E;
                if (k == pick) at_pick = E;
            }
            emin[r * G + g] = best;
            epick[r * G + g] = at_pick;
            group_error(w + g * GROUP, alpha[pick] * base, e + g * GROUP);
        }
        free(e);
    }
}
