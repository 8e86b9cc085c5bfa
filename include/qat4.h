/*
 * qat4.h -- C ABI of libqat4, a B200 (sm_100a) implementation of the
 * group-32 symmetric INT4 weight quantizer used for quantization-aware
 * training with a W4A16 export:
 *
 *   (a) calibration Hessian            H = X^T X / n
 *   (b) Hessian-weighted scale search  Delta* = argmin over a grid of
 *                                      e H_gg e^T, e = w_g - Q_Delta(w_g)
 *   (c) LSQ fake-quant forward         Q = Delta * clamp(rint(w / Delta), -8, 7)
 *       LSQ backward                   straight-through grad to W, step grad to Delta
 *       W4A16 export                   4-bit codes + binary16 scales
 *
 * Sources: the model card "Opt.Gear-1B-qat-int4-per-channel-unquantized"
 * (section "Quantization Configuration": symmetric INT4 with zero-point 0,
 * and the per-group objective Delta* = argmin ||W X - Q_Delta(W) X||_F^2;
 * section "QAT Highlights": group size 32 and one grid for initialisation,
 * QAT and export) and the blog post "Opt.Gear-QAT: Preserving On-Device
 * Performance with QAT" (section "Quantization parameters of Opt.Gear-1B":
 * one scale per 32 weights; section 2 "Hessian-based scale initialize";
 * section 3 "LSQ-based QAT").
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Data pointers are DEVICE pointers owned by the caller.  The library
 *    never allocates device or host memory and keeps no per-call state.
 *  - Matrices are row-major and dense (row stride = number of columns)
 *    unless a leading dimension is given.  A weight matrix W is [R, C]
 *    (R output rows, C input columns); group (r, g) is W[r, 32g : 32g+32],
 *    so C must be a positive multiple of 32.  Per-group arrays are
 *    [R, C/32] row-major.
 *  - Every call is asynchronous on `stream` (0 = legacy default stream).
 *    Argument errors are detected on the host before anything is launched
 *    and nothing is written; launch failures return QAT4_ERR_CUDA.
 *  - Pointers must be 16-byte aligned (QAT4_ERR_ALIGN otherwise).
 *  - Inputs are assumed finite.  Delta = 0 is allowed (it only arises for an
 *    all-zero group): such a group quantizes to 0, its weight gradient is G
 *    and its step gradient is 0.
 *  - Rounding: w / Delta is an IEEE binary32 division, round() is
 *    round-half-to-even, Delta * q is one binary32 multiply; integer codes,
 *    Q, grad_W and packed bytes are therefore exactly reproducible.
 */
#ifndef QAT4_H
#define QAT4_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QAT4_OK = 0,
    QAT4_ERR_NULL = 1,       /* a required pointer is NULL */
    QAT4_ERR_SHAPE = 2,      /* R, C, n or K out of range, C % 32 != 0, ldh < C */
    QAT4_ERR_ALIGN = 3,      /* a pointer is not 16-byte aligned */
    QAT4_ERR_DTYPE = 4,      /* unknown qat4_dtype */
    QAT4_ERR_WORKSPACE = 5,  /* workspace missing or smaller than required */
    QAT4_ERR_CUDA = 6,       /* a CUDA runtime/driver call or a launch failed */
    QAT4_ERR_TIMEOUT = 7     /* a kernel gave up a bounded wait (see qat4_sync_check) */
} qat4_status;

typedef enum { QAT4_F32 = 0, QAT4_BF16 = 1 } qat4_dtype;

/* Human-readable name of a status code (static storage, never NULL). */
const char *qat4_status_string(qat4_status status);

/* ABI version of this header (incremented on incompatible changes). */
int qat4_abi_version(void);

/* ---------------------------------------------------------------- (a)
 * Calibration Hessian H = X^T X / n  (blog section 2: layer sensitivity
 * from calibration inputs, the second-order output-reconstruction view).
 *
 *  X          bf16 bit patterns, [n, C] row-major (n calibration tokens).
 *  n          1 <= n <= 2^31 - 1.
 *  C          number of input channels, multiple of 32, 32 <= C <= 65536.
 *  H          float32 [C, C] row-major, written in full (both triangles,
 *             bitwise symmetric).  Products are exact, sums are float32 on
 *             the tensor cores (bf16 x bf16 -> fp32), scaled by 1/n.
 *  workspace  device scratch of at least qat4_hessian_workspace_bytes(n, C)
 *             bytes (may be NULL when that is 0); contents on entry are
 *             ignored.  The result does not depend on the device's SM count.
 *  Errors: QAT4_ERR_NULL, _SHAPE, _ALIGN, _WORKSPACE, _CUDA.  A bounded
 *  wait that gives up inside the kernel is reported by qat4_sync_check.
 */
size_t qat4_hessian_workspace_bytes(int64_t n, int64_t C);
qat4_status qat4_hessian(const uint16_t *X, int64_t n, int64_t C, float *H,
                         void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* One rank's share of a Hessian whose calibration rows are split across GPUs:
 * H = X^T X / n_total over the n rows of X (n <= n_total), everything else as
 * qat4_hessian (same workspace size for the same n and C).  Summing the
 * partials of all shards (an all-reduce) gives X_all^T X_all / n_total:
 * the split-n form of the exchange step of the Hessian on several GPUs. */
qat4_status qat4_hessian_partial(const uint16_t *X, int64_t n, int64_t C, int64_t n_total, float *H,
                                 void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------- (b)
 * Hessian-weighted per-group scale search (model card, "Quantization
 * Configuration": Delta* = argmin ||W X - Q_Delta(W) X||_F^2 per group,
 * read block-diagonally: each group minimises e H_gg e^T with the other
 * groups at zero error; blog section 2).
 *
 *  W         float32 [R, C].
 *  H         float32, row stride ldh >= C; only the C/32 diagonal 32x32
 *            blocks H[32g:32g+32, 32g:32g+32] are read.  H must be
 *            symmetric positive semi-definite for the exact-argmin
 *            guarantee below (any Hessian from qat4_hessian is).
 *  alpha     float32 [K], K >= 1: candidate multipliers.  Candidate k of
 *            group (r, g) is Delta_k = fl(alpha[k] * fl(max|w_g| / 7)).
 *  delta     out float32 [R, C/32]: the chosen Delta_k.
 *  idx       out int32   [R, C/32]: the chosen k (smallest k on exact ties).
 *  best_err  out float32 [R, C/32] (may be NULL): e H_gg e^T at the chosen k,
 *            rounded to float32 from a float64 evaluation.
 *  Every candidate is screened on the tensor cores (e H e^T with the error
 *  vector in binary16 and H split into two binary16 parts, float32 sums)
 *  together with a rigorous rounding-error bound; the candidates that the
 *  bound cannot separate from the minimum are re-scored in float64, so idx
 *  equals the argmin of the float64 objective except for candidates whose
 *  objectives agree to ~1e-15.
 *  Errors: QAT4_ERR_NULL, _SHAPE, _ALIGN, _CUDA.
 */
qat4_status qat4_scale_search(const float *W, int64_t R, int64_t C,
                              const float *H, int64_t ldh,
                              const float *alpha, int32_t K,
                              float *delta, int32_t *idx, float *best_err,
                              cudaStream_t stream);

/* ---------------------------------------------------------------- (c)
 * LSQ fake-quant forward (blog section 3: the forward pass emulates the
 * deployment INT4 grid):  Q = Delta * clamp(rint(w / Delta), -8, 7).
 *
 *  W      float32 [R, C];  delta float32 [R, C/32];  Q out float32 [R, C].
 *  Errors: QAT4_ERR_NULL, _SHAPE, _ALIGN, _CUDA.
 */
qat4_status qat4_lsq_fwd(const float *W, const float *delta, int64_t R, int64_t C,
                         float *Q, cudaStream_t stream);

/* LSQ backward (blog section 3: straight-through estimator for round; the
 * step-size gradient normalised by the group's element count and the
 * number of positive levels; Esser et al., "Learned Step Size
 * Quantization", ICLR 2020).  With v = w / Delta:
 *    grad_W     = G                       if -8 <= v <= 7, else 0
 *    dQ/dDelta  = rint(v) - v             if -8 <  v <  7
 *               = -8 if v <= -8,  7 if v >= 7
 *    grad_delta = grad_scale * sum over the group of G * dQ/dDelta
 *  G           [R, C], float32 (QAT4_F32) or bf16 bit patterns (QAT4_BF16).
 *  grad_scale  normally 1/sqrt(32 * 7).
 *  grad_W      out float32 [R, C];  grad_delta out float32 [R, C/32]
 *              (overwritten, not accumulated).
 *  Errors: QAT4_ERR_NULL, _SHAPE, _ALIGN, _DTYPE, _CUDA.
 */
qat4_status qat4_lsq_bwd(const float *W, const float *delta, const void *G, qat4_dtype g_dtype,
                         int64_t R, int64_t C, float grad_scale,
                         float *grad_W, float *grad_delta, cudaStream_t stream);

/* Forward and backward in one pass over W and G (the outputs of
 * qat4_lsq_fwd and qat4_lsq_bwd, bit-identical Q and grad_W). */
qat4_status qat4_lsq_fwd_bwd(const float *W, const float *delta, const void *G, qat4_dtype g_dtype,
                             int64_t R, int64_t C, float grad_scale,
                             float *Q, float *grad_W, float *grad_delta, cudaStream_t stream);

/* LSQ step of a whole layer from and to HOST memory (the blog's QAT step on
 * weights that live on the host): the rows are streamed through the GPU in
 * chunks of about 2 M weights, each chunk uploaded on `stream`, run through
 * the fused forward/backward kernel, and downloaded on `copy_stream`, so the
 * uploads of one chunk overlap the downloads of the previous one (PCIe is
 * full duplex).  Results are identical to qat4_lsq_fwd_bwd on the same data.
 *
 *  W, delta, G, Q, grad_W, grad_delta   HOST pointers with the shapes and
 *            dtypes of qat4_lsq_fwd_bwd; page-locked memory is needed for the
 *            copies to overlap (pageable memory is correct but serialises).
 *  workspace DEVICE memory, 256-byte aligned, at least
 *            qat4_lsq_fwd_bwd_host_workspace_bytes(R, C, g_dtype) bytes
 *            (two chunks of every operand).
 *  stream, copy_stream   the call returns once everything is enqueued; when
 *            `stream` has completed (cudaStreamSynchronize), the outputs are
 *            on the host.  copy_stream may equal stream (then nothing overlaps).
 *  The call creates and releases five CUDA events per call; it allocates no
 *  memory.  Errors: QAT4_ERR_NULL, _SHAPE, _DTYPE, _WORKSPACE, _ALIGN (all
 *  before anything is enqueued) and _CUDA (a copy, launch or event call
 *  failed; the outputs are then incomplete, and `stream` still waits for the
 *  copies that were enqueued).
 */
size_t qat4_lsq_fwd_bwd_host_workspace_bytes(int64_t R, int64_t C, qat4_dtype g_dtype);
qat4_status qat4_lsq_fwd_bwd_host(const float *W, const float *delta, const void *G, qat4_dtype g_dtype,
                                  int64_t R, int64_t C, float grad_scale,
                                  float *Q, float *grad_W, float *grad_delta,
                                  void *workspace, size_t workspace_bytes,
                                  cudaStream_t stream, cudaStream_t copy_stream);

/* W4A16 export (model card, "QAT Highlights": the same INT4 grid at
 * initialisation, QAT and export).  Codes are the forward codes
 * clamp(rint(w / Delta), -8, 7) for the float32 Delta.
 *
 *  packed  out uint8 [R, C/2]: byte j of a row holds element 2j in its low
 *          nibble and element 2j+1 in its high nibble (4-bit two's complement).
 *  scales  out binary16 bit patterns [R, C/32]: Delta rounded to nearest even.
 *  Errors: QAT4_ERR_NULL, _SHAPE, _ALIGN, _CUDA.
 */
qat4_status qat4_pack_w4a16(const float *W, const float *delta, int64_t R, int64_t C,
                            uint8_t *packed, uint16_t *scales, cudaStream_t stream);

/* Same result as qat4_hessian, for callers that cannot allocate device memory
 * themselves -- for example code running inside an engine or framework that
 * owns all device memory through its own allocator or a fixed budget, or a
 * latency-critical loop where cudaMalloc/cudaFree (which may synchronise the
 * device) are not acceptable.  The pages describe no such variant; it has no
 * counterpart there.
 *
 *  X, n, C, H  as for qat4_hessian.  No workspace argument: the scratch is a
 *              static device array of 19,398,656 bytes (18.5 MiB) inside the
 *              library, which every GPU that loads the library holds until the
 *              process exits.  It covers every (n, C) the planner accepts;
 *              a shape that needed more would be rejected with
 *              QAT4_ERR_WORKSPACE.
 *  The call allocates nothing: no cudaMalloc, cudaFree or allocating library
 *  routine.  Its first call on a device (with that device current) looks up
 *  the array's device address once and keeps it; make that first call before
 *  any stream capture.  The kept address belongs to the device's context: the
 *  call compares the current context's id (cuCtxGetId) with the one the
 *  address was looked up in, and after cudaDeviceReset, whose next CUDA call
 *  runs in a new context, it looks the address up again -- so the first call
 *  after a reset is again a set-up call and must also come before any
 *  capture.  All calls on a device share the one array: two calls whose
 *  kernels overlap on the GPU (different streams, or other host threads)
 *  race on it and must be ordered by the caller.  Every byte of the scratch
 *  that is read is first written by the same call, so nothing from the
 *  previous call leaks into the result.
 *  Errors: QAT4_ERR_NULL, _SHAPE, _ALIGN, _WORKSPACE, _CUDA. */
qat4_status qat4_hessian_noalloc(const uint16_t *X, int64_t n, int64_t C, float *H, cudaStream_t stream);

/* ---------------------------------------------------------------- per-channel
 * The same quantizer with one scale per output row (model card
 * "Opt.Gear-1B-qat-int4-per-channel-unquantized": per-channel symmetric INT4
 * weights with learned channel-wise scales, W4A16 export).  Arguments as for
 * the group-32 calls, except that delta, grad_delta and scales hold one value
 * per row ([R]), the step gradient of a row sums all C weights, and the
 * normalisation passed in is normally grad_scale = 1/sqrt(C * 7).  The codes,
 * Q, grad_W and packed bytes equal those of the group-32 calls given the row's
 * scale in every group of the row.
 *  Errors: QAT4_ERR_NULL, _SHAPE, _ALIGN, _DTYPE (LSQ backward), _CUDA. */
qat4_status qat4_lsq_fwd_rowwise(const float *W, const float *delta, int64_t R, int64_t C,
                                 float *Q, cudaStream_t stream);
qat4_status qat4_lsq_bwd_rowwise(const float *W, const float *delta, const void *G, qat4_dtype g_dtype,
                                 int64_t R, int64_t C, float grad_scale,
                                 float *grad_W, float *grad_delta, cudaStream_t stream);
qat4_status qat4_lsq_fwd_bwd_rowwise(const float *W, const float *delta, const void *G, qat4_dtype g_dtype,
                                     int64_t R, int64_t C, float grad_scale,
                                     float *Q, float *grad_W, float *grad_delta, cudaStream_t stream);
qat4_status qat4_pack_w4a16_rowwise(const float *W, const float *delta, int64_t R, int64_t C,
                                    uint8_t *packed, uint16_t *scales, cudaStream_t stream);

/* Per-channel scale search: for every row r and candidate
 * Delta_k = fl(alpha[k] * fl(max_c |W[r,c]| / 7)) the full quadratic form
 * E_k = e H e^T, e = w_r - Q_{Delta_k}(w_r) (exact difference), over all C x C
 * entries of H (model card objective with one scale per row).
 *  W          float32 [R, C], C <= 8192.
 *  H          float32 [C, C], row stride ldh >= C; must be symmetric.
 *  alpha, K   candidate multipliers, as for qat4_scale_search.
 *  delta, idx, best_err   out [R]; idx is the argmin of E_k (smallest k on
 *             ties); E_k is evaluated in binary64 (exact up to binary64
 *             rounding and a dropped term below 1e-14 relative).
 *  workspace  at least qat4_scale_search_rowwise_workspace_bytes(R, C) bytes
 *             (16 R C + 4 R, rounded up): H w and H q for every row.  Large
 *             matrices can be searched in row chunks to bound it.
 *  Errors: QAT4_ERR_NULL, _SHAPE (C > 8192, ldh < C, K < 1), _ALIGN,
 *  _WORKSPACE, _CUDA. */
size_t qat4_scale_search_rowwise_workspace_bytes(int64_t R, int64_t C);
qat4_status qat4_scale_search_rowwise(const float *W, int64_t R, int64_t C,
                                      const float *H, int64_t ldh,
                                      const float *alpha, int32_t K,
                                      float *delta, int32_t *idx, float *best_err,
                                      void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* ------------------------------------------------ full-objective refinement
 * The model card ("Quantization Configuration") writes the scale objective
 * over the whole layer, argmin ||W X - Q_Delta(W) X||_F^2: per row of W the
 * quadratic form e H e^T of e = w - Q_Delta(w) over all C columns, including
 * the cross-group blocks of H that qat4_scale_search leaves out.  Starting
 * from the given candidate indices (normally the search's), each of `sweeps`
 * passes visits the groups of a row in order and moves each to the candidate
 * of its own grid (Delta_k = alpha_k * fl(max|w_g| / 7)) that minimises the
 * full objective with the other groups held; ties go to the smallest k.  The
 * objective never increases.  Arithmetic: exact codes, exact binary64 errors,
 * binary64 objective differences (v = H e kept per row).
 *  W      float32 [R, C];  H float32 [C, C] (row stride ldh >= C, ldh % 4 == 0),
 *         symmetric (as qat4_hessian writes it);  alpha float32 [K].
 *  idx    int32 [R, C/32], in: start indices in [0, K) (others are clamped),
 *         out: refined indices.
 *  delta  out float32 [R, C/32]: alpha[idx] * fl(max|w_g| / 7).
 *  obj    out float64 [R] (nullable): the final e H e^T of every row.
 *  workspace  >= qat4_refine_workspace_bytes(R, C) bytes (2 R C binary64).
 *  sweeps >= 0 (0 only evaluates the start).
 *  Errors: QAT4_ERR_NULL, _SHAPE, _ALIGN, _WORKSPACE, _CUDA. */
size_t qat4_refine_workspace_bytes(int64_t R, int64_t C);
qat4_status qat4_refine(const float *W, int64_t R, int64_t C, const float *H, int64_t ldh, const float *alpha,
                        int32_t K, int32_t sweeps, int32_t *idx, float *delta, double *obj, void *workspace,
                        size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------- inference
 * The product on the W4A16 export (model card "Opt.Gear-1B-qat-int4-per-
 * channel-unquantized", section "Quantization Configuration": INT4 weights,
 * 16-bit activations), for decode-sized batches:
 *     y[m, r] = sum_c x[m, c] * (scale[r, c / group] * code[r, c])
 *  x       bf16 bit patterns [M, C] (M tokens, 1 <= M <= 65535; processed up to eight
 *          tokens per pass -- fewer when x of a wide row does not fit shared memory -- so
 *          the codes are read once per pass).
 *  packed  uint8 [R, C/2], the layout of qat4_pack_w4a16 (element 2j in the low nibble of
 *          byte j, 4-bit two's complement).
 *  scales  binary16 bit patterns [R, C/group]: group = 32 for the export of
 *          qat4_pack_w4a16, group = C for qat4_pack_w4a16_rowwise (any multiple of 32 that
 *          divides C is accepted).
 *  y       out float32 [M, R]; zeroed on the stream first, then written.  Products are
 *          exact (bf16 codes times bf16 x on the tensor cores), sums float32 in an order
 *          fixed by (R, C, M) and the SM count.
 *  C must be a multiple of 32 and small enough that one token's x (bf16) and three 16 KB
 *  stages fit the opt-in shared memory of a block (C <= 88064 on B200); else _SHAPE.
 *  Errors: QAT4_ERR_NULL, _SHAPE, _ALIGN, _CUDA. */
qat4_status qat4_w4a16_gemv(const uint16_t *x, int64_t M, const uint8_t *packed, const uint16_t *scales,
                            int64_t R, int64_t C, int64_t group, float *y, cudaStream_t stream);

/* ------------------------------------------------ fake-quant forward GEMM
 * The forward of a quantized linear layer in a QAT step (blog "Opt.Gear-QAT",
 * section 3 "LSQ-based QAT": the forward pass runs on the weights projected
 * onto the deployment INT4 grid), with the quantizer fused into the GEMM:
 *     Y[t, r] = sum_c X[t, c] * bf16(Q_Delta(W)[r, c])
 *  X      bf16 bit patterns [T, C], row-major (T tokens).
 *  W      float32 [R, C], delta float32 [R, C/32]: Q_Delta(w) = Delta *
 *         clamp(rint(w / Delta), -8, 7) exactly as qat4_lsq_fwd computes it,
 *         then rounded to bf16 to nearest even (the operand precision of a bf16
 *         forward); products exact, sums float32 on the tensor cores.
 *  Y      out float32 [T, R], row-major.
 *  C must be a multiple of 32; T, R >= 1.  Pointers 16-byte aligned.
 *  Errors: QAT4_ERR_NULL, _SHAPE, _ALIGN, _CUDA; a bounded wait that gives up
 *  leaves QAT4_ERR_TIMEOUT for qat4_sync_check. */
qat4_status qat4_fq_gemm(const uint16_t *X, int64_t T, const float *W, const float *delta, int64_t R, int64_t C,
                         float *Y, cudaStream_t stream);

/* The same product in two kernels: the quantizer writes bf16(Q_Delta(W))
 * (the same values the fused call forms in shared memory) into `workspace`,
 * then a persistent tcgen05 GEMM computes Y = X * Qb^T.  Arguments as for
 * qat4_fq_gemm, plus
 *  workspace  device scratch of at least
 *             qat4_fq_gemm_staged_workspace_bytes(R, C) bytes (R * C bf16,
 *             rounded up to 256), 256-byte aligned; contents on entry are
 *             ignored, on return it holds bf16(Q_Delta(W)) [R, C].
 *  Same result as qat4_fq_gemm up to the order of the float32 sums.
 *  Errors: QAT4_ERR_NULL, _SHAPE, _ALIGN, _WORKSPACE, _CUDA; a bounded wait
 *  that gives up leaves QAT4_ERR_TIMEOUT for qat4_sync_check. */
size_t qat4_fq_gemm_staged_workspace_bytes(int64_t R, int64_t C);
qat4_status qat4_fq_gemm_staged(const uint16_t *X, int64_t T, const float *W, const float *delta, int64_t R,
                                int64_t C, float *Y, void *workspace, size_t workspace_bytes, cudaStream_t stream);

/* Synchronises `stream`, then reads and clears the library's device error
 * word for the current device.  Returns QAT4_ERR_TIMEOUT if a kernel gave up
 * a bounded wait since the last check, QAT4_ERR_CUDA if synchronisation
 * failed, QAT4_OK otherwise. */
qat4_status qat4_sync_check(cudaStream_t stream);

/* Exercises the bounded-wait path: launches one tiny kernel that waits on a
 * barrier which nothing ever completes, for at most limit_ns nanoseconds
 * (1 <= limit_ns <= 10^10), after which it records a timeout in the device
 * error word and returns.  qat4_sync_check then returns QAT4_ERR_TIMEOUT. */
qat4_status qat4_selftest_bounded_wait(int64_t limit_ns, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* QAT4_H */
