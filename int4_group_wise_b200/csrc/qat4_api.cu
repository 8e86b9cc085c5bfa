// qat4_api.cu -- the C ABI of libqat4 (declared in include/qat4.h): argument
// validation on the host, launch configuration, and the device error word.
// All kernels live in the headers included below; this is the only
// translation unit of the library.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "../../include/qat4.h"
#include "device_common.cuh"
#include "hessian.cuh"
#include "lsq_pack.cuh"
#include "scale_search.cuh"
#include "rowwise.cuh"
#include "rowwise_search.cuh"
#include "w4a16_gemv.cuh"
#include "fq_gemm.cuh"
#include "fq_staged.cuh"
#include "refine.cuh"

namespace {

constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool valid_rc(int64_t R, int64_t C) {
    return R >= 1 && C >= 32 && (C % 32) == 0 && R <= (int64_t(1) << 31) - 1 &&
           C <= (int64_t(1) << 31) - 1 && R * C <= (int64_t(1) << 40);
}

struct DeviceInfo {
    unsigned long long ctx_id = 0;   // context the cached set-up below belongs to
    int sms = 0;
    bool hessian_attr = false;
    bool search_attr = false;
    bool rowsearch_attr = false;
    int smem_optin = 0;       // opt-in shared memory per block; gemv attributes set when > 0
    bool fq_attr = false;
    bool gemm_attr = false;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mutex;

// Unique id of the calling thread's current CUDA context (the driver never
// reuses one within a process), or 0 if it cannot be read.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

unsigned long long current_ctx_id() {
    static std::once_flag once;
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    if (!get_current || !get_id) return 0;
    CUcontext c = nullptr;
    unsigned long long id = 0;
    if (get_current(&c) != CUDA_SUCCESS || c == nullptr || get_id(c, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// Current device and its cached set-up (SM count, kernel attributes); false on
// any CUDA error.  The set-up is tied to the device's context: when the context
// has changed since it was made (cudaDeviceReset destroys the primary context,
// and the next call runs in a new one), it is dropped and made again.
bool device_info(int* dev_out, DeviceInfo** info) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    unsigned long long ctx = current_ctx_id();
    if (ctx == 0) {   // no context current yet: cudaSetDevice creates and binds it
        if (cudaSetDevice(dev) != cudaSuccess) return false;
        ctx = current_ctx_id();
    }
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo& d = g_dev[dev];
    if (ctx != 0 && ctx != d.ctx_id) {
        d = DeviceInfo{};
        d.ctx_id = ctx;
    }
    if (d.sms == 0) {
        int sms = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
            return false;
        d.sms = sms;
    }
    *dev_out = dev;
    *info = &d;
    return true;
}

qat4_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? QAT4_OK : QAT4_ERR_CUDA;
}

// --------------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

}  // namespace

extern "C" {

const char* qat4_status_string(qat4_status s) {
    switch (s) {
        case QAT4_OK: return "QAT4_OK";
        case QAT4_ERR_NULL: return "QAT4_ERR_NULL: a required pointer is NULL";
        case QAT4_ERR_SHAPE: return "QAT4_ERR_SHAPE: size out of range or C not a multiple of 32";
        case QAT4_ERR_ALIGN: return "QAT4_ERR_ALIGN: pointer not 16-byte aligned";
        case QAT4_ERR_DTYPE: return "QAT4_ERR_DTYPE: unknown gradient dtype";
        case QAT4_ERR_WORKSPACE: return "QAT4_ERR_WORKSPACE: workspace missing or too small";
        case QAT4_ERR_CUDA: return "QAT4_ERR_CUDA: a CUDA call or kernel launch failed";
        case QAT4_ERR_TIMEOUT: return "QAT4_ERR_TIMEOUT: a kernel gave up a bounded wait";
    }
    return "QAT4_ERR_UNKNOWN";
}

int qat4_abi_version(void) { return 1; }

// ------------------------------------------------------------------ Hessian
size_t qat4_hessian_workspace_bytes(int64_t n, int64_t C) {
    if (n < 1 || C < 32 || C % 32 != 0 || C > 65536) return 0;
    const qat4::HessPlan plan = qat4::hess_plan(n, C);
    if (plan.split <= 1) return 0;
    return static_cast<size_t>(plan.tiles - plan.split0) * plan.split * qat4::kPTile * qat4::kPTile * sizeof(float);
}

}  // extern "C"

namespace {

// H = X^T X / n_norm over the n rows of X (n_norm = n for the Hessian itself).
qat4_status hessian_run(const uint16_t* X, int64_t n, int64_t C, int64_t n_norm, float* H, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
    if (!X || !H) return QAT4_ERR_NULL;
    if (n < 1 || n > (int64_t(1) << 31) - 1 || C < 32 || C % 32 != 0 || C > 65536 || n_norm < 1)
        return QAT4_ERR_SHAPE;
    if (!aligned16(X) || !aligned16(H) || (workspace && !aligned16(workspace))) return QAT4_ERR_ALIGN;
    const size_t need = qat4_hessian_workspace_bytes(n, C);
    if (workspace_bytes < need || (need > 0 && !workspace)) return QAT4_ERR_WORKSPACE;

    int dev;
    DeviceInfo* info;
    if (!device_info(&dev, &info)) return QAT4_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!info->hessian_attr) {
            if (cudaFuncSetAttribute(qat4::hessian_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(qat4::kPSmemBytes)) != cudaSuccess)
                return QAT4_ERR_CUDA;
            info->hessian_attr = true;
        }
    }
    EncodeTiledFn encode = encode_tiled();
    if (!encode) return QAT4_ERR_CUDA;

    CUtensorMap tmap;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(n)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(C) * 2};
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(qat4::kPBK)};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return QAT4_ERR_CUDA;

    qat4::HessParams p;
    p.n = n;
    p.C = static_cast<int>(C);
    p.plan = qat4::hess_plan(n, C);
    p.inv_n = static_cast<float>(1.0 / static_cast<double>(n_norm));
    // generous bound: 4 s plus 100 ns per calibration row (a chunk of the
    // mainloop takes ~2 ns per row at full rate)
    p.limit_ns = 4000000000ull + 100ull * static_cast<uint64_t>(n);
    const unsigned ctas = 2u * static_cast<unsigned>(p.plan.units);
    qat4::hessian_pair_kernel<<<ctas, qat4::kPThreads, qat4::kPSmemBytes, stream>>>(
        tmap, p, H, static_cast<float*>(workspace));
    if (cudaGetLastError() != cudaSuccess) return QAT4_ERR_CUDA;
    if (p.plan.split > 1) {   // the tiles cut into parts
        const dim3 grid(static_cast<unsigned>(p.plan.tiles - p.plan.split0), 64);
        qat4::hessian_reduce_kernel<<<grid, 256, 0, stream>>>(static_cast<const float*>(workspace), p, H);
    }
    return launch_status();
}

}  // namespace

extern "C" {

qat4_status qat4_hessian(const uint16_t* X, int64_t n, int64_t C, float* H,
                         void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    return hessian_run(X, n, C, n, H, workspace, workspace_bytes, stream);
}

qat4_status qat4_hessian_partial(const uint16_t* X, int64_t n, int64_t C, int64_t n_total, float* H,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (n_total < n) return QAT4_ERR_SHAPE;
    return hessian_run(X, n, C, n_total, H, workspace, workspace_bytes, stream);
}

// -------------------------------------------------------------- scale search
qat4_status qat4_scale_search(const float* W, int64_t R, int64_t C, const float* H, int64_t ldh,
                              const float* alpha, int32_t K, float* delta, int32_t* idx,
                              float* best_err, cudaStream_t stream) {
    if (!W || !H || !alpha || !delta || !idx) return QAT4_ERR_NULL;
    if (!valid_rc(R, C) || K < 1 || ldh < C || C / 32 > 65535) return QAT4_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(H) || !aligned16(alpha) || !aligned16(delta) || !aligned16(idx) ||
        (best_err && !aligned16(best_err)) || (ldh % 4) != 0)
        return QAT4_ERR_ALIGN;
    int dev;
    DeviceInfo* info;
    if (!device_info(&dev, &info)) return QAT4_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!info->search_attr) {
            if (cudaFuncSetAttribute(qat4::scale_search_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(qat4::kTcSmemBytes)) != cudaSuccess)
                return QAT4_ERR_CUDA;
            info->search_attr = true;
        }
    }
    const dim3 grid(static_cast<unsigned>((R + qat4::kTcRows - 1) / qat4::kTcRows), static_cast<unsigned>(C / 32));
    // each wait covers one candidate's four small MMAs; the limit only catches a tensor core that never answers
    qat4::scale_search_kernel<4><<<grid, qat4::kTcRows, qat4::kTcSmemBytes, stream>>>(
        W, static_cast<int>(R), static_cast<int>(C), H, ldh, alpha, K, delta, idx, best_err, 4000000000ull);
    return launch_status();
}

// ---------------------------------------------------------------------- LSQ
static qat4_status lsq_common(const float* W, const float* delta, const void* G, qat4_dtype g_dtype,
                              int64_t R, int64_t C, float grad_scale, float* Q, float* grad_W,
                              float* grad_delta, bool fwd, bool bwd, cudaStream_t stream) {
    if (!W || !delta || (fwd && !Q) || (bwd && (!G || !grad_W || !grad_delta))) return QAT4_ERR_NULL;
    if (!valid_rc(R, C)) return QAT4_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(delta) || (fwd && !aligned16(Q)) ||
        (bwd && (!aligned16(G) || !aligned16(grad_W) || !aligned16(grad_delta))))
        return QAT4_ERR_ALIGN;
    if (bwd && g_dtype != QAT4_F32 && g_dtype != QAT4_BF16) return QAT4_ERR_DTYPE;
    int dev;
    DeviceInfo* info;
    if (!device_info(&dev, &info)) return QAT4_ERR_CUDA;
    // short 128-thread blocks, two quads per thread, all loads issued up front; R * C <= 2^40
    // keeps the grid below 2^32 blocks
    const int64_t nquads = R * C / 4;
    constexpr int kU = 2;
    const unsigned blocks = static_cast<unsigned>((nquads + qat4::kLsqBlock * kU - 1) / (qat4::kLsqBlock * kU));
    const unsigned th = qat4::kLsqBlock;
    if (fwd && !bwd) {
        qat4::lsq_blocks_kernel<float, true, false, kU><<<blocks, th, 0, stream>>>(W, delta, nullptr, nquads, 0.f, Q,
                                                                                  nullptr, nullptr);
    } else if (g_dtype == QAT4_F32) {
        const float* g = static_cast<const float*>(G);
        if (fwd)
            qat4::lsq_blocks_kernel<float, true, true, kU><<<blocks, th, 0, stream>>>(W, delta, g, nquads, grad_scale,
                                                                                     Q, grad_W, grad_delta);
        else
            qat4::lsq_blocks_kernel<float, false, true, kU><<<blocks, th, 0, stream>>>(W, delta, g, nquads,
                                                                                      grad_scale, nullptr, grad_W,
                                                                                      grad_delta);
    } else {
        const uint16_t* g = static_cast<const uint16_t*>(G);
        if (fwd)
            qat4::lsq_blocks_kernel<uint16_t, true, true, kU><<<blocks, th, 0, stream>>>(W, delta, g, nquads,
                                                                                        grad_scale, Q, grad_W,
                                                                                        grad_delta);
        else
            qat4::lsq_blocks_kernel<uint16_t, false, true, kU><<<blocks, th, 0, stream>>>(W, delta, g, nquads,
                                                                                         grad_scale, nullptr, grad_W,
                                                                                         grad_delta);
    }
    return launch_status();
}

qat4_status qat4_lsq_fwd(const float* W, const float* delta, int64_t R, int64_t C, float* Q,
                         cudaStream_t stream) {
    return lsq_common(W, delta, nullptr, QAT4_F32, R, C, 0.f, Q, nullptr, nullptr, true, false, stream);
}

qat4_status qat4_lsq_bwd(const float* W, const float* delta, const void* G, qat4_dtype g_dtype, int64_t R,
                         int64_t C, float grad_scale, float* grad_W, float* grad_delta,
                         cudaStream_t stream) {
    return lsq_common(W, delta, G, g_dtype, R, C, grad_scale, nullptr, grad_W, grad_delta, false, true,
                      stream);
}

qat4_status qat4_lsq_fwd_bwd(const float* W, const float* delta, const void* G, qat4_dtype g_dtype,
                             int64_t R, int64_t C, float grad_scale, float* Q, float* grad_W,
                             float* grad_delta, cudaStream_t stream) {
    return lsq_common(W, delta, G, g_dtype, R, C, grad_scale, Q, grad_W, grad_delta, true, true, stream);
}

// --------------------------------------------------------------------- pack
qat4_status qat4_pack_w4a16(const float* W, const float* delta, int64_t R, int64_t C, uint8_t* packed,
                            uint16_t* scales, cudaStream_t stream) {
    if (!W || !delta || !packed || !scales) return QAT4_ERR_NULL;
    if (!valid_rc(R, C)) return QAT4_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(delta) || !aligned16(packed) || !aligned16(scales)) return QAT4_ERR_ALIGN;
    int dev;
    DeviceInfo* info;
    if (!device_info(&dev, &info)) return QAT4_ERR_CUDA;
    // 128-thread blocks of 4 octets per thread; R * C <= 2^40 keeps the grid below 2^28 blocks
    const int64_t noct = R * C / 8;   // C % 32 == 0: octets never straddle a group
    constexpr int kU = 4;
    const int64_t blocks = (noct + qat4::kPackBlock * kU - 1) / (qat4::kPackBlock * kU);
    qat4::pack_w4a16_blocks_kernel<kU, false><<<static_cast<unsigned>(blocks), qat4::kPackBlock, 0, stream>>>(
        W, delta, noct, 4, 0.25, reinterpret_cast<uint32_t*>(packed), scales);
    return launch_status();
}

// ------------------------------------------------- LSQ step from host memory
// Rows per chunk of the host-buffer pipeline: about 2 M weights, at least one row.
static int64_t host_chunk_rows(int64_t R, int64_t C) {
    return std::max<int64_t>(1, std::min<int64_t>(R, (int64_t(1) << 21) / C));
}
static size_t host_chunk_bytes(int64_t rows, int64_t C, qat4_dtype g_dtype) {
    const int64_t n = rows * C;
    const size_t gb = g_dtype == QAT4_BF16 ? 2 : 4;
    // W, G, Q, grad_W, delta, grad_delta of one chunk, each rounded up to 256 bytes
    auto r256 = [](size_t b) { return (b + 255) & ~size_t(255); };
    return r256(n * 4) + r256(n * gb) + r256(n * 4) + r256(n * 4) + 2 * r256(n / 32 * 4);
}

size_t qat4_lsq_fwd_bwd_host_workspace_bytes(int64_t R, int64_t C, qat4_dtype g_dtype) {
    if (!valid_rc(R, C) || (g_dtype != QAT4_F32 && g_dtype != QAT4_BF16)) return 0;
    return 2 * host_chunk_bytes(host_chunk_rows(R, C), C, g_dtype);
}

qat4_status qat4_lsq_fwd_bwd_host(const float* W, const float* delta, const void* G, qat4_dtype g_dtype,
                                  int64_t R, int64_t C, float grad_scale, float* Q, float* grad_W,
                                  float* grad_delta, void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream, cudaStream_t copy_stream) {
    if (!W || !delta || !G || !Q || !grad_W || !grad_delta || !workspace) return QAT4_ERR_NULL;
    if (!valid_rc(R, C)) return QAT4_ERR_SHAPE;
    if (g_dtype != QAT4_F32 && g_dtype != QAT4_BF16) return QAT4_ERR_DTYPE;
    if (workspace_bytes < qat4_lsq_fwd_bwd_host_workspace_bytes(R, C, g_dtype)) return QAT4_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return QAT4_ERR_ALIGN;
    const int64_t crow = host_chunk_rows(R, C);
    const size_t gb = g_dtype == QAT4_BF16 ? 2 : 4;
    const size_t stage = host_chunk_bytes(crow, C, g_dtype);
    auto r256 = [](size_t b) { return (b + 255) & ~size_t(255); };
    struct Buf { float *w, *q, *gw, *d, *gd; void* g; };
    Buf buf[2];
    for (int b = 0; b < 2; ++b) {
        uint8_t* p = static_cast<uint8_t*>(workspace) + b * stage;
        const int64_t n = crow * C;
        buf[b].w = reinterpret_cast<float*>(p);            p += r256(n * 4);
        buf[b].g = p;                                       p += r256(n * gb);
        buf[b].q = reinterpret_cast<float*>(p);            p += r256(n * 4);
        buf[b].gw = reinterpret_cast<float*>(p);           p += r256(n * 4);
        buf[b].d = reinterpret_cast<float*>(p);            p += r256(n / 32 * 4);
        buf[b].gd = reinterpret_cast<float*>(p);
    }
    cudaEvent_t done[2] = {nullptr, nullptr}, freed[2] = {nullptr, nullptr}, last = nullptr;
    bool made = true;
    for (int b = 0; b < 2; ++b) {
        made = made && cudaEventCreateWithFlags(&done[b], cudaEventDisableTiming) == cudaSuccess;
        made = made && cudaEventCreateWithFlags(&freed[b], cudaEventDisableTiming) == cudaSuccess;
    }
    made = made && cudaEventCreateWithFlags(&last, cudaEventDisableTiming) == cudaSuccess;
    qat4_status st = made ? QAT4_OK : QAT4_ERR_CUDA;
    const auto H2D = cudaMemcpyHostToDevice;
    const auto D2H = cudaMemcpyDeviceToHost;
    int64_t chunk = 0;
    for (int64_t r0 = 0; st == QAT4_OK && r0 < R; r0 += crow, ++chunk) {
        const int b = static_cast<int>(chunk & 1);
        const int64_t nr = std::min(crow, R - r0);
        const size_t n = static_cast<size_t>(nr * C);
        const size_t off = static_cast<size_t>(r0 * C);
        bool ok = true;
        // the stage's outputs of two chunks ago must be on the host before it is refilled
        if (chunk >= 2) ok &= cudaStreamWaitEvent(stream, freed[b], 0) == cudaSuccess;
        ok &= cudaMemcpyAsync(buf[b].w, W + off, n * 4, H2D, stream) == cudaSuccess;
        ok &= cudaMemcpyAsync(buf[b].g, static_cast<const uint8_t*>(G) + off * gb, n * gb, H2D, stream) == cudaSuccess;
        ok &= cudaMemcpyAsync(buf[b].d, delta + off / 32, n / 32 * 4, H2D, stream) == cudaSuccess;
        if (!ok) { st = QAT4_ERR_CUDA; break; }
        st = lsq_common(buf[b].w, buf[b].d, buf[b].g, g_dtype, nr, C, grad_scale, buf[b].q, buf[b].gw, buf[b].gd,
                        true, true, stream);
        if (st != QAT4_OK) break;
        ok &= cudaEventRecord(done[b], stream) == cudaSuccess;
        // downloads on the copy stream overlap the next chunk's uploads (PCIe is full duplex)
        ok &= cudaStreamWaitEvent(copy_stream, done[b], 0) == cudaSuccess;
        ok &= cudaMemcpyAsync(Q + off, buf[b].q, n * 4, D2H, copy_stream) == cudaSuccess;
        ok &= cudaMemcpyAsync(grad_W + off, buf[b].gw, n * 4, D2H, copy_stream) == cudaSuccess;
        ok &= cudaMemcpyAsync(grad_delta + off / 32, buf[b].gd, n / 32 * 4, D2H, copy_stream) == cudaSuccess;
        ok &= cudaEventRecord(freed[b], copy_stream) == cudaSuccess;
        if (!ok) st = QAT4_ERR_CUDA;
    }
    // completion is observable on `stream`: it waits for the last download (also after an error
    // part-way, so that nothing of this call is still running when `stream` has completed)
    if (made && (cudaEventRecord(last, copy_stream) != cudaSuccess ||
                 cudaStreamWaitEvent(stream, last, 0) != cudaSuccess))
        st = QAT4_ERR_CUDA;
    // release whatever was created (destruction of a pending event is deferred by the runtime)
    for (int b = 0; b < 2; ++b) {
        if (done[b]) cudaEventDestroy(done[b]);
        if (freed[b]) cudaEventDestroy(freed[b]);
    }
    if (last) cudaEventDestroy(last);
    return st;
}

// -------------------------------------------------------------- per-channel
static qat4_status lsq_rowwise_common(const float* W, const float* delta, const void* G, qat4_dtype g_dtype,
                                      int64_t R, int64_t C, float grad_scale, float* Q, float* grad_W,
                                      float* grad_delta, bool fwd, bool bwd, cudaStream_t stream) {
    if (!W || !delta || (fwd && !Q) || (bwd && (!G || !grad_W || !grad_delta))) return QAT4_ERR_NULL;
    if (!valid_rc(R, C)) return QAT4_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(delta) || (fwd && !aligned16(Q)) ||
        (bwd && (!aligned16(G) || !aligned16(grad_W) || !aligned16(grad_delta))))
        return QAT4_ERR_ALIGN;
    if (bwd && g_dtype != QAT4_F32 && g_dtype != QAT4_BF16) return QAT4_ERR_DTYPE;
    const unsigned grid = static_cast<unsigned>(R);
    const unsigned th = qat4::kRowThreads;
    const int c = static_cast<int>(C);
    if (fwd && !bwd) {
        qat4::lsq_rowwise_kernel<float, true, false><<<grid, th, 0, stream>>>(W, delta, nullptr, c, 0.f, Q,
                                                                             nullptr, nullptr);
    } else if (g_dtype == QAT4_F32) {
        const float* g = static_cast<const float*>(G);
        if (fwd)
            qat4::lsq_rowwise_kernel<float, true, true><<<grid, th, 0, stream>>>(W, delta, g, c, grad_scale, Q,
                                                                                grad_W, grad_delta);
        else
            qat4::lsq_rowwise_kernel<float, false, true><<<grid, th, 0, stream>>>(W, delta, g, c, grad_scale,
                                                                                 nullptr, grad_W, grad_delta);
    } else {
        const uint16_t* g = static_cast<const uint16_t*>(G);
        if (fwd)
            qat4::lsq_rowwise_kernel<uint16_t, true, true><<<grid, th, 0, stream>>>(W, delta, g, c, grad_scale,
                                                                                   Q, grad_W, grad_delta);
        else
            qat4::lsq_rowwise_kernel<uint16_t, false, true><<<grid, th, 0, stream>>>(W, delta, g, c, grad_scale,
                                                                                    nullptr, grad_W, grad_delta);
    }
    return launch_status();
}

qat4_status qat4_lsq_fwd_rowwise(const float* W, const float* delta, int64_t R, int64_t C, float* Q,
                                 cudaStream_t stream) {
    return lsq_rowwise_common(W, delta, nullptr, QAT4_F32, R, C, 0.f, Q, nullptr, nullptr, true, false, stream);
}

qat4_status qat4_lsq_bwd_rowwise(const float* W, const float* delta, const void* G, qat4_dtype g_dtype,
                                 int64_t R, int64_t C, float grad_scale, float* grad_W, float* grad_delta,
                                 cudaStream_t stream) {
    return lsq_rowwise_common(W, delta, G, g_dtype, R, C, grad_scale, nullptr, grad_W, grad_delta, false, true,
                              stream);
}

qat4_status qat4_lsq_fwd_bwd_rowwise(const float* W, const float* delta, const void* G, qat4_dtype g_dtype,
                                     int64_t R, int64_t C, float grad_scale, float* Q, float* grad_W,
                                     float* grad_delta, cudaStream_t stream) {
    return lsq_rowwise_common(W, delta, G, g_dtype, R, C, grad_scale, Q, grad_W, grad_delta, true, true, stream);
}

qat4_status qat4_pack_w4a16_rowwise(const float* W, const float* delta, int64_t R, int64_t C, uint8_t* packed,
                                    uint16_t* scales, cudaStream_t stream) {
    if (!W || !delta || !packed || !scales) return QAT4_ERR_NULL;
    if (!valid_rc(R, C)) return QAT4_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(delta) || !aligned16(packed) || !aligned16(scales)) return QAT4_ERR_ALIGN;
    // the short-block export in its row mode: C / 8 octets share one scale
    const int64_t noct = R * C / 8;
    constexpr int kU = 4;
    const int64_t blocks = (noct + qat4::kPackBlock * kU - 1) / (qat4::kPackBlock * kU);
    const int64_t row_oct = C / 8;
    qat4::pack_w4a16_blocks_kernel<kU, true><<<static_cast<unsigned>(blocks), qat4::kPackBlock, 0, stream>>>(
        W, delta, noct, row_oct, 1.0 / static_cast<double>(row_oct), reinterpret_cast<uint32_t*>(packed), scales);
    return launch_status();
}

size_t qat4_scale_search_rowwise_workspace_bytes(int64_t R, int64_t C) {
    if (R < 1 || C < 32 || C % 32 != 0 || C > qat4::kRsMaxC) return 0;
    const size_t hq = static_cast<size_t>(R) * static_cast<size_t>(C) * 2 * sizeof(double);
    return hq + ((static_cast<size_t>(R) * sizeof(float) + 255) / 256) * 256;
}

qat4_status qat4_scale_search_rowwise(const float* W, int64_t R, int64_t C, const float* H, int64_t ldh,
                                      const float* alpha, int32_t K, float* delta, int32_t* idx,
                                      float* best_err, void* workspace, size_t workspace_bytes,
                                      cudaStream_t stream) {
    if (!W || !H || !alpha || !delta || !idx || !workspace) return QAT4_ERR_NULL;
    if (!valid_rc(R, C) || C > qat4::kRsMaxC || K < 1 || ldh < C || R > (int64_t(1) << 22)) return QAT4_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(H) || !aligned16(alpha) || !aligned16(delta) || !aligned16(idx) ||
        (best_err && !aligned16(best_err)) || !aligned16(workspace))
        return QAT4_ERR_ALIGN;
    if (workspace_bytes < qat4_scale_search_rowwise_workspace_bytes(R, C)) return QAT4_ERR_WORKSPACE;
    const int ept = C <= 2048 ? 8 : (C <= 4096 ? 16 : 32);
    const size_t smem = static_cast<size_t>(C) * (sizeof(double) + sizeof(uint32_t));
    int dev;
    DeviceInfo* info;
    if (!device_info(&dev, &info)) return QAT4_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!info->rowsearch_attr) {
            const int mx = static_cast<int>(qat4::kRsMaxC * (sizeof(double) + sizeof(uint32_t)));
            if (cudaFuncSetAttribute(qat4::rowwise_sweep_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx) != cudaSuccess ||
                cudaFuncSetAttribute(qat4::rowwise_sweep_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx) != cudaSuccess ||
                cudaFuncSetAttribute(qat4::rowwise_sweep_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx) != cudaSuccess)
                return QAT4_ERR_CUDA;
            info->rowsearch_attr = true;
        }
    }
    double* hbuf = static_cast<double*>(workspace);
    double* tbuf = hbuf + R * C;
    float* base = reinterpret_cast<float*>(tbuf + R * C);
    const int r = static_cast<int>(R), c = static_cast<int>(C);
    qat4::rowwise_base_kernel<<<static_cast<unsigned>((R * 32 + 255) / 256), 256, 0, stream>>>(W, r, c, base);
    const dim3 g1(static_cast<unsigned>((C + qat4::kHqTile - 1) / qat4::kHqTile),
                  static_cast<unsigned>((R + qat4::kHqTile - 1) / qat4::kHqTile));
    qat4::rowwise_hq_kernel<<<g1, 256, 0, stream>>>(W, r, c, H, ldh, base, alpha, hbuf, tbuf);
    const unsigned g2 = static_cast<unsigned>(R);
    if (ept == 8)
        qat4::rowwise_sweep_kernel<8><<<g2, qat4::kRsThreads, smem, stream>>>(W, c, H, ldh, alpha, K, base, hbuf, tbuf,
                                                                            delta, idx, best_err);
    else if (ept == 16)
        qat4::rowwise_sweep_kernel<16><<<g2, qat4::kRsThreads, smem, stream>>>(W, c, H, ldh, alpha, K, base, hbuf, tbuf,
                                                                             delta, idx, best_err);
    else
        qat4::rowwise_sweep_kernel<32><<<g2, qat4::kRsThreads, smem, stream>>>(W, c, H, ldh, alpha, K, base, hbuf, tbuf,
                                                                             delta, idx, best_err);
    return launch_status();
}

// ---------------------------------------------------------- W4A16 inference
qat4_status qat4_w4a16_gemv(const uint16_t* x, int64_t M, const uint8_t* packed, const uint16_t* scales,
                            int64_t R, int64_t C, int64_t group, float* y, cudaStream_t stream) {
    if (!x || !packed || !scales || !y) return QAT4_ERR_NULL;
    if (M < 1 || M > 65535 || !valid_rc(R, C) || group < 32 || group % 32 != 0 || C % group != 0)
        return QAT4_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(packed) || !aligned16(scales) || !aligned16(y)) return QAT4_ERR_ALIGN;
    int dev = 0;
    DeviceInfo* info = nullptr;
    if (!device_info(&dev, &info)) return QAT4_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (info->smem_optin == 0) {
            int optin = 0;
            if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
                return QAT4_ERR_CUDA;
            if (cudaFuncSetAttribute(qat4::w4a16_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, optin))
                return QAT4_ERR_CUDA;
            info->smem_optin = optin;
        }
    }
    const size_t optin = static_cast<size_t>(info->smem_optin);
    const int c = static_cast<int>(C);
    // tokens per pass: up to 8, fewer when x of a wide row leaves under three ring slots
    int mt_max = qat4::kGmMaxTokens;
    while (mt_max > 0 && qat4::gemv_smem_bytes(mt_max, c, 3) > optin) --mt_max;
    if (mt_max == 0) return QAT4_ERR_SHAPE;

    EncodeTiledFn encode = encode_tiled();
    if (!encode) return QAT4_ERR_CUDA;
    CUtensorMap tmap;   // codes as uint32 words [R, C/8]; one box = 16 rows x 128 bytes, 128-byte swizzle
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(C / 8), static_cast<cuuint64_t>(R)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(C / 2)};
        const cuuint32_t box[2] = {32, static_cast<cuuint32_t>(qat4::kGmRows)};
        const cuuint32_t estr[2] = {1, 1};
        if (encode(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint8_t*>(packed), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return QAT4_ERR_CUDA;
    }
    // both launches may overlap the previous kernel of the stream (programmatic dependent launch);
    // each waits for it before it reads x or writes y
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    {
        const int64_t ny = M * R;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>((ny / 4 + 255) / 256 + 1, 4 * info->sms)));
        cfg.blockDim = dim3(256);
        cfg.stream = stream;
        cfg.attrs = pdl;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, qat4::gemv_zero_kernel, y, ny) != cudaSuccess) return QAT4_ERR_CUDA;
    }
    qat4::GemvParams p;
    p.scales = scales;
    p.R = static_cast<int>(R);
    p.C = c;
    p.group = static_cast<int>(group);
    p.G = static_cast<int>(C / group);
    p.nblocks = static_cast<int>((R + qat4::kGmRows - 1) / qat4::kGmRows);
    p.nchunks = static_cast<int>((C + qat4::kGmChunkCols - 1) / qat4::kGmChunkCols);
    p.xstride = qat4::gemv_xstride(c);
    p.dmask = 0x000F000Fu;        // nibbles at bits 0..3 and 16..19
    p.dbits = 0x43084308u;        // bf16 exponent of 128 in both halves, plus the nibbles' top bit
    for (int64_t m0 = 0; m0 < M; m0 += mt_max) {
        const int mt = static_cast<int>(M - m0 < mt_max ? M - m0 : mt_max);
        // two CTAs per SM when two 5-stage rings fit, else one with as many stages as fit
        int per_sm = 2, stages = 5;
        if (2 * (qat4::gemv_smem_bytes(mt, c, stages) + 1024) > 228u * 1024u) {
            per_sm = 1;
            stages = qat4::kGmMaxStages;
            while (stages > 3 && qat4::gemv_smem_bytes(mt, c, stages) > optin) --stages;
        }
        const int64_t want = static_cast<int64_t>(info->sms) * per_sm;
        const int grid = static_cast<int>(p.nblocks < want ? p.nblocks : want);   // ranges >= one row block
        const int64_t per_cta = (static_cast<int64_t>(p.nblocks) * p.nchunks + grid - 1) / grid;
        // generous bound: 4 s plus 20 us per stage of a CTA (a stage streams in well under 1 us)
        p.limit_ns = 4000000000ull + 20000ull * static_cast<uint64_t>(per_cta);
        p.stages = stages;
        p.MT = mt;
        p.x = x + m0 * C;
        p.y = y + m0 * R;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid));
        cfg.blockDim = dim3(qat4::kGmThreads);
        cfg.dynamicSmemBytes = qat4::gemv_smem_bytes(mt, c, stages);
        cfg.stream = stream;
        cfg.attrs = pdl;
        cfg.numAttrs = 1;
        if (cudaLaunchKernelEx(&cfg, qat4::w4a16_gemv_kernel, tmap, p) != cudaSuccess) return QAT4_ERR_CUDA;
    }
    return QAT4_OK;
}

// ------------------------------------------------------ fake-quant forward GEMM
qat4_status qat4_fq_gemm(const uint16_t* X, int64_t T, const float* W, const float* delta, int64_t R, int64_t C,
                         float* Y, cudaStream_t stream) {
    if (!X || !W || !delta || !Y) return QAT4_ERR_NULL;
    if (T < 1 || T > (int64_t(1) << 31) - 1 || !valid_rc(R, C) || T * R > (int64_t(1) << 40)) return QAT4_ERR_SHAPE;
    if (!aligned16(X) || !aligned16(W) || !aligned16(delta) || !aligned16(Y)) return QAT4_ERR_ALIGN;
    const int64_t tiles_m = (T + qat4::kFqTile * qat4::kFqMTiles - 1) / (qat4::kFqTile * qat4::kFqMTiles);
    const int64_t tiles_r = (R + qat4::kFqTile - 1) / qat4::kFqTile;
    if (2 * tiles_m * tiles_r > (int64_t(1) << 31) - 1) return QAT4_ERR_SHAPE;
    int dev = 0;
    DeviceInfo* info = nullptr;
    if (!device_info(&dev, &info)) return QAT4_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!info->fq_attr) {
            if (cudaFuncSetAttribute(qat4::fq_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(qat4::kFqSmemBytes)) != cudaSuccess)
                return QAT4_ERR_CUDA;
            info->fq_attr = true;
        }
    }
    EncodeTiledFn encode = encode_tiled();
    if (!encode) return QAT4_ERR_CUDA;
    CUtensorMap tx, tw;
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(T)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(C) * 2};
        const cuuint32_t box[2] = {static_cast<cuuint32_t>(qat4::kFqBK), static_cast<cuuint32_t>(qat4::kFqHalf)};
        const cuuint32_t estr[2] = {1, 1};
        if (encode(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return QAT4_ERR_CUDA;
    }
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(R)};
        const cuuint64_t strides[1] = {static_cast<cuuint64_t>(C) * 4};
        const cuuint32_t box[2] = {32, static_cast<cuuint32_t>(qat4::kFqHalf)};
        const cuuint32_t estr[2] = {1, 1};
        if (encode(&tw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(W), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return QAT4_ERR_CUDA;
    }
    qat4::FqParams p;
    p.delta = delta;
    p.Y = Y;
    p.T = static_cast<int>(T);
    p.R = static_cast<int>(R);
    p.C = static_cast<int>(C);
    p.G = static_cast<int>(C / 32);
    p.tiles_r = static_cast<int>(tiles_r);
    p.ksteps = static_cast<int>((C + qat4::kFqBK - 1) / qat4::kFqBK);
    // generous bound: 4 s plus 10 us per 64-column step (a step takes well under 1 us)
    p.limit_ns = 4000000000ull + 10000ull * static_cast<uint64_t>(p.ksteps);
    const unsigned grid = static_cast<unsigned>(2 * tiles_m * tiles_r);
    qat4::fq_gemm_kernel<<<grid, qat4::kFqThreads, qat4::kFqSmemBytes, stream>>>(tx, tw, p);
    return launch_status();
}

size_t qat4_fq_gemm_staged_workspace_bytes(int64_t R, int64_t C) {
    if (!valid_rc(R, C)) return 0;
    return (static_cast<size_t>(R) * static_cast<size_t>(C) * 2 + 255) & ~size_t(255);
}

qat4_status qat4_fq_gemm_staged(const uint16_t* X, int64_t T, const float* W, const float* delta, int64_t R,
                                int64_t C, float* Y, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (!X || !W || !delta || !Y || !workspace) return QAT4_ERR_NULL;
    if (T < 1 || T > (int64_t(1) << 31) - 1 || !valid_rc(R, C) || T * R > (int64_t(1) << 40)) return QAT4_ERR_SHAPE;
    if (!aligned16(X) || !aligned16(W) || !aligned16(delta) || !aligned16(Y) ||
        (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
        return QAT4_ERR_ALIGN;
    if (workspace_bytes < qat4_fq_gemm_staged_workspace_bytes(R, C)) return QAT4_ERR_WORKSPACE;
    const int64_t tiles_m = (T + qat4::kGTile - 1) / qat4::kGTile;
    const int64_t tiles_n = (R + qat4::kGTile - 1) / qat4::kGTile;
    if (tiles_m * tiles_n > (int64_t(1) << 31) - 1) return QAT4_ERR_SHAPE;
    int dev = 0;
    DeviceInfo* info = nullptr;
    if (!device_info(&dev, &info)) return QAT4_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(g_mutex);
        if (!info->gemm_attr) {
            if (cudaFuncSetAttribute(qat4::gemm_bf16_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(qat4::kGSmemBytes)) != cudaSuccess)
                return QAT4_ERR_CUDA;
            info->gemm_attr = true;
        }
    }
    EncodeTiledFn encode = encode_tiled();
    if (!encode) return QAT4_ERR_CUDA;
    uint16_t* Qb = static_cast<uint16_t*>(workspace);
    // both operands bf16 K-major [rows, C]: one box = 128 rows x 64 columns (128 bytes), 128-byte swizzle
    CUtensorMap ta, tb;
    const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(qat4::kGHalf)};
    const cuuint32_t estr[2] = {1, 1};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(C) * 2};
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(T)};
        if (encode(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return QAT4_ERR_CUDA;
    }
    {
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(R)};
        if (encode(&tb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Qb, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return QAT4_ERR_CUDA;
    }
    CUtensorMap ty = {};
    const bool tma_store = (R % 4) == 0;     // rows of Y 16-byte aligned
    if (tma_store) {   // Y float32 [T, R]: one box = 32 rows x 32 columns (128 bytes), 128-byte swizzle
        const cuuint64_t dims[2] = {static_cast<cuuint64_t>(R), static_cast<cuuint64_t>(T)};
        const cuuint64_t ystr[1] = {static_cast<cuuint64_t>(R) * 4};
        const cuuint32_t ybox[2] = {32, 32};
        if (encode(&ty, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, Y, dims, ystr, ybox, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return QAT4_ERR_CUDA;
    }
    // 1. Qb = bf16(Q_Delta(W)), 16 weights per thread
    const int64_t nhalf = R * C / 16;
    qat4::fq_quantize_kernel<<<static_cast<unsigned>((nhalf + qat4::kFqQuantBlock - 1) / qat4::kFqQuantBlock),
                               qat4::kFqQuantBlock, 0, stream>>>(W, delta, nhalf, Qb);
    if (cudaGetLastError() != cudaSuccess) return QAT4_ERR_CUDA;
    // 2. Y = X Qb^T on the tensor cores, one persistent pair per SM pair
    qat4::GemmParams p;
    p.Y = Y;
    p.T = static_cast<int>(T);
    p.R = static_cast<int>(R);
    p.C = static_cast<int>(C);
    p.tiles_m = static_cast<int>(tiles_m);
    p.tiles = static_cast<int>(tiles_m * tiles_n);
    p.ksteps = static_cast<int>((C + qat4::kGBK - 1) / qat4::kGBK);
    p.tma_store = tma_store ? 1 : 0;
    const int pairs = static_cast<int>(std::min<int64_t>(qat4::kGPairsPerGpu, tiles_m * tiles_n));
    const int64_t per_pair = (tiles_m * tiles_n + pairs - 1) / pairs;
    // generous bound: 4 s plus 10 us per 128-column step of a pair's tiles (a step takes well under 1 us)
    p.limit_ns = 4000000000ull + 10000ull * static_cast<uint64_t>(per_pair * p.ksteps);
    // launched early (programmatic dependent launch): its producer waits for the quantizer
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(2 * pairs));
    cfg.blockDim = dim3(qat4::kGThreads);
    cfg.dynamicSmemBytes = qat4::kGSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, qat4::gemm_bf16_pair_kernel, ta, tb, ty, p) != cudaSuccess) return QAT4_ERR_CUDA;
    return launch_status();
}

// ------------------------------------------------------ full-objective refinement
size_t qat4_refine_workspace_bytes(int64_t R, int64_t C) {
    if (!valid_rc(R, C)) return 0;
    return 2 * static_cast<size_t>(R) * static_cast<size_t>(C) * sizeof(double);
}

qat4_status qat4_refine(const float* W, int64_t R, int64_t C, const float* H, int64_t ldh, const float* alpha,
                        int32_t K, int32_t sweeps, int32_t* idx, float* delta, double* obj, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
    if (!W || !H || !alpha || !idx || !delta) return QAT4_ERR_NULL;
    if (!valid_rc(R, C) || K < 1 || sweeps < 0 || ldh < C || R > 65535 * int64_t(qat4::kRfTileR))
        return QAT4_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(H) || !aligned16(alpha) || !aligned16(idx) || !aligned16(delta) ||
        (obj && !aligned16(obj)) || (ldh % 4) != 0 || (workspace && !aligned16(workspace)))
        return QAT4_ERR_ALIGN;
    const size_t need = qat4_refine_workspace_bytes(R, C);
    if (!workspace || workspace_bytes < need) return QAT4_ERR_WORKSPACE;
    int dev = 0;
    DeviceInfo* info = nullptr;
    if (!device_info(&dev, &info)) return QAT4_ERR_CUDA;
    double* E = static_cast<double*>(workspace);
    double* V = E + R * C;
    const int64_t ngroups = R * (C / 32);
    const int64_t err_blocks = (ngroups + 7) / 8;
    const unsigned eb = static_cast<unsigned>(err_blocks < int64_t(info->sms) * 16 ? err_blocks : int64_t(info->sms) * 16);
    qat4::refine_err_kernel<<<eb, 256, 0, stream>>>(W, ngroups, alpha, K, idx, E);
    if (cudaGetLastError() != cudaSuccess) return QAT4_ERR_CUDA;
    const dim3 vgrid(static_cast<unsigned>((C + qat4::kRfTileC - 1) / qat4::kRfTileC),
                     static_cast<unsigned>((R + qat4::kRfTileR - 1) / qat4::kRfTileR));
    qat4::refine_v_kernel<<<vgrid, 256, 0, stream>>>(E, static_cast<int>(R), static_cast<int>(C), H, ldh, V);
    if (cudaGetLastError() != cudaSuccess) return QAT4_ERR_CUDA;
    const unsigned sgrid = static_cast<unsigned>((R + qat4::kRfWarps - 1) / qat4::kRfWarps);
    qat4::refine_sweep_kernel<<<sgrid, 32 * qat4::kRfWarps, 0, stream>>>(
        W, static_cast<int>(R), static_cast<int>(C), H, ldh, alpha, K, sweeps, idx, delta, obj, V);
    return launch_status();
}

// ------------------------------------------------------------ error handling
qat4_status qat4_sync_check(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return QAT4_ERR_CUDA;
    int word = 0;
    if (cudaMemcpyFromSymbol(&word, qat4::g_dev_error, sizeof word) != cudaSuccess) return QAT4_ERR_CUDA;
    if (word != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(qat4::g_dev_error, &zero, sizeof zero) != cudaSuccess) return QAT4_ERR_CUDA;
        if (word & qat4::QAT4_DEV_ERR_TIMEOUT) return QAT4_ERR_TIMEOUT;
    }
    return QAT4_OK;
}

}  // extern "C"

namespace qat4 {
__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // nothing ever arrives on `bar`: the wait runs into its limit and returns
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, limit_ns);
}
}  // namespace qat4

extern "C" qat4_status qat4_selftest_bounded_wait(int64_t limit_ns, cudaStream_t stream) {
    if (limit_ns < 1 || limit_ns > 10000000000ll) return QAT4_ERR_SHAPE;
    qat4::bounded_wait_selftest_kernel<<<1, 32, 0, stream>>>(static_cast<uint64_t>(limit_ns));
    return launch_status();
}

// ------------------------------------------------------ no-allocation variant
// Some callers of this library cannot allocate device memory themselves: code
// that runs inside an engine or framework which owns every byte of device
// memory (a caching allocator or a fixed memory budget that a stray cudaMalloc
// would break), and latency-critical loops in which cudaMalloc/cudaFree, which
// may synchronise the device, are not acceptable.  qat4_hessian_noalloc serves
// them: its scratch is the file-scope array below, which every GPU that loads
// this library holds until the process exits.
namespace {

// Largest workspace the Hessian planner can ask for: at most 74 parts of cut
// tiles, each one 256 x 256 fp32 partial.
constexpr size_t kNoallocScratchBytes =
    static_cast<size_t>(qat4::kPPairsPerGpu) * qat4::kPTile * qat4::kPTile * sizeof(float);  // 18.5 MiB

static __device__ __align__(256) unsigned char g_hessian_scratch[kNoallocScratchBytes];

void* g_scratch_addr[kMaxDevices] = {};              // device address of g_hessian_scratch
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // the context that address belongs to

}  // namespace

extern "C" qat4_status qat4_hessian_noalloc(const uint16_t* X, int64_t n, int64_t C, float* H,
                                            cudaStream_t stream) {
    if (!X || !H) return QAT4_ERR_NULL;
    if (n < 1 || n > (int64_t(1) << 31) - 1 || C < 32 || C % 32 != 0 || C > 65536) return QAT4_ERR_SHAPE;
    const size_t need = qat4_hessian_workspace_bytes(n, C);
    if (need > kNoallocScratchBytes) return QAT4_ERR_WORKSPACE;   // larger than the built-in scratch
    int dev = 0;
    DeviceInfo* info = nullptr;
    if (!device_info(&dev, &info)) return QAT4_ERR_CUDA;           // also makes the context current
    const unsigned long long ctx = current_ctx_id();
    void* scratch = nullptr;
    {
        // Set-up once per device (and again if its context has been replaced, as after
        // cudaDeviceReset), with that device current: host code only knows a stand-in
        // for the array, so its device address is looked up.
        std::lock_guard<std::mutex> lock(g_mutex);
        if (g_scratch_addr[dev] == nullptr || ctx == 0 || ctx != g_scratch_ctx[dev]) {
            void* addr = nullptr;
            if (cudaGetSymbolAddress(&addr, g_hessian_scratch) != cudaSuccess || addr == nullptr)
                return QAT4_ERR_CUDA;
            g_scratch_addr[dev] = addr;
            g_scratch_ctx[dev] = ctx;
        }
        scratch = g_scratch_addr[dev];
    }
    // The kernels overwrite every scratch byte they later read, so the previous
    // call's contents need no clearing.
    return qat4_hessian(X, n, C, H, scratch, kNoallocScratchBytes, stream);
}
