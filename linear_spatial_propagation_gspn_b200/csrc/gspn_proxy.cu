// gspn_proxy.cu -- compressive channel proxy around the propagation.
//
// "GSPN-2: Efficient Parallel Sequence Modeling" paper notes, section "Optimisation 2: compact
// channel propagation": the C input channels are projected to C_proxy << C channels, the
// propagation runs in that proxy space, and a 1x1 convolution restores C channels. Per pixel
// the projections are dense matrix products over channels, i.e. per batch item a GEMM of a
// C_proxy x C (or C x C_proxy) matrix with a C x HW (C_proxy x HW) activation: the one dense
// contraction of the path. They run on the tensor cores as strided batched GEMMs through
// cuBLAS (plain library GEMMs); the propagation in between is gspn_forward.
//
// Row-major operands through a column-major library: Xp (Cp x HW) = P_in (Cp x C) . X (C x HW)
// is Xp^T (HW x Cp) = X^T (HW x C) . P_in^T (C x Cp) in column-major terms, where each row-major
// matrix is the column-major matrix of its transpose: m = HW, n = Cp, k = C, A = X (lda = HW),
// B = P_in (ldb = C), C = Xp (ldc = HW); likewise for the output projection.
#include <cublas_v2.h>

#include <mutex>

#include "gspn_common.cuh"
#include "gspn_internal.h"

namespace gspn {
namespace {

// One cuBLAS handle per device, created on first use and kept for the process; calls take the
// lock while they set the stream and enqueue (enqueueing is fast; the GEMMs run asynchronously).
std::mutex g_blas_mutex;
cublasHandle_t g_blas[64] = {};

cublasHandle_t blas_handle(int dev) {
    if (dev < 0 || dev >= 64) return nullptr;
    if (!g_blas[dev]) {
        cublasHandle_t h = nullptr;
        if (cublasCreate(&h) != CUBLAS_STATUS_SUCCESS) return nullptr;
        g_blas[dev] = h;
    }
    return g_blas[dev];
}

// Y (rows x HW, row-major, per batch item) = M (rows x inner, row-major, shared) . X (inner x HW)
cublasStatus_t project(cublasHandle_t h, int dtype, int rows, int inner, long long HW, int batch, const void* M,
                       const void* X, void* Y) {
    const float one = 1.f, zero = 0.f;
    const bool bf = dtype == GSPN_BF16;
    const cudaDataType_t t = bf ? CUDA_R_16BF : CUDA_R_32F;
    const cublasComputeType_t ct = bf ? CUBLAS_COMPUTE_32F : CUBLAS_COMPUTE_32F_PEDANTIC;
    return cublasGemmStridedBatchedEx(h, CUBLAS_OP_N, CUBLAS_OP_N, (int)HW, rows, inner, &one, X, t, (int)HW,
                                      (long long)inner * HW, M, t, inner, 0, &zero, Y, t, (int)HW,
                                      (long long)rows * HW, batch, ct, CUBLAS_GEMM_DEFAULT);
}

}  // namespace
}  // namespace gspn

using namespace gspn;

extern "C" {

GSPN_API size_t gspn_proxy_workspace_size(const gspn_desc* desc, int c_full) {
    if (!desc || c_full < 1) return 0;
    if ((long long)desc->N * c_full * desc->H * desc->W > (1LL << 40)) return 0;
    const size_t scan = gspn_workspace_size(desc, 0);
    if (scan == 0) return 0;
    const size_t es = desc->dtype == GSPN_F32 ? 4 : 2;
    const size_t proxy = (size_t)desc->N * desc->C * desc->H * desc->W * es;
    return align256(scan) + 2 * align256(proxy);
}

GSPN_API gspn_status gspn_proxy_forward(const gspn_desc* desc, int c_full, const void* x, const void* p_in,
                                        const void* a, const void* lam, const void* u, const void* p_out, void* y,
                                        void* ws, size_t ws_bytes, void* stream) {
    const size_t need = gspn_proxy_workspace_size(desc, c_full);
    if (need == 0) return GSPN_ERR_INVALID_ARG;
    if (!x || !p_in || !a || !lam || !u || !p_out || !y || !ws) return GSPN_ERR_INVALID_ARG;
    for (const void* q : {x, p_in, a, lam, u, p_out, (const void*)y, (const void*)ws})
        if (((uintptr_t)q & 15u) != 0) return GSPN_ERR_ALIGNMENT;
    if (ws_bytes < need) return GSPN_ERR_WORKSPACE;
    if ((long long)desc->H * desc->W > 0x7fffffffLL || c_full > 0x7fffffff / 2) return GSPN_ERR_UNSUPPORTED;
    const size_t scan = gspn_workspace_size(desc, 0);
    const size_t es = desc->dtype == GSPN_F32 ? 4 : 2;
    const size_t proxy = (size_t)desc->N * desc->C * desc->H * desc->W * es;
    char* base = (char*)ws;
    void* xp = base + align256(scan);
    void* yp = base + align256(scan) + align256(proxy);
    const long long HW = (long long)desc->H * desc->W;
    cudaStream_t st = (cudaStream_t)stream;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return GSPN_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lock(g_blas_mutex);
        cublasHandle_t h = blas_handle(dev);
        if (!h || cublasSetStream(h, st) != CUBLAS_STATUS_SUCCESS) return GSPN_ERR_CUDA;
        if (project(h, desc->dtype, desc->C, c_full, HW, desc->N, p_in, x, xp) != CUBLAS_STATUS_SUCCESS)
            return GSPN_ERR_CUDA;
    }
    const gspn_status s = gspn_forward(desc, xp, a, lam, u, yp, ws, scan, stream);
    if (s != GSPN_OK) return s;
    {
        std::lock_guard<std::mutex> lock(g_blas_mutex);
        cublasHandle_t h = blas_handle(dev);
        if (!h || cublasSetStream(h, st) != CUBLAS_STATUS_SUCCESS) return GSPN_ERR_CUDA;
        if (project(h, desc->dtype, c_full, desc->C, HW, desc->N, p_out, yp, y) != CUBLAS_STATUS_SUCCESS)
            return GSPN_ERR_CUDA;
    }
    return GSPN_OK;
}

}  // extern "C"
