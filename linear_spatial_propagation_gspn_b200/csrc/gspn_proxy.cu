// gspn_proxy.cu -- compressive channel proxy around the propagation.
//
// "GSPN-2: Efficient Parallel Sequence Modeling" paper notes, section "Optimisation 2: compact
// channel propagation": the C input channels are projected to C_proxy << C channels, the
// propagation runs in that proxy space, and a 1x1 convolution restores C channels. Per pixel
// the projections are dense matrix products over channels, i.e. per batch item a GEMM of a
// C_proxy x C (or C x C_proxy) matrix with a C x HW (C_proxy x HW) activation: the one dense
// contraction of the path, run by the library's own projection kernels (k_proj.cu: tcgen05 tensor
// cores for bf16, exact fp32 otherwise); the propagation in between is gspn_forward.
#include "gspn_common.cuh"
#include "gspn_internal.h"

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
    unsigned* status = (unsigned*)ws;   // device status word, cleared once for the three stages
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned), st) != cudaSuccess) return GSPN_ERR_CUDA;
    if (launch_projection(desc->dtype, desc->C, c_full, HW, desc->N, p_in, x, xp, status, st) != cudaSuccess)
        return GSPN_ERR_CUDA;
    const gspn_status s = forward_internal(desc, xp, a, lam, u, yp, ws, scan, stream, false);
    if (s != GSPN_OK) return s;
    if (launch_projection(desc->dtype, c_full, desc->C, HW, desc->N, p_out, yp, y, status, st) != cudaSuccess)
        return GSPN_ERR_CUDA;
    return GSPN_OK;
}

}  // extern "C"
