// gspn_internal.h -- host-side declarations shared by the libgspn translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "gspn.h"

namespace gspn {

struct Problem {
    int N, C, H, W;
    int Cw;          // C (per-channel) or 1 (shared)
    int D;           // number of directions in the mask
    int wmode;
    unsigned mask;
    int dtype;       // GSPN_F32 / GSPN_BF16
    int chunk;       // lines per local chunk (0: global)
    int per_dir;     // lam and u carry a direction axis
    long long LU;    // elements of lam (and of u): U, or D * U with per_dir
    long long HW;    // H * W
    long long U;     // N * C * H * W
    long long A;     // D * N * Cw * 3 * H * W
    int esize() const { return dtype == GSPN_F32 ? 4 : 2; }
};

inline size_t align256(size_t b) { return (b + 255) & ~(size_t)255; }

// Workspace carving: a bump allocator over the caller's buffer (never allocates memory).
struct WsCarver {
    char* base;
    size_t off;
    explicit WsCarver(void* ws) : base((char*)ws), off(256) {}
    template <typename T> T* take(size_t count) {
        T* p = (T*)(base + off);
        off += align256(count * sizeof(T));
        return p;
    }
};

// ---- generic family (any shape) -------------------------------------------------------
size_t generic_ws_bytes(const Problem& p, bool bwd);
bool generic_supports(const Problem& p, bool bwd);
bool generic_fast_backward(const Problem& p);
cudaError_t generic_backward_saved(const Problem& p, const void* x, const void* a, const void* lam, const void* u,
                                   const void* dy, const float* hsaved, void* dx, void* da, void* dlam, void* du,
                                   void* ws, cudaStream_t st);
cudaError_t generic_forward(const Problem& p, const void* x, const void* a, const void* lam, const void* u,
                            void* y, void* ws, cudaStream_t st);
cudaError_t generic_backward(const Problem& p, const void* x, const void* a, const void* lam, const void* u,
                             const void* dy, void* dx, void* da, void* dlam, void* du, void* ws,
                             cudaStream_t st);

// ---- plane family (small maps, whole plane on chip) ------------------------------------
size_t plane_ws_bytes(const Problem& p, bool bwd);
bool plane_supports(const Problem& p, bool bwd);
bool plane_can_save(const Problem& p);
cudaError_t plane_forward_save(const Problem& p, const void* x, const void* a, const void* lam, const void* u,
                               void* y, float* hsave, cudaStream_t st);
cudaError_t plane_forward(const Problem& p, const void* x, const void* a, const void* lam, const void* u,
                          void* y, void* ws, cudaStream_t st);
cudaError_t plane_backward(const Problem& p, const void* x, const void* a, const void* lam, const void* u,
                           const void* dy, void* dx, void* da, void* dlam, void* du, void* ws,
                           cudaStream_t st);

// ---- sweep family (large maps, TMA-fed line sweeps) ------------------------------------
size_t sweep_ws_bytes(const Problem& p, bool bwd);
bool sweep_supports(const Problem& p, bool bwd);
cudaError_t sweep_forward(const Problem& p, const void* x, const void* a, const void* lam, const void* u,
                          void* y, void* ws, cudaStream_t st);
cudaError_t sweep_backward(const Problem& p, const void* x, const void* a, const void* lam, const void* u,
                           const void* dy, void* dx, void* da, void* dlam, void* du, void* ws,
                           cudaStream_t st);

// Weight table of the line sweeps: for every direction slot and (n, cw) plane, the outer weights
// (w0, w2) of each normalised tridiagonal row, in TableT of the storage dtype (fp32, or fp16 for
// bf16 storage). Slots from tslot0 on are written transposed ([W][H] per plane).
cudaError_t launch_weight_table(const Problem& P, const void* a, void* table, int tslot0, cudaStream_t st);

// ---- band family (large square maps): checkpointed scans with band recompute ----------------
bool band_supports(const Problem& p);
size_t band_ws_bytes(const Problem& p);
cudaError_t band_forward(const Problem& p, const void* x, const void* a, const void* lam, const void* u, void* y,
                         void* ws, cudaStream_t st);

// gspn_forward with the option of keeping the device status word (callers that launched their own
// kernels on the same workspace first clear it themselves).
gspn_status forward_internal(const gspn_desc* desc, const void* x, const void* a, const void* lam, const void* u,
                             void* y, void* ws, size_t ws_bytes, void* stream, bool clear_status);

// ---- channel projections of the compressive proxy (k_proj.cu) -----------------------------
// Y[n] (Mo x HW) = P (Mo x K) . X[n] (K x HW) for n < batch, row-major, storage dtype: a tcgen05
// GEMM for bf16 with 16-byte rows (K and HW multiples of 8), an exact fp32 SIMT GEMM otherwise.
bool proj_uses_tc(int dtype, int Mo, int K, long long HW);
cudaError_t launch_projection(int dtype, int Mo, int K, long long HW, int batch, const void* P, const void* X, void* Y,
                              unsigned* status, cudaStream_t st);

// ---- per-launch timing hooks (gspn_forward_timed) ---------------------------------------
// Kernel families call launch_begin / launch_end around every kernel launch. When a timed
// call is active on this host thread they record the caller's events on the launch stream.
void launch_begin(cudaStream_t st);
void launch_end(cudaStream_t st);

// ---- misc ------------------------------------------------------------------------------
// True when the descriptor is well formed (the checks gspn_forward reports as
// GSPN_ERR_INVALID_ARG); says nothing about whether a kernel family supports it.
bool desc_valid(const gspn_desc* d);
cudaError_t launch_copy(const void* src, void* dst, size_t bytes, cudaStream_t st);
cudaError_t launch_wait_probe(unsigned* status, const unsigned* flag, unsigned long long limit_ns,
                              cudaStream_t st);
int device_sm_count();

}  // namespace gspn
