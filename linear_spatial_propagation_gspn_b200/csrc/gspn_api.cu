// gspn_api.cu -- the C ABI of libgspn: argument checks, workspace sizing, kernel-family
// selection and the small utility kernels (copy ceiling, bounded-wait probe).
#include <atomic>
#include <stdint.h>
#include <string.h>

#include <algorithm>

#include "gspn_common.cuh"
#include "gspn_internal.h"

namespace gspn {
namespace {

bool make_problem(const gspn_desc* d, Problem* p) {
    if (!d) return false;
    if (d->N < 1 || d->C < 1 || d->H < 1 || d->W < 1) return false;
    if (d->wmode != GSPN_W_PER_CHANNEL && d->wmode != GSPN_W_SHARED) return false;
    if (d->dir_mask < 1u || d->dir_mask > 15u) return false;
    if (d->dtype != GSPN_F32 && d->dtype != GSPN_BF16) return false;
    if (d->algo < GSPN_ALGO_AUTO || d->algo > GSPN_ALGO_BAND) return false;
    if (d->chunk < 0) return false;
    if (d->per_dir != 0 && d->per_dir != 1) return false;
    if ((long long)d->N * d->C > 0x7fffffffLL) return false;
    p->N = d->N; p->C = d->C; p->H = d->H; p->W = d->W;
    p->wmode = d->wmode;
    p->mask = d->dir_mask;
    p->dtype = d->dtype;
    // a chunk at least as long as both axes is the global scan
    p->chunk = d->chunk >= (d->H > d->W ? d->H : d->W) ? 0 : d->chunk;
    p->Cw = d->wmode == GSPN_W_SHARED ? 1 : d->C;
    p->D = __builtin_popcount(d->dir_mask);
    p->HW = (long long)d->H * d->W;
    p->U = (long long)d->N * d->C * p->HW;
    p->A = (long long)p->D * d->N * p->Cw * 3 * p->HW;
    p->per_dir = d->per_dir;
    p->LU = d->per_dir ? p->D * p->U : p->U;
    return true;
}

int select_algo(const gspn_desc* d, const Problem& p, bool bwd) {
    // per-direction lambda / u: the sweep family does not run it
    if (p.per_dir && d->algo == GSPN_ALGO_SWEEP) return -1;
    switch (d->algo) {
    case GSPN_ALGO_GENERIC: return generic_supports(p, bwd) ? GSPN_ALGO_GENERIC : -1;
    case GSPN_ALGO_PLANE: return plane_supports(p, bwd) ? GSPN_ALGO_PLANE : -1;
    case GSPN_ALGO_SWEEP: return sweep_supports(p, bwd) ? GSPN_ALGO_SWEEP : -1;
    case GSPN_ALGO_BAND: return (!bwd && band_supports(p)) ? GSPN_ALGO_BAND : -1;
    default:
        if (bwd && generic_fast_backward(p)) return GSPN_ALGO_GENERIC;
        if (plane_supports(p, bwd)) return GSPN_ALGO_PLANE;
        if (!p.per_dir && sweep_supports(p, bwd)) return GSPN_ALGO_SWEEP;
        if (generic_supports(p, bwd)) return GSPN_ALGO_GENERIC;
        return -1;
    }
}

size_t ws_for(int algo, const Problem& p, bool bwd) {
    switch (algo) {
    case GSPN_ALGO_GENERIC: return generic_ws_bytes(p, bwd);
    case GSPN_ALGO_PLANE: return plane_ws_bytes(p, bwd);
    case GSPN_ALGO_SWEEP: return sweep_ws_bytes(p, bwd);
    case GSPN_ALGO_BAND: return bwd ? 0 : band_ws_bytes(p);
    default: return 0;
    }
}

bool aligned16(const void* ptr) { return ((uintptr_t)ptr & 15u) == 0; }

gspn_status to_status(cudaError_t e) { return e == cudaSuccess ? GSPN_OK : GSPN_ERR_CUDA; }

// ---------------------------------------------------------------- utility kernels
__global__ void k_copy16(const uint4* __restrict__ src, uint4* __restrict__ dst, long long n16) {
    long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x;
    const long long stride = (long long)gridDim.x * blockDim.x;
    // 4 independent 16-byte loads in flight per thread
    for (; i + 3 * stride < n16; i += 4 * stride) {
        uint4 v0 = src[i], v1 = src[i + stride], v2 = src[i + 2 * stride], v3 = src[i + 3 * stride];
        dst[i] = v0;
        dst[i + stride] = v1;
        dst[i + 2 * stride] = v2;
        dst[i + 3 * stride] = v3;
    }
    for (; i < n16; i += stride) dst[i] = src[i];
}

__global__ void k_wait_probe(unsigned* status, const unsigned* flag, unsigned long long limit_ns) {
    if (threadIdx.x == 0) wait_flag_bounded((const volatile unsigned*)flag, limit_ns, status);
}

struct Hooks {
    cudaEvent_t const* ev = nullptr;
    int n_ev = 0;
    int launches = 0;
    bool on = false;
};
thread_local Hooks g_hooks;

}  // namespace

bool desc_valid(const gspn_desc* d) {
    Problem p;
    return make_problem(d, &p);
}

void launch_begin(cudaStream_t st) {
    if (g_hooks.on && 2 * g_hooks.launches + 1 < g_hooks.n_ev) cudaEventRecord(g_hooks.ev[2 * g_hooks.launches], st);
}

void launch_end(cudaStream_t st) {
    if (!g_hooks.on) return;
    if (2 * g_hooks.launches + 1 < g_hooks.n_ev) cudaEventRecord(g_hooks.ev[2 * g_hooks.launches + 1], st);
    ++g_hooks.launches;
}

// SM count of the current device, queried once per device (host-side planning asks for it
// several times per call).
int device_sm_count() {
    static std::atomic<int> cache[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int sms = 148;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (dev >= 0 && dev < 64) cache[dev].store(sms, std::memory_order_relaxed);
    return sms;
}

cudaError_t launch_copy(const void* src, void* dst, size_t bytes, cudaStream_t st) {
    const long long n16 = (long long)(bytes / 16);
    const int blocks = device_sm_count() * 4;
    k_copy16<<<blocks, 512, 0, st>>>((const uint4*)src, (uint4*)dst, n16);
    return cudaGetLastError();
}

cudaError_t launch_wait_probe(unsigned* status, const unsigned* flag, unsigned long long limit_ns, cudaStream_t st) {
    k_wait_probe<<<1, 32, 0, st>>>(status, flag, limit_ns);
    return cudaGetLastError();
}

}  // namespace gspn

using namespace gspn;

extern "C" {

int gspn_version(void) { return 2; }

const char* gspn_status_string(gspn_status s) {
    switch (s) {
    case GSPN_OK: return "ok";
    case GSPN_ERR_INVALID_ARG: return "invalid argument";
    case GSPN_ERR_UNSUPPORTED: return "unsupported shape for the requested kernel family";
    case GSPN_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case GSPN_ERR_WORKSPACE: return "workspace too small";
    case GSPN_ERR_CUDA: return "CUDA error";
    case GSPN_ERR_DEVICE_TIMEOUT: return "bounded device wait timed out";
    default: return "unknown status";
    }
}

size_t gspn_workspace_size(const gspn_desc* desc, int for_backward) {
    Problem p;
    if (!make_problem(desc, &p)) return 0;
    const int algo = select_algo(desc, p, for_backward != 0);
    if (algo < 0) return 0;
    return ws_for(algo, p, for_backward != 0);
}

int gspn_selected_algo(const gspn_desc* desc, int for_backward) {
    Problem p;
    if (!make_problem(desc, &p)) return -1;
    return select_algo(desc, p, for_backward != 0);
}

gspn_status gspn_forward(const gspn_desc* desc, const void* x, const void* a, const void* lam, const void* u, void* y,
                         void* ws, size_t ws_bytes, void* stream) {
    return gspn::forward_internal(desc, x, a, lam, u, y, ws, ws_bytes, stream, true);
}

}  // extern "C"

gspn_status gspn::forward_internal(const gspn_desc* desc, const void* x, const void* a, const void* lam, const void* u,
                                   void* y, void* ws, size_t ws_bytes, void* stream, bool clear_status) {
    Problem p;
    if (!make_problem(desc, &p)) return GSPN_ERR_INVALID_ARG;
    if (!x || !a || !lam || !u || !y || !ws) return GSPN_ERR_INVALID_ARG;
    if (!aligned16(x) || !aligned16(a) || !aligned16(lam) || !aligned16(u) || !aligned16(y) || !aligned16(ws))
        return GSPN_ERR_ALIGNMENT;
    const int algo = select_algo(desc, p, false);
    if (algo < 0) return GSPN_ERR_UNSUPPORTED;
    if (ws_bytes < ws_for(algo, p, false)) return GSPN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = clear_status ? cudaMemsetAsync(ws, 0, sizeof(unsigned), st) : cudaSuccess;
    if (e != cudaSuccess) return GSPN_ERR_CUDA;
    switch (algo) {
    case GSPN_ALGO_PLANE: e = plane_forward(p, x, a, lam, u, y, ws, st); break;
    case GSPN_ALGO_SWEEP: e = sweep_forward(p, x, a, lam, u, y, ws, st); break;
    case GSPN_ALGO_BAND: e = band_forward(p, x, a, lam, u, y, ws, st); break;
    default: e = generic_forward(p, x, a, lam, u, y, ws, st); break;
    }
    return to_status(e);
}

extern "C" {

gspn_status gspn_forward_timed(const gspn_desc* desc, const void* x, const void* a, const void* lam, const void* u,
                               void* y, void* ws, size_t ws_bytes, void* stream, void* const* events, int n_events,
                               int* n_launches) {
    g_hooks.ev = (cudaEvent_t const*)events;
    g_hooks.n_ev = events ? n_events : 0;
    g_hooks.launches = 0;
    g_hooks.on = true;
    gspn_status s = gspn_forward(desc, x, a, lam, u, y, ws, ws_bytes, stream);
    g_hooks.on = false;
    if (n_launches) *n_launches = g_hooks.launches;
    return s;
}

gspn_status gspn_backward(const gspn_desc* desc, const void* x, const void* a, const void* lam, const void* u,
                          const void* dy, void* dx, void* da, void* dlam, void* du, void* ws, size_t ws_bytes,
                          void* stream) {
    Problem p;
    if (!make_problem(desc, &p)) return GSPN_ERR_INVALID_ARG;
    if (!x || !a || !lam || !u || !dy || !dx || !da || !dlam || !du || !ws) return GSPN_ERR_INVALID_ARG;
    const void* ptrs[] = {x, a, lam, u, dy, dx, da, dlam, du, ws};
    for (const void* q : ptrs)
        if (!aligned16(q)) return GSPN_ERR_ALIGNMENT;
    const int algo = select_algo(desc, p, true);
    if (algo < 0) return GSPN_ERR_UNSUPPORTED;
    if (ws_bytes < ws_for(algo, p, true)) return GSPN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(unsigned), st);
    if (e != cudaSuccess) return GSPN_ERR_CUDA;
    switch (algo) {
    case GSPN_ALGO_PLANE: e = plane_backward(p, x, a, lam, u, dy, dx, da, dlam, du, ws, st); break;
    case GSPN_ALGO_SWEEP: e = sweep_backward(p, x, a, lam, u, dy, dx, da, dlam, du, ws, st); break;
    default: e = generic_backward(p, x, a, lam, u, dy, dx, da, dlam, du, ws, st); break;
    }
    return to_status(e);
}

// The training pair applies: forward on the concurrent-direction plane kernel, backward on the
// all-directions kernels.
static bool pair_ok(const gspn_desc* desc, const Problem& p) {
    return gspn::select_algo(desc, p, false) == GSPN_ALGO_PLANE && gspn::plane_can_save(p) &&
           gspn::select_algo(desc, p, true) == GSPN_ALGO_GENERIC && gspn::generic_fast_backward(p);
}

size_t gspn_hsave_size(const gspn_desc* desc) {
    Problem p;
    if (!make_problem(desc, &p) || !pair_ok(desc, p)) return 0;
    return (size_t)p.D * p.U * sizeof(float);
}

gspn_status gspn_forward_save(const gspn_desc* desc, const void* x, const void* a, const void* lam, const void* u,
                              void* y, void* hsave, void* ws, size_t ws_bytes, void* stream) {
    Problem p;
    if (!make_problem(desc, &p)) return GSPN_ERR_INVALID_ARG;
    if (!x || !a || !lam || !u || !y || !hsave || !ws) return GSPN_ERR_INVALID_ARG;
    const void* ptrs[] = {x, a, lam, u, y, hsave, ws};
    for (const void* q : ptrs)
        if (!aligned16(q)) return GSPN_ERR_ALIGNMENT;
    if (!pair_ok(desc, p)) return GSPN_ERR_UNSUPPORTED;
    if (ws_bytes < ws_for(GSPN_ALGO_PLANE, p, false)) return GSPN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(unsigned), st);
    if (e != cudaSuccess) return GSPN_ERR_CUDA;
    return to_status(gspn::plane_forward_save(p, x, a, lam, u, y, (float*)hsave, st));
}

gspn_status gspn_backward_saved(const gspn_desc* desc, const void* x, const void* a, const void* lam, const void* u,
                                const void* dy, const void* hsave, void* dx, void* da, void* dlam, void* du, void* ws,
                                size_t ws_bytes, void* stream) {
    Problem p;
    if (!make_problem(desc, &p)) return GSPN_ERR_INVALID_ARG;
    if (!x || !a || !lam || !u || !dy || !hsave || !dx || !da || !dlam || !du || !ws) return GSPN_ERR_INVALID_ARG;
    const void* ptrs[] = {x, a, lam, u, dy, hsave, dx, da, dlam, du, ws};
    for (const void* q : ptrs)
        if (!aligned16(q)) return GSPN_ERR_ALIGNMENT;
    if (!pair_ok(desc, p)) return GSPN_ERR_UNSUPPORTED;
    if (ws_bytes < ws_for(GSPN_ALGO_GENERIC, p, true)) return GSPN_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(unsigned), st);
    if (e != cudaSuccess) return GSPN_ERR_CUDA;
    return to_status(gspn::generic_backward_saved(p, x, a, lam, u, dy, (const float*)hsave, dx, da, dlam, du, ws, st));
}

size_t gspn_forward_host_buffer_size(const gspn_desc* desc) {
    Problem p;
    if (!make_problem(desc, &p)) return 0;
    const size_t ws = gspn_workspace_size(desc, 0);
    if (ws == 0) return 0;
    const size_t es = p.esize();
    return 2 * align256(p.U * es) + 2 * align256(p.LU * es) + align256(p.A * es) + align256(ws);
}

gspn_status gspn_forward_host(const gspn_desc* desc, const void* hx, const void* ha, const void* hlam, const void* hu,
                              void* hy, void* dev, size_t dev_bytes, void* stream) {
    Problem p;
    if (!make_problem(desc, &p)) return GSPN_ERR_INVALID_ARG;
    if (!hx || !ha || !hlam || !hu || !hy || !dev) return GSPN_ERR_INVALID_ARG;
    if (!aligned16(dev)) return GSPN_ERR_ALIGNMENT;
    const size_t need = gspn_forward_host_buffer_size(desc);
    if (need == 0) return GSPN_ERR_UNSUPPORTED;
    if (dev_bytes < need) return GSPN_ERR_WORKSPACE;
    const size_t es = p.esize();
    const size_t ub = p.U * es, lb = p.LU * es, ab = p.A * es;
    char* base = (char*)dev;
    char* dx = base;
    char* dlam = dx + align256(ub);
    char* du = dlam + align256(lb);
    char* dyo = du + align256(lb);
    char* da = dyo + align256(ub);
    char* dws = da + align256(ab);
    const size_t wsb = dev_bytes - (size_t)(dws - base);
    cudaStream_t st = (cudaStream_t)stream;
    // Once a copy is queued, every return waits for the stream first: the caller may free or
    // reuse its host buffers as soon as this call returns, error or not.
    auto fail = [&](gspn_status s) {
        cudaStreamSynchronize(st);
        return s;
    };
    if (cudaMemcpyAsync(dx, hx, ub, cudaMemcpyHostToDevice, st) != cudaSuccess) return fail(GSPN_ERR_CUDA);
    if (cudaMemcpyAsync(da, ha, ab, cudaMemcpyHostToDevice, st) != cudaSuccess) return fail(GSPN_ERR_CUDA);
    if (cudaMemcpyAsync(dlam, hlam, lb, cudaMemcpyHostToDevice, st) != cudaSuccess) return fail(GSPN_ERR_CUDA);
    if (cudaMemcpyAsync(du, hu, lb, cudaMemcpyHostToDevice, st) != cudaSuccess) return fail(GSPN_ERR_CUDA);
    gspn_status s = gspn_forward(desc, dx, da, dlam, du, dyo, dws, wsb, stream);
    if (s != GSPN_OK) return fail(s);
    if (cudaMemcpyAsync(hy, dyo, ub, cudaMemcpyDeviceToHost, st) != cudaSuccess) return fail(GSPN_ERR_CUDA);
    if (cudaStreamSynchronize(st) != cudaSuccess) return GSPN_ERR_CUDA;
    return GSPN_OK;
}

gspn_status gspn_device_status(void* ws, void* stream) {
    if (!ws) return GSPN_ERR_INVALID_ARG;
    cudaStream_t st = (cudaStream_t)stream;
    unsigned word = 0;
    if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, st) != cudaSuccess) return GSPN_ERR_CUDA;
    if (cudaMemsetAsync(ws, 0, sizeof(word), st) != cudaSuccess) return GSPN_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return GSPN_ERR_CUDA;
    if (word & kDevTimeout) return GSPN_ERR_DEVICE_TIMEOUT;
    return GSPN_OK;
}

gspn_status gspn_debug_wait_timeout(void* ws, size_t ws_bytes, unsigned long long limit_ns, void* stream) {
    if (!ws || ws_bytes < kStatusBytes) return GSPN_ERR_INVALID_ARG;
    if (!aligned16(ws)) return GSPN_ERR_ALIGNMENT;
    if (limit_ns > 5000000000ULL) return GSPN_ERR_INVALID_ARG;  // never wait more than 5 s
    cudaStream_t st = (cudaStream_t)stream;
    unsigned* status = (unsigned*)ws;
    unsigned* flag = status + 16;  // inside the reserved 256 bytes; nothing ever sets it
    if (cudaMemsetAsync(ws, 0, kStatusBytes, st) != cudaSuccess) return GSPN_ERR_CUDA;
    return to_status(launch_wait_probe(status, flag, limit_ns, st));
}

gspn_status gspn_copy_ceiling(const void* src, void* dst, size_t bytes, void* stream) {
    if (!src || !dst) return GSPN_ERR_INVALID_ARG;
    if (!aligned16(src) || !aligned16(dst) || (bytes & 15u)) return GSPN_ERR_ALIGNMENT;
    return to_status(launch_copy(src, dst, bytes, (cudaStream_t)stream));
}

}  // extern "C"
