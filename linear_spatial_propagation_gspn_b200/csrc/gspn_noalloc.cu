// gspn_noalloc.cu -- gspn_forward_noalloc: the forward pass with its scratch memory taken from
// a fixed device array compiled into the library, for callers that cannot allocate.
//
// Who needs this: some callers cannot allocate device memory at the moment they call us. The
// usual cases are code running inside a component that owns the device allocator (a framework
// caching allocator or an inference server with a pre-planned memory arena, where a foreign
// cudaMalloc would fragment or exceed the plan), and code on a latency-critical host path, where
// cudaMalloc / cudaFree can implicitly synchronise the whole device and stall other streams.
// Those callers still provide the inputs and the output; the workspace the forward needs comes
// from g_noalloc_scratch below instead of from them.
//
// The array is a file-scope __device__ variable: every GPU that loads this library holds
// GSPN_NOALLOC_SCRATCH_BYTES of it until the process exits. In host code its name is only a
// host-side stand-in, so every call looks up the device address with cudaGetSymbolAddress (with
// the target device current) and hands that to the kernels. The lookup is a host-side query that
// allocates nothing; doing it per call (instead of caching it) keeps the address right even after
// a cudaDeviceReset has reloaded the module at another address.
#include "gspn.h"
#include "gspn_internal.h"

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[GSPN_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch on the current device.
gspn_status scratch_for_current_device(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return GSPN_ERR_CUDA;
    *out = p;
    return GSPN_OK;
}

}  // namespace

extern "C" gspn_status gspn_forward_noalloc(const gspn_desc* desc, const void* x, const void* a, const void* lam,
                                            const void* u, void* y, void* stream) {
    // Descriptor first (malformed: GSPN_ERR_INVALID_ARG, as gspn_forward reports it), then the
    // size check: nothing touches the device for a problem that does not fit.
    if (!gspn::desc_valid(desc)) return GSPN_ERR_INVALID_ARG;
    const size_t need = gspn_workspace_size(desc, 0);
    if (need == 0) return GSPN_ERR_UNSUPPORTED;
    if (need > (size_t)GSPN_NOALLOC_SCRATCH_BYTES) return GSPN_ERR_WORKSPACE;
    if (!x || !a || !lam || !u || !y) return GSPN_ERR_INVALID_ARG;
    void* scratch = nullptr;
    const gspn_status s = scratch_for_current_device(&scratch);
    if (s != GSPN_OK) return s;
    // gspn_forward clears the status word at the start of the scratch before launching, and
    // every other byte it reads from the workspace is written earlier in the same call, so the
    // previous call's contents never leak into this one.
    return gspn_forward(desc, x, a, lam, u, y, scratch, (size_t)GSPN_NOALLOC_SCRATCH_BYTES, stream);
}
