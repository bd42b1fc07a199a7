// k_plane.cu -- small-map kernel family (placeholder until the fused kernel lands).
#include "gspn_internal.h"

namespace gspn {
bool plane_supports(const Problem&, bool) { return false; }
size_t plane_ws_bytes(const Problem&, bool) { return 0; }
cudaError_t plane_forward(const Problem&, const void*, const void*, const void*, const void*, void*, void*,
                          cudaStream_t) { return cudaErrorNotSupported; }
cudaError_t plane_backward(const Problem&, const void*, const void*, const void*, const void*, const void*, void*,
                           void*, void*, void*, void*, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace gspn
