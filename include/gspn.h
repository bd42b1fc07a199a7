/*
 * gspn.h -- C ABI of libgspn, the sm_100a (B200) implementation of the GSPN 4-direction
 * line-scan propagation.
 *
 * The operation ("GSPN-2: Efficient Parallel Sequence Modeling" paper notes, section
 * "2D spatial propagation review"; "Parallel Sequence Modeling via Generalized Spatial
 * Propagation Network" summary, section "Approach"):
 *
 *   for every plane (n, c) and every direction d in dir_mask, in scan coordinates
 *   (step i along the scan axis, lane j across it):
 *       h_{-1} = 0,   h_i[j] = sum_{k in range} w_i[j][k] h_{i-1}[j+k-1] + lam_i[j] x_i[j]
 *   with w_i[j][k] = sigmoid(a_k) / sum_{k' in range} sigmoid(a_k') over the neighbours
 *   j-1, j, j+1 that lie inside the line (a tridiagonal, row-stochastic matrix), and
 *       y = u * sum_{d in dir_mask} h^d      (h^d taken back to image coordinates).
 *   The display equation of the pages did not survive extraction; this is the reading the
 *   library implements (stated in full in the repository's design notes).
 *
 * Directions and scan coordinates (r = image row, c = image column):
 *   TB: r = i, c = j     BT: r = H-1-i, c = j     LR: r = j, c = i     RL: r = j, c = W-1-i
 * Neighbour k = 0, 1, 2 is lane j-1, j, j+1: ordered by increasing image coordinate on the
 * axis across the scan, for every direction. The three logits of hidden pixel (r, c) are
 * stored at image position (r, c).
 *
 * Weight modes: per-channel w_{i,c} (GSPN-1) or one w_i shared by all channels of a batch
 * item with per-channel lam (GSPN-2, "GSPN-2 ..." paper notes, section "Optimisation 2:
 * compact channel propagation").
 *
 * Layouts (all contiguous, all in the one storage dtype of the descriptor):
 *   x, lam, u, y, dy, dx, dlam, du : N x C x H x W
 *   a, da                          : D x N x Cw x 3 x H x W
 *     D  = popcount(dir_mask); slots in the fixed order TB, BT, LR, RL keeping only the
 *          directions in the mask;
 *     Cw = C (GSPN_W_PER_CHANNEL) or 1 (GSPN_W_SHARED).
 * Arithmetic is fp32 for both storage dtypes (bf16 values are widened on load and rounded to
 * nearest-even on store).
 *
 * Ownership and conventions:
 *   - The caller owns every buffer. The library never allocates, never keeps a pointer after
 *     a call returns, and never synchronises except in gspn_device_status and
 *     gspn_forward_host.
 *   - Work is enqueued on `stream` (a cudaStream_t passed as void*; NULL = legacy stream).
 *   - Outputs are overwritten, never accumulated into. In the shared mode da is the sum over
 *     channels.
 *   - Device pointers must be 16-byte aligned (else GSPN_ERR_ALIGNMENT), shapes must have
 *     N, C, H, W >= 1 and 1 <= dir_mask <= 15 (else GSPN_ERR_INVALID_ARG), and the workspace
 *     must be at least gspn_workspace_size() bytes (else GSPN_ERR_WORKSPACE). All of these
 *     are checked on the host before anything is launched.
 *   - A launch failure returns GSPN_ERR_CUDA. Kernels never trap; a bounded device-side wait
 *     that runs out records GSPN_ERR_DEVICE_TIMEOUT in the workspace status word, which
 *     gspn_device_status reports.
 *   - Calls sharing one workspace must not overlap on the GPU.
 */
#ifndef GSPN_H
#define GSPN_H

#include <stddef.h>

#if defined(__GNUC__)
#define GSPN_API __attribute__((visibility("default")))
#else
#define GSPN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GSPN_OK = 0,
    GSPN_ERR_INVALID_ARG = 1,
    GSPN_ERR_UNSUPPORTED = 2,
    GSPN_ERR_ALIGNMENT = 3,
    GSPN_ERR_WORKSPACE = 4,
    GSPN_ERR_CUDA = 5,
    GSPN_ERR_DEVICE_TIMEOUT = 6
} gspn_status;

typedef enum { GSPN_F32 = 0, GSPN_BF16 = 1 } gspn_dtype;
typedef enum { GSPN_W_PER_CHANNEL = 0, GSPN_W_SHARED = 1 } gspn_wmode;
enum { GSPN_DIR_TB = 1, GSPN_DIR_BT = 2, GSPN_DIR_LR = 4, GSPN_DIR_RL = 8, GSPN_DIR_ALL = 15 };

/* Kernel family. AUTO picks the fastest one that supports the shape; the others force a
 * family (GSPN_ERR_UNSUPPORTED if it cannot run the shape) so that every path can be tested
 * on the same inputs.
 *   GENERIC: any shape; one CTA per plane and direction, hidden line in shared memory.
 *   PLANE:   small maps; the whole plane stays on chip and all directions run in one pass.
 *   SWEEP:   large maps (forward): persistent line sweeps fed by per-thread asynchronous copies,
 *            one launch per direction plus one for the weights.
 *   BAND:    1024 x 1024 maps, all four directions, forward only, never chosen by AUTO: the
 *            ascending scans keep a checkpoint of their line every 8 lines and the descending
 *            scans recompute them band by band, so partial sums never cross HBM between the two
 *            scans of a pair (fewer DRAM bytes than SWEEP, but more rows streamed per SM). */
enum { GSPN_ALGO_AUTO = 0, GSPN_ALGO_GENERIC = 1, GSPN_ALGO_PLANE = 2, GSPN_ALGO_SWEEP = 3, GSPN_ALGO_BAND = 4 };

/* chunk: 0 = global propagation over the whole map. K > 0 = local propagation: the map is cut
 * along each direction's scan axis into chunks of K lines aligned to image line 0 (rows for
 * top->bottom / bottom->top, columns for left->right / right->left) and propagation does not
 * cross a chunk boundary (the scan restarts from h = 0 at the first line of every chunk in scan
 * order; the logits of that line get zero gradient). The pages contrast local and global GSPN
 * ("Parallel Sequence Modeling via Generalized Spatial Propagation Network" summary, section
 * "Measured effects") and give the fused kernel a chunk grid axis ("GSPN-2: Efficient Parallel
 * Sequence Modeling" paper notes, "Optimisation 1"). Negative: GSPN_ERR_INVALID_ARG. */
typedef struct {
    int N, C, H, W;
    int wmode;          /* gspn_wmode */
    unsigned dir_mask;  /* GSPN_DIR_* bits */
    int dtype;          /* gspn_dtype */
    int algo;           /* GSPN_ALGO_*, 0 = AUTO */
    int chunk;          /* lines per local chunk; 0 = global */
    int per_dir;        /* 1: lam and u have a direction axis (see below); 0: shared */
} gspn_desc;

/* per_dir = 1: lam and u are D x N x C x H x W (slots ordered as the logits' direction slots);
 * direction d's scan is driven by lam_d * x and the output is y = sum_d u_d * h^d, a learnable
 * per-pixel weighting of the directions (the pages' models merge the four directions with a
 * learnable merge: "Parallel Sequence Modeling via Generalized Spatial Propagation Network"
 * summary, section "Measured effects"). Gradients: dlam_d = x * delta^d, du_d = dy * h^d,
 * dx = sum_d lam_d * delta^d, with g^d = u_d * dy starting each reverse scan. The generic family
 * runs it forward and backward, the plane family forward; values other than 0 / 1:
 * GSPN_ERR_INVALID_ARG. */

/* Bytes of device workspace that gspn_forward (for_backward = 0) or gspn_backward
 * (for_backward = 1) needs for this descriptor; 0 if the descriptor is invalid or its
 * forced algo cannot run it. The first 256 bytes hold the device status word. */
GSPN_API size_t gspn_workspace_size(const gspn_desc *desc, int for_backward);

/* Kernel family that AUTO (or the forced algo) uses for this descriptor, or -1. */
GSPN_API int gspn_selected_algo(const gspn_desc *desc, int for_backward);

/* y = u * sum_d h^d (definition above). x, a, lam, u, y, ws: device pointers. */
GSPN_API gspn_status gspn_forward(const gspn_desc *desc, const void *x, const void *a, const void *lam,
                         const void *u, void *y, void *ws, size_t ws_bytes, void *stream);

/* Gradients of the scalar sum(dy * y) with respect to x, a, lam and u (reverse scans):
 *   g = u * dy; per direction delta_i = g_i + w_{i+1}^T delta_{i+1}; dz = sum_d delta^d;
 *   dx = lam * dz; dlam = x * dz; du = dy * sum_d h^d;
 *   da_k = s_k (1 - s_k) (dw_k - sum_k' w_k' dw_k') / S with dw_i[j][k] = delta_i[j] h_{i-1}[j+k-1],
 *   zero for out-of-range k and on the first step of each scan.
 * All pointers are device pointers; da has the layout of a. */
GSPN_API gspn_status gspn_backward(const gspn_desc *desc, const void *x, const void *a, const void *lam,
                          const void *u, const void *dy, void *dx, void *da, void *dlam, void *du,
                          void *ws, size_t ws_bytes, void *stream);

/* Training pair. gspn_forward_save is gspn_forward that also writes each direction's hidden
 * state h^d into hsave; gspn_backward_saved returns the gradients of gspn_backward reading h^d
 * from hsave instead of recomputing the forward scans (the reverse scans need h_{i-1} of every
 * line). hsave is caller-owned device memory of gspn_hsave_size bytes, fp32: slot k (the k-th
 * direction of the mask) at k * N * C * H * W floats, vertical directions in the image layout,
 * horizontal ones transposed per plane (W x H); it is only meaningful between a
 * gspn_forward_save and a gspn_backward_saved on the same inputs. The pair applies when AUTO
 * (or the forced algo) runs the forward on the plane family's concurrent-direction kernel and
 * the backward on the generic family's all-directions kernels; otherwise gspn_hsave_size
 * returns 0 and both calls return GSPN_ERR_UNSUPPORTED before any launch. Workspace: the same as
 * gspn_forward / gspn_backward. Argument errors as gspn_forward / gspn_backward. */
GSPN_API size_t gspn_hsave_size(const gspn_desc *desc);
GSPN_API gspn_status gspn_forward_save(const gspn_desc *desc, const void *x, const void *a, const void *lam,
                              const void *u, void *y, void *hsave, void *ws, size_t ws_bytes, void *stream);
GSPN_API gspn_status gspn_backward_saved(const gspn_desc *desc, const void *x, const void *a, const void *lam,
                                const void *u, const void *dy, const void *hsave, void *dx, void *da,
                                void *dlam, void *du, void *ws, size_t ws_bytes, void *stream);

/* gspn_forward that also records CUDA events around each kernel launch it makes, for
 * per-kernel timing on the launching stream: events[2k] before and events[2k+1] after launch k
 * (cudaEvent_t handles created by the caller). *n_launches receives the number of launches;
 * launches beyond n_events/2 are not timed. Otherwise identical to gspn_forward. */
GSPN_API gspn_status gspn_forward_timed(const gspn_desc *desc, const void *x, const void *a, const void *lam,
                               const void *u, void *y, void *ws, size_t ws_bytes, void *stream,
                               void *const *events, int n_events, int *n_launches);

/* Bytes of device staging buffer that gspn_forward_host needs (inputs, output and
 * workspace, each 256-byte aligned). */
GSPN_API size_t gspn_forward_host_buffer_size(const gspn_desc *desc);

/* End-to-end forward from HOST buffers: copies x, a, lam, u from host memory (pinned memory
 * gives asynchronous copies) into the caller's device buffer `dev`, runs gspn_forward there,
 * copies y back to host memory `hy` and synchronises `stream`. Returns the first error; once a
 * copy has been queued it synchronises `stream` before returning on every path, so the host
 * buffers may be reused as soon as the call returns. */
GSPN_API gspn_status gspn_forward_host(const gspn_desc *desc, const void *hx, const void *ha,
                              const void *hlam, const void *hu, void *hy, void *dev,
                              size_t dev_bytes, void *stream);

/* Synchronises `stream`, reads and clears the device status word at the start of `ws`.
 * Returns GSPN_OK, GSPN_ERR_DEVICE_TIMEOUT (a bounded device wait ran out) or GSPN_ERR_CUDA. */
GSPN_API gspn_status gspn_device_status(void *ws, void *stream);

/* Test hook for the failure path: launches one CTA that waits, through the same kind of bounded
 * wait the kernels' hand-offs use, on a flag in `ws` that nothing sets, giving up after
 * `limit_ns` nanoseconds and recording GSPN_ERR_DEVICE_TIMEOUT in the status word. */
GSPN_API gspn_status gspn_debug_wait_timeout(void *ws, size_t ws_bytes, unsigned long long limit_ns,
                                    void *stream);

/* Plain device-to-device copy of `bytes` (multiple of 16, 16-byte aligned pointers) with a
 * vectorised grid-stride kernel: the bandwidth ceiling the sweeps are compared with. */
GSPN_API gspn_status gspn_copy_ceiling(const void *src, void *dst, size_t bytes, void *stream);

/* Compressive channel proxy around the propagation ("GSPN-2: Efficient Parallel Sequence
 * Modeling" paper notes, "Optimisation 2: compact channel propagation": project the C channels
 * to a low-dimensional proxy, propagate there, restore with a 1x1 convolution):
 *     xp = P_in x,   yp = propagation of xp (gspn_forward),   y = P_out yp,
 * per pixel, with P_in a C_proxy x C and P_out a C x C_proxy matrix (row-major, storage dtype).
 * `desc` describes the proxy-space propagation: desc->C = C_proxy, and the logits a, lam and u
 * are in proxy space (shapes as for gspn_forward with C = C_proxy). x and y: N x c_full x H x W.
 * The projections are the library's own GEMM kernels: for bf16 storage with C and C_proxy
 * multiples of 8 and H*W a multiple of 8, tcgen05 tensor-core MMAs on TMA-loaded tiles (bf16
 * operands, fp32 accumulation); otherwise an exact fp32 GEMM on the CUDA cores. xp and yp live in
 * the workspace in the storage dtype. All pointers are device pointers. */
GSPN_API size_t gspn_proxy_workspace_size(const gspn_desc *desc, int c_full);
GSPN_API gspn_status gspn_proxy_forward(const gspn_desc *desc, int c_full, const void *x, const void *p_in,
                               const void *a, const void *lam, const void *u, const void *p_out,
                               void *y, void *ws, size_t ws_bytes, void *stream);

/* Size of the fixed device scratch array used by gspn_forward_noalloc (64 MiB). */
#define GSPN_NOALLOC_SCRATCH_BYTES (64u << 20)

/* gspn_forward without any allocation by anyone: the workspace comes from a fixed device array
 * of GSPN_NOALLOC_SCRATCH_BYTES compiled into the library (the pages have no counterpart; this
 * exists for callers that cannot allocate device memory at call time, e.g. code running under
 * another component's allocator or on a path where cudaMalloc/cudaFree would synchronise the
 * device). x, a, lam, u, y are device pointers on the current device; `stream` belongs to it.
 *   - Returns GSPN_ERR_INVALID_ARG for a malformed descriptor or a null pointer,
 *     GSPN_ERR_UNSUPPORTED for a well-formed one no kernel family runs, and GSPN_ERR_WORKSPACE,
 *     before touching the device, if the descriptor needs more workspace than
 *     GSPN_NOALLOC_SCRATCH_BYTES (gspn_workspace_size(desc, 0) tells).
 *   - Every call looks up the array's device address on the current device (a host-side query
 *     that allocates nothing), so the address stays right across a cudaDeviceReset.
 *   - Every call on a device shares the one array, which keeps the last call's contents (each
 *     call rewrites what it reads): calls that overlap on the GPU, from any stream or thread,
 *     race on it. Serialise them.
 *   - Every GPU that loads the library holds the array until the process exits. */
GSPN_API gspn_status gspn_forward_noalloc(const gspn_desc *desc, const void *x, const void *a,
                                          const void *lam, const void *u, void *y, void *stream);

GSPN_API const char *gspn_status_string(gspn_status s);
GSPN_API int gspn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GSPN_H */
