// k_plane.cu -- small-map kernel family of libgspn: the whole plane stays on chip.
//
// One CTA owns one (n, c) plane at a time (persistent over planes). Shared memory holds the
// plane's z = lambda * x, the running sum over directions and the current direction's weights,
// all fp32 with an odd row stride so that walking a row (vertical scans) or a column
// (horizontal scans) across the 32 lanes of a warp is bank-conflict-free. x, lambda and u are
// read once, every logit is read once, y is written once: the HBM traffic is the compulsory
// one. Per direction, all threads form the normalised weights from coalesced logit reads
// ("Parallel Sequence Modeling via Generalized Spatial Propagation Network" summary, section
// "Approach": sigmoid then normalisation over the in-range neighbours), then one warp runs the
// sequential scan with the line held in registers and the j +- 1 neighbours exchanged by warp
// shuffles ("GSPN-2: Efficient Parallel Sequence Modeling" paper notes, section "Optimisation 3":
// keep h_{i-1} on chip). Several CTAs per SM overlap one plane's scan with another's loads.
// Directions are added to the sum one after another in the fixed order TB, BT, LR, RL, so the
// result is deterministic.
#include <algorithm>

#include "gspn_common.cuh"
#include "gspn_internal.h"

namespace gspn {
namespace {

constexpr int kPlaneThreads = 128;
constexpr int kPlaneBwdThreads = 256;          // the backward runs one or two CTAs per SM: more warps
                                               // for its parallel phases
constexpr int kPlaneMaxLanes = 128;            // scan lanes held by one warp (4 per thread)
constexpr size_t kPlaneSmemBudget = 225 * 1024;

struct PlaneArgs {
    const void* x;
    const void* lam;
    const void* u;
    const void* a;
    void* y;
    int N, C, H, W, Cw, Wp;
    unsigned mask;
    int chunk;     // lines per local chunk (0: global)
    float* hsave;  // concurrent forward only, may be null: each direction's h for the backward,
                   // slot k (k-th direction of the mask) at k U, vertical slots in the image layout,
                   // horizontal ones transposed per plane ([W][H])
};

// Weights of one pixel for direction d (w1 = 1 - w0 - w2 is re-derived by the scan). Fast MUFU
// form; the rare max-shifted form for logits below -40 is applied behind a warp vote.
template <unsigned D>
__device__ __forceinline__ void pixel_weights(float a0, float a1, float a2, int r, int col, int H, int W,
                                              float& w0, float& w2) {
    constexpr bool V = D == kTB || D == kBT;
    const bool hl = V ? col > 0 : r > 0;
    const bool hr = V ? col < W - 1 : r < H - 1;
    Wts w = lane_weights_fast_nocheck(a0, a1, a2, hl, hr);
    const bool shift = weights_need_shift(a0, a1, a2, hl, hr);
    if (__any_sync(__activemask(), shift) && shift) w = weights_shifted(a0, a1, a2, hl, hr);
    w0 = w.w0;
    w2 = w.w2;
}

// Shared-memory offset of scan position (i, j) of direction D.
template <unsigned D>
__device__ __forceinline__ int plane_pix(int H, int W, int Wp, int i, int j) {
    if (D == kTB) return i * Wp + j;
    if (D == kBT) return (H - 1 - i) * Wp + j;
    if (D == kLR) return j * Wp + i;
    return j * Wp + (W - 1 - i);
}

// One warp scans the whole plane for direction D; lane j is held by thread j / LPT. Software
// pipelined: the shared-memory operands of step i + 1 (z, w0, w2 and the running sum) are
// loaded while step i's new line is formed, so a step waits only for the shuffles and FMAs of
// the recurrence. Lanes past the line (j >= M) read index 0 and contribute nothing.
// PD (per-direction lambda / u): the scan writes h^D over z (each z value is read before its
// pixel's h is written) and leaves the running sum to the caller, which weights h^D by u_D.
template <unsigned D, int LPT, bool LOCAL, bool PD = false>
__device__ __forceinline__ void plane_scan(float* z, const float* w0b, const float* w2b, float* acc, int H,
                                           int W, int Wp, int chunk, int lane) {
    constexpr bool V = D == kTB || D == kBT;
    const int L = V ? H : W, M = V ? W : H;
    float h[LPT], cz[LPT], cw0[LPT], cw2[LPT], ca[LPT];
    int cq[LPT];
    bool on[LPT];
    int crem = first_chunk_len(scan_ascending(D), L, chunk);   // steps left in this chunk
    const int clen = chunk > 0 ? chunk : L;
#pragma unroll
    for (int e = 0; e < LPT; ++e) {
        h[e] = 0.f;
        const int j = lane * LPT + e;
        on[e] = j < M;
        cq[e] = on[e] ? plane_pix<D>(H, W, Wp, 0, j) : 0;
        cz[e] = z[cq[e]];
        cw0[e] = 0.f;   // step 0 has no predecessor: h_0 = z
        cw2[e] = 0.f;
        ca[e] = PD ? 0.f : acc[cq[e]];
    }
    for (int i = 0; i < L; ++i) {
        // operands of step i + 1
        float nz[LPT], nw0[LPT], nw2[LPT], na[LPT];
        int nq[LPT];
        const bool more = i + 1 < L;
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            const int j = lane * LPT + e;
            nq[e] = (more && on[e]) ? plane_pix<D>(H, W, Wp, i + 1, j) : 0;
            nz[e] = z[nq[e]];
            nw0[e] = w0b[nq[e]];
            nw2[e] = w2b[nq[e]];
        }
        float hl = __shfl_up_sync(0xffffffffu, h[LPT - 1], 1);
        float hr = __shfl_down_sync(0xffffffffu, h[0], 1);
        if (lane == 0) hl = 0.f;
        if (lane == 31) hr = 0.f;
        float hn[LPT];
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            const float left = e == 0 ? hl : h[e - 1];
            const float right = e == LPT - 1 ? hr : h[e + 1];
            const float v = fmaf(cw0[e], left, fmaf(1.f - cw0[e] - cw2[e], h[e], fmaf(cw2[e], right, cz[e])));
            hn[e] = on[e] ? v : 0.f;
            if (on[e]) {
                if (PD) z[cq[e]] = v;
                else acc[cq[e]] = ca[e] + v;
            }
        }
        // the running sum of step i + 1 is read after this step's writes (different pixels
        // except at the same lane, which this thread owns); a chunk's first step starts from
        // h = 0 (local propagation; counted down, no division per step)
        bool restart = false;
        if constexpr (LOCAL) {
            restart = --crem == 0;
            if (restart) crem = clen;
        }
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            na[e] = PD ? 0.f : acc[nq[e]];
            h[e] = restart ? 0.f : hn[e];
            cz[e] = nz[e];
            cw0[e] = nw0[e];
            cw2[e] = nw2[e];
            ca[e] = na[e];
            cq[e] = nq[e];
        }
    }
}

// Weights of direction D for the whole plane into w0b / w2b (all threads; 4 pixels per
// iteration when a row is a multiple of 4 long).
template <typename T, unsigned D, int NT = kPlaneThreads>
__device__ __forceinline__ void plane_weights(const T* a3, float* w0b, float* w2b, int H, int W, int Wp, int tid) {
    const int HW = H * W;
    if (W % 4 == 0) {
        // each iteration's logits are loaded one iteration ahead, so the global-load latency is
        // paid about once per direction instead of once per iteration
        float a0[4], a1[4], a2[4];
        int e = tid * 4;
        if (e < HW) {
            ld_lanes<T, 4>(a3 + e, a0);
            ld_lanes<T, 4>(a3 + HW + e, a1);
            ld_lanes<T, 4>(a3 + 2 * HW + e, a2);
        }
        for (; e < HW; e += NT * 4) {
            float b0[4], b1[4], b2[4];
            const int en = e + NT * 4;
            if (en < HW) {
                ld_lanes<T, 4>(a3 + en, b0);
                ld_lanes<T, 4>(a3 + HW + en, b1);
                ld_lanes<T, 4>(a3 + 2 * HW + en, b2);
            }
            const int r = e / W, col = e - r * W;
#pragma unroll
            for (int k = 0; k < 4; ++k)
                pixel_weights<D>(a0[k], a1[k], a2[k], r, col + k, H, W, w0b[r * Wp + col + k], w2b[r * Wp + col + k]);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                a0[k] = b0[k];
                a1[k] = b1[k];
                a2[k] = b2[k];
            }
        }
    } else {
        for (int e = tid; e < HW; e += NT) {
            const int r = e / W, col = e - r * W;
            pixel_weights<D>(Io<T>::ld(a3 + e), Io<T>::ld(a3 + HW + e), Io<T>::ld(a3 + 2 * HW + e), r, col, H, W,
                             w0b[r * Wp + col], w2b[r * Wp + col]);
        }
    }
}

template <typename T, unsigned D, int LPT, bool LOCAL, bool PD = false>
__device__ __forceinline__ void plane_direction(const T* a3, float* z, float* w0b, float* w2b, float* acc, int H,
                                                int W, int Wp, int chunk, int tid) {
    plane_weights<T, D>(a3, w0b, w2b, H, W, Wp, tid);
    __syncthreads();
    if (tid < 32) plane_scan<D, LPT, LOCAL, PD>(z, w0b, w2b, acc, H, W, Wp, chunk, tid);
    __syncthreads();
}

// z = lam * x over the plane (all threads; plane layout with row stride Wp).
template <typename T>
__device__ __forceinline__ void plane_load_z(const T* x, const T* lam, float* z, int H, int W, int Wp, int tid) {
    const int HW = H * W;
    if (W % 4 == 0) {
        for (int e = tid * 4; e < HW; e += kPlaneThreads * 4) {
            const int r = e / W, col = e - r * W;
            float xv[4], lv[4];
            ld_lanes<T, 4>(x + e, xv);
            ld_lanes<T, 4>(lam + e, lv);
#pragma unroll
            for (int k = 0; k < 4; ++k) z[r * Wp + col + k] = lv[k] * xv[k];
        }
    } else {
        for (int e = tid; e < HW; e += kPlaneThreads) {
            const int r = e / W, col = e - r * W;
            z[r * Wp + col] = Io<T>::ld(lam + e) * Io<T>::ld(x + e);
        }
    }
}

// acc (+)= g * src over the plane, g a storage-dtype tensor in image layout (all threads).
template <typename T, bool FIRST>
__device__ __forceinline__ void plane_axpy(const T* g, const float* src, float* acc, int H, int W, int Wp, int tid) {
    const int HW = H * W;
    for (int e = tid; e < HW; e += kPlaneThreads) {
        const int q = (e / W) * Wp + e % W;
        const float v = Io<T>::ld(g + e) * src[q];
        acc[q] = FIRST ? v : acc[q] + v;
    }
}

template <typename T, int LPT, bool LOCAL, bool PD>
__global__ void __launch_bounds__(kPlaneThreads) k_plane_fwd(PlaneArgs p) {
    extern __shared__ float sm[];
    const int H = p.H, W = p.W, Wp = p.Wp;
    const int HWs = H * Wp;
    float* z = sm;
    float* acc = z + HWs;
    float* w0b = acc + HWs;
    float* w2b = w0b + HWs;
    const int tid = threadIdx.x;
    const int HW = H * W;
    const int nplanes = p.N * p.C;
    const long long U = (long long)nplanes * HW;   // one N x C x H x W tensor (per-direction stride)
    for (int plane = blockIdx.x; plane < nplanes; plane += gridDim.x) {
        const int n = plane / p.C, c = plane % p.C;
        const long long po = (long long)plane * HW;
        const T* x = (const T*)p.x + po;
        T* y = (T*)p.y + po;
        // shared lam / u: z = lambda * x once and sum = 0; per-direction: sum = 0 (z per direction)
        if (!PD) plane_load_z<T>(x, (const T*)p.lam + po, z, H, W, Wp, tid);
        for (int e = tid; e < HW; e += kPlaneThreads) acc[(e / W) * Wp + e % W] = 0.f;
        int slot = 0;
        auto a_of = [&](int s) {
            return (const T*)p.a + (((long long)s * p.N + n) * p.Cw + (p.Cw == 1 ? 0 : c)) * 3 * HW;
        };
        // per-direction lam / u: z = lam_s x before the direction (its first barrier orders it),
        // the scan leaves h^D in z, and sum += u_s h^D after it
        auto pre = [&](int s) {
            if (PD) plane_load_z<T>(x, (const T*)p.lam + s * U + po, z, H, W, Wp, tid);
        };
        auto post = [&](int s) {
            if (PD) {
                plane_axpy<T, false>((const T*)p.u + s * U + po, z, acc, H, W, Wp, tid);
                __syncthreads();
            }
        };
        if (p.mask & kTB) { pre(slot); plane_direction<T, kTB, LPT, LOCAL, PD>(a_of(slot), z, w0b, w2b, acc, H, W, Wp, p.chunk, tid); post(slot++); }
        if (p.mask & kBT) { pre(slot); plane_direction<T, kBT, LPT, LOCAL, PD>(a_of(slot), z, w0b, w2b, acc, H, W, Wp, p.chunk, tid); post(slot++); }
        if (p.mask & kLR) { pre(slot); plane_direction<T, kLR, LPT, LOCAL, PD>(a_of(slot), z, w0b, w2b, acc, H, W, Wp, p.chunk, tid); post(slot++); }
        if (p.mask & kRL) { pre(slot); plane_direction<T, kRL, LPT, LOCAL, PD>(a_of(slot), z, w0b, w2b, acc, H, W, Wp, p.chunk, tid); post(slot++); }
        // y = u * sum (shared u) or y = sum (per-direction u already applied)
        const T* u = (const T*)p.u + po;
        if (W % 4 == 0) {
            for (int e = tid * 4; e < HW; e += kPlaneThreads * 4) {
                const int r = e / W, col = e - r * W;
                float uv[4] = {1.f, 1.f, 1.f, 1.f};
                if (!PD) ld_lanes<T, 4>(u + e, uv);
#pragma unroll
                for (int k = 0; k < 4; ++k) uv[k] *= acc[r * Wp + col + k];
                st_lanes<T, 4>(y + e, uv);
            }
        } else {
            for (int e = tid; e < HW; e += kPlaneThreads) {
                const int r = e / W, col = e - r * W;
                Io<T>::st(y + e, (PD ? 1.f : Io<T>::ld(u + e)) * acc[r * Wp + col]);
            }
        }
        __syncthreads();
    }
}

// ====================================================== forward, directions scanned concurrently
// fp32 storage. The four line scans of a plane are independent given z = lambda x and are only
// added at the end ("GSPN-2: Efficient Parallel Sequence Modeling" paper notes, section "2D
// spatial propagation review": one scan per direction, then the merge), so they run at the same
// time here: one CTA per plane (persistent over planes), one warp per direction, each warp
// writing its h^d to a plane buffer of its own; y = u * (h^TB + h^BT + h^LR + h^RL) is then
// summed in that fixed order, so the result does not depend on warp timing. Each scanning warp
// streams its three logit planes through a ring of NSL strips of K = 16 / sizeof(T) scan lines
// filled with 16-byte cp.async copies that bypass L1: the logits are read from HBM exactly once,
// and the transposed walks of the horizontal directions read one 16-byte run per lane and
// strip. The weights of a whole strip are formed before its K recurrence steps, off the h chain.
// Lane j of a scan line is held by thread j % 32 as its element j / 32 (interleaved), which keeps
// every row and column walk of the odd-stride planes conflict-free.

__device__ __forceinline__ uint32_t cd_saddr(const void* ptr) { return (uint32_t)__cvta_generic_to_shared(ptr); }
__device__ __forceinline__ void cd_cp16(void* dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(cd_saddr(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cd_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cd_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Float offset of the rings in shared memory: after z and the nd h planes, rounded up to 16 bytes.
__host__ __device__ constexpr int cd_ring_offset(int nd, int HWs) { return ((1 + nd) * HWs + 3) & ~3; }
// The same for h planes of hbytes per element (the forward keeps them in the storage type: bf16
// planes take half the shared memory, so more CTAs fit on an SM; the sum over directions is then
// formed from h rounded to bf16, well inside the bf16 output's tolerance).
__host__ __device__ constexpr int cd_ring_offset_h(int nd, int HWs, int hbytes) {
    return ((HWs * 4 + nd * HWs * hbytes + 15) / 16) * 4;
}

template <typename T> struct CdGeom {
    static constexpr int K = 16 / (int)sizeof(T);   // scan lines per ring strip = elements per 16 bytes
};
// 32-bit words of one ring strip: 3 logit planes x K lines x 32 LPT lanes (both storage types).
template <int LPT> __host__ __device__ constexpr int cd_slot_words() { return 384 * LPT; }

// Geometry of one direction as seen by its scanning warp. Scan position (i, j) (line i, lane j)
// is plane-buffer element p0 + i si + j sj (row stride Wp) and image element g0 + i gi + j gj.
// The direction is a runtime value so that the four warps of a CTA run the same instructions.
struct CdDir {
    bool vert, asc;
    int L, M;
    int p0, si, sj;
    int g0, gi, gj;
    int s0, ssi;   // the direction's scan layout (line i, lane j at s0 + i ssi + j): the image for
                   // vertical directions, the transposed plane (W x H) for horizontal ones
};

__device__ __forceinline__ CdDir cd_dir(unsigned d, int H, int W, int Wp) {
    CdDir g;
    g.vert = d == kTB || d == kBT;
    g.asc = d == kTB || d == kLR;
    g.L = g.vert ? H : W;
    g.M = g.vert ? W : H;
    if (d == kTB) { g.p0 = 0; g.si = Wp; g.sj = 1; g.g0 = 0; g.gi = W; g.gj = 1; g.s0 = 0; g.ssi = W; }
    else if (d == kBT) {
        g.p0 = (H - 1) * Wp; g.si = -Wp; g.sj = 1; g.g0 = (H - 1) * W; g.gi = -W; g.gj = 1;
        g.s0 = (H - 1) * W; g.ssi = -W;
    } else if (d == kLR) { g.p0 = 0; g.si = 1; g.sj = Wp; g.g0 = 0; g.gi = 1; g.gj = W; g.s0 = 0; g.ssi = H; }
    else { g.p0 = W - 1; g.si = -1; g.sj = Wp; g.g0 = W - 1; g.gi = -1; g.gj = W; g.s0 = (W - 1) * H; g.ssi = -H; }
    return g;
}

// Issues the copies of strip q (scan lines q K .. q K + K - 1) into one ring slot, all 16-byte
// cp.async that bypass L1 (image rows are a multiple of 16 bytes). Vertical strips: the K image
// rows are copied chunk by chunk (the warp's 32 copies cover consecutive chunks) and land
// line-major, element (k, s, j) at element offset (k K + s) 32 LPT + j. Horizontal strips: every
// lane (image row) j copies its own 16-byte run of K columns of each logit plane to chunk
// k 32 LPT + j, read back whole by that thread. Copies past the plane are skipped.
template <typename T, int LPT>
__device__ __forceinline__ void cd_fetch(uint32_t* slot, const T* a3, const CdDir& g, int HW, int W, int q, int lane) {
    constexpr int K = CdGeom<T>::K;
    const int i0 = q * K;
    if (g.vert) {
        const int nc = g.M / K;               // chunks per image row
        const int rows = min(K, g.L - i0);    // lines of this strip inside the plane
        const int per_k = rows * nc;
        T* dst0 = reinterpret_cast<T*>(slot);
        for (int idx = lane; idx < 3 * per_k; idx += 32) {
            const int k = idx / per_k, rem = idx - k * per_k;
            const int s = rem / nc, c = rem - s * nc;
            cd_cp16(dst0 + (k * K + s) * 32 * LPT + c * K, a3 + k * HW + g.g0 + (i0 + s) * g.gi + c * K);
        }
    } else {
        const int col = g.asc ? i0 : W - K - i0;   // first column of the run
#pragma unroll
        for (int k = 0; k < 3; ++k)
#pragma unroll
            for (int e = 0; e < LPT; ++e) {
                const int j = e * 32 + lane;
                if (j < g.M) cd_cp16(slot + (k * 32 * LPT + j) * 4, a3 + k * HW + j * W + col);
            }
    }
}

// Logits of KH lines of the strip (lines s0 .. s0 + KH - 1) for this thread's lanes:
// lg[k][s][e] = logit k of line s0 + s, lane e 32 + lane.
template <typename T, int LPT, int KH>
__device__ __forceinline__ void cd_strip_logits(const uint32_t* slot, const CdDir& g, int lane, int s0,
                                                float (&lg)[3][KH][LPT]) {
    constexpr int K = CdGeom<T>::K;
    if (g.vert) {
        const T* src = reinterpret_cast<const T*>(slot);
#pragma unroll
        for (int k = 0; k < 3; ++k)
#pragma unroll
            for (int s = 0; s < KH; ++s)
#pragma unroll
                for (int e = 0; e < LPT; ++e)
                    lg[k][s][e] = Io<T>::ld(src + (k * K + s0 + s) * 32 * LPT + e * 32 + lane);
    } else {
#pragma unroll
        for (int k = 0; k < 3; ++k)
#pragma unroll
            for (int e = 0; e < LPT; ++e) {
                const uint4 v = reinterpret_cast<const uint4*>(slot)[k * 32 * LPT + e * 32 + lane];
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                float f[K];   // columns in ascending order
                if constexpr (sizeof(T) == 4) {
#pragma unroll
                    for (int q = 0; q < 4; ++q) f[q] = __uint_as_float(w[q]);
                } else {
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 t = unpack2<T>(w[q]);
                        f[2 * q] = t.x;
                        f[2 * q + 1] = t.y;
                    }
                }
#pragma unroll
                for (int s = 0; s < KH; ++s) lg[k][s][e] = g.asc ? f[s0 + s] : f[K - 1 - s0 - s];
            }
    }
}

// Issues the first NSL strips (one commit group per strip, empty past the end).
template <typename T, int LPT, int NSL>
__device__ __forceinline__ void cd_prime(uint32_t* ring, const T* a3, const CdDir& g, int HW, int W, int lane) {
    constexpr int K = CdGeom<T>::K;
    const int nq = (g.L + K - 1) / K;
#pragma unroll
    for (int q = 0; q < NSL; ++q) {
        if (q < nq) cd_fetch<T, LPT>(ring + q * cd_slot_words<LPT>(), a3, g, HW, W, q, lane);
        cd_commit();
    }
}

// Scan of one direction by one warp: h of the plane into hb (plane layout, row stride Wp). The
// ring already holds strips 0 .. NSL - 1 (issued by cd_prime).
template <typename T, int LPT, bool LOCAL, int NSL, typename HB = float>
__device__ __forceinline__ void cd_scan(const float* z, HB* hb, uint32_t* ring, const T* a3, const CdDir& g,
                                        int HW, int W, int chunk, int lane, float* hg = nullptr) {
    constexpr int K = CdGeom<T>::K;
    constexpr int SLOT = cd_slot_words<LPT>();
    const int L = g.L, M = g.M;
    const int nq = (L + K - 1) / K;
    float h[LPT];
    bool on[LPT], hl[LPT], hr[LPT];
    int pj[LPT];   // plane offset of (line 0, lane j)
#pragma unroll
    for (int e = 0; e < LPT; ++e) {
        const int j = e * 32 + lane;
        h[e] = 0.f;
        on[e] = j < M;
        hl[e] = j > 0;
        hr[e] = j < M - 1;
        pj[e] = on[e] ? g.p0 + j * g.sj : 0;
    }
    int crem = first_chunk_len(g.asc, L, chunk);   // lines left in this chunk
    const int clen = chunk > 0 ? chunk : L;
    constexpr int KH = 4;                // lines whose weights are formed together
    for (int q = 0; q < nq; ++q) {
        cd_wait<NSL - 1>();
        __syncwarp();
        uint32_t* slot = ring + (q % NSL) * SLOT;
#pragma unroll
        for (int s0 = 0; s0 < K; s0 += KH) {
            // normalised weights of KH lines of the strip (independent of h)
            float w0[KH][LPT], w2[KH][LPT];
            bool shift = false;
            {
                float lg[3][KH][LPT];
                cd_strip_logits<T, LPT, KH>(slot, g, lane, s0, lg);
#pragma unroll
                for (int s = 0; s < KH; ++s)
#pragma unroll
                    for (int e = 0; e < LPT; ++e) {
                        const Wts w = lane_weights_fast_nocheck(lg[0][s][e], lg[1][s][e], lg[2][s][e], hl[e], hr[e]);
                        shift |= on[e] && q * K + s0 + s < L &&
                                 weights_need_shift(lg[0][s][e], lg[1][s][e], lg[2][s][e], hl[e], hr[e]);
                        w0[s][e] = w.w0;
                        w2[s][e] = w.w2;
                    }
                if (__any_sync(0xffffffffu, shift)) {   // rare: some logit below the fast form's range
#pragma unroll
                    for (int s = 0; s < KH; ++s)
#pragma unroll
                        for (int e = 0; e < LPT; ++e)
                            if (weights_need_shift(lg[0][s][e], lg[1][s][e], lg[2][s][e], hl[e], hr[e])) {
                                const Wts w = weights_shifted(lg[0][s][e], lg[1][s][e], lg[2][s][e], hl[e], hr[e]);
                                w0[s][e] = w.w0;
                                w2[s][e] = w.w2;
                            }
                }
            }
            if (s0 + KH == K) {
                // the strip's logits are consumed: refill its slot now, NSL strips ahead of use
                __syncwarp();
                if (q + NSL < nq) cd_fetch<T, LPT>(slot, a3, g, HW, W, q + NSL, lane);
                cd_commit();
            }
#pragma unroll
            for (int s = 0; s < KH; ++s) {
                const int i = q * K + s0 + s;
                if (i < L) {   // warp-uniform
                    const int di = i * g.si;
                    float zi[LPT];
#pragma unroll
                    for (int e = 0; e < LPT; ++e) zi[e] = z[on[e] ? pj[e] + di : 0];
                    // neighbours j - 1 and j + 1: rotate each element across the warp by one lane;
                    // lane 0 / 31 take the wrapped value of the previous / next element
                    float rl[LPT], rr[LPT];
#pragma unroll
                    for (int e = 0; e < LPT; ++e) {
                        rl[e] = __shfl_sync(0xffffffffu, h[e], (lane + 31) & 31);
                        rr[e] = __shfl_sync(0xffffffffu, h[e], (lane + 1) & 31);
                    }
                    bool restart = false;
                    if constexpr (LOCAL) {
                        restart = --crem == 0;
                        if (restart) crem = clen;
                    }
#pragma unroll
                    for (int e = 0; e < LPT; ++e) {
                        const float left = lane > 0 ? rl[e] : (e > 0 ? rl[e - 1] : 0.f);
                        const float right = lane < 31 ? rr[e] : (e < LPT - 1 ? rr[e + 1] : 0.f);
                        const float a = w0[s][e], c = w2[s][e];
                        const float v = fmaf(a, left, fmaf(1.f - a - c, h[e], fmaf(c, right, zi[e])));
                        if (on[e]) {
                            Io<HB>::st(hb + pj[e] + di, v);
                            // h for the backward, fp32 in the scan layout (a warp's lanes are
                            // consecutive there, so the store is coalesced)
                            if (hg) hg[g.s0 + i * g.ssi + e * 32 + lane] = v;
                        }
                        h[e] = (on[e] && !restart) ? v : 0.f;
                    }
                }
            }
        }
    }
}

constexpr int kCdThreads = 128;   // one warp per direction

template <typename T, int LPT, bool LOCAL, int NSL>
__global__ void __launch_bounds__(kCdThreads) k_plane_fwd_cd(PlaneArgs p) {
    extern __shared__ __align__(16) float sm[];
    constexpr int UNR = 4;   // vectors of 4 per thread whose loads are in flight together
    const int H = p.H, W = p.W, Wp = p.Wp;
    const int HW = H * W, HWs = H * Wp;
    const int nd = __popc(p.mask);
    float* z = sm;
    T* hb = reinterpret_cast<T*>(z + HWs);                      // nd planes (storage type), slot order
    // nd rings of NSL strips, 16-byte aligned for the copies and the 16-byte reads
    uint32_t* rings = reinterpret_cast<uint32_t*>(sm + cd_ring_offset_h(nd, HWs, (int)sizeof(T)));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    // this warp's direction: the warp-th set bit of the mask (its logit slot is warp)
    unsigned dir = 0;
    {
        unsigned m = p.mask;
        for (int k = 0; k < warp && m; ++k) m &= m - 1;
        dir = m & (0u - m);
    }
    const CdDir geo = cd_dir(dir, H, W, Wp);
    const bool scans = warp < nd;
    uint32_t* ring = rings + warp * NSL * cd_slot_words<LPT>();
    T* hw = hb + warp * HWs;
    const int nplanes = p.N * p.C;
    for (int plane = blockIdx.x; plane < nplanes; plane += gridDim.x) {
        const int n = plane / p.C, c = plane % p.C;
        const long long po = (long long)plane * HW;
        const T* a3 = (const T*)p.a + (((long long)warp * p.N + n) * p.Cw + (p.Cw == 1 ? 0 : c)) * 3 * HW;
        // the first logit strips go out before z is formed
        if (scans) cd_prime<T, LPT, NSL>(ring, a3, geo, HW, W, lane);
        {
            const T* x = (const T*)p.x + po;
            const T* lam = (const T*)p.lam + po;
            for (int e0 = tid * 4; e0 < HW; e0 += kCdThreads * 4 * UNR) {
                float xv[UNR][4], lv[UNR][4];
#pragma unroll
                for (int r = 0; r < UNR; ++r) {
                    const int e = e0 + r * kCdThreads * 4;
                    if (e < HW) {
                        ld_lanes<T, 4>(x + e, xv[r]);
                        ld_lanes<T, 4>(lam + e, lv[r]);
                    }
                }
#pragma unroll
                for (int r = 0; r < UNR; ++r) {
                    const int e = e0 + r * kCdThreads * 4;
                    if (e < HW) {
                        const int row = e / W, col = e - row * W;
#pragma unroll
                        for (int k = 0; k < 4; ++k) z[row * Wp + col + k] = lv[r][k] * xv[r][k];
                    }
                }
            }
        }
        __syncthreads();
        if (scans)
            cd_scan<T, LPT, LOCAL, NSL, T>(z, hw, ring, a3, geo, HW, W, p.chunk, lane,
                                           p.hsave ? p.hsave + (long long)warp * p.N * p.C * HW + po : nullptr);
        __syncthreads();
        // y = u * sum_d h^d, summed in slot order
        {
            const T* u = (const T*)p.u + po;
            T* y = (T*)p.y + po;
            for (int e0 = tid * 4; e0 < HW; e0 += kCdThreads * 4 * UNR) {
                float uv[UNR][4];
#pragma unroll
                for (int r = 0; r < UNR; ++r) {
                    const int e = e0 + r * kCdThreads * 4;
                    if (e < HW) ld_lanes<T, 4>(u + e, uv[r]);
                }
#pragma unroll
                for (int r = 0; r < UNR; ++r) {
                    const int e = e0 + r * kCdThreads * 4;
                    if (e < HW) {
                        const int row = e / W, col = e - row * W;
                        float v[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const int q = row * Wp + col + k;
                            float s = Io<T>::ld(hb + q);
                            for (int d = 1; d < nd; ++d) s += Io<T>::ld(hb + d * HWs + q);
                            v[k] = uv[r][k] * s;
                        }
                        st_lanes<T, 4>(y + e, v);
                    }
                }
            }
        }
        // the next plane's z and h writes come after its first barrier, which every thread
        // reaches only after this plane's sum
    }
}

// ================================================================== backward (per-channel)
struct PlaneBwdArgs {
    const void* x;
    const void* lam;
    const void* u;
    const void* a;
    const void* dy;
    void* dx;
    void* da;
    void* dlam;
    void* du;
    int N, C, H, W, Wp;
    unsigned mask;
    int chunk;   // lines per local chunk (0: global)
};

// Forward recompute of direction D by one warp: hb = h^D (plane layout), acc += h^D. Software
// pipelined like plane_scan.
template <unsigned D, int LPT, bool LOCAL>
__device__ __forceinline__ void plane_recompute(const float* z, const float* w0b, const float* w2b, float* hb,
                                                float* acc, int H, int W, int Wp, int chunk, int lane) {
    constexpr bool V = D == kTB || D == kBT;
    const int L = V ? H : W, M = V ? W : H;
    float h[LPT], cz[LPT], cw0[LPT], cw2[LPT];
    int cq[LPT];
    bool on[LPT];
    int crem = first_chunk_len(scan_ascending(D), L, chunk);   // steps left in this chunk
    const int clen = chunk > 0 ? chunk : L;
#pragma unroll
    for (int e = 0; e < LPT; ++e) {
        h[e] = 0.f;
        const int j = lane * LPT + e;
        on[e] = j < M;
        cq[e] = on[e] ? plane_pix<D>(H, W, Wp, 0, j) : 0;
        cz[e] = z[cq[e]];
        cw0[e] = cw2[e] = 0.f;   // step 0: h_0 = z
    }
    for (int i = 0; i < L; ++i) {
        float nz[LPT], nw0[LPT], nw2[LPT];
        int nq[LPT];
        const bool more = i + 1 < L;
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            nq[e] = (more && on[e]) ? plane_pix<D>(H, W, Wp, i + 1, lane * LPT + e) : 0;
            nz[e] = z[nq[e]];
            nw0[e] = w0b[nq[e]];
            nw2[e] = w2b[nq[e]];
        }
        float hl = __shfl_up_sync(0xffffffffu, h[LPT - 1], 1);
        float hr = __shfl_down_sync(0xffffffffu, h[0], 1);
        if (lane == 0) hl = 0.f;
        if (lane == 31) hr = 0.f;
        float hn[LPT];
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            const float left = e == 0 ? hl : h[e - 1];
            const float right = e == LPT - 1 ? hr : h[e + 1];
            const float v = fmaf(cw0[e], left, fmaf(1.f - cw0[e] - cw2[e], h[e], fmaf(cw2[e], right, cz[e])));
            hn[e] = on[e] ? v : 0.f;
            if (on[e]) {
                hb[cq[e]] = v;
                acc[cq[e]] += v;
            }
        }
        bool restart = false;
        if constexpr (LOCAL) {
            restart = --crem == 0;
            if (restart) crem = clen;
        }
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            h[e] = restart ? 0.f : hn[e];
            cz[e] = nz[e];
            cw0[e] = nw0[e];
            cw2[e] = nw2[e];
            cq[e] = nq[e];
        }
    }
}

// Reverse scan of direction D by one warp, delta only (no global memory):
//   delta_i[j] = g_i[j] + w_{i+1}[j-1][2] delta_{i+1}[j-1] + w_{i+1}[j][1] delta_{i+1}[j]
//                + w_{i+1}[j+1][0] delta_{i+1}[j+1]
// into db (plane layout), and dz += delta. The operands of step i - 1 are loaded while step i
// is formed.
template <unsigned D, int LPT, bool LOCAL>
__device__ __forceinline__ void plane_reverse(const float* g, const float* w0b, const float* w2b, float* db, float* dz,
                                             int H, int W, int Wp, int chunk, int lane) {
    constexpr bool V = D == kTB || D == kBT;
    const int L = V ? H : W, M = V ? W : H;
    float del[LPT], pw0[LPT], pw1[LPT], pw2[LPT];   // delta and weights of step i + 1
    float cg[LPT], cw0[LPT], cw2[LPT];              // g and weights of step i
    // steps from the start of the chunk holding step i (0: step i starts a chunk), counted down
    const int cfirst = first_chunk_len(scan_ascending(D), L, chunk);
    const int clen = chunk > 0 ? chunk : L;
    int kin = L - 1 < cfirst ? L - 1 : (L - 1 - cfirst) % clen;
    int cq[LPT];
    bool on[LPT];
#pragma unroll
    for (int e = 0; e < LPT; ++e) {
        del[e] = pw0[e] = pw1[e] = pw2[e] = 0.f;
        const int j = lane * LPT + e;
        on[e] = j < M;
        cq[e] = on[e] ? plane_pix<D>(H, W, Wp, L - 1, j) : 0;
        cg[e] = g[cq[e]];
        cw0[e] = w0b[cq[e]];
        cw2[e] = w2b[cq[e]];
    }
    for (int i = L - 1; i >= 0; --i) {
        float ng[LPT], nw0[LPT], nw2[LPT];
        int nq[LPT];
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            nq[e] = (i > 0 && on[e]) ? plane_pix<D>(H, W, Wp, i - 1, lane * LPT + e) : 0;
            ng[e] = g[nq[e]];
            nw0[e] = w0b[nq[e]];
            nw2[e] = w2b[nq[e]];
        }
        // neighbour terms of w_{i+1}^T delta_{i+1}: lane j-1's (w2 delta) and lane j+1's (w0 delta)
        float fromL = __shfl_up_sync(0xffffffffu, pw2[LPT - 1] * del[LPT - 1], 1);
        float fromR = __shfl_down_sync(0xffffffffu, pw0[0] * del[0], 1);
        if (lane == 0) fromL = 0.f;
        if (lane == 31) fromR = 0.f;
        float dn[LPT];
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            const float l = e == 0 ? fromL : pw2[e - 1] * del[e - 1];
            const float r = e == LPT - 1 ? fromR : pw0[e + 1] * del[e + 1];
            const float d = fmaf(pw1[e], del[e], cg[e]) + l + r;
            dn[e] = on[e] ? d : 0.f;
            if (on[e]) {
                db[cq[e]] = d;
                dz[cq[e]] += d;
            }
        }
        // step i's weights become the "next step" weights of step i - 1; a step that starts a
        // chunk (step 0 included) does not see h_{i-1}, so nothing flows back through it
        bool live = i != 0;
        if constexpr (LOCAL) {
            live = kin != 0;
            kin = kin != 0 ? kin - 1 : (i - 1 < cfirst ? i - 1 : clen - 1);
        }
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            del[e] = dn[e];
            pw0[e] = (on[e] && live) ? cw0[e] : 0.f;
            pw2[e] = (on[e] && live) ? cw2[e] : 0.f;
            pw1[e] = (on[e] && live) ? 1.f - cw0[e] - cw2[e] : 0.f;
            cg[e] = ng[e];
            cw0[e] = nw0[e];
            cw2[e] = nw2[e];
            cq[e] = nq[e];
        }
    }
}

// Logit gradients of direction D for the whole plane (all threads, image order, vector loads
// and stores when W % 4 == 0): at scan position (i, j) with i > 0,
//   dw_k = delta_i[j] h_{i-1}[j+k-1],  da_k = w_k sigmoid(-a_k) (dw_k - sum_k' w_k' dw_k')
// (zero for out-of-range k); row i = 0 has zero gradient (its weights multiply h_{-1} = 0).
template <typename T, unsigned D, int NT>
__device__ __forceinline__ void plane_logit_grads(const T* a3, T* da3, const float* w0b, const float* w2b,
                                                  const float* hb, const float* db, int H, int W, int Wp, int chunk,
                                                  int tid) {
    constexpr bool V = D == kTB || D == kBT;
    const int M = V ? W : H;
    const int HW = H * W;
    auto grad = [&](float a0, float a1, float a2, int r, int c, float& g0, float& g1, float& g2) {
        const int i = D == kTB ? r : D == kBT ? H - 1 - r : D == kLR ? c : W - 1 - c;
        const int j = V ? c : r;
        g0 = g1 = g2 = 0.f;
        if (!chunk_start(scan_ascending(D), V ? H : W, chunk, i)) {
            const int q = r * Wp + c;
            const float w0 = w0b[q], w2 = w2b[q], w1 = 1.f - w0 - w2;
            const bool hasl = j > 0, hasr = j < M - 1;
            const float d = db[q];
            const float h0 = hasl ? hb[plane_pix<D>(H, W, Wp, i - 1, j - 1)] : 0.f;
            const float h1 = hb[plane_pix<D>(H, W, Wp, i - 1, j)];
            const float h2 = hasr ? hb[plane_pix<D>(H, W, Wp, i - 1, j + 1)] : 0.f;
            const float dw0 = d * h0, dw1 = d * h1, dw2 = d * h2;
            const float sdw = w0 * dw0 + w1 * dw1 + w2 * dw2;
            // sigmoid(-a) = 1 / (1 + exp(a)) from the MUFU exponential (relative error a few ulp,
            // far inside the gradient tolerance); the argument is clamped at 80 so exp stays
            // finite (sigmoid(-80) is 2e-35, indistinguishable from the limit 0 here)
            auto sgm = [](float a) { return __fdividef(1.f, 1.f + __expf(fminf(a, 80.f))); };
            g0 = hasl ? w0 * sgm(a0) * (dw0 - sdw) : 0.f;
            g1 = w1 * sgm(a1) * (dw1 - sdw);
            g2 = hasr ? w2 * sgm(a2) * (dw2 - sdw) : 0.f;
        }
    };
    if (W % 4 == 0) {
        for (int e = tid * 4; e < HW; e += NT * 4) {
            const int r = e / W, c = e - r * W;
            float a0[4], a1[4], a2[4], g0[4], g1[4], g2[4];
            ld_lanes<T, 4>(a3 + e, a0);
            ld_lanes<T, 4>(a3 + HW + e, a1);
            ld_lanes<T, 4>(a3 + 2 * HW + e, a2);
#pragma unroll
            for (int k = 0; k < 4; ++k) grad(a0[k], a1[k], a2[k], r, c + k, g0[k], g1[k], g2[k]);
            st_lanes<T, 4>(da3 + e, g0);
            st_lanes<T, 4>(da3 + HW + e, g1);
            st_lanes<T, 4>(da3 + 2 * HW + e, g2);
        }
    } else {
        for (int e = tid; e < HW; e += NT) {
            const int r = e / W, c = e - r * W;
            float g0, g1, g2;
            grad(Io<T>::ld(a3 + e), Io<T>::ld(a3 + HW + e), Io<T>::ld(a3 + 2 * HW + e), r, c, g0, g1, g2);
            Io<T>::st(da3 + e, g0);
            Io<T>::st(da3 + HW + e, g1);
            Io<T>::st(da3 + 2 * HW + e, g2);
        }
    }
}

template <typename T, unsigned D, int LPT, bool LOCAL>
__device__ __forceinline__ void plane_bwd_direction(const T* a3, T* da3, const float* z, const float* g, float* w0b,
                                                    float* w2b, float* hb, float* db, float* acc, float* dz, int H,
                                                    int W, int Wp, int chunk, int tid) {
    plane_weights<T, D, kPlaneBwdThreads>(a3, w0b, w2b, H, W, Wp, tid);
    __syncthreads();
    if (tid < 32) {
        plane_recompute<D, LPT, LOCAL>(z, w0b, w2b, hb, acc, H, W, Wp, chunk, tid);
        __syncwarp();
        plane_reverse<D, LPT, LOCAL>(g, w0b, w2b, db, dz, H, W, Wp, chunk, tid);
    }
    __syncthreads();
    plane_logit_grads<T, D, kPlaneBwdThreads>(a3, da3, w0b, w2b, hb, db, H, W, Wp, chunk, tid);
    __syncthreads();
}

template <typename T, int LPT, bool LOCAL>
__global__ void __launch_bounds__(kPlaneBwdThreads) k_plane_bwd(PlaneBwdArgs p) {
    extern __shared__ float sm[];
    const int H = p.H, W = p.W, Wp = p.Wp;
    const int HWs = H * Wp;
    float* z = sm;
    float* g = z + HWs;
    float* acc = g + HWs;
    float* dz = acc + HWs;
    float* hb = dz + HWs;
    float* db = hb + HWs;
    float* w0b = db + HWs;
    float* w2b = w0b + HWs;
    const int tid = threadIdx.x;
    const int HW = H * W;
    const int nplanes = p.N * p.C;
    for (int plane = blockIdx.x; plane < nplanes; plane += gridDim.x) {
        const int n = plane / p.C, c = plane % p.C;
        const long long po = (long long)plane * HW;
        const T *x = (const T*)p.x + po, *lam = (const T*)p.lam + po, *u = (const T*)p.u + po, *dy = (const T*)p.dy + po;
        for (int e = tid; e < HW; e += kPlaneBwdThreads) {
            const int q = (e / W) * Wp + e % W;
            z[q] = Io<T>::ld(lam + e) * Io<T>::ld(x + e);
            g[q] = Io<T>::ld(u + e) * Io<T>::ld(dy + e);
            acc[q] = 0.f;
            dz[q] = 0.f;
        }
        __syncthreads();
        int slot = 0;
        auto aoff = [&](int s) { return (((long long)s * p.N + n) * p.C + c) * 3 * HW; };
        if (p.mask & kTB) { const long long o = aoff(slot++); plane_bwd_direction<T, kTB, LPT, LOCAL>((const T*)p.a + o, (T*)p.da + o, z, g, w0b, w2b, hb, db, acc, dz, H, W, Wp, p.chunk, tid); }
        if (p.mask & kBT) { const long long o = aoff(slot++); plane_bwd_direction<T, kBT, LPT, LOCAL>((const T*)p.a + o, (T*)p.da + o, z, g, w0b, w2b, hb, db, acc, dz, H, W, Wp, p.chunk, tid); }
        if (p.mask & kLR) { const long long o = aoff(slot++); plane_bwd_direction<T, kLR, LPT, LOCAL>((const T*)p.a + o, (T*)p.da + o, z, g, w0b, w2b, hb, db, acc, dz, H, W, Wp, p.chunk, tid); }
        if (p.mask & kRL) { const long long o = aoff(slot++); plane_bwd_direction<T, kRL, LPT, LOCAL>((const T*)p.a + o, (T*)p.da + o, z, g, w0b, w2b, hb, db, acc, dz, H, W, Wp, p.chunk, tid); }
        for (int e = tid; e < HW; e += kPlaneBwdThreads) {
            const int q = (e / W) * Wp + e % W;
            Io<T>::st((T*)p.dx + po + e, Io<T>::ld(lam + e) * dz[q]);
            Io<T>::st((T*)p.dlam + po + e, Io<T>::ld(x + e) * dz[q]);
            Io<T>::st((T*)p.du + po + e, Io<T>::ld(dy + e) * acc[q]);
        }
        __syncthreads();
    }
}

// ====================================================== backward, directions scanned concurrently
// fp32 storage, per-channel weights. Warp d takes the d-th direction of the mask: it recomputes
// that direction's h into a plane of its own (cd_scan, the forward's strip scan), then runs the
// reverse scan delta_i = g_i + w_{i+1}^T delta_{i+1} into a second plane of its own, streaming the
// direction's logits through its ring again, strips in reverse order. The directions' scans are
// independent given z and g, so the D warps run them at the same time. Afterwards all threads form
// every direction's logit gradients from its delta and h planes (coalesced, image order) and
// dx = lam dz, dlam = x dz, du = dy sum_d h^d with dz = sum_d delta^d, both sums in slot order, so
// the result does not depend on warp timing.

// Primes the ring with the last NSL strips, last first (one commit group per strip).
template <typename T, int LPT, int NSL>
__device__ __forceinline__ void cd_prime_rev(uint32_t* ring, const T* a3, const CdDir& g, int HW, int W, int lane) {
    constexpr int K = CdGeom<T>::K;
    const int nq = (g.L + K - 1) / K;
#pragma unroll
    for (int q = 0; q < NSL; ++q) {
        if (q < nq) cd_fetch<T, LPT>(ring + q * cd_slot_words<LPT>(), a3, g, HW, W, nq - 1 - q, lane);
        cd_commit();
    }
}

// Reverse scan of one direction by one warp over the lines L-1 .. 0: delta into db (plane layout).
// (w_{i+1}^T delta)[j] = w_{i+1}[j-1][2] delta[j-1] + w_{i+1}[j][1] delta[j] + w_{i+1}[j+1][0] delta[j+1];
// no delta flows back through the first line of a chunk (its weights multiply h = 0).
template <typename T, int LPT, bool LOCAL, int NSL>
__device__ __forceinline__ void cd_reverse(const float* gz, float* db, uint32_t* ring, const T* a3, const CdDir& g,
                                           int HW, int W, int chunk, int lane) {
    constexpr int K = CdGeom<T>::K;
    constexpr int SLOT = cd_slot_words<LPT>();
    const int L = g.L, M = g.M;
    const int nq = (L + K - 1) / K;
    float del[LPT], pw0[LPT], pw1[LPT], pw2[LPT];   // delta and weights of line i + 1
    bool on[LPT], hl[LPT], hr[LPT];
    int pj[LPT];
#pragma unroll
    for (int e = 0; e < LPT; ++e) {
        const int j = e * 32 + lane;
        del[e] = pw0[e] = pw1[e] = pw2[e] = 0.f;
        on[e] = j < M;
        hl[e] = j > 0;
        hr[e] = j < M - 1;
        pj[e] = on[e] ? g.p0 + j * g.sj : 0;
    }
    for (int qr = 0; qr < nq; ++qr) {
        const int q = nq - 1 - qr;
        cd_wait<NSL - 1>();
        __syncwarp();
        uint32_t* slot = ring + (qr % NSL) * SLOT;
        float w0[K][LPT], w2[K][LPT];
        bool shift = false;
        {
            float lg[3][K][LPT];
            cd_strip_logits<T, LPT, K>(slot, g, lane, 0, lg);
#pragma unroll
            for (int s = 0; s < K; ++s)
#pragma unroll
                for (int e = 0; e < LPT; ++e) {
                    const Wts w = lane_weights_fast_nocheck(lg[0][s][e], lg[1][s][e], lg[2][s][e], hl[e], hr[e]);
                    shift |= on[e] && q * K + s < L &&
                             weights_need_shift(lg[0][s][e], lg[1][s][e], lg[2][s][e], hl[e], hr[e]);
                    w0[s][e] = w.w0;
                    w2[s][e] = w.w2;
                }
            if (__any_sync(0xffffffffu, shift)) {   // rare: some logit below the fast form's range
#pragma unroll
                for (int s = 0; s < K; ++s)
#pragma unroll
                    for (int e = 0; e < LPT; ++e)
                        if (weights_need_shift(lg[0][s][e], lg[1][s][e], lg[2][s][e], hl[e], hr[e])) {
                            const Wts w = weights_shifted(lg[0][s][e], lg[1][s][e], lg[2][s][e], hl[e], hr[e]);
                            w0[s][e] = w.w0;
                            w2[s][e] = w.w2;
                        }
            }
        }
        __syncwarp();
        if (qr + NSL < nq) cd_fetch<T, LPT>(slot, a3, g, HW, W, nq - 1 - (qr + NSL), lane);
        cd_commit();
#pragma unroll
        for (int s = K - 1; s >= 0; --s) {
            const int i = q * K + s;
            if (i < L) {   // warp-uniform
                const int di = i * g.si;
                float tl[LPT], tr[LPT], rl[LPT], rr[LPT];
#pragma unroll
                for (int e = 0; e < LPT; ++e) {
                    tl[e] = pw2[e] * del[e];   // lane j's term for lane j + 1
                    tr[e] = pw0[e] * del[e];   // lane j's term for lane j - 1
                }
#pragma unroll
                for (int e = 0; e < LPT; ++e) {
                    rl[e] = __shfl_sync(0xffffffffu, tl[e], (lane + 31) & 31);
                    rr[e] = __shfl_sync(0xffffffffu, tr[e], (lane + 1) & 31);
                }
                bool live = i != 0;
                if constexpr (LOCAL) live = !chunk_start(g.asc, L, chunk, i);
#pragma unroll
                for (int e = 0; e < LPT; ++e) {
                    const float left = lane > 0 ? rl[e] : (e > 0 ? rl[e - 1] : 0.f);
                    const float right = lane < 31 ? rr[e] : (e < LPT - 1 ? rr[e + 1] : 0.f);
                    const float gi = gz[on[e] ? pj[e] + di : 0];
                    const float d = on[e] ? fmaf(pw1[e], del[e], gi) + left + right : 0.f;
                    if (on[e]) db[pj[e] + di] = d;
                    del[e] = d;
                    const bool keep = on[e] && live;
                    pw0[e] = keep ? w0[s][e] : 0.f;
                    pw2[e] = keep ? w2[s][e] : 0.f;
                    pw1[e] = keep ? 1.f - w0[s][e] - w2[s][e] : 0.f;
                }
            }
        }
    }
}

// Logit gradients of direction D from its delta and h planes, weights formed again from the logits
// (all threads, image order, vector loads and stores; W % 4 == 0): at scan position (i, j), i > 0,
//   dw_k = delta_i[j] h_{i-1}[j+k-1],  da_k = w_k sigmoid(-a_k) (dw_k - sum_k' w_k' dw_k')
// (zero for out-of-range k and for the first line of a chunk).
template <typename T, unsigned D, int NT>
__device__ __forceinline__ void cd_logit_grads(const T* a3, T* da3, const float* hb, const float* db, int H, int W,
                                               int Wp, int chunk, int tid) {
    constexpr bool V = D == kTB || D == kBT;
    const int M = V ? W : H;
    const int HW = H * W;
    for (int e0 = tid * 4; e0 < HW; e0 += NT * 4) {
        const int r = e0 / W, c0 = e0 - r * W;
        float a0[4], a1[4], a2[4], g0[4], g1[4], g2[4];
        ld_lanes<T, 4>(a3 + e0, a0);
        ld_lanes<T, 4>(a3 + HW + e0, a1);
        ld_lanes<T, 4>(a3 + 2 * HW + e0, a2);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int c = c0 + k;
            const int i = D == kTB ? r : D == kBT ? H - 1 - r : D == kLR ? c : W - 1 - c;
            const int j = V ? c : r;
            g0[k] = g1[k] = g2[k] = 0.f;
            if (!chunk_start(scan_ascending(D), V ? H : W, chunk, i)) {
                const bool hasl = j > 0, hasr = j < M - 1;
                const LaneJac J = lane_jacobian(a0[k], a1[k], a2[k], hasl, hasr);
                const float d = db[r * Wp + c];
                const float h0 = hasl ? hb[plane_pix<D>(H, W, Wp, i - 1, j - 1)] : 0.f;
                const float h1 = hb[plane_pix<D>(H, W, Wp, i - 1, j)];
                const float h2 = hasr ? hb[plane_pix<D>(H, W, Wp, i - 1, j + 1)] : 0.f;
                const float dw0 = d * h0, dw1 = d * h1, dw2 = d * h2;
                const float sdw = J.w0 * dw0 + J.w1 * dw1 + J.w2 * dw2;
                g0[k] = J.g0 * (dw0 - sdw);
                g1[k] = J.g1 * (dw1 - sdw);
                g2[k] = J.g2 * (dw2 - sdw);
            }
        }
        st_lanes<T, 4>(da3 + e0, g0);
        st_lanes<T, 4>(da3 + HW + e0, g1);
        st_lanes<T, 4>(da3 + 2 * HW + e0, g2);
    }
}

// Shared memory of the concurrent-direction backward (floats): z, g, then nd h planes and nd delta
// planes, then nd rings of NSL strips (16-byte aligned).
__host__ __device__ constexpr int cdb_ring_offset(int nd, int HWs) { return ((2 + 2 * nd) * HWs + 3) & ~3; }
// One warp per direction scans; all eight warps share the parallel phases (loads, logit gradients,
// the final products), which are latency-bound at one CTA per SM.
constexpr int kCdbThreads = 256;

template <typename T, int LPT, bool LOCAL, int NSL>
__global__ void __launch_bounds__(kCdbThreads) k_plane_bwd_cd(PlaneBwdArgs p) {
    extern __shared__ __align__(16) float sm[];
    const int H = p.H, W = p.W, Wp = p.Wp;
    const int HW = H * W, HWs = H * Wp;
    const int nd = __popc(p.mask);
    float* z = sm;
    float* gpl = z + HWs;
    float* hb = gpl + HWs;          // nd planes, slot order
    float* db = hb + nd * HWs;      // nd planes, slot order
    uint32_t* rings = reinterpret_cast<uint32_t*>(sm + cdb_ring_offset(nd, HWs));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    unsigned dir = 0;   // this warp's direction: the warp-th set bit of the mask (its slot is warp)
    {
        unsigned m = p.mask;
        for (int k = 0; k < warp && m; ++k) m &= m - 1;
        dir = m & (0u - m);
    }
    const CdDir geo = cd_dir(dir, H, W, Wp);
    const bool scans = warp < nd;
    uint32_t* ring = rings + warp * NSL * cd_slot_words<LPT>();
    float* hw = hb + warp * HWs;
    float* dw = db + warp * HWs;
    const int nplanes = p.N * p.C;
    for (int plane = blockIdx.x; plane < nplanes; plane += gridDim.x) {
        const int n = plane / p.C, c = plane % p.C;
        const long long po = (long long)plane * HW;
        auto aoff = [&](int s) { return (((long long)s * p.N + n) * p.C + c) * 3 * HW; };
        const T* a3 = (const T*)p.a + aoff(warp);
        const T *x = (const T*)p.x + po, *lam = (const T*)p.lam + po, *u = (const T*)p.u + po;
        const T* dy = (const T*)p.dy + po;
        if (scans) cd_prime<T, LPT, NSL>(ring, a3, geo, HW, W, lane);
        for (int e0 = tid * 4; e0 < HW; e0 += kCdbThreads * 4) {   // z = lam x, g = u dy
            float xv[4], lv[4], uv[4], dv[4];
            ld_lanes<T, 4>(x + e0, xv);
            ld_lanes<T, 4>(lam + e0, lv);
            ld_lanes<T, 4>(u + e0, uv);
            ld_lanes<T, 4>(dy + e0, dv);
            const int row = e0 / W, col = e0 - row * W;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                z[row * Wp + col + k] = lv[k] * xv[k];
                gpl[row * Wp + col + k] = uv[k] * dv[k];
            }
        }
        __syncthreads();
        if (scans) {
            cd_scan<T, LPT, LOCAL, NSL>(z, hw, ring, a3, geo, HW, W, p.chunk, lane);
            __syncwarp();   // every lane has read its last strip before the ring is refilled
            cd_prime_rev<T, LPT, NSL>(ring, a3, geo, HW, W, lane);
            cd_reverse<T, LPT, LOCAL, NSL>(gpl, dw, ring, a3, geo, HW, W, p.chunk, lane);
        }
        __syncthreads();
        // logit gradients, one direction after another (slot order)
        {
            int slot = 0;
            if (p.mask & kTB) { const long long o = aoff(slot); cd_logit_grads<T, kTB, kCdbThreads>((const T*)p.a + o, (T*)p.da + o, hb + slot * HWs, db + slot * HWs, H, W, Wp, p.chunk, tid); ++slot; }
            if (p.mask & kBT) { const long long o = aoff(slot); cd_logit_grads<T, kBT, kCdbThreads>((const T*)p.a + o, (T*)p.da + o, hb + slot * HWs, db + slot * HWs, H, W, Wp, p.chunk, tid); ++slot; }
            if (p.mask & kLR) { const long long o = aoff(slot); cd_logit_grads<T, kLR, kCdbThreads>((const T*)p.a + o, (T*)p.da + o, hb + slot * HWs, db + slot * HWs, H, W, Wp, p.chunk, tid); ++slot; }
            if (p.mask & kRL) { const long long o = aoff(slot); cd_logit_grads<T, kRL, kCdbThreads>((const T*)p.a + o, (T*)p.da + o, hb + slot * HWs, db + slot * HWs, H, W, Wp, p.chunk, tid); ++slot; }
        }
        // dx = lam dz, dlam = x dz, du = dy sum_d h^d (sums in slot order)
        for (int e0 = tid * 4; e0 < HW; e0 += kCdbThreads * 4) {
            float xv[4], lv[4], dv[4], ox[4], ol[4], ou[4];
            ld_lanes<T, 4>(x + e0, xv);
            ld_lanes<T, 4>(lam + e0, lv);
            ld_lanes<T, 4>(dy + e0, dv);
            const int row = e0 / W, col = e0 - row * W;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int q = row * Wp + col + k;
                float dz = db[q], hs = hb[q];
                for (int d = 1; d < nd; ++d) {
                    dz += db[d * HWs + q];
                    hs += hb[d * HWs + q];
                }
                ox[k] = lv[k] * dz;
                ol[k] = xv[k] * dz;
                ou[k] = dv[k] * hs;
            }
            st_lanes<T, 4>((T*)p.dx + po + e0, ox);
            st_lanes<T, 4>((T*)p.dlam + po + e0, ol);
            st_lanes<T, 4>((T*)p.du + po + e0, ou);
        }
        __syncthreads();   // the next plane overwrites z, g and the planes
    }
}

int plane_wp(const Problem& P) { return P.W % 2 == 0 ? P.W + 1 : P.W; }
size_t plane_smem(const Problem& P) { return 4 * (size_t)P.H * plane_wp(P) * sizeof(float); }
int plane_lanes(const Problem& P) {
    const int M = std::max(P.H, P.W);
    return M <= 32 ? 1 : (M <= 64 ? 2 : 4);
}

size_t plane_bwd_smem(const Problem& P) { return 8 * (size_t)P.H * plane_wp(P) * sizeof(float); }

template <typename T, int LPT, bool LOCAL>
cudaError_t plane_bwd_launch3(const Problem& P, const PlaneBwdArgs& a, cudaStream_t st) {
    const size_t smem = plane_bwd_smem(P);
    cudaError_t e = cudaFuncSetAttribute(k_plane_bwd<T, LPT, LOCAL>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaFuncSetAttribute(k_plane_bwd<T, LPT, LOCAL>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    int per_sm = 1;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_plane_bwd<T, LPT, LOCAL>, kPlaneBwdThreads, smem);
    if (e != cudaSuccess) return e;
    const long long want = (long long)std::max(1, per_sm) * device_sm_count();
    const int grid = (int)std::min<long long>(want, (long long)P.N * P.C);
    launch_begin(st);
    k_plane_bwd<T, LPT, LOCAL><<<grid, kPlaneBwdThreads, smem, st>>>(a);
    launch_end(st);
    return cudaGetLastError();
}

template <typename T, int LPT, bool LOCAL, bool PD>
cudaError_t plane_fwd_launch3(const Problem& P, const PlaneArgs& a, cudaStream_t st) {
    const size_t smem = plane_smem(P);
    cudaError_t e = cudaFuncSetAttribute(k_plane_fwd<T, LPT, LOCAL, PD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaFuncSetAttribute(k_plane_fwd<T, LPT, LOCAL, PD>, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    int per_sm = 1;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_plane_fwd<T, LPT, LOCAL, PD>, kPlaneThreads, smem);
    if (e != cudaSuccess) return e;
    const long long want = (long long)std::max(1, per_sm) * device_sm_count();
    const int grid = (int)std::min<long long>(want, (long long)P.N * P.C);
    launch_begin(st);
    k_plane_fwd<T, LPT, LOCAL, PD><<<grid, kPlaneThreads, smem, st>>>(a);
    launch_end(st);
    return cudaGetLastError();
}

size_t cd_smem(const Problem& P, int nsl, int lpt) {
    const int nd = __builtin_popcount(P.mask);
    const int slot = 384 * lpt;   // words per ring strip (cd_slot_words)
    return (size_t)cd_ring_offset_h(nd, P.H * plane_wp(P), (int)P.esize()) * sizeof(float) + (size_t)nd * nsl * slot * 4;
}
// Ring depth of the concurrent-direction forward: three strips when two CTAs still fit on an SM,
// else two; 0 when the kernel does not apply (per-direction lambda / u, rows not a whole number of
// 16-byte chunks, or the planes do not fit). bf16 storage keeps its h planes in bf16 (half the
// shared memory of fp32 ones) and forms the weights of a strip four lines at a time (160
// registers instead of 255), which made it faster than the direction-serial kernel on the
// 56 x 56 classifier maps (1.30 ms against 1.43 ms per forward).
int cd_ring_depth(const Problem& P) {
    // rows of whole 16-byte chunks: 4 fp32 or 8 bf16 elements
    if (P.per_dir || P.W % (P.dtype == GSPN_F32 ? 4 : 8) != 0) return 0;
    const int lpt = plane_lanes(P);
    if (cd_smem(P, 3, lpt) <= kPlaneSmemBudget / 2) return 3;
    return cd_smem(P, 2, lpt) <= kPlaneSmemBudget ? 2 : 0;
}

template <typename T, int LPT, bool LOCAL, int NSL>
cudaError_t plane_cd_launch4(const Problem& P, const PlaneArgs& a, cudaStream_t st) {
    const size_t smem = cd_smem(P, NSL, LPT);
    auto kern = k_plane_fwd_cd<T, LPT, LOCAL, NSL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    int per_sm = 1;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kCdThreads, smem);
    if (e != cudaSuccess) return e;
    const long long want = (long long)std::max(1, per_sm) * device_sm_count();
    const int grid = (int)std::min<long long>(want, (long long)P.N * P.C);
    launch_begin(st);
    kern<<<grid, kCdThreads, smem, st>>>(a);
    launch_end(st);
    return cudaGetLastError();
}
template <typename T, int LPT, bool LOCAL>
cudaError_t plane_cd_launch3(const Problem& P, const PlaneArgs& a, cudaStream_t st) {
    return cd_ring_depth(P) == 3 ? plane_cd_launch4<T, LPT, LOCAL, 3>(P, a, st)
                                 : plane_cd_launch4<T, LPT, LOCAL, 2>(P, a, st);
}

// Local propagation has its own instantiations, so the global scans carry no chunk counters.
template <typename T, int LPT>
cudaError_t plane_fwd_launch(const Problem& P, const PlaneArgs& a, cudaStream_t st) {
    if (cd_ring_depth(P) > 0)
        return P.chunk > 0 ? plane_cd_launch3<T, LPT, true>(P, a, st) : plane_cd_launch3<T, LPT, false>(P, a, st);
    if (P.per_dir)
        return P.chunk > 0 ? plane_fwd_launch3<T, LPT, true, true>(P, a, st)
                           : plane_fwd_launch3<T, LPT, false, true>(P, a, st);
    return P.chunk > 0 ? plane_fwd_launch3<T, LPT, true, false>(P, a, st)
                       : plane_fwd_launch3<T, LPT, false, false>(P, a, st);
}
size_t cdb_smem(const Problem& P, int nsl, int lpt) {
    const int nd = __builtin_popcount(P.mask);
    return (size_t)cdb_ring_offset(nd, P.H * plane_wp(P)) * sizeof(float) + (size_t)nd * nsl * 384 * lpt * 4;
}
// Ring depth of the concurrent-direction backward (fp32, rows of whole 16-byte chunks): 3 strips if
// they fit, else 2; 0 when the kernel does not apply.
int cdb_ring_depth(const Problem& P) {
    if (P.dtype != GSPN_F32 || P.per_dir || P.W % 4 != 0 || P.wmode != GSPN_W_PER_CHANNEL) return 0;
    const int lpt = plane_lanes(P);
    if (cdb_smem(P, 3, lpt) <= kPlaneSmemBudget) return 3;
    return cdb_smem(P, 2, lpt) <= kPlaneSmemBudget ? 2 : 0;
}
template <typename T, int LPT, bool LOCAL, int NSL>
cudaError_t plane_bwd_cd_launch4(const Problem& P, const PlaneBwdArgs& a, cudaStream_t st) {
    const size_t smem = cdb_smem(P, NSL, LPT);
    auto kern = k_plane_bwd_cd<T, LPT, LOCAL, NSL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    int per_sm = 1;
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kCdbThreads, smem);
    if (e != cudaSuccess) return e;
    const long long want = (long long)std::max(1, per_sm) * device_sm_count();
    const int grid = (int)std::min<long long>(want, (long long)P.N * P.C);
    launch_begin(st);
    kern<<<grid, kCdbThreads, smem, st>>>(a);
    launch_end(st);
    return cudaGetLastError();
}
template <typename T, int LPT, bool LOCAL>
cudaError_t plane_bwd_cd_launch3(const Problem& P, const PlaneBwdArgs& a, cudaStream_t st) {
    return cdb_ring_depth(P) == 3 ? plane_bwd_cd_launch4<T, LPT, LOCAL, 3>(P, a, st)
                                  : plane_bwd_cd_launch4<T, LPT, LOCAL, 2>(P, a, st);
}
template <typename T, int LPT>
cudaError_t plane_bwd_launch(const Problem& P, const PlaneBwdArgs& a, cudaStream_t st) {
    if constexpr (sizeof(T) == 4) {
        if (cdb_ring_depth(P) > 0)
            return P.chunk > 0 ? plane_bwd_cd_launch3<T, LPT, true>(P, a, st)
                               : plane_bwd_cd_launch3<T, LPT, false>(P, a, st);
    }
    return P.chunk > 0 ? plane_bwd_launch3<T, LPT, true>(P, a, st) : plane_bwd_launch3<T, LPT, false>(P, a, st);
}

template <typename T>
cudaError_t plane_forward_t(const Problem& P, const void* x, const void* a, const void* lam, const void* u, void* y,
                            void* hsave, cudaStream_t st) {
    PlaneArgs args{x, lam, u, a, y, P.N, P.C, P.H, P.W, P.Cw, plane_wp(P), P.mask, P.chunk, (float*)hsave};
    switch (plane_lanes(P)) {
    case 1: return plane_fwd_launch<T, 1>(P, args, st);
    case 2: return plane_fwd_launch<T, 2>(P, args, st);
    default: return plane_fwd_launch<T, 4>(P, args, st);
    }
}

}  // namespace

bool plane_supports(const Problem& P, bool bwd) {
    if (std::max(P.H, P.W) > kPlaneMaxLanes) return false;
    if ((long long)P.H * P.W > (1LL << 20)) return false;
    if (bwd) return P.wmode == GSPN_W_PER_CHANNEL && !P.per_dir && plane_bwd_smem(P) <= kPlaneSmemBudget;
    return plane_smem(P) <= kPlaneSmemBudget;
}

size_t plane_ws_bytes(const Problem&, bool) { return 256; }

cudaError_t plane_forward(const Problem& P, const void* x, const void* a, const void* lam, const void* u, void* y,
                          void*, cudaStream_t st) {
    if (P.dtype == GSPN_F32) return plane_forward_t<float>(P, x, a, lam, u, y, nullptr, st);
    return plane_forward_t<__nv_bfloat16>(P, x, a, lam, u, y, nullptr, st);
}

// The forward keeps each direction's h when the concurrent-direction kernel runs it (it holds all
// four h planes in shared memory at the end of a plane).
bool plane_can_save(const Problem& P) { return plane_supports(P, false) && cd_ring_depth(P) > 0; }

cudaError_t plane_forward_save(const Problem& P, const void* x, const void* a, const void* lam, const void* u,
                               void* y, float* hsave, cudaStream_t st) {
    if (!plane_can_save(P)) return cudaErrorNotSupported;
    if (P.dtype == GSPN_F32) return plane_forward_t<float>(P, x, a, lam, u, y, hsave, st);
    return plane_forward_t<__nv_bfloat16>(P, x, a, lam, u, y, hsave, st);
}

cudaError_t plane_backward(const Problem& P, const void* x, const void* a, const void* lam, const void* u,
                           const void* dy, void* dx, void* da, void* dlam, void* du, void*, cudaStream_t st) {
    PlaneBwdArgs args{x, lam, u, a, dy, dx, da, dlam, du, P.N, P.C, P.H, P.W, plane_wp(P), P.mask, P.chunk};
    const int lpt = plane_lanes(P);
    if (P.dtype == GSPN_F32)
        return lpt == 1 ? plane_bwd_launch<float, 1>(P, args, st)
                        : (lpt == 2 ? plane_bwd_launch<float, 2>(P, args, st) : plane_bwd_launch<float, 4>(P, args, st));
    return lpt == 1 ? plane_bwd_launch<__nv_bfloat16, 1>(P, args, st)
                    : (lpt == 2 ? plane_bwd_launch<__nv_bfloat16, 2>(P, args, st)
                                : plane_bwd_launch<__nv_bfloat16, 4>(P, args, st));
}

}  // namespace gspn
