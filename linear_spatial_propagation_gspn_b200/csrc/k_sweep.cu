// k_sweep.cu -- large-map kernel family of libgspn: persistent line sweeps.
//
// One sweep per direction in the mask, in the order TB, BT, LR, RL. Every sweep is one
// persistent kernel: each CTA owns whole planes (a line of a scan couples all its lanes, so a
// line cannot be split across CTAs without a per-step exchange) and runs the sequential scan
// over the plane with the running line h_{i-1} in registers; one barrier per step exchanges the
// neighbour values across warps. Inputs stream through a shared-memory ring filled with
// per-thread asynchronous copies (cp.async): each thread copies exactly the lanes it will read,
// several steps ahead, so no thread waits for another's data. (Measured on B200: a TMA bulk copy
// costs about 285 ns per operation per SM whatever its size up to 32 KB, and the operations of
// one SM are serialised; a sweep needs 5-7 row-sized copies per step, which capped it near
// 1.2-1.9 us per step. Per-thread copies have no such per-operation cost.)
//   - vertical sweeps (TB, BT): thread t owns LPT consecutive lanes of a row; its copies are
//     contiguous across the warp (fully coalesced);
//   - horizontal sweeps (LR, RL): column tiles of 16 bytes per row (4 fp32 or 8 bf16 steps, a
//     staged transpose); thread t owns rows t, t+T, ..., copies and reads 16 bytes per row per
//     tensor (conflict-free), and writes its outputs back as 16-byte row segments.
// No direction issues strided per-element HBM traffic. The first sweep reads x and lambda and
// writes z = lambda * x and the partial sum; later sweeps read z and the partial sum (both in the
// storage dtype); the last one reads u and writes y = u * (partial + h). ("GSPN-2: Efficient
// Parallel Sequence Modeling" paper notes, section "Optimisation 3: efficient CUDA extension":
// coalesced access and on-chip reuse of h_{i-1} were the decisive optimisations on A100.)
#include <stdlib.h>

#include <algorithm>
#include <type_traits>

#include "gspn_common.cuh"
#include "gspn_internal.h"

namespace gspn {
namespace {

enum { M_FIRST = 0, M_ONLY = 1, M_MID = 2, M_LAST = 3 };

// TOUT: outputs leave through a shared-memory staging block and are written lane-major
// (transposed); a final sweep then applies u while flushing, so u is not in the ring.
template <int MODE, bool TOUT = false> struct ModeT {
    static constexpr bool XL = MODE == M_FIRST || MODE == M_ONLY;     // read x, lam (else z)
    static constexpr bool ACCIN = MODE == M_MID || MODE == M_LAST;    // read the partial sum
    static constexpr bool FINAL = MODE == M_ONLY || MODE == M_LAST;   // read u, write y
    static constexpr bool ZOUT = MODE == M_FIRST || (TOUT && !FINAL); // write z (z^T when TOUT)
    static constexpr bool URING = FINAL && !TOUT;                     // u comes through the ring
    // storage-dtype tensors per stage: x lam | z, [acc], [u]  (plus the two fp32 weight rows)
    static constexpr int NTEN = (XL ? 2 : 1) + (ACCIN ? 1 : 0) + (URING ? 1 : 0);
    // staged outputs when TOUT: z and acc, or the unscaled sum for a final sweep
    static constexpr int NSTG = TOUT ? (FINAL ? 1 : 2) : 0;
};

// Steps per staging block of a transposed-output sweep (64 bytes of fp32 per lane).
constexpr int kTB_STEPS = 16;

// Sweep arguments in scan coordinates: H = scan length (steps), W = lanes. A horizontal scan
// over transposed buffers passes (H, W) = (image width, image height).
struct SweepArgs {
    const void* x;
    const void* lam;
    const void* u;    // scan-major, or lane-major (image layout) for a transposed-output final sweep
    const float* wt;  // weight table of this direction's slot: [N][Cw][2][H][W] fp32 (w0, w2)
    void* z;          // workspace, storage dtype, scan-major
    void* acc;        // workspace, storage dtype, scan-major
    void* y;          // output (scan-major, or lane-major when TOUT)
    void* zt;         // lane-major z   (TOUT, non-final)
    void* acct;       // lane-major acc (TOUT, non-final)
    int N, C, H, W, Cw;
};

struct WeightArgs {
    const void* a;    // logits [D][N][Cw][3][H][W]
    float* wt;        // table  [D][N][Cw][2][H][W] (transposed planes: [W][H])
    int N, Cw, H, W, D;
    int plane0;       // first (slot, n, cw) plane handled by the launch
    unsigned dirs[4]; // direction bit of each slot
};

// ------------------------------------------------------------------ async copies
__device__ __forceinline__ uint32_t smem_u32(const void* ptr) { return (uint32_t)__cvta_generic_to_shared(ptr); }

// Global -> shared copy of BYTES (4, 8 or 16) bytes, both addresses aligned to BYTES. 16-byte
// copies bypass L1 (.cg); smaller ones must use .ca.
template <int BYTES>
__device__ __forceinline__ void cp_async(void* dst, const void* src) {
    if constexpr (BYTES == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(smem_u32(dst)), "l"(src), "n"(BYTES)
                     : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------------------ 16-byte row segments
// 16 bytes = 4 fp32 or 8 bf16 consecutive steps of one lane.
template <typename T> struct Seg;
template <> struct Seg<float> {
    static constexpr int S = 4;
    static __device__ __forceinline__ float get(const uint4& r, int s) {
        return __uint_as_float(s == 0 ? r.x : s == 1 ? r.y : s == 2 ? r.z : r.w);
    }
    static __device__ __forceinline__ void put(uint4& r, int s, float v) {
        const uint32_t b = __float_as_uint(v);
        if (s == 0) r.x = b; else if (s == 1) r.y = b; else if (s == 2) r.z = b; else r.w = b;
    }
};
template <> struct Seg<__nv_bfloat16> {
    static constexpr int S = 8;
    static __device__ __forceinline__ float get(const uint4& r, int s) {
        const uint32_t w = (s >> 1) == 0 ? r.x : (s >> 1) == 1 ? r.y : (s >> 1) == 2 ? r.z : r.w;
        const uint32_t bits = (s & 1) ? (w & 0xffff0000u) : (w << 16);
        return __uint_as_float(bits);
    }
    static __device__ __forceinline__ void put(uint4& r, int s, float v) {
        const uint32_t h = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(v));
        uint32_t* w = (s >> 1) == 0 ? &r.x : (s >> 1) == 1 ? &r.y : (s >> 1) == 2 ? &r.z : &r.w;
        *w = (s & 1) ? ((*w & 0x0000ffffu) | (h << 16)) : ((*w & 0xffff0000u) | h);
    }
};

__device__ __forceinline__ unsigned char* align128(unsigned char* ptr) {
    return (unsigned char*)(((uintptr_t)ptr + 127) & ~(uintptr_t)127);
}

// A thread's LPT lanes of one row in shared memory. With fp32 and LPT = 8 a thread owns 32
// bytes, and threads t and t+4 would hit the same banks in a 16-byte load phase; the thread
// therefore stores its two 16-byte chunks in swapped order when bit 2 of its index is set
// (`sw`), which makes every load phase conflict-free. Each thread writes and reads only its own
// chunks, so the swizzle is private to the thread.
template <typename T, int LPT>
__device__ __forceinline__ void copy_lanes(unsigned char* dst, const T* src, int sw) {
    constexpr int VB = LPT * (int)sizeof(T);
    if constexpr (VB == 32) {
        cp_async<16>(dst + 16 * sw, src);
        cp_async<16>(dst + 16 * (1 - sw), src + 4);
    } else {
        cp_async<VB>(dst, src);
    }
}
template <typename T, int LPT>
__device__ __forceinline__ void read_lanes(const unsigned char* srcs, float (&v)[LPT], int sw) {
    constexpr int VB = LPT * (int)sizeof(T);
    if constexpr (VB == 32) {
        const float4 q0 = *(const float4*)(srcs + 16 * sw), q1 = *(const float4*)(srcs + 16 * (1 - sw));
        v[0] = q0.x; v[1] = q0.y; v[2] = q0.z; v[3] = q0.w;
        v[4] = q1.x; v[5] = q1.y; v[6] = q1.z; v[7] = q1.w;
    } else {
        ld_lanes<T, LPT>(srcs, v);
    }
}


// ================================================================== weight formation (A1)
// Turns the logits of every (slot, n, cw) plane into the two outer weights w0, w2 of each
// normalised tridiagonal row; the sweeps re-derive w1 = 1 - w0 - w2, so every row sums to one.
// Elementwise and memory-bound: one thread per 4 consecutive pixels of a row, accurate expf and
// IEEE reciprocal. blockIdx.y = plane, so no 64-bit division is needed.
template <typename T>
__global__ void __launch_bounds__(256) k_sweep_weights(WeightArgs p) {
    const long long HW = (long long)p.H * p.W;
    const int plane = p.plane0 + (int)blockIdx.y;      // (slot, n, cw)
    const int slot = plane / (p.N * p.Cw);
    const unsigned d = p.dirs[slot];
    const T* a3 = (const T*)p.a + (long long)plane * 3 * HW;
    float* wt = p.wt + (long long)plane * 2 * HW;
    const int quads = (int)(HW / 4);
    for (int q = blockIdx.x * blockDim.x + threadIdx.x; q < quads; q += gridDim.x * blockDim.x) {
        const int pix = q * 4;
        const int r = pix / p.W, c0 = pix - r * p.W;
        float a0[4], a1[4], a2[4], w0[4], w2[4];
        ld_lanes<T, 4>(a3 + pix, a0);
        ld_lanes<T, 4>(a3 + HW + pix, a1);
        ld_lanes<T, 4>(a3 + 2 * HW + pix, a2);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int c = c0 + k;
            const bool hl = is_vertical(d) ? c > 0 : r > 0;
            const bool hr = is_vertical(d) ? c < p.W - 1 : r < p.H - 1;
            const Wts w = lane_weights_acc(a0[k], a1[k], a2[k], hl, hr);
            w0[k] = w.w0;
            w2[k] = w.w2;
        }
        st_lanes<float, 4>(wt + pix, w0);
        st_lanes<float, 4>(wt + HW + pix, w2);
    }
}

// Same table, written transposed ([W][H] per plane: element (column c, row r) at c*H + r) for
// horizontal scans run over transposed buffers. 32x32 pixel tiles through shared memory keep
// both the logit reads and the table writes coalesced.
template <typename T>
__global__ void __launch_bounds__(256) k_sweep_weights_t(WeightArgs p) {
    __shared__ float tile[2][32][33];
    const long long HW = (long long)p.H * p.W;
    const int plane = p.plane0 + (int)blockIdx.z;
    const int slot = plane / (p.N * p.Cw);
    const unsigned d = p.dirs[slot];
    const T* a3 = (const T*)p.a + (long long)plane * 3 * HW;
    float* wt = p.wt + (long long)plane * 2 * HW;
    const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 32 x 8
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int r = r0 + ty + 8 * k, c = c0 + tx;
        float w0 = 0.f, w2 = 0.f;
        if (r < p.H && c < p.W) {
            const long long q = (long long)r * p.W + c;
            const bool hl = is_vertical(d) ? c > 0 : r > 0;
            const bool hr = is_vertical(d) ? c < p.W - 1 : r < p.H - 1;
            const Wts w = lane_weights_acc(Io<T>::ld(a3 + q), Io<T>::ld(a3 + HW + q), Io<T>::ld(a3 + 2 * HW + q), hl, hr);
            w0 = w.w0;
            w2 = w.w2;
        }
        tile[0][ty + 8 * k][tx] = w0;
        tile[1][ty + 8 * k][tx] = w2;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int c = c0 + ty + 8 * k, r = r0 + tx;
        if (r < p.H && c < p.W) {
            const long long q = (long long)c * p.H + r;
            wt[q] = tile[0][tx][ty + 8 * k];
            wt[HW + q] = tile[1][tx][ty + 8 * k];
        }
    }
}

// ================================================================== vertical sweep
// CTA = one plane at a time (persistent over planes b, b + grid, ...); thread t owns lanes
// [LPT t, LPT t + LPT). Ring of NS stages; a stage is one image row of the two fp32 weight
// rows and of each storage-dtype input. Every thread keeps NS rows of its own lanes in flight.
// The loop is software-pipelined by one step: while step g's new line is exchanged at the
// barrier, every thread has already pulled step g+1's inputs out of the ring.
template <typename T, unsigned DIR, int MODE, int LPT, int NS, bool TOUT>
__global__ void __launch_bounds__(LPT == 8 ? 512 : 1024, 1) k_vsweep(SweepArgs p) {
    using Md = ModeT<MODE, TOUT>;
    constexpr int NTEN = Md::NTEN;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align128(smem_raw);
    const int H = p.H, W = p.W;
    const int rowB = W * (int)sizeof(T);
    const int wrowB = W * 4;
    const int stageB = 2 * wrowB + NTEN * rowB;
    float* halo = (float*)(smem + (size_t)NS * stageB);   // [2 parity][2 lo/hi][32 warps]
    // TOUT staging: Md::NSTG blocks of [kTB_STEPS][R] in the storage dtype (the values are
    // stored in that dtype anyway). R is W rounded up to 32 plus 16 bytes, so every staging row
    // starts 16-byte aligned (vector stores) and consecutive rows shift the bank pattern.
    T* stg = (T*)(halo + 128);
    const int R = ((W + 31) / 32) * 32 + 16 / (int)sizeof(T);
    // TOUT final: u of the next staging block, prefetched lane-major, 16 bytes per chunk id
    constexpr int CH = 16 / (int)sizeof(T);          // steps per 16-byte chunk
    constexpr int CPL = kTB_STEPS / CH;              // chunks per lane segment
    uint4* ubuf = (uint4*)align128((unsigned char*)(stg + (size_t)Md::NSTG * kTB_STEPS * R));
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int j0 = tid * LPT;
    const bool active = j0 < W;
    const int sw = (tid >> 2) & 1;
    const long long HW = (long long)H * W;
    const int nplanes = p.N * p.C;
    const int my_planes = (nplanes - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const long long total = (long long)my_planes * H;
    const size_t wofs = (size_t)j0 * 4;                                  // this thread in a weight row
    const size_t tofs = 2 * (size_t)wrowB + (size_t)j0 * sizeof(T);      // ... in the first T row

    // Issue cursor: rows are requested strictly in step order, so plane, row and stage advance
    // incrementally (no division inside the loop).
    long long iss_left = total;
    int iss_i = 0, iss_s = 0, iss_plane = (int)blockIdx.x;
    const float* iss_wt = nullptr;
    long long iss_poff = 0;
    auto iss_plane_setup = [&]() {
        const int n = iss_plane / p.C, c = iss_plane % p.C;
        iss_wt = p.wt + ((long long)n * p.Cw + (p.Cw == 1 ? 0 : c)) * 2 * HW;
        iss_poff = (long long)iss_plane * HW;
    };
    auto issue = [&]() {
        if (iss_left > 0) {
            if (active) {
                const int r = DIR == kTB ? iss_i : H - 1 - iss_i;
                unsigned char* st = smem + (size_t)iss_s * stageB;
                const long long ro = (long long)r * W + j0;
                copy_lanes<float, LPT>(st + wofs, iss_wt + ro, sw);
                copy_lanes<float, LPT>(st + wrowB + wofs, iss_wt + HW + ro, sw);
                const long long off = iss_poff + ro;
                unsigned char* sd = st + tofs;
                int t = 0;
                if (Md::XL) {
                    copy_lanes<T, LPT>(sd + (t++) * rowB, (const T*)p.x + off, sw);
                    copy_lanes<T, LPT>(sd + (t++) * rowB, (const T*)p.lam + off, sw);
                } else {
                    copy_lanes<T, LPT>(sd + (t++) * rowB, (const T*)p.z + off, sw);
                }
                if (Md::ACCIN) copy_lanes<T, LPT>(sd + (t++) * rowB, (const T*)p.acc + off, sw);
                if (Md::URING) copy_lanes<T, LPT>(sd + (t++) * rowB, (const T*)p.u + off, sw);
            }
            --iss_left;
            if (++iss_s == NS) iss_s = 0;
            if (++iss_i == H) {
                iss_i = 0;
                iss_plane += (int)gridDim.x;
                if (iss_plane < nplanes) iss_plane_setup();
            }
        }
        cp_async_commit();   // always one group per call, so the wait counts stay uniform
    };
    // Final transposed-output sweep: copy u of the staging block that contains scan row `row`
    // of plane offset `po` into ubuf (same chunk ids as the flush). The copies join the ring's
    // next commit group, which is complete at least kTB_STEPS - NS steps before the flush.
    auto prefetch_u = [&](int row, long long po) {
        if constexpr (TOUT && Md::FINAL) {
            const int s_base = row - row % kTB_STEPS;
            const int nvalid = min(kTB_STEPS, H - s_base);
            const int q = tid % CPL, jstep = (int)blockDim.x / CPL;
            if (q * CH < nvalid) {
                const T* src = (const T*)p.u + po + (long long)(tid / CPL) * H + s_base + q * CH;
                for (int j = tid / CPL; j < W; j += jstep, src += (long long)jstep * H)
                    cp_async<16>(ubuf + j * CPL + q, src);
            }
        }
    };
    prefetch_u(DIR == kTB ? 0 : H - 1, (long long)blockIdx.x * HW);
    iss_plane_setup();
#pragma unroll
    for (int q = 0; q < NS; ++q) issue();

    // inputs of the next step, already out of shared memory
    float nz[LPT], nacc[LPT], nu[LPT], nw0[LPT], nw2[LPT];
#pragma unroll
    for (int e = 0; e < LPT; ++e) nz[e] = nacc[e] = nu[e] = nw0[e] = nw2[e] = 0.f;
    int fs = 0;   // consumer stage
    auto fetch = [&]() {
        cp_async_wait<NS - 1>();
        if (active) {
            const unsigned char* st = smem + (size_t)fs * stageB;
            read_lanes<float, LPT>(st + wofs, nw0, sw);
            read_lanes<float, LPT>(st + wrowB + wofs, nw2, sw);
            const unsigned char* sd = st + tofs;
            read_lanes<T, LPT>(sd, nz, sw);
            if (Md::XL) {
                float l2[LPT];
                read_lanes<T, LPT>(sd + rowB, l2, sw);
#pragma unroll
                for (int e = 0; e < LPT; ++e) nz[e] *= l2[e];     // z = x * lam
            }
            int t = Md::XL ? 2 : 1;
            if (Md::ACCIN) read_lanes<T, LPT>(sd + (t++) * rowB, nacc, sw);
            if (Md::URING) read_lanes<T, LPT>(sd + (t++) * rowB, nu, sw);
        }
        if (++fs == NS) fs = 0;
        issue();   // this thread has consumed its lanes of the stage: refill it NS steps ahead
    };

    fetch();
    float h[LPT];
#pragma unroll
    for (int e = 0; e < LPT; ++e) h[e] = 0.f;
    int i = 0;                                   // step within the plane
    long long poff = (long long)blockIdx.x * HW;
    int plane = (int)blockIdx.x;
    for (long long g = 0; g < total; ++g) {
        float cz[LPT], cacc[LPT], cu[LPT], cw0[LPT], cw2[LPT];
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            cz[e] = nz[e]; cacc[e] = nacc[e]; cu[e] = nu[e]; cw0[e] = nw0[e]; cw2[e] = nw2[e];
            if (i == 0) h[e] = 0.f;
        }
        if constexpr (TOUT && Md::FINAL) {
            // first step of a staging block (after the first): the previous block was flushed
            // behind a barrier at the end of the last iteration, so ubuf is free. The copies
            // join the commit group of this iteration's fetch.
            const int rc = DIR == kTB ? i : H - 1 - i;
            const bool starts = DIR == kTB ? rc % kTB_STEPS == 0 : (rc % kTB_STEPS == kTB_STEPS - 1 || rc == H - 1);
            if (g > 0 && starts) prefetch_u(rc, poff);
        }
        // neighbours from the previous step: lane j0-1 and lane j0+LPT
        const float* hprev = halo + ((g + 1) & 1) * 64;
        float hl = __shfl_up_sync(0xffffffffu, h[LPT - 1], 1);
        float hr = __shfl_down_sync(0xffffffffu, h[0], 1);
        const float edge = lane == 0 ? hprev[32 + warp - 1 + (warp == 0)] : hprev[warp + 1 - (warp == nw - 1)];
        if (lane == 0) hl = warp > 0 ? edge : 0.f;
        if (lane == 31) hr = warp < nw - 1 ? edge : 0.f;
        float hn[LPT];
#pragma unroll
        for (int e = 0; e < LPT; ++e) hn[e] = 0.f;
        if (active) {
#pragma unroll
            for (int e = 0; e < LPT; ++e) {
                hn[e] = cz[e];
                if (i > 0) {
                    const float left = e == 0 ? hl : h[e - 1];
                    const float right = e == LPT - 1 ? hr : h[e + 1];
                    const float w1 = 1.f - cw0[e] - cw2[e];
                    hn[e] = fmaf(cw0[e], left, fmaf(w1, h[e], fmaf(cw2[e], right, hn[e])));
                }
            }
            const int r = DIR == kTB ? i : H - 1 - i;
            const long long off = poff + (long long)r * W + j0;
            float o[LPT];
#pragma unroll
            for (int e = 0; e < LPT; ++e) {
                o[e] = Md::ACCIN ? cacc[e] + hn[e] : hn[e];
                if (Md::URING) o[e] *= cu[e];
            }
            if constexpr (TOUT) {
                T* srow = stg + (size_t)(r % kTB_STEPS) * R + j0;
                if constexpr (Md::FINAL) {
                    st_lanes<T, LPT>(srow, o);
                } else {
                    st_lanes<T, LPT>(srow, cz);
                    st_lanes<T, LPT>(srow + kTB_STEPS * R, o);
                }
            } else {
                st_lanes<T, LPT>((T*)(Md::FINAL ? p.y : p.acc) + off, o);
                if (Md::ZOUT) st_lanes<T, LPT>((T*)p.z + off, cz);
            }
        }
        float* hcur = halo + (g & 1) * 64;
        if (lane == 0) hcur[warp] = hn[0];
        if (lane == 31) hcur[32 + warp] = hn[LPT - 1];
        if (g + 1 < total) fetch();
        __syncthreads();
#pragma unroll
        for (int e = 0; e < LPT; ++e) h[e] = hn[e];
        if constexpr (TOUT) {
            // a staging block is complete: write it lane-major, 16 bytes per chunk
            const int r = DIR == kTB ? i : H - 1 - i;
            const bool flush = DIR == kTB ? (r % kTB_STEPS == kTB_STEPS - 1 || r == H - 1) : (r % kTB_STEPS == 0);
            if (flush) {
                const int s_base = r - r % kTB_STEPS;
                const int nvalid = min(kTB_STEPS, H - s_base);
                // The ring's waits already cover the u copies of a block longer than NS steps
                // (issued with the block's first step); short blocks and the last step wait here.
                if constexpr (Md::FINAL)
                    if (nvalid <= NS || g + 1 >= total) cp_async_wait<0>();
                // Thread t writes chunk q = t % CPL of lanes t / CPL, t / CPL + T / CPL, ...: a warp
                // covers 32 / CPL whole lane segments per store; its shared reads are runs of
                // consecutive lanes in CPL staging rows (R = 4 mod 32: at most two threads per bank).
                const int q = tid % CPL, jstep = (int)blockDim.x / CPL;
                if (q * CH < nvalid) {
                    const long long gstep = (long long)jstep * H;
                    const T* sp = stg + (size_t)(q * CH) * R + tid / CPL;
                    const long long g0 = poff + (long long)(tid / CPL) * H + s_base + q * CH;
                    if constexpr (Md::FINAL) {
                        T* gp = (T*)p.y + g0;
                        const uint4* up = ubuf + (tid / CPL) * CPL + q;
#pragma unroll 4
                        for (int j = tid / CPL; j < W; j += jstep, sp += jstep, gp += gstep, up += jstep * CPL) {
                            float v[CH], uu[CH];
                            ld_lanes<T, CH>(up, uu);
#pragma unroll
                            for (int k = 0; k < CH; ++k) v[k] = Io<T>::ld(sp + k * R) * uu[k];
                            st_lanes<T, CH>(gp, v);
                        }
                    } else {
                        T* gz = (T*)p.zt + g0;
                        T* ga = (T*)p.acct + g0;
                        const size_t second = (size_t)kTB_STEPS * R;
#pragma unroll 4
                        for (int j = tid / CPL; j < W; j += jstep, sp += jstep, gz += gstep, ga += gstep) {
                            float v[CH], va[CH];
#pragma unroll
                            for (int k = 0; k < CH; ++k) {
                                v[k] = Io<T>::ld(sp + k * R);
                                va[k] = Io<T>::ld(sp + second + k * R);
                            }
                            st_lanes<T, CH>(gz, v);
                            st_lanes<T, CH>(ga, va);
                        }
                    }
                }
                __syncthreads();   // the staging block is reused by the next step
            }
        }
        if (++i == H) {
            i = 0;
            plane += (int)gridDim.x;
            poff = (long long)plane * HW;
        }
    }
    cp_async_wait<0>();
}

// ================================================================== horizontal sweep
__device__ __forceinline__ float u4_get(const uint4& r, int c) {
    return __uint_as_float(c == 0 ? r.x : c == 1 ? r.y : c == 2 ? r.z : r.w);
}

// CTA = one plane at a time. Thread t owns rows t + T*g for g < G. Ring of NS column tiles; a
// tile holds, for every row, S steps: 16 bytes of each storage-dtype input and S*4 bytes of each
// fp32 weight row (WC = S/4 chunks of 16 bytes), laid out [slot][row][16 B] so that
// consecutive threads read consecutive 16-byte chunks.
template <typename T, unsigned DIR, int MODE, int G, int NS>
__global__ void __launch_bounds__(G == 4 ? 256 : (G == 2 ? 512 : 1024), 1) k_hsweep(SweepArgs p, int Hpad) {
    using Md = ModeT<MODE>;
    using SG = Seg<T>;
    constexpr int NTEN = Md::NTEN;
    constexpr int S = SG::S;
    constexpr int WC = S / 4;                             // 16-byte chunks per weight row segment
    constexpr int NSLOT = 2 * WC + NTEN;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align128(smem_raw);
    const int H = p.H, W = p.W;
    const int slotB = Hpad * 16;
    const int stageB = NSLOT * slotB;
    float* halo = (float*)(smem + (size_t)NS * stageB);    // [2 parity][2 lo/hi][G][32 warps]
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int T_ = blockDim.x;
    const long long HW = (long long)H * W;
    const int nb = W / S;                                 // column tiles per plane (W % S == 0)
    const int nplanes = p.N * p.C;
    const int my_planes = (nplanes - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const long long total = (long long)my_planes * nb;

    // Issue cursor (per thread): tiles are requested strictly in order.
    long long iss_left = total;
    int iss_bt = 0, iss_s = 0, iss_plane = (int)blockIdx.x;
    const float* iss_wt = nullptr;
    long long iss_poff = 0;
    auto iss_plane_setup = [&]() {
        const int n = iss_plane / p.C, c = iss_plane % p.C;
        iss_wt = p.wt + ((long long)n * p.Cw + (p.Cw == 1 ? 0 : c)) * 2 * HW;
        iss_poff = (long long)iss_plane * HW;
    };
    auto issue = [&]() {
        if (iss_left > 0) {
            const int b = DIR == kLR ? iss_bt : nb - 1 - iss_bt;
            unsigned char* st = smem + (size_t)iss_s * stageB;
#pragma unroll
            for (int gg = 0; gg < G; ++gg) {
                const int row = tid + T_ * gg;
                if (row < H) {
                    const long long ro = (long long)row * W + (long long)b * S;
                    unsigned char* d = st + (size_t)row * 16;
#pragma unroll
                    for (int k = 0; k < WC; ++k) {
                        cp_async<16>(d + k * slotB, iss_wt + ro + 4 * k);
                        cp_async<16>(d + (WC + k) * slotB, iss_wt + HW + ro + 4 * k);
                    }
                    const long long off = iss_poff + ro;
                    unsigned char* dt = d + 2 * WC * slotB;
                    int t = 0;
                    if (Md::XL) {
                        cp_async<16>(dt + (t++) * slotB, (const T*)p.x + off);
                        cp_async<16>(dt + (t++) * slotB, (const T*)p.lam + off);
                    } else {
                        cp_async<16>(dt + (t++) * slotB, (const T*)p.z + off);
                    }
                    if (Md::ACCIN) cp_async<16>(dt + (t++) * slotB, (const T*)p.acc + off);
                    if (Md::FINAL) cp_async<16>(dt + (t++) * slotB, (const T*)p.u + off);
                }
            }
            --iss_left;
            if (++iss_s == NS) iss_s = 0;
            if (++iss_bt == nb) {
                iss_bt = 0;
                iss_plane += (int)gridDim.x;
                if (iss_plane < nplanes) iss_plane_setup();
            }
        }
        cp_async_commit();
    };
    iss_plane_setup();
#pragma unroll
    for (int q = 0; q < NS; ++q) issue();

    float h[G];
#pragma unroll
    for (int gg = 0; gg < G; ++gg) h[gg] = 0.f;
    long long gstep = 0;   // global step counter (halo parity)
    int bt = 0, cs = 0;    // tile within plane, consumer stage
    long long poff = (long long)blockIdx.x * HW;
    int plane = (int)blockIdx.x;
    for (long long tg = 0; tg < total; ++tg) {
        const int b = DIR == kLR ? bt : nb - 1 - bt;
        if (bt == 0) {
#pragma unroll
            for (int gg = 0; gg < G; ++gg) h[gg] = 0.f;
        }
        // pull this thread's rows of the tile into registers, then refill the stage
        cp_async_wait<NS - 1>();
        uint4 rw0[G][WC], rw2[G][WC], rs0[G], rs1[G], racc[G], ru[G], out0[G], out1[G];
        const unsigned char* st = smem + (size_t)cs * stageB;
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
            const int row = tid + T_ * gg;
            const size_t o = (size_t)row * 16;
#pragma unroll
            for (int k = 0; k < WC; ++k) rw0[gg][k] = rw2[gg][k] = make_uint4(0, 0, 0, 0);
            rs0[gg] = rs1[gg] = racc[gg] = ru[gg] = make_uint4(0, 0, 0, 0);
            if (row < H) {
#pragma unroll
                for (int k = 0; k < WC; ++k) {
                    rw0[gg][k] = *(const uint4*)(st + k * slotB + o);
                    rw2[gg][k] = *(const uint4*)(st + (WC + k) * slotB + o);
                }
                const unsigned char* dt = st + 2 * WC * slotB + o;
                int t = 0;
                rs0[gg] = *(const uint4*)(dt + (t++) * slotB);
                if (Md::XL) rs1[gg] = *(const uint4*)(dt + (t++) * slotB);
                if (Md::ACCIN) racc[gg] = *(const uint4*)(dt + (t++) * slotB);
                if (Md::FINAL) ru[gg] = *(const uint4*)(dt + (t++) * slotB);
            }
            out0[gg] = make_uint4(0, 0, 0, 0);
            out1[gg] = make_uint4(0, 0, 0, 0);
        }
        if (++cs == NS) cs = 0;
        issue();
#pragma unroll
        for (int sj = 0; sj < S; ++sj) {
            const int sl = DIR == kLR ? sj : S - 1 - sj;     // segment slot (column b*S + sl)
            const int col = b * S + sl;
            const int i = DIR == kLR ? col : W - 1 - col;    // scan step
            const float* hprev = halo + ((gstep + 1) & 1) * (2 * G * 32);
            float hn[G];
#pragma unroll
            for (int gg = 0; gg < G; ++gg) {
                const int row = tid + T_ * gg;
                float hl = __shfl_up_sync(0xffffffffu, h[gg], 1);
                float hr = __shfl_down_sync(0xffffffffu, h[gg], 1);
                // edge lanes take the neighbour warp's value (or the previous / next row group's)
                const int il = warp > 0 ? G * 32 + gg * 32 + warp - 1 : G * 32 + (gg > 0 ? gg - 1 : 0) * 32 + nw - 1;
                const int ir = warp < nw - 1 ? gg * 32 + warp + 1 : (gg < G - 1 ? gg + 1 : gg) * 32;
                const float eh = hprev[lane == 0 ? il : ir];
                if (lane == 0) hl = (warp > 0 || gg > 0) ? eh : 0.f;
                if (lane == 31) hr = (warp < nw - 1 || gg < G - 1) ? eh : 0.f;
                float v = 0.f;
                if (row < H) {
                    float zz = SG::get(rs0[gg], sl);
                    if (Md::XL) zz *= SG::get(rs1[gg], sl);
                    v = zz;
                    if (i > 0) {
                        const float w0 = u4_get(rw0[gg][sl >> 2], sl & 3);
                        const float w2 = u4_get(rw2[gg][sl >> 2], sl & 3);
                        v = fmaf(w0, hl, fmaf(1.f - w0 - w2, h[gg], fmaf(w2, hr, v)));
                    }
                    float accv = v;
                    if (Md::ACCIN) accv += SG::get(racc[gg], sl);
                    if (Md::FINAL) SG::put(out0[gg], sl, accv * SG::get(ru[gg], sl));
                    else SG::put(out0[gg], sl, accv);
                    if (Md::ZOUT) SG::put(out1[gg], sl, zz);
                }
                hn[gg] = v;
            }
            float* hcur = halo + (gstep & 1) * (2 * G * 32);
#pragma unroll
            for (int gg = 0; gg < G; ++gg) {
                if (lane == 0) hcur[gg * 32 + warp] = hn[gg];
                if (lane == 31) hcur[G * 32 + gg * 32 + warp] = hn[gg];
                h[gg] = hn[gg];
            }
            __syncthreads();
            ++gstep;
        }
        // write back the tile's outputs as 16-byte row segments
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
            const int row = tid + T_ * gg;
            if (row < H) {
                const long long off = poff + (long long)row * W + (long long)b * S;
                *(uint4*)((T*)(Md::FINAL ? p.y : p.acc) + off) = out0[gg];
                if (Md::ZOUT) *(uint4*)((T*)p.z + off) = out1[gg];
            }
        }
        if (++bt == nb) {
            bt = 0;
            plane += (int)gridDim.x;
            poff = (long long)plane * HW;
        }
    }
    cp_async_wait<0>();
}

// ================================================================== host side
constexpr size_t kSmemBudget = 225 * 1024;

int ntensors(int mode, bool tout = false) {
    switch (mode) {
    case M_FIRST: return tout ? ModeT<M_FIRST, true>::NTEN : ModeT<M_FIRST>::NTEN;
    case M_ONLY: return ModeT<M_ONLY>::NTEN;
    case M_MID: return tout ? ModeT<M_MID, true>::NTEN : ModeT<M_MID>::NTEN;
    default: return tout ? ModeT<M_LAST, true>::NTEN : ModeT<M_LAST>::NTEN;
    }
}
int nstaged(int mode, bool tout) {
    if (!tout) return 0;
    return (mode == M_LAST || mode == M_ONLY) ? 1 : 2;
}

int mode_of(int v, int D) {
    if (D == 1) return M_ONLY;
    if (v == 0) return M_FIRST;
    return v == D - 1 ? M_LAST : M_MID;
}

// ---- vertical geometry: lanes per thread (8, or 4 when W is not a multiple of 8), ring depth
int v_lanes(const Problem& P) {
    int lpt = 8;
    if (const char* e = getenv("GSPN_VLPT")) lpt = atoi(e) == 4 ? 4 : 8;
    if (P.W % 8 != 0) lpt = 4;   // 8 lanes per thread only when every thread's lanes lie in the row
    return lpt;
}
int v_threads(const Problem& P) { return std::max(32, ((P.W / v_lanes(P) + 31) / 32) * 32); }
size_t v_smem(const Problem& P, int mode, int ns, bool tout) {
    const size_t R = ((size_t)(P.W + 31) / 32) * 32 + 16 / P.esize();
    const bool ubuf = tout && (mode == M_LAST || mode == M_ONLY);
    return 128 + (size_t)ns * (2 * (size_t)P.W * 4 + (size_t)ntensors(mode, tout) * P.W * P.esize()) + 512 +
           (size_t)nstaged(mode, tout) * kTB_STEPS * R * P.esize() + 128 +
           (ubuf ? (size_t)P.W * kTB_STEPS * P.esize() : 0);
}
// 4 stages when they fit; 2 when there are more planes than SMs and the shorter ring lets twice
// as many CTAs (planes) share an SM, which hides more of the per-step latency.
int v_stages(const Problem& P, int mode, bool tout = false) {
    const size_t s4 = v_smem(P, mode, 4, tout), s2 = v_smem(P, mode, 2, tout);
    if (s2 > kSmemBudget) return 0;
    if (s4 > kSmemBudget) return 2;
    const bool many = (long long)P.N * P.C > device_sm_count();
    if (many && kSmemBudget / s2 >= 2 * (kSmemBudget / s4)) return 2;
    return 4;
}

// ---- horizontal geometry: threads, rows per thread (as instantiated), padded rows, ring depth
int h_pref_rows() {
    if (const char* e = getenv("GSPN_HROWS")) {
        const int g = atoi(e);
        if (g == 1 || g == 2 || g == 4) return g;
    }
    return 1;
}
int h_threads(const Problem& P) {
    const int t = ((P.H + h_pref_rows() - 1) / h_pref_rows() + 31) / 32 * 32;
    return std::min(1024, std::max(t, ((P.H + 3) / 4 + 31) / 32 * 32));
}
// Rows per thread as instantiated (1, 2 or 4): the kernel's halo and the shared-memory size
// below are both laid out for this value, never for the raw quotient.
int h_rows(const Problem& P) {
    const int g = (P.H + h_threads(P) - 1) / h_threads(P);
    return g <= 1 ? 1 : (g <= 2 ? 2 : 4);
}
int h_pad(const Problem& P) { return ((P.H + 7) / 8) * 8; }
int h_slots(const Problem& P, int mode) { return 2 * ((16 / P.esize()) / 4) + ntensors(mode); }
size_t h_smem(const Problem& P, int mode, int ns) {
    return 128 + (size_t)ns * h_slots(P, mode) * h_pad(P) * 16 + 2 * 2 * h_rows(P) * 32 * sizeof(float);
}
int h_stages(const Problem& P, int mode) {
    if (h_smem(P, mode, 4) <= kSmemBudget) return 4;
    return h_smem(P, mode, 2) <= kSmemBudget ? 2 : 0;
}

// Persistent grid: as many CTAs as fit on the device at once, but never more than planes. Each
// CTA runs one plane's scan at a time, so several CTAs per SM hide the per-step latency when
// there are more planes than SMs.
template <typename K>
int sweep_grid(const Problem& P, K kern, int threads, size_t smem) {
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    return (int)std::min<long long>((long long)per_sm * device_sm_count(), (long long)P.N * P.C);
}

template <typename T, unsigned DIR, int MODE, bool TOUT, int LPT, int NS>
cudaError_t launch_v4(const Problem& P, const SweepArgs& a, cudaStream_t st) {
    const size_t smem = v_smem(P, MODE, NS, TOUT);
    auto kern = k_vsweep<T, DIR, MODE, LPT, NS, TOUT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    const int grid = sweep_grid(P, kern, v_threads(P), smem);
    launch_begin(st);
    k_vsweep<T, DIR, MODE, LPT, NS, TOUT><<<grid, v_threads(P), smem, st>>>(a);
    launch_end(st);
    return cudaGetLastError();
}

template <typename T, unsigned DIR, int MODE, bool TOUT, int LPT>
cudaError_t launch_v3(const Problem& P, const SweepArgs& a, cudaStream_t st) {
    return v_stages(P, MODE, TOUT) == 4 ? launch_v4<T, DIR, MODE, TOUT, LPT, 4>(P, a, st)
                                        : launch_v4<T, DIR, MODE, TOUT, LPT, 2>(P, a, st);
}

template <typename T, unsigned DIR, int MODE, bool TOUT = false>
cudaError_t launch_v(const Problem& P, const SweepArgs& a, cudaStream_t st) {
    return v_lanes(P) == 4 ? launch_v3<T, DIR, MODE, TOUT, 4>(P, a, st)
                           : launch_v3<T, DIR, MODE, TOUT, 8>(P, a, st);
}

template <typename T, unsigned DIR, int MODE, int G, int NS>
cudaError_t launch_h4(const Problem& P, const SweepArgs& a, cudaStream_t st) {
    const size_t smem = h_smem(P, MODE, NS);
    auto kern = k_hsweep<T, DIR, MODE, G, NS>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    const int grid = sweep_grid(P, kern, h_threads(P), smem);
    launch_begin(st);
    k_hsweep<T, DIR, MODE, G, NS><<<grid, h_threads(P), smem, st>>>(a, h_pad(P));
    launch_end(st);
    return cudaGetLastError();
}

template <typename T, unsigned DIR, int MODE, int G>
cudaError_t launch_h3(const Problem& P, const SweepArgs& a, cudaStream_t st) {
    return h_stages(P, MODE) == 4 ? launch_h4<T, DIR, MODE, G, 4>(P, a, st)
                                  : launch_h4<T, DIR, MODE, G, 2>(P, a, st);
}

template <typename T, unsigned DIR, int MODE>
cudaError_t launch_h(const Problem& P, const SweepArgs& a, cudaStream_t st) {
    switch (h_rows(P)) {
    case 1: return launch_h3<T, DIR, MODE, 1>(P, a, st);
    case 2: return launch_h3<T, DIR, MODE, 2>(P, a, st);
    default: return launch_h3<T, DIR, MODE, 4>(P, a, st);
    }
}

template <typename T, unsigned DIR>
cudaError_t launch_dir(const Problem& P, const SweepArgs& a, int mode, cudaStream_t st) {
    if constexpr (DIR == kTB || DIR == kBT) {
        switch (mode) {
        case M_FIRST: return launch_v<T, DIR, M_FIRST>(P, a, st);
        case M_ONLY: return launch_v<T, DIR, M_ONLY>(P, a, st);
        case M_MID: return launch_v<T, DIR, M_MID>(P, a, st);
        default: return launch_v<T, DIR, M_LAST>(P, a, st);
        }
    } else {
        switch (mode) {
        case M_FIRST: return launch_h<T, DIR, M_FIRST>(P, a, st);
        case M_ONLY: return launch_h<T, DIR, M_ONLY>(P, a, st);
        case M_MID: return launch_h<T, DIR, M_MID>(P, a, st);
        default: return launch_h<T, DIR, M_LAST>(P, a, st);
        }
    }
}

size_t table_floats(const Problem& P) { return (size_t)P.D * P.N * P.Cw * 2 * (size_t)P.HW; }

// The transposed path: when the mask has vertical and horizontal directions and both image
// axes give 16-byte rows, the last vertical sweep writes z and the partial sum transposed and
// the horizontal scans run as vertical-style sweeps over those transposed buffers.
Problem swapped(const Problem& P) {
    Problem Q = P;
    std::swap(Q.H, Q.W);
    return Q;
}
bool tpath(const Problem& P) {
    return (P.mask & (kTB | kBT)) && (P.mask & (kLR | kRL)) && (P.H * P.esize()) % 16 == 0 &&
           (P.W * P.esize()) % 16 == 0 && P.H <= 4096;
}
int n_vertical(const Problem& P) { return ((P.mask & kTB) ? 1 : 0) + ((P.mask & kBT) ? 1 : 0); }

template <typename T, unsigned DIR>
cudaError_t launch_vt(const Problem& P, const SweepArgs& a, int mode, bool tout, cudaStream_t st) {
    if (!tout) return launch_dir<T, DIR>(P, a, mode, st);
    switch (mode) {
    case M_FIRST: return launch_v<T, DIR, M_FIRST, true>(P, a, st);
    case M_MID: return launch_v<T, DIR, M_MID, true>(P, a, st);
    case M_LAST: return launch_v<T, DIR, M_LAST, true>(P, a, st);
    default: return cudaErrorNotSupported;
    }
}

template <typename T>
cudaError_t sweep_forward_t(const Problem& P, const void* x, const void* a, const void* lam, const void* u, void* y,
                            void* ws, cudaStream_t st) {
    const bool tp = tpath(P);
    const int nV = n_vertical(P);
    WsCarver wc(ws);
    float* table = wc.take<float>(table_floats(P));
    void* z = P.D > 1 ? wc.take<T>(P.U) : nullptr;
    void* acc = P.D > 1 ? wc.take<T>(P.U) : nullptr;
    void* zt = tp ? wc.take<T>(P.U) : nullptr;
    void* acct = tp ? wc.take<T>(P.U) : nullptr;
    // A1: weight formation for every direction, once per (n, cw) plane
    WeightArgs wa{a, table, P.N, P.Cw, P.H, P.W, P.D, 0, {0u, 0u, 0u, 0u}};
    for (int v = 0, k = 0; k < 4; ++k)
        if (P.mask & (1u << k)) wa.dirs[v++] = 1u << k;
    const int per_slot = P.N * P.Cw;
    const int row_planes = (tp ? nV : P.D) * per_slot;
    cudaError_t e;
    if (row_planes > 0) {
        const int quads = (int)(P.HW / 4);
        const dim3 wgrid((unsigned)std::max(1, std::min((quads + 255) / 256, 64)), (unsigned)row_planes);
        launch_begin(st);
        k_sweep_weights<T><<<wgrid, 256, 0, st>>>(wa);
        launch_end(st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    if (tp) {
        wa.plane0 = nV * per_slot;
        const dim3 tgrid((unsigned)((P.W + 31) / 32), (unsigned)((P.H + 31) / 32), (unsigned)((P.D - nV) * per_slot));
        launch_begin(st);
        k_sweep_weights_t<T><<<tgrid, 256, 0, st>>>(wa);
        launch_end(st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // A2-A6: one sweep per direction
    const size_t slot_floats = (size_t)per_slot * 2 * (size_t)P.HW;
    const Problem PS = swapped(P);
    int v = 0;
    for (unsigned d = kTB; d <= kRL; d <<= 1) {
        if (!(P.mask & d)) continue;
        const int mode = mode_of(v, P.D);
        SweepArgs args{x, lam, u, table + v * slot_floats, z, acc, y, zt, acct, P.N, P.C, P.H, P.W, P.Cw};
        if (is_vertical(d)) {
            const bool tout = tp && v == nV - 1;
            e = d == kTB ? launch_vt<T, kTB>(P, args, mode, tout, st) : launch_vt<T, kBT>(P, args, mode, tout, st);
        } else if (tp) {
            // horizontal scan over the transposed buffers: scan length W, lanes H
            args.z = zt;
            args.acc = acct;
            args.H = PS.H;
            args.W = PS.W;
            const bool tout = v == P.D - 1;
            e = d == kLR ? launch_vt<T, kTB>(PS, args, mode, tout, st) : launch_vt<T, kBT>(PS, args, mode, tout, st);
        } else {
            e = d == kLR ? launch_dir<T, kLR>(P, args, mode, st) : launch_dir<T, kRL>(P, args, mode, st);
        }
        if (e != cudaSuccess) return e;
        ++v;
    }
    return cudaSuccess;
}

}  // namespace

bool sweep_supports(const Problem& P, bool bwd) {
    if (bwd) return false;
    if ((P.W * P.esize()) % 16 != 0) return false;   // 16-byte rows and column tiles
    if (P.W > 4096) return false;
    if ((long long)P.D * P.N * P.Cw > 65535) return false;   // weight-formation grid.y / grid.z
    const bool tp = tpath(P);
    const int nV = n_vertical(P);
    const Problem PS = swapped(P);
    for (int v = 0, k = 0; k < 4; ++k) {
        const unsigned d = 1u << k;
        if (!(P.mask & d)) continue;
        const int mode = mode_of(v, P.D);
        bool ok;
        if (is_vertical(d)) ok = v_stages(P, mode, tp && v == nV - 1) > 0;
        else if (tp) ok = v_stages(PS, mode, v == P.D - 1) > 0;
        else ok = P.H <= 1024 && h_stages(P, mode) > 0;
        if (!ok) return false;
        ++v;
    }
    return true;
}

size_t sweep_ws_bytes(const Problem& P, bool bwd) {
    if (bwd) return 0;
    size_t b = 256 + align256(table_floats(P) * sizeof(float));
    if (P.D > 1) b += 2 * align256((size_t)P.U * P.esize());
    if (tpath(P)) b += 2 * align256((size_t)P.U * P.esize());
    return b;
}

cudaError_t sweep_forward(const Problem& P, const void* x, const void* a, const void* lam, const void* u, void* y,
                          void* ws, cudaStream_t st) {
    if (P.dtype == GSPN_F32) return sweep_forward_t<float>(P, x, a, lam, u, y, ws, st);
    return sweep_forward_t<__nv_bfloat16>(P, x, a, lam, u, y, ws, st);
}

cudaError_t sweep_backward(const Problem&, const void*, const void*, const void*, const void*, const void*, void*,
                           void*, void*, void*, void*, cudaStream_t) {
    return cudaErrorNotSupported;
}

}  // namespace gspn
