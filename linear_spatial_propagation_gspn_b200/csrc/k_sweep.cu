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
//
// Horizontal directions. When both image axes give 16-byte rows, the vertical sweeps also write
// z and the partial sum lane-major (transposed), and the horizontal scans run on the vertical
// kernel over those buffers; the last one writes y back in the image layout. A lane-major output
// leaves through a double-buffered shared-memory staging block of KST steps that dedicated
// writer warps drain as one 32- or 64-byte segment per lane while the scan warps go on (hand-off
// by mbarriers), so the scattered segment writes stay off the scan's critical path. Otherwise
// the horizontal scans read column tiles of 16 bytes per row (k_hsweep).
//
// The first sweep reads x and lambda (z = lambda * x); later sweeps read z or recompute it, and
// the partial sum (both in the storage dtype); the last one applies u and writes y. No direction
// issues strided per-element HBM traffic. ("GSPN-2: Efficient Parallel Sequence Modeling" paper
// notes, section "Optimisation 3: efficient CUDA extension": coalesced access and on-chip reuse
// of h_{i-1} were the decisive optimisations on A100.)
#include <stdlib.h>

#include <algorithm>
#include <type_traits>

#include "gspn_common.cuh"
#include "gspn_internal.h"
#include "sweep_io.cuh"

namespace gspn {
namespace {

using namespace sio;

enum { M_FIRST = 0, M_ONLY = 1, M_MID = 2, M_LAST = 3 };

// Column-tile sweep modes (k_hsweep).
template <int MODE> struct ModeT {
    static constexpr bool XL = MODE == M_FIRST || MODE == M_ONLY;     // read x, lam (else z)
    static constexpr bool ACCIN = MODE == M_MID || MODE == M_LAST;    // read the partial sum
    static constexpr bool FINAL = MODE == M_ONLY || MODE == M_LAST;   // read u, write y
    static constexpr bool ZOUT = MODE == M_FIRST;                     // write z
    static constexpr bool URING = FINAL;                              // u comes through the ring
    // storage-dtype tensors per stage: x lam | z, [acc], [u]  (plus the two fp32 weight rows)
    static constexpr int NTEN = (XL ? 2 : 1) + (ACCIN ? 1 : 0) + (URING ? 1 : 0);
};

struct WeightArgs {
    const void* a;    // logits [D][N][Cw][3][H][W]
    void* wt;         // table  [D][N][Cw][2][H][W] of TableT (slots from tslot0 on: [W][H] planes)
    int N, Cw, H, W, D;
    int tslot0;       // first slot written transposed (D: none)
    unsigned dirs[4]; // direction bit of each slot
};

// ================================================================== weight formation (A1)
// Turns the logits of every (slot, n, cw) plane into the two outer weights w0, w2 of each
// normalised tridiagonal row; the sweeps re-derive w1 = 1 - w0 - w2. Elementwise and
// memory-bound, one launch for all slots. A persistent CTA (512 threads) takes tiles of 32 rows
// x 128 columns: thread (tx, ty) loads 4 consecutive columns (one vector per logit row) of rows
// ty and ty + 16, forms the 8 weights (MUFU exponential and reciprocal, the normalisation
// applied afterwards so every row still sums to one up to a few ulp; the max-shifted form for
// logits below -40), and writes them in the image layout straight from registers, or, for the
// transposed slots ([W][H] planes: element (column c, row r) at c * H + r), through a
// shared-memory tile read column-wise (row stride 129 words: conflict-free) so that the table
// writes stay coalesced. Needs W % 4 == 0.
constexpr int kWTileR = 32, kWTileC = 128, kWThreads = 512;

template <typename T>
__global__ void __launch_bounds__(kWThreads) k_weights(WeightArgs p, int tiles_x, int tiles_y, int ntiles) {
    using WT = typename TableT<T>::type;
    constexpr int RPT = kWTileR * 32 / kWThreads;   // rows per thread (2)
    constexpr int RSTEP = kWThreads / 32;           // 16
    __shared__ float tile[2][kWTileR][kWTileC + 1];
    const int H = p.H, W = p.W;
    const long long HW = (long long)H * W;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    const int per_plane = tiles_x * tiles_y;
    const int planes_per_slot = p.N * p.Cw;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
        const int plane = t / per_plane, tt = t - plane * per_plane;
        const int by = tt / tiles_x, bx = tt - by * tiles_x;
        const int slot = plane / planes_per_slot;
        const bool vert = is_vertical(p.dirs[slot]);
        const T* a3 = (const T*)p.a + (long long)plane * 3 * HW;
        WT* wt = (WT*)p.wt + (long long)plane * 2 * HW;
        const int r0 = by * kWTileR, c0 = bx * kWTileC;
        const int c = c0 + 4 * tx;
        const bool cin = c < W;   // W % 4 == 0: a quad is all in or all out
        float l0[RPT][4], l1[RPT][4], l2[RPT][4];
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const int r = r0 + ty + RSTEP * k;
#pragma unroll
            for (int e = 0; e < 4; ++e) l0[k][e] = l1[k][e] = l2[k][e] = 0.f;
            if (cin && r < H) {
                const long long q = (long long)r * W + c;
                ld_lanes<T, 4>(a3 + q, l0[k]);
                ld_lanes<T, 4>(a3 + HW + q, l1[k]);
                ld_lanes<T, 4>(a3 + 2 * HW + q, l2[k]);
            }
        }
        float w0[RPT][4], w2[RPT][4];
#pragma unroll
        for (int k = 0; k < RPT; ++k) {
            const int r = r0 + ty + RSTEP * k;
            const bool in = cin && r < H;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int cc = c + e;
                const bool hl = vert ? cc > 0 : r > 0;
                const bool hr = vert ? cc < W - 1 : r < H - 1;
                Wts w = lane_weights_fast_nocheck(l0[k][e], l1[k][e], l2[k][e], hl, hr);
                if (weights_need_shift(l0[k][e], l1[k][e], l2[k][e], hl, hr))
                    w = weights_shifted(l0[k][e], l1[k][e], l2[k][e], hl, hr);
                w0[k][e] = in ? w.w0 : 0.f;
                w2[k][e] = in ? w.w2 : 0.f;
            }
        }
        if (slot < p.tslot0) {   // image layout, straight from registers
#pragma unroll
            for (int k = 0; k < RPT; ++k) {
                const int r = r0 + ty + RSTEP * k;
                if (cin && r < H) {
                    const long long q = (long long)r * W + c;
                    st_lanes<WT, 4>(wt + q, w0[k]);
                    st_lanes<WT, 4>(wt + HW + q, w2[k]);
                }
            }
        } else {                 // transposed planes (uniform per tile: the barriers are safe)
#pragma unroll
            for (int k = 0; k < RPT; ++k)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    tile[0][ty + RSTEP * k][4 * tx + e] = w0[k][e];
                    tile[1][ty + RSTEP * k][4 * tx + e] = w2[k][e];
                }
            __syncthreads();
            // warp ty writes columns ty, ty + 16, ...: 32 consecutive rows each (lane = row)
            const int r = r0 + tx;
            if (r < H) {
#pragma unroll 4
                for (int cc = ty; cc < kWTileC; cc += RSTEP) {
                    const int col = c0 + cc;
                    if (col < W) {
                        const long long q = (long long)col * H + r;
                        Io<WT>::st(wt + q, tile[0][tx][cc]);
                        Io<WT>::st(wt + HW + q, tile[1][tx][cc]);
                    }
                }
            }
            __syncthreads();
        }
    }
}

// ================================================================== vertical sweep
// CTA = one plane at a time (persistent over planes b, b + grid, ...). Scan thread t owns lanes
// [LPT t, LPT t + LPT). Ring of NS stages; a stage is one image row of the two fp32 weight rows
// and of each storage-dtype input, and every scan thread keeps NS rows of its own lanes in
// flight. The loop is software-pipelined by one step (while step g's new line is exchanged at
// the barrier, every thread has already pulled step g+1's inputs out of the ring) and unrolled by
// NS, so ring stages and halo buffers are compile-time. Bookkeeping is incremental: 32-bit row
// offsets within the plane, plane base pointers set once per plane. A plane starts from h = 0 and
// a zero halo, so its first step needs no special case (h_0 = z exactly). Lane-major roles
// (NSTG > 0) launch as many writer threads as scan threads (write_blocks above); the scan warps
// then synchronise among themselves with named barrier 1.
template <typename T, unsigned DIR, int ROLE, int LPT, int NS, int SEGB>
__global__ void __launch_bounds__(LPT == 8 ? 512 : 1024, 1) k_vsweep(SweepArgs p) {
    using Rl = RoleT<ROLE>;
    constexpr int NTEN = Rl::NTEN;
    constexpr int NSTG = Rl::NSTG;
    constexpr int KST = SEGB / (int)sizeof(T);   // steps per staging block (a power of two)
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align128(smem_raw);
    const int H = p.H, W = p.W;
    const int rowB = W * (int)sizeof(T);
    using WT = typename TableT<T>::type;
    const int wrowB = W * (int)sizeof(WT);
    const int stageB = 2 * wrowB + NTEN * rowB;
    // halo, per step parity: lo[0..32] (lane 0 of warp w writes lo[w]) and hi[0..32] (lane 31 of
    // warp w writes hi[w + 1]); hi[0] and lo[nw] are never written and stay zero, so the first
    // lane's left and the last lane's right neighbour read zero without a test.
    float* halo = (float*)(smem + (size_t)NS * stageB);   // [2 parity][lo 33 | pad | hi 33 | pad] = 2 x 68
    uint64_t* bars = (uint64_t*)(halo + 136);             // full[2], free[2]
    // Staging: two buffers of NSTG blocks [KST][R] in the storage dtype (the values are stored in
    // that dtype anyway). R is W rounded up to 32 plus 16 bytes: every staging row starts 16-byte
    // aligned and consecutive rows shift the bank pattern.
    T* stg = (T*)(bars + 4);
    const int R = ((W + 31) / 32) * 32 + 16 / (int)sizeof(T);
    const size_t stg_buf = (size_t)NSTG * KST * R;
    T* ubuf = stg + 2 * stg_buf;   // final lane-major sweep: u of two blocks, [2][W][KST]
    const int nsc = NSTG > 0 ? (int)blockDim.x / 2 : (int)blockDim.x;
    const int tid = threadIdx.x;
    const long long HW = (long long)H * W;
    const int nplanes = p.N * p.C;
    const int my_planes = (nplanes - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;

    for (int k = tid; k < 2 * 68; k += blockDim.x) halo[k] = 0.f;
    if constexpr (NSTG > 0) {
        if (tid == 0) {
            mbar_init(&bars[0], (unsigned)nsc);
            mbar_init(&bars[1], (unsigned)nsc);
            mbar_init(&bars[2], blockDim.x - (unsigned)nsc);
            mbar_init(&bars[3], blockDim.x - (unsigned)nsc);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
    }
    __syncthreads();
    if constexpr (NSTG > 0) {
        if (tid >= nsc) {
            write_blocks<T, DIR, ROLE, KST>(p, stg, stg_buf, R, bars, ubuf, tid - nsc, (int)blockDim.x - nsc, my_planes);
            return;
        }
    }

    const int lane = tid & 31, warp = tid >> 5;
    const int j0 = tid * LPT;
    const bool active = j0 < W;
    const int sw = (tid >> 2) & 1;
    const int total = my_planes * H;                               // rows this CTA scans
    const int dstep = DIR == kTB ? W : -W;                         // row-offset step in scan order
    const int off0 = (DIR == kTB ? 0 : (H - 1) * W) + j0;          // first row offset of a plane
    const int r0 = DIR == kTB ? 0 : H - 1;                         // first row of a plane
    const int rstep = DIR == kTB ? 1 : -1;
    unsigned char* const wdst = smem + (size_t)j0 * sizeof(WT);                        // + stage
    unsigned char* const tdst = smem + 2 * (size_t)wrowB + (size_t)j0 * sizeof(T);    // + stage

    // ---- issue cursor (rows requested strictly in scan order, NS rows ahead of the consumer)
    int iss_left = total, iss_rows = H, iss_off = off0, iss_plane = (int)blockIdx.x;
    const WT* iw0 = nullptr;
    const WT* iw2 = nullptr;
    const T* isrc[NTEN];
    auto iss_setup = [&]() {
        const int n = iss_plane / p.C, c = iss_plane - n * p.C;
        iw0 = (const WT*)p.wt + ((long long)n * p.Cw + (p.Cw == 1 ? 0 : c)) * 2 * HW;
        iw2 = iw0 + HW;
        const long long po = (long long)iss_plane * HW;
        int t = 0;
        if (Rl::XL) {
            isrc[t++] = (const T*)p.x + po;
            isrc[t++] = (const T*)p.lam + po;
        } else {
            isrc[t++] = (const T*)p.z + po;
        }
        if (Rl::ACCIN) isrc[t++] = (const T*)p.acc + po;
        if (Rl::URING) isrc[t++] = (const T*)p.u + po;
    };
    auto issue = [&](int s) {   // s: compile-time after unrolling
        if (iss_left > 0) {
            if (active) {
                unsigned char* ws = wdst + (size_t)s * stageB;
                copy_lanes<WT, LPT>(ws, iw0 + iss_off, sw);
                copy_lanes<WT, LPT>(ws + wrowB, iw2 + iss_off, sw);
                unsigned char* ts = tdst + (size_t)s * stageB;
#pragma unroll
                for (int t = 0; t < NTEN; ++t) copy_lanes<T, LPT>(ts + t * rowB, isrc[t] + iss_off, sw);
            }
            --iss_left;
            iss_off += dstep;
            if (--iss_rows == 0) {
                iss_rows = H;
                iss_off = off0;
                iss_plane += (int)gridDim.x;
                if (iss_plane < nplanes) iss_setup();
            }
        }
        cp_async_commit();   // always one group per call, so the wait counts stay uniform
    };
    iss_setup();
#pragma unroll
    for (int s = 0; s < NS; ++s) issue(s);

    // ---- inputs of the next step, already out of shared memory (inactive threads keep zeros,
    //      which make their lanes compute h = 0)
    float nz[LPT], nacc[LPT], nu[LPT], nw0[LPT], nw2[LPT];
#pragma unroll
    for (int e = 0; e < LPT; ++e) nz[e] = nacc[e] = nu[e] = nw0[e] = nw2[e] = 0.f;
    auto fetch = [&](int s) {   // s: compile-time after unrolling
        cp_async_wait<NS - 1>();
        if (active) {
            const unsigned char* ws = wdst + (size_t)s * stageB;
            read_lanes<WT, LPT>(ws, nw0, sw);
            read_lanes<WT, LPT>(ws + wrowB, nw2, sw);
            const unsigned char* ts = tdst + (size_t)s * stageB;
            read_lanes<T, LPT>(ts, nz, sw);
            if (Rl::XL) {
                float l2[LPT];
                read_lanes<T, LPT>(ts + rowB, l2, sw);
#pragma unroll
                for (int e = 0; e < LPT; ++e) nz[e] *= l2[e];     // z = x * lam
            }
            int t = Rl::XL ? 2 : 1;
            if (Rl::ACCIN) read_lanes<T, LPT>(ts + (t++) * rowB, nacc, sw);
            if (Rl::URING) read_lanes<T, LPT>(ts + (t++) * rowB, nu, sw);
        }
        issue(s);   // this thread has consumed its lanes of the stage: refill it NS rows ahead
    };
    fetch(0);

    // ---- consumer cursor
    int c_rows = H, c_off = off0, c_r = r0, c_plane = (int)blockIdx.x;
    T* oacc = nullptr;
    T* oy = nullptr;
    T* oz = nullptr;
    auto out_setup = [&]() {
        const long long po = (long long)c_plane * HW;
        if (Rl::ANAT) oacc = (T*)p.acc + po;
        if (Rl::YNAT) oy = (T*)p.y + po;
        if (Rl::ZNAT) oz = (T*)p.z + po;
    };
    out_setup();
    int kblk = 0;        // staging blocks completed by this CTA
    bool dead = false;   // a hand-off wait timed out: stop waiting
    // local propagation: steps left in the current chunk (the plane end also ends a chunk)
    const int cfirst = first_chunk_len(DIR == kTB, H, p.chunk);
    const int clen = p.chunk > 0 ? p.chunk : H;
    int crem = cfirst;
    float h[LPT];
#pragma unroll
    for (int e = 0; e < LPT; ++e) h[e] = 0.f;

    auto step = [&](int u) {   // u: position in the unrolled group (compile-time)
        const float* lo_prev = halo + ((u + 1) & 1) * 68;
        float* lo_cur = halo + (u & 1) * 68;
        float hl = __shfl_up_sync(0xffffffffu, h[LPT - 1], 1);
        float hr = __shfl_down_sync(0xffffffffu, h[0], 1);
        if (lane == 0) hl = lo_prev[34 + warp];          // hi of the warp to the left (0 for warp 0)
        if (lane == 31) hr = lo_prev[warp + 1];          // lo of the warp to the right (0 for the last)
        float hn[LPT];
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            const float left = e == 0 ? hl : h[e - 1];
            const float right = e == LPT - 1 ? hr : h[e + 1];
            const float w1 = 1.f - nw0[e] - nw2[e];
            hn[e] = fmaf(nw0[e], left, fmaf(w1, h[e], fmaf(nw2[e], right, nz[e])));
        }
        float o[LPT];
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            o[e] = Rl::ACCIN ? nacc[e] + hn[e] : hn[e];
            if (Rl::URING) o[e] *= nu[e];
        }
        if (active) {
            if (Rl::ANAT) st_lanes<T, LPT>(oacc + c_off, o);
            if (Rl::YNAT) st_lanes<T, LPT>(oy + c_off, o);
            if (Rl::ZNAT) st_lanes<T, LPT>(oz + c_off, nz);
        }
        if constexpr (NSTG > 0) {
            // staging row of this step; wait for the writers to have emptied the buffer (used
            // two blocks ago) before the block's first row, hand the block over after its last
            const int rb = c_r & (KST - 1);
            const bool bstart = DIR == kTB ? rb == 0 : (rb == KST - 1 || c_r == H - 1);
            const bool bend = DIR == kTB ? (rb == KST - 1 || c_r == H - 1) : rb == 0;
            const int b = kblk & 1;
            if (bstart && kblk >= 2 && !dead)
                dead = !mbar_wait_bounded<false>(&bars[2 + b], (unsigned)((kblk >> 1) - 1) & 1u, p.status);
            if (active) {
                T* srow = stg + (size_t)b * stg_buf + (size_t)rb * R + j0;
                if (Rl::ZSTG) st_lanes<T, LPT>(srow, nz);
                if (Rl::ASTG) st_lanes<T, LPT>(srow + (Rl::ZSTG ? (size_t)KST * R : 0), o);
            }
            if (bend) {
                mbar_arrive(&bars[b]);
                ++kblk;
            }
        }
        // the last row of a chunk or of the plane hands zeros to the next step (a short last
        // chunk ends with the plane)
        const bool last = crem == 1 || c_rows == 1;
        if (lane == 0) lo_cur[warp] = last ? 0.f : hn[0];
        if (lane == 31) lo_cur[34 + warp + 1] = last ? 0.f : hn[LPT - 1];
        fetch((u + 1) % NS);
        if constexpr (NSTG > 0)
            asm volatile("bar.sync 1, %0;" ::"r"(nsc) : "memory");
        else
            __syncthreads();
#pragma unroll
        for (int e = 0; e < LPT; ++e) h[e] = hn[e];
        if (--crem == 0) {
            crem = clen;
#pragma unroll
            for (int e = 0; e < LPT; ++e) h[e] = 0.f;
        }
        c_off += dstep;
        c_r += rstep;
        if (--c_rows == 0) {
            crem = cfirst;
#pragma unroll
            for (int e = 0; e < LPT; ++e) h[e] = 0.f;
            c_rows = H;
            c_off = off0;
            c_r = r0;
            c_plane += (int)gridDim.x;
            if (c_plane < nplanes) out_setup();
        }
    };
    for (int g = 0; g < total; g += NS) {
#pragma unroll
        for (int u = 0; u < NS; ++u)
            if (g + u < total) step(u);
    }
    cp_async_wait<0>();
}

// Fixed-width variant of k_vsweep for lines of WL lanes (WL a multiple of 32 * LPT) and scan
// lengths that are a multiple of 32 (so of NS and of every staging block). With the line width
// known at compile time every ring, halo and staging address is a per-thread base plus an
// immediate, and the plane loop is split so that neither cursor tests for a plane change inside
// the step: per step a scan warp executes little more than its loads, its 6-7 floating-point
// operations per lane, the neighbour exchange and the barrier. Same roles, layouts and
// hand-off protocol as k_vsweep.
template <typename T, unsigned DIR, int ROLE, int LPT, int NS, int SEGB, int WL>
__global__ void __launch_bounds__(2 * WL / LPT, 1) k_vsweep_w(SweepArgs p) {
    using Rl = RoleT<ROLE>;
    constexpr int NTEN = Rl::NTEN;
    constexpr int NSTG = Rl::NSTG;
    constexpr int KST = SEGB / (int)sizeof(T);
    constexpr int NSC = WL / LPT;                         // scan threads
    constexpr int ROWB = WL * (int)sizeof(T);
    using WT = typename TableT<T>::type;
    constexpr int WROWB = WL * (int)sizeof(WT);
    constexpr int STAGEB = 2 * WROWB + NTEN * ROWB;
    constexpr int R = ((WL + 31) / 32) * 32 + 16 / (int)sizeof(T);
    constexpr int STG_BUF = NSTG * KST * R;               // elements per staging buffer
    static_assert(WL % (32 * LPT) == 0, "whole warps of active lanes");
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align128(smem_raw);
    const int H = p.H;
    // [2 parity][lo 33 | pad | hi 33 | pad | sink]: every lane loads and stores one halo word per
    // step at a precomputed address (lanes other than 0 and 31 use a sink word), so the
    // exchange has no branches
    float* halo = (float*)(smem + (size_t)NS * STAGEB);
    uint64_t* bars = (uint64_t*)(halo + 136);
    T* stg = (T*)(bars + 4);
    T* ubuf = stg + 2 * STG_BUF;
    const int tid = threadIdx.x;
    const long long HW = (long long)H * WL;
    const int nplanes = p.N * p.C;
    const int my_planes = (nplanes - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;

    for (int k = tid; k < 2 * 68; k += blockDim.x) halo[k] = 0.f;
    if constexpr (NSTG > 0) {
        if (tid == 0) {
            mbar_init(&bars[0], (unsigned)NSC);
            mbar_init(&bars[1], (unsigned)NSC);
            mbar_init(&bars[2], blockDim.x - (unsigned)NSC);
            mbar_init(&bars[3], blockDim.x - (unsigned)NSC);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
    }
    __syncthreads();
    if constexpr (NSTG > 0) {
        if (tid >= NSC) {
            write_blocks<T, DIR, ROLE, KST>(p, stg, (size_t)STG_BUF, R, bars, ubuf, tid - NSC, (int)blockDim.x - NSC,
                                            my_planes);
            return;
        }
    }

    const int lane = tid & 31, warp = tid >> 5;
    const int j0 = tid * LPT;
    const int sw = (tid >> 2) & 1;
    const bool first = lane == 0, lastl = lane == 31;
    // halo word this lane reads (lane 0: hi of the warp to the left; lane 31: lo of the warp to
    // the right) and writes (lane 0: its lo; lane 31: its hi), per parity offset 0 / 68
    const int hread = first ? 34 + warp : (lastl ? warp + 1 : 67);
    const int hwrite = first ? warp : (lastl ? 34 + warp + 1 : 67);
    constexpr int DSTEP = DIR == kTB ? WL : -WL;
    const int off0 = (DIR == kTB ? 0 : (H - 1) * WL) + j0;
    unsigned char* const wdst = smem + (size_t)j0 * sizeof(WT);
    unsigned char* const tdst = smem + 2 * (size_t)WROWB + (size_t)j0 * sizeof(T);

    // ---- issue cursor: plane bases and a 32-bit row offset
    int iss_off = off0;
    const WT* iw0 = nullptr;
    const WT* iw2 = nullptr;
    const T* isrc[NTEN];
    auto iss_setup = [&](int plane) {
        const int n = plane / p.C, c = plane - n * p.C;
        iw0 = (const WT*)p.wt + ((long long)n * p.Cw + (p.Cw == 1 ? 0 : c)) * 2 * HW;
        iw2 = iw0 + HW;
        const long long po = (long long)plane * HW;
        int t = 0;
        if (Rl::XL) {
            isrc[t++] = (const T*)p.x + po;
            isrc[t++] = (const T*)p.lam + po;
        } else {
            isrc[t++] = (const T*)p.z + po;
        }
        if (Rl::ACCIN) isrc[t++] = (const T*)p.acc + po;
        if (Rl::URING) isrc[t++] = (const T*)p.u + po;
        iss_off = off0;
    };
    auto issue = [&](int s, bool live) {   // s compile-time; live: uniform
        if (live) {
            unsigned char* ws = wdst + s * STAGEB;
            copy_lanes<WT, LPT>(ws, iw0 + iss_off, sw);
            copy_lanes<WT, LPT>(ws + WROWB, iw2 + iss_off, sw);
            unsigned char* ts = tdst + s * STAGEB;
#pragma unroll
            for (int t = 0; t < NTEN; ++t) copy_lanes<T, LPT>(ts + t * ROWB, isrc[t] + iss_off, sw);
            iss_off += DSTEP;
        }
        cp_async_commit();
    };
    float nz[LPT], nacc[LPT], nu[LPT], nw0[LPT], nw2[LPT];
#pragma unroll
    for (int e = 0; e < LPT; ++e) nz[e] = nacc[e] = nu[e] = nw0[e] = nw2[e] = 0.f;
    auto fetch = [&](int s, bool live) {
        cp_async_wait<NS - 1>();
        const unsigned char* ws = wdst + s * STAGEB;
        read_lanes<WT, LPT>(ws, nw0, sw);
        read_lanes<WT, LPT>(ws + WROWB, nw2, sw);
        const unsigned char* ts = tdst + s * STAGEB;
        read_lanes<T, LPT>(ts, nz, sw);
        if (Rl::XL) {
            float l2[LPT];
            read_lanes<T, LPT>(ts + ROWB, l2, sw);
#pragma unroll
            for (int e = 0; e < LPT; ++e) nz[e] *= l2[e];
        }
        int t = Rl::XL ? 2 : 1;
        if (Rl::ACCIN) read_lanes<T, LPT>(ts + (t++) * ROWB, nacc, sw);
        if (Rl::URING) read_lanes<T, LPT>(ts + (t++) * ROWB, nu, sw);
        issue(s, live);
    };

    // ---- consumer state
    int c_off = off0;
    T* oacc = nullptr;
    T* oy = nullptr;
    T* oz = nullptr;
    auto out_setup = [&](int plane) {
        const long long po = (long long)plane * HW;
        if (Rl::ANAT) oacc = (T*)p.acc + po;
        if (Rl::YNAT) oy = (T*)p.y + po;
        if (Rl::ZNAT) oz = (T*)p.z + po;
        c_off = off0;
    };
    int kblk = 0;
    bool dead = false;
    // local propagation: steps left in the current chunk (the plane end also ends a chunk)
    const int cfirst = first_chunk_len(DIR == kTB, H, p.chunk);
    const int clen = p.chunk > 0 ? p.chunk : H;
    int crem = cfirst;
    float h[LPT];
#pragma unroll
    for (int e = 0; e < LPT; ++e) h[e] = 0.f;

    // one step: i = step within the plane (its low bits give the staging row), u = position in
    // the unrolled group, live = the refill has a row to fetch
    auto step = [&](int i, int u, bool live) {
        const float* lo_prev = halo + ((u + 1) & 1) * 68;
        float* lo_cur = halo + (u & 1) * 68;
        const float hx = lo_prev[hread];
        float hl = __shfl_up_sync(0xffffffffu, h[LPT - 1], 1);
        float hr = __shfl_down_sync(0xffffffffu, h[0], 1);
        hl = first ? hx : hl;
        hr = lastl ? hx : hr;
        float hn[LPT];
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            const float left = e == 0 ? hl : h[e - 1];
            const float right = e == LPT - 1 ? hr : h[e + 1];
            const float w1 = 1.f - nw0[e] - nw2[e];
            hn[e] = fmaf(nw0[e], left, fmaf(w1, h[e], fmaf(nw2[e], right, nz[e])));
        }
        float o[LPT];
#pragma unroll
        for (int e = 0; e < LPT; ++e) {
            o[e] = Rl::ACCIN ? nacc[e] + hn[e] : hn[e];
            if (Rl::URING) o[e] *= nu[e];
        }
        if (Rl::ANAT) st_lanes<T, LPT>(oacc + c_off, o);
        if (Rl::YNAT) st_lanes<T, LPT>(oy + c_off, o);
        if (Rl::ZNAT) st_lanes<T, LPT>(oz + c_off, nz);
        if constexpr (NSTG > 0) {
            const int ib = i & (KST - 1);
            const int rb = DIR == kTB ? ib : KST - 1 - ib;
            const int b = kblk & 1;
            if (ib == 0 && kblk >= 2 && !dead)
                dead = !mbar_wait_bounded<false>(&bars[2 + b], (unsigned)((kblk >> 1) - 1) & 1u, p.status);
            T* srow = stg + b * STG_BUF + rb * R + j0;
            if (Rl::ZSTG) st_lanes<T, LPT>(srow, nz);
            if (Rl::ASTG) st_lanes<T, LPT>(srow + (Rl::ZSTG ? KST * R : 0), o);
            if (ib == KST - 1) {
                mbar_arrive(&bars[b]);
                ++kblk;
            }
        }
        // the last row of a chunk or of the plane hands zeros to the next step (a short last
        // chunk ends with the plane)
        const bool last = crem == 1 || i == H - 1;
        lo_cur[hwrite] = last ? 0.f : (lastl ? hn[LPT - 1] : hn[0]);
        fetch((u + 1) % NS, live);
        if constexpr (NSTG > 0)
            asm volatile("bar.sync 1, %0;" ::"n"(NSC) : "memory");
        else
            __syncthreads();
#pragma unroll
        for (int e = 0; e < LPT; ++e) h[e] = hn[e];
        if (--crem == 0) {
            crem = clen;
#pragma unroll
            for (int e = 0; e < LPT; ++e) h[e] = 0.f;
        }
        c_off += DSTEP;
    };

    // Ring protocol: rows 0..NS-1 are issued up front; the fetch of step i (which reads row i + 1)
    // refills the stage it frees with row i + 1 + NS. So in a plane, steps 0..H-NS-2 refill with
    // this plane's rows and steps H-NS-1..H-1 with the next plane's rows 0..NS (the same stream
    // the prologue starts).
    int plane = (int)blockIdx.x;
    iss_setup(plane);
#pragma unroll
    for (int s = 0; s < NS; ++s) issue(s, true);
    fetch(0, true);
    for (int pl = 0; pl < my_planes; ++pl, plane += (int)gridDim.x) {
        out_setup(plane);
        crem = cfirst;
        const bool more = pl + 1 < my_planes;
        int i = 0;
        for (; i < H - 2 * NS; i += NS) {
#pragma unroll
            for (int u = 0; u < NS; ++u) step(i + u, u, true);
        }
#pragma unroll
        for (int u = 0; u < NS; ++u) {
            if (u == NS - 1 && more) iss_setup(plane + (int)gridDim.x);
            step(i + u, u, u < NS - 1 || more);
        }
        i += NS;
#pragma unroll
        for (int u = 0; u < NS; ++u) step(i + u, u, more);
#pragma unroll
        for (int e = 0; e < LPT; ++e) h[e] = 0.f;
    }
    cp_async_wait<0>();
}

// ================================================================== horizontal sweep
__device__ __forceinline__ float u4_get(const uint4& r, int c) {
    return __uint_as_float(c == 0 ? r.x : c == 1 ? r.y : c == 2 ? r.z : r.w);
}
// Weight sl of a row segment held as WC 16-byte chunks of table elements.
template <typename WT, int WC>
__device__ __forceinline__ float wt_get(const uint4 (&r)[WC], int sl) {
    if constexpr (std::is_same<WT, float>::value) {
        return u4_get(r[sl >> 2], sl & 3);
    } else {
        const uint4& q = r[sl >> 3];
        const int e = sl & 7;
        const uint32_t w = (e >> 1) == 0 ? q.x : (e >> 1) == 1 ? q.y : (e >> 1) == 2 ? q.z : q.w;
        const float2 f = unpack2<WT>(w);
        return (e & 1) ? f.y : f.x;
    }
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
    using WT = typename TableT<T>::type;
    constexpr int WC = S * (int)sizeof(WT) / 16;          // 16-byte chunks per weight row segment
    constexpr int WPC = 16 / (int)sizeof(WT);             // weights per chunk
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
    const WT* iss_wt = nullptr;
    long long iss_poff = 0;
    auto iss_plane_setup = [&]() {
        const int n = iss_plane / p.C, c = iss_plane % p.C;
        iss_wt = (const WT*)p.wt + ((long long)n * p.Cw + (p.Cw == 1 ? 0 : c)) * 2 * HW;
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
                        cp_async<16>(d + k * slotB, iss_wt + ro + WPC * k);
                        cp_async<16>(d + (WC + k) * slotB, iss_wt + HW + ro + WPC * k);
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
                    if (!chunk_start(DIR == kLR, W, p.chunk, i)) {
                        const float w0 = wt_get<WT, WC>(rw0[gg], sl);
                        const float w2 = wt_get<WT, WC>(rw2[gg], sl);
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
constexpr size_t kSmemBudget = 225 * 1024;   // dynamic shared memory of one CTA
constexpr size_t kSmemSM = 228 * 1024;       // shared memory of one SM (1 KB of it reserved per CTA)

int ntensors(int mode) {   // horizontal column-tile sweep
    switch (mode) {
    case M_FIRST: return ModeT<M_FIRST>::NTEN;
    case M_ONLY: return ModeT<M_ONLY>::NTEN;
    case M_MID: return ModeT<M_MID>::NTEN;
    default: return ModeT<M_LAST>::NTEN;
    }
}
struct RoleInfo {
    int nten, nstg, ystg, ns_a, seg_a, ns_b2, ns_b4, seg_b;   // ns_b2 / ns_b4: 2- / 4-byte storage
};
template <int ROLE> constexpr RoleInfo role_info_t() {
    using Rl = RoleT<ROLE>;
    return {Rl::NTEN, Rl::NSTG, Rl::YSTG ? 1 : 0, Rl::NS_A, Rl::SEG_A,
            Rl::template ns_b<__nv_bfloat16>(), Rl::template ns_b<float>(), Rl::SEG_B};
}
RoleInfo role_info(int role) {
    switch (role) {
    case R_FIRST: return role_info_t<R_FIRST>();
    case R_ONLY: return role_info_t<R_ONLY>();
    case R_MID: return role_info_t<R_MID>();
    case R_LAST: return role_info_t<R_LAST>();
    case R_SZ: return role_info_t<R_SZ>();
    case R_SA: return role_info_t<R_SA>();
    case R_SZA: return role_info_t<R_SZA>();
    default: return role_info_t<R_SY>();
    }
}

int mode_of(int v, int D) {
    if (D == 1) return M_ONLY;
    if (v == 0) return M_FIRST;
    return v == D - 1 ? M_LAST : M_MID;
}

// ---- vertical geometry: lanes per thread, ring depth
// 8 lanes per thread, or 4: when W is not a multiple of 8 (every thread's lanes must lie in the
// row), and for 1024-lane lines when every plane has an SM to itself (one CTA per SM: twice the
// warps per scheduler hide the per-step latency; with more planes than SMs, the smaller blocks
// of 8 lanes per thread let more CTAs share an SM instead).
constexpr int kFixedLanes = 1024;
int v_lanes(const Problem& P) {
    if (P.W % 8 != 0) return 4;
    if (P.W == kFixedLanes && P.H % 32 == 0 && (long long)P.N * P.C <= device_sm_count()) return 4;
    return 8;
}
int v_threads(const Problem& P) { return std::max(32, ((P.W / v_lanes(P) + 31) / 32) * 32); }
// Weight-table element bytes (TableT): 4 for fp32 storage, 2 (fp16) for bf16 storage.
size_t table_esize(const Problem& P) { return P.dtype == GSPN_F32 ? 4 : 2; }
size_t table_elems(const Problem& P) { return (size_t)P.D * P.N * P.Cw * 2 * (size_t)P.HW; }

int v_block_threads(const Problem& P, int role) { return (role_info(role).nstg ? 2 : 1) * v_threads(P); }
int v_max_threads(const Problem& P) { return v_lanes(P) == 8 ? 512 : 1024; }
size_t v_smem(const Problem& P, int role, int ns, int segb) {
    const RoleInfo ri = role_info(role);
    const size_t R = ((size_t)(P.W + 31) / 32) * 32 + 16 / P.esize();
    const size_t kst = (size_t)segb / P.esize();
    return 128 + (size_t)ns * (2 * (size_t)P.W * table_esize(P) + (size_t)ri.nten * P.W * P.esize()) + 2 * 68 * 4 + 32 +
           2 * (size_t)ri.nstg * kst * R * P.esize() + (ri.ystg ? 2 * (size_t)P.W * kst * P.esize() : 0);
}
// Resident CTAs per SM by shared memory and, assuming the 128-register cap of the 8-lane
// kernels (the largest of them use about that many), by registers.
int ctas_per_sm(size_t smem, int threads) {
    if (smem > kSmemBudget) return 0;
    const int by_smem = (int)(kSmemSM / (smem + 1024));
    const int by_regs = 65536 / (threads * 128);
    return std::max(0, std::min(by_smem, by_regs));
}

// Ring depth and staging segment of a vertical sweep; ns == 0: not supported.
//  - no staged output: 4 stages, or 2 when there are more planes than SMs and the shorter ring
//    lets more CTAs (planes) share an SM, which hides more of the per-step latency;
//  - staged output: configuration A or B of the role, whichever runs more of the planes at once
//    (A on a tie).
struct VCfg {
    int ns, segb;
};
VCfg v_config(const Problem& P, int role) {
    const RoleInfo ri = role_info(role);
    const int threads = v_block_threads(P, role);
    if (ri.nstg == 0) {
        const size_t s4 = v_smem(P, role, 4, 16), s2 = v_smem(P, role, 2, 16);
        if (s2 > kSmemBudget) return {0, 16};
        if (s4 > kSmemBudget) return {2, 16};
        const bool many = (long long)P.N * P.C > device_sm_count();
        if (many && ctas_per_sm(s2, threads) > ctas_per_sm(s4, threads)) return {2, 16};
        return {4, 16};
    }
    if (threads > v_max_threads(P)) return {0, 0};
    const long long planes = (long long)P.N * P.C, sms = device_sm_count();
    const int need = (int)std::min<long long>(64, (planes + sms - 1) / sms);
    const int ns_b = P.esize() == 2 ? ri.ns_b2 : ri.ns_b4;
    const int ua = std::min(ctas_per_sm(v_smem(P, role, ri.ns_a, ri.seg_a), threads), need);
    const int ub = std::min(ctas_per_sm(v_smem(P, role, ns_b, ri.seg_b), threads), need);
    if (ua == 0 && ub == 0) return {0, 0};
    return ua >= ub ? VCfg{ri.ns_a, ri.seg_a} : VCfg{ns_b, ri.seg_b};
}

// ---- horizontal geometry: threads, rows per thread (as instantiated), padded rows, ring depth
int h_pref_rows() { return 1; }
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
// One 16-byte chunk per weight row segment: 4 fp32 or 8 fp16 weights, as many as storage
// elements in a 16-byte segment.
int h_slots(const Problem&, int mode) { return 2 + ntensors(mode); }
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


template <typename T, unsigned DIR, int ROLE, int LPT, int NS, int SEGB>
cudaError_t launch_v4(const Problem& P, const SweepArgs& a, cudaStream_t st) {
    const size_t smem = v_smem(P, ROLE, NS, SEGB);
    const int threads = v_block_threads(P, ROLE);
    auto kern = k_vsweep<T, DIR, ROLE, LPT, NS, SEGB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    const int grid = sweep_grid(P, kern, threads, smem);
    launch_begin(st);
    k_vsweep<T, DIR, ROLE, LPT, NS, SEGB><<<grid, threads, smem, st>>>(a);
    launch_end(st);
    return cudaGetLastError();
}

template <typename T, unsigned DIR, int ROLE, int LPT>
cudaError_t launch_v3(const Problem& P, const SweepArgs& a, const VCfg& c, cudaStream_t st) {
    using Rl = RoleT<ROLE>;
    if constexpr (Rl::NSTG == 0) {
        return c.ns == 4 ? launch_v4<T, DIR, ROLE, LPT, 4, 16>(P, a, st) : launch_v4<T, DIR, ROLE, LPT, 2, 16>(P, a, st);
    } else {
        constexpr int NSB = Rl::template ns_b<T>();
        return (c.ns == Rl::NS_A && c.segb == Rl::SEG_A) ? launch_v4<T, DIR, ROLE, LPT, Rl::NS_A, Rl::SEG_A>(P, a, st)
                                                         : launch_v4<T, DIR, ROLE, LPT, NSB, Rl::SEG_B>(P, a, st);
    }
}

// Fixed-width kernel: 1024-lane lines (the 1024 x 1024 maps in both scan orientations), scan
// lengths a multiple of 32.
bool use_fixed(const Problem& P) {
    return P.W == kFixedLanes && P.H % 32 == 0 && P.H >= 32;
}

template <typename T, unsigned DIR, int ROLE, int LPT, int NS, int SEGB>
cudaError_t launch_w4(const Problem& P, const SweepArgs& a, cudaStream_t st) {
    const size_t smem = v_smem(P, ROLE, NS, SEGB);
    const int threads = v_block_threads(P, ROLE);
    auto kern = k_vsweep_w<T, DIR, ROLE, LPT, NS, SEGB, kFixedLanes>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    const int grid = sweep_grid(P, kern, threads, smem);
    launch_begin(st);
    k_vsweep_w<T, DIR, ROLE, LPT, NS, SEGB, kFixedLanes><<<grid, threads, smem, st>>>(a);
    launch_end(st);
    return cudaGetLastError();
}

template <typename T, unsigned DIR, int ROLE, int LPT>
cudaError_t launch_w3(const Problem& P, const SweepArgs& a, const VCfg& c, cudaStream_t st) {
    using Rl = RoleT<ROLE>;
    if constexpr (Rl::NSTG == 0) {
        return c.ns == 4 ? launch_w4<T, DIR, ROLE, LPT, 4, 16>(P, a, st) : launch_w4<T, DIR, ROLE, LPT, 2, 16>(P, a, st);
    } else {
        constexpr int NSB = Rl::template ns_b<T>();
        return (c.ns == Rl::NS_A && c.segb == Rl::SEG_A) ? launch_w4<T, DIR, ROLE, LPT, Rl::NS_A, Rl::SEG_A>(P, a, st)
                                                         : launch_w4<T, DIR, ROLE, LPT, NSB, Rl::SEG_B>(P, a, st);
    }
}

template <typename T, unsigned DIR, int ROLE>
cudaError_t launch_v(const Problem& P, const SweepArgs& a, cudaStream_t st) {
    const VCfg c = v_config(P, ROLE);
    if (c.ns == 0) return cudaErrorNotSupported;
    if (use_fixed(P))
        return v_lanes(P) == 4 ? launch_w3<T, DIR, ROLE, 4>(P, a, c, st) : launch_w3<T, DIR, ROLE, 8>(P, a, c, st);
    return v_lanes(P) == 4 ? launch_v3<T, DIR, ROLE, 4>(P, a, c, st) : launch_v3<T, DIR, ROLE, 8>(P, a, c, st);
}

// A vertical-kernel sweep in scan order `asc` (top->bottom / left->right) or descending.
template <typename T>
cudaError_t launch_role(bool asc, const Problem& P, const SweepArgs& a, int role, cudaStream_t st) {
    switch (role) {
    case R_FIRST: return asc ? launch_v<T, kTB, R_FIRST>(P, a, st) : launch_v<T, kBT, R_FIRST>(P, a, st);
    case R_ONLY: return asc ? launch_v<T, kTB, R_ONLY>(P, a, st) : launch_v<T, kBT, R_ONLY>(P, a, st);
    case R_MID: return asc ? launch_v<T, kTB, R_MID>(P, a, st) : launch_v<T, kBT, R_MID>(P, a, st);
    case R_LAST: return asc ? launch_v<T, kTB, R_LAST>(P, a, st) : launch_v<T, kBT, R_LAST>(P, a, st);
    case R_SZ: return asc ? launch_v<T, kTB, R_SZ>(P, a, st) : cudaErrorNotSupported;
    case R_SA: return asc ? cudaErrorNotSupported : launch_v<T, kBT, R_SA>(P, a, st);
    case R_SZA: return asc ? launch_v<T, kTB, R_SZA>(P, a, st) : launch_v<T, kBT, R_SZA>(P, a, st);
    case R_SY: return asc ? launch_v<T, kTB, R_SY>(P, a, st) : launch_v<T, kBT, R_SY>(P, a, st);
    default: return cudaErrorNotSupported;
    }
}

template <typename T, unsigned DIR>
cudaError_t launch_hdir(const Problem& P, const SweepArgs& a, int mode, cudaStream_t st) {
    switch (mode) {
    case M_FIRST: return launch_h<T, DIR, M_FIRST>(P, a, st);
    case M_ONLY: return launch_h<T, DIR, M_ONLY>(P, a, st);
    case M_MID: return launch_h<T, DIR, M_MID>(P, a, st);
    default: return launch_h<T, DIR, M_LAST>(P, a, st);
    }
}


// The transposed path: when the mask has vertical and horizontal directions, both image axes
// give 16-byte rows and a line fits a CTA with its writer warps (at most 2048 lanes), the
// vertical sweeps hand z and the partial sum over lane-major and the horizontal scans run as
// vertical-kernel sweeps over those buffers.
Problem swapped(const Problem& P) {
    Problem Q = P;
    std::swap(Q.H, Q.W);
    return Q;
}
bool tpath_geometry(const Problem& P) {
    return (P.mask & (kTB | kBT)) && (P.mask & (kLR | kRL)) && (P.H * P.esize()) % 16 == 0 &&
           (P.W * P.esize()) % 16 == 0 && P.H <= 2048 && P.W <= 2048;
}
int n_vertical(const Problem& P) { return ((P.mask & kTB) ? 1 : 0) + ((P.mask & kBT) ? 1 : 0); }

// How the vertical sweeps hand their results to the horizontal ones on the transposed path: TB
// writes the partial sum scan-major and z lane-major; BT recomputes z from x and lambda, adds its
// scan and writes the partial sum lane-major (one staged output each). With one vertical
// direction it writes both lane-major.

// Role of visit v (direction d).
int visit_role(const Problem& P, unsigned d, int v, bool tp) {
    if (!tp) return mode_of(v, P.D);   // R_FIRST..R_LAST coincide with M_FIRST..M_LAST
    if (is_vertical(d)) {
        if (n_vertical(P) == 1) return R_SZA;
        return v == 0 ? R_SZ : R_SA;
    }
    return v == P.D - 1 ? R_SY : R_MID;
}

// The transposed path is taken when its geometry holds and every one of its sweeps fits a CTA;
// otherwise the horizontal scans fall back to column tiles.
bool tpath(const Problem& P) {
    if (!tpath_geometry(P)) return false;
    const Problem PS = swapped(P);
    for (int v = 0, k = 0; k < 4; ++k) {
        const unsigned d = 1u << k;
        if (!(P.mask & d)) continue;
        if (v_config(is_vertical(d) ? P : PS, visit_role(P, d, v, true)).ns == 0) return false;
        ++v;
    }
    return true;
}

template <typename T>
cudaError_t sweep_forward_t(const Problem& P, const void* x, const void* a, const void* lam, const void* u, void* y,
                            void* ws, cudaStream_t st) {
    const bool tp = tpath(P);
    const int nV = n_vertical(P);
    using WT = typename TableT<T>::type;
    WsCarver wc(ws);
    WT* table = wc.take<WT>(table_elems(P));
    void *z = nullptr, *acc = nullptr, *zt = nullptr, *acct = nullptr;
    if (tp) {
        if (nV == 2) acc = wc.take<T>(P.U);
        zt = wc.take<T>(P.U);
        acct = wc.take<T>(P.U);
    } else if (P.D > 1) {
        z = wc.take<T>(P.U);
        acc = wc.take<T>(P.U);
    }
    // A1: weight formation for every direction, once per (n, cw) plane, in one launch; on the
    // transposed path the horizontal slots (which follow the vertical ones) are written [W][H]
    cudaError_t e = launch_weight_table(P, a, table, tp ? nV : P.D, st);
    if (e != cudaSuccess) return e;
    const int per_slot = P.N * P.Cw;
    // A2-A6: one sweep per direction
    const size_t slot_elems = (size_t)per_slot * 2 * (size_t)P.HW;
    const Problem PS = swapped(P);
    int v = 0;
    for (unsigned d = kTB; d <= kRL; d <<= 1) {
        if (!(P.mask & d)) continue;
        SweepArgs args{x, lam, u, table + v * slot_elems, z, acc, y, zt, acct, (unsigned*)ws,
                       P.N, P.C, P.H, P.W, P.Cw, P.chunk};
        const int role = visit_role(P, d, v, tp);
        const bool asc = d == kTB || d == kLR;
        if (is_vertical(d)) {
            e = launch_role<T>(asc, P, args, role, st);
        } else if (tp) {
            // horizontal scan over the lane-major buffers: scan length W, lanes H
            args.z = zt;
            args.acc = acct;
            args.H = PS.H;
            args.W = PS.W;
            e = launch_role<T>(asc, PS, args, role, st);
        } else {
            e = d == kLR ? launch_hdir<T, kLR>(P, args, role, st) : launch_hdir<T, kRL>(P, args, role, st);
        }
        if (e != cudaSuccess) return e;
        ++v;
    }
    return cudaSuccess;
}

}  // namespace

cudaError_t launch_weight_table(const Problem& P, const void* a, void* table, int tslot0, cudaStream_t st) {
    const bool bf = P.dtype != GSPN_F32;
    WeightArgs wa{a, table, P.N, P.Cw, P.H, P.W, P.D, tslot0, {0u, 0u, 0u, 0u}};
    for (int v = 0, k = 0; k < 4; ++k)
        if (P.mask & (1u << k)) wa.dirs[v++] = 1u << k;
    const int tiles_x = (P.W + kWTileC - 1) / kWTileC, tiles_y = (P.H + kWTileR - 1) / kWTileR;
    const long long ntiles = (long long)P.D * P.N * P.Cw * tiles_x * tiles_y;
    int per_sm = 1;
    const cudaError_t oe = bf ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_weights<__nv_bfloat16>, kWThreads, 0)
                              : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_weights<float>, kWThreads, 0);
    if (oe != cudaSuccess || per_sm < 1) per_sm = 1;
    const int grid = (int)std::min<long long>(ntiles, (long long)per_sm * device_sm_count());
    launch_begin(st);
    if (bf)
        k_weights<__nv_bfloat16><<<grid, kWThreads, 0, st>>>(wa, tiles_x, tiles_y, (int)ntiles);
    else
        k_weights<float><<<grid, kWThreads, 0, st>>>(wa, tiles_x, tiles_y, (int)ntiles);
    launch_end(st);
    return cudaGetLastError();
}

bool sweep_supports(const Problem& P, bool bwd) {
    if (bwd) return false;
    if ((P.W * P.esize()) % 16 != 0) return false;   // 16-byte rows and column tiles
    if (P.W > 4096) return false;
    if ((long long)P.D * P.N * P.Cw * ((P.H + kWTileR - 1) / kWTileR) * ((P.W + kWTileC - 1) / kWTileC) > 0x7fffffffLL)
        return false;   // weight-formation tile count
    const bool tp = tpath(P);
    const Problem PS = swapped(P);
    for (int v = 0, k = 0; k < 4; ++k) {
        const unsigned d = 1u << k;
        if (!(P.mask & d)) continue;
        const int role = visit_role(P, d, v, tp);
        bool ok;
        if (is_vertical(d)) ok = v_config(P, role).ns > 0;
        else if (tp) ok = v_config(PS, role).ns > 0;
        else ok = P.H <= 1024 && h_stages(P, role) > 0;
        if (!ok) return false;
        ++v;
    }
    return true;
}

size_t sweep_ws_bytes(const Problem& P, bool bwd) {
    if (bwd) return 0;
    size_t b = 256 + align256(table_elems(P) * table_esize(P));
    const size_t ub = align256((size_t)P.U * P.esize());
    if (tpath(P)) b += (n_vertical(P) == 2 ? 3 : 2) * ub;
    else if (P.D > 1) b += 2 * ub;
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
