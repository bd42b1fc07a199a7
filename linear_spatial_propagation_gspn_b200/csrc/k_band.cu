// k_band.cu -- large-map forward of libgspn with checkpointed scans and band recompute (sm_100a).
//
// The four directions of the forward ("GSPN-2: Efficient Parallel Sequence Modeling" paper notes,
// section "2D spatial propagation review": top->bottom, bottom->top, left->right, right->left,
// summed) come in two opposite pairs. The sum of a pair at one pixel needs both scans' values
// there, but the two scans reach the pixel at opposite ends of their 1024-step chains, so one of
// them must be carried over. Carrying a whole partial-sum plane through HBM costs two plane
// transfers per pair; carrying only the running line every 8 steps (a checkpoint, 1/8 of a plane)
// and recomputing the other scan band by band costs a fraction of that. Per plane:
//
//   P1  top->bottom over x, lambda (z = lambda x): writes z lane-major (for the horizontal pair)
//       and the top->bottom line entering every band of 8 rows (checkpoints);
//   P2  left->right over lane-major z: writes its checkpoints;
//   P3  bottom->top over the bands from the last to the first, interleaved with the top->bottom
//       recompute of the band it will visit next (from that band's checkpoint): one barrier step
//       advances both chains; writes the vertical sum lane-major;
//   P4  the same for right->left with the left->right recompute over lane-major z, adding the
//       vertical sum and writing y = u * (sum of the four) in the image layout.
//
// Each pass is one persistent launch: a CTA owns a whole plane (a line couples all its lanes), the
// running lines live in registers (4 lanes per thread), the j +- 1 neighbours come from warp
// shuffles plus one shared-memory word per warp edge, and one barrier per step orders the
// exchange. Rows stream through a shared-memory ring of per-thread asynchronous copies fed from L2
// (each band's rows are prefetched into L2 a band ahead); lane-major outputs leave through the
// staging blocks and writer warps of the line sweeps (sweep_io.cuh).
#include <algorithm>

#include "gspn_common.cuh"
#include "gspn_internal.h"
#include "sweep_io.cuh"

namespace gspn {
namespace {

using namespace sio;

constexpr int kBand = 8;   // lines per band = checkpoint interval
constexpr int kLpt = 4;    // lanes per scan thread

enum { B_CKZ = 0, B_CK = 1, B_RS = 2, B_RY = 3 };

// Pass arguments in scan coordinates (s.H = steps, s.W = lanes). Fields of s by pass:
//   P1: x, lam, wt (top->bottom slot), zt (z out, lane-major);  P2: z (lane-major z read as rows),
//   wt (left->right slot);  P3: x, lam, wt (bottom->top), acct (sum out, lane-major);  P4: z
//   (lane-major z), acc (vertical sum, lane-major), u, y, wt (right->left).
struct BandArgs {
    SweepArgs s;
    const void* wt_rec;   // recompute chain's table slot (P3: top->bottom; P4: left->right)
    void* ckpt;           // [planes][K][lanes] of T: the ascending chain's line entering band k (k = 0: zeros)
};

// ---- band cursor: element offsets (including the thread's first lane) of one band of one plane
struct Cur {
    long long to;   // weight table: plane slot base + band's first row
    long long po;   // storage tensors: plane base + band's first row
    long long ck;   // checkpoint row of the band
    int plane, bi;  // plane, band index in processing order
    bool live;
};

// Band bi of `plane` in processing order; bands ascend (asc) or descend.
__device__ __forceinline__ void band_setup(Cur& c, const SweepArgs& p, int plane, int bi, bool asc, int K,
                                           long long HW, int WL, int j0) {
    c.plane = plane;
    c.bi = bi;
    c.live = plane < p.N * p.C;
    if (!c.live) return;
    const int b = asc ? bi : K - 1 - bi;
    const int n = plane / p.C, cc = plane - n * p.C;
    const long long tplane = (long long)n * p.Cw + (p.Cw == 1 ? 0 : cc);
    c.to = tplane * 2 * HW + (long long)b * kBand * WL + j0;
    c.po = (long long)plane * HW + (long long)b * kBand * WL + j0;
    c.ck = ((long long)plane * K + b) * WL + j0;
}
__device__ __forceinline__ void band_next(const Cur& c, Cur& n, const SweepArgs& p, bool asc, int K, long long HW,
                                          int WL, int j0) {
    if (c.bi + 1 < K) band_setup(n, p, c.plane, c.bi + 1, asc, K, HW, WL, j0);
    else band_setup(n, p, c.plane + (int)gridDim.x, 0, asc, K, HW, WL, j0);
}

// L2 prefetch of the band's 8 rows of a [rows][WL] tensor with element size esz, starting at
// element offset off (which includes the thread's j0): thread t covers line t % LPR of row
// t / LPR (LPR 128-byte lines per row), so one pass covers NSC / LPR rows.
__device__ __forceinline__ void prefetch_rows(const void* base, long long off, int esz, int WL, int nsc, int tid,
                                              int j0) {
    const int lpr = WL * esz / 128;
    const int per = nsc / lpr;
    for (int r = tid / lpr; r < kBand; r += per) {
        const char* a = (const char*)base + (off - j0 + (long long)r * WL) * esz + (tid % lpr) * 128;
        asm volatile("prefetch.global.L2 [%0];" ::"l"(a));
    }
}

// One recurrence step over a thread's LPT lanes: hn = w0 * left + (1 - w0 - w2) * h + w2 * right + z,
// with the neighbours from warp shuffles and, at the warp edges, hx (a halo word).
template <int LPT>
__device__ __forceinline__ void advance(const float (&h)[LPT], float hx, const float (&w0)[LPT],
                                        const float (&w2)[LPT], const float (&z)[LPT], bool first, bool lastl,
                                        float (&hn)[LPT]) {
    float hl = __shfl_up_sync(0xffffffffu, h[LPT - 1], 1);
    float hr = __shfl_down_sync(0xffffffffu, h[0], 1);
    hl = first ? hx : hl;
    hr = lastl ? hx : hr;
#pragma unroll
    for (int e = 0; e < LPT; ++e) {
        const float left = e == 0 ? hl : h[e - 1];
        const float right = e == LPT - 1 ? hr : h[e + 1];
        const float w1 = 1.f - w0[e] - w2[e];
        hn[e] = fmaf(w0[e], left, fmaf(w1, h[e], fmaf(w2[e], right, z[e])));
    }
}

// ================================================================== single-chain passes (P1, P2)
template <int BR> struct OneRole {
    static constexpr int NT = BR == B_CKZ ? 2 : 1;   // storage rows per ring stage: x, lam | z
    static constexpr bool STG = BR == B_CKZ;         // z leaves lane-major through the writers
};

template <typename T, int BR>
size_t one_smem(int WL, int NS, int SEGB) {
    using WT = typename TableT<T>::type;
    const size_t es = sizeof(T);
    size_t b = 128 + (size_t)NS * (2 * (size_t)WL * sizeof(WT) + (size_t)OneRole<BR>::NT * WL * es) + 2 * 68 * 4 + 4 * 8;
    if (OneRole<BR>::STG) b += 2 * ((size_t)SEGB / es) * ((size_t)WL + 16 / es) * es;
    return b;
}

// Ascending scan of every plane; checkpoints at every band boundary (band 0: zeros); P1 also
// stages z for the lane-major copy.
template <typename T, int BR, int NS, int SEGB, int WL>
__global__ void __launch_bounds__((OneRole<BR>::STG ? 2 : 1) * WL / kLpt, 1) k_band_one(BandArgs P) {
    using Rl = OneRole<BR>;
    using WT = typename TableT<T>::type;
    constexpr int LPT = kLpt;
    constexpr int NSC = WL / LPT;
    constexpr int KST = SEGB / (int)sizeof(T);
    constexpr int ROWB = WL * (int)sizeof(T);
    constexpr int WROWB = WL * (int)sizeof(WT);
    constexpr int STAGEB = 2 * WROWB + Rl::NT * ROWB;
    constexpr int R = WL + 16 / (int)sizeof(T);
    constexpr int STG_BUF = Rl::STG ? KST * R : 0;
    static_assert(WL % (32 * LPT) == 0, "whole warps of lanes");
    // the refill of step u reads step u + NS, at most one band ahead
    static_assert(kBand % NS == 0 && NS < kBand, "ring stages divide a band and look less than a band ahead");
    static_assert(!Rl::STG || KST % kBand == 0 || kBand % KST == 0, "staging blocks align with bands");
    const SweepArgs& p = P.s;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align128(smem_raw);
    unsigned char* ring = smem;
    float* halo = (float*)(smem + (size_t)NS * STAGEB);   // [2 parity][68]
    uint64_t* bars = (uint64_t*)(halo + 2 * 68);
    T* stg = (T*)(bars + 4);

    const int H = p.H, K = H / kBand;
    const long long HW = (long long)H * WL;
    const int tid = threadIdx.x;
    const int nplanes = p.N * p.C;
    const int my_planes = (nplanes - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    for (int k = tid; k < 2 * 68; k += blockDim.x) halo[k] = 0.f;
    if constexpr (Rl::STG) {
        if (tid == 0) {
            mbar_init(&bars[0], (unsigned)NSC);
            mbar_init(&bars[1], (unsigned)NSC);
            mbar_init(&bars[2], blockDim.x - (unsigned)NSC);
            mbar_init(&bars[3], blockDim.x - (unsigned)NSC);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
    }
    __syncthreads();
    if constexpr (Rl::STG) {
        if (tid >= NSC) {
            write_blocks<T, kTB, R_SZ, KST>(p, stg, (size_t)STG_BUF, R, bars, nullptr, tid - NSC, (int)blockDim.x - NSC,
                                            my_planes);
            return;
        }
    }
    const int lane = tid & 31, warp = tid >> 5, j0 = tid * LPT;
    const bool first = lane == 0, lastl = lane == 31;
    const int hread = first ? 34 + warp : (lastl ? warp + 1 : 67);
    const int hwrite = first ? warp : (lastl ? 34 + warp + 1 : 67);

    auto issue_step = [&](int u, const Cur& c) {   // u: step within the band (compile-time)
        if (c.live) {
            unsigned char* st = ring + (u % NS) * STAGEB;
            const WT* tb = (const WT*)p.wt + c.to + u * WL;
            copy_lanes<WT, LPT>(st + j0 * sizeof(WT), tb, 0);
            copy_lanes<WT, LPT>(st + WROWB + j0 * sizeof(WT), tb + HW, 0);
            unsigned char* ts = st + 2 * WROWB + j0 * sizeof(T);
            const long long ro = c.po + u * WL;
            if constexpr (BR == B_CKZ) {
                copy_lanes<T, LPT>(ts, (const T*)p.x + ro, 0);
                copy_lanes<T, LPT>(ts + ROWB, (const T*)p.lam + ro, 0);
            } else {
                copy_lanes<T, LPT>(ts, (const T*)p.z + ro, 0);
            }
        }
        cp_async_commit();   // one group per step, so the wait counts stay uniform
    };
    auto prefetch_band = [&](const Cur& c) {
        if (!c.live) return;
        prefetch_rows(p.wt, c.to, sizeof(WT), WL, NSC, tid, j0);
        prefetch_rows(p.wt, c.to + HW, sizeof(WT), WL, NSC, tid, j0);
        if constexpr (BR == B_CKZ) {
            prefetch_rows(p.x, c.po, sizeof(T), WL, NSC, tid, j0);
            prefetch_rows(p.lam, c.po, sizeof(T), WL, NSC, tid, j0);
        } else {
            prefetch_rows(p.z, c.po, sizeof(T), WL, NSC, tid, j0);
        }
    };
    float nw0[LPT], nw2[LPT], nz[LPT];
    auto fetch = [&](int u, const Cur& cur, const Cur& nxt) {   // u in 0..kBand (compile-time)
        cp_async_wait<NS - 1>();
        const unsigned char* st = ring + ((u % kBand) % NS) * STAGEB;
        read_lanes<WT, LPT>(st + j0 * sizeof(WT), nw0, 0);
        read_lanes<WT, LPT>(st + WROWB + j0 * sizeof(WT), nw2, 0);
        const unsigned char* ts = st + 2 * WROWB + j0 * sizeof(T);
        read_lanes<T, LPT>(ts, nz, 0);
        if constexpr (BR == B_CKZ) {
            float l2[LPT];
            read_lanes<T, LPT>(ts + ROWB, l2, 0);
#pragma unroll
            for (int e = 0; e < LPT; ++e) nz[e] *= l2[e];   // z = x * lambda
        }
        const int ui = u + NS;
        if (ui < kBand) issue_step(ui, cur);
        else issue_step(ui - kBand, nxt);
    };
    auto sync_scan = [&]() {
        if constexpr (Rl::STG) asm volatile("bar.sync 1, %0;" ::"n"(NSC) : "memory");
        else __syncthreads();
    };

    float h[LPT];
#pragma unroll
    for (int e = 0; e < LPT; ++e) h[e] = 0.f;
    int kblk = 0;
    bool dead = false;
    Cur cur, nxt;
    band_setup(cur, p, (int)blockIdx.x, 0, true, K, HW, WL, j0);
    band_next(cur, nxt, p, true, K, HW, WL, j0);
    prefetch_band(cur);
#pragma unroll
    for (int u = 0; u < NS; ++u) issue_step(u, cur);
    fetch(0, cur, nxt);
    while (cur.live) {
        const bool plane_end = cur.bi == K - 1;
        T* ck = (T*)P.ckpt + cur.ck;
        if (cur.bi == 0) {
            const float zero[LPT] = {};
            st_lanes<T, LPT>(ck, zero);
        }
#pragma unroll
        for (int s = 0; s < kBand; ++s) {
            const float hx = halo[((s + 1) & 1) * 68 + hread];
            float hn[LPT];
            advance<LPT>(h, hx, nw0, nw2, nz, first, lastl, hn);
            const bool last_step = plane_end && s == kBand - 1;
            if (s == kBand - 1 && !plane_end) st_lanes<T, LPT>(ck + WL, hn);   // line entering the next band
            if constexpr (Rl::STG) {
                const int ib = (cur.bi * kBand + s) & (KST - 1);
                const int b = kblk & 1;
                if (ib == 0 && kblk >= 2 && !dead)
                    dead = !mbar_wait_bounded<false>(&bars[2 + b], (unsigned)((kblk >> 1) - 1) & 1u, p.status);
                st_lanes<T, LPT>(stg + b * STG_BUF + ib * R + j0, nz);
                if (ib == KST - 1) {
                    mbar_arrive(&bars[b]);
                    ++kblk;
                }
            }
            halo[(s & 1) * 68 + hwrite] = last_step ? 0.f : (lastl ? hn[LPT - 1] : hn[0]);
            if (s == 0) prefetch_band(nxt);
            fetch(s + 1, cur, nxt);
            sync_scan();
#pragma unroll
            for (int e = 0; e < LPT; ++e) h[e] = last_step ? 0.f : hn[e];
        }
        cur = nxt;
        band_next(cur, nxt, p, true, K, HW, WL, j0);
    }
    cp_async_wait<0>();
}

// ================================================================== two-chain passes (P3, P4)
// A period advances the main (descending) chain through band B_{t-1} and the recompute (ascending)
// chain through band B_t, step by step under one barrier: the recompute of a band is ready when
// the main chain reaches it one period later. The recompute's lines and z of a band live in 8
// register slots per lane: at every step the main chain reads a slot and the recompute writes its
// new value into the same slot (slot s in even periods, 7 - s in odd ones), which is exactly the
// slot that the main chain reads for that row one period later.
template <int BR> struct TwoRole {
    static constexpr int WROLE = BR == B_RS ? R_SA : R_SY;   // writers: the sum lane-major, or y with u
    static constexpr bool YSTG = BR == B_RY;
    static constexpr int WRITERS = 128;                      // writer threads
};

template <typename T, int BR>
size_t two_smem(int WL, int NS, int SEGB) {
    using WT = typename TableT<T>::type;
    const size_t es = sizeof(T);
    const size_t kst = (size_t)SEGB / es;
    size_t b = 128 + (size_t)NS * (4 * (size_t)WL * sizeof(WT) + 2 * (size_t)WL * es) + 4 * 68 * 4 + 4 * 8;
    b += 2 * ((size_t)WL + 2 * 16 / es) * es;                 // checkpoint rows
    b += 2 * kst * ((size_t)WL + 16 / es) * es;               // staging
    if (TwoRole<BR>::YSTG) b += 2 * (size_t)WL * kst * es;    // u of two blocks
    return b;
}

template <typename T, int BR, int NS, int SEGB, int WL>
__global__ void __launch_bounds__(WL / kLpt + TwoRole<BR>::WRITERS, 1) k_band_two(BandArgs P) {
    using Rl = TwoRole<BR>;
    using WT = typename TableT<T>::type;
    constexpr int LPT = kLpt;
    constexpr int NSC = WL / LPT;
    constexpr int KST = SEGB / (int)sizeof(T);
    constexpr int ROWB = WL * (int)sizeof(T);
    constexpr int WROWB = WL * (int)sizeof(WT);
    constexpr int STAGEB = 4 * WROWB + 2 * ROWB;   // main w0 w2 | recompute w0 w2 | two storage rows
    constexpr int R = WL + 16 / (int)sizeof(T);
    constexpr int STG_BUF = KST * R;
    constexpr int CKPAD = 16 / (int)sizeof(T);
    constexpr int CKROW = WL + 2 * CKPAD;
    static_assert(WL % (32 * LPT) == 0, "whole warps of lanes");
    static_assert(kBand % NS == 0 && NS < kBand, "ring stages divide a period and look less than a period ahead");
    static_assert(KST % kBand == 0 || kBand % KST == 0, "staging blocks align with bands");
    const SweepArgs& p = P.s;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align128(smem_raw);
    unsigned char* ring = smem;
    float* halo_m = (float*)(smem + (size_t)NS * STAGEB);   // main chain [2 parity][68]
    float* halo_r = halo_m + 2 * 68;                        // recompute chain
    uint64_t* bars = (uint64_t*)(halo_r + 2 * 68);
    T* ckbuf = (T*)(bars + 4);                              // [2][CKROW], lanes from CKPAD, zero padding
    T* stg = ckbuf + 2 * CKROW;
    T* ubuf = stg + 2 * STG_BUF;

    const int H = p.H, K = H / kBand;
    const long long HW = (long long)H * WL;
    const int tid = threadIdx.x;
    const int nplanes = p.N * p.C;
    const int my_planes = (nplanes - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    for (int k = tid; k < 4 * 68; k += blockDim.x) halo_m[k] = 0.f;
    for (int k = tid; k < 2 * CKROW; k += blockDim.x) ckbuf[k] = T(0.f);
    if (tid == 0) {
        mbar_init(&bars[0], (unsigned)NSC);
        mbar_init(&bars[1], (unsigned)NSC);
        mbar_init(&bars[2], blockDim.x - (unsigned)NSC);
        mbar_init(&bars[3], blockDim.x - (unsigned)NSC);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (tid >= NSC) {
        write_blocks<T, kBT, Rl::WROLE, KST>(p, stg, (size_t)STG_BUF, R, bars, ubuf, tid - NSC, (int)blockDim.x - NSC,
                                             my_planes);
        return;
    }
    const int lane = tid & 31, warp = tid >> 5, j0 = tid * LPT;
    const bool first = lane == 0, lastl = lane == 31;
    const int hread = first ? 34 + warp : (lastl ? warp + 1 : 67);
    const int hwrite = first ? warp : (lastl ? 34 + warp + 1 : 67);

    // stage of step u of a period: main part from band m (rows descending), recompute part from r
    auto issue_step = [&](int u, const Cur& m, const Cur& r) {
        unsigned char* st = ring + (u % NS) * STAGEB;
        unsigned char* ts = st + 4 * WROWB + j0 * sizeof(T);
        if (m.live) {
            const WT* tb = (const WT*)p.wt + m.to + (kBand - 1 - u) * WL;
            copy_lanes<WT, LPT>(st + j0 * sizeof(WT), tb, 0);
            copy_lanes<WT, LPT>(st + WROWB + j0 * sizeof(WT), tb + HW, 0);
            if constexpr (BR == B_RY) copy_lanes<T, LPT>(ts + ROWB, (const T*)p.acc + m.po + (kBand - 1 - u) * WL, 0);
        }
        if (r.live) {
            const WT* tb = (const WT*)P.wt_rec + r.to + u * WL;
            copy_lanes<WT, LPT>(st + 2 * WROWB + j0 * sizeof(WT), tb, 0);
            copy_lanes<WT, LPT>(st + 3 * WROWB + j0 * sizeof(WT), tb + HW, 0);
            if constexpr (BR == B_RS) {
                copy_lanes<T, LPT>(ts, (const T*)p.x + r.po + u * WL, 0);
                copy_lanes<T, LPT>(ts + ROWB, (const T*)p.lam + r.po + u * WL, 0);
            } else {
                copy_lanes<T, LPT>(ts, (const T*)p.z + r.po + u * WL, 0);
            }
        }
        cp_async_commit();   // one group per step
    };
    // checkpoint row of band c into buffer buf (joins the next ring group)
    auto issue_ck = [&](const Cur& c, int buf) {
        if (c.live) cp_async<LPT * (int)sizeof(T)>(ckbuf + buf * CKROW + CKPAD + j0, (const T*)P.ckpt + c.ck);
    };
    // the next period's rows into L2: main rows of band m, recompute rows of band r
    auto prefetch_period = [&](const Cur& m, const Cur& r) {
        if (m.live) {
            prefetch_rows(p.wt, m.to, sizeof(WT), WL, NSC, tid, j0);
            prefetch_rows(p.wt, m.to + HW, sizeof(WT), WL, NSC, tid, j0);
            if constexpr (BR == B_RY) prefetch_rows(p.acc, m.po, sizeof(T), WL, NSC, tid, j0);
        }
        if (r.live) {
            prefetch_rows(P.wt_rec, r.to, sizeof(WT), WL, NSC, tid, j0);
            prefetch_rows(P.wt_rec, r.to + HW, sizeof(WT), WL, NSC, tid, j0);
            if constexpr (BR == B_RS) {
                prefetch_rows(p.x, r.po, sizeof(T), WL, NSC, tid, j0);
                prefetch_rows(p.lam, r.po, sizeof(T), WL, NSC, tid, j0);
            } else {
                prefetch_rows(p.z, r.po, sizeof(T), WL, NSC, tid, j0);
            }
        }
    };
    float mw0[LPT], mw2[LPT], rw0[LPT], rw2[LPT], nz[LPT], nacc[LPT];
    // step u (0..kBand, compile-time) out of its stage; refill with step u + NS (next period's
    // stage if it falls beyond this one: main part from cr, recompute part from cn)
    auto fetch = [&](int u, const Cur& cm, const Cur& cr, const Cur& cn) {
        cp_async_wait<NS - 1>();
        const unsigned char* st = ring + ((u % kBand) % NS) * STAGEB;
        read_lanes<WT, LPT>(st + j0 * sizeof(WT), mw0, 0);
        read_lanes<WT, LPT>(st + WROWB + j0 * sizeof(WT), mw2, 0);
        read_lanes<WT, LPT>(st + 2 * WROWB + j0 * sizeof(WT), rw0, 0);
        read_lanes<WT, LPT>(st + 3 * WROWB + j0 * sizeof(WT), rw2, 0);
        const unsigned char* ts = st + 4 * WROWB + j0 * sizeof(T);
        read_lanes<T, LPT>(ts, nz, 0);
        if constexpr (BR == B_RS) {
            float l2[LPT];
            read_lanes<T, LPT>(ts + ROWB, l2, 0);
#pragma unroll
            for (int e = 0; e < LPT; ++e) nz[e] *= l2[e];   // z = x * lambda
        } else {
            read_lanes<T, LPT>(ts + ROWB, nacc, 0);
        }
        const int ui = u + NS;
        if (ui < kBand) issue_step(ui, cm, cr);
        else issue_step(ui - kBand, cr, cn);
    };
    auto sync_scan = [&]() { asm volatile("bar.sync 1, %0;" ::"n"(NSC) : "memory"); };

    float hm[LPT], hr[LPT];
    float zR[kBand][LPT], hR[kBand][LPT];
#pragma unroll
    for (int e = 0; e < LPT; ++e) hm[e] = hr[e] = 0.f;
    int kblk = 0;
    bool dead = false;
    Cur cm, cr, cn;   // B_{t-1} (main), B_t (recompute), B_{t+1}
    cm.live = false;
    cm.bi = 0;
    cm.plane = 0;
    band_setup(cr, p, (int)blockIdx.x, 0, false, K, HW, WL, j0);
    band_next(cr, cn, p, false, K, HW, WL, j0);
    issue_ck(cr, 0);
    prefetch_period(cm, cr);
#pragma unroll
    for (int u = 0; u < NS; ++u) issue_step(u, cm, cr);
    fetch(0, cm, cr, cn);
    sync_scan();   // the first checkpoint row is visible to every scan thread

    // one period; PAR (the period's parity) fixes the register slots and the checkpoint buffer
    auto period = [&](auto par_tag) {
        constexpr int PAR = decltype(par_tag)::value;
        const bool mlive = cm.live, rlive = cr.live;
        const bool plane_end = cm.bi == K - 1;
        if (rlive) {
            const T* ck = ckbuf + PAR * CKROW + CKPAD + j0;
#pragma unroll
            for (int e = 0; e < LPT; ++e) hr[e] = Io<T>::ld(ck + e);
        }
#pragma unroll
        for (int s = 0; s < kBand; ++s) {
            const int slot = PAR == 0 ? s : kBand - 1 - s;
            float hnm[LPT];
            bool last_step = false;
            if (mlive) {
                // ---- main step s: row 8b + 7 - s of band B_{t-1}
                const float hx = halo_m[((s + 1) & 1) * 68 + hread];
                advance<LPT>(hm, hx, mw0, mw2, zR[slot], first, lastl, hnm);
                last_step = plane_end && s == kBand - 1;
                float o[LPT];
#pragma unroll
                for (int e = 0; e < LPT; ++e) {
                    o[e] = hnm[e] + hR[slot][e];
                    if constexpr (BR == B_RY) o[e] += nacc[e];
                }
                const int ib = (cm.bi * kBand + s) & (KST - 1);
                const int rb = KST - 1 - ib;
                const int b = kblk & 1;
                if (ib == 0 && kblk >= 2 && !dead)
                    dead = !mbar_wait_bounded<false>(&bars[2 + b], (unsigned)((kblk >> 1) - 1) & 1u, p.status);
                st_lanes<T, LPT>(stg + b * STG_BUF + rb * R + j0, o);
                if (ib == KST - 1) {
                    mbar_arrive(&bars[b]);
                    ++kblk;
                }
                // the last step of a plane hands zeros to the next plane's first step
                halo_m[(s & 1) * 68 + hwrite] = last_step ? 0.f : (lastl ? hnm[LPT - 1] : hnm[0]);
            }
            if (rlive) {
                // ---- recompute step s: row 8b' + s of band B_t, from its checkpoint at s = 0
                float hx;
                if (s == 0) hx = Io<T>::ld(ckbuf + PAR * CKROW + CKPAD + (first ? j0 - 1 : j0 + LPT));
                else hx = halo_r[((s + 1) & 1) * 68 + hread];
                float hnr[LPT];
                advance<LPT>(hr, hx, rw0, rw2, nz, first, lastl, hnr);
#pragma unroll
                for (int e = 0; e < LPT; ++e) {
                    zR[slot][e] = nz[e];
                    hR[slot][e] = hnr[e];
                    hr[e] = hnr[e];
                }
                halo_r[(s & 1) * 68 + hwrite] = lastl ? hnr[LPT - 1] : hnr[0];
            }
            if (s == 0) {
                issue_ck(cn, PAR ^ 1);     // joins the group of the next refill
                prefetch_period(cr, cn);   // the next period's rows
            }
            fetch(s + 1, cm, cr, cn);
            sync_scan();
            if (mlive) {
#pragma unroll
                for (int e = 0; e < LPT; ++e) hm[e] = last_step ? 0.f : hnm[e];
            }
        }
        cm = cr;
        cr = cn;
        band_next(cr, cn, p, false, K, HW, WL, j0);
    };
    while (cm.live || cr.live) {
        period(std::integral_constant<int, 0>{});
        if (!(cm.live || cr.live)) break;
        period(std::integral_constant<int, 1>{});
    }
    cp_async_wait<0>();
}

// ================================================================== host side
constexpr int kBandLanes = 1024;
constexpr size_t kSmemBudget = 225 * 1024;

// Ring depth and staging segment per pass: 4 stages (the ring reads rows prefetched into L2 a
// band ahead); 32-byte lane-major segments, except in the final pass with 4-byte storage, which
// also keeps u of two staging blocks and so stages 16-byte segments (4 steps).
template <typename T, int BR> struct BandCfgT {
    static constexpr int NS = 4;
    static constexpr int SEGB = (BR == B_RY && sizeof(T) == 4) ? 16 : 32;
};
template <typename T, int BR>
size_t band_smem_cfg() {
    constexpr int NS = BandCfgT<T, BR>::NS, SEGB = BandCfgT<T, BR>::SEGB;
    return (BR == B_CKZ || BR == B_CK) ? one_smem<T, BR>(kBandLanes, NS, SEGB) : two_smem<T, BR>(kBandLanes, NS, SEGB);
}

template <typename T, int BR>
cudaError_t launch_band(const Problem& P, const BandArgs& a, cudaStream_t st) {
    constexpr int NS = BandCfgT<T, BR>::NS, SEGB = BandCfgT<T, BR>::SEGB;
    constexpr bool one = BR == B_CKZ || BR == B_CK;
    const size_t smem = band_smem_cfg<T, BR>();
    if (smem > kSmemBudget) return cudaErrorNotSupported;
    int threads;
    void (*kern)(BandArgs);
    if constexpr (one) {
        kern = k_band_one<T, BR, NS, SEGB, kBandLanes>;
        threads = (OneRole<BR>::STG ? 2 : 1) * kBandLanes / kLpt;
    } else {
        kern = k_band_two<T, BR, NS, SEGB, kBandLanes>;
        threads = kBandLanes / kLpt + TwoRole<BR>::WRITERS;
    }
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    int per_sm = 1;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, threads, smem) != cudaSuccess || per_sm < 1)
        per_sm = 1;
    const int grid = (int)std::min<long long>((long long)per_sm * device_sm_count(), (long long)P.N * P.C);
    launch_begin(st);
    kern<<<grid, threads, smem, st>>>(a);
    launch_end(st);
    return cudaGetLastError();
}

template <typename T>
cudaError_t band_forward_t(const Problem& P, const void* x, const void* a, const void* lam, const void* u, void* y,
                           void* ws, cudaStream_t st) {
    using WT = typename TableT<T>::type;
    WsCarver wc(ws);
    const size_t slot = (size_t)P.N * P.Cw * 2 * (size_t)P.HW;
    WT* table = wc.take<WT>(4 * slot);
    T* zt = wc.take<T>(P.U);
    T* sv = wc.take<T>(P.U);
    T* ckv = wc.take<T>((size_t)P.N * P.C * (P.H / kBand) * (size_t)P.W);
    T* ckh = wc.take<T>((size_t)P.N * P.C * (P.W / kBand) * (size_t)P.H);
    cudaError_t e = launch_weight_table(P, a, table, 2, st);   // TB, BT image layout; LR, RL transposed
    if (e != cudaSuccess) return e;
    unsigned* status = (unsigned*)ws;
    // vertical coordinates: steps = rows (H), lanes = columns (W); horizontal: swapped
    const SweepArgs sv_args{x, lam, u, nullptr, nullptr, nullptr, y, zt, sv, status, P.N, P.C, P.H, P.W, P.Cw, 0};
    const SweepArgs sh_args{x, lam, u, nullptr, zt, sv, y, zt, sv, status, P.N, P.C, P.W, P.H, P.Cw, 0};
    BandArgs b1{sv_args, nullptr, ckv};   // P1: top->bottom checkpoints, z lane-major
    b1.s.wt = table + 0 * slot;
    if ((e = launch_band<T, B_CKZ>(P, b1, st)) != cudaSuccess) return e;
    BandArgs b2{sh_args, nullptr, ckh};   // P2: left->right checkpoints over lane-major z
    b2.s.wt = table + 2 * slot;
    if ((e = launch_band<T, B_CK>(P, b2, st)) != cudaSuccess) return e;
    BandArgs b3{sv_args, table + 0 * slot, ckv};   // P3: bottom->top + top->bottom recompute
    b3.s.wt = table + 1 * slot;
    if ((e = launch_band<T, B_RS>(P, b3, st)) != cudaSuccess) return e;
    BandArgs b4{sh_args, table + 2 * slot, ckh};   // P4: right->left + left->right recompute, y
    b4.s.wt = table + 3 * slot;
    return launch_band<T, B_RY>(P, b4, st);
}

}  // namespace

// The band forward runs the global scan of all four directions on 1024 x 1024 maps with lambda and
// u shared by the directions, when the caller asks for it (GSPN_ALGO_BAND).
bool band_supports(const Problem& P) {
    if (P.mask != 15u || P.chunk != 0 || P.per_dir) return false;
    if (P.H != kBandLanes || P.W != kBandLanes) return false;
    if ((long long)P.N * P.C > 0x7fffffffLL / 2) return false;
    size_t worst;
    if (P.dtype != GSPN_F32)
        worst = std::max({band_smem_cfg<__nv_bfloat16, B_CKZ>(), band_smem_cfg<__nv_bfloat16, B_CK>(),
                          band_smem_cfg<__nv_bfloat16, B_RS>(), band_smem_cfg<__nv_bfloat16, B_RY>()});
    else
        worst = std::max({band_smem_cfg<float, B_CKZ>(), band_smem_cfg<float, B_CK>(), band_smem_cfg<float, B_RS>(),
                          band_smem_cfg<float, B_RY>()});
    return worst <= kSmemBudget;
}

size_t band_ws_bytes(const Problem& P) {
    const size_t es = P.esize();
    const size_t tb = (size_t)P.D * P.N * P.Cw * 2 * (size_t)P.HW * (P.dtype == GSPN_F32 ? 4 : 2);
    const size_t ck = (size_t)P.N * P.C * ((size_t)P.H / kBand * P.W) * es;
    return 256 + align256(tb) + 2 * align256((size_t)P.U * es) + 2 * align256(ck) + 256;
}

cudaError_t band_forward(const Problem& P, const void* x, const void* a, const void* lam, const void* u, void* y,
                         void* ws, cudaStream_t st) {
    if (P.dtype == GSPN_F32) return band_forward_t<float>(P, x, a, lam, u, y, ws, st);
    return band_forward_t<__nv_bfloat16>(P, x, a, lam, u, y, ws, st);
}

}  // namespace gspn
