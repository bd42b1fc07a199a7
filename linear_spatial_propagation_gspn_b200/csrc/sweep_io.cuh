// sweep_io.cuh -- data movement shared by the line-sweep kernels of libgspn (sm_100a):
// per-thread asynchronous copies into shared-memory rings, 16-byte row segments, the weight-table
// element type, the lane-major staging protocol between scan warps and writer warps (mbarrier
// hand-off, bounded waits) and the writer loop itself.
#pragma once

#include <stdint.h>

#include <type_traits>

#include "gspn_common.cuh"

namespace gspn {
namespace sio {

// Sweep arguments in scan coordinates: H = scan length (steps), W = lanes. A horizontal scan
// over transposed buffers passes (H, W) = (image width, image height).
struct SweepArgs {
    const void* x;
    const void* lam;
    const void* u;    // scan-major, or lane-major (image layout) for a lane-major final sweep
    const void* wt;   // weight table of this direction's slot: [N][Cw][2][H][W] of TableT (w0, w2)
    void* z;          // workspace, storage dtype, scan-major
    void* acc;        // workspace, storage dtype, scan-major
    void* y;          // output (scan-major, or lane-major for a lane-major final sweep)
    void* zt;         // lane-major z
    void* acct;       // lane-major partial sum
    unsigned* status; // device status word (hand-off timeouts)
    int N, C, H, W, Cw;
    int chunk;        // lines per local chunk along the scan (0: global)
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

// Table element type: fp32 for fp32 storage, fp16 for bf16 storage. The weights lie in [0, 1],
// so fp16's 11-bit significand bounds their relative rounding error by 2^-12, far inside the
// bf16 tolerance (and the sweeps re-derive w1 = 1 - w0 - w2 in fp32, so every row still sums to
// one); it halves the table's traffic and the weight rows of a sweep's ring.
template <typename T> struct TableT { using type = float; };
template <> struct TableT<__nv_bfloat16> { using type = __half; };

// Roles of a vertical sweep. On the transposed path (a vertical and a horizontal direction in the
// mask, 16-byte rows on both axes) the vertical sweeps hand z and the partial sum over
// lane-major, the horizontal scans run as vertical sweeps over those buffers with H and W
// swapped, and the last of them writes y back in the image layout.
enum {
    R_FIRST = 0,   // x, lam -> z, partial                          (scan-major)
    R_ONLY = 1,    // x, lam, u -> y                                (scan-major)
    R_MID = 2,     // z, partial -> partial                         (scan-major)
    R_LAST = 3,    // z, partial, u -> y                            (scan-major)
    R_SZ = 4,      // x, lam -> partial (scan-major), z (lane-major)
    R_SA = 5,      // x, lam, partial -> partial (lane-major)
    R_SZA = 6,     // x, lam -> z and partial (lane-major)
    R_SY = 7,      // z, partial -> y (lane-major, u applied while writing)
};
template <int ROLE> struct RoleT {
    static constexpr bool XL = ROLE == R_FIRST || ROLE == R_ONLY || ROLE == R_SZ || ROLE == R_SA || ROLE == R_SZA;
    static constexpr bool ACCIN = ROLE == R_MID || ROLE == R_LAST || ROLE == R_SA || ROLE == R_SY;
    static constexpr bool URING = ROLE == R_ONLY || ROLE == R_LAST;   // u through the ring
    static constexpr bool ZNAT = ROLE == R_FIRST;
    static constexpr bool ANAT = ROLE == R_FIRST || ROLE == R_MID || ROLE == R_SZ;
    static constexpr bool YNAT = ROLE == R_ONLY || ROLE == R_LAST;
    static constexpr bool ZSTG = ROLE == R_SZ || ROLE == R_SZA;
    static constexpr bool ASTG = ROLE == R_SA || ROLE == R_SZA || ROLE == R_SY;
    static constexpr bool YSTG = ROLE == R_SY;
    // storage-dtype tensors per ring stage: x lam | z, [partial], [u]  (plus two fp32 weight rows)
    static constexpr int NTEN = (XL ? 2 : 1) + (ACCIN ? 1 : 0) + (URING ? 1 : 0);
    static constexpr int NSTG = (ZSTG ? 1 : 0) + (ASTG ? 1 : 0);   // staged (lane-major) outputs
    // (ring stages, lane-major segment bytes) of the two launch configurations: A, and B with
    // less shared memory for more CTAs per SM (a shorter ring at 4-byte storage; at 2-byte
    // storage the halved staging suffices). A final lane-major sweep also keeps u of two blocks.
    static constexpr int NS_A = 4, SEG_A = (NSTG == 1 && !YSTG) ? 64 : 32;
    static constexpr int SEG_B = 32;
    template <typename T> static constexpr int ns_b() { return sizeof(T) == 2 ? 4 : 2; }
};

// ---- mbarrier hand-off between the scan warps and the writer warps of a lane-major sweep
constexpr unsigned long long kHandoffLimitNs = 1000000000ull;   // 1 s: far above any block's time

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, unsigned parity) {
    unsigned ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok)
                 : "r"(smem_u32(bar)), "r"(parity)
                 : "memory");
    return ok != 0u;
}
// Waits for the phase of `bar` with this parity. Gives up after kHandoffLimitNs: the timeout is
// recorded in the status word and the caller carries on as if the phase had completed (its
// outputs are then garbage, but every thread still reaches every barrier, so the kernel ends).
// SLEEP: back off between polls (the writer warps, which wait most of the time and would
// otherwise take issue slots from the scan warps on the same scheduler).
template <bool SLEEP>
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, unsigned parity, unsigned* status) {
    if (mbar_test(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (!mbar_test(bar, parity)) {
        if (globaltimer_ns() - t0 > kHandoffLimitNs) {
            report_timeout(status);
            return false;
        }
        if (SLEEP) __nanosleep(128);
    }
    return true;
}

// Writer warps of a lane-major sweep. The scan warps fill staging block k (KST steps of every
// lane, [step][lane]) in buffer k % 2 and arrive on full[k % 2]; the writers wait for it, write
// each lane's KST steps as one segment of KST * sizeof(T) bytes of the lane-major output, and
// arrive on free[k % 2], which the scan warps wait for before refilling that buffer two blocks
// later. Writer thread f handles chunk q = f % CPL (16 bytes) of lanes f / CPL, f / CPL + nfl /
// CPL, ...: a warp store covers 32 / CPL whole segments. For y, the writers multiply by u, which
// they copy (cp.async, the same chunks) into ubuf[(k + 1) % 2] one block ahead: scattered
// segment reads are latency-bound, so they must be in flight long before they are needed.
template <typename T, unsigned DIR, int ROLE, int KST>
__device__ __forceinline__ void write_blocks(const SweepArgs& p, const T* stg, size_t stg_buf, int R, uint64_t* bars,
                                             T* ubuf, int f, int nfl, int my_planes) {
    using Rl = RoleT<ROLE>;
    constexpr int CH = 16 / (int)sizeof(T);   // steps per 16-byte chunk
    constexpr int CPL = KST / CH;             // chunks per lane segment
    const int H = p.H, W = p.W;
    const long long HW = (long long)H * W;
    const int nbp = (H + KST - 1) / KST;
    const int nblk = my_planes * nbp;
    const int q = f % CPL, j1 = f / CPL, jstep = nfl / CPL;
    // block k -> (plane offset, first step, valid steps)
    auto block_at = [&](int k, long long& poff, int& s_base, int& nvalid) {
        const int pl = k / nbp, bi = k - pl * nbp;
        poff = (long long)((int)blockIdx.x + pl * (int)gridDim.x) * HW;
        s_base = (DIR == kTB ? bi : nbp - 1 - bi) * KST;
        nvalid = min(KST, H - s_base);
    };
    // y only: copy u of block k into ubuf[k % 2] (this thread's chunks), one commit group
    auto prefetch_u = [&](int k) {
        if constexpr (Rl::YSTG) {
            if (k < nblk) {
                long long poff;
                int s_base, nvalid;
                block_at(k, poff, s_base, nvalid);
                if (q * CH < nvalid) {
                    const T* src = (const T*)p.u + poff + s_base + q * CH;
                    T* dst = ubuf + (size_t)(k & 1) * W * KST + q * CH;
                    for (int j = j1; j < W; j += jstep) cp_async<16>(dst + (size_t)j * KST, src + (long long)j * H);
                }
            }
            cp_async_commit();
        }
    };
    prefetch_u(0);
    bool dead = false;
    for (int k = 0; k < nblk; ++k) {
        prefetch_u(k + 1);
        const int b = k & 1;
        if (!dead) dead = !mbar_wait_bounded<true>(&bars[b], (unsigned)(k >> 1) & 1u, p.status);
        long long poff;
        int s_base, nvalid;
        block_at(k, poff, s_base, nvalid);
        if (q * CH < nvalid) {   // H is a multiple of CH: a chunk is either all valid or absent
            const T* sb = stg + (size_t)b * stg_buf + (size_t)(q * CH) * R;
            const long long g0 = poff + s_base + q * CH;
#pragma unroll
            for (int s = 0; s < Rl::NSTG; ++s) {
                const T* ss = sb + (size_t)s * KST * R;
                T* dst = (T*)(Rl::YSTG ? p.y : ((Rl::ZSTG && s == 0) ? p.zt : p.acct));
                if constexpr (Rl::YSTG) {
                    cp_async_wait<1>();   // block k's u has landed (block k + 1's may be in flight)
                    const T* ub = ubuf + (size_t)b * W * KST + q * CH;
#pragma unroll 4
                    for (int j = j1; j < W; j += jstep) {
                        const uint4 uu = *(const uint4*)(ub + (size_t)j * KST);
                        float v[CH];
#pragma unroll
                        for (int kk = 0; kk < CH; ++kk) v[kk] = Io<T>::ld(ss + kk * R + j) * Seg<T>::get(uu, kk);
                        st_lanes<T, CH>(dst + g0 + (long long)j * H, v);
                    }
                } else {
#pragma unroll 4
                    for (int j = j1; j < W; j += jstep) {
                        float v[CH];
#pragma unroll
                        for (int kk = 0; kk < CH; ++kk) v[kk] = Io<T>::ld(ss + kk * R + j);
                        st_lanes<T, CH>(dst + g0 + (long long)j * H, v);
                    }
                }
            }
        }
        mbar_arrive(&bars[2 + b]);
    }
    if constexpr (Rl::YSTG) cp_async_wait<0>();
}

}  // namespace sio
}  // namespace gspn
