// k_sweep.cu -- large-map kernel family of libgspn: persistent, TMA-fed line sweeps.
//
// One sweep per direction in the mask, in the order TB, BT, LR, RL. Every sweep is one
// persistent kernel: each CTA owns whole planes (a line of a scan couples all its lanes, so
// a line cannot be split across CTAs without a per-step exchange) and runs the sequential
// scan over the plane with the running line h_{i-1} in registers. Inputs stream through a
// shared-memory ring filled by the TMA engine; every step ends with one named barrier that
// also exchanges the neighbour values across warps, and after it thread 0 refills the stage
// that was just consumed. No direction issues strided HBM traffic:
//   - vertical sweeps (TB, BT) read whole image rows with 1D bulk copies; each thread owns 4
//     consecutive lanes, read with one 16-byte (fp32) or 8-byte (bf16) shared load;
//   - horizontal sweeps (LR, RL) read [H rows x 16 bytes] column tiles with 2D tensor copies
//     (a staged transpose); each thread owns rows t, t+T, ... and reads 16 bytes (4 fp32 or
//     8 bf16 steps) of each of its rows, conflict-free; outputs are gathered for the tile and
//     written back as 16-byte row segments.
// The first sweep reads x and lambda and writes z = lambda * x and the partial sum; later
// sweeps read z and the partial sum (both in the storage dtype); the last one reads u and
// writes y = u * (partial + h). ("GSPN-2: Efficient Parallel Sequence Modeling" paper notes,
// section "Optimisation 3: efficient CUDA extension": coalesced access and on-chip reuse of
// h_{i-1} were the decisive optimisations on A100; here the line stays in registers.)
#include <algorithm>

#include "gspn_common.cuh"
#include "gspn_internal.h"
#include "tma.cuh"

namespace gspn {
namespace {

enum { M_FIRST = 0, M_ONLY = 1, M_MID = 2, M_LAST = 3 };

template <int MODE> struct ModeT {
    static constexpr bool XL = MODE == M_FIRST || MODE == M_ONLY;     // read x, lam (else z)
    static constexpr bool ACCIN = MODE == M_MID || MODE == M_LAST;    // read the partial sum
    static constexpr bool FINAL = MODE == M_ONLY || MODE == M_LAST;   // read u, write y
    static constexpr bool ZOUT = MODE == M_FIRST;                     // write z
    // tensors per stage: a0 a1 a2, x lam | z, [acc], [u]
    static constexpr int NTEN = 3 + (XL ? 2 : 1) + (ACCIN ? 1 : 0) + (FINAL ? 1 : 0);
};

struct SweepArgs {
    const void* x;
    const void* lam;
    const void* u;
    const void* a;
    void* z;       // workspace, storage dtype
    void* acc;     // workspace, storage dtype
    void* y;
    int N, C, H, W, Cw;
    int slot;
    int ns;        // pipeline stages
    unsigned* status;
    unsigned long long limit_ns;
};

constexpr unsigned long long kWaitLimitNs = 2000000000ULL;  // 2 s

// ------------------------------------------------------------------ 4-lane vectors
template <typename T> struct V4;
template <> struct V4<float> {
    static __device__ __forceinline__ void ld(const void* p, float v[4]) {
        float4 q = *(const float4*)p;
        v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    }
    static __device__ __forceinline__ void st(void* p, const float v[4]) { *(float4*)p = make_float4(v[0], v[1], v[2], v[3]); }
};
template <> struct V4<__nv_bfloat16> {
    static __device__ __forceinline__ void ld(const void* p, float v[4]) {
        uint2 q = *(const uint2*)p;
        float2 f0 = __bfloat1622float2(*(const __nv_bfloat162*)&q.x);
        float2 f1 = __bfloat1622float2(*(const __nv_bfloat162*)&q.y);
        v[0] = f0.x; v[1] = f0.y; v[2] = f1.x; v[3] = f1.y;
    }
    static __device__ __forceinline__ void st(void* p, const float v[4]) {
        __nv_bfloat162 b0 = __floats2bfloat162_rn(v[0], v[1]);
        __nv_bfloat162 b1 = __floats2bfloat162_rn(v[2], v[3]);
        uint2 q;
        q.x = *(const uint32_t*)&b0;
        q.y = *(const uint32_t*)&b1;
        *(uint2*)p = q;
    }
};

// 16-byte row segment: 4 fp32 or 8 bf16 consecutive steps of one lane.
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

__device__ __forceinline__ unsigned char* align128(unsigned char* p) {
    return (unsigned char*)(((uintptr_t)p + 127) & ~(uintptr_t)127);
}

// ================================================================== vertical sweep
// CTA = one plane at a time (persistent over planes b, b + grid, ...), blockDim = W/4 rounded
// up to a warp multiple. Stage = one image row of each input tensor.
template <typename T, unsigned DIR, int MODE>
__global__ void __launch_bounds__(1024, 1) k_vsweep(SweepArgs p) {
    using Md = ModeT<MODE>;
    constexpr int NTEN = Md::NTEN;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align128(smem_raw);
    const int H = p.H, W = p.W, NS = p.ns;
    const int rowB = W * (int)sizeof(T);
    const int stageB = NTEN * rowB;
    unsigned char* stages = smem;
    float* halo = (float*)(smem + (size_t)NS * stageB);   // [2 parity][2 lo/hi][32 warps]
    uint64_t* full = (uint64_t*)(halo + 128);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int j0 = tid * 4;
    const bool active = j0 < W;
    const long long HW = (long long)H * W;
    const int nplanes = p.N * p.C;
    const int my_planes = (nplanes - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const long long total = (long long)my_planes * H;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();

    auto issue = [&](long long g) {
        const int k = (int)(g / H), i = (int)(g % H);
        const int plane = (int)blockIdx.x + k * (int)gridDim.x;
        const int n = plane / p.C, c = plane % p.C;
        const int r = DIR == kTB ? i : H - 1 - i;
        unsigned char* st = stages + (size_t)(g % NS) * stageB;
        uint64_t* bar = &full[g % NS];
        mbar_arrive_expect_tx(bar, (uint32_t)stageB);
        const T* a3 = (const T*)p.a + (((long long)p.slot * p.N + n) * p.Cw + (p.Cw == 1 ? 0 : c)) * 3 * HW +
                      (long long)r * W;
        tma_load_1d(st, a3, rowB, bar);
        tma_load_1d(st + rowB, a3 + HW, rowB, bar);
        tma_load_1d(st + 2 * rowB, a3 + 2 * HW, rowB, bar);
        const long long off = (long long)plane * HW + (long long)r * W;
        int t = 3;
        if (Md::XL) {
            tma_load_1d(st + (t++) * rowB, (const T*)p.x + off, rowB, bar);
            tma_load_1d(st + (t++) * rowB, (const T*)p.lam + off, rowB, bar);
        } else {
            tma_load_1d(st + (t++) * rowB, (const T*)p.z + off, rowB, bar);
        }
        if (Md::ACCIN) tma_load_1d(st + (t++) * rowB, (const T*)p.acc + off, rowB, bar);
        if (Md::FINAL) tma_load_1d(st + (t++) * rowB, (const T*)p.u + off, rowB, bar);
    };
    if (tid == 0)
        for (long long g = 0; g < NS && g < total; ++g) issue(g);

    float h[4] = {0.f, 0.f, 0.f, 0.f};
    long long g = 0;
    bool failed = false;
    for (; g < total; ++g) {
        const int i = (int)(g % H);
        const int k = (int)(g / H);
        if (i == 0) { h[0] = h[1] = h[2] = h[3] = 0.f; }
        const int s = (int)(g % NS);
        const bool ok = mbar_wait_bounded(&full[s], (uint32_t)((g / NS) & 1), p.limit_ns, p.status);
        // neighbours from the previous step: lane j0-1 and lane j0+4
        const float* hprev = halo + ((g + 1) & 1) * 64;
        float hl = __shfl_up_sync(0xffffffffu, h[3], 1);
        float hr = __shfl_down_sync(0xffffffffu, h[0], 1);
        if (lane == 0) hl = warp > 0 ? hprev[32 + warp - 1] : 0.f;
        if (lane == 31) hr = warp < nw - 1 ? hprev[warp + 1] : 0.f;
        float hn[4] = {0.f, 0.f, 0.f, 0.f};
        if (active) {
            const unsigned char* st = stages + (size_t)s * stageB + (size_t)j0 * sizeof(T);
            float zz[4], src1[4];
            V4<T>::ld(st + (Md::XL ? 3 : 3) * rowB, zz);
            if (Md::XL) {
                V4<T>::ld(st + 4 * rowB, src1);
#pragma unroll
                for (int e = 0; e < 4; ++e) zz[e] *= src1[e];   // z = x * lam
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) hn[e] = zz[e];
            if (i > 0) {
                float a0[4], a1[4], a2[4];
                V4<T>::ld(st, a0);
                V4<T>::ld(st + rowB, a1);
                V4<T>::ld(st + 2 * rowB, a2);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = j0 + e;
                    float w0, w1, w2;
                    lane_weights(a0[e], a1[e], a2[e], j > 0, j < W - 1, w0, w1, w2);
                    const float left = e == 0 ? hl : h[e - 1];
                    const float right = e == 3 ? hr : h[e + 1];
                    hn[e] = fmaf(w0, left, fmaf(w1, h[e], fmaf(w2, right, hn[e])));
                }
            }
            const int plane = (int)blockIdx.x + k * (int)gridDim.x;
            const int r = DIR == kTB ? i : H - 1 - i;
            const long long off = (long long)plane * HW + (long long)r * W + j0;
            int t = Md::XL ? 5 : 4;
            float acc[4];
            if (Md::ACCIN) {
                V4<T>::ld(st + (t++) * rowB, acc);
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[e] += hn[e];
            } else {
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[e] = hn[e];
            }
            if (Md::FINAL) {
                float uu[4];
                V4<T>::ld(st + (t++) * rowB, uu);
#pragma unroll
                for (int e = 0; e < 4; ++e) uu[e] *= acc[e];
                V4<T>::st((T*)p.y + off, uu);
            } else {
                V4<T>::st((T*)p.acc + off, acc);
            }
            if (Md::ZOUT) V4<T>::st((T*)p.z + off, zz);
        }
        float* hcur = halo + (g & 1) * 64;
        if (lane == 0) hcur[warp] = hn[0];
        if (lane == 31) hcur[32 + warp] = hn[3];
        const bool any_fail = bar_red_or(1, blockDim.x, !ok);
#pragma unroll
        for (int e = 0; e < 4; ++e) h[e] = hn[e];
        if (any_fail) { failed = true; break; }
        if (tid == 0 && g + NS < total) issue(g + NS);
    }
    if (failed && tid == 0) {
        // drain the copies still in flight before the CTA's shared memory is released
        for (long long q = g + 1; q < total && q < g + NS; ++q)
            mbar_wait_bounded(&full[q % NS], (uint32_t)((q / NS) & 1), p.limit_ns, p.status);
    }
}

// ================================================================== horizontal sweep
struct HMaps {
    CUtensorMap a, src0, src1, acc, u;   // src0/src1 = x/lam, or z/-
};

// CTA = one plane at a time. blockDim T = min(512, H rounded up to 32); thread t owns rows
// t + T*g for g < G. Stage = one column tile [Hpad rows x 16 bytes] of each input tensor.
template <typename T, unsigned DIR, int MODE, int G>
__global__ void __launch_bounds__(512, 1) k_hsweep(SweepArgs p, const __grid_constant__ HMaps maps, int box_rows,
                                                   int nbox) {
    using Md = ModeT<MODE>;
    using SG = Seg<T>;
    constexpr int NTEN = Md::NTEN;
    constexpr int S = SG::S;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align128(smem_raw);
    const int H = p.H, W = p.W, NS = p.ns;
    const int Hpad = box_rows * nbox;
    const int tenB = Hpad * 16;
    const int stageB = NTEN * tenB;
    unsigned char* stages = smem;
    float* halo = (float*)(smem + (size_t)NS * stageB);    // [2 parity][2 lo/hi][G][16 warps]
    uint64_t* full = (uint64_t*)(halo + 2 * 2 * G * 16);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    const int T_ = blockDim.x;
    const long long HW = (long long)H * W;
    const int nb = (W + S - 1) / S;                       // column tiles per plane
    const int nplanes = p.N * p.C;
    const int my_planes = (nplanes - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const long long total = (long long)my_planes * nb;

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(&full[s], 1);
        fence_mbar_init();
    }
    __syncthreads();

    auto issue = [&](long long tg) {
        const int k = (int)(tg / nb), bt = (int)(tg % nb);
        const int b = DIR == kLR ? bt : nb - 1 - bt;
        const int plane = (int)blockIdx.x + k * (int)gridDim.x;
        const int n = plane / p.C, c = plane % p.C;
        unsigned char* st = stages + (size_t)(tg % NS) * stageB;
        uint64_t* bar = &full[tg % NS];
        mbar_arrive_expect_tx(bar, (uint32_t)stageB);
        const int x0 = b * S;
        const int arow = (int)((((long long)p.slot * p.N + n) * p.Cw + (p.Cw == 1 ? 0 : c)) * 3 * H);
        const int prow = plane * H;
        for (int bx = 0; bx < nbox; ++bx) {
            const int ro = bx * box_rows;
            unsigned char* d = st + (size_t)ro * 16;
            tma_load_2d(d, &maps.a, x0, arow + ro, bar);
            tma_load_2d(d + tenB, &maps.a, x0, arow + H + ro, bar);
            tma_load_2d(d + 2 * tenB, &maps.a, x0, arow + 2 * H + ro, bar);
            int t = 3;
            tma_load_2d(d + (t++) * tenB, &maps.src0, x0, prow + ro, bar);
            if (Md::XL) tma_load_2d(d + (t++) * tenB, &maps.src1, x0, prow + ro, bar);
            if (Md::ACCIN) tma_load_2d(d + (t++) * tenB, &maps.acc, x0, prow + ro, bar);
            if (Md::FINAL) tma_load_2d(d + (t++) * tenB, &maps.u, x0, prow + ro, bar);
        }
    };
    if (tid == 0)
        for (long long q = 0; q < NS && q < total; ++q) issue(q);

    float h[G];
#pragma unroll
    for (int gg = 0; gg < G; ++gg) h[gg] = 0.f;
    long long tg = 0;
    long long gstep = 0;   // global step counter (halo parity)
    bool failed = false;
    for (; tg < total; ++tg) {
        const int k = (int)(tg / nb), bt = (int)(tg % nb);
        const int b = DIR == kLR ? bt : nb - 1 - bt;
        if (bt == 0) {
#pragma unroll
            for (int gg = 0; gg < G; ++gg) h[gg] = 0.f;
        }
        const int s = (int)(tg % NS);
        const bool ok = mbar_wait_bounded(&full[s], (uint32_t)((tg / NS) & 1), p.limit_ns, p.status);
        // pull this thread's rows of the tile into registers
        uint4 ra0[G], ra1[G], ra2[G], rs0[G], rs1[G], racc[G], ru[G], out0[G], out1[G];
        const unsigned char* st = stages + (size_t)s * stageB;
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
            const int row = tid + T_ * gg;
            const size_t o = (size_t)row * 16;
            if (row < H) {
                ra0[gg] = *(const uint4*)(st + o);
                ra1[gg] = *(const uint4*)(st + tenB + o);
                ra2[gg] = *(const uint4*)(st + 2 * tenB + o);
                int t = 3;
                rs0[gg] = *(const uint4*)(st + (t++) * tenB + o);
                if (Md::XL) rs1[gg] = *(const uint4*)(st + (t++) * tenB + o);
                if (Md::ACCIN) racc[gg] = *(const uint4*)(st + (t++) * tenB + o);
                if (Md::FINAL) ru[gg] = *(const uint4*)(st + (t++) * tenB + o);
            }
            out0[gg] = make_uint4(0, 0, 0, 0);
            out1[gg] = make_uint4(0, 0, 0, 0);
        }
        const int plane = (int)blockIdx.x + k * (int)gridDim.x;
#pragma unroll
        for (int sj = 0; sj < S; ++sj) {
            const int sl = DIR == kLR ? sj : S - 1 - sj;     // segment slot (column b*S + sl)
            const int col = b * S + sl;
            const bool valid = col < W;                      // uniform across the CTA
            const int i = DIR == kLR ? col : W - 1 - col;    // scan step
            const float* hprev = halo + ((gstep + 1) & 1) * (2 * G * 16);
            float hn[G];
#pragma unroll
            for (int gg = 0; gg < G; ++gg) {
                const int row = tid + T_ * gg;
                float hl = __shfl_up_sync(0xffffffffu, h[gg], 1);
                float hr = __shfl_down_sync(0xffffffffu, h[gg], 1);
                if (lane == 0) {
                    if (warp > 0) hl = hprev[G * 16 + gg * 16 + warp - 1];
                    else hl = gg > 0 ? hprev[G * 16 + (gg - 1) * 16 + nw - 1] : 0.f;
                }
                if (lane == 31) {
                    if (warp < nw - 1) hr = hprev[gg * 16 + warp + 1];
                    else hr = gg < G - 1 ? hprev[(gg + 1) * 16] : 0.f;
                }
                float v = 0.f;
                if (valid && row < H) {
                    float zz = SG::get(rs0[gg], sl);
                    if (Md::XL) zz *= SG::get(rs1[gg], sl);
                    v = zz;
                    if (i > 0) {
                        float w0, w1, w2;
                        lane_weights(SG::get(ra0[gg], sl), SG::get(ra1[gg], sl), SG::get(ra2[gg], sl), row > 0,
                                     row < H - 1, w0, w1, w2);
                        v = fmaf(w0, hl, fmaf(w1, h[gg], fmaf(w2, hr, v)));
                    }
                    float accv = v;
                    if (Md::ACCIN) accv += SG::get(racc[gg], sl);
                    if (Md::FINAL) SG::put(out0[gg], sl, accv * SG::get(ru[gg], sl));
                    else SG::put(out0[gg], sl, accv);
                    if (Md::ZOUT) SG::put(out1[gg], sl, zz);
                }
                hn[gg] = valid ? v : h[gg];
            }
            float* hcur = halo + (gstep & 1) * (2 * G * 16);
#pragma unroll
            for (int gg = 0; gg < G; ++gg) {
                if (lane == 0) hcur[gg * 16 + warp] = hn[gg];
                if (lane == 31) hcur[G * 16 + gg * 16 + warp] = hn[gg];
                h[gg] = hn[gg];
            }
            const bool any_fail = bar_red_or(1, blockDim.x, !ok);
            ++gstep;
            if (any_fail) { failed = true; break; }
            // every thread copied its rows of this stage into registers before the first
            // barrier of the tile, so the stage can be refilled now
            if (sj == 0 && tid == 0 && tg + NS < total) issue(tg + NS);
        }
        if (failed) break;
        // write back the tile's outputs as 16-byte row segments
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
            const int row = tid + T_ * gg;
            if (row < H) {
                const long long off = (long long)plane * HW + (long long)row * W + (long long)b * S;
                const bool full_seg = (b + 1) * S <= W;
                T* dst = Md::FINAL ? (T*)p.y : (T*)p.acc;
                if (full_seg) {
                    *(uint4*)(dst + off) = out0[gg];
                    if (Md::ZOUT) *(uint4*)((T*)p.z + off) = out1[gg];
                } else {
                    for (int sl = 0; sl < W - b * S; ++sl) {
                        Io<T>::st(dst + off + sl, SG::get(out0[gg], sl));
                        if (Md::ZOUT) Io<T>::st((T*)p.z + off + sl, SG::get(out1[gg], sl));
                    }
                }
            }
        }
    }
    if (failed && tid == 0) {
        for (long long q = tg + 1; q < total && q < tg + NS; ++q)
            mbar_wait_bounded(&full[q % NS], (uint32_t)((q / NS) & 1), p.limit_ns, p.status);
    }
}

// ================================================================== host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)ptr;
    }
    return fn;
}

// 2D map over a [rows x W] row-major tensor with a box of [box_rows x 16 bytes].
bool make_map(CUtensorMap* m, const void* base, int dtype, long long rows, int W, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const int es = dtype == GSPN_F32 ? 4 : 2;
    cuuint64_t dims[2] = {(cuuint64_t)W, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)W * es};
    cuuint32_t box[2] = {(cuuint32_t)(16 / es), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, dtype == GSPN_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

constexpr int kSmemBudget = 225 * 1024;

int ntensors(int mode) {
    switch (mode) {
    case M_FIRST: return ModeT<M_FIRST>::NTEN;
    case M_ONLY: return ModeT<M_ONLY>::NTEN;
    case M_MID: return ModeT<M_MID>::NTEN;
    default: return ModeT<M_LAST>::NTEN;
    }
}

int v_stages(const Problem& P, int mode) {
    const size_t stageB = (size_t)ntensors(mode) * P.W * P.esize();
    int ns = (int)((kSmemBudget - 1024) / stageB);
    return std::min(ns, 4);
}

void h_geometry(const Problem& P, int* box_rows, int* nbox, int* threads, int* G) {
    *box_rows = std::min(256, ((P.H + 7) / 8) * 8);
    *nbox = (P.H + *box_rows - 1) / *box_rows;
    *threads = std::min(512, ((P.H + 31) / 32) * 32);
    *G = (*nbox * *box_rows + *threads - 1) / *threads;
}

int h_stages(const Problem& P, int mode) {
    int br, nbox, thr, G;
    h_geometry(P, &br, &nbox, &thr, &G);
    const size_t stageB = (size_t)ntensors(mode) * br * nbox * 16;
    int ns = (int)((kSmemBudget - 4096) / stageB);
    return std::min(ns, 3);
}

int mode_of(int v, int D) {
    if (D == 1) return M_ONLY;
    if (v == 0) return M_FIRST;
    return v == D - 1 ? M_LAST : M_MID;
}

template <typename T, unsigned DIR, int MODE>
cudaError_t launch_v(const Problem& P, SweepArgs a, cudaStream_t st) {
    a.ns = v_stages(P, MODE);
    const int threads = std::max(32, ((P.W / 4 + 31) / 32) * 32);
    const size_t smem = 128 + (size_t)a.ns * ModeT<MODE>::NTEN * P.W * sizeof(T) + 128 * sizeof(float) + 8 * 8;
    const int grid = std::min(P.N * P.C, device_sm_count());
    cudaFuncSetAttribute(k_vsweep<T, DIR, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_begin(st);
    k_vsweep<T, DIR, MODE><<<grid, threads, smem, st>>>(a);
    launch_end(st);
    return cudaGetLastError();
}

template <typename T, unsigned DIR, int MODE, int G>
cudaError_t launch_h_g(const Problem& P, SweepArgs a, const HMaps& maps, int br, int nbox, int threads,
                       cudaStream_t st) {
    a.ns = h_stages(P, MODE);
    const size_t smem = 128 + (size_t)a.ns * ModeT<MODE>::NTEN * br * nbox * 16 + 2 * 2 * G * 16 * sizeof(float) + 8 * 8;
    const int grid = std::min(P.N * P.C, device_sm_count());
    cudaFuncSetAttribute(k_hsweep<T, DIR, MODE, G>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    launch_begin(st);
    k_hsweep<T, DIR, MODE, G><<<grid, threads, smem, st>>>(a, maps, br, nbox);
    launch_end(st);
    return cudaGetLastError();
}

template <typename T, unsigned DIR, int MODE>
cudaError_t launch_h(const Problem& P, SweepArgs a, const HMaps& maps, cudaStream_t st) {
    int br, nbox, threads, G;
    h_geometry(P, &br, &nbox, &threads, &G);
    switch (G) {
    case 1: return launch_h_g<T, DIR, MODE, 1>(P, a, maps, br, nbox, threads, st);
    case 2: return launch_h_g<T, DIR, MODE, 2>(P, a, maps, br, nbox, threads, st);
    default: return cudaErrorNotSupported;
    }
}

template <typename T, unsigned DIR>
cudaError_t launch_dir(const Problem& P, SweepArgs a, int mode, const HMaps* maps, cudaStream_t st) {
    const bool vert = DIR == kTB || DIR == kBT;
    switch (mode) {
    case M_FIRST: return vert ? launch_v<T, DIR, M_FIRST>(P, a, st) : launch_h<T, DIR, M_FIRST>(P, a, *maps, st);
    case M_ONLY: return vert ? launch_v<T, DIR, M_ONLY>(P, a, st) : launch_h<T, DIR, M_ONLY>(P, a, *maps, st);
    case M_MID: return vert ? launch_v<T, DIR, M_MID>(P, a, st) : launch_h<T, DIR, M_MID>(P, a, *maps, st);
    default: return vert ? launch_v<T, DIR, M_LAST>(P, a, st) : launch_h<T, DIR, M_LAST>(P, a, *maps, st);
    }
}

template <typename T>
cudaError_t sweep_forward_t(const Problem& P, const void* x, const void* a, const void* lam, const void* u, void* y,
                            void* ws, cudaStream_t st) {
    WsCarver wc(ws);
    void* z = P.D > 1 ? wc.take<T>(P.U) : nullptr;
    void* acc = P.D > 1 ? wc.take<T>(P.U) : nullptr;
    SweepArgs args{x, lam, u, a, z, acc, y, P.N, P.C, P.H, P.W, P.Cw, 0, 2, (unsigned*)ws, kWaitLimitNs};
    int v = 0;
    for (unsigned d = kTB; d <= kRL; d <<= 1) {
        if (!(P.mask & d)) continue;
        const int mode = mode_of(v, P.D);
        args.slot = v;
        HMaps maps;
        if (!is_vertical(d)) {
            int br, nbox, thr, G;
            h_geometry(P, &br, &nbox, &thr, &G);
            const long long prow = (long long)P.N * P.C * P.H;
            const long long arow = (long long)P.D * P.N * P.Cw * 3 * P.H;
            const bool xl = mode == M_FIRST || mode == M_ONLY;
            bool ok = make_map(&maps.a, a, P.dtype, arow, P.W, br);
            ok = ok && make_map(&maps.src0, xl ? x : z, P.dtype, prow, P.W, br);
            ok = ok && make_map(&maps.src1, xl ? lam : x, P.dtype, prow, P.W, br);
            ok = ok && make_map(&maps.acc, acc ? acc : x, P.dtype, prow, P.W, br);
            ok = ok && make_map(&maps.u, u, P.dtype, prow, P.W, br);
            if (!ok) return cudaErrorInvalidValue;
        }
        cudaError_t e;
        switch (d) {
        case kTB: e = launch_dir<T, kTB>(P, args, mode, nullptr, st); break;
        case kBT: e = launch_dir<T, kBT>(P, args, mode, nullptr, st); break;
        case kLR: e = launch_dir<T, kLR>(P, args, mode, &maps, st); break;
        default: e = launch_dir<T, kRL>(P, args, mode, &maps, st); break;
        }
        if (e != cudaSuccess) return e;
        ++v;
    }
    return cudaSuccess;
}

}  // namespace

bool sweep_supports(const Problem& P, bool bwd) {
    if (bwd) return false;
    if ((P.W * P.esize()) % 16 != 0) return false;
    if (P.W > 4096 || P.H > 1024) return false;
    // TMA row coordinates are 32-bit
    if ((long long)P.D * P.N * P.Cw * 3 * P.H >= (1LL << 31) || (long long)P.N * P.C * P.H >= (1LL << 31)) return false;
    if (!encode_fn()) return false;
    for (int mode = 0; mode < 4; ++mode) {
        if ((P.mask & (kTB | kBT)) && v_stages(P, mode) < 2) return false;
        if ((P.mask & (kLR | kRL)) && h_stages(P, mode) < 2) return false;
    }
    return true;
}

size_t sweep_ws_bytes(const Problem& P, bool bwd) {
    if (bwd) return 0;
    size_t b = 256;
    if (P.D > 1) b += 2 * align256((size_t)P.U * P.esize());
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
