// k_proj.cu -- the channel projections of the compressive proxy ("GSPN-2: Efficient Parallel
// Sequence Modeling" paper notes, section "Optimisation 2: compact channel propagation"): per batch
// item n, Y[n] (Mo x HW) = P (Mo x K) . X[n] (K x HW), row-major, NCHW activations. This is the
// one dense contraction of the path.
//
// bf16 storage: a tcgen05 GEMM on the 5th-generation tensor cores. A CTA owns 128 pixels x BN
// output channels; the accumulator (fp32) lives in tensor memory. Operands come by TMA into a ring
// of 128-byte-swizzled shared-memory stages: A = the X tile, 64 k-rows x 128 pixels with pixels
// contiguous (an MN-major operand: two boxes of 64 pixels), B = the P tile, BN rows x 64 k with k
// contiguous (K-major). Warp 0 issues the TMA loads, warp 1 owns the tensor memory and issues the
// MMAs (one thread; each k-chunk is 4 MMAs of K = 16, committed to the stage's "empty" barrier so
// the producer can refill it), and all four warps read the accumulator back (tcgen05.ld) and write
// bf16 rows of Y. Every wait is bounded; a wait that runs out records GSPN_ERR_DEVICE_TIMEOUT in
// the status word and the kernel winds down normally (tensor memory is always freed).
//
// fp32 storage (and channel counts whose rows are not 16-byte multiples): an exact fp32 SIMT GEMM
// (64 x 64 output tiles, k staged through shared memory), since the tensor cores' fp32 formats
// would round the operands.
#include <cuda.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "gspn_common.cuh"
#include "gspn_internal.h"

namespace gspn {
namespace {

constexpr int kPM = 128;            // pixels per tile (MMA M)
constexpr int kPK = 64;             // k per stage (one 128-byte swizzle row of bf16)
constexpr unsigned long long kWaitNs = 1000000000ull;

__device__ __forceinline__ uint32_t s32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mb_init(uint64_t* b, unsigned n) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(s32(b)), "r"(n) : "memory");
}
__device__ __forceinline__ void mb_expect_tx(uint64_t* b, unsigned bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(s32(b)), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mb_try(uint64_t* b, unsigned parity) {
    unsigned ok;
    asm volatile("{ .reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p; }"
                 : "=r"(ok)
                 : "r"(s32(b)), "r"(parity)
                 : "memory");
    return ok != 0u;
}
// Bounded wait for the phase with this parity; false (and a recorded timeout) after kWaitNs.
__device__ __forceinline__ bool mb_wait(uint64_t* b, unsigned parity, unsigned* status) {
    if (mb_try(b, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (!mb_try(b, parity)) {
        if (globaltimer_ns() - t0 > kWaitNs) {
            report_timeout(status);
            return false;
        }
    }
    return true;
}

// TMA tile loads into this CTA's own shared memory, completion counted in bytes on the mbarrier.
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];" ::
            "r"(s32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(c2), "r"(s32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
                     "r"(s32(dst)), "l"(map), "r"(c0), "r"(c1), "r"(s32(bar))
                 : "memory");
}

// Shared-memory matrix descriptor (tcgen05): start address, leading / stride byte offsets (all >> 4),
// descriptor version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3fffu);
    d |= (uint64_t)((lbo >> 4) & 0x3fffu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3fffu) << 32;
    d |= (uint64_t)1 << 46;   // version
    d |= (uint64_t)2 << 61;   // SWIZZLE_128B
    return d;
}
// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, M = 128; a_mn / b_mn: the
// operand is MN-major (else K-major); n = N.
__device__ __forceinline__ uint32_t instr_desc(bool a_mn, bool b_mn, int n) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kPM >> 4) << 24);
}

struct ProjArgs {
    __nv_bfloat16* y;     // [batch][Mo][HW]
    unsigned* status;
    int Mo, K, HW;        // output rows, contraction length, pixels
    int tile_rows;        // output rows of one tile (multiple of 16, at most 256)
    int tiles_p, tiles_n, batch;
    int acc_cols;         // tensor-memory columns of one accumulator (power of two); two are allocated
    int stages;           // shared-memory operand stages (as many as fit beside the staging tiles)
    int ybufs;            // output staging tiles (1 or 2)
};

// Persistent: a CTA walks the tiles blockIdx.x, blockIdx.x + gridDim.x, ... Tiles are ordered with
// the pixel tile fastest and the row tile slowest, so the CTAs running at the same time write
// neighbouring 256-byte pieces of the same output rows (DRAM page locality for the 2.4 GB output of
// a C_proxy -> C projection). Warp 0 = TMA producer, warp 1 = tensor-memory owner and MMA issuer,
// warps 2..5 = epilogue. Two accumulators in tensor memory: the epilogue of one tile overlaps the
// MMAs of the next. A stage holds the X tile (two blocks of [64 k][64 px], 8 KB each, MN-major) and
// the P tile (tile_rows rows of 64 k, K-major). MMA M = 128 pixels, N = tile_rows (A = X, B = P):
// the accumulator's lanes are pixels. The epilogue converts the tile to bf16 into a shared-memory
// staging tile and one thread writes it out with a single TMA store (the output of a
// C_proxy -> C projection is 2.4 GB; per-thread 2-byte stores, and TMA stores of 16-row chunks
// behind a barrier and a proxy fence each, measured slower).
constexpr int kEpiWarps = 4;
constexpr int kProjThreads = 64 + 32 * kEpiWarps;

__device__ __forceinline__ void decode_tile(const ProjArgs& a, long long t, int& n, int& p0, int& r0) {
    const int tn = (int)(t % a.tiles_n);
    t /= a.tiles_n;
    const int tp = (int)(t % a.tiles_p);
    n = (int)(t / a.tiles_p);
    p0 = tp * kPM;
    r0 = tn * a.tile_rows;
}

__global__ void __launch_bounds__(kProjThreads, 1) k_proj_tc(const __grid_constant__ CUtensorMap mapA,
                                                              const __grid_constant__ CUtensorMap mapB,
                                                              const __grid_constant__ CUtensorMap mapY, ProjArgs a) {
    extern __shared__ unsigned char smem_raw[];
    // 1024-byte alignment: the swizzle pattern is anchored to address bits 7..9
    unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    constexpr int xB = kPM * kPK * 2;              // X tile bytes per stage (16 KB)
    const int stageB = xB + a.tile_rows * kPK * 2;
    const int nst = a.stages;
    uint64_t* full = (uint64_t*)(smem + nst * stageB);
    uint64_t* empty = full + nst;
    uint64_t* accf = empty + nst;       // accumulator b holds a finished tile
    uint64_t* acce = accf + 2;          // accumulator b has been read out
    uint32_t* tmem_slot = (uint32_t*)(acce + 2);
    // ybufs output staging tiles [tile_rows][128 pixels] of bf16
    __nv_bfloat16* ystage = (__nv_bfloat16*)((unsigned char*)full + 1024);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long total = (long long)a.tiles_p * a.tiles_n * a.batch;
    const int nk = (a.K + kPK - 1) / kPK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < nst; ++s) {
            mb_init(&full[s], 1);
            mb_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mb_init(&accf[b], 1);
            mb_init(&acce[b], kEpiWarps);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s32(tmem_slot)),
                     "r"(2 * a.acc_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    bool ok = true;   // false once a wait has run out: stop waiting, wind down

    if (warp == 0) {
        if (lane == 0) {
            // ---- TMA producer: two 64-pixel X blocks and the P rows per 64-wide k-chunk
            long long g = 0;
            for (long long t = blockIdx.x; t < total; t += gridDim.x) {
                int n, p0, r0;
                decode_tile(a, t, n, p0, r0);
                for (int kc = 0; kc < nk; ++kc, ++g) {
                    const int s = (int)(g % nst);
                    if (g >= nst && ok) ok = mb_wait(&empty[s], (unsigned)((g / nst) - 1) & 1u, a.status);
                    unsigned char* st = smem + s * stageB;
                    mb_expect_tx(&full[s], (unsigned)stageB);
                    tma_load_3d(st, &mapA, p0, kc * kPK, n, &full[s]);
                    tma_load_3d(st + 8192, &mapA, p0 + 64, kc * kPK, n, &full[s]);
                    tma_load_2d(st + xB, &mapB, kc * kPK, r0, &full[s]);
                }
            }
            // wind down: every load has landed before the CTA may exit (bounded)
            for (long long q = (g > nst ? g - nst : 0); q < g; ++q)
                mb_wait(&full[q % nst], (unsigned)(q / nst) & 1u, a.status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issuer: per k-chunk 4 MMAs of K = 16 into accumulator (tile & 1)
            const uint32_t idesc = instr_desc(true, false, a.tile_rows);
            long long g = 0;
            int it = 0;
            for (long long t = blockIdx.x; t < total; t += gridDim.x, ++it) {
                const int b = it & 1;
                if (it >= 2 && ok) ok = mb_wait(&acce[b], (unsigned)((it >> 1) - 1) & 1u, a.status);
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t dt = tmem + (uint32_t)(b * a.acc_cols);
                for (int kc = 0; kc < nk; ++kc, ++g) {
                    const int s = (int)(g % nst);
                    if (ok) ok = mb_wait(&full[s], (unsigned)(g / nst) & 1u, a.status);
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                    const uint32_t xbase = s32(smem + s * stageB);
                    const uint32_t pbase = xbase + xB;
                    // the last chunk may hold fewer than 64 valid k (TMA zero-fills the rest): no MMA
                    // for the 16-wide steps that lie wholly past K
                    const int kks = min(kPK / 16, (a.K - kc * kPK + 15) / 16);
#pragma unroll
                    for (int kk = 0; kk < kPK / 16; ++kk) {
                        if (kk >= kks) break;
                        // X: 16 k-rows = two 8-row atoms (1024 B each) further; 64-pixel blocks 8 KB apart
                        const uint64_t ad = smem_desc(xbase + kk * 2048, 8192, 1024);
                        // P: 16 k = 32 bytes further along each 128-byte row; 8-row groups 1024 B apart
                        const uint64_t bd = smem_desc(pbase + kk * 32, 16, 1024);
                        const uint32_t accum = (kc > 0 || kk > 0) ? 1u : 0u;
                        asm volatile(
                            "{ .reg .pred p; setp.ne.u32 p, %4, 0;\n"
                            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(dt),
                            "l"(ad), "l"(bd), "r"(idesc), "r"(accum)
                            : "memory");
                    }
                    // the stage is free once these MMAs have read it
                    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                     s32(&empty[s]))
                                 : "memory");
                }
                asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                                 s32(&accf[b]))
                             : "memory");
            }
        }
    } else {
        // ---- epilogue: warp w reads the accumulator lanes (pixels) of quadrant w % 4, 16 columns
        // (output rows) at a time, and converts them into its 32-pixel quarter of a staging tile
        // [tile_rows][128 pixels]; thread 64 then writes the tile out with one TMA store. With two
        // staging tiles the store of one tile overlaps the conversion of the next.
        const int q = warp & 3;
        const bool issuer = threadIdx.x == 64;
        int it = 0;
        for (long long t = blockIdx.x; t < total; t += gridDim.x, ++it) {
            const int b = it & 1;
            __nv_bfloat16* tile = ystage + (it % a.ybufs) * (a.tile_rows * kPM);
            if (ok) ok = mb_wait(&accf[b], (unsigned)(it >> 1) & 1u, a.status);
            __syncwarp();
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            int n, p0, r0;
            decode_tile(a, t, n, p0, r0);
            // the store issued from this staging tile ybufs tiles ago has finished reading it
            if (issuer) {
                if (a.ybufs == 2)
                    asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                else
                    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            }
            asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpiWarps) : "memory");
            __nv_bfloat16* col = tile + q * 32 + lane;
            for (int c0 = 0; c0 < a.tile_rows; c0 += 16) {
                uint32_t v[16];
                const uint32_t taddr = tmem + (uint32_t)(b * a.acc_cols) + ((uint32_t)(q * 32) << 16) + (uint32_t)c0;
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, "
                    "%13, %14, %15}, [%16];"
                    : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                      "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]),
                      "=r"(v[15])
                    : "r"(taddr));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                for (int j = 0; j < 16; ++j) col[(c0 + j) * kPM] = __float2bfloat16_rn(__uint_as_float(v[j]));
            }
            // the accumulator may be overwritten once every epilogue warp has read it
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(s32(&acce[b])) : "memory");
            // the staging writes (generic proxy) before the TMA store (async proxy) reads them
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            asm volatile("bar.sync 1, %0;" ::"n"(32 * kEpiWarps) : "memory");
            if (issuer) {
                asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                                 &mapY),
                             "r"(p0), "r"(r0), "r"(n), "r"(s32(tile))
                             : "memory");
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
            }
        }
        if (issuer) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");   // every store has completed
    }
    __syncwarp();   // the single-lane roles rejoin their warps before the block barrier
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * a.acc_cols)
                     : "memory");
    }
}

// ---- exact fp32 (SIMT) projection: 64 rows x 64 pixels per 256-thread block, 4 x 4 per thread,
// k staged through shared memory 16 at a time; fp32 accumulation for both storage dtypes.
template <typename T>
__global__ void __launch_bounds__(256) k_proj_simt(const T* __restrict__ P, const T* __restrict__ X, T* __restrict__ Y,
                                                   int Mo, int K, int HW) {
    __shared__ float Ps[16][64 + 4];
    __shared__ float Xs[16][64 + 4];
    const int n = blockIdx.z;
    const int m0 = blockIdx.y * 64, p0 = blockIdx.x * 64;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const T* Xn = X + (long long)n * K * HW;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 16) {
        for (int e = threadIdx.x; e < 16 * 64; e += 256) {
            const int kk = e / 64, c = e % 64;
            const int m = m0 + c, k = k0 + kk, p = p0 + c;
            Ps[kk][c] = (m < Mo && k < K) ? Io<T>::ld(P + (long long)m * K + k) : 0.f;
            Xs[kk][c] = (p < HW && k < K) ? Io<T>::ld(Xn + (long long)k * HW + p) : 0.f;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) {
            float pm[4], xp[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                pm[i] = Ps[kk][ty * 4 + i];
                xp[i] = Xs[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(pm[i], xp[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int m = m0 + ty * 4 + i;
        if (m >= Mo) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int p = p0 + tx * 4 + j;
            if (p < HW) Io<T>::st(Y + ((long long)n * Mo + m) * HW + p, acc[i][j]);
        }
    }
}

// ---- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    });
    return fn;
}

int pow2_at_least(int v) {
    int c = 32;
    while (c < v) c <<= 1;
    return c;
}

// Rows per tile: a multiple of 16 up to 256 that covers Mo in as few tiles as possible with the
// least padding.
int pick_bn(int Mo) {
    const int tiles = (Mo + 255) / 256;
    const int per = (Mo + tiles - 1) / tiles;
    return ((per + 15) / 16) * 16;
}

// Shared memory: alignment slack, the operand stages, 1 KB of barriers and the tensor-memory slot,
// then the staging tiles. Two staging tiles where three or more operand stages still fit beside
// them, else one; then as many stages as fit in the opt-in maximum, at most 8.
constexpr size_t kSmemMax = 232448;
struct TcPlan {
    int stages, ybufs;
    size_t smem;
};
TcPlan tc_plan(int rows) {
    const size_t stageB = (size_t)(kPM + rows) * kPK * 2, tileB = (size_t)rows * kPM * 2;
    const size_t room = kSmemMax - 2048;
    TcPlan p;
    p.ybufs = (room - 2 * tileB) / stageB >= 3 ? 2 : 1;
    p.stages = (int)std::min<size_t>(8, (room - p.ybufs * tileB) / stageB);
    p.smem = 2048 + p.stages * stageB + p.ybufs * tileB;
    return p;
}


}  // namespace

// The tensor-core path needs 16-byte rows for the TMA maps (K and HW multiples of 8) and 16-bit
// operands.
bool proj_uses_tc(int dtype, int Mo, int K, long long HW) {
    return dtype == GSPN_BF16 && K % 8 == 0 && HW % 8 == 0 && HW < (1LL << 31) && Mo >= 1 && encode_fn() != nullptr;
}

cudaError_t launch_projection(int dtype, int Mo, int K, long long HW, int batch, const void* P, const void* X, void* Y,
                              unsigned* status, cudaStream_t st) {
    if (!proj_uses_tc(dtype, Mo, K, HW)) {
        dim3 grid((unsigned)((HW + 63) / 64), (unsigned)((Mo + 63) / 64), (unsigned)batch);
        launch_begin(st);
        if (dtype == GSPN_F32)
            k_proj_simt<float><<<grid, 256, 0, st>>>((const float*)P, (const float*)X, (float*)Y, Mo, K, (int)HW);
        else
            k_proj_simt<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)P, (const __nv_bfloat16*)X,
                                                             (__nv_bfloat16*)Y, Mo, K, (int)HW);
        launch_end(st);
        return cudaGetLastError();
    }
    EncodeTiledFn enc = encode_fn();
    const int tile_rows = pick_bn(Mo);
    CUtensorMap mapA, mapB;
    {   // X as [batch][K][HW] bf16; box 64 pixels x 64 k x 1
        const cuuint64_t dims[3] = {(cuuint64_t)HW, (cuuint64_t)K, (cuuint64_t)batch};
        const cuuint64_t strides[2] = {(cuuint64_t)HW * 2, (cuuint64_t)K * HW * 2};
        const cuuint32_t box[3] = {64, (cuuint32_t)kPK, 1};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&mapA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(X), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    {   // P as [Mo][K] bf16; box 64 k x tile_rows rows
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)Mo};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kPK, (cuuint32_t)tile_rows};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&mapB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(P), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    CUtensorMap mapY;
    {   // Y as [batch][Mo][HW] bf16; box 128 pixels x tile_rows x 1 (stores clip at the edges)
        const cuuint64_t dims[3] = {(cuuint64_t)HW, (cuuint64_t)Mo, (cuuint64_t)batch};
        const cuuint64_t strides[2] = {(cuuint64_t)HW * 2, (cuuint64_t)Mo * HW * 2};
        const cuuint32_t box[3] = {(cuuint32_t)kPM, (cuuint32_t)tile_rows, 1};
        const cuuint32_t es[3] = {1, 1, 1};
        if (enc(&mapY, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, Y, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    ProjArgs a;
    a.y = (__nv_bfloat16*)Y;
    a.status = status;
    a.Mo = Mo;
    a.K = K;
    a.HW = (int)HW;
    a.tile_rows = tile_rows;
    a.tiles_p = (int)((HW + kPM - 1) / kPM);
    a.tiles_n = (Mo + tile_rows - 1) / tile_rows;
    a.batch = batch;
    a.acc_cols = pow2_at_least(tile_rows);
    const TcPlan plan = tc_plan(tile_rows);
    a.stages = plan.stages;
    a.ybufs = plan.ybufs;
    const size_t smem = plan.smem;
    auto kern = k_proj_tc;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long tiles = (long long)a.tiles_p * a.tiles_n * batch;
    const int grid = (int)std::min<long long>(tiles, device_sm_count());
    launch_begin(st);
    kern<<<grid, kProjThreads, smem, st>>>(mapA, mapB, mapY, a);
    launch_end(st);
    return cudaGetLastError();
}

}  // namespace gspn
