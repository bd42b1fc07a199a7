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

#include <mutex>

#include "gspn_common.cuh"
#include "gspn_internal.h"

namespace gspn {
namespace {

constexpr int kPM = 128;            // pixels per tile (MMA M)
constexpr int kPK = 64;             // k per stage (one 128-byte swizzle row of bf16)
constexpr int kStages = 3;
constexpr int kATileB = kPK * kPM * 2;   // 16 KB: two [64 k][64 px] swizzled halves
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

// TMA tile loads (no multicast), completion counted in bytes on the mbarrier.
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
// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, A MN-major, B K-major, M = 128.
__device__ __forceinline__ uint32_t instr_desc(int bn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | ((uint32_t)(bn >> 3) << 17) | ((uint32_t)(kPM >> 4) << 24);
}

struct ProjArgs {
    __nv_bfloat16* y;     // [N][Mo][HW]
    unsigned* status;
    int Mo, K, HW, bn;    // output rows, contraction length, pixels, output rows per tile (multiple of 16)
    int tiles_p, tiles_n; // pixel tiles, row tiles
    int tmem_cols;        // power of two >= bn
};

__global__ void __launch_bounds__(128, 1) k_proj_tc(const __grid_constant__ CUtensorMap mapA,
                                                     const __grid_constant__ CUtensorMap mapB, ProjArgs a) {
    extern __shared__ unsigned char smem_raw[];
    // 1024-byte alignment: the swizzle pattern is anchored to address bits 7..9
    unsigned char* smem = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    const int btile = a.bn * kPK * 2;
    const int stageB = kATileB + btile;
    uint64_t* full = (uint64_t*)(smem + kStages * stageB);
    uint64_t* empty = full + kStages;
    uint64_t* done = empty + kStages;
    uint32_t* tmem_slot = (uint32_t*)(done + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int t = blockIdx.x;
    const int tp = t % a.tiles_p;
    t /= a.tiles_p;
    const int tn = t % a.tiles_n;
    const int n = t / a.tiles_n;
    const int p0 = tp * kPM, r0 = tn * a.bn;
    const int nk = (a.K + kPK - 1) / kPK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mb_init(&full[s], 1);
            mb_init(&empty[s], 1);
        }
        mb_init(done, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s32(tmem_slot)),
                     "r"(a.tmem_cols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;
    bool ok = true;

    if (warp == 0 && lane == 0) {
        // ---- TMA producer
        for (int kc = 0; kc < nk; ++kc) {
            const int s = kc % kStages;
            if (kc >= kStages && ok) ok = mb_wait(&empty[s], (unsigned)((kc / kStages) - 1) & 1u, a.status);
            unsigned char* st = smem + s * stageB;
            mb_expect_tx(&full[s], (unsigned)stageB);
            tma_load_3d(st, &mapA, p0, kc * kPK, n, &full[s]);
            tma_load_3d(st + kATileB / 2, &mapA, p0 + 64, kc * kPK, n, &full[s]);
            tma_load_2d(st + kATileB, &mapB, kc * kPK, r0, &full[s]);
        }
        // wind down: every load has landed before the CTA may exit (bounded)
        for (int kc = (nk > kStages ? nk - kStages : 0); kc < nk; ++kc) {
            const int s = kc % kStages;
            mb_wait(&full[s], (unsigned)(kc / kStages) & 1u, a.status);
        }
    } else if (warp == 1 && lane == 0) {
        // ---- MMA issuer: 4 MMAs of K = 16 per stage
        const uint32_t idesc = instr_desc(a.bn);
        for (int kc = 0; kc < nk; ++kc) {
            const int s = kc % kStages;
            if (ok) ok = mb_wait(&full[s], (unsigned)(kc / kStages) & 1u, a.status);
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const uint32_t abase = s32(smem + s * stageB);
            const uint32_t bbase = abase + kATileB;
#pragma unroll
            for (int kk = 0; kk < kPK / 16; ++kk) {
                // A: 16 k-rows = two 8-row atoms (1024 B each) further; halves of 64 px 8 KB apart
                const uint64_t ad = smem_desc(abase + kk * 2048, kATileB / 2, 1024);
                // B: 16 k = 32 bytes further along each 128-byte row; 8-row groups 1024 B apart
                const uint64_t bd = smem_desc(bbase + kk * 32, 16, 1024);
                const uint32_t accum = (kc > 0 || kk > 0) ? 1u : 0u;
                asm volatile(
                    "{ .reg .pred p; setp.ne.u32 p, %4, 0;\n"
                    "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p; }" ::"r"(tmem),
                    "l"(ad), "l"(bd), "r"(idesc), "r"(accum)
                    : "memory");
            }
            // the stage is free once these MMAs have read it
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                             s32(&empty[s]))
                         : "memory");
        }
        asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(s32(done))
                     : "memory");
    }
    __syncwarp();

    // ---- epilogue: warp w reads accumulator lanes 32w..32w+31 (pixels), 16 columns at a time
    mb_wait(done, 0u, a.status);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const int px = p0 + warp * 32 + lane;
    __nv_bfloat16* yrow = a.y + ((long long)n * a.Mo + r0) * a.HW + px;
    for (int c0 = 0; c0 < a.bn; c0 += 16) {
        uint32_t v[16];
        const uint32_t taddr = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0;
        asm volatile(
            "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
            "%15}, [%16];"
            : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
              "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
            : "r"(taddr));
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        if (px < a.HW) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int r = r0 + c0 + j;
                if (r < a.Mo) yrow[(long long)(c0 + j) * a.HW] = __float2bfloat16_rn(__uint_as_float(v[j]));
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 1) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(a.tmem_cols) : "memory");
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

size_t tc_smem(int bn) { return 1024 + (size_t)kStages * (kATileB + (size_t)bn * kPK * 2) + 8 * (2 * kStages + 1) + 16; }

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
    const int bn = pick_bn(Mo);
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
    {   // P as [Mo][K] bf16; box 64 k x bn rows
        const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)Mo};
        const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
        const cuuint32_t box[2] = {(cuuint32_t)kPK, (cuuint32_t)bn};
        const cuuint32_t es[2] = {1, 1};
        if (enc(&mapB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(P), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    ProjArgs a;
    a.y = (__nv_bfloat16*)Y;
    a.status = status;
    a.Mo = Mo;
    a.K = K;
    a.HW = (int)HW;
    a.bn = bn;
    a.tiles_p = (int)((HW + kPM - 1) / kPM);
    a.tiles_n = (Mo + bn - 1) / bn;
    a.tmem_cols = pow2_at_least(bn);
    const size_t smem = tc_smem(bn);
    cudaError_t e = cudaFuncSetAttribute(k_proj_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long blocks = (long long)a.tiles_p * a.tiles_n * batch;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
    launch_begin(st);
    k_proj_tc<<<(unsigned)blocks, 128, smem, st>>>(mapA, mapB, a);
    launch_end(st);
    return cudaGetLastError();
}

}  // namespace gspn
