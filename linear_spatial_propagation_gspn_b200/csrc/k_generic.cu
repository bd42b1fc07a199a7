// k_generic.cu -- the any-shape kernel family of libgspn.
//
// One CTA per (plane, direction) runs the whole sequential scan of that direction
// ("GSPN-2: Efficient Parallel Sequence Modeling" paper notes, section "Optimisation 1:
// single-kernel fusion": all steps of a scan inside one kernel, looping over lines). The
// previous hidden line lives in shared memory (double-buffered, one barrier per step) and
// lanes are strided over the CTA's threads. Directions run one after another so the
// partial sum over directions can be kept in an fp32 workspace without races. This family
// exists for coverage (any N, C, H, W, odd sizes, any direction mask); the plane and sweep
// families are the fast paths.
#include <algorithm>

#include "gspn_common.cuh"
#include "gspn_internal.h"

namespace gspn {
namespace {

constexpr int kGenFwdMaxLanes = 28 * 1024;  // 2 fp32 lines in 224 KB of shared memory
constexpr int kGenBwdMaxLanes = 7 * 1024;   // 8 fp32 lines

struct GenArgs {
    const void* x;
    const void* a;
    const void* lam;
    const void* u;
    void* y;            // forward output (storage dtype)
    float* acc;         // fp32 partial sum over directions (N*C*H*W), may be null if D == 1
    float* hstore;      // backward recompute: h of this direction in image coordinates
    int N, C, H, W, Cw, D;
    unsigned dir;
    int slot;
    int first, last;    // first / last direction of the mask
    int chunk;          // lines per local chunk (0: global)
    int per_dir;        // lam and u carry a direction axis: this direction's are at slot * U
};

// The scans are latency-bound: every step's loads depend on nothing but the step index, so each
// thread asks L2 for its lanes' elements kPrefetch steps ahead (one prefetch per array; the lanes
// of a warp share one request per line). Only vertical scans do this: their lines are rows, so a
// warp's prefetches cover whole lines (horizontal scans here only occur on the per-direction path,
// whose columns would cost a request per lane).
constexpr int kPrefetch = 8;
__device__ __forceinline__ void pf_l2(const void* p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// Forward scan of one direction for plane blockIdx.x. Writes y (last direction), the fp32
// partial sum (other directions) and, when hstore is set, this direction's h.
template <typename T, unsigned DIR>
__global__ void k_gen_fwd(GenArgs p) {
    extern __shared__ float sh[];
    const int plane = blockIdx.x;
    const int n = plane / p.C, c = plane % p.C;
    const long long HW = (long long)p.H * p.W;
    const int L = is_vertical(DIR) ? p.H : p.W;
    const int M = is_vertical(DIR) ? p.W : p.H;
    const long long lu = p.per_dir ? (long long)p.slot * p.N * p.C * HW : 0;   // this direction's lam / u
    const T* x = (const T*)p.x + plane * HW;
    const T* lam = (const T*)p.lam + lu + plane * HW;
    const T* u = (const T*)p.u + lu + plane * HW;
    T* y = (T*)p.y + plane * HW;
    const T* a3 = (const T*)p.a + (((long long)p.slot * p.N + n) * p.Cw + (p.Cw == 1 ? 0 : c)) * 3 * HW;
    float* acc = p.acc ? p.acc + plane * HW : nullptr;
    float* hst = p.hstore ? p.hstore + plane * HW : nullptr;
    float* hp = sh;
    float* hc = sh + M;
    const bool pf = is_vertical(DIR);
    for (int i = 0; i < L; ++i) {
        for (int j = threadIdx.x; j < M; j += blockDim.x) {
            const long long q = scan_pixel(DIR, p.H, p.W, i, j);
            if (pf && i + kPrefetch < L) {
                const long long f = scan_pixel(DIR, p.H, p.W, i + kPrefetch, j);
                pf_l2(x + f);
                pf_l2(lam + f);
                pf_l2(a3 + f);
                pf_l2(a3 + HW + f);
                pf_l2(a3 + 2 * HW + f);
                if (acc && !p.first) pf_l2(acc + f);
                if (p.per_dir || (p.last && !hst)) pf_l2(u + f);
            }
            float h = Io<T>::ld(lam + q) * Io<T>::ld(x + q);
            if (!chunk_start(scan_ascending(DIR), L, p.chunk, i)) {
                const Wts w = lane_weights_fast(Io<T>::ld(a3 + q), Io<T>::ld(a3 + HW + q),
                                                Io<T>::ld(a3 + 2 * HW + q), j > 0, j < M - 1);
                if (j > 0) h = fmaf(w.w0, hp[j - 1], h);
                h = fmaf(w.w1, hp[j], h);
                if (j < M - 1) h = fmaf(w.w2, hp[j + 1], h);
            }
            hc[j] = h;
            if (hst) hst[q] = h;
            // shared u gates the sum once at the end; a per-direction u weights each term
            const float hv = p.per_dir ? Io<T>::ld(u + q) * h : h;
            if (p.first && p.last) {
                if (y != nullptr && !hst) Io<T>::st(y + q, p.per_dir ? hv : Io<T>::ld(u + q) * h);
                if (acc) acc[q] = hv;
            } else if (p.first) {
                acc[q] = hv;
            } else if (p.last && !hst) {
                Io<T>::st(y + q, p.per_dir ? acc[q] + hv : Io<T>::ld(u + q) * (acc[q] + h));
            } else {
                acc[q] += hv;
            }
        }
        __syncthreads();
        float* t = hp;
        hp = hc;
        hc = t;
    }
}

// Channel-shared logit gradients are sums over channels accumulated with atomics from many CTAs.
// They are summed as 64-bit fixed-point integers (2^32 units): integer addition does not depend on
// the order, so the result is the same on every run. A term is an fp32 value scaled by a power of
// two (exact) and rounded to 2^-32; it is clamped to |v| <= 2^19 so that 2048 terms cannot overflow.
constexpr float kFixScale = 4294967296.f;   // 2^32
__device__ __forceinline__ unsigned long long to_fixed(float v) {
    v = fminf(fmaxf(v, -524288.f), 524288.f);
    return (unsigned long long)__float2ll_rn(v * kFixScale);
}
__device__ __forceinline__ float from_fixed(unsigned long long q) { return (float)(long long)q * (1.f / kFixScale); }

struct GenBwdArgs {
    const void* a;
    const void* u;
    const void* dy;
    void* da;            // per-channel mode: written directly (storage dtype)
    unsigned long long* dacc;   // shared mode: fixed-point sum over channels (zeroed before)
    float* dz;           // fp32, N*C*H*W
    const float* hstore; // h of this direction, image coordinates, fp32
    int N, C, H, W, Cw;
    unsigned dir;
    int slot;
    int first;
    int chunk;           // lines per local chunk (0: global)
    int per_dir;         // lam and u carry a direction axis (then dlam, du are written here)
    const void* x;       // per_dir: x, this direction's lam, dlam_d and du_d outputs
    const void* lam;
    void* dlam;
    void* du;
};

// Reverse scan of one direction for plane blockIdx.x:
//   delta_i = u dy + w_{i+1}^T delta_{i+1};  dz (+)= delta;  da from dw_i[j][k] = delta_i[j] h_{i-1}[j+k-1].
template <typename T, unsigned DIR>
__global__ void k_gen_bwd(GenBwdArgs p) {
    extern __shared__ float sh[];
    const int plane = blockIdx.x;
    const int n = plane / p.C, c = plane % p.C;
    const long long HW = (long long)p.H * p.W;
    const int L = is_vertical(DIR) ? p.H : p.W;
    const int M = is_vertical(DIR) ? p.W : p.H;
    const long long lu = p.per_dir ? (long long)p.slot * p.N * p.C * HW : 0;   // this direction's lam / u
    const T* u = (const T*)p.u + lu + plane * HW;
    const T* dy = (const T*)p.dy + plane * HW;
    const long long abase = (((long long)p.slot * p.N + n) * p.Cw + (p.Cw == 1 ? 0 : c)) * 3 * HW;
    const T* a3 = (const T*)p.a + abase;
    T* da3 = p.da ? (T*)p.da + abase : nullptr;
    unsigned long long* dacc3 = p.dacc ? p.dacc + (((long long)p.slot * p.N + n) * 3) * HW : nullptr;
    float* dz = p.dz + plane * HW;
    const float* hs = p.hstore + plane * HW;
    // [delta prev | delta cur | w(prev buffer) x3 | w(cur buffer) x3]
    float* dprev = sh;
    float* dcur = sh + M;
    float* wprev = sh + 2 * M;
    float* wcur = sh + 5 * M;
    const bool pf = is_vertical(DIR);
    for (int i = L - 1; i >= 0; --i) {
        for (int j = threadIdx.x; j < M; j += blockDim.x) {
            const long long q = scan_pixel(DIR, p.H, p.W, i, j);
            if (pf && i - kPrefetch >= 1) {
                const long long f = scan_pixel(DIR, p.H, p.W, i - kPrefetch, j);
                pf_l2(u + f);
                pf_l2(dy + f);
                pf_l2(a3 + f);
                pf_l2(a3 + HW + f);
                pf_l2(a3 + 2 * HW + f);
                pf_l2(hs + scan_pixel(DIR, p.H, p.W, i - kPrefetch - 1, j));
                if (!p.first) pf_l2(dz + f);
                if (dacc3) {
                    pf_l2(dacc3 + f);
                    pf_l2(dacc3 + HW + f);
                    pf_l2(dacc3 + 2 * HW + f);
                }
                if (p.per_dir) {
                    const long long pq = lu + plane * HW + f;
                    pf_l2((const T*)p.lam + pq);
                    pf_l2((const T*)p.x + plane * HW + f);
                }
            }
            float del = Io<T>::ld(u + q) * Io<T>::ld(dy + q);
            // no delta flows back through the first line of a chunk (it does not see h_{i-1})
            if (i < L - 1 && !chunk_start(scan_ascending(DIR), L, p.chunk, i + 1)) {
                // (w_{i+1}^T delta_{i+1})[j] = w[j-1][2] d[j-1] + w[j][1] d[j] + w[j+1][0] d[j+1]
                if (j > 0) del = fmaf(wprev[2 * M + j - 1], dprev[j - 1], del);
                del = fmaf(wprev[M + j], dprev[j], del);
                if (j < M - 1) del = fmaf(wprev[j + 1], dprev[j + 1], del);
            }
            dcur[j] = del;
            if (p.per_dir) {
                // dlam_d = x delta^d, du_d = dy h^d; dz accumulates dx = sum_d lam_d delta^d
                const long long pq = lu + plane * HW + q;
                const float lamv = Io<T>::ld((const T*)p.lam + pq);
                Io<T>::st((T*)p.dlam + pq, Io<T>::ld((const T*)p.x + plane * HW + q) * del);
                Io<T>::st((T*)p.du + pq, Io<T>::ld(dy + q) * hs[q]);
                if (p.first) dz[q] = lamv * del;
                else dz[q] += lamv * del;
            } else {
                if (p.first) dz[q] = del;
                else dz[q] += del;
            }
            if (!chunk_start(scan_ascending(DIR), L, p.chunk, i)) {
                const bool hl = j > 0, hr = j < M - 1;
                const LaneJac J = lane_jacobian_fast(Io<T>::ld(a3 + q), Io<T>::ld(a3 + HW + q),
                                                     Io<T>::ld(a3 + 2 * HW + q), hl, hr);
                const float h0 = hl ? hs[scan_pixel(DIR, p.H, p.W, i - 1, j - 1)] : 0.f;
                const float h1 = hs[scan_pixel(DIR, p.H, p.W, i - 1, j)];
                const float h2 = hr ? hs[scan_pixel(DIR, p.H, p.W, i - 1, j + 1)] : 0.f;
                const float dw0 = del * h0, dw1 = del * h1, dw2 = del * h2;
                const float s = J.w0 * dw0 + J.w1 * dw1 + J.w2 * dw2;
                const float g0 = J.g0 * (dw0 - s), g1 = J.g1 * (dw1 - s), g2 = J.g2 * (dw2 - s);
                if (da3) {
                    Io<T>::st(da3 + q, g0);
                    Io<T>::st(da3 + HW + q, g1);
                    Io<T>::st(da3 + 2 * HW + q, g2);
                } else {
                    atomicAdd(dacc3 + q, to_fixed(g0));
                    atomicAdd(dacc3 + HW + q, to_fixed(g1));
                    atomicAdd(dacc3 + 2 * HW + q, to_fixed(g2));
                }
                wcur[j] = J.w0;
                wcur[M + j] = J.w1;
                wcur[2 * M + j] = J.w2;
            } else if (da3) {
                Io<T>::st(da3 + q, 0.f);
                Io<T>::st(da3 + HW + q, 0.f);
                Io<T>::st(da3 + 2 * HW + q, 0.f);
            }
        }
        __syncthreads();
        float* t = dprev; dprev = dcur; dcur = t;
        t = wprev; wprev = wcur; wcur = t;
    }
}

// dx = lam dz, dlam = x dz, du = dy acc.
template <typename T>
__global__ void k_gen_bwd_final(const T* x, const T* lam, const T* dy, const float* dz, const float* acc, T* dx,
                                T* dlam, T* du, long long U) {
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < U; e += (long long)gridDim.x * blockDim.x) {
        const float g = dz[e];
        Io<T>::st(dx + e, Io<T>::ld(lam + e) * g);
        Io<T>::st(dlam + e, Io<T>::ld(x + e) * g);
        Io<T>::st(du + e, Io<T>::ld(dy + e) * acc[e]);
    }
}

template <typename T>
__global__ void k_f32_to(const float* src, T* dst, long long n) {
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x)
        Io<T>::st(dst + e, src[e]);
}

template <typename T>
__global__ void k_fixed_to(const unsigned long long* src, T* dst, long long n) {
    for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x)
        Io<T>::st(dst + e, from_fixed(src[e]));
}

// Batched transpose dst[b][c][r] (+)= src[b][r][c] for b < B (R x Cc planes), through 32 x 32
// shared-memory tiles (coalesced both ways). Src: storage type, fp32 or 64-bit fixed point.
template <typename S> __device__ __forceinline__ float ld_any(const S* p) { return Io<S>::ld(p); }
template <> __device__ __forceinline__ float ld_any<unsigned long long>(const unsigned long long* p) {
    return from_fixed(*p);
}
template <typename S, typename D, bool ADD>
__global__ void k_transpose(const S* __restrict__ src, D* __restrict__ dst, int R, int Cc) {
    __shared__ float tile[32][33];
    const long long b = blockIdx.z;
    const int r0 = blockIdx.y * 32, c0 = blockIdx.x * 32;
    const S* sp = src + b * (long long)R * Cc;
    D* dp = dst + b * (long long)R * Cc;
    for (int k = threadIdx.y; k < 32; k += 8) {
        const int r = r0 + k, c = c0 + threadIdx.x;
        if (r < R && c < Cc) tile[k][threadIdx.x] = ld_any(sp + (long long)r * Cc + c);
    }
    __syncthreads();
    for (int k = threadIdx.y; k < 32; k += 8) {
        const int c = c0 + k, r = r0 + threadIdx.x;
        if (r < R && c < Cc) {
            D* q = dp + (long long)c * R + r;
            const float v = tile[threadIdx.x][k];
            Io<D>::st(q, ADD ? Io<D>::ld(q) + v : v);
        }
    }
}
template <typename S, typename D, bool ADD>
cudaError_t launch_transpose(const S* src, D* dst, long long B, int R, int Cc, cudaStream_t st) {
    const long long plane = (long long)R * Cc;
    for (long long b0 = 0; b0 < B; b0 += 65535) {   // grid z is limited to 65535
        const long long nb = std::min<long long>(65535, B - b0);
        dim3 grid((unsigned)((Cc + 31) / 32), (unsigned)((R + 31) / 32), (unsigned)nb);
        k_transpose<S, D, ADD><<<grid, dim3(32, 8), 0, st>>>(src + b0 * plane, dst + b0 * plane, R, Cc);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

int gen_threads(int M) { return std::min(1024, std::max(32, ((M + 31) / 32) * 32)); }

// One launch of the forward / reverse scan of direction d (the direction is a template argument,
// so the pixel indexing folds to a row base plus the lane).
template <typename T, unsigned D>
cudaError_t gen_fwd_launch_d(const GenArgs& g, int M, cudaStream_t st) {
    const size_t smem = 2 * (size_t)M * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(k_gen_fwd<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    launch_begin(st);
    k_gen_fwd<T, D><<<g.N * g.C, gen_threads(M), smem, st>>>(g);
    launch_end(st);
    return cudaGetLastError();
}
template <typename T>
cudaError_t gen_fwd_launch(const GenArgs& g, int M, cudaStream_t st) {
    switch (g.dir) {
    case kTB: return gen_fwd_launch_d<T, kTB>(g, M, st);
    case kBT: return gen_fwd_launch_d<T, kBT>(g, M, st);
    case kLR: return gen_fwd_launch_d<T, kLR>(g, M, st);
    default: return gen_fwd_launch_d<T, kRL>(g, M, st);
    }
}
template <typename T, unsigned D>
cudaError_t gen_bwd_launch_d(const GenBwdArgs& b, int M, cudaStream_t st) {
    const size_t smem = 8 * (size_t)M * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(k_gen_bwd<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    launch_begin(st);
    k_gen_bwd<T, D><<<b.N * b.C, gen_threads(M), smem, st>>>(b);
    launch_end(st);
    return cudaGetLastError();
}
template <typename T>
cudaError_t gen_bwd_launch(const GenBwdArgs& b, int M, cudaStream_t st) {
    switch (b.dir) {
    case kTB: return gen_bwd_launch_d<T, kTB>(b, M, st);
    case kBT: return gen_bwd_launch_d<T, kBT>(b, M, st);
    case kLR: return gen_bwd_launch_d<T, kLR>(b, M, st);
    default: return gen_bwd_launch_d<T, kRL>(b, M, st);
    }
}

template <typename T>
cudaError_t gen_forward_t(const Problem& P, const void* x, const void* a, const void* lam, const void* u, void* y,
                          void* ws, cudaStream_t st) {
    WsCarver wc(ws);
    float* acc = P.D > 1 ? wc.take<float>(P.U) : nullptr;
    int slot = 0, seen = 0;
    for (unsigned d = kTB; d <= kRL; d <<= 1) {
        if (!(P.mask & d)) continue;
        GenArgs g{x, a, lam, u, y, acc, nullptr, P.N, P.C, P.H, P.W, P.Cw, P.D, d, slot, seen == 0, seen == P.D - 1,
                  P.chunk, P.per_dir};
        const cudaError_t e = gen_fwd_launch<T>(g, is_vertical(d) ? P.W : P.H, st);
        if (e != cudaSuccess) return e;
        ++slot;
        ++seen;
    }
    return cudaSuccess;
}

// Direction-serial backward with the per-direction lam / u of the learnable merge: every direction
// on the image-layout buffers (horizontal directions walk columns).
template <typename T>
cudaError_t gen_backward_perdir(const Problem& P, const void* x, const void* a, const void* lam, const void* u,
                                const void* dy, void* dx, void* da, void* dlam, void* du, void* ws, cudaStream_t st) {
    WsCarver wc(ws);
    float* acc = wc.take<float>(P.U);
    float* dz = wc.take<float>(P.U);
    float* hstore = wc.take<float>(P.U);
    unsigned long long* dacc = P.wmode == GSPN_W_SHARED ? wc.take<unsigned long long>(P.A) : nullptr;
    cudaError_t e;
    if (dacc && (e = cudaMemsetAsync(dacc, 0, P.A * sizeof(unsigned long long), st)) != cudaSuccess) return e;
    int slot = 0;
    for (unsigned d = kTB; d <= kRL; d <<= 1) {
        if (!(P.mask & d)) continue;
        const int M = is_vertical(d) ? P.W : P.H;
        GenArgs g{x, a, lam, u, nullptr, acc, hstore, P.N, P.C, P.H, P.W, P.Cw, P.D, d, slot, slot == 0, false,
                  P.chunk, P.per_dir};
        if ((e = gen_fwd_launch<T>(g, M, st)) != cudaSuccess) return e;
        GenBwdArgs b{a, u, dy, dacc ? nullptr : da, dacc, dz, hstore, P.N, P.C, P.H, P.W, P.Cw, d, slot, slot == 0,
                     P.chunk, P.per_dir, x, lam, dlam, du};
        if ((e = gen_bwd_launch<T>(b, M, st)) != cudaSuccess) return e;
        ++slot;
    }
    const int blocks = (int)std::max<long long>(1, std::min<long long>(4096, (P.U + 255) / 256));
    k_f32_to<T><<<blocks, 256, 0, st>>>(dz, (T*)dx, P.U);   // dlam_d, du_d written per direction
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (dacc) {
        const int ab = (int)std::max<long long>(1, std::min<long long>(4096, (P.A + 255) / 256));
        k_fixed_to<T><<<ab, 256, 0, st>>>(dacc, (T*)da, P.A);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// Recompute + reverse scan of one direction, which runs as a vertical scan (TB or BT) of the
// problem with H x W lanes given: the image itself for the vertical directions, its transpose for
// the horizontal ones.
template <typename T>
cudaError_t gen_direction_bwd(const Problem& P, int H, int W, unsigned vdir, int slot, bool first, const void* x,
                              const void* a, const void* lam, const void* u, const void* dy, void* da,
                              unsigned long long* dacc, float* acc, float* dz, float* hstore, cudaStream_t st) {
    const int M = W;
    GenArgs g{x, a, lam, u, nullptr, acc, hstore, P.N, P.C, H, W, P.Cw, P.D, vdir, slot, first, false, P.chunk, 0};
    cudaError_t e = gen_fwd_launch<T>(g, M, st);
    if (e != cudaSuccess) return e;
    GenBwdArgs b{a, u, dy, dacc ? nullptr : da, dacc, dz, hstore, P.N, P.C, H, W, P.Cw, vdir, slot, first,
                 P.chunk, 0, x, lam, nullptr, nullptr};
    return gen_bwd_launch<T>(b, M, st);
}

int n_vert(const Problem& P) { return ((P.mask & kTB) ? 1 : 0) + ((P.mask & kBT) ? 1 : 0); }
int n_horz(const Problem& P) { return P.D - n_vert(P); }

// Backward with lam and u shared by the directions. The vertical directions scan the image-layout
// buffers; the horizontal ones scan transposed copies of x, lam, u, dy and of their logit slots
// (left->right is then top->bottom of the transpose, right->left bottom->top), so every scan reads
// and writes whole rows. Their sums over directions and their logit gradients are transposed back.
template <typename T>
cudaError_t gen_backward_t(const Problem& P, const void* x, const void* a, const void* lam, const void* u,
                           const void* dy, void* dx, void* da, void* dlam, void* du, void* ws, cudaStream_t st) {
    if (P.per_dir) return gen_backward_perdir<T>(P, x, a, lam, u, dy, dx, da, dlam, du, ws, st);
    const bool shared = P.wmode == GSPN_W_SHARED;
    const int nV = n_vert(P), nH = n_horz(P);
    const long long slotA = (long long)P.N * P.Cw * 3 * P.HW;   // logits of one direction slot
    const long long slotD = (long long)P.N * 3 * P.HW;          // shared-mode gradient of one slot
    WsCarver wc(ws);
    float* acc = wc.take<float>(P.U);
    float* dz = wc.take<float>(P.U);
    float* hstore = wc.take<float>(P.U);
    unsigned long long* dacc = shared ? wc.take<unsigned long long>((size_t)P.D * slotD) : nullptr;
    float *accT = nullptr, *dzT = nullptr;
    T *xT = nullptr, *lamT = nullptr, *uT = nullptr, *dyT = nullptr, *aT = nullptr, *daT = nullptr;
    if (nH > 0) {
        accT = wc.take<float>(P.U);
        dzT = wc.take<float>(P.U);
        xT = wc.take<T>(P.U);
        lamT = wc.take<T>(P.U);
        uT = wc.take<T>(P.U);
        dyT = wc.take<T>(P.U);
        aT = wc.take<T>((size_t)nH * slotA);
        if (!shared) daT = wc.take<T>((size_t)nH * slotA);
    }
    cudaError_t e;
    if (dacc && (e = cudaMemsetAsync(dacc, 0, (size_t)P.D * slotD * sizeof(unsigned long long), st)) != cudaSuccess)
        return e;
    const long long planes = (long long)P.N * P.C;
    if (nH > 0) {
        if ((e = launch_transpose<T, T, false>((const T*)x, xT, planes, P.H, P.W, st)) != cudaSuccess) return e;
        if ((e = launch_transpose<T, T, false>((const T*)lam, lamT, planes, P.H, P.W, st)) != cudaSuccess) return e;
        if ((e = launch_transpose<T, T, false>((const T*)u, uT, planes, P.H, P.W, st)) != cudaSuccess) return e;
        if ((e = launch_transpose<T, T, false>((const T*)dy, dyT, planes, P.H, P.W, st)) != cudaSuccess) return e;
        // the horizontal slots follow the vertical ones: one batch of nH * N * Cw * 3 planes
        if ((e = launch_transpose<T, T, false>((const T*)a + nV * slotA, aT, (long long)nH * P.N * P.Cw * 3, P.H,
                                               P.W, st)) != cudaSuccess)
            return e;
    }
    int v = 0, h = 0;
    for (unsigned d = kTB; d <= kRL; d <<= 1) {
        if (!(P.mask & d)) continue;
        if (is_vertical(d)) {
            e = gen_direction_bwd<T>(P, P.H, P.W, d, v, v == 0, x, a, lam, u, dy, da, dacc, acc, dz, hstore, st);
            ++v;
        } else {
            e = gen_direction_bwd<T>(P, P.W, P.H, d == kLR ? kTB : kBT, h, h == 0, xT, aT, lamT, uT, dyT, daT,
                                     dacc ? dacc + nV * slotD : nullptr, accT, dzT, hstore, st);
            ++h;
        }
        if (e != cudaSuccess) return e;
    }
    if (nH > 0) {   // sums of the horizontal directions back to the image layout
        if (nV > 0) {
            if ((e = launch_transpose<float, float, true>(accT, acc, planes, P.W, P.H, st)) != cudaSuccess) return e;
            if ((e = launch_transpose<float, float, true>(dzT, dz, planes, P.W, P.H, st)) != cudaSuccess) return e;
        } else {
            if ((e = launch_transpose<float, float, false>(accT, acc, planes, P.W, P.H, st)) != cudaSuccess) return e;
            if ((e = launch_transpose<float, float, false>(dzT, dz, planes, P.W, P.H, st)) != cudaSuccess) return e;
        }
    }
    const int blocks = (int)std::max<long long>(1, std::min<long long>(4096, (P.U + 255) / 256));
    k_gen_bwd_final<T><<<blocks, 256, 0, st>>>((const T*)x, (const T*)lam, (const T*)dy, dz, acc, (T*)dx, (T*)dlam,
                                               (T*)du, P.U);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (shared) {
        if (nV > 0) {
            const long long nv = (long long)nV * slotD;
            const int ab = (int)std::max<long long>(1, std::min<long long>(4096, (nv + 255) / 256));
            k_fixed_to<T><<<ab, 256, 0, st>>>(dacc, (T*)da, nv);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
        }
        if (nH > 0 &&
            (e = launch_transpose<unsigned long long, T, false>(dacc + nV * slotD, (T*)da + nV * slotA,
                                                                (long long)nH * P.N * 3, P.W, P.H, st)) != cudaSuccess)
            return e;
    } else if (nH > 0) {
        if ((e = launch_transpose<T, T, false>(daT, (T*)da + nV * slotA, (long long)nH * P.N * P.Cw * 3, P.W, P.H,
                                               st)) != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace

bool generic_supports(const Problem& p, bool bwd) {
    const int M = std::max(p.H, p.W);
    return M <= (bwd ? kGenBwdMaxLanes : kGenFwdMaxLanes);
}

size_t generic_ws_bytes(const Problem& p, bool bwd) {
    size_t b = 256;
    if (!bwd) {
        if (p.D > 1) b += align256(p.U * sizeof(float));
        return b;
    }
    b += 3 * align256(p.U * sizeof(float));
    if (p.wmode == GSPN_W_SHARED) b += align256(p.A * sizeof(unsigned long long));
    const int nh = ((p.mask & kLR) ? 1 : 0) + ((p.mask & kRL) ? 1 : 0);
    if (!p.per_dir && nh > 0) {
        const size_t es = p.esize();
        const size_t slot_a = (size_t)p.N * p.Cw * 3 * p.HW;
        b += 2 * align256(p.U * sizeof(float)) + 4 * align256(p.U * es) + align256(nh * slot_a * es);
        if (p.wmode != GSPN_W_SHARED) b += align256(nh * slot_a * es);
    }
    return b;
}

cudaError_t generic_forward(const Problem& p, const void* x, const void* a, const void* lam, const void* u, void* y,
                            void* ws, cudaStream_t st) {
    if (p.dtype == GSPN_F32) return gen_forward_t<float>(p, x, a, lam, u, y, ws, st);
    return gen_forward_t<__nv_bfloat16>(p, x, a, lam, u, y, ws, st);
}

cudaError_t generic_backward(const Problem& p, const void* x, const void* a, const void* lam, const void* u,
                             const void* dy, void* dx, void* da, void* dlam, void* du, void* ws, cudaStream_t st) {
    if (p.dtype == GSPN_F32) return gen_backward_t<float>(p, x, a, lam, u, dy, dx, da, dlam, du, ws, st);
    return gen_backward_t<__nv_bfloat16>(p, x, a, lam, u, dy, dx, da, dlam, du, ws, st);
}

}  // namespace gspn
