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

// Forward scan of one direction for plane blockIdx.x. Writes y (last direction), the fp32
// partial sum (other directions) and, when hstore is set, this direction's h.
template <typename T>
__global__ void k_gen_fwd(GenArgs p) {
    extern __shared__ float sh[];
    const int plane = blockIdx.x;
    const int n = plane / p.C, c = plane % p.C;
    const long long HW = (long long)p.H * p.W;
    const int L = is_vertical(p.dir) ? p.H : p.W;
    const int M = is_vertical(p.dir) ? p.W : p.H;
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
    for (int i = 0; i < L; ++i) {
        for (int j = threadIdx.x; j < M; j += blockDim.x) {
            const long long q = scan_pixel(p.dir, p.H, p.W, i, j);
            float h = Io<T>::ld(lam + q) * Io<T>::ld(x + q);
            if (!chunk_start(scan_ascending(p.dir), L, p.chunk, i)) {
                float w0, w1, w2;
                lane_weights(Io<T>::ld(a3 + q), Io<T>::ld(a3 + HW + q), Io<T>::ld(a3 + 2 * HW + q), j > 0,
                             j < M - 1, w0, w1, w2);
                if (j > 0) h = fmaf(w0, hp[j - 1], h);
                h = fmaf(w1, hp[j], h);
                if (j < M - 1) h = fmaf(w2, hp[j + 1], h);
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

struct GenBwdArgs {
    const void* a;
    const void* u;
    const void* dy;
    void* da;            // per-channel mode: written directly (storage dtype)
    float* dacc;         // shared mode: fp32 sum over channels (zeroed before)
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
template <typename T>
__global__ void k_gen_bwd(GenBwdArgs p) {
    extern __shared__ float sh[];
    const int plane = blockIdx.x;
    const int n = plane / p.C, c = plane % p.C;
    const long long HW = (long long)p.H * p.W;
    const int L = is_vertical(p.dir) ? p.H : p.W;
    const int M = is_vertical(p.dir) ? p.W : p.H;
    const long long lu = p.per_dir ? (long long)p.slot * p.N * p.C * HW : 0;   // this direction's lam / u
    const T* u = (const T*)p.u + lu + plane * HW;
    const T* dy = (const T*)p.dy + plane * HW;
    const long long abase = (((long long)p.slot * p.N + n) * p.Cw + (p.Cw == 1 ? 0 : c)) * 3 * HW;
    const T* a3 = (const T*)p.a + abase;
    T* da3 = p.da ? (T*)p.da + abase : nullptr;
    float* dacc3 = p.dacc ? p.dacc + (((long long)p.slot * p.N + n) * 3) * HW : nullptr;
    float* dz = p.dz + plane * HW;
    const float* hs = p.hstore + plane * HW;
    // [delta prev | delta cur | w(prev buffer) x3 | w(cur buffer) x3]
    float* dprev = sh;
    float* dcur = sh + M;
    float* wprev = sh + 2 * M;
    float* wcur = sh + 5 * M;
    for (int i = L - 1; i >= 0; --i) {
        for (int j = threadIdx.x; j < M; j += blockDim.x) {
            const long long q = scan_pixel(p.dir, p.H, p.W, i, j);
            float del = Io<T>::ld(u + q) * Io<T>::ld(dy + q);
            // no delta flows back through the first line of a chunk (it does not see h_{i-1})
            if (i < L - 1 && !chunk_start(scan_ascending(p.dir), L, p.chunk, i + 1)) {
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
            if (!chunk_start(scan_ascending(p.dir), L, p.chunk, i)) {
                const bool hl = j > 0, hr = j < M - 1;
                LaneJac J = lane_jacobian(Io<T>::ld(a3 + q), Io<T>::ld(a3 + HW + q), Io<T>::ld(a3 + 2 * HW + q),
                                          hl, hr);
                const float h0 = hl ? hs[scan_pixel(p.dir, p.H, p.W, i - 1, j - 1)] : 0.f;
                const float h1 = hs[scan_pixel(p.dir, p.H, p.W, i - 1, j)];
                const float h2 = hr ? hs[scan_pixel(p.dir, p.H, p.W, i - 1, j + 1)] : 0.f;
                const float dw0 = del * h0, dw1 = del * h1, dw2 = del * h2;
                const float s = J.w0 * dw0 + J.w1 * dw1 + J.w2 * dw2;
                const float g0 = J.g0 * (dw0 - s), g1 = J.g1 * (dw1 - s), g2 = J.g2 * (dw2 - s);
                if (da3) {
                    Io<T>::st(da3 + q, g0);
                    Io<T>::st(da3 + HW + q, g1);
                    Io<T>::st(da3 + 2 * HW + q, g2);
                } else {
                    atomicAdd(dacc3 + q, g0);
                    atomicAdd(dacc3 + HW + q, g1);
                    atomicAdd(dacc3 + 2 * HW + q, g2);
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

int gen_threads(int M) { return std::min(1024, std::max(32, ((M + 31) / 32) * 32)); }

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
        const int M = is_vertical(d) ? P.W : P.H;
        const size_t smem = 2 * (size_t)M * sizeof(float);
        cudaFuncSetAttribute(k_gen_fwd<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        launch_begin(st);
        k_gen_fwd<T><<<P.N * P.C, gen_threads(M), smem, st>>>(g);
        launch_end(st);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
        ++slot;
        ++seen;
    }
    return cudaSuccess;
}

template <typename T>
cudaError_t gen_backward_t(const Problem& P, const void* x, const void* a, const void* lam, const void* u,
                           const void* dy, void* dx, void* da, void* dlam, void* du, void* ws, cudaStream_t st) {
    WsCarver wc(ws);
    float* acc = wc.take<float>(P.U);
    float* dz = wc.take<float>(P.U);
    float* hstore = wc.take<float>(P.U);
    float* dacc = P.wmode == GSPN_W_SHARED ? wc.take<float>(P.A) : nullptr;
    cudaError_t e;
    if (dacc) {
        e = cudaMemsetAsync(dacc, 0, P.A * sizeof(float), st);
        if (e != cudaSuccess) return e;
    }
    int slot = 0, seen = 0;
    for (unsigned d = kTB; d <= kRL; d <<= 1) {
        if (!(P.mask & d)) continue;
        const int M = is_vertical(d) ? P.W : P.H;
        // 1) recompute this direction's h (image coordinates) and accumulate sum_d h for du
        GenArgs g{x, a, lam, u, nullptr, acc, hstore, P.N, P.C, P.H, P.W, P.Cw, P.D, d, slot, seen == 0, false,
                  P.chunk, P.per_dir};
        if (P.D == 1) g.first = 1;
        size_t smem = 2 * (size_t)M * sizeof(float);
        cudaFuncSetAttribute(k_gen_fwd<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_gen_fwd<T><<<P.N * P.C, gen_threads(M), smem, st>>>(g);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        // 2) reverse scan
        GenBwdArgs b{a, u, dy, dacc ? nullptr : da, dacc, dz, hstore, P.N, P.C, P.H, P.W, P.Cw, d, slot, seen == 0,
                     P.chunk, P.per_dir, x, lam, dlam, du};
        smem = 8 * (size_t)M * sizeof(float);
        cudaFuncSetAttribute(k_gen_bwd<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k_gen_bwd<T><<<P.N * P.C, gen_threads(M), smem, st>>>(b);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        ++slot;
        ++seen;
    }
    const int blocks = (int)std::max<long long>(1, std::min<long long>(4096, (P.U + 255) / 256));
    if (P.per_dir) {
        k_f32_to<T><<<blocks, 256, 0, st>>>(dz, (T*)dx, P.U);   // dlam_d, du_d written per direction
    } else {
        k_gen_bwd_final<T><<<blocks, 256, 0, st>>>((const T*)x, (const T*)lam, (const T*)dy, dz, acc, (T*)dx,
                                                   (T*)dlam, (T*)du, P.U);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (dacc) {
        const int ab = (int)std::max<long long>(1, std::min<long long>(4096, (P.A + 255) / 256));
        k_f32_to<T><<<ab, 256, 0, st>>>(dacc, (T*)da, P.A);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
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
    if (p.wmode == GSPN_W_SHARED) b += align256(p.A * sizeof(float));
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
