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

// Weights and Jacobian factors of one lane (see lane_jacobian) with one reciprocal: with
// p_k = 1 + e_k, e_k = exp(-a_k), the in-range numerators q_k (products of the other two p's),
// D = q0 + q1 + q2, P = the product of the in-range p's and r = 1 / (P D): w_k = q_k P r and
// sigmoid(a_k) = 1 / p_k = q_k D r, so g_k = w_k (1 - sigmoid(a_k)) = w_k e_k q_k D r. P D stays
// finite while every in-range logit is >= kJacBelow; otherwise the accurate form is used. w1 is
// taken as 1 - w0 - w2.
constexpr float kJacBelow = -17.f;
__device__ __forceinline__ LaneJac lane_jacobian_1r(float a0, float a1, float a2, bool has_l, bool has_r) {
    const float amin = fminf(a1, fminf(has_l ? a0 : a1, has_r ? a2 : a1));
    if (amin < kJacBelow) return lane_jacobian(a0, a1, a2, has_l, has_r);
    // out-of-range logits are clamped so that they cannot produce inf * 0
    const float e0 = __expf(-fmaxf(a0, kJacBelow));
    const float e1 = __expf(-fmaxf(a1, kJacBelow));
    const float e2 = __expf(-fmaxf(a2, kJacBelow));
    const float p0 = 1.f + e0, p1 = 1.f + e1, p2 = 1.f + e2;
    const Wts q = weights_from_p(p0, p1, p2, has_l, has_r);
    const float Dn = q.w0 + q.w1 + q.w2;
    const float P = (has_l ? p0 : 1.f) * p1 * (has_r ? p2 : 1.f);
    const float r = __fdividef(1.f, P * Dn);
    const float inv = P * r, dr = Dn * r;
    LaneJac J;
    J.w0 = q.w0 * inv;
    J.w2 = q.w2 * inv;
    // the row sums to one exactly (a single in-range neighbour gets w1 = 1 and no gradient)
    J.w1 = 1.f - J.w0 - J.w2;
    J.g0 = J.w0 * e0 * (q.w0 * dr);
    J.g1 = J.w1 * e1 * (q.w1 * dr);
    J.g2 = J.w2 * e2 * (q.w2 * dr);
    return J;
}

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
                const LaneJac J = lane_jacobian_1r(Io<T>::ld(a3 + q), Io<T>::ld(a3 + HW + q),
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

// ---- Concurrent backward for lam and u shared by the directions: every direction of every plane
// in one launch (grid y = direction), the horizontal directions as top->bottom / bottom->top scans
// of transposed copies, so every line is a row. Each direction writes its own slots of h, of the
// partial sum and of the adjoint (no read-modify-write across directions), which lets the SMs hold
// CTAs of several planes and directions at once and hide one plane's step latency behind another's.
// A thread owns LPT lanes strided by the block size (lane j = thread + k * blockDim), so every
// warp-wide load, store and fixed-point atomic touches consecutive addresses. The loads of the next
// step are issued before the current step's arithmetic (they do not depend on it), and rows
// kPrefetch steps ahead are requested from L2. The lines in shared memory carry kPad zero lanes on
// each side, so edge lanes read zeros. Same arithmetic and summation order per lane as k_gen_fwd /
// k_gen_bwd.
constexpr int kPad = 4;
constexpr int kTT = 64;   // tile edge of the transposes
constexpr int kGenvLPT = 4;
constexpr int kGenvMaxLanes = 1024;

struct GenvDir {         // one direction's buffers, in the layout it scans (image or transposed)
    const void* x;
    const void* lam;
    const void* u;
    const void* dy;
    const void* a;       // this direction's logit slot: N x Cw x 3 x H x W
    float* hs;           // h of this direction (recompute -> reverse scan; summed by the final kernel)
    float* dz;           // adjoint delta of this direction
    void* da;            // per-channel mode: this direction's logit-gradient slot
    unsigned long long* dacc;   // shared mode: fixed-point sum over channels, N x 3 x H x W
    int H, W;            // scan length, lanes
    int asc;             // top->bottom (1) or bottom->top (0)
    const float* zp;     // non-null: z = lam x of this direction, formed beforehand (read instead of x, lam)
    const float* gp;     // non-null: g = u dy of this direction, formed beforehand (read instead of u, dy)
};
struct GenvArgs {
    GenvDir d[4];
    int N, C, Cw, chunk;
};

// Warp 0 asks L2 for every 128-byte line of a row (one line per lane, strided by 32 lines); the
// other warps skip the prefetch block.
template <typename E>
__device__ __forceinline__ void pf_row(const E* row, int W, int t) {
    const int bytes = W * (int)sizeof(E);   // at most 32 lines for 4-byte lanes, 64 for 8-byte ones
    if (t * 128 < bytes) pf_l2((const char*)row + t * 128);
    if constexpr (sizeof(E) > 4)
        if ((t + 32) * 128 < bytes) pf_l2((const char*)row + (t + 32) * 128);
}

template <typename T, int LPT, int NT>
__global__ void __launch_bounds__(NT, 2) k_genv_fwd(GenvArgs p) {
    extern __shared__ float sh[];
    const GenvDir& D = p.d[blockIdx.y];
    const bool asc = D.asc != 0;
    const int plane = blockIdx.x;
    const int n = plane / p.C, c = plane % p.C;
    const int H = D.H, W = D.W, LW = W + 2 * kPad;
    const long long HW = (long long)H * W;
    const T* x = (const T*)D.x + plane * HW;
    const T* lam = (const T*)D.lam + plane * HW;
    const float* zp = D.zp ? D.zp + plane * HW : nullptr;
    const T* a0p = (const T*)D.a + ((long long)n * p.Cw + (p.Cw == 1 ? 0 : c)) * 3 * HW;
    const T* a1p = a0p + HW;
    const T* a2p = a1p + HW;
    float* hst = D.hs + plane * HW;
    float* hp = sh;
    float* hc = sh + LW;
    for (int e = threadIdx.x; e < 2 * LW; e += NT) sh[e] = 0.f;
    const int t = threadIdx.x;
    auto rowo = [&](int i) { return (asc ? i : H - 1 - i) * W; };   // row offset in the plane
    float nx[LPT], nl[LPT], n0[LPT], n1[LPT], n2[LPT];
    auto fetch = [&](int i) {
        const int o = rowo(i) + t;
#pragma unroll
        for (int k = 0; k < LPT; ++k) {
            if (t + k * NT >= W) break;
            if (zp) {   // h starts from z = 1 * z, the same product
                nx[k] = zp[o + k * NT];
                nl[k] = 1.f;
            } else {
                nx[k] = Io<T>::ld(x + o + k * NT);
                nl[k] = Io<T>::ld(lam + o + k * NT);
            }
            n0[k] = Io<T>::ld(a0p + o + k * NT);
            n1[k] = Io<T>::ld(a1p + o + k * NT);
            n2[k] = Io<T>::ld(a2p + o + k * NT);
        }
    };
    fetch(0);
    __syncthreads();
    for (int i = 0; i < H; ++i) {
        float cx[LPT], cl[LPT], c0[LPT], c1[LPT], c2[LPT];
#pragma unroll
        for (int k = 0; k < LPT; ++k) {
            cx[k] = nx[k]; cl[k] = nl[k]; c0[k] = n0[k]; c1[k] = n1[k]; c2[k] = n2[k];
        }
        if (i + 1 < H) fetch(i + 1);
        if (t < 32 && i + kPrefetch < H) {   // warp 0 alone (pf_row strides over the row)
            const int f = rowo(i + kPrefetch);
            if (zp) {
                pf_row(zp + f, W, t);
            } else {
                pf_row(x + f, W, t);
                pf_row(lam + f, W, t);
            }
            pf_row(a0p + f, W, t);
            pf_row(a1p + f, W, t);
            pf_row(a2p + f, W, t);
        }
        const int o = rowo(i) + t;
        const bool cs = chunk_start(asc, H, p.chunk, i);
#pragma unroll
        for (int k = 0; k < LPT; ++k) {
            const int j = t + k * NT;
            if (j >= W) break;
            float h = cl[k] * cx[k];
            if (!cs) {
                const Wts w = lane_weights_fast(c0[k], c1[k], c2[k], j > 0, j < W - 1);
                if (j > 0) h = fmaf(w.w0, hp[kPad + j - 1], h);
                h = fmaf(w.w1, hp[kPad + j], h);
                if (j < W - 1) h = fmaf(w.w2, hp[kPad + j + 1], h);
            }
            hc[kPad + j] = h;
            hst[o + k * NT] = h;
        }
        __syncthreads();
        float* tt = hp;
        hp = hc;
        hc = tt;
    }
}

template <typename T, bool SHARED, int LPT, int NT>
__global__ void __launch_bounds__(NT, 2) k_genv_bwd(GenvArgs p) {
    extern __shared__ float sh[];
    const GenvDir& D = p.d[blockIdx.y];
    const bool asc = D.asc != 0;
    const int plane = blockIdx.x;
    const int n = plane / p.C, c = plane % p.C;
    const int H = D.H, W = D.W, LW = W + 2 * kPad;
    const long long HW = (long long)H * W;
    const T* u = (const T*)D.u + plane * HW;
    const T* dy = (const T*)D.dy + plane * HW;
    const float* gp = D.gp ? D.gp + plane * HW : nullptr;
    const long long abase = ((long long)n * p.Cw + (p.Cw == 1 ? 0 : c)) * 3 * HW;
    const T* a0p = (const T*)D.a + abase;
    const T* a1p = a0p + HW;
    const T* a2p = a1p + HW;
    T* da0 = SHARED ? nullptr : (T*)D.da + abase;
    unsigned long long* dq0 = SHARED ? D.dacc + (long long)n * 3 * HW : nullptr;
    float* dz = D.dz + plane * HW;
    const float* hs = D.hs + plane * HW;
    // [delta prev | delta cur | w prev x3 | w cur x3 | h of line i-1, two buffers], each padded
    float* dprev = sh;
    float* dcur = sh + LW;
    float* wprev = sh + 2 * LW;
    float* wcur = sh + 5 * LW;
    float* hb = sh + 8 * LW;
    for (int e = threadIdx.x; e < 10 * LW; e += NT) sh[e] = 0.f;
    const int t = threadIdx.x;
    auto rowo = [&](int i) { return (asc ? i : H - 1 - i) * W; };
    float nu[LPT], ndy[LPT], n0[LPT], n1[LPT], n2[LPT], nh[LPT];
    // the loads of step i: u, dy, logits of line i and h of line i - 1 (its neighbours are read
    // from the shared copy that step i's predecessor writes, one barrier later)
    auto fetch = [&](int i) {
        const int o = rowo(i) + t;
        const int o1 = i > 0 ? rowo(i - 1) + t : 0;
#pragma unroll
        for (int k = 0; k < LPT; ++k) {
            if (t + k * NT >= W) break;
            if (gp) {   // delta starts from g = g * 1, the same product
                nu[k] = gp[o + k * NT];
                ndy[k] = 1.f;
            } else {
                nu[k] = Io<T>::ld(u + o + k * NT);
                ndy[k] = Io<T>::ld(dy + o + k * NT);
            }
            n0[k] = Io<T>::ld(a0p + o + k * NT);
            n1[k] = Io<T>::ld(a1p + o + k * NT);
            n2[k] = Io<T>::ld(a2p + o + k * NT);
            nh[k] = i > 0 ? hs[o1 + k * NT] : 0.f;
        }
    };
    fetch(H - 1);
    int hbuf = 0;
    {   // h of line H - 2 into the shared copy for the first step
        float* hl = hb + kPad;
#pragma unroll
        for (int k = 0; k < LPT; ++k)
            if (t + k * NT < W) hl[t + k * NT] = nh[k];
    }
    __syncthreads();
    for (int i = H - 1; i >= 0; --i) {
        float cu[LPT], cdy[LPT], c0[LPT], c1[LPT], c2[LPT];
#pragma unroll
        for (int k = 0; k < LPT; ++k) {
            cu[k] = nu[k]; cdy[k] = ndy[k]; c0[k] = n0[k]; c1[k] = n1[k]; c2[k] = n2[k];
        }
        const float* hl = hb + hbuf * LW + kPad;   // h of line i - 1 (all lanes, from the previous step)
        if (i > 0) {
            fetch(i - 1);
            // h of line i - 2 for the next step, into the other buffer
            float* hn = hb + (hbuf ^ 1) * LW + kPad;
#pragma unroll
            for (int k = 0; k < LPT; ++k)
                if (t + k * NT < W) hn[t + k * NT] = nh[k];
        }
        if (t < 32 && i - kPrefetch >= 1) {   // warp 0 alone (pf_row strides over the row)
            const int f = rowo(i - kPrefetch);
            if (gp) {
                pf_row(gp + f, W, t);
            } else {
                pf_row(u + f, W, t);
                pf_row(dy + f, W, t);
            }
            pf_row(a0p + f, W, t);
            pf_row(a1p + f, W, t);
            pf_row(a2p + f, W, t);
            pf_row(hs + rowo(i - kPrefetch - 1), W, t);
            if (SHARED) {
                pf_row(dq0 + f, W, t);
                pf_row(dq0 + HW + f, W, t);
                pf_row(dq0 + 2 * HW + f, W, t);
            }
        }
        const int o = rowo(i) + t;
        // no delta flows back through the first line of a chunk (it does not see h_{i-1})
        const bool back = i < H - 1 && !chunk_start(asc, H, p.chunk, i + 1);
        const bool cs = chunk_start(asc, H, p.chunk, i);
        const float* dpv = dprev + kPad;
        const float* w0v = wprev + kPad;
        const float* w1v = wprev + LW + kPad;
        const float* w2v = wprev + 2 * LW + kPad;
#pragma unroll
        for (int k = 0; k < LPT; ++k) {
            const int j = t + k * NT;
            if (j >= W) break;
            float d = cu[k] * cdy[k];
            if (back) {
                // (w_{i+1}^T delta_{i+1})[j] = w[j-1][2] d[j-1] + w[j][1] d[j] + w[j+1][0] d[j+1]
                if (j > 0) d = fmaf(w2v[j - 1], dpv[j - 1], d);
                d = fmaf(w1v[j], dpv[j], d);
                if (j < W - 1) d = fmaf(w0v[j + 1], dpv[j + 1], d);
            }
            dcur[kPad + j] = d;
            dz[o + k * NT] = d;
            float g0 = 0.f, g1 = 0.f, g2 = 0.f;
            if (!cs) {
                const LaneJac J = lane_jacobian_1r(c0[k], c1[k], c2[k], j > 0, j < W - 1);
                const float dw0 = d * hl[j - 1], dw1 = d * hl[j], dw2 = d * hl[j + 1];
                const float sm = J.w0 * dw0 + J.w1 * dw1 + J.w2 * dw2;
                g0 = J.g0 * (dw0 - sm);
                g1 = J.g1 * (dw1 - sm);
                g2 = J.g2 * (dw2 - sm);
                wcur[kPad + j] = J.w0;
                wcur[LW + kPad + j] = J.w1;
                wcur[2 * LW + kPad + j] = J.w2;
                if constexpr (SHARED) {
                    atomicAdd(dq0 + o + k * NT, to_fixed(g0));
                    atomicAdd(dq0 + HW + o + k * NT, to_fixed(g1));
                    atomicAdd(dq0 + 2 * HW + o + k * NT, to_fixed(g2));
                }
            }
            if constexpr (!SHARED) {
                Io<T>::st(da0 + o + k * NT, g0);
                Io<T>::st(da0 + HW + o + k * NT, g1);
                Io<T>::st(da0 + 2 * HW + o + k * NT, g2);
            }
        }
        __syncthreads();
        float* tt = dprev; dprev = dcur; dcur = tt;
        tt = wprev; wprev = wcur; wcur = tt;
        hbuf ^= 1;
    }
}

// dx = lam dz, dlam = x dz, du = dy acc with dz and acc the sums of the directions' slots: up to
// two image-layout slots (the vertical directions) and up to two transposed ones ([W][H] per plane,
// the horizontal directions), the latter read through a 64 x 64 shared-memory transpose per tile
// (coalesced on both sides). Null slots are absent directions. Per element the sum is taken as
// (horizontal 0 + horizontal 1) + vertical 0 + vertical 1.
struct GenvFinal {
    const float *accV0, *accV1, *dzV0, *dzV1;   // image layout
    const float *accH0, *accH1, *dzH0, *dzH1;   // transposed layout
};
template <typename T>
__global__ void __launch_bounds__(256) k_genv_final(GenvFinal f, const T* __restrict__ x, const T* __restrict__ lam,
                                                    const T* __restrict__ dy, T* dx, T* dlam, T* du, int H, int W) {
    __shared__ float ta[kTT][kTT + 1];
    __shared__ float tz[kTT][kTT + 1];
    const long long HW = (long long)H * W, pb = blockIdx.z * HW;
    const int r0 = blockIdx.y * kTT, c0 = blockIdx.x * kTT;
    const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
    if (f.accH0) {
        // transposed slots: image (r, c) at [c][r]; this thread reads rows c0 + ty + 4k, column r0 + tx
#pragma unroll 4
        for (int k = 0; k < 16; ++k) {
            const int c = c0 + ty + 4 * k, r = r0 + tx;
            float va = 0.f, vz = 0.f;
            if (r < H && c < W) {
                const long long q = pb + (long long)c * H + r;
                va = f.accH0[q];
                vz = f.dzH0[q];
                if (f.accH1) {
                    va += f.accH1[q];
                    vz += f.dzH1[q];
                }
            }
            ta[ty + 4 * k][tx] = va;
            tz[ty + 4 * k][tx] = vz;
        }
    }
    __syncthreads();
#pragma unroll 4
    for (int k = 0; k < 16; ++k) {
        const int r = r0 + ty + 4 * k, c = c0 + tx;
        if (r >= H || c >= W) continue;
        const long long e = pb + (long long)r * W + c;
        float a = f.accH0 ? ta[tx][ty + 4 * k] : 0.f;
        float z = f.accH0 ? tz[tx][ty + 4 * k] : 0.f;
        if (f.accV0) {
            a += f.accV0[e];
            z += f.dzV0[e];
        }
        if (f.accV1) {
            a += f.accV1[e];
            z += f.dzV1[e];
        }
        Io<T>::st(dx + e, Io<T>::ld(lam + e) * z);
        Io<T>::st(dlam + e, Io<T>::ld(x + e) * z);
        Io<T>::st(du + e, Io<T>::ld(dy + e) * a);
    }
}

// Per-direction lambda / u (the learnable merge): y = sum_d u_d h_d with h_d driven by lambda_d x,
// so dx = sum_d lambda_d delta_d, dlambda_d = x delta_d and du_d = dy h_d. Same tiling as
// k_genv_final; slot d of h and delta is image layout (vertical) or transposed (horizontal), and
// slot d of lambda, dlambda and du is image layout at d * U. dx sums the slots in direction order.
struct GenvFinalPD {
    const float* hs[4];
    const float* dz[4];
    int vert[4];
    int D;
    long long U;
};
template <typename T>
__global__ void __launch_bounds__(256) k_genv_final_pd(GenvFinalPD f, const T* __restrict__ x, const T* __restrict__ lam,
                                                       const T* __restrict__ dy, T* dx, T* dlam, T* du, int H, int W) {
    __shared__ float th[kTT][kTT + 1];
    __shared__ float tz[kTT][kTT + 1];
    const long long HW = (long long)H * W, pb = blockIdx.z * HW;
    const int r0 = blockIdx.y * kTT, c0 = blockIdx.x * kTT;
    const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
    float sx[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) sx[k] = 0.f;
    for (int d = 0; d < f.D; ++d) {
        const float* hsd = f.hs[d] + pb;
        const float* dzd = f.dz[d] + pb;
        const bool vert = f.vert[d] != 0;
        if (!vert) {   // transposed slot: image (r, c) at [c][r]
#pragma unroll 4
            for (int k = 0; k < 16; ++k) {
                const int c = c0 + ty + 4 * k, r = r0 + tx;
                const bool in = r < H && c < W;
                th[ty + 4 * k][tx] = in ? hsd[(long long)c * H + r] : 0.f;
                tz[ty + 4 * k][tx] = in ? dzd[(long long)c * H + r] : 0.f;
            }
        }
        __syncthreads();
#pragma unroll 4
        for (int k = 0; k < 16; ++k) {
            const int r = r0 + ty + 4 * k, c = c0 + tx;
            if (r >= H || c >= W) continue;
            const long long e = pb + (long long)r * W + c;
            const float hv = vert ? hsd[e - pb] : th[tx][ty + 4 * k];
            const float zv = vert ? dzd[e - pb] : tz[tx][ty + 4 * k];
            const long long ed = d * f.U + e;
            sx[k] += Io<T>::ld(lam + ed) * zv;
            Io<T>::st(dlam + ed, Io<T>::ld(x + e) * zv);
            Io<T>::st(du + ed, Io<T>::ld(dy + e) * hv);
        }
        __syncthreads();
    }
#pragma unroll 4
    for (int k = 0; k < 16; ++k) {
        const int r = r0 + ty + 4 * k, c = c0 + tx;
        if (r < H && c < W) Io<T>::st(dx + pb + (long long)r * W + c, sx[k]);
    }
}

// Forward output from the per-direction h slots: y = sum_d u_d h_d (per-direction u, slot d of u
// at d * U) or y = u sum_d h_d (shared u), the slots summed in direction order; horizontal slots
// read through a 64 x 64 shared-memory transpose per tile.
template <typename T>
__global__ void __launch_bounds__(256) k_genv_y(GenvFinalPD f, const T* __restrict__ u, T* y, int H, int W,
                                                int per_dir) {
    __shared__ float th[kTT][kTT + 1];
    const long long HW = (long long)H * W, pb = blockIdx.z * HW;
    const int r0 = blockIdx.y * kTT, c0 = blockIdx.x * kTT;
    const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
    float sy[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) sy[k] = 0.f;
    for (int d = 0; d < f.D; ++d) {
        const float* hsd = f.hs[d] + pb;
        const bool vert = f.vert[d] != 0;
        if (!vert) {   // transposed slot: image (r, c) at [c][r]
#pragma unroll 4
            for (int k = 0; k < 16; ++k) {
                const int c = c0 + ty + 4 * k, r = r0 + tx;
                th[ty + 4 * k][tx] = (r < H && c < W) ? hsd[(long long)c * H + r] : 0.f;
            }
        }
        __syncthreads();
#pragma unroll 4
        for (int k = 0; k < 16; ++k) {
            const int r = r0 + ty + 4 * k, c = c0 + tx;
            if (r >= H || c >= W) continue;
            const long long e = (long long)r * W + c;
            const float hv = vert ? hsd[e] : th[tx][ty + 4 * k];
            sy[k] += per_dir ? Io<T>::ld(u + d * f.U + pb + e) * hv : hv;
        }
        __syncthreads();
    }
#pragma unroll 4
    for (int k = 0; k < 16; ++k) {
        const int r = r0 + ty + 4 * k, c = c0 + tx;
        if (r >= H || c >= W) continue;
        const long long e = pb + (long long)r * W + c;
        Io<T>::st(y + e, per_dir ? sy[k] : Io<T>::ld(u + e) * sy[k]);
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
// Batched transpose of R x Cc planes through 64 x 64 shared tiles; a thread moves 16 elements and
// issues all 16 loads before the first shared-memory store (enough bytes in flight per SM to keep
// HBM busy). ADD adds the transposed values onto dst.
template <typename S, typename D, bool ADD>
__global__ void __launch_bounds__(256) k_transpose(const S* __restrict__ src, D* __restrict__ dst, int R, int Cc) {
    __shared__ float tile[kTT][kTT + 1];
    const long long b = blockIdx.z;
    const int r0 = blockIdx.y * kTT, c0 = blockIdx.x * kTT;
    const S* sp = src + b * (long long)R * Cc;
    D* dp = dst + b * (long long)R * Cc;
    const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;   // 64 x 4 threads
    float v[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const int r = r0 + ty + 4 * k, c = c0 + tx;
        v[k] = (r < R && c < Cc) ? ld_any(sp + (long long)r * Cc + c) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) tile[ty + 4 * k][tx] = v[k];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const int c = c0 + ty + 4 * k, r = r0 + tx;
        if (r < R && c < Cc) {
            D* q = dp + (long long)c * R + r;
            const float t = tile[tx][ty + 4 * k];
            Io<D>::st(q, ADD ? Io<D>::ld(q) + t : t);
        }
    }
}
template <typename S, typename D, bool ADD>
cudaError_t launch_transpose(const S* src, D* dst, long long B, int R, int Cc, cudaStream_t st) {
    const long long plane = (long long)R * Cc;
    for (long long b0 = 0; b0 < B; b0 += 65535) {   // grid z is limited to 65535
        const long long nb = std::min<long long>(65535, B - b0);
        dim3 grid((unsigned)((Cc + kTT - 1) / kTT), (unsigned)((R + kTT - 1) / kTT), (unsigned)nb);
        k_transpose<S, D, ADD><<<grid, 256, 0, st>>>(src + b0 * plane, dst + b0 * plane, R, Cc);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

// dst = transpose(a * b) per plane, in fp32: the product the horizontal scans consume (z = lam x
// for the recompute, g = u dy for the reverse scan), formed while transposing so that one plane
// set crosses HBM instead of two.
template <typename S>
__global__ void __launch_bounds__(256) k_transpose_mul(const S* __restrict__ a, const S* __restrict__ b,
                                                       float* __restrict__ dst, int R, int Cc) {
    __shared__ float tile[kTT][kTT + 1];
    const long long pb = (long long)blockIdx.z * R * Cc;
    const int r0 = blockIdx.y * kTT, c0 = blockIdx.x * kTT;
    const int tx = threadIdx.x & 63, ty = threadIdx.x >> 6;
    float v[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const int r = r0 + ty + 4 * k, c = c0 + tx;
        const long long q = pb + (long long)r * Cc + c;
        v[k] = (r < R && c < Cc) ? Io<S>::ld(a + q) * Io<S>::ld(b + q) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < 16; ++k) tile[ty + 4 * k][tx] = v[k];
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        const int c = c0 + ty + 4 * k, r = r0 + tx;
        if (r < R && c < Cc) dst[pb + (long long)c * R + r] = tile[tx][ty + 4 * k];
    }
}
// planes of a (a_planes of them, each multiplied by the plane of b with the same index modulo
// b_planes) transposed into dst.
template <typename S>
cudaError_t launch_transpose_mul(const S* a, const S* b, float* dst, long long a_planes, long long b_planes, int R,
                                 int Cc, cudaStream_t st) {
    const long long plane = (long long)R * Cc;
    for (long long s0 = 0; s0 < a_planes; s0 += b_planes) {   // one launch per set of b_planes
        for (long long b0 = 0; b0 < b_planes; b0 += 65535) {   // grid z is limited to 65535
            const long long nb = std::min<long long>(65535, b_planes - b0);
            dim3 grid((unsigned)((Cc + kTT - 1) / kTT), (unsigned)((R + kTT - 1) / kTT), (unsigned)nb);
            k_transpose_mul<S><<<grid, 256, 0, st>>>(a + (s0 + b0) * plane, b + b0 * plane, dst + (s0 + b0) * plane,
                                                      R, Cc);
            const cudaError_t e = cudaGetLastError();
            if (e != cudaSuccess) return e;
        }
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
    GenBwdArgs b{a, u, dy, dacc ? nullptr : da, dacc, dz, hstore, P.N, P.C, H, W, P.Cw, vdir, slot, first,
                 P.chunk, 0, x, lam, nullptr, nullptr};
    cudaError_t e = gen_fwd_launch<T>(g, M, st);
    if (e != cudaSuccess) return e;
    return gen_bwd_launch<T>(b, M, st);
}

int n_vert(const Problem& P) { return ((P.mask & kTB) ? 1 : 0) + ((P.mask & kBT) ? 1 : 0); }
int n_horz(const Problem& P) { return P.D - n_vert(P); }

// Launches the recompute (and, unless fwd_only, the reverse scan) over grid (planes, D). A thread
// owns LPT lanes at stride NT: one lane per thread up to 256 lanes (64, 128 or 256 threads, so
// small maps do not leave warps idle), four beyond.
template <typename T, int LPT, int NT>
cudaError_t genv_scans_cfg(const GenvArgs& g, int lanes, long long planes, int D, bool shared, bool fwd_only,
                           bool bwd_only, cudaStream_t st) {
    const size_t lw = (size_t)lanes + 2 * kPad;
    const dim3 grid((unsigned)planes, (unsigned)D);
    cudaError_t e;
    if (!bwd_only) {
        e = cudaFuncSetAttribute(k_genv_fwd<T, LPT, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(2 * lw * sizeof(float)));
        if (e != cudaSuccess) return e;
        launch_begin(st);
        k_genv_fwd<T, LPT, NT><<<grid, NT, 2 * lw * sizeof(float), st>>>(g);
        launch_end(st);
        if ((e = cudaGetLastError()) != cudaSuccess || fwd_only) return e;
    }
    auto kb = shared ? k_genv_bwd<T, true, LPT, NT> : k_genv_bwd<T, false, LPT, NT>;
    if ((e = cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(10 * lw * sizeof(float)))) !=
        cudaSuccess)
        return e;
    launch_begin(st);
    kb<<<grid, NT, 10 * lw * sizeof(float), st>>>(g);
    launch_end(st);
    return cudaGetLastError();
}
template <typename T>
cudaError_t genv_scans(const GenvArgs& g, int lanes, long long planes, int D, bool shared, bool fwd_only,
                       cudaStream_t st, bool bwd_only = false) {
    if (lanes <= 64) return genv_scans_cfg<T, 1, 64>(g, lanes, planes, D, shared, fwd_only, bwd_only, st);
    if (lanes <= 128) return genv_scans_cfg<T, 1, 128>(g, lanes, planes, D, shared, fwd_only, bwd_only, st);
    if (lanes <= 256) return genv_scans_cfg<T, 1, 256>(g, lanes, planes, D, shared, fwd_only, bwd_only, st);
    return genv_scans_cfg<T, kGenvLPT, kGenvMaxLanes / kGenvLPT>(g, lanes, planes, D, shared, fwd_only, bwd_only,
                                                                 st);
}

// The concurrent backward runs lines of at most kGenvMaxLanes lanes.
bool genv_ok(const Problem& P) {
    auto lanes_ok = [](int L) { return L <= kGenvMaxLanes; };
    return P.HW < (1LL << 31) && (n_vert(P) == 0 || lanes_ok(P.W)) && (n_horz(P) == 0 || lanes_ok(P.H));
}

// hsaved: each direction's h kept by the forward (slot k at k U, vertical slots in the image layout,
// horizontal ones transposed per plane), or null to recompute it.
template <typename T>
cudaError_t gen_backward_cc(const Problem& P, const void* x, const void* a, const void* lam, const void* u,
                            const void* dy, void* dx, void* da, void* dlam, void* du, void* ws, cudaStream_t st,
                            const float* hsaved = nullptr) {
    const bool shared = P.wmode == GSPN_W_SHARED;
    const int nV = n_vert(P), nH = n_horz(P);
    const long long slotA = (long long)P.N * P.Cw * 3 * P.HW;   // logits of one direction slot
    const long long slotD = (long long)P.N * 3 * P.HW;          // shared-mode gradient of one slot
    const long long planes = (long long)P.N * P.C;
    WsCarver wc(ws);
    float* hs = wc.take<float>((size_t)P.D * P.U);   // h per direction: also the terms of du
    if (hsaved) hs = const_cast<float*>(hsaved);     // kept by the forward: read only
    float* dz = wc.take<float>((size_t)P.D * P.U);
    unsigned long long* dacc = shared ? wc.take<unsigned long long>((size_t)P.D * slotD) : nullptr;
    T *aT = nullptr, *daT = nullptr;
    float *zT = nullptr, *gT = nullptr;   // z = lam x and g = u dy of the horizontal scans, transposed
    const int nlu = P.per_dir ? nH : 1;   // lambda / u planes sets the horizontal scans read
    if (nH > 0) {
        zT = wc.take<float>((size_t)nlu * P.U);
        gT = wc.take<float>((size_t)nlu * P.U);
        aT = wc.take<T>((size_t)nH * slotA);
        if (!shared) daT = wc.take<T>((size_t)nH * slotA);
    }
    cudaError_t e;
    if (dacc && (e = cudaMemsetAsync(dacc, 0, (size_t)P.D * slotD * sizeof(unsigned long long), st)) != cudaSuccess)
        return e;
    if (nH > 0) {
        // per-direction lambda / u: the horizontal slots follow the vertical ones
        const size_t lu0 = P.per_dir ? (size_t)nV * P.U : 0;
        if ((e = launch_transpose_mul<T>((const T*)lam + lu0, (const T*)x, zT, nlu * planes, planes, P.H, P.W, st)) !=
            cudaSuccess)
            return e;
        if ((e = launch_transpose_mul<T>((const T*)u + lu0, (const T*)dy, gT, nlu * planes, planes, P.H, P.W, st)) !=
            cudaSuccess)
            return e;
        // the horizontal slots follow the vertical ones: one batch of nH * N * Cw * 3 planes
        if ((e = launch_transpose<T, T, false>((const T*)a + nV * slotA, aT, (long long)nH * P.N * P.Cw * 3, P.H,
                                               P.W, st)) != cudaSuccess)
            return e;
    }
    GenvArgs g;
    g.N = P.N;
    g.C = P.C;
    g.Cw = P.Cw;
    g.chunk = P.chunk;
    int v = 0, h = 0, k = 0, lanes = 0;
    for (unsigned d = kTB; d <= kRL; d <<= 1) {
        if (!(P.mask & d)) continue;
        GenvDir& G = g.d[k];
        G.hs = hs + (size_t)k * P.U;
        G.dz = dz + (size_t)k * P.U;
        if (is_vertical(d)) {
            const size_t lu = P.per_dir ? (size_t)v * P.U : 0;
            G.x = x; G.lam = (const T*)lam + lu; G.u = (const T*)u + lu; G.dy = dy;
            G.zp = nullptr; G.gp = nullptr;
            G.a = (const T*)a + v * slotA;
            G.da = shared ? nullptr : (void*)((T*)da + v * slotA);
            G.dacc = shared ? dacc + v * slotD : nullptr;
            G.H = P.H; G.W = P.W; G.asc = d == kTB;
            ++v;
        } else {
            const size_t lu = P.per_dir ? (size_t)h * P.U : 0;
            G.x = x; G.lam = lam; G.u = u; G.dy = dy;   // not read: the scans take z and g
            G.zp = zT + lu; G.gp = gT + lu;
            G.a = aT + h * slotA;
            G.da = shared ? nullptr : (void*)(daT + h * slotA);
            G.dacc = shared ? dacc + (nV + h) * slotD : nullptr;
            G.H = P.W; G.W = P.H; G.asc = d == kLR;
            ++h;
        }
        lanes = std::max(lanes, G.W);
        ++k;
    }
    if ((e = genv_scans<T>(g, lanes, planes, P.D, shared, false, st, hsaved != nullptr)) != cudaSuccess) return e;
    for (long long b0 = 0; b0 < planes; b0 += 65535) {   // grid z is limited to 65535
        const long long nb = std::min<long long>(65535, planes - b0);
        const size_t off = (size_t)b0 * P.HW;
        auto slot = [&](float* base, int i) -> const float* { return base + (size_t)i * P.U + off; };
        const dim3 fg((unsigned)((P.W + kTT - 1) / kTT), (unsigned)((P.H + kTT - 1) / kTT), (unsigned)nb);
        if (P.per_dir) {
            GenvFinalPD f{};
            f.D = P.D;
            f.U = (long long)P.U;
            for (int i = 0; i < P.D; ++i) {
                f.hs[i] = slot(hs, i);
                f.dz[i] = slot(dz, i);
                f.vert[i] = i < nV;
            }
            launch_begin(st);
            k_genv_final_pd<T><<<fg, 256, 0, st>>>(f, (const T*)x + off, (const T*)lam + off, (const T*)dy + off,
                                                   (T*)dx + off, (T*)dlam + off, (T*)du + off, P.H, P.W);
            launch_end(st);
            if ((e = cudaGetLastError()) != cudaSuccess) return e;
            continue;
        }
        GenvFinal f{};
        if (nV > 0) { f.accV0 = slot(hs, 0); f.dzV0 = slot(dz, 0); }
        if (nV > 1) { f.accV1 = slot(hs, 1); f.dzV1 = slot(dz, 1); }
        if (nH > 0) { f.accH0 = slot(hs, nV); f.dzH0 = slot(dz, nV); }
        if (nH > 1) { f.accH1 = slot(hs, nV + 1); f.dzH1 = slot(dz, nV + 1); }
        launch_begin(st);
        k_genv_final<T><<<fg, 256, 0, st>>>(f, (const T*)x + off, (const T*)lam + off, (const T*)dy + off,
                                            (T*)dx + off, (T*)dlam + off, (T*)du + off, P.H, P.W);
        launch_end(st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
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

// Backward with lam and u shared by the directions. The vertical directions scan the image-layout
// buffers; the horizontal ones scan transposed copies of x, lam, u, dy and of their logit slots
// (left->right is then top->bottom of the transpose, right->left bottom->top), so every scan reads
// and writes whole rows. Their sums over directions and their logit gradients are transposed back.
// Forward with per-direction lambda / u on lines of at most kGenvMaxLanes lanes: the recompute
// kernel of the backward (all directions of all planes in one launch, horizontal directions on
// transposed x and lambda_d) writes h per direction, and k_genv_y forms y.
// (Measured on the shared-lambda workloads, this path is slower than the plane and sweep
// forwards: training 1.12 against 0.81 ms, classifier 2.04 against 1.28 ms, highres 4.34 against
// 1.87 ms; it serves the per-direction mode, which those families do not run on large maps.)
bool genv_fwd_ok(const Problem& P) { return P.per_dir && genv_ok(P); }

template <typename T>
cudaError_t gen_forward_cc(const Problem& P, const void* x, const void* a, const void* lam, const void* u, void* y,
                           void* ws, cudaStream_t st) {
    const int nV = n_vert(P), nH = n_horz(P);
    const long long slotA = (long long)P.N * P.Cw * 3 * P.HW;
    const long long planes = (long long)P.N * P.C;
    WsCarver wc(ws);
    float* hs = wc.take<float>((size_t)P.D * P.U);
    T* aT = nullptr;
    float* zT = nullptr;                   // z = lam x of the horizontal scans, transposed
    const int nlu = P.per_dir ? nH : 1;   // lambda planes sets the horizontal scans read
    if (nH > 0) {
        zT = wc.take<float>((size_t)nlu * P.U);
        aT = wc.take<T>((size_t)nH * slotA);
    }
    cudaError_t e;
    if (nH > 0) {
        const size_t lu0 = P.per_dir ? (size_t)nV * P.U : 0;
        if ((e = launch_transpose_mul<T>((const T*)lam + lu0, (const T*)x, zT, nlu * planes, planes, P.H, P.W, st)) !=
            cudaSuccess)
            return e;
        if ((e = launch_transpose<T, T, false>((const T*)a + nV * slotA, aT, (long long)nH * P.N * P.Cw * 3, P.H,
                                               P.W, st)) != cudaSuccess)
            return e;
    }
    GenvArgs g{};
    g.N = P.N;
    g.C = P.C;
    g.Cw = P.Cw;
    g.chunk = P.chunk;
    int v = 0, h = 0, k = 0, lanes = 0;
    for (unsigned d = kTB; d <= kRL; d <<= 1) {
        if (!(P.mask & d)) continue;
        GenvDir& G = g.d[k];
        G.hs = hs + (size_t)k * P.U;
        if (is_vertical(d)) {
            G.x = x;
            G.lam = (const T*)lam + (P.per_dir ? (size_t)v * P.U : 0);
            G.a = (const T*)a + v * slotA;
            G.H = P.H; G.W = P.W; G.asc = d == kTB;
            ++v;
        } else {
            G.x = x;      // not read: the scan takes z
            G.lam = lam;
            G.zp = zT + (P.per_dir ? (size_t)h * P.U : 0);
            G.a = aT + h * slotA;
            G.H = P.W; G.W = P.H; G.asc = d == kLR;
            ++h;
        }
        lanes = std::max(lanes, G.W);
        ++k;
    }
    if ((e = genv_scans<T>(g, lanes, planes, P.D, false, true, st)) != cudaSuccess) return e;
    for (long long b0 = 0; b0 < planes; b0 += 65535) {   // grid z is limited to 65535
        const long long nb = std::min<long long>(65535, planes - b0);
        const size_t off = (size_t)b0 * P.HW;
        GenvFinalPD f{};
        f.D = P.D;
        f.U = (long long)P.U;
        for (int i = 0; i < P.D; ++i) {
            f.hs[i] = hs + (size_t)i * P.U + off;
            f.vert[i] = i < nV;
        }
        const dim3 fg((unsigned)((P.W + kTT - 1) / kTT), (unsigned)((P.H + kTT - 1) / kTT), (unsigned)nb);
        launch_begin(st);
        k_genv_y<T><<<fg, 256, 0, st>>>(f, (const T*)u + off, (T*)y + off, P.H, P.W, P.per_dir);
        launch_end(st);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

template <typename T>
cudaError_t gen_backward_t(const Problem& P, const void* x, const void* a, const void* lam, const void* u,
                           const void* dy, void* dx, void* da, void* dlam, void* du, void* ws, cudaStream_t st) {
    if (genv_ok(P)) return gen_backward_cc<T>(P, x, a, lam, u, dy, dx, da, dlam, du, ws, st);
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

// The all-directions-at-once backward applies (lines of at most 1024 lanes): faster than the plane
// family's backward on small maps as well (measured: training 64 x 64 fp32 2.36 ms against 4.60 ms,
// classifier 56 x 56 bf16 4.12 ms against 5.70 ms), so AUTO prefers it for the backward.
bool generic_fast_backward(const Problem& p) { return genv_ok(p) && generic_supports(p, true); }

bool generic_supports(const Problem& p, bool bwd) {
    const int M = std::max(p.H, p.W);
    return M <= (bwd ? kGenBwdMaxLanes : kGenFwdMaxLanes);
}

size_t generic_ws_bytes(const Problem& p, bool bwd) {
    size_t b = 256;
    if (!bwd) {
        if (genv_fwd_ok(p)) {   // the layout gen_forward_cc carves
            const int nh = ((p.mask & kLR) ? 1 : 0) + ((p.mask & kRL) ? 1 : 0);
            const size_t es = p.esize();
            b += align256((size_t)p.D * p.U * sizeof(float));
            if (nh > 0)
                b += align256((size_t)(p.per_dir ? nh : 1) * p.U * sizeof(float)) +
                     align256((size_t)nh * p.N * p.Cw * 3 * p.HW * es);
            return b;
        }
        if (p.D > 1) b += align256(p.U * sizeof(float));
        return b;
    }
    const int nh = ((p.mask & kLR) ? 1 : 0) + ((p.mask & kRL) ? 1 : 0);
    if (genv_ok(p)) {   // the layout gen_backward_cc carves
        const size_t es = p.esize();
        const size_t slot_a = (size_t)p.N * p.Cw * 3 * p.HW, slot_d = (size_t)p.N * 3 * p.HW;
        b += 2 * align256((size_t)p.D * p.U * sizeof(float));
        if (p.wmode == GSPN_W_SHARED) b += align256((size_t)p.D * slot_d * sizeof(unsigned long long));
        if (nh > 0) {
            const size_t nlu = p.per_dir ? nh : 1;
            b += 2 * align256(nlu * p.U * sizeof(float)) + align256(nh * slot_a * es);
            if (p.wmode != GSPN_W_SHARED) b += align256(nh * slot_a * es);
        }
        return b;
    }
    b += 3 * align256(p.U * sizeof(float));
    if (p.wmode == GSPN_W_SHARED) b += align256(p.A * sizeof(unsigned long long));
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
    if (genv_fwd_ok(p))
        return p.dtype == GSPN_F32 ? gen_forward_cc<float>(p, x, a, lam, u, y, ws, st)
                                   : gen_forward_cc<__nv_bfloat16>(p, x, a, lam, u, y, ws, st);
    if (p.dtype == GSPN_F32) return gen_forward_t<float>(p, x, a, lam, u, y, ws, st);
    return gen_forward_t<__nv_bfloat16>(p, x, a, lam, u, y, ws, st);
}

cudaError_t generic_backward_saved(const Problem& p, const void* x, const void* a, const void* lam, const void* u,
                                   const void* dy, const float* hsaved, void* dx, void* da, void* dlam, void* du,
                                   void* ws, cudaStream_t st) {
    if (!genv_ok(p)) return cudaErrorNotSupported;
    if (p.dtype == GSPN_F32)
        return gen_backward_cc<float>(p, x, a, lam, u, dy, dx, da, dlam, du, ws, st, hsaved);
    return gen_backward_cc<__nv_bfloat16>(p, x, a, lam, u, dy, dx, da, dlam, du, ws, st, hsaved);
}

cudaError_t generic_backward(const Problem& p, const void* x, const void* a, const void* lam, const void* u,
                             const void* dy, void* dx, void* da, void* dlam, void* du, void* ws, cudaStream_t st) {
    if (p.dtype == GSPN_F32) return gen_backward_t<float>(p, x, a, lam, u, dy, dx, da, dlam, du, ws, st);
    return gen_backward_t<__nv_bfloat16>(p, x, a, lam, u, dy, dx, da, dlam, du, ws, st);
}

}  // namespace gspn
