// gspn_common.cuh -- device helpers shared by the libgspn kernels (sm_100a).
//
// Weight formation follows "Parallel Sequence Modeling via Generalized Spatial Propagation
// Network" (summary), section "Approach": sigmoid of the three neighbour logits, then division
// by their sum over the neighbours that lie inside the line, so each row of the tridiagonal
// propagation matrix sums to one.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>

#include "gspn.h"

namespace gspn {

// ------------------------------------------------------------------ storage dtypes
template <typename T> struct Io;
template <> struct Io<float> {
    static __device__ __forceinline__ float ld(const float* p) { return *p; }
    static __device__ __forceinline__ void st(float* p, float v) { *p = v; }
};
template <> struct Io<__nv_bfloat16> {
    static __device__ __forceinline__ float ld(const __nv_bfloat16* p) { return __bfloat162float(*p); }
    static __device__ __forceinline__ void st(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }
};

template <> struct Io<__half> {
    static __device__ __forceinline__ float ld(const __half* p) { return __half2float(*p); }
    static __device__ __forceinline__ void st(__half* p, float v) { *p = __float2half_rn(v); }
};

// ------------------------------------------------------------------ vector lanes
// Two 16-bit values (bf16 or fp16) packed in a word, to and from floats (round to nearest even).
template <typename T> __device__ __forceinline__ float2 unpack2(uint32_t w);
template <> __device__ __forceinline__ float2 unpack2<__nv_bfloat16>(uint32_t w) {
    return __bfloat1622float2(*(const __nv_bfloat162*)&w);
}
template <> __device__ __forceinline__ float2 unpack2<__half>(uint32_t w) { return __half22float2(*(const __half2*)&w); }
template <typename T> __device__ __forceinline__ uint32_t pack2(float a, float b);
template <> __device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float a, float b) {
    const __nv_bfloat162 q = __floats2bfloat162_rn(a, b);
    return *(const uint32_t*)&q;
}
template <> __device__ __forceinline__ uint32_t pack2<__half>(float a, float b) {
    const __half2 q = __floats2half2_rn(a, b);
    return *(const uint32_t*)&q;
}

// L consecutive lanes of storage type T (float, bf16 or fp16; aligned to L elements).
template <typename T, int L>
__device__ __forceinline__ void ld_lanes(const void* ptr, float (&v)[L]) {
    if constexpr (std::is_same<T, float>::value) {
        if constexpr (L == 1) {
            v[0] = *(const float*)ptr;
        } else if constexpr (L == 2) {
            const float2 q = *(const float2*)ptr;
            v[0] = q.x; v[1] = q.y;
        } else if constexpr (L == 4) {
            const float4 q = *(const float4*)ptr;
            v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
        } else {
            const float4 q0 = *(const float4*)ptr, q1 = *((const float4*)ptr + 1);
            v[0] = q0.x; v[1] = q0.y; v[2] = q0.z; v[3] = q0.w;
            v[4] = q1.x; v[5] = q1.y; v[6] = q1.z; v[7] = q1.w;
        }
    } else {
        if constexpr (L == 1) {
            v[0] = Io<T>::ld((const T*)ptr);
        } else if constexpr (L == 2) {
            const float2 f = unpack2<T>(*(const uint32_t*)ptr);
            v[0] = f.x; v[1] = f.y;
        } else if constexpr (L == 4) {
            const uint2 q = *(const uint2*)ptr;
            const float2 f0 = unpack2<T>(q.x), f1 = unpack2<T>(q.y);
            v[0] = f0.x; v[1] = f0.y; v[2] = f1.x; v[3] = f1.y;
        } else {
            const uint4 q = *(const uint4*)ptr;
            const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float2 f = unpack2<T>(w[k]);
                v[2 * k] = f.x;
                v[2 * k + 1] = f.y;
            }
        }
    }
}

template <typename T, int L>
__device__ __forceinline__ void st_lanes(void* ptr, const float (&v)[L]) {
    if constexpr (std::is_same<T, float>::value) {
        if constexpr (L == 1) *(float*)ptr = v[0];
        else if constexpr (L == 2) *(float2*)ptr = make_float2(v[0], v[1]);
        else if constexpr (L == 4) *(float4*)ptr = make_float4(v[0], v[1], v[2], v[3]);
        else {
            *(float4*)ptr = make_float4(v[0], v[1], v[2], v[3]);
            *((float4*)ptr + 1) = make_float4(v[4], v[5], v[6], v[7]);
        }
    } else {
        if constexpr (L == 1) {
            Io<T>::st((T*)ptr, v[0]);
        } else if constexpr (L == 2) {
            *(uint32_t*)ptr = pack2<T>(v[0], v[1]);
        } else if constexpr (L == 4) {
            *(uint2*)ptr = make_uint2(pack2<T>(v[0], v[1]), pack2<T>(v[2], v[3]));
        } else {
            *(uint4*)ptr = make_uint4(pack2<T>(v[0], v[1]), pack2<T>(v[2], v[3]), pack2<T>(v[4], v[5]),
                                      pack2<T>(v[6], v[7]));
        }
    }
}

// ------------------------------------------------------------------ geometry
// Directions as bit masks, slot order TB, BT, LR, RL.
constexpr unsigned kTB = 1u, kBT = 2u, kLR = 4u, kRL = 8u;

__host__ __device__ __forceinline__ bool is_vertical(unsigned d) { return d == kTB || d == kBT; }

// Image offset (r * W + c) of scan position (i, j) of direction d.
__host__ __device__ __forceinline__ long long scan_pixel(unsigned d, int H, int W, int i, int j) {
    int r, c;
    if (d == kTB)      { r = i;         c = j; }
    else if (d == kBT) { r = H - 1 - i; c = j; }
    else if (d == kLR) { r = j;         c = i; }
    else               { r = j;         c = W - 1 - i; }
    return (long long)r * W + c;
}

// Slot of direction d among the directions set in mask (order TB, BT, LR, RL).
__host__ __device__ __forceinline__ int dir_slot(unsigned mask, unsigned d) {
    int s = 0;
    for (unsigned b = 1u; b < d; b <<= 1) s += (mask & b) ? 1 : 0;
    return s;
}

// ------------------------------------------------------------------ local (chunked) scans
// Local propagation restarts a scan from h = 0 at the first line, in scan order, of every chunk
// of `chunk` image lines along the scan axis (chunks aligned to image line 0; 0 = global). In
// scan coordinates with L steps an ascending scan (TB, LR) restarts at i % chunk == 0 and a
// descending one (BT, RL) at i == 0 and wherever (L - i) % chunk == 0 (the step whose image line
// is the last of its chunk).
__host__ __device__ __forceinline__ bool chunk_start(bool asc, int L, int chunk, int i) {
    if (i == 0) return true;
    if (chunk <= 0) return false;
    return asc ? (i % chunk == 0) : ((L - i) % chunk == 0);
}
// Steps in a scan's first chunk; every later chunk has `chunk` steps (the last may be short).
// Scan loops count down from it instead of dividing every step. Global: L.
__host__ __device__ __forceinline__ int first_chunk_len(bool asc, int L, int chunk) {
    if (chunk <= 0 || chunk >= L) return L;
    return asc ? chunk : ((L - 1) % chunk) + 1;
}
__host__ __device__ __forceinline__ bool scan_ascending(unsigned d) { return d == kTB || d == kLR; }

// ------------------------------------------------------------------ weights
// Normalised weights (w0, w1, w2) of one hidden lane from its logits. has_l / has_r tell
// whether lanes j-1 / j+1 exist. With p_k = 1 + exp(-a_k) (so sigmoid = 1/p_k), multiplying
// numerator and denominator by p0 p1 p2 gives w0 = p1 p2 / D, w1 = p0 p2 / D, w2 = p0 p1 / D
// with D = p1 p2 + p0 p2 + p0 p1: three exponentials and one reciprocal per lane. The
// products stay finite while every in-range logit is >= -40; below that the weights are
// formed from log-sigmoids shifted by their maximum, which is finite for every finite logit.
// Everything here is inline and returns by value, so no weight ever touches local memory.
struct Wts {
    float w0, w1, w2;
};

constexpr float kShiftBelow = -40.f;

// True when some in-range logit is below kShiftBelow (then the shifted form must be used).
__device__ __forceinline__ bool weights_need_shift(float a0, float a1, float a2, bool has_l, bool has_r) {
    const float amin = fminf(a1, fminf(has_l ? a0 : a1, has_r ? a2 : a1));
    return amin < kShiftBelow;
}

// log sigmoid(a) = -softplus(-a) = -(max(-a, 0) + log1p(exp(-|a|))); weights = exp(l_k - max l).
__device__ __forceinline__ Wts weights_shifted(float a0, float a1, float a2, bool has_l, bool has_r) {
    auto logsig = [](float a) { return -(fmaxf(-a, 0.f) + log1pf(expf(-fabsf(a)))); };
    const float l0 = has_l ? logsig(a0) : -INFINITY;
    const float l1 = logsig(a1);
    const float l2 = has_r ? logsig(a2) : -INFINITY;
    const float m = fmaxf(l1, fmaxf(l0, l2));
    const float e0 = has_l ? expf(l0 - m) : 0.f;
    const float e1 = expf(l1 - m);
    const float e2 = has_r ? expf(l2 - m) : 0.f;
    const float inv = 1.0f / (e0 + e1 + e2);
    return Wts{e0 * inv, e1 * inv, e2 * inv};
}

// Common-denominator numerators with the out-of-range terms removed (branch-free in edge lanes):
// interior q = (p1 p2, p0 p2, p0 p1); no left (0, p2, p1); no right (p1, p0, 0); single (0, 1, 0).
__device__ __forceinline__ Wts weights_from_p(float p0, float p1, float p2, bool has_l, bool has_r) {
    const float l = has_l ? p0 : 1.f;
    const float r = has_r ? p2 : 1.f;
    return Wts{has_l ? p1 * r : 0.f, l * r, has_r ? p1 * l : 0.f};
}

// Accurate form (expf, IEEE reciprocal); used by the generic family and the backward.
__device__ __forceinline__ Wts lane_weights_acc(float a0, float a1, float a2, bool has_l, bool has_r) {
    if (weights_need_shift(a0, a1, a2, has_l, has_r)) return weights_shifted(a0, a1, a2, has_l, has_r);
    const Wts q = weights_from_p(1.f + expf(-a0), 1.f + expf(-a1), 1.f + expf(-a2), has_l, has_r);
    const float inv = __frcp_rn(q.w0 + q.w1 + q.w2);
    return Wts{q.w0 * inv, q.w1 * inv, q.w2 * inv};
}

__device__ __forceinline__ void lane_weights(float a0, float a1, float a2, bool has_l, bool has_r,
                                             float& w0, float& w1, float& w2) {
    const Wts w = lane_weights_acc(a0, a1, a2, has_l, has_r);
    w0 = w.w0;
    w1 = w.w1;
    w2 = w.w2;
}

// Fast form from the MUFU approximations (__expf: relative error about 2 ulp plus the rounding
// of the scaled argument; __fdividef: about 2 ulp). The normalisation is applied after the
// approximations, so every row still sums to one up to a few ulp and the small weight errors do
// not compound along the scan. Branch-free: the arguments are clamped at kShiftBelow so the
// products never overflow; a caller must redo lanes for which weights_need_shift() holds with
// weights_shifted() (kernels do that behind one warp vote per step, the path is rare).
__device__ __forceinline__ Wts lane_weights_fast_nocheck(float a0, float a1, float a2, bool has_l, bool has_r) {
    const float p0 = 1.f + __expf(-fmaxf(a0, kShiftBelow));
    const float p1 = 1.f + __expf(-fmaxf(a1, kShiftBelow));
    const float p2 = 1.f + __expf(-fmaxf(a2, kShiftBelow));
    const Wts q = weights_from_p(p0, p1, p2, has_l, has_r);
    const float inv = __fdividef(1.f, q.w0 + q.w1 + q.w2);
    return Wts{q.w0 * inv, q.w1 * inv, q.w2 * inv};
}

// Weights and Jacobian factors of one lane for the backward:
// da_k = s_k (1 - s_k) (dw_k - sum_k' w_k' dw_k') / S = g_k (dw_k - sum_k' w_k' dw_k').
struct LaneJac {
    float w0, w1, w2;     // normalised weights
    float g0, g1, g2;     // s_k (1 - s_k) / S  (0 out of range)
};

__device__ __forceinline__ float sigmoidf_(float a) { return 1.0f / (1.0f + expf(-a)); }

__device__ __forceinline__ LaneJac lane_jacobian(float a0, float a1, float a2, bool has_l, bool has_r) {
    LaneJac J;
    lane_weights(a0, a1, a2, has_l, has_r, J.w0, J.w1, J.w2);
    // s_k / S = w_k, so s_k (1 - s_k) / S = w_k (1 - s_k) = w_k sigmoid(-a_k).
    J.g0 = has_l ? J.w0 * sigmoidf_(-a0) : 0.f;
    J.g1 = J.w1 * sigmoidf_(-a1);
    J.g2 = has_r ? J.w2 * sigmoidf_(-a2) : 0.f;
    return J;
}

// Fast forms for the scans whose step cost is instruction issue (the generic family): MUFU
// exponentials and divisions (relative error a few ulp, normalised after the approximations) when
// every in-range logit is >= kShiftBelow, else the accurate shifted form. Out-of-range logits are
// clamped before the exponential so that they cannot produce inf * 0.
__device__ __forceinline__ Wts lane_weights_fast(float a0, float a1, float a2, bool has_l, bool has_r) {
    if (weights_need_shift(a0, a1, a2, has_l, has_r)) return weights_shifted(a0, a1, a2, has_l, has_r);
    return lane_weights_fast_nocheck(a0, a1, a2, has_l, has_r);
}
__device__ __forceinline__ LaneJac lane_jacobian_fast(float a0, float a1, float a2, bool has_l, bool has_r) {
    if (weights_need_shift(a0, a1, a2, has_l, has_r)) return lane_jacobian(a0, a1, a2, has_l, has_r);
    const float e0 = __expf(-fmaxf(a0, kShiftBelow));
    const float e1 = __expf(-fmaxf(a1, kShiftBelow));
    const float e2 = __expf(-fmaxf(a2, kShiftBelow));
    const float p0 = 1.f + e0, p1 = 1.f + e1, p2 = 1.f + e2;
    const Wts q = weights_from_p(p0, p1, p2, has_l, has_r);
    const float inv = __fdividef(1.f, q.w0 + q.w1 + q.w2);
    LaneJac J;
    J.w0 = q.w0 * inv;
    J.w1 = q.w1 * inv;
    J.w2 = q.w2 * inv;
    // s_k (1 - s_k) / S = w_k sigmoid(-a_k) = w_k e_k / p_k (0 out of range, where w_k = 0)
    J.g0 = J.w0 * __fdividef(e0, p0);
    J.g1 = J.w1 * __fdividef(e1, p1);
    J.g2 = J.w2 * __fdividef(e2, p2);
    return J;
}

// ------------------------------------------------------------------ status word and waits
// Workspace bytes [0, 256) hold the device status; kernels only ever OR bits into word 0.
constexpr size_t kStatusBytes = 256;
constexpr unsigned kDevTimeout = 1u;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void report_timeout(unsigned* status) {
    if (status) atomicOr(status, kDevTimeout);
}

// Bounded wait on a global flag becoming non-zero. Returns false (and records a timeout)
// after limit_ns nanoseconds.
__device__ __forceinline__ bool wait_flag_bounded(const volatile unsigned* flag, unsigned long long limit_ns,
                                                  unsigned* status) {
    unsigned long long t0 = globaltimer_ns();
    while (*flag == 0u) {
        if (globaltimer_ns() - t0 > limit_ns) {
            report_timeout(status);
            return false;
        }
        __nanosleep(256);
    }
    return true;
}

}  // namespace gspn
