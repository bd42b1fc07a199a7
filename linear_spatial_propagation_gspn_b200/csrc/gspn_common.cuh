// gspn_common.cuh -- device helpers shared by the libgspn kernels (sm_100a).
//
// Weight formation follows "Parallel Sequence Modeling via Generalized Spatial Propagation
// Network" (summary), section "Approach": sigmoid of the three neighbour logits, then division
// by their sum over the neighbours that lie inside the line, so each row of the tridiagonal
// propagation matrix sums to one.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

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

// ------------------------------------------------------------------ weights
// Normalised weights (w0, w1, w2) of one hidden lane from its logits. has_l / has_r tell
// whether lanes j-1 / j+1 exist. With p_k = 1 + exp(-a_k) (so sigmoid = 1/p_k), multiplying
// numerator and denominator by p0 p1 p2 gives w0 = p1 p2 / D, w1 = p0 p2 / D, w2 = p0 p1 / D
// with D = p1 p2 + p0 p2 + p0 p1: three exponentials and one reciprocal per lane. The
// products stay finite while every in-range logit is >= -40; below that the weights are
// formed from log-sigmoids shifted by their maximum, which is finite for every finite logit.
static __device__ __noinline__ void weights_slow(float a0, float a1, float a2, bool has_l, bool has_r,
                                          float& w0, float& w1, float& w2) {
    // log sigmoid(a) = -softplus(-a) = -(max(-a, 0) + log1p(exp(-|a|)))
    auto logsig = [](float a) { return -(fmaxf(-a, 0.f) + log1pf(expf(-fabsf(a)))); };
    float l0 = has_l ? logsig(a0) : -INFINITY;
    float l1 = logsig(a1);
    float l2 = has_r ? logsig(a2) : -INFINITY;
    float m = fmaxf(l1, fmaxf(l0, l2));
    float e0 = has_l ? expf(l0 - m) : 0.f;
    float e1 = expf(l1 - m);
    float e2 = has_r ? expf(l2 - m) : 0.f;
    float inv = 1.0f / (e0 + e1 + e2);
    w0 = e0 * inv;
    w1 = e1 * inv;
    w2 = e2 * inv;
}

__device__ __forceinline__ void lane_weights(float a0, float a1, float a2, bool has_l, bool has_r,
                                             float& w0, float& w1, float& w2) {
    float amin = fminf(a1, fminf(has_l ? a0 : a1, has_r ? a2 : a1));
    if (amin < -40.f) {
        weights_slow(a0, a1, a2, has_l, has_r, w0, w1, w2);
        return;
    }
    float p0 = 1.f + expf(-a0);
    float p1 = 1.f + expf(-a1);
    float p2 = 1.f + expf(-a2);
    if (has_l && has_r) {
        float q0 = p1 * p2, q1 = p0 * p2, q2 = p0 * p1;
        float inv = __frcp_rn(q0 + q1 + q2);
        w0 = q0 * inv;
        w1 = q1 * inv;
        w2 = q2 * inv;
    } else if (has_r) {          // lane 0: neighbours k = 1, 2
        float inv = __frcp_rn(p1 + p2);
        w0 = 0.f;
        w1 = p2 * inv;
        w2 = p1 * inv;
    } else if (has_l) {          // last lane: neighbours k = 0, 1
        float inv = __frcp_rn(p0 + p1);
        w0 = p1 * inv;
        w1 = p0 * inv;
        w2 = 0.f;
    } else {                     // single lane
        w0 = 0.f;
        w1 = 1.f;
        w2 = 0.f;
    }
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
