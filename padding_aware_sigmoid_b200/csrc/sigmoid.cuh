// In-register evaluation of sigma(x) = 1 / (1 + e^-x) and sigma'(x) for the
// bf16 kernels, two scores at a time so that the FMA work issues as packed
// f32x2 instructions.  Two modes:
//
//  TANH: sigma(x) = 0.5 tanh(x / 2) + 0.5 with the hardware tanh.approx.f32,
//        the form the kernel pages describe (paper.rainbus.top summary,
//        method step (3)).  One MUFU op per score.  Near sigma -> 0 the sum
//        0.5 + 0.5 t cancels, so its relative accuracy in the left tail is
//        bounded by the absolute accuracy of tanh.approx near -1.
//
//  EXP:  u = e^-|x| with the hardware ex2.approx.ftz.f32 (one MUFU op), then
//        g = 1 / (1 + u) for u in (0, 1] by a degree-4 polynomial, and
//        sigma = g for x >= 0, u g for x < 0.  The polynomial is the minimax
//        fit of 1/(1+u) on [0, 1] in relative error, fitted for this library
//        by iteratively reweighted least squares; its maximum relative error
//        is 3.4e-4 (bf16 rounding of P is 2^-9 = 2.0e-3) and its sign
//        alternates across the interval.  Nothing cancels in either tail.
//        sigma'(x) = sigma(x) sigma(-x) = u g^2 for either sign of x.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace sigattn {

enum SigmoidMode : int { kSigmoidTanh = 0, kSigmoidExp = 1 };

__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// minimax coefficients of 1/(1+u) on [0, 1], lowest degree first
constexpr float kG0 = 0.999782274f;
constexpr float kG1 = -0.986068382f;
constexpr float kG2 = 0.870132568f;
constexpr float kG3 = -0.537934966f;
constexpr float kG4 = 0.154207251f;

constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

// 1/(1+u) for u in [0, 1], on a pair
__device__ __forceinline__ float2 recip1p2(float2 u) {
    float2 g = fma2(u, f2(kG4, kG4), f2(kG3, kG3));
    g = fma2(g, u, f2(kG2, kG2));
    g = fma2(g, u, f2(kG1, kG1));
    return fma2(g, u, f2(kG0, kG0));
}

// Coefficients that turn a raw score s = q.k into the argument each mode
// needs, so that the per-score cost before the MUFU op is one (packed) FMA.
struct SigmoidCoef {
    float a, c;  // TANH: y = a s + c = (alpha s + b) / 2;  EXP: y = (alpha s + b) log2 e
};

template <int MODE>
__host__ __device__ __forceinline__ SigmoidCoef make_coef(float alpha, float bias) {
    if (MODE == kSigmoidTanh) return SigmoidCoef{0.5f * alpha, 0.5f * bias};
    return SigmoidCoef{alpha * kLog2e, bias * kLog2e};
}

__device__ __forceinline__ float2 scale2(float s0, float s1, const SigmoidCoef &cf) {
    return fma2(f2(s0, s1), f2(cf.a, cf.a), f2(cf.c, cf.c));
}

// sigma of two pre-scaled arguments (see SigmoidCoef).
template <int MODE>
__device__ __forceinline__ float2 sigma2(float2 y) {
    if (MODE == kSigmoidTanh) {
        const float2 t = f2(tanh_approx(y.x), tanh_approx(y.y));
        return fma2(t, f2(0.5f, 0.5f), f2(0.5f, 0.5f));
    } else {
        const float2 u = f2(ex2_approx(-fabsf(y.x)), ex2_approx(-fabsf(y.y)));
        const float2 g = recip1p2(u);
        const float2 m = f2(y.x >= 0.0f ? 1.0f : u.x, y.y >= 0.0f ? 1.0f : u.y);
        return mul2(g, m);
    }
}

// sigma and sigma' of two pre-scaled arguments.
template <int MODE>
__device__ __forceinline__ void sigma_grad2(float2 y, float2 &p, float2 &dp) {
    if (MODE == kSigmoidTanh) {
        const float2 t = f2(tanh_approx(y.x), tanh_approx(y.y));
        p = fma2(t, f2(0.5f, 0.5f), f2(0.5f, 0.5f));
        // (1 - t^2) / 4
        dp = fma2(mul2(t, f2(-0.25f, -0.25f)), t, f2(0.25f, 0.25f));
    } else {
        const float2 u = f2(ex2_approx(-fabsf(y.x)), ex2_approx(-fabsf(y.y)));
        const float2 g = recip1p2(u);
        const float2 ug = mul2(u, g);
        p = f2(y.x >= 0.0f ? g.x : ug.x, y.y >= 0.0f ? g.y : ug.y);
        dp = mul2(ug, g);
    }
}

}  // namespace sigattn
