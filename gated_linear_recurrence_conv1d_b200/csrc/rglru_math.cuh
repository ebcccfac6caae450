// rglru_math.cuh -- element-wise arithmetic of the tensor-core kernels (sm_100a).
//
// One definition of the gate / decay / input-normalisation / GeLU steps shared by the fused
// prefill, the decode step and the persistent decode, in scalar and packed-fp32x2 forms.  It
// follows "Griffin Guide: RecurrentGemma, RG-LRU & Hybrid Attention", "1. Formulation of the
// RG-LRU Gating Mechanism":
//
//   r_t = sigma(W_a x_t + b_a), i_t = sigma(W_x x_t + b_x), log a_t = c r_t log sigma(Lambda),
//   u_t = sqrt(1 - a_t^2) (i_t x_t),
//
// with these choices, each exact to a few fp32 ulps (no hardware tanh):
//
//   * sigma(v) = 1 / (1 + 2^(-v log2 e)): one ex2 and one reciprocal; the gate bias enters as
//     the addend of the FMA that scales the contraction by -log2 e (nb = -b log2 e);
//   * a_t = 1 + E with E = expm1(K r_t), K = c log sigma(Lambda) <= 0: the series to l^5 when
//     K >= -1/8 (|l| <= 1/8, relative error below 6e-9, and no cancellation in 1 - a^2 near
//     a = 1), else ex2(l log2 e) - 1;
//   * 1 - a_t^2 = -E (2 + E);  sqrt(1 - a^2) i_t = q rsqrt(q (1 + e_x)^2) with q = 1 - a^2 and
//     e_x = 2^(-v_x log2 e): one reciprocal square root for both the square root and the
//     division of the input gate (q clamped below at 1e-30 inside the rsqrt);
//   * GeLU, erf form: y Phi(y) = max(y, 0) - s exp(-s^2/2) R(s), s = |y|, with R a degree-10
//     polynomial fitted to Q(s) exp(s^2/2) on [0, 5.5] (Q the normal upper tail; the fit is
//     printed by gelu_tail_fit.py beside this file; |GeLU error| < 2e-6); the constants below
//     are -R's coefficients;
//   * GeLU, tanh form: (y/2)(1 + tanh(k (y + 0.044715 y^3))) = y sigma(2 k (y + 0.044715 y^3)).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "sm100.cuh"

namespace rglru {
namespace fm {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kSqrt2OverPi = 0.79788456080286535588f;

// -R(s), R(s) = Q(s) exp(s^2 / 2) on [0, 5.5]
constexpr float kNR0 = -4.999885559e-01f;
constexpr float kNR1 = 3.986470401e-01f;
constexpr float kNR2 = -2.480954677e-01f;
constexpr float kNR3 = 1.275549978e-01f;
constexpr float kNR4 = -5.391246453e-02f;
constexpr float kNR5 = 1.802178286e-02f;
constexpr float kNR6 = -4.527380690e-03f;
constexpr float kNR7 = 8.083113353e-04f;
constexpr float kNR8 = -9.561613842e-05f;
constexpr float kNR9 = 6.667832167e-06f;
constexpr float kNR10 = -2.065398093e-07f;
constexpr float kGeluSMax = 5.5f;

__device__ __forceinline__ float ex2f(float x) { return sm100::ex2_approx(x); }
__device__ __forceinline__ float rcpf(float x) {
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ float rsqrtf_(float x) {
    float r;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// ---------------------------------------------------------------- packed fp32x2 -----------
__device__ __forceinline__ float2 f2(float v) { return make_float2(v, v); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 ex2_2(float2 v) { return make_float2(ex2f(v.x), ex2f(v.y)); }
__device__ __forceinline__ float2 rcp2(float2 v) { return make_float2(rcpf(v.x), rcpf(v.y)); }

// expm1(l) for -1/8 <= l <= 0 by its series to l^5
__device__ __forceinline__ float expm1_series(float l) {
    float p = fmaf(l, 1.0f / 720.0f, 1.0f / 120.0f);
    p = fmaf(l, p, 1.0f / 24.0f);
    p = fmaf(l, p, 1.0f / 6.0f);
    p = fmaf(l, p, 0.5f);
    p = fmaf(l, p, 1.0f);
    return l * p;
}
__device__ __forceinline__ float2 expm1_series2(float2 l) {
    float2 p = fma2(l, f2(1.0f / 720.0f), f2(1.0f / 120.0f));
    p = fma2(l, p, f2(1.0f / 24.0f));
    p = fma2(l, p, f2(1.0f / 6.0f));
    p = fma2(l, p, f2(0.5f));
    p = fma2(l, p, f2(1.0f));
    return mul2(l, p);
}
// any l <= 0
__device__ __forceinline__ float expm1_any(float l) {
    return l > -0.125f ? expm1_series(l) : ex2f(l * kLog2e) - 1.0f;
}

// a_t and u_t = sqrt(1 - a_t^2) i_t x_t from the bias-free gate contractions da, dx; nba, nbx =
// -b log2 e; K = c log sigma(Lambda); xc the fp32 conv output.  SERIES: K >= -1/8 is known.
template <bool SERIES>
__device__ __forceinline__ void gates1(float da, float dx, float nba, float nbx, float K, float xc, float& a,
                                       float& u) {
    const float ea = ex2f(fmaf(da, -kLog2e, nba));
    const float r = rcpf(1.0f + ea);
    const float l = r * K;
    const float em = SERIES ? expm1_series(l) : expm1_any(l);
    a = 1.0f + em;
    const float q = em * fmaf(em, -1.0f, -2.0f);
    const float ex = ex2f(fmaf(dx, -kLog2e, nbx));
    const float d = 1.0f + ex;
    const float s = fmaxf(q * (d * d), 1e-30f);
    u = (q * xc) * rsqrtf_(s);
}
template <bool SERIES>
__device__ __forceinline__ void gates2(float2 da, float2 dx, float2 nba, float2 nbx, float2 K, float2 xc, float2& a,
                                       float2& u) {
    const float2 ea = ex2_2(fma2(da, f2(-kLog2e), nba));
    const float2 r = rcp2(add2(ea, f2(1.0f)));
    const float2 l = mul2(r, K);
    float2 em;
    if constexpr (SERIES) em = expm1_series2(l);
    else em = make_float2(expm1_any(l.x), expm1_any(l.y));
    a = add2(em, f2(1.0f));
    const float2 q = mul2(em, fma2(em, f2(-1.0f), f2(-2.0f)));
    const float2 ex = ex2_2(fma2(dx, f2(-kLog2e), nbx));
    const float2 d = add2(ex, f2(1.0f));
    const float2 s = mul2(q, mul2(d, d));
    const float2 rs = make_float2(rsqrtf_(fmaxf(s.x, 1e-30f)), rsqrtf_(fmaxf(s.y, 1e-30f)));
    u = mul2(mul2(q, xc), rs);
}

// GeLU, erf form (see the header)
__device__ __forceinline__ float gelu_erf1(float y) {
    const float sc = fminf(fabsf(y), kGeluSMax);
    const float e = ex2f((y * y) * (-0.5f * kLog2e));
    float p = fmaf(kNR10, sc, kNR9);
    p = fmaf(p, sc, kNR8);
    p = fmaf(p, sc, kNR7);
    p = fmaf(p, sc, kNR6);
    p = fmaf(p, sc, kNR5);
    p = fmaf(p, sc, kNR4);
    p = fmaf(p, sc, kNR3);
    p = fmaf(p, sc, kNR2);
    p = fmaf(p, sc, kNR1);
    p = fmaf(p, sc, kNR0);
    return fmaf(sc * e, p, fmaxf(y, 0.0f));
}
__device__ __forceinline__ float2 gelu_erf2(float2 y) {
    const float2 sc = make_float2(fminf(fabsf(y.x), kGeluSMax), fminf(fabsf(y.y), kGeluSMax));
    const float2 e = ex2_2(mul2(mul2(y, y), f2(-0.5f * kLog2e)));
    float2 p = fma2(f2(kNR10), sc, f2(kNR9));
    p = fma2(p, sc, f2(kNR8));
    p = fma2(p, sc, f2(kNR7));
    p = fma2(p, sc, f2(kNR6));
    p = fma2(p, sc, f2(kNR5));
    p = fma2(p, sc, f2(kNR4));
    p = fma2(p, sc, f2(kNR3));
    p = fma2(p, sc, f2(kNR2));
    p = fma2(p, sc, f2(kNR1));
    p = fma2(p, sc, f2(kNR0));
    return fma2(mul2(sc, e), p, make_float2(fmaxf(y.x, 0.0f), fmaxf(y.y, 0.0f)));
}
// GeLU, tanh form
__device__ __forceinline__ float gelu_tanh1(float y) {
    const float c1 = -2.0f * kSqrt2OverPi * kLog2e, c3 = c1 * 0.044715f;
    const float e = ex2f(y * fmaf(y * y, c3, c1));
    return y * rcpf(1.0f + e);
}
__device__ __forceinline__ float2 gelu_tanh2(float2 y) {
    const float c1 = -2.0f * kSqrt2OverPi * kLog2e, c3 = c1 * 0.044715f;
    const float2 e = ex2_2(mul2(y, fma2(mul2(y, y), f2(c3), f2(c1))));
    return mul2(y, rcp2(add2(e, f2(1.0f))));
}
__device__ __forceinline__ float gelu1(float y, int tanh_form) { return tanh_form ? gelu_tanh1(y) : gelu_erf1(y); }

// Phi(v) to ~1e-7 without erfc, for the gradients: with s = |v| and e = exp(-v^2 / 2) (one exp2,
// returned too), the upper tail Q(s) = e R(s), R a degree-14 polynomial in t = (s - 2.75) / 2.75
// on s in [0, 5.5] (s clamped there; beyond it Q < 2e-8), fitted by gelu_tail_fit.py --precise
// beside this file (max |Phi error| 1.1e-7 in fp32); Phi(v) = 1 - Q for v >= 0, Q otherwise.
constexpr float kPhiR0 = 1.307247281e-01f;
constexpr float kPhiR1 = -1.084856018e-01f;
constexpr float kPhiR2 = 8.409250528e-02f;
constexpr float kPhiR3 = -6.148617715e-02f;
constexpr float kPhiR4 = 4.272365198e-02f;
constexpr float kPhiR5 = -2.843398601e-02f;
constexpr float kPhiR6 = 1.814154349e-02f;
constexpr float kPhiR7 = -1.083536446e-02f;
constexpr float kPhiR8 = 6.395316683e-03f;
constexpr float kPhiR9 = -4.469349980e-03f;
constexpr float kPhiR10 = 2.545840805e-03f;
constexpr float kPhiR11 = -3.012927773e-04f;
constexpr float kPhiR12 = 1.266671024e-04f;
constexpr float kPhiR13 = -8.168322383e-04f;
constexpr float kPhiR14 = 4.210809420e-04f;
__device__ __forceinline__ float phi_precise(float v, float& e) {
    e = ex2f((v * v) * (-0.5f * kLog2e));
    const float t = fmaf(fminf(fabsf(v), 5.5f), 1.0f / 2.75f, -1.0f);
    float r = kPhiR14;
    r = fmaf(r, t, kPhiR13);
    r = fmaf(r, t, kPhiR12);
    r = fmaf(r, t, kPhiR11);
    r = fmaf(r, t, kPhiR10);
    r = fmaf(r, t, kPhiR9);
    r = fmaf(r, t, kPhiR8);
    r = fmaf(r, t, kPhiR7);
    r = fmaf(r, t, kPhiR6);
    r = fmaf(r, t, kPhiR5);
    r = fmaf(r, t, kPhiR4);
    r = fmaf(r, t, kPhiR3);
    r = fmaf(r, t, kPhiR2);
    r = fmaf(r, t, kPhiR1);
    r = fmaf(r, t, kPhiR0);
    const float q = e * r;
    return v >= 0.f ? 1.0f - q : q;
}

}  // namespace fm
}  // namespace rglru
