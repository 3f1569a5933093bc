// screen.cuh -- exact candidate selection by screening and verification.
//
// The scale search must return exactly the candidate that the definition
// picks: the first candidate (ascending bit pattern / exponent) whose loss,
// accumulated in binary32 as
//   r = x*inv; q = E2M1(r); y = RN(q*d); e = RN(x - y); L = RN(L + RN(e*e))
// (WMSE: L = RN(L + RN(w*RN(e*e)))), is smallest.  Evaluating that loss for
// every candidate costs six FMA-pipe operations per element and candidate,
// which made the sweep arithmetic-bound.  Instead:
//
// 1. Screen.  For every candidate compute the loss in units of the step d:
//      et = RN(q - r)  (one mixed f16/f32 subtract, q exact in f16)
//      Lt = RN(Lt + et*et)  (fused)            WMSE: Lt = RN(Lt + RN(w*et)*et)
//    and lam = RN(v^2 * Lt), where d = RN(v*S) (NVFP4: v the E4M3 value of
//    the pattern, S the global scale; MXFP4: v = 2^(e-e0), S = 2^e0).  This is
//    three FMA-pipe operations per element and candidate.  It uses the same r
//    and q as the definition, so it differs from L/S^2 only by rounding.
// 2. Bound.  With u = 2^-24, alpha = ||x||/S (WMSE: sqrt(sum w x^2)/S) and
//    tau an absolute allowance for results that fall in the subnormal range,
//    the true loss l = L/S^2 of every candidate obeys
//      |l - lam| <= D(max(l, lam)),
//      D(z) = u*(K1*z + K2*alpha*sqrt(z)) + K3*u^2*alpha^2 + tau,
//    because (a) y, e and r carry one rounding each, so |e - (-d*et)| <=
//    u*(3|x| + 3|E|)*(1+2u) with E = x - q*d the exact error, which gives
//    |e^2 - d^2 et^2| <= 6u(|x||E| + E^2) + O(u^2) and, summed with
//    Cauchy-Schwarz, the alpha*sqrt(l) and l terms; (b) both 16-term
//    (32-term for MXFP4) sequential sums round at most n+2 times relative to
//    their terms; (c) d^2 = v^2 S^2 (1+delta)^2.  The constants K1 = 128,
//    K2 = 16, K3 = 64 are about twice what (a)-(c) need for 32-term blocks.
//    Let M = min lam (candidate w).  The winner's true loss is at most U, the
//    root of U = M + D(U), and a candidate k can only win if
//    lam_k - D(lam_k) <= U; using sqrt(z) <= (z/sqrt(U) + sqrt(U))/2 this holds
//    whenever lam_k <= T = (U + u*K2*alpha*sqrt(U)/2 + K3*u^2*alpha^2 + tau) /
//    (1 - u*K1 - u*K2*alpha/(2*sqrt(U))), so every candidate with lam_k > T is
//    excluded.  survivor_threshold evaluates an upper bound of T with
//    approximate square roots and reciprocals, each widened, and widens the
//    result by another 2^-10 relative, far more than their errors.
// 3. Verify.  The survivors (the screening minimum always survives; on
//    typical weights about 1.002 per block) are evaluated with the exact
//    definition in ascending order and the first minimum wins.  With a single
//    survivor that candidate is the winner and its exact loss comes out of
//    the emit stage, which computes q*d anyway for the reconstruction.
//
// Every excluded candidate has a true loss above the winner's, so the result
// is the definition's result bit for bit; the screening only saves work.
#pragma once

#include "device.cuh"

namespace fp4q {

constexpr float kU = 0x1p-24f;
constexpr float kK1 = 128.0f;
constexpr float kK2 = 16.0f;
constexpr float kK3 = 64.0f;

// Approximate square root, reciprocal square root and reciprocal (flush-to-zero
// forms, single hardware instructions); callers widen every result so that the
// threshold only grows, and pass normal inputs.
__device__ __forceinline__ float sqrt_approx(float x)
{
    float r;
    asm("sqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float rsqrt_approx(float x)
{
    float r;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

__device__ __forceinline__ float rcp_approx(float x)
{
    float r;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
    return r;
}

// Largest screened loss that can still belong to the exact winner.
//   M      minimum screened loss lam over the candidates
//   alpha2 an upper bound of ||x||^2 / S^2 (or of the weighted norm); the
//          bound D grows with alpha, so any upper bound keeps it valid
//   tau    absolute allowance, in units of S^2 (at least 2^-120)
// With a = 1 - u*K1, b = u*K2*alpha and c >= M + K3*u^2*alpha^2 + tau:
//   sqrt(U) = (b + sqrt(b^2 + 4*a*c')) / (2a) <= (b + sqrt(c)) / a =: s (c' <= c),
// and 1/s <= min(rho, 1/b) with rho >= 1/sqrt(c).  Any t > 0 may stand for
// sqrt(U) in the bound sqrt(z) <= (z/t + t)/2; with t = s,
//   T = (s^2 + b*s/2 + K3*u^2*alpha^2 + tau) / (1 - u*K1 - min(b*rho/2, 1/2)),
// whose denominator is at least 1/2 - u*K1 (every candidate is kept if a NaN
// makes it fail the test below).
__device__ __forceinline__ float survivor_threshold(float M, float alpha2, float tau)
{
    const float alpha = sqrt_approx(fmaxf(alpha2, 0x1p-126f)) * (1.0f + 0x1p-16f);
    const float hb = (0.5f * kU * kK2) * alpha;                    // b/2
    const float k3 = (kK3 * kU * kU) * alpha2;
    const float c = (M + k3 + tau) * (1.0f + 0x1p-16f);
    const float rho = rsqrt_approx(c) * (1.0f + 0x1p-16f);         // >= 1/sqrt(c)
    const float s = (2.0f * hb + c * rho) * (1.0f + 0x1p-15f);    // >= sqrt(U)
    const float den = (1.0f - kU * kK1) - fminf(hb * rho, 0.5f);
    if (!(den > 0.25f)) return __int_as_float(0x7F800000);          // keep all
    const float T = (s * s + hb * s + k3 + tau) * rcp_approx(den);
    return T * (1.0f + 0x1p-10f);
}

// f16x2 of the E2M1 rounding of (lo, hi); the code byte stays in a PTX .b8.
__device__ __forceinline__ uint32_t e2m1x2_round_h(float lo, float hi)
{
    uint32_t h2;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(h2) : "f"(hi), "f"(lo));
    return h2;
}

// (q_lo - r_lo, q_hi - r_hi) from the f16x2 pair q and the f32 pair r: two
// mixed-precision subtracts (each one rounding; the f16 operand is exact).
__device__ __forceinline__ uint64_t sub_h2_f2(uint32_t q2, float rlo, float rhi)
{
    uint64_t r;    // the two results are formed in place as one register pair
    asm("{\n\t.reg .f16 l, h;\n\t.reg .f32 a, b;\n\t"
        "mov.b32 {l, h}, %1;\n\t"
        "sub.rn.f32.f16 a, l, %2;\n\t"
        "sub.rn.f32.f16 b, h, %3;\n\t"
        "mov.b64 %0, {a, b};\n\t}"
        : "=l"(r) : "r"(q2), "f"(rlo), "f"(rhi));
    return r;
}

// Exact binary32 value of an f16x2 pair, via mixed adds of -0 (exact; the
// full-rate path, unlike a plain f16->f32 conversion).  `nz` must be a runtime
// -0.0f so that the adds are not folded away.
__device__ __forceinline__ uint64_t h2_to_f2(uint32_t q2, float nz)
{
    uint64_t r;
    asm("{\n\t.reg .f16 l, h;\n\t.reg .f32 a, b;\n\t"
        "mov.b32 {l, h}, %1;\n\t"
        "add.rn.f32.f16 a, l, %2;\n\t"
        "add.rn.f32.f16 b, h, %2;\n\t"
        "mov.b64 %0, {a, b};\n\t}"
        : "=l"(r) : "r"(q2), "f"(nz));
    return r;
}

__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c)
{
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
    return r;
}

}  // namespace fp4q
