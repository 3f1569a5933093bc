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
//    Let M = min lam.  Bounding the square-root term linearly (see
//    survivor_threshold) gives a threshold T = (M + 2b) / (1 - a)^2 above
//    which no candidate can hold the exact minimum, so every candidate with
//    lam_k > T is excluded.
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

// Largest screened loss that can still belong to the exact winner.
//   M      minimum screened loss lam over the candidates
//   alpha2 an upper bound of ||x||^2 / S^2 (or of the weighted norm); the
//          bound D grows with alpha, so any upper bound keeps it valid
//   tau    absolute allowance, in units of S^2 (at least 2^-120)
// The square-root term is bounded linearly: sqrt(z) <= (z/(g alpha) + g alpha)/2
// for g = 2^-8, so D(z) <= a z + b with
//   a = u (K1 + K2 / (2g)),   b = u K2 g alpha^2 / 2 + K3 u^2 alpha^2 + tau.
// The winner's true loss is at most that of the screening minimum, which is at
// most U = (M + b) / (1 - a).  A candidate k can only win if l_k <= U, and
// l_k >= lam_k - a max(l_k, lam_k) - b, so it needs lam_k <= (U + b) / (1 - a)
// <= (M + 2b) / (1 - a)^2.  That threshold is widened by another 2^-10
// relative (and b by 2^-16), far more than the two roundings of its
// evaluation; a = 2176 u, so it admits candidates within about 0.12% of the
// minimum on a typical block.
__device__ __forceinline__ float survivor_threshold(float M, float alpha2, float tau)
{
    constexpr float kG = 0x1p-8f;
    constexpr float kA = kU * (kK1 + kK2 / (2.0f * kG));
    constexpr float kB = 0.5f * kU * kK2 * kG + kK3 * kU * kU;
    constexpr float kC = (1.0f + 0x1p-10f) / ((1.0f - kA) * (1.0f - kA));
    const float b = __fmaf_rn(alpha2, kB * (1.0f + 0x1p-16f), tau);
    return __fmaf_rn(2.0f, b, M) * kC;
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
