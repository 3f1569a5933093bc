// mxfp4_block.cuh -- MXFP4 quantization of one 32-element block with the
// E8M0 exponent sweep, optionally after the random-sign block Hadamard; shared
// by the per-tensor kernel and the batch kernel.
//
// "Bridging the Gap Between Promise and Performance for Microscaling FP4
// Quantization" (gist.science, arXiv 2509.23202), technical summary:
//   sec. 1  MXFP4 groups of 32 elements share one power-of-two (E8M0) scale;
//   sec. 2  the group scales are chosen to minimise the MSE ("Grade Otimizada
//           por MSE"), and block Hadamard micro-rotations are fused into the
//           GPU kernel ("Rotacoes Online Fundidas").
// "Resumo Tecnico: TORQ" (arXiv 2605.19561) sec. 2.B: the S-step maps the
// block maximum onto the largest code, which gives the centre exponent e0 =
// the smallest e with 6*2^e >= amax; the sweep visits e0-1, e0, e0+1.
//
// One thread owns one block: the rotation (sign flips, five in-register
// butterfly stages h = 1..16, the 1/sqrt(32) multiply) and the sequential loss
// stay in registers.  The three exponents are selected by screen-then-verify
// (screen.cuh) in units of 2^e0, each exponent two elements at a time (e0+1
// is never the first minimum and is not screened, see kMxScreened).  The Hadamard runs on the CUDA cores:
// it has to reproduce the stage order bit for bit, which a tensor-core
// contraction does not, and it costs 6 adds/multiplies per element against a
// memory budget of ~4.5 bytes per element.
#pragma once

#include "device.cuh"
#include "screen.cuh"

namespace fp4q {

constexpr float kInvSqrt32 = 0x1.6a09e6p-3f;   // RN(1/sqrt(32))

// Candidates screened: e0-1 and e0 only.  e0 is the smallest exponent whose
// grid 2^e0 * {0, .5, 1, 1.5, 2, 3, 4, 6} covers the block maximum, and the
// grid of e0+1 inside [0, 6 * 2^e0] is {0, 1, 2, 3, 4, 6} * 2^e0, a subset of
// it: the nearest point of e0+1 is never nearer than that of e0, for every
// element.  With power-of-two steps r = x * 2^-e and y = q * 2^e are exact
// (an element too small for that has q = 0 under both), and RN(x - y),
// RN(e * e) and the running sum are monotone, so the definition's loss at
// e0+1 is never below the loss at e0 and the first minimum is never e0+1
// (after clamping at 127 the two are the same exponent).  Its screened loss is
// set to +inf: it survives only when the threshold is infinite, and then the
// exact verification decides, as for any candidate.
constexpr int kMxScreened = 2;

// The 32 bf16 elements of a block from its 64 raw bytes, and max|w| as bits.
__device__ __forceinline__ void unpack32_bf16_amax(const uint4* u, float (&x)[32], uint32_t& wmax)
{
    uint32_t m2 = 0;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        const uint4 t = u[v];
        bf16x2_to_f32(t.x, x[8 * v + 0], x[8 * v + 1]);
        bf16x2_to_f32(t.y, x[8 * v + 2], x[8 * v + 3]);
        bf16x2_to_f32(t.z, x[8 * v + 4], x[8 * v + 5]);
        bf16x2_to_f32(t.w, x[8 * v + 6], x[8 * v + 7]);
        m2 = __vmaxu2(m2, __vmaxu2(t.x & 0x7FFF7FFFu, t.y & 0x7FFF7FFFu));
        m2 = __vmaxu2(m2, __vmaxu2(t.z & 0x7FFF7FFFu, t.w & 0x7FFF7FFFu));
    }
    wmax = max(m2 & 0xFFFFu, m2 >> 16) << 16;
}

// max(bits_of(m), |v|) as binary32 bits, m a non-negative float's bits: a NaN
// input gives the canonical NaN 0x7FFFFFFF, above Inf, above every finite value.
__device__ __forceinline__ uint32_t max_nan_abs(uint32_t m, float v)
{
    float r;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(r) : "f"(__uint_as_float(m)), "f"(fabsf(v)));
    return __float_as_uint(r);
}

// Neighbour-paired form (elements 2j, 2j+1 in a register pair).
template <typename T, bool HAD>
__device__ __forceinline__ uint32_t mxfp4_block_pairs_of_neighbours(const T* __restrict__ src, uint32_t sign_mask,
                                                uint8_t* __restrict__ codes16, uint8_t* __restrict__ scale,
                                                T* __restrict__ deq32, float* __restrict__ loss,
                                                int32_t* __restrict__ d_status, uint64_t z2, float neg_zero)
{
    float x[32];
    uint32_t wmax;         // max |w| bits of the unrotated block
    load_block_amax<32>(src, x, wmax);
    uint32_t abits = wmax; // max |y| bits of the block that is quantized
    if (HAD) {
        const uint32_t m = sign_mask;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            x[j] = __uint_as_float(__float_as_uint(x[j]) ^ (((m >> j) & 1u) << 31));
#pragma unroll
        for (int h = 1; h < 32; h *= 2) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (i & h) continue;
                const float a = x[i], c = x[i + h];
                x[i] = __fadd_rn(a, c);
                x[i + h] = __fsub_rn(a, c);
            }
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) x[j] = __fmul_rn(x[j], kInvSqrt32);
        abits = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) abits = max(abits, __float_as_uint(x[j]) & 0x7FFFFFFFu);
    }
    // From here on the search works on the signed values: E2M1 rounding and
    // every loss term are symmetric in the sign.
    if (abits >= 0x7F800000u) atomicOr(d_status, kFlagNonfinite);
    int e0 = -127;
    if (abits >= 0x00800000u) {
        const int a = (int)(abits >> 23) - 127;                 // floor(log2 amax)
        e0 = a - 2 + ((abits & 0x7FFFFFu) > 0x400000u ? 1 : 0);  // 6*2^(a-2) = 1.5*2^a
        e0 = min(max(e0, -127), 127);
    }
    // candidate k = 0, 1, 2 is the exponent e0 - 1 + k, clamped to [-127, 127]
#define FP4Q_EK(k) min(max(e0 - 1 + (k), -127), 127)

    // 1. screen the three exponents in units of 2^e0 (S = 2^e0, v = 2^(e-e0))
    const float inv0 = exp2i(-e0);
    const float as = __uint_as_float(abits) * inv0;      // sum y^2 / S^2 <= 32 amax^2 / S^2
    const float alpha2 = (32.0f * as * as) * (1.0f + 0x1p-16f);
    const float tS = 0x1p-70f * inv0;
    const float tau = tS * tS + 0x1p-120f;
    float lam[3];
    {   // e0-1 and e0, two elements at a time; e0+1 never wins (kMxScreened)
        uint64_t inv2[kMxScreened], L2[kMxScreened];
#pragma unroll
        for (int k = 0; k < kMxScreened; ++k) {
            const float ik = exp2i(-FP4Q_EK(k));
            inv2[k] = pk(ik, ik);
            L2[k] = pk(0.0f, 0.0f);
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            const uint64_t xp = pk(x[2 * j], x[2 * j + 1]);
#pragma unroll
            for (int k = 0; k < kMxScreened; ++k) {
                float ra, rb;
                upk(mul2(xp, inv2[k]), ra, rb);
                const uint64_t et = sub_h2_f2(e2m1x2_round_h(ra, rb), ra, rb);
                L2[k] = fma2(et, et, L2[k]);
            }
        }
#pragma unroll
        for (int k = 0; k < kMxScreened; ++k) {
            float lo, hi;
            upk(L2[k], lo, hi);
            lam[k] = (lo + hi) * exp2i(2 * (FP4Q_EK(k) - e0));
        }
        lam[2] = __int_as_float(0x7F800000);
    }
    const float M = fminf(fminf(lam[0], lam[1]), lam[2]);
    const float thr = survivor_threshold(M, alpha2, tau);
    uint32_t mask = (lam[0] <= thr ? 1u : 0u) | (lam[1] <= thr ? 2u : 0u) | (lam[2] <= thr ? 4u : 0u);
    if (mask == 0) mask = 7u;                  // unreachable for finite inputs; evaluate all

    // 2. verify: exact loss of the survivors, first minimum wins
    int be;
    if ((mask & (mask - 1)) == 0) {
        be = FP4Q_EK(__ffs(mask) - 1);
    } else {
        float best = 0.0f;
        bool first = true;
        be = FP4Q_EK(0);
        while (mask) {
            const int k = __ffs(mask) - 1;
            mask &= mask - 1;
            const int e = FP4Q_EK(k);
            const uint64_t d2 = pk(exp2i(e), exp2i(e)), inv2 = pk(exp2i(-e), exp2i(-e));
            float L = 0.0f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint64_t xp = pk(x[2 * j], x[2 * j + 1]);
                float r0, r1;
                upk(mul2(xp, inv2), r0, r1);
                const uint64_t q2 = h2_to_f2(e2m1x2_round_h(r0, r1), neg_zero);
                const uint64_t e2 = sub2(xp, mul2_nofuse(q2, d2, z2));
                float s0, s1;
                upk(mul2_nofuse(e2, e2, z2), s0, s1);
                L = __fadd_rn(__fadd_rn(L, s0), s1);
            }
            if (first || L < best) { best = L; be = e; }
            first = false;
        }
    }

    // 3. emit the winner with its exact loss
    const float d = exp2i(be), inv = exp2i(-be);
    const uint64_t d2 = pk(d, d), inv2 = pk(inv, inv);
    uint32_t word[4];
    float L = 0.0f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {          // 8 elements per chunk: one 16-byte bf16 store
        float y[8], r[8];
        uint32_t q2[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) upk(mul2(pk(x[8 * c + 2 * j], x[8 * c + 2 * j + 1]), inv2), r[2 * j], r[2 * j + 1]);
        word[c] = e2m1x8_encode(r, q2);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = 8 * c + 2 * j;
            const uint64_t y2 = mul2_nofuse(f16x2_to_f2(q2[j]), d2, z2);
            upk(y2, y[2 * j], y[2 * j + 1]);
            if (loss) {     // the winner is known; its exact loss is only an output
                const uint64_t e2 = sub2(pk(x[i], x[i + 1]), y2);
                float s0, s1;
                upk(mul2_nofuse(e2, e2, z2), s0, s1);
                L = __fadd_rn(__fadd_rn(L, s0), s1);
            }
        }
        if (deq32) store_block<8>(deq32 + 8 * c, y);
    }
#undef FP4Q_EK
    st_stream(codes16, make_uint4(word[0], word[1], word[2], word[3]));
    *scale = (uint8_t)(be + 127);
    if (loss) *loss = L;
    return wmax;

}

// Half-paired form (elements j, j+16 in a register pair), for the rotation.
// PF < 0: the block is loaded from src here.  PF >= 0 (bf16 only): the block's
// 64 bytes arrive in `cur`, and the 64 bytes at `next` (if not null) are loaded
// into `nxt` before any of this block's work.
template <typename T, bool HAD, int PF = -1>
__device__ __forceinline__ uint32_t mxfp4_block_pairs_of_halves(const T* __restrict__ src, uint32_t sign_mask,
                                                uint8_t* __restrict__ codes16, uint8_t* __restrict__ scale,
                                                T* __restrict__ deq32, float* __restrict__ loss,
                                                int32_t* __restrict__ d_status, uint64_t z2, float neg_zero,
                                                const uint4* cur = nullptr, const T* __restrict__ next = nullptr,
                                                uint4* nxt = nullptr)
{
    // The block lives in 16 register pairs P[j].  With the rotation, P[j]
    // holds elements j and j+16: the butterfly stages h = 1, 2, 4, 8 act on
    // both alike and run as packed adds, stage h = 16 combines the two halves
    // of each pair; every element sees the operations of the stage-by-stage
    // definition in its order.  (Without the rotation P[j] would hold the
    // neighbours 2j, 2j+1.)  The search and the emit work on whatever pairing
    // P has; E(j, h) is the element held in half h of P[j].
#define FP4Q_E(j, h) (HAD ? (j) + 16 * (h) : 2 * (j) + (h))
    float x[32];
    uint32_t wmax;         // max |w| bits of the unrotated block
    if constexpr (PF < 0) {
        load_block_amax<32>(src, x, wmax);
    } else {
        unpack32_bf16_amax(cur, x, wmax);
#pragma unroll
        for (int v = 0; v < 4; ++v) nxt[v] = next ? ld_stream(next + 8 * v) : make_uint4(0, 0, 0, 0);
    }
    uint32_t abits = wmax; // max |y| bits of the block that is quantized
    uint64_t P[16];
    if (HAD) {
        const uint32_t m = sign_mask;
#pragma unroll
        for (int j = 0; j < 32; ++j)
            x[j] = __uint_as_float(__float_as_uint(x[j]) ^ (((m >> j) & 1u) << 31));
#pragma unroll
        for (int j = 0; j < 16; ++j) P[j] = pk(x[j], x[j + 16]);
#pragma unroll
        for (int h = 1; h < 16; h *= 2) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                if (i & h) continue;
                const uint64_t a = P[i], c = P[i + h];
                P[i] = add2(a, c);
                P[i + h] = sub2(a, c);
            }
        }
        const uint64_t c2 = pk(kInvSqrt32, kInvSqrt32);
        abits = 0;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            float a, c;
            upk(P[j], a, c);
            P[j] = mul2(pk(__fadd_rn(a, c), __fsub_rn(a, c)), c2);
            upk(P[j], a, c);
            abits = max_nan_abs(max_nan_abs(abits, a), c);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) P[j] = pk(x[2 * j], x[2 * j + 1]);
    }
    // From here on the search works on the signed values: E2M1 rounding and
    // every loss term are symmetric in the sign.
    if (abits >= 0x7F800000u) atomicOr(d_status, kFlagNonfinite);
    int e0 = -127;
    if (abits >= 0x00800000u) {
        const int a = (int)(abits >> 23) - 127;                 // floor(log2 amax)
        e0 = a - 2 + ((abits & 0x7FFFFFu) > 0x400000u ? 1 : 0);  // 6*2^(a-2) = 1.5*2^a
        e0 = min(max(e0, -127), 127);
    }
    // candidate k = 0, 1, 2 is the exponent e0 - 1 + k, clamped to [-127, 127]
#define FP4Q_EK(k) min(max(e0 - 1 + (k), -127), 127)

    // 1. screen the three exponents in units of 2^e0 (S = 2^e0, v = 2^(e-e0))
    const float inv0 = exp2i(-e0);
    const float as = __uint_as_float(abits) * inv0;      // sum y^2 / S^2 <= 32 amax^2 / S^2
    const float alpha2 = (32.0f * as * as) * (1.0f + 0x1p-16f);
    const float tS = 0x1p-70f * inv0;
    const float tau = tS * tS + 0x1p-120f;
    float lam[3];
    {   // e0-1 and e0, one register pair at a time; e0+1 never wins (kMxScreened)
        uint64_t inv2[kMxScreened], L2[kMxScreened];
#pragma unroll
        for (int k = 0; k < kMxScreened; ++k) {
            const float ik = exp2i(-FP4Q_EK(k));
            inv2[k] = pk(ik, ik);
            L2[k] = pk(0.0f, 0.0f);
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) {
#pragma unroll
            for (int k = 0; k < kMxScreened; ++k) {
                float ra, rb;
                upk(mul2(P[j], inv2[k]), ra, rb);
                const uint64_t et = sub_h2_f2(e2m1x2_round_h(ra, rb), ra, rb);
                L2[k] = fma2(et, et, L2[k]);
            }
        }
#pragma unroll
        for (int k = 0; k < kMxScreened; ++k) {
            float lo, hi;
            upk(L2[k], lo, hi);
            lam[k] = (lo + hi) * exp2i(2 * (FP4Q_EK(k) - e0));
        }
        lam[2] = __int_as_float(0x7F800000);
    }
    const float M = fminf(fminf(lam[0], lam[1]), lam[2]);
    const float thr = survivor_threshold(M, alpha2, tau);
    uint32_t mask = (lam[0] <= thr ? 1u : 0u) | (lam[1] <= thr ? 2u : 0u) | (lam[2] <= thr ? 4u : 0u);
    if (mask == 0) mask = 7u;                  // unreachable for finite inputs; evaluate all

    // 2. verify: exact loss of the survivors (summed in element order), first minimum wins
    int be;
    if ((mask & (mask - 1)) == 0) {
        be = FP4Q_EK(__ffs(mask) - 1);
    } else {
        float best = 0.0f;
        bool first = true;
        be = FP4Q_EK(0);
        while (mask) {
            const int k = __ffs(mask) - 1;
            mask &= mask - 1;
            const int e = FP4Q_EK(k);
            const uint64_t d2 = pk(exp2i(e), exp2i(e)), inv2 = pk(exp2i(-e), exp2i(-e));
            float s[32];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float r0, r1;
                upk(mul2(P[j], inv2), r0, r1);
                const uint64_t q2 = h2_to_f2(e2m1x2_round_h(r0, r1), neg_zero);
                const uint64_t e2 = sub2(P[j], mul2_nofuse(q2, d2, z2));
                upk(mul2_nofuse(e2, e2, z2), s[FP4Q_E(j, 0)], s[FP4Q_E(j, 1)]);
            }
            float L = 0.0f;
#pragma unroll
            for (int i = 0; i < 32; ++i) L = __fadd_rn(L, s[i]);
            if (first || L < best) { best = L; be = e; }
            first = false;
        }
    }

    // 3. emit the winner: codes, reconstruction q*d and, when requested, its
    //    exact loss in element order
    const float d = exp2i(be), inv = exp2i(-be);
    const uint64_t d2 = pk(d, d), inv2 = pk(inv, inv);
    uint32_t word[4];
    float L = 0.0f;
    // one 8-element chunk: its 8 quotients in element order -> word[c] and deq
    auto emit_chunk = [&](int c, const float (&rc)[8]) {
        float y[8];
        uint32_t q2[4];
        word[c] = e2m1x8_encode(rc, q2);
#pragma unroll
        for (int j = 0; j < 4; ++j) upk(mul2_nofuse(f16x2_to_f2(q2[j]), d2, z2), y[2 * j], y[2 * j + 1]);
        if (deq32) store_block<8>(deq32 + 8 * c, y);
    };
    if (HAD) {
        // pairs 8g..8g+7 hold elements 8g..8g+7 (low halves, chunk g) and
        // 16+8g..16+8g+7 (high halves, chunk 2+g)
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            float rl[8], rh[8];
#pragma unroll
            for (int m = 0; m < 8; ++m) upk(mul2(P[8 * g + m], inv2), rl[m], rh[m]);
            emit_chunk(g, rl);
            emit_chunk(2 + g, rh);
        }
        if (loss) {     // the winner is known; its exact loss is only an output
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float lo, hi;
                upk(P[i & 15], lo, hi);
                const float xi = i < 16 ? lo : hi;
                const uint32_t code = e2m1x2(__fmul_rn(xi, inv), 0.0f) & 0xFu;
                float q, unused;
                f16x2_to_f32(e2m1x2_to_f16x2(code), q, unused);
                const float e = __fsub_rn(xi, __fmul_rn(q, d));
                L = __fadd_rn(L, __fmul_rn(e, e));
            }
        }
    } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float rc[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) upk(mul2(P[4 * c + j], inv2), rc[2 * j], rc[2 * j + 1]);
            emit_chunk(c, rc);
        }
        if (loss) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float r0, r1;
                upk(mul2(P[j], inv2), r0, r1);
                const uint64_t y2 = mul2_nofuse(e2m1x2_decode(e2m1x2(r0, r1)), d2, z2);
                const uint64_t e2 = sub2(P[j], y2);
                float s0, s1;
                upk(mul2_nofuse(e2, e2, z2), s0, s1);
                L = __fadd_rn(__fadd_rn(L, s0), s1);
            }
        }
    }
#undef FP4Q_E
#undef FP4Q_EK
    st_stream(codes16, make_uint4(word[0], word[1], word[2], word[3]));
    *scale = (uint8_t)(be + 127);
    if (loss) *loss = L;
    return wmax;

}

// Quantize one 32-element block; returns max|w| (as binary32 bits) of the
// unrotated block, for a fused global max.
//   src      the block's 32 input elements; sign_mask: its sign mask (HAD only)
//   codes16  16 bytes of packed nibbles; scale: the E8M0 byte
//   deq32    32 reconstructed elements or nullptr; loss: the block's loss or nullptr
// Both forms compute the same bytes; the rotated one keeps elements j and j+16
// in one register pair so that four of the five butterfly stages run packed.
template <typename T, bool HAD>
__device__ __forceinline__ uint32_t mxfp4_block(const T* __restrict__ src, uint32_t sign_mask,
                                                uint8_t* __restrict__ codes16, uint8_t* __restrict__ scale,
                                                T* __restrict__ deq32, float* __restrict__ loss,
                                                int32_t* __restrict__ d_status, uint64_t z2, float neg_zero)
{
    if constexpr (HAD)
        return mxfp4_block_pairs_of_halves<T, true>(src, sign_mask, codes16, scale, deq32, loss, d_status, z2, neg_zero);
    else
        return mxfp4_block_pairs_of_neighbours<T, false>(src, sign_mask, codes16, scale, deq32, loss, d_status, z2,
                                                         neg_zero);
}

}  // namespace fp4q
