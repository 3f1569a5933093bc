// nvfp4_block.cuh -- the NVFP4 ScaleSweep of one 16-element block, shared by
// the per-tensor sweep kernel and the batch kernel.
//
// ScaleSweep summary (gist.science, arXiv 2606.07618), "Metodologia":
//   sec. 2  S = max|x| / (256*6); s_base = the block maximum relative to S
//           rounded to FP8 (pattern p = E4M3_rne_sat(amax / (6*S)));
//           Lemma 4.1 bounds the optimum by 12/7 s_base (pattern offset +7),
//           Lemma 4.3 by 4/5 s_base for MSE (offset -3), and the WMSE lower
//           bound is set empirically to 1/2 s_base (offset -8);
//   sec. 3  sweep the FP8 bit patterns of that window and keep the one that
//           minimises the objective (sec. 1: MSE, or importance-weighted MSE).
//
// One thread owns one block, so each candidate's loss is accumulated
// sequentially in column order in one thread's registers.  The candidate is
// selected by screen-then-verify (screen.cuh): every candidate of the window
// is screened in step units (two candidates per packed operation, element by
// element so that the (x, x) pair is built once; an odd last candidate two
// elements at a time), candidates whose screened loss exceeds the rigorous
// threshold are dropped, the rest are evaluated with the exact definition,
// and the emit stage writes the winner's codes, its reconstruction q*d and,
// when requested, its exact loss.  All steps d = RN(E4M3(p)*S), reciprocals
// and v^2 come from shared-memory tables built once per global scale.
#pragma once

#include <type_traits>

#include "device.cuh"
#include "screen.cuh"

namespace fp4q {

// Per-global-scale tables in shared memory: (d, inv, v^2) per E4M3 pattern;
// then, for every window position j = p' + kNvOff (p' = p + LO + 2k runs from
// -8 to 141), the pairs (inv[p'], inv[p'+1]) and (v^2[p'], v^2[p'+1]) with each
// pattern clipped to 0x01..0x7E, so that one aligned 8-byte shared load yields
// a candidate pair's operands.
constexpr int kNvPairs = 152, kNvOff = 8;
struct NvTables {
    float4 step[128];
    float2 inv_pair[kNvPairs];
    float2 vsq_pair[kNvPairs];
};

// Scalars derived from the global scale.
struct NvScale {
    float S, t6, invS, tau0;
};

// FP4Q flag for a global max that cannot be used (0 if it can).
__device__ __forceinline__ int32_t nvfp4_gmax_flag(float gmax)
{
    const uint32_t gbits = __float_as_uint(gmax);
    if (gbits >= 0x7F800000u) return kFlagNonfinite;                 // NaN or Inf
    if (gbits != 0u && (gmax < 0x1p-64f || gmax > 0x1p64f)) return kFlagRange;
    return 0;
}

// S = gmax / 1536 (S = 1 for gmax = 0) and the bound's constants.
__device__ __forceinline__ NvScale nvfp4_scale(float gmax)
{
    NvScale c;
    c.S = __float_as_uint(gmax) != 0u ? __fdiv_rn(gmax, 1536.0f) : 1.0f;
    c.t6 = __fmul_rn(6.0f, c.S);
    c.invS = 1.0f / c.S;                              // bound only
    const float tS = 0x1p-70f * c.invS;
    c.tau0 = tS * tS + 0x1p-120f;                     // subnormal allowance, S^2 units
    return c;
}

// Fill the tables for global scale S.  Every thread of the thread block must
// call it (it synchronises twice); any block size.
__device__ __forceinline__ void nvfp4_tables(NvTables& t, float S)
{
    for (int i = threadIdx.x; i < 128; i += blockDim.x) {
        const uint32_t p = i == 0 ? 1u : (i == 127 ? 126u : (uint32_t)i);
        const float v = e4m3_value(p);
        const float d = __fmul_rn(v, S);
        t.step[i] = make_float4(d, __frcp_rn(d), __fmul_rn(v, v), 0.0f);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < kNvPairs; i += blockDim.x) {
        const int pa = min(max(i - kNvOff, 1), 126);
        const int pb = min(max(i - kNvOff + 1, 1), 126);
        t.inv_pair[i] = make_float2(t.step[pa].y, t.step[pb].y);
        t.vsq_pair[i] = make_float2(t.step[pa].z, t.step[pb].z);
    }
    __syncthreads();
}

// Choose the pattern of one block: the screen, the survivor threshold and the
// exact verification below, on the block's 16 values x (amax = max|x|;
// wt the importance weights for WMSE; alpha2, tau and prune as in
// screen.cuh).  Returns the winning E4M3 pattern.
template <int LO, int NREAL, bool WMSE>
__device__ __forceinline__ int nvfp4_select(const NvTables& tb, const NvScale& c, const float (&x)[16], float amax,
                                            const float (&wt)[16], float alpha2, float tau, bool prune,
                                            uint64_t z2, float neg_zero)
{
    constexpr int NC = (NREAL + 1) & ~1;
    const int p = (int)e4m3_rn_sat(__fdiv_rn(amax, c.t6));   // s_base pattern

    // 1. screen every candidate of the window
    constexpr int NP = NREAL / 2;          // candidate pairs screened together
    float lam[NC];
    {
        uint64_t inv2[NP], L2[NP];
        const uint64_t* invp = reinterpret_cast<const uint64_t*>(tb.inv_pair) + (p + LO + kNvOff);
#pragma unroll
        for (int k = 0; k < NP; ++k) {
            inv2[k] = invp[2 * k];
            L2[k] = pk(0.0f, 0.0f);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {     // element outer: the (x, x) pair is built once
            const uint64_t aa = pk(x[i], x[i]);
            const uint64_t w2 = WMSE ? pk(wt[i], wt[i]) : 0;
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                float ra, rb;
                upk(mul2(aa, inv2[k]), ra, rb);
                const uint64_t et = sub_h2_f2(e2m1x2_round_h(ra, rb), ra, rb);
                L2[k] = fma2(WMSE ? mul2(w2, et) : et, et, L2[k]);
            }
        }
        const uint64_t* vsqp = reinterpret_cast<const uint64_t*>(tb.vsq_pair) + (p + LO + kNvOff);
#pragma unroll
        for (int k = 0; k < NP; ++k) upk(mul2(L2[k], vsqp[2 * k]), lam[2 * k], lam[2 * k + 1]);
    }
    if (NREAL & 1) {    // the odd last candidate, two elements per packed operation
        const float il = tb.inv_pair[p + LO + NREAL - 1 + kNvOff].x;
        const float vl = tb.vsq_pair[p + LO + NREAL - 1 + kNvOff].x;
        const uint64_t inv2 = pk(il, il);
        uint64_t L2 = pk(0.0f, 0.0f);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            float ra, rb;
            upk(mul2(pk(x[2 * j], x[2 * j + 1]), inv2), ra, rb);
            const uint64_t et = sub_h2_f2(e2m1x2_round_h(ra, rb), ra, rb);
            L2 = fma2(WMSE ? mul2(pk(wt[2 * j], wt[2 * j + 1]), et) : et, et, L2);
        }
        float lo, hi;
        upk(L2, lo, hi);
        lam[NREAL - 1] = (lo + hi) * vl;
    }
    float M = lam[0];
#pragma unroll
    for (int k = 1; k < NREAL; ++k) M = fminf(M, lam[k]);
    const float thr = prune ? survivor_threshold(M, alpha2, tau) : __int_as_float(0x7F800000);
    uint32_t mask = 0;
#pragma unroll
    for (int k = 0; k < NREAL; ++k) mask |= (lam[k] <= thr ? 1u : 0u) << k;
    if (mask == 0) mask = (1u << NREAL) - 1;   // unreachable for finite inputs; evaluate all

    // 2. verify: exact loss of the survivors, first minimum wins
    int bp;
    if ((mask & (mask - 1)) == 0) {
        bp = min(max(p + LO + __ffs(mask) - 1, 1), 126);
    } else {
        float best = 0.0f;
        bool first = true;
        bp = 1;
        while (mask) {
            const int k = __ffs(mask) - 1;
            mask &= mask - 1;
            const int pp = min(max(p + LO + k, 1), 126);
            const float4 sc = tb.step[pp];
            const uint64_t d2 = pk(sc.x, sc.x), inv2 = pk(sc.y, sc.y);
            float L = 0.0f;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const uint64_t xp = pk(x[2 * j], x[2 * j + 1]);
                float r0, r1;
                upk(mul2(xp, inv2), r0, r1);
                const uint64_t q2 = h2_to_f2(e2m1x2_round_h(r0, r1), neg_zero);
                const uint64_t e2 = sub2(xp, mul2_nofuse(q2, d2, z2));
                uint64_t s2 = mul2_nofuse(e2, e2, z2);
                if (WMSE) s2 = mul2_nofuse(pk(wt[2 * j], wt[2 * j + 1]), s2, z2);
                float s0, s1;
                upk(s2, s0, s1);
                L = __fadd_rn(__fadd_rn(L, s0), s1);
            }
            if (first || L < best) { best = L; bp = pp; }
            first = false;
        }
    }

    return bp;
}

// Quantize one 16-element block.
//   src        the block's 16 input elements
//   wimp       the block's 16 importance weights (WMSE only)
//   codes8     8 bytes of packed nibbles; scale: the E4M3 pattern byte
//   deq16      16 reconstructed elements or nullptr; loss: the block's loss or nullptr
template <typename T, int LO, int NREAL, bool WMSE>
__device__ __forceinline__ void nvfp4_block(const NvTables& tb, const NvScale& c, const T* __restrict__ src,
                                            const float* __restrict__ wimp, uint8_t* __restrict__ codes8,
                                            uint8_t* __restrict__ scale, T* __restrict__ deq16,
                                            float* __restrict__ loss, uint64_t z2, float neg_zero)
{
    // The search works on the signed values: E2M1 rounding and every loss
    // term are symmetric in the sign, so the losses equal those of |x|.
    float x[16];
    uint32_t abits;
    if constexpr (std::is_same<T, __nv_bfloat16>::value) {
        // the global max was checked finite, so no NaN can reach this block:
        // a float max of |x| is the block maximum
        load_block<16>(src, x);
        float m = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(x[i]));
        abits = __float_as_uint(m);
    } else {
        load_block_amax<16>(src, x, abits);
    }
    const float amax = __uint_as_float(abits);
    float alpha2;
    float wt[16];
    float tau = c.tau0;
    bool prune = true;
    if (WMSE) {
        const float4* wp = reinterpret_cast<const float4*>(wimp);
        uint32_t wbits = 0;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const float4 t = __ldg(wp + v);
            wt[4 * v + 0] = t.x; wt[4 * v + 1] = t.y; wt[4 * v + 2] = t.z; wt[4 * v + 3] = t.w;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) wbits = max(wbits, __float_as_uint(wt[i]));
        // the bound assumes 0 <= w <= 2^64 (sign bit clear, at most 2^64)
        prune = wbits <= 0x5F800000u;
        tau = c.tau0 * (1.0f + __uint_as_float(min(wbits, 0x5F800000u)));
        uint64_t al2 = pk(0.0f, 0.0f);
        const uint64_t invS2 = pk(c.invS, c.invS);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint64_t xs = mul2(pk(x[2 * j], x[2 * j + 1]), invS2);
            al2 = fma2(mul2(pk(wt[2 * j], wt[2 * j + 1]), xs), xs, al2);
        }
        float lo, hi;
        upk(al2, lo, hi);
        alpha2 = (lo + hi) * (1.0f + 0x1p-16f);   // bound only: rounded up generously
    } else {
        const float as = amax * c.invS;            // sum x^2 / S^2 <= 16 amax^2 / S^2
        alpha2 = (16.0f * as * as) * (1.0f + 0x1p-16f);
    }
    const int bp = nvfp4_select<LO, NREAL, WMSE>(tb, c, x, amax, wt, alpha2, tau, prune, z2, neg_zero);

    // 3. emit the winner: codes from the signed values, reconstruction q*d,
    //    and its exact loss when requested
    const float4 sw = tb.step[bp];
    const uint64_t d2 = pk(sw.x, sw.x), inv2 = pk(sw.y, sw.y);
    uint32_t word[2];
    float y[16];
    float L = 0.0f;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float r[8];
        uint32_t q2[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) upk(mul2(pk(x[8 * h + 2 * j], x[8 * h + 2 * j + 1]), inv2), r[2 * j], r[2 * j + 1]);
        word[h] = e2m1x8_encode(r, q2);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int i = 8 * h + 2 * j;
            const uint64_t y2 = mul2_nofuse(f16x2_to_f2(q2[j]), d2, z2);
            upk(y2, y[i], y[i + 1]);
            if (loss) {     // the winner is known; its exact loss is only an output
                const uint64_t e2 = sub2(pk(x[i], x[i + 1]), y2);
                uint64_t s2 = mul2_nofuse(e2, e2, z2);
                if (WMSE) s2 = mul2_nofuse(pk(wt[i], wt[i + 1]), s2, z2);
                float s0, s1;
                upk(s2, s0, s1);
                L = __fadd_rn(__fadd_rn(L, s0), s1);
            }
        }
    }
    st_stream64(codes8, make_uint2(word[0], word[1]));
    *scale = (uint8_t)bp;
    if (loss) *loss = L;
    if (deq16) store_block<16>(deq16, y);
}

}  // namespace fp4q
