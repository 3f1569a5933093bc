// nvfp4.cu -- NVFP4 ScaleSweep: per-block E4M3 scale search (MSE / WMSE).
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
// Mapping.  One thread owns one 16-element block, so each candidate's loss is
// accumulated sequentially in column order in one thread's registers (the
// fixed order that makes the result reproducible bit for bit).  A warp covers
// 32 consecutive blocks = 512 contiguous elements: the two 16-byte loads per
// lane, the 8-byte code stores, the 1-byte scale stores and the 32-byte
// reconstruction stores of a warp are all contiguous.
//
// Inner loop.  Candidates are evaluated two at a time with sm_100a f32x2
// arithmetic: for element x the pair (r_k, r_k+1) = (|x|, |x|) * (inv_k,
// inv_k+1) is one packed multiply, one cvt.e2m1x2 rounds both to E2M1 (ties to
// even, saturating), one cvt back to f16x2 and two exact widenings give
// (q_k, q_k+1); then y = q*d, e = |x| - y, e*e (and w*(e*e)) and L += are four
// packed RN operations (the two products that feed an add are issued as fma
// with a -0 addend so that ptxas cannot fuse them into the add; see
// mul2_nofuse).  Working on |x| gives the same e*e as the signed value
// because round-to-nearest is symmetric.  Per-candidate steps d = RN(E4M3(p)*S)
// and inv = RN(1/d) for all 126 patterns are computed once per thread block
// into shared memory.  The window is clamped to 0x01..0x7E by clamping each
// candidate pattern: a clamped duplicate has the same loss as its original and
// so never wins a strict comparison, which keeps every lane on the same path.
#include "device.cuh"
#include "launch.h"
#include "screen.cuh"

namespace fp4q {

namespace {

constexpr int kThreads = 256;

template <typename T, int LO, int NREAL, bool WMSE>
__global__ void __launch_bounds__(kThreads)
nvfp4_sweep_kernel(const T* __restrict__ w, int64_t nblocks, int64_t blocks_per_row,
                   const float* __restrict__ d_amax, const float* __restrict__ importance,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                   float* __restrict__ d_S, T* __restrict__ deq, float* __restrict__ loss,
                   int32_t* __restrict__ d_status, float neg_zero)
{
    constexpr int NC = (NREAL + 1) & ~1;
    // Per E4M3 pattern: (d, inv, v^2); then, for every window position j = p' + 8
    // (p' = p + LO + 2k may run from -8 to 140), the pairs (inv[p'], inv[p'+1])
    // and (v^2[p'], v^2[p'+1]) with each pattern clipped to 0x01..0x7E, so that
    // one aligned 8-byte shared load yields a candidate pair's operands.
    constexpr int kPairs = 152, kOff = 8;
    __shared__ float4 step[128];
    __shared__ float2 inv_pair[kPairs], vsq_pair[kPairs];

    const float gmax = __ldg(d_amax);
    const uint32_t gbits = __float_as_uint(gmax);
    if (gbits >= 0x7F800000u) {            // NaN or Inf reached the global max
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(d_status, kFlagNonfinite);
        return;
    }
    if (gbits != 0u && (gmax < 0x1p-64f || gmax > 0x1p64f)) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(d_status, kFlagRange);
        return;
    }
    const float S = gbits != 0u ? __fdiv_rn(gmax, 1536.0f) : 1.0f;
    if (blockIdx.x == 0 && threadIdx.x == 0) *d_S = S;
    if (threadIdx.x < 128) {
        const uint32_t p = threadIdx.x == 0 ? 1u : (threadIdx.x == 127 ? 126u : threadIdx.x);
        const float v = e4m3_value(p);
        const float d = __fmul_rn(v, S);
        step[threadIdx.x] = make_float4(d, __frcp_rn(d), __fmul_rn(v, v), 0.0f);
    }
    __syncthreads();
    if (threadIdx.x < kPairs) {
        const int pa = min(max((int)threadIdx.x - kOff, 1), 126);
        const int pb = min(max((int)threadIdx.x - kOff + 1, 1), 126);
        inv_pair[threadIdx.x] = make_float2(step[pa].y, step[pb].y);
        vsq_pair[threadIdx.x] = make_float2(step[pa].z, step[pb].z);
    }
    __syncthreads();
    const float t6 = __fmul_rn(6.0f, S);
    const float invS = 1.0f / S;                              // bound only
    const float tS = 0x1p-70f * invS;
    const float tau0 = tS * tS + 0x1p-120f;                   // subnormal allowance, S^2 units
    const uint64_t z2 = pk(neg_zero, neg_zero);

    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride) {
        float x[16];
        load_block<16>(w + b * 16, x);
        float amax = 0.0f, alpha2 = 0.0f;
        float wt[16];
        float tau = tau0;
        bool prune = true;
        if (WMSE) {
            const float4* wp = reinterpret_cast<const float4*>(importance + (b % blocks_per_row) * 16);
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
            tau = tau0 * (1.0f + __uint_as_float(min(wbits, 0x5F800000u)));
        }
        float a[16];        // |x|, shared by every stage below
#pragma unroll
        for (int i = 0; i < 16; ++i) a[i] = fabsf(x[i]);
        uint64_t al2 = pk(0.0f, 0.0f);
        const uint64_t invS2 = pk(invS, invS);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            amax = fmaxf(amax, fmaxf(a[2 * j], a[2 * j + 1]));
            const uint64_t as = mul2(pk(a[2 * j], a[2 * j + 1]), invS2);
            al2 = fma2(WMSE ? mul2(pk(wt[2 * j], wt[2 * j + 1]), as) : as, as, al2);
        }
        {
            float lo, hi;
            upk(al2, lo, hi);
            alpha2 = (lo + hi) * (1.0f + 0x1p-16f);   // bound only: rounded up generously
        }
        const int p = (int)e4m3_rn_sat(__fdiv_rn(amax, t6));   // s_base pattern

        // 1. screen every candidate of the window
        constexpr int NP = NREAL / 2;          // candidate pairs screened together
        float lam[NC];
        {
            uint64_t inv2[NP], L2[NP];
            const uint64_t* invp = reinterpret_cast<const uint64_t*>(inv_pair) + (p + LO + kOff);
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                inv2[k] = invp[2 * k];
                L2[k] = pk(0.0f, 0.0f);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {     // element outer: the (|x|, |x|) pair is built once
                const uint64_t aa = pk(a[i], a[i]);
                const uint64_t w2 = WMSE ? pk(wt[i], wt[i]) : 0;
#pragma unroll
                for (int k = 0; k < NP; ++k) {
                    float ra, rb;
                    upk(mul2(aa, inv2[k]), ra, rb);
                    const uint64_t et = sub_h2_f2(e2m1x2_round_h(ra, rb), ra, rb);
                    L2[k] = fma2(WMSE ? mul2(w2, et) : et, et, L2[k]);
                }
            }
            const uint64_t* vsqp = reinterpret_cast<const uint64_t*>(vsq_pair) + (p + LO + kOff);
#pragma unroll
            for (int k = 0; k < NP; ++k) upk(mul2(L2[k], vsqp[2 * k]), lam[2 * k], lam[2 * k + 1]);
        }
        if (NREAL & 1) {    // the odd last candidate, two elements per packed operation
            const float il = inv_pair[p + LO + NREAL - 1 + kOff].x;
            const float vl = vsq_pair[p + LO + NREAL - 1 + kOff].x;
            const uint64_t inv2 = pk(il, il);
            uint64_t L2 = pk(0.0f, 0.0f);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float ra, rb;
                upk(mul2(pk(a[2 * j], a[2 * j + 1]), inv2), ra, rb);
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
        const float T = prune ? survivor_threshold(M, alpha2, tau) : __int_as_float(0x7F800000);
        uint32_t mask = 0;
#pragma unroll
        for (int k = 0; k < NREAL; ++k) mask |= (lam[k] <= T ? 1u : 0u) << k;
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
                const float4 sc = step[pp];
                const uint64_t d2 = pk(sc.x, sc.x), inv2 = pk(sc.y, sc.y);
                float L = 0.0f;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint64_t ap = pk(a[2 * j], a[2 * j + 1]);
                    float r0, r1;
                    upk(mul2(ap, inv2), r0, r1);
                    const uint64_t q2 = h2_to_f2(e2m1x2_round_h(r0, r1), neg_zero);
                    const uint64_t e2 = sub2(ap, mul2_nofuse(q2, d2, z2));
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

        // 3. emit the winner: codes from the signed values, reconstruction
        //    q*d, and its exact loss
        const float4 sw = step[bp];
        const uint64_t d2 = pk(sw.x, sw.x), inv2 = pk(sw.y, sw.y);
        uint32_t byte[8];
        float y[16];
        float L = 0.0f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const uint64_t xp = pk(x[2 * j], x[2 * j + 1]);
            float r0, r1;
            upk(mul2(xp, inv2), r0, r1);
            byte[j] = e2m1x2(r0, r1);
            const uint64_t y2 = mul2_nofuse(h2_to_f2(e2m1x2_to_f16x2(byte[j]), neg_zero), d2, z2);
            upk(y2, y[2 * j], y[2 * j + 1]);
            if (loss) {     // the winner is known; its exact loss is only an output
                const uint64_t e2 = sub2(xp, y2);
                uint64_t s2 = mul2_nofuse(e2, e2, z2);
                if (WMSE) s2 = mul2_nofuse(pk(wt[2 * j], wt[2 * j + 1]), s2, z2);
                float s0, s1;
                upk(s2, s0, s1);
                L = __fadd_rn(__fadd_rn(L, s0), s1);
            }
        }
        uint2 packed;
        packed.x = byte[0] | byte[1] << 8 | byte[2] << 16 | byte[3] << 24;
        packed.y = byte[4] | byte[5] << 8 | byte[6] << 16 | byte[7] << 24;
        st_stream64(codes + b * 8, packed);
        scales[b] = (uint8_t)bp;
        if (loss) loss[b] = L;
        if (deq) store_block<16>(deq + b * 16, y);
    }
}

template <typename T, int LO, int NREAL, bool WMSE>
void launch_typed(const void* w, int64_t rows, int64_t cols, const float* d_amax,
                  const float* importance, uint8_t* codes, uint8_t* scales, float* d_S,
                  void* deq, float* loss, int32_t* d_status, cudaStream_t s)
{
    const int64_t nblocks = rows * (cols / 16);
    const int64_t grid = resident_grid(nvfp4_sweep_kernel<T, LO, NREAL, WMSE>, kThreads, 0, nblocks);
    nvfp4_sweep_kernel<T, LO, NREAL, WMSE><<<(unsigned)grid, kThreads, 0, s>>>(
        static_cast<const T*>(w), nblocks, cols / 16, d_amax, importance, codes, scales, d_S,
        static_cast<T*>(deq), loss, d_status, -0.0f);
}

}  // namespace

void launch_nvfp4_sweep(const void* w, bool bf16, int64_t rows, int64_t cols, const float* d_amax,
                        const float* importance, uint8_t* codes, uint8_t* scales, float* d_S,
                        void* deq, float* loss, int32_t* d_status, cudaStream_t s)
{
    if (importance == nullptr) {
        if (bf16)
            launch_typed<__nv_bfloat16, -3, 11, false>(w, rows, cols, d_amax, nullptr, codes, scales,
                                                        d_S, deq, loss, d_status, s);
        else
            launch_typed<float, -3, 11, false>(w, rows, cols, d_amax, nullptr, codes, scales, d_S,
                                               deq, loss, d_status, s);
    } else {
        if (bf16)
            launch_typed<__nv_bfloat16, -8, 16, true>(w, rows, cols, d_amax, importance, codes,
                                                       scales, d_S, deq, loss, d_status, s);
        else
            launch_typed<float, -8, 16, true>(w, rows, cols, d_amax, importance, codes, scales, d_S,
                                              deq, loss, d_status, s);
    }
}

}  // namespace fp4q
