// mxfp4.cu -- MXFP4 with an E8M0 exponent sweep, optionally after a fused
// random-sign 32-point block Hadamard rotation.
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
// Mapping.  One thread owns one 32-element block: the rotation (sign flips,
// five in-register butterfly stages h = 1..16, the 1/sqrt(32) multiply) and
// the sequential loss of each candidate stay in registers.  The candidates are
// powers of two, so r = y * 2^-e and q * 2^e are exact scalings; three
// candidates are padded to four (a clamped duplicate never wins) and evaluated
// as two f32x2 pairs like the NVFP4 sweep.  The Hadamard runs on the CUDA
// cores: it has to reproduce the stage order bit for bit, which a tensor-core
// contraction does not, and it costs 6 adds/multiplies per element against a
// memory budget of ~4.5 bytes per element.
#include "device.cuh"
#include "launch.h"
#include "screen.cuh"

namespace fp4q {

namespace {

constexpr int kThreads = 256;
constexpr float kInvSqrt32 = 0x1.6a09e6p-3f;   // RN(1/sqrt(32))

// AMAX: also reduce max|w| of the unrotated input into *gmax_bits (an atomic
// max on the binary32 bit pattern, which keeps NaN and Inf), for the NVFP4
// global scale of the same weight.
template <typename T, bool HAD, bool AMAX>
__global__ void __launch_bounds__(kThreads, 3)
mxfp4_kernel(const T* __restrict__ w, int64_t nblocks, int64_t blocks_per_row,
             const uint32_t* __restrict__ masks, uint8_t* __restrict__ codes,
             uint8_t* __restrict__ scales, T* __restrict__ deq, float* __restrict__ loss,
             int32_t* __restrict__ d_status, float neg_zero, unsigned* __restrict__ gmax_bits)
{
    const uint64_t z2 = pk(neg_zero, neg_zero);
    uint32_t wmax = 0;     // AMAX: max |w| bits over this thread's blocks
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride) {
        float x[32];
        load_block<32>(w + b * 32, x);
        if (HAD && AMAX) {
#pragma unroll
            for (int j = 0; j < 32; ++j) wmax = max(wmax, __float_as_uint(x[j]) & 0x7FFFFFFFu);
        }
        if (HAD) {
            const uint32_t m = __ldg(masks + (b % blocks_per_row));
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
        }
        float a[32];        // |y|, shared by every stage below
        uint32_t abits = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
            a[j] = fabsf(x[j]);
            abits = max(abits, __float_as_uint(a[j]));
        }
        if (abits >= 0x7F800000u) atomicOr(d_status, kFlagNonfinite);
        if (!HAD && AMAX) wmax = max(wmax, abits);
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
        float alpha2;
        {
            uint64_t al2 = pk(0.0f, 0.0f);
            const uint64_t inv02 = pk(inv0, inv0);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const uint64_t as = mul2(pk(a[2 * j], a[2 * j + 1]), inv02);
                al2 = fma2(as, as, al2);
            }
            float lo, hi;
            upk(al2, lo, hi);
            alpha2 = (lo + hi) * (1.0f + 0x1p-16f);   // bound only: rounded up generously
        }
        const float tS = 0x1p-70f * inv0;
        const float tau = tS * tS + 0x1p-120f;
        float lam[3];
        {   // exponents e0-1 and e0 as a pair, one element at a time
            const int ea = FP4Q_EK(0), eb = FP4Q_EK(1);
            const uint64_t inv2 = pk(exp2i(-ea), exp2i(-eb));
            uint64_t L2 = pk(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float ra, rb;
                upk(mul2(pk(a[i], a[i]), inv2), ra, rb);
                const uint64_t et = sub_h2_f2(e2m1x2_round_h(ra, rb), ra, rb);
                L2 = fma2(et, et, L2);
            }
            upk(mul2(L2, pk(exp2i(2 * (ea - e0)), exp2i(2 * (eb - e0)))), lam[0], lam[1]);
        }
        {   // exponent e0+1, two elements at a time
            const int ec = FP4Q_EK(2);
            const float invc = exp2i(-ec);
            const uint64_t inv2 = pk(invc, invc);
            uint64_t L2 = pk(0.0f, 0.0f);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float ra, rb;
                upk(mul2(pk(a[2 * j], a[2 * j + 1]), inv2), ra, rb);
                const uint64_t et = sub_h2_f2(e2m1x2_round_h(ra, rb), ra, rb);
                L2 = fma2(et, et, L2);
            }
            float lo, hi;
            upk(L2, lo, hi);
            lam[2] = (lo + hi) * exp2i(2 * (ec - e0));
        }
        const float M = fminf(fminf(lam[0], lam[1]), lam[2]);
        const float T = survivor_threshold(M, alpha2, tau);
        uint32_t mask = (lam[0] <= T ? 1u : 0u) | (lam[1] <= T ? 2u : 0u) | (lam[2] <= T ? 4u : 0u);
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
                    const uint64_t ap = pk(a[2 * j], a[2 * j + 1]);
                    float r0, r1;
                    upk(mul2(ap, inv2), r0, r1);
                    const uint64_t q2 = h2_to_f2(e2m1x2_round_h(r0, r1), neg_zero);
                    const uint64_t e2 = sub2(ap, mul2_nofuse(q2, d2, z2));
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
            float y[8];
            word[c] = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = 8 * c + 2 * j;
                const uint64_t xp = pk(x[i], x[i + 1]);
                float r0, r1;
                upk(mul2(xp, inv2), r0, r1);
                const uint32_t byte = e2m1x2(r0, r1);
                word[c] |= byte << (8 * j);
                const uint64_t y2 = mul2_nofuse(h2_to_f2(e2m1x2_to_f16x2(byte), neg_zero), d2, z2);
                upk(y2, y[2 * j], y[2 * j + 1]);
                if (loss) {     // the winner is known; its exact loss is only an output
                    const uint64_t e2 = sub2(xp, y2);
                    float s0, s1;
                    upk(mul2_nofuse(e2, e2, z2), s0, s1);
                    L = __fadd_rn(__fadd_rn(L, s0), s1);
                }
            }
            if (deq) store_block<8>(deq + b * 32 + 8 * c, y);
        }
#undef FP4Q_EK
        st_stream(codes + b * 16, make_uint4(word[0], word[1], word[2], word[3]));
        scales[b] = (uint8_t)(be + 127);
        if (loss) loss[b] = L;
    }
    if (AMAX) {
        __shared__ uint32_t warp_max[kThreads / 32];
        wmax = __reduce_max_sync(0xFFFFFFFFu, wmax);
        if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = wmax;
        __syncthreads();
        if (threadIdx.x < 32) {
            wmax = threadIdx.x < kThreads / 32 ? warp_max[threadIdx.x] : 0u;
            wmax = __reduce_max_sync(0xFFFFFFFFu, wmax);
            if (threadIdx.x == 0 && wmax != 0u) atomicMax(gmax_bits, wmax);
        }
    }
}

template <typename T, bool HAD, bool AMAX>
void launch_typed(const void* w, int64_t rows, int64_t cols, const uint32_t* masks, uint8_t* codes,
                  uint8_t* scales, void* deq, float* loss, int32_t* d_status, unsigned* gmax_bits,
                  cudaStream_t s)
{
    const int64_t nblocks = rows * (cols / 32);
    const int64_t grid = resident_grid(mxfp4_kernel<T, HAD, AMAX>, kThreads, 0, nblocks);
    mxfp4_kernel<T, HAD, AMAX><<<(unsigned)grid, kThreads, 0, s>>>(
        static_cast<const T*>(w), nblocks, cols / 32, masks, codes, scales, static_cast<T*>(deq),
        loss, d_status, -0.0f, gmax_bits);
}

template <typename T, bool AMAX>
void launch_rot(const void* w, int64_t rows, int64_t cols, const uint32_t* masks, uint8_t* codes,
                uint8_t* scales, void* deq, float* loss, int32_t* d_status, unsigned* gmax_bits,
                cudaStream_t s)
{
    if (masks)
        launch_typed<T, true, AMAX>(w, rows, cols, masks, codes, scales, deq, loss, d_status, gmax_bits, s);
    else
        launch_typed<T, false, AMAX>(w, rows, cols, nullptr, codes, scales, deq, loss, d_status, gmax_bits, s);
}

}  // namespace

void launch_mxfp4(const void* w, bool bf16, int64_t rows, int64_t cols, const uint32_t* sign_masks,
                  uint8_t* codes, uint8_t* scales, void* deq, float* loss, int32_t* d_status,
                  float* d_amax, cudaStream_t s)
{
    unsigned* g = reinterpret_cast<unsigned*>(d_amax);
    if (d_amax) {
        cudaMemsetAsync(d_amax, 0, sizeof(float), s);
        if (bf16)
            launch_rot<__nv_bfloat16, true>(w, rows, cols, sign_masks, codes, scales, deq, loss, d_status, g, s);
        else
            launch_rot<float, true>(w, rows, cols, sign_masks, codes, scales, deq, loss, d_status, g, s);
    } else {
        if (bf16)
            launch_rot<__nv_bfloat16, false>(w, rows, cols, sign_masks, codes, scales, deq, loss, d_status, g, s);
        else
            launch_rot<float, false>(w, rows, cols, sign_masks, codes, scales, deq, loss, d_status, g, s);
    }
}

}  // namespace fp4q
