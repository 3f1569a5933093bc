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

namespace fp4q {

namespace {

constexpr int kThreads = 256;
constexpr float kInvSqrt32 = 0x1.6a09e6p-3f;   // RN(1/sqrt(32))

template <typename T, bool HAD>
__global__ void __launch_bounds__(kThreads)
mxfp4_kernel(const T* __restrict__ w, int64_t nblocks, int64_t blocks_per_row,
             const uint32_t* __restrict__ masks, uint8_t* __restrict__ codes,
             uint8_t* __restrict__ scales, T* __restrict__ deq, float* __restrict__ loss,
             int32_t* __restrict__ d_status, float neg_zero)
{
    const uint64_t z2 = pk(neg_zero, neg_zero);
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride) {
        float x[32];
        load_block<32>(w + b * 32, x);
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
        uint32_t abits = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) abits = max(abits, __float_as_uint(x[j]) & 0x7FFFFFFFu);
        if (abits >= 0x7F800000u) atomicOr(d_status, kFlagNonfinite);
        int e0 = -127;
        if (abits >= 0x00800000u) {
            const int a = (int)(abits >> 23) - 127;                 // floor(log2 amax)
            e0 = a - 2 + ((abits & 0x7FFFFFu) > 0x400000u ? 1 : 0);  // 6*2^(a-2) = 1.5*2^a
            e0 = min(max(e0, -127), 127);
        }
        const int ea = max(e0 - 1, -127), ec = min(e0 + 1, 127);
        float best = 0.0f;
        int be = ea;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const int e_lo = k == 0 ? ea : ec;
            const int e_hi = k == 0 ? e0 : ec;
            const uint64_t inv2 = pk(exp2i(-e_lo), exp2i(-e_hi));
            const uint64_t d2 = pk(exp2i(e_lo), exp2i(e_hi));
            uint64_t L2 = pk(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const float a = fabsf(x[i]);
                const uint64_t aa = pk(a, a);
                float ra, rb;
                upk(mul2(aa, inv2), ra, rb);
                const uint64_t q2 = e2m1x2_round(ra, rb);
                const uint64_t e2 = sub2(aa, mul2_nofuse(q2, d2, z2));
                L2 = add2(L2, mul2_nofuse(e2, e2, z2));
            }
            float La, Lb;
            upk(L2, La, Lb);
            if (k == 0 || La < best) { best = La; be = e_lo; }
            if (Lb < best) { best = Lb; be = e_hi; }
        }
        const float d = exp2i(be), inv = exp2i(-be);
        uint32_t byte[16];
#pragma unroll
        for (int j = 0; j < 16; ++j)
            byte[j] = e2m1x2(__fmul_rn(x[2 * j], inv), __fmul_rn(x[2 * j + 1], inv));
        uint4 packed;
        packed.x = byte[0] | byte[1] << 8 | byte[2] << 16 | byte[3] << 24;
        packed.y = byte[4] | byte[5] << 8 | byte[6] << 16 | byte[7] << 24;
        packed.z = byte[8] | byte[9] << 8 | byte[10] << 16 | byte[11] << 24;
        packed.w = byte[12] | byte[13] << 8 | byte[14] << 16 | byte[15] << 24;
        st_stream(codes + b * 16, packed);
        scales[b] = (uint8_t)(be + 127);
        if (loss) loss[b] = best;
        if (deq) {
            float y[32];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                float qa, qb;
                upk(e2m1x2_decode(byte[j]), qa, qb);
                y[2 * j] = __fmul_rn(qa, d);
                y[2 * j + 1] = __fmul_rn(qb, d);
            }
            store_block<32>(deq + b * 32, y);
        }
    }
}

template <typename T, bool HAD>
void launch_typed(const void* w, int64_t rows, int64_t cols, const uint32_t* masks, uint8_t* codes,
                  uint8_t* scales, void* deq, float* loss, int32_t* d_status, cudaStream_t s)
{
    const int64_t nblocks = rows * (cols / 32);
    const int64_t per_wave = (int64_t)sm_count() * 8 * kThreads;
    const int64_t waves = (nblocks + per_wave - 1) / per_wave;
    int64_t grid = (nblocks + kThreads * waves - 1) / (kThreads * waves);
    if (grid < 1) grid = 1;
    mxfp4_kernel<T, HAD><<<(unsigned)grid, kThreads, 0, s>>>(
        static_cast<const T*>(w), nblocks, cols / 32, masks, codes, scales, static_cast<T*>(deq),
        loss, d_status, -0.0f);
}

}  // namespace

void launch_mxfp4(const void* w, bool bf16, int64_t rows, int64_t cols, const uint32_t* sign_masks,
                  uint8_t* codes, uint8_t* scales, void* deq, float* loss, int32_t* d_status,
                  cudaStream_t s)
{
    if (sign_masks) {
        if (bf16)
            launch_typed<__nv_bfloat16, true>(w, rows, cols, sign_masks, codes, scales, deq, loss,
                                              d_status, s);
        else
            launch_typed<float, true>(w, rows, cols, sign_masks, codes, scales, deq, loss, d_status, s);
    } else {
        if (bf16)
            launch_typed<__nv_bfloat16, false>(w, rows, cols, nullptr, codes, scales, deq, loss,
                                               d_status, s);
        else
            launch_typed<float, false>(w, rows, cols, nullptr, codes, scales, deq, loss, d_status, s);
    }
}

}  // namespace fp4q
