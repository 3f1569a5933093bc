// focus.cu -- the FOCUS forward quantizer and the inverse block Hadamard.
//
// "FOCUS" summary (gist.science, arXiv 2608.01847), "Metodologia" 2-3: the
// stored (dequantization) scale S_dq of a hardware block keeps its format
// (E4M3 x S for NVFP4, E8M0 for MXFP4), while the quantization scale is
// relaxed to S_q = S_dq * c_k with a full-precision coefficient per sub-block
// (CRS: one per block; DGS: one per sub-block of e.g. 8 elements).  The codes
// are Q(W_k / S_q) and the reconstruction is q * S_dq.  Per sub-block k:
//   dq = RN(d * c_k);  inv = RN(1 / dq);  r = x * inv;  q = E2M1(r);
//   y = RN(q * d);     loss = sum over the block of RN(x - y)^2, column order
// with d = RN(E4M3(p) * S) (NVFP4) or 2^(b - 127) (MXFP4).  One thread per
// hardware block, loads and stores as in the quantizer kernels.
//
// MR-GPTQ summary, technical sec. 2: MXFP4 weights are stored rotated by the
// random-sign block Hadamard y = c * H32 * (sigma o x).  Since (c * H32)^2 = I
// and sigma o sigma = 1, x = sigma o (c * H32 * y): the same five butterfly
// stages, the multiply by c, then the sign flips map a rotated-domain
// reconstruction back to the original domain.
#include <cuda_fp16.h>

#include "device.cuh"
#include "launch.h"
#include "mxfp4_block.cuh"

namespace fp4q {

namespace {

constexpr int kThreads = 256;

template <typename T, int BS, int SUB>
__global__ void __launch_bounds__(kThreads)
focus_kernel(const T* __restrict__ w, int64_t nblocks, const uint8_t* __restrict__ scales,
             const float* __restrict__ d_S, const __half* __restrict__ coeffs, uint8_t* __restrict__ codes,
             T* __restrict__ deq, float* __restrict__ loss, int32_t* __restrict__ d_status, float neg_zero)
{
    constexpr bool NV = BS == 16;
    const float S = NV ? __ldg(d_S) : 1.0f;
    const uint64_t z2 = pk(neg_zero, neg_zero);
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    int32_t flags = 0;
    for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride) {
        float x[BS];
        uint32_t abits;
        load_block_amax<BS>(w + b * BS, x, abits);
        if (abits >= 0x7F800000u) flags |= kFlagNonfinite;
        const uint32_t sb = __ldg(scales + b);
        float d;
        if (NV) {
            if (sb < 1u || sb > 126u) flags |= kFlagRange;
            d = __fmul_rn(e4m3_value(sb & 0x7Fu), S);
        } else {
            if (sb == 255u) flags |= kFlagRange;
            d = exp2i((int)sb - 127);
        }
        // the reciprocal quantization step of every sub-block
        float inv[BS / SUB];
#pragma unroll
        for (int k = 0; k < BS / SUB; ++k) {
            const __half h = coeffs[(b * BS) / SUB + k];
            const uint16_t hb = __half_as_ushort(h);
            if ((hb & 0x8000u) || hb == 0u || (hb & 0x7C00u) == 0x7C00u) flags |= kFlagRange;
            inv[k] = __frcp_rn(__fmul_rn(d, __half2float(h)));
        }
        const uint64_t d2 = pk(d, d);
        uint32_t word[BS / 8];
        float y[BS];
        float L = 0.0f;
#pragma unroll
        for (int h = 0; h < BS / 8; ++h) {
            float r[8];
            uint32_t q2[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = 8 * h + 2 * j;
                const float iv = inv[i / SUB];
                upk(mul2(pk(x[i], x[i + 1]), pk(iv, iv)), r[2 * j], r[2 * j + 1]);
            }
            word[h] = e2m1x8_encode(r, q2);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = 8 * h + 2 * j;
                const uint64_t y2 = mul2_nofuse(f16x2_to_f2(q2[j]), d2, z2);
                upk(y2, y[i], y[i + 1]);
                if (loss) {
                    const uint64_t e2 = sub2(pk(x[i], x[i + 1]), y2);
                    float s0, s1;
                    upk(mul2_nofuse(e2, e2, z2), s0, s1);
                    L = __fadd_rn(__fadd_rn(L, s0), s1);
                }
            }
        }
        if (NV)
            st_stream64(codes + b * 8, make_uint2(word[0], word[1]));
        else
            st_stream(codes + b * 16, make_uint4(word[0], word[1], word[2], word[3]));
        if (loss) loss[b] = L;
        if (deq) store_block<BS>(deq + b * BS, y);
    }
    if (flags) atomicOr(d_status, flags);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
unrotate_kernel(const T* __restrict__ y, int64_t nblocks, int64_t blocks_per_row,
                const uint32_t* __restrict__ sign_masks, T* __restrict__ out)
{
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride) {
        float v[32];
        load_block<32>(y + b * 32, v);
#pragma unroll
        for (int h = 1; h < 32; h *= 2) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if (i & h) continue;
                const float a = v[i], c = v[i + h];
                v[i] = __fadd_rn(a, c);
                v[i + h] = __fsub_rn(a, c);
            }
        }
        const uint32_t m = __ldg(sign_masks + (b % blocks_per_row));
#pragma unroll
        for (int j = 0; j < 32; ++j)
            v[j] = __uint_as_float(__float_as_uint(__fmul_rn(v[j], kInvSqrt32)) ^ (((m >> j) & 1u) << 31));
        store_block<32>(out + b * 32, v);
    }
}

template <typename T, int BS, int SUB>
void launch_focus_typed(const void* w, int64_t rows, int64_t cols, const uint8_t* scales, const float* d_S,
                        const void* coeffs, uint8_t* codes, void* deq, float* loss, int32_t* d_status,
                        cudaStream_t s)
{
    const int64_t nblocks = rows * (cols / BS);
    const int64_t grid = resident_grid(focus_kernel<T, BS, SUB>, kThreads, 0, nblocks);
    focus_kernel<T, BS, SUB><<<(unsigned)grid, kThreads, 0, s>>>(
        static_cast<const T*>(w), nblocks, scales, d_S, static_cast<const __half*>(coeffs), codes,
        static_cast<T*>(deq), loss, d_status, -0.0f);
}

template <typename T, int BS>
bool launch_focus_sub(int sub, const void* w, int64_t rows, int64_t cols, const uint8_t* scales,
                      const float* d_S, const void* coeffs, uint8_t* codes, void* deq, float* loss,
                      int32_t* d_status, cudaStream_t s)
{
    switch (sub) {
    case 4: launch_focus_typed<T, BS, 4>(w, rows, cols, scales, d_S, coeffs, codes, deq, loss, d_status, s); return true;
    case 8: launch_focus_typed<T, BS, 8>(w, rows, cols, scales, d_S, coeffs, codes, deq, loss, d_status, s); return true;
    case 16: launch_focus_typed<T, BS, 16>(w, rows, cols, scales, d_S, coeffs, codes, deq, loss, d_status, s); return true;
    case 32:
        if (BS != 32) return false;
        launch_focus_typed<T, 32, 32>(w, rows, cols, scales, d_S, coeffs, codes, deq, loss, d_status, s);
        return true;
    }
    return false;
}

}  // namespace

bool launch_focus(bool mx, bool bf16, int sub, const void* w, int64_t rows, int64_t cols, const uint8_t* scales,
                  const float* d_S, const void* coeffs, uint8_t* codes, void* deq, float* loss,
                  int32_t* d_status, cudaStream_t s)
{
    if (mx)
        return bf16 ? launch_focus_sub<__nv_bfloat16, 32>(sub, w, rows, cols, scales, d_S, coeffs, codes, deq,
                                                          loss, d_status, s)
                    : launch_focus_sub<float, 32>(sub, w, rows, cols, scales, d_S, coeffs, codes, deq, loss,
                                                  d_status, s);
    return bf16 ? launch_focus_sub<__nv_bfloat16, 16>(sub, w, rows, cols, scales, d_S, coeffs, codes, deq, loss,
                                                      d_status, s)
                : launch_focus_sub<float, 16>(sub, w, rows, cols, scales, d_S, coeffs, codes, deq, loss, d_status,
                                              s);
}

void launch_unrotate(bool bf16, const void* y, int64_t rows, int64_t cols, const uint32_t* sign_masks, void* out,
                     cudaStream_t s)
{
    const int64_t nblocks = rows * (cols / 32);
    if (bf16) {
        const int64_t grid = resident_grid(unrotate_kernel<__nv_bfloat16>, kThreads, 0, nblocks);
        unrotate_kernel<__nv_bfloat16><<<(unsigned)grid, kThreads, 0, s>>>(
            static_cast<const __nv_bfloat16*>(y), nblocks, cols / 32, sign_masks, static_cast<__nv_bfloat16*>(out));
    } else {
        const int64_t grid = resident_grid(unrotate_kernel<float>, kThreads, 0, nblocks);
        unrotate_kernel<float><<<(unsigned)grid, kThreads, 0, s>>>(static_cast<const float*>(y), nblocks, cols / 32,
                                                                   sign_masks, static_cast<float*>(out));
    }
}

}  // namespace fp4q
