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
    constexpr int NC = (NREAL + 1) & ~1;   // candidates evaluated in pairs
    const uint64_t z2 = pk(neg_zero, neg_zero);
    __shared__ float2 step[128];           // (d, inv) per E4M3 pattern

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
        const float d = __fmul_rn(e4m3_value(p), S);
        step[threadIdx.x] = make_float2(d, __frcp_rn(d));
    }
    __syncthreads();
    const float t6 = __fmul_rn(6.0f, S);

    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride) {
        float x[16];
        load_block<16>(w + b * 16, x);
        uint64_t aa[16];
        float amax = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float a = fabsf(x[i]);
            amax = fmaxf(amax, a);
            aa[i] = pk(a, a);
        }
        uint64_t ww[16];
        if (WMSE) {
            const float4* wp = reinterpret_cast<const float4*>(importance + (b % blocks_per_row) * 16);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const float4 t = __ldg(wp + v);
                ww[4 * v + 0] = pk(t.x, t.x);
                ww[4 * v + 1] = pk(t.y, t.y);
                ww[4 * v + 2] = pk(t.z, t.z);
                ww[4 * v + 3] = pk(t.w, t.w);
            }
        }
        const int p = (int)e4m3_rn_sat(__fdiv_rn(amax, t6));   // s_base pattern

        float best = 0.0f;
        int bp = 1;
#pragma unroll
        for (int k = 0; k < NC; k += 2) {
            const int pa = min(max(p + LO + min(k, NREAL - 1), 1), 126);
            const int pb = min(max(p + LO + min(k + 1, NREAL - 1), 1), 126);
            const float2 sa = step[pa], sb = step[pb];
            const uint64_t inv2 = pk(sa.y, sb.y), d2 = pk(sa.x, sb.x);
            uint64_t L2 = pk(0.0f, 0.0f);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float ra, rb;
                upk(mul2(aa[i], inv2), ra, rb);
                const uint64_t q2 = e2m1x2_round(ra, rb);
                const uint64_t e2 = sub2(aa[i], mul2_nofuse(q2, d2, z2));
                uint64_t s2 = mul2_nofuse(e2, e2, z2);
                if (WMSE) s2 = mul2_nofuse(ww[i], s2, z2);
                L2 = add2(L2, s2);
            }
            float La, Lb;
            upk(L2, La, Lb);
            if (k == 0 || La < best) { best = La; bp = pa; }
            if (Lb < best) { best = Lb; bp = pb; }
        }

        // emit the winner: codes from the signed values, reconstruction q*d
        const float2 sw = step[bp];
        uint32_t byte[8];
#pragma unroll
        for (int j = 0; j < 8; ++j)
            byte[j] = e2m1x2(__fmul_rn(x[2 * j], sw.y), __fmul_rn(x[2 * j + 1], sw.y));
        uint2 packed;
        packed.x = byte[0] | byte[1] << 8 | byte[2] << 16 | byte[3] << 24;
        packed.y = byte[4] | byte[5] << 8 | byte[6] << 16 | byte[7] << 24;
        st_stream64(codes + b * 8, packed);
        scales[b] = (uint8_t)bp;
        if (loss) loss[b] = best;
        if (deq) {
            float y[16];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float qa, qb;
                upk(e2m1x2_decode(byte[j]), qa, qb);
                y[2 * j] = __fmul_rn(qa, sw.x);
                y[2 * j + 1] = __fmul_rn(qb, sw.x);
            }
            store_block<16>(deq + b * 16, y);
        }
    }
}

template <typename T, int LO, int NREAL, bool WMSE>
void launch_typed(const void* w, int64_t rows, int64_t cols, const float* d_amax,
                  const float* importance, uint8_t* codes, uint8_t* scales, float* d_S,
                  void* deq, float* loss, int32_t* d_status, cudaStream_t s)
{
    const int64_t nblocks = rows * (cols / 16);
    // balanced waves of at most 8 resident thread blocks per SM
    const int64_t per_wave = (int64_t)sm_count() * 8 * kThreads;
    const int64_t waves = (nblocks + per_wave - 1) / per_wave;
    int64_t grid = (nblocks + kThreads * waves - 1) / (kThreads * waves);
    if (grid < 1) grid = 1;
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
