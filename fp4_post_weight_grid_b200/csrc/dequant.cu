// dequant.cu -- decode packed E2M1 codes with their block scales, and the
// diagnostic probes of the rounding primitives.
//
// NVFP4 (ScaleSweep summary, "Declaracao do Problema": E2M1 elements with an
// FP8 block scale and an FP32 global scale): out = RN(q * RN(E4M3(s) * S)).
// MXFP4 (MR-GPTQ summary, technical sec. 1: power-of-two E8M0 scales):
// out = q * 2^(b-127).  Both equal the quantizers' reconstruction bit for bit.
// One thread decodes one block; loads and stores are 8/16-byte vectors.
#include <cmath>

#include "device.cuh"
#include "launch.h"
#include "wait.cuh"

namespace fp4q {

namespace {

constexpr int kThreads = 256;

// Signed E4M3 pattern -> value; 0x7F / 0xFF are NaN.
__device__ __forceinline__ float e4m3_signed(uint32_t s)
{
    const uint32_t p = s & 0x7Fu;
    const float v = p == 0x7Fu ? __uint_as_float(0x7FC00000u) : e4m3_value(p);
    return (s & 0x80u) ? -v : v;
}

// E8M0 byte -> 2^(b-127); 0xFF is NaN.
__device__ __forceinline__ float e8m0_value(uint32_t b)
{
    return b == 0xFFu ? __uint_as_float(0x7FC00000u) : exp2i((int)b - 127);
}

template <typename T, bool MX>
__global__ void __launch_bounds__(kThreads)
dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
               const float* __restrict__ d_S, int64_t nblocks, T* __restrict__ out)
{
    constexpr int B = MX ? 32 : 16;
    const float S = MX ? 1.0f : __ldg(d_S);
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride) {
        const uint32_t s = scales[b];
        const float d = MX ? e8m0_value(s) : __fmul_rn(e4m3_signed(s), S);
        uint32_t word[B / 8];
        if (MX) {
            const uint4 u = *reinterpret_cast<const uint4*>(codes + b * 16);
            word[0] = u.x; word[1] = u.y; word[2] = u.z; word[3] = u.w;
        } else {
            const uint2 u = *reinterpret_cast<const uint2*>(codes + b * 8);
            word[0] = u.x; word[1] = u.y;
        }
        float y[B];
#pragma unroll
        for (int j = 0; j < B / 2; ++j) {
            float qa, qb;
            upk(e2m1x2_decode((word[j / 4] >> (8 * (j % 4))) & 0xFFu), qa, qb);
            y[2 * j] = __fmul_rn(qa, d);
            y[2 * j + 1] = __fmul_rn(qb, d);
        }
        store_block<B>(out + b * B, y);
    }
}

// A plain streaming copy (16-byte loads and stores, four in flight per
// thread, grid-stride): the copy bandwidth this library's own loads and
// stores reach, for the HBM roofline of the benchmark.
__global__ void __launch_bounds__(kThreads) probe_copy_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                                              int64_t n16)
{
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    for (; i + 3 * stride < n16; i += 4 * stride) {
        const uint4 a = ld_stream(src + i), b = ld_stream(src + i + stride);
        const uint4 c = ld_stream(src + i + 2 * stride), d = ld_stream(src + i + 3 * stride);
        st_stream(dst + i, a);
        st_stream(dst + i + stride, b);
        st_stream(dst + i + 2 * stride, c);
        st_stream(dst + i + 3 * stride, d);
    }
    for (; i < n16; i += stride) st_stream(dst + i, ld_stream(src + i));
}

// The library's bounded spin-wait on its own: one thread waits for *flag >=
// target and raises FP4Q_FLAG_TIMEOUT if that does not happen within `limit`
// polls, so that tests can watch a wait run out without any fault.
__global__ void probe_wait_kernel(const unsigned* flag, unsigned target, unsigned limit, int32_t* d_status)
{
    if (!wait_geq(flag, target, limit)) atomicOr(d_status, kFlagTimeout);
}

__global__ void probe_e2m1_kernel(const float* __restrict__ r, uint8_t* __restrict__ out, int64_t n)
{
    const int64_t npair = (n + 1) / 2;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < npair;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float lo = r[2 * i];
        const float hi = 2 * i + 1 < n ? r[2 * i + 1] : 0.0f;
        const uint32_t byte = e2m1x2(lo, hi);
        out[2 * i] = (uint8_t)(byte & 15u);
        if (2 * i + 1 < n) out[2 * i + 1] = (uint8_t)(byte >> 4);
    }
}

__global__ void probe_e4m3_kernel(const float* __restrict__ v, uint8_t* __restrict__ out, int64_t n)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        out[i] = (uint8_t)e4m3_rn_sat(v[i]);
}

int64_t grid_for(int64_t items)
{
    int64_t g = (items + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)sm_count() * 16;
    if (g > cap) g = cap;
    return g < 1 ? 1 : g;
}

}  // namespace

void launch_dequant(bool mx, const uint8_t* codes, const uint8_t* scales, const float* d_S,
                    int64_t rows, int64_t cols, void* out, bool out_bf16, cudaStream_t s)
{
    const int64_t nb = rows * (cols / (mx ? 32 : 16));
    const unsigned g = (unsigned)grid_for(nb);
    if (mx) {
        if (out_bf16)
            dequant_kernel<__nv_bfloat16, true><<<g, kThreads, 0, s>>>(codes, scales, d_S, nb,
                                                                       static_cast<__nv_bfloat16*>(out));
        else
            dequant_kernel<float, true><<<g, kThreads, 0, s>>>(codes, scales, d_S, nb,
                                                               static_cast<float*>(out));
    } else {
        if (out_bf16)
            dequant_kernel<__nv_bfloat16, false><<<g, kThreads, 0, s>>>(codes, scales, d_S, nb,
                                                                        static_cast<__nv_bfloat16*>(out));
        else
            dequant_kernel<float, false><<<g, kThreads, 0, s>>>(codes, scales, d_S, nb,
                                                                static_cast<float*>(out));
    }
}

void launch_probe_copy(const void* src, void* dst, int64_t bytes, cudaStream_t s)
{
    const int64_t n16 = bytes / 16;
    int64_t grid = (n16 + 4 * kThreads - 1) / (4 * kThreads);
    const int64_t cap = (int64_t)sm_count() * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    probe_copy_kernel<<<(unsigned)grid, kThreads, 0, s>>>(static_cast<const uint4*>(src), static_cast<uint4*>(dst),
                                                           n16);
}

void launch_probe_wait(const unsigned* flag, unsigned target, unsigned limit, int32_t* d_status, cudaStream_t s)
{
    probe_wait_kernel<<<1, 1, 0, s>>>(flag, target, limit, d_status);
}

void launch_probe_e2m1(const float* r, uint8_t* out, int64_t n, cudaStream_t s)
{
    probe_e2m1_kernel<<<(unsigned)grid_for((n + 1) / 2), kThreads, 0, s>>>(r, out, n);
}

void launch_probe_e4m3(const float* v, uint8_t* out, int64_t n, cudaStream_t s)
{
    probe_e4m3_kernel<<<(unsigned)grid_for(n), kThreads, 0, s>>>(v, out, n);
}

}  // namespace fp4q
