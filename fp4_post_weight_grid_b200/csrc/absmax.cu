// absmax.cu -- grid-wide max|x| for the NVFP4 global scale.
//
// ScaleSweep summary, "Metodologia" sec. 2: S = max|x| / (256*6) needs the
// tensor's largest magnitude before any block is quantized.  This is one
// streaming read of W: 16-byte loads, four in flight per thread, the maximum
// kept as an unsigned bit pattern of |x| (non-negative binary32 values order
// like unsigned integers and every NaN pattern sorts above +Inf, so NaN and
// Inf survive the reduction), a warp reduction, then one atomicMax per thread
// block on the caller's float.
#include "device.cuh"
#include "launch.h"
#include "nvfp4_block.cuh"

namespace fp4q {

namespace {

constexpr int kThreads = 512;

__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b)
{
    uint32_t r;
    asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

template <bool BF16>
__device__ __forceinline__ uint32_t merge(uint32_t m, uint4 u)
{
    if (BF16) {
        m = vmax_u16x2(m, u.x & 0x7FFF7FFFu);
        m = vmax_u16x2(m, u.y & 0x7FFF7FFFu);
        m = vmax_u16x2(m, u.z & 0x7FFF7FFFu);
        m = vmax_u16x2(m, u.w & 0x7FFF7FFFu);
    } else {
        m = max(m, u.x & 0x7FFFFFFFu);
        m = max(m, u.y & 0x7FFFFFFFu);
        m = max(m, u.z & 0x7FFFFFFFu);
        m = max(m, u.w & 0x7FFFFFFFu);
    }
    return m;
}

template <bool BF16>
__global__ void __launch_bounds__(kThreads) absmax_kernel(const void* __restrict__ x, int64_t n,
                                                          unsigned* __restrict__ out)
{
    constexpr int kPerVec = BF16 ? 8 : 4;
    const int64_t nvec = n / kPerVec;
    const uint4* v = static_cast<const uint4*>(x);
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    uint32_t m = 0;
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        uint4 a = ld_stream(v + i);
        uint4 b = ld_stream(v + i + stride);
        uint4 c = ld_stream(v + i + 2 * stride);
        uint4 d = ld_stream(v + i + 3 * stride);
        m = merge<BF16>(m, a);
        m = merge<BF16>(m, b);
        m = merge<BF16>(m, c);
        m = merge<BF16>(m, d);
    }
    for (; i < nvec; i += stride) m = merge<BF16>(m, ld_stream(v + i));
    if (BF16) m = max(m & 0xFFFFu, m >> 16) << 16;     // bf16 pattern -> binary32 pattern
    // the last n % kPerVec elements
    if (blockIdx.x == 0 && threadIdx.x < (unsigned)(n - nvec * kPerVec)) {
        const int64_t k = nvec * kPerVec + threadIdx.x;
        uint32_t t = BF16 ? ((uint32_t)static_cast<const uint16_t*>(x)[k] & 0x7FFFu) << 16
                          : static_cast<const uint32_t*>(x)[k] & 0x7FFFFFFFu;
        m = max(m, t);
    }
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    __shared__ uint32_t warp_max[kThreads / 32];
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = threadIdx.x < kThreads / 32 ? warp_max[threadIdx.x] : 0u;
        m = __reduce_max_sync(0xFFFFFFFFu, m);
        if (threadIdx.x == 0 && m != 0u) atomicMax(out, m);
    }
}

// After the reduction: flag a global max that the NVFP4 sweep cannot use
// (NaN/Inf, or nonzero outside [2^-64, 2^64]), one warp, one word read.
__global__ void __launch_bounds__(32) absmax_check_kernel(const float* __restrict__ d_amax,
                                                          int32_t* __restrict__ d_status)
{
    if (threadIdx.x == 0) {
        const int32_t flag = nvfp4_gmax_flag(*d_amax);
        if (flag) atomicOr(d_status, flag);
    }
}

}  // namespace

void launch_absmax(const void* x, bool bf16, int64_t n, float* d_amax, int32_t* d_status, cudaStream_t s)
{
    cudaMemsetAsync(d_amax, 0, sizeof(float), s);
    if (n <= 0) return;
    const int64_t nvec = n / (bf16 ? 8 : 4);
    int64_t blocks = (nvec + 4 * kThreads - 1) / (4 * kThreads);
    const int64_t cap = (int64_t)sm_count() * 4;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    unsigned* out = reinterpret_cast<unsigned*>(d_amax);
    if (bf16)
        absmax_kernel<true><<<(unsigned)blocks, kThreads, 0, s>>>(x, n, out);
    else
        absmax_kernel<false><<<(unsigned)blocks, kThreads, 0, s>>>(x, n, out);
    if (d_status) absmax_check_kernel<<<1, 32, 0, s>>>(d_amax, d_status);
}

}  // namespace fp4q
