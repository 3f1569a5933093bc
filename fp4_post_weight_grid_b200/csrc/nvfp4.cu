// nvfp4.cu -- NVFP4 ScaleSweep kernel for one weight: one thread per
// 16-element block over a grid-stride loop; the per-block search is
// nvfp4_block (nvfp4_block.cuh), the global scale comes from *d_amax
// (ScaleSweep summary, "Metodologia: ScaleSweep" sec. 2).
#include "device.cuh"
#include "launch.h"
#include "nvfp4_block.cuh"

namespace fp4q {

namespace {

constexpr int kThreads = 256;

template <typename T, int LO, int NREAL, bool WMSE>
__global__ void __launch_bounds__(kThreads, WMSE ? 3 : 5)
nvfp4_sweep_kernel(const T* __restrict__ w, int64_t nblocks, int64_t blocks_per_row,
                   const float* __restrict__ d_amax, const float* __restrict__ importance,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                   float* __restrict__ d_S, T* __restrict__ deq, float* __restrict__ loss,
                   int32_t* __restrict__ d_status, float neg_zero)
{
    __shared__ NvTables tb;
    const float gmax = __ldg(d_amax);
    const int32_t flag = nvfp4_gmax_flag(gmax);
    if (flag) {
        if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(d_status, flag);
        return;
    }
    const NvScale c = nvfp4_scale(gmax);
    if (blockIdx.x == 0 && threadIdx.x == 0) *d_S = c.S;
    nvfp4_tables(tb, c.S);
    const uint64_t z2 = pk(neg_zero, neg_zero);
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride)
        nvfp4_block<T, LO, NREAL, WMSE>(tb, c, w + b * 16, WMSE ? importance + (b % blocks_per_row) * 16 : nullptr,
                                        codes + b * 8, scales + b, deq ? deq + b * 16 : nullptr,
                                        loss ? loss + b : nullptr, z2, neg_zero);
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
