// nvfp4.cu -- NVFP4 ScaleSweep kernels for one weight and for a group of
// weights in one launch: one thread per 16-element block over a grid-stride
// loop; the per-block search is nvfp4_block (nvfp4_block.cuh), the global
// scale comes from *d_amax (ScaleSweep summary, "Metodologia: ScaleSweep"
// sec. 2).
#include "device.cuh"
#include "launch.h"
#include "nvfp4_block.cuh"

namespace fp4q {

namespace {

constexpr int kThreads = 256;

// The sweep of one weight by thread blocks cta = 0 .. nctas-1 of a launch.
template <typename T, int LO, int NREAL, bool WMSE>
__device__ __forceinline__ void nvfp4_sweep_body(NvTables& tb, const T* __restrict__ w, int64_t nblocks,
                                                 int64_t blocks_per_row, const float* __restrict__ d_amax,
                                                 const float* __restrict__ importance, uint8_t* __restrict__ codes,
                                                 uint8_t* __restrict__ scales, float* __restrict__ d_S,
                                                 T* __restrict__ deq, float* __restrict__ loss,
                                                 int32_t* __restrict__ d_status, float neg_zero, unsigned cta,
                                                 unsigned nctas)
{
    const float gmax = __ldg(d_amax);
    const int32_t flag = nvfp4_gmax_flag(gmax);
    if (flag) {                                  // uniform across the thread block
        if (cta == 0 && threadIdx.x == 0) atomicOr(d_status, flag);
        return;
    }
    const NvScale c = nvfp4_scale(gmax);
    if (cta == 0 && threadIdx.x == 0) *d_S = c.S;
    nvfp4_tables(tb, c.S);
    const uint64_t z2 = pk(neg_zero, neg_zero);
    const int64_t stride = (int64_t)nctas * kThreads;
    for (int64_t b = (int64_t)cta * kThreads + threadIdx.x; b < nblocks; b += stride)
        nvfp4_block<T, LO, NREAL, WMSE>(tb, c, w + b * 16, WMSE ? importance + (b % blocks_per_row) * 16 : nullptr,
                                        codes + b * 8, scales + b, deq ? deq + b * 16 : nullptr,
                                        loss ? loss + b : nullptr, z2, neg_zero);
}

template <typename T, int LO, int NREAL, bool WMSE>
__global__ void __launch_bounds__(kThreads, WMSE ? 3 : 5)
nvfp4_sweep_kernel(const T* __restrict__ w, int64_t nblocks, int64_t blocks_per_row,
                   const float* __restrict__ d_amax, const float* __restrict__ importance,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                   float* __restrict__ d_S, T* __restrict__ deq, float* __restrict__ loss,
                   int32_t* __restrict__ d_status, float neg_zero)
{
    __shared__ NvTables tb;
    nvfp4_sweep_body<T, LO, NREAL, WMSE>(tb, w, nblocks, blocks_per_row, d_amax, importance, codes, scales, d_S,
                                         deq, loss, d_status, neg_zero, blockIdx.x, gridDim.x);
}

// Several weights in one launch: weight t owns thread blocks
// [cta0, cta0 + nctas); a thread block works on its own weight only (its
// tables are that weight's), exactly as the single-weight kernel would.
struct NvGroupParams {
    int32_t n;
    struct Item {
        const void* w;
        const float* amax;
        const float* importance;
        uint8_t* codes;
        uint8_t* scales;
        float* S;
        void* deq;
        float* loss;
        int64_t nblocks, blocks_per_row, cta0, nctas;
    } t[kGroupMax];
};

template <typename T, int LO, int NREAL, bool WMSE>
__global__ void __launch_bounds__(kThreads, WMSE ? 3 : 5)
nvfp4_group_kernel(const __grid_constant__ NvGroupParams P, int32_t* __restrict__ d_status, float neg_zero)
{
    __shared__ NvTables tb;
    int t = 0;
    while (t + 1 < P.n && (int64_t)blockIdx.x >= P.t[t + 1].cta0) ++t;
    const NvGroupParams::Item& it = P.t[t];
    nvfp4_sweep_body<T, LO, NREAL, WMSE>(tb, static_cast<const T*>(it.w), it.nblocks, it.blocks_per_row, it.amax,
                                         it.importance, it.codes, it.scales, it.S, static_cast<T*>(it.deq),
                                         it.loss, d_status, neg_zero, (unsigned)(blockIdx.x - it.cta0), (unsigned)it.nctas);
}

template <typename T, int LO, int NREAL, bool WMSE>
void launch_group_typed(const GroupItem* items, int n, int32_t* d_status, cudaStream_t s)
{
    auto kernel = nvfp4_group_kernel<T, LO, NREAL, WMSE>;
    NvGroupParams P{};
    int64_t total = 0;
    for (int i = 0; i < n; ++i) total += items[i].rows * (items[i].cols / 16);
    const int64_t rounds = grid_rounds(kernel, kThreads, 0, total);
    int64_t cta = 0;
    P.n = 0;
    for (int i = 0; i < n; ++i) {
        const int64_t nblocks = items[i].rows * (items[i].cols / 16);
        if (nblocks == 0) continue;                  // nothing to write, as the single call
        NvGroupParams::Item& d = P.t[P.n++];
        d = {items[i].w, items[i].amax, items[i].importance, items[i].codes, items[i].scales,
             items[i].global_scale, items[i].deq, items[i].loss, nblocks, items[i].cols / 16, cta,
             (nblocks + kThreads * rounds - 1) / (kThreads * rounds)};
        cta += d.nctas;
    }
    if (P.n == 0) return;
    kernel<<<(unsigned)cta, kThreads, 0, s>>>(P, d_status, -0.0f);
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

void launch_nvfp4_group(const GroupItem* items, int n, bool bf16, bool wmse, int32_t* d_status, cudaStream_t s)
{
    if (!wmse) {
        if (bf16) launch_group_typed<__nv_bfloat16, -3, 11, false>(items, n, d_status, s);
        else launch_group_typed<float, -3, 11, false>(items, n, d_status, s);
    } else {
        if (bf16) launch_group_typed<__nv_bfloat16, -8, 16, true>(items, n, d_status, s);
        else launch_group_typed<float, -8, 16, true>(items, n, d_status, s);
    }
}

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
