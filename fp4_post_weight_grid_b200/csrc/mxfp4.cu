// mxfp4.cu -- MXFP4 kernels for one weight and for a group of weights in one
// launch: one thread per 32-element block over a grid-stride loop; the
// per-block work is mxfp4_block (mxfp4_block.cuh).
#include <type_traits>

#include "device.cuh"
#include "launch.h"
#include "mxfp4_block.cuh"

namespace fp4q {

namespace {

constexpr int kThreads = 256;

// One weight.  AMAX: also reduce max|w| of the unrotated input into
// *gmax_bits (an atomic max on the binary32 bit pattern, which keeps NaN and
// Inf), for the NVFP4 global scale of the same weight.
template <typename T, bool HAD, bool AMAX>
__global__ void __launch_bounds__(kThreads, 4)
mxfp4_kernel(const T* __restrict__ w, int64_t nblocks, int64_t blocks_per_row,
             const uint32_t* __restrict__ masks, uint8_t* __restrict__ codes,
             uint8_t* __restrict__ scales, T* __restrict__ deq, float* __restrict__ loss,
             int32_t* __restrict__ d_status, float neg_zero, unsigned* __restrict__ gmax_bits)
{
    const uint64_t z2 = pk(neg_zero, neg_zero);
    uint32_t wmax = 0;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride) {
        const uint32_t m = HAD ? __ldg(masks + (b % blocks_per_row)) : 0u;
        const uint32_t bm = mxfp4_block<T, HAD>(w + b * 32, m, codes + b * 16, scales + b,
                                                deq ? deq + b * 32 : nullptr, loss ? loss + b : nullptr,
                                                d_status, z2, neg_zero);
        if (AMAX) wmax = max(wmax, bm);
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

// Several weights in one launch, each with the fused max: weight t owns
// thread blocks [cta0, cta0 + nctas).
constexpr int kMxGroupBlocksPerSm = 2;    // grid cap of the grouped launch
struct MxGroupParams {
    int32_t n;
    struct Item {
        const void* w;
        const uint32_t* masks;
        uint8_t* codes;
        uint8_t* scales;
        void* deq;
        float* loss;
        unsigned* gmax_bits;
        int64_t nblocks, blocks_per_row, cta0, nctas;
    } t[kGroupMax];
};

// The thread block's item sits in shared memory and its pointers are read
// there (volatile, so not hoisted into registers) at every block.  Three
// thread blocks per SM, not the single-weight kernel's four: the grouped
// MXFP4 launch runs beside the NVFP4 sweep of the previous group, and fewer
// resident MXFP4 warps leave room for the sweep (whole-model step 18.33/18.25
// -> 17.93/17.90 ms on one box; two blocks per SM: 18.74 ms).
template <typename T, bool HAD>
__global__ void __launch_bounds__(kThreads, 3)
mxfp4_group_kernel(const __grid_constant__ MxGroupParams P, int32_t* __restrict__ d_status, float neg_zero)
{
    __shared__ MxGroupParams::Item item;
    __shared__ uint32_t warp_max[kThreads / 32];
    if (threadIdx.x == 0) {
        int t = 0;
        while (t + 1 < P.n && (int64_t)blockIdx.x >= P.t[t + 1].cta0) ++t;
        item = P.t[t];
    }
    __syncthreads();
    const volatile MxGroupParams::Item& it = item;
    const uint64_t z2 = pk(neg_zero, neg_zero);
    uint32_t wmax = 0;
    for (int64_t b = ((int64_t)blockIdx.x - it.cta0) * kThreads + threadIdx.x; b < it.nblocks;
         b += it.nctas * kThreads) {
        const uint32_t m = HAD ? __ldg(it.masks + (b % it.blocks_per_row)) : 0u;
        T* deq = static_cast<T*>(it.deq);
        float* loss = it.loss;
        const uint32_t bm = mxfp4_block<T, HAD>(static_cast<const T*>(it.w) + b * 32, m, it.codes + b * 16,
                                                it.scales + b, deq ? deq + b * 32 : nullptr,
                                                loss ? loss + b : nullptr, d_status, z2, neg_zero);
        wmax = max(wmax, bm);
    }
    wmax = __reduce_max_sync(0xFFFFFFFFu, wmax);
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = wmax;
    __syncthreads();
    if (threadIdx.x < 32) {
        wmax = threadIdx.x < kThreads / 32 ? warp_max[threadIdx.x] : 0u;
        wmax = __reduce_max_sync(0xFFFFFFFFu, wmax);
        if (threadIdx.x == 0 && wmax != 0u) atomicMax(it.gmax_bits, wmax);
    }
}

template <typename T, bool HAD>
void launch_group_typed(const GroupItem* items, int n, int32_t* d_status, cudaStream_t s)
{
    auto kernel = mxfp4_group_kernel<T, HAD>;
    MxGroupParams P{};
    int64_t total = 0;
    for (int i = 0; i < n; ++i) total += items[i].rows * (items[i].cols / 32);
    // At most two thread blocks per SM over the whole launch (each takes more
    // rounds), so that the pass stays beside the NVFP4 sweep for longer with
    // fewer warps instead of filling the SMs and finishing early: whole-model
    // step 17.84 -> 17.66-17.69 ms (one per SM: 20.8 ms).
    int64_t rounds = grid_rounds(kernel, kThreads, 0, total);
    const int64_t per_launch = (int64_t)kMxGroupBlocksPerSm * sm_count() * kThreads;
    if ((total + per_launch - 1) / per_launch > rounds) rounds = (total + per_launch - 1) / per_launch;
    int64_t cta = 0;
    P.n = 0;
    for (int i = 0; i < n; ++i) {
        cudaMemsetAsync(items[i].amax, 0, sizeof(float), s);     // max over no elements: 0
        const int64_t nblocks = items[i].rows * (items[i].cols / 32);
        if (nblocks == 0) continue;
        MxGroupParams::Item& d = P.t[P.n++];
        d = {items[i].w, items[i].sign_masks, items[i].codes, items[i].scales, items[i].deq, items[i].loss,
             reinterpret_cast<unsigned*>(items[i].amax), nblocks, items[i].cols / 32, cta,
             (nblocks + kThreads * rounds - 1) / (kThreads * rounds)};
        cta += d.nctas;
    }
    if (P.n == 0) return;
    kernel<<<(unsigned)cta, kThreads, 0, s>>>(P, d_status, -0.0f);
}

// Rotated bf16 with at least two blocks per thread: the next block's 64 bytes
// are loaded at the top of this block's work, so that every thread has one
// load in flight while it computes.  That holds 16 more registers (119 in all,
// two thread blocks per SM instead of four) and removes the spills of the
// 64-register form; with the load latency hidden the fewer warps issue more
// (16384x8192: 158 -> 145 us).  The column group index of the sign mask
// advances with the stride instead of a division per block.  (The plain form
// gains 131 -> 125 us alone, but it runs beside the NVFP4 sweep in the
// whole-model step, where its fewer resident warps cost more than they gain.)
constexpr int kPfThreads = 256;
#ifndef FP4Q_SIGN_TABLE
#define FP4Q_SIGN_TABLE 1
#endif
// TABLE: the sign flips come from a shared-memory table of every column
// group's 16 sign words (bit 15 and bit 31 of the bf16 pair word k carry mask
// bits 2k and 2k+1), built once per thread block and XORed into the raw words
// before they are unpacked: four 16-byte shared loads and sixteen XORs per
// block instead of a shift and a XOR per element.
template <bool AMAX, bool TABLE>
__global__ void __launch_bounds__(kPfThreads, 2)
mxfp4_rot_pf_kernel(const __nv_bfloat16* __restrict__ w, int64_t nblocks, int64_t blocks_per_row,
                const uint32_t* __restrict__ masks, uint8_t* __restrict__ codes,
                uint8_t* __restrict__ scales, __nv_bfloat16* __restrict__ deq, float* __restrict__ loss,
                int32_t* __restrict__ d_status, float neg_zero, unsigned* __restrict__ gmax_bits)
{
    extern __shared__ uint4 sign_tab[];               // TABLE: blocks_per_row x 4
    const uint64_t z2 = pk(neg_zero, neg_zero);
    uint32_t wmax = 0;
    const int64_t stride = (int64_t)gridDim.x * kPfThreads;
    const int64_t step_col = stride % blocks_per_row;
    int64_t b = (int64_t)blockIdx.x * kPfThreads + threadIdx.x;
    int64_t col = b % blocks_per_row;
    uint4 u[4];
#pragma unroll
    for (int v = 0; v < 4; ++v) u[v] = b < nblocks ? ld_stream(w + b * 32 + 8 * v) : make_uint4(0, 0, 0, 0);
    if (TABLE) {
        for (int64_t g = threadIdx.x; g < blocks_per_row; g += kPfThreads) {
            const uint32_t m = __ldg(masks + g);
            uint32_t sw[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) sw[k] = ((m >> (2 * k)) & 1u) << 15 | ((m >> (2 * k + 1)) & 1u) << 31;
#pragma unroll
            for (int v = 0; v < 4; ++v) sign_tab[g * 4 + v] = make_uint4(sw[4 * v], sw[4 * v + 1], sw[4 * v + 2], sw[4 * v + 3]);
        }
        __syncthreads();
    }
    for (; b < nblocks; b += stride) {
        const int64_t nb = b + stride;
        const __nv_bfloat16* next = nb < nblocks ? w + nb * 32 : nullptr;
        uint4 nu[4];
        uint32_t bm;
        if (TABLE) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const uint4 t = sign_tab[col * 4 + v];
                u[v] = make_uint4(u[v].x ^ t.x, u[v].y ^ t.y, u[v].z ^ t.z, u[v].w ^ t.w);
            }
            bm = mxfp4_block_pairs_of_halves<__nv_bfloat16, true, 0>(
                nullptr, 0u, codes + b * 16, scales + b, deq ? deq + b * 32 : nullptr,
                loss ? loss + b : nullptr, d_status, z2, neg_zero, u, next, nu);
        } else {
            bm = mxfp4_block_pairs_of_halves<__nv_bfloat16, true, 0>(
                nullptr, __ldg(masks + col), codes + b * 16, scales + b, deq ? deq + b * 32 : nullptr,
                loss ? loss + b : nullptr, d_status, z2, neg_zero, u, next, nu);
        }
        col += step_col;
        if (col >= blocks_per_row) col -= blocks_per_row;
#pragma unroll
        for (int v = 0; v < 4; ++v) u[v] = nu[v];
        if (AMAX) wmax = max(wmax, bm);
    }
    if (AMAX) {
        __shared__ uint32_t warp_max[kPfThreads / 32];
        wmax = __reduce_max_sync(0xFFFFFFFFu, wmax);
        if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = wmax;
        __syncthreads();
        if (threadIdx.x < 32) {
            wmax = threadIdx.x < kPfThreads / 32 ? warp_max[threadIdx.x] : 0u;
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
    if constexpr (HAD && std::is_same<T, __nv_bfloat16>::value) {
        const int64_t bpr = cols / 32;
        if (FP4Q_SIGN_TABLE && bpr <= 1024) {            // table of at most 64 KB
            auto kernel = mxfp4_rot_pf_kernel<AMAX, true>;
            const size_t tab = (size_t)bpr * sizeof(uint4) * 4;
            if (grid_rounds(kernel, kPfThreads, tab, nblocks) >= 2) {
                const int64_t grid = resident_grid(kernel, kPfThreads, tab, nblocks);
                kernel<<<(unsigned)grid, kPfThreads, tab, s>>>(
                    static_cast<const __nv_bfloat16*>(w), nblocks, bpr, masks, codes, scales,
                    static_cast<__nv_bfloat16*>(deq), loss, d_status, -0.0f, gmax_bits);
                return;
            }
        }
        if (grid_rounds(mxfp4_rot_pf_kernel<AMAX, false>, kPfThreads, 0, nblocks) >= 2) {
            const int64_t grid = resident_grid(mxfp4_rot_pf_kernel<AMAX, false>, kPfThreads, 0, nblocks);
            mxfp4_rot_pf_kernel<AMAX, false><<<(unsigned)grid, kPfThreads, 0, s>>>(
                static_cast<const __nv_bfloat16*>(w), nblocks, cols / 32, masks, codes, scales,
                static_cast<__nv_bfloat16*>(deq), loss, d_status, -0.0f, gmax_bits);
            return;
        }
    }
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

void launch_mxfp4_group(const GroupItem* items, int n, bool bf16, bool had, int32_t* d_status, cudaStream_t s)
{
    if (had) {
        if (bf16) launch_group_typed<__nv_bfloat16, true>(items, n, d_status, s);
        else launch_group_typed<float, true>(items, n, d_status, s);
    } else {
        if (bf16) launch_group_typed<__nv_bfloat16, false>(items, n, d_status, s);
        else launch_group_typed<float, false>(items, n, d_status, s);
    }
}

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
