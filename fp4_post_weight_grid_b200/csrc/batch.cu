// batch.cu -- one persistent launch that quantizes a list of weights to both
// NVFP4 (ScaleSweep) and MXFP4 (E8M0 sweep).
//
// NVFP4 needs each weight's global max before any of its blocks can be swept
// (ScaleSweep summary, "Metodologia: ScaleSweep" sec. 2: S = max|x|/(256*6));
// the MXFP4 pass computes every block's max anyway.  The kernel therefore
// works through a queue of tiles (16384 elements each) in the order
//   MX(0) MX(1) NV(0) MX(2) NV(1) ... MX(n-1) NV(n-2) NV(n-1)
// where MX(t) are the MXFP4 tiles of weight t (which also merge max|w| into a
// per-weight counter) and NV(t) its NVFP4 tiles.  A thread block takes the
// next tile with one atomic add.  Before an NV(t) tile it waits until every
// MX(t) tile has finished; those tiles were all taken from the queue before
// any NV(t) tile, by thread blocks that are running and never wait
// themselves, so the wait always ends (it is also bounded: after about two
// seconds the tile is skipped and FP4Q_FLAG_TIMEOUT is raised).  Memory-bound
// MXFP4 tiles and arithmetic-bound NVFP4 tiles are resident on the same SMs at
// the same time, and the whole list costs one launch.
//
// The per-block arithmetic is exactly that of the single-weight kernels
// (nvfp4_block.cuh, mxfp4_block.cuh), so the results are bit-identical.  The
// MXFP4 tiles use the neighbour-paired form for both plain and rotated
// blocks: one kernel holds both, and the half-paired form's extra registers
// would spill here.
#include <mutex>

#include "batch.h"
#include "device.cuh"
#include "launch.h"
#include "mxfp4_block.cuh"
#include "nvfp4_block.cuh"
#include "wait.cuh"

namespace fp4q {

namespace {

constexpr int kThreads = 256;
constexpr int kMxBlocksPerThread = 2;   // 512 MXFP4 blocks = 16384 elements per tile
constexpr int kNvBlocksPerThread = 4;   // 1024 NVFP4 blocks = 16384 elements per tile

__device__ __forceinline__ unsigned ld_volatile(const unsigned* p)
{
    return *reinterpret_cast<const volatile unsigned*>(p);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, 4)
batch_kernel(const __grid_constant__ BatchParams P, unsigned* __restrict__ ws, int32_t* __restrict__ d_status,
             float neg_zero)
{
    __shared__ NvTables tb;
    __shared__ int s_item, s_seg;
    __shared__ unsigned s_gmax, s_skip;
    __shared__ uint32_t warp_max[kThreads / 32];
    unsigned* queue = ws;
    unsigned* gmax = ws + kWsHeader;
    unsigned* done = ws + kWsHeader + kMaxBatch;
    const uint64_t z2 = pk(neg_zero, neg_zero);
    int tables_for = -1;        // the weight whose NVFP4 tables are in shared memory
    NvScale c{};

    for (;;) {
        if (threadIdx.x == 0) {
            const int item = (int)atomicAdd(queue, 1u);
            int lo = 0, hi = 2 * P.n;               // seg_start[lo] <= item < seg_start[hi]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (P.seg_start[mid] <= item) lo = mid; else hi = mid;
            }
            s_item = item;
            s_seg = lo;
        }
        __syncthreads();
        const int item = s_item;
        if (item >= P.seg_start[2 * P.n]) break;
        const int seg = s_seg;
        const int t = P.seg_tensor[seg];
        const int tile = item - P.seg_start[seg];
        const BatchTensor& d = P.t[t];

        if (!P.seg_nv[seg]) {
            // ---------------- MXFP4 tile of weight t (and its max |w|)
            const int64_t nb = d.rows * (d.cols / 32);
            const int64_t bpr = d.cols / 32;
            uint32_t m = 0;
#pragma unroll 1
            for (int j = 0; j < kMxBlocksPerThread; ++j) {
                const int64_t b = (int64_t)tile * (kThreads * kMxBlocksPerThread) + j * kThreads + threadIdx.x;
                if (b >= nb) break;
                const T* src = static_cast<const T*>(d.w) + b * 32;
                T* dq = d.mx_deq ? static_cast<T*>(d.mx_deq) + b * 32 : nullptr;
                float* ls = d.mx_loss ? d.mx_loss + b : nullptr;
                uint32_t bm;
                if (d.sign_masks)
                    bm = mxfp4_block_pairs_of_neighbours<T, true>(src, __ldg(d.sign_masks + (b % bpr)), d.mx_codes + b * 16,
                                              d.mx_scales + b, dq, ls, d_status, z2, neg_zero);
                else
                    bm = mxfp4_block_pairs_of_neighbours<T, false>(src, 0u, d.mx_codes + b * 16, d.mx_scales + b, dq, ls,
                                               d_status, z2, neg_zero);
                m = max(m, bm);
            }
            m = __reduce_max_sync(0xFFFFFFFFu, m);
            if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
            __syncthreads();
            if (threadIdx.x < 32) {
                m = threadIdx.x < kThreads / 32 ? warp_max[threadIdx.x] : 0u;
                m = __reduce_max_sync(0xFFFFFFFFu, m);
                if (threadIdx.x == 0) {
                    if (m != 0u) atomicMax(gmax + t, m);
                    __threadfence();                 // outputs and max before the count
                    atomicAdd(done + t, 1u);
                }
            }
        } else {
            // ---------------- NVFP4 tile of weight t: wait for its max
            if (threadIdx.x == 0) {
                unsigned skip = 0;
                if (!wait_geq(done + t, (unsigned)P.mx_tiles[t], kWaitLimit)) {
                    atomicOr(d_status, kFlagTimeout);
                    skip = 1;
                }
                __threadfence();
                s_gmax = ld_volatile(gmax + t);
                s_skip = skip;
            }
            __syncthreads();
            const float g = __uint_as_float(s_gmax);
            const int32_t flag = nvfp4_gmax_flag(g);
            if (tile == 0 && threadIdx.x == 0) {
                *d.amax = g;
                if (flag) atomicOr(d_status, flag);
            }
            if (!s_skip && !flag) {
                if (tables_for != t) {               // uniform across the thread block
                    c = nvfp4_scale(g);
                    nvfp4_tables(tb, c.S);
                    tables_for = t;
                }
                if (tile == 0 && threadIdx.x == 0) *d.global_scale = c.S;
                const int64_t nb = d.rows * (d.cols / 16);
                const int64_t bpr = d.cols / 16;
#pragma unroll 1
                for (int j = 0; j < kNvBlocksPerThread; ++j) {
                    const int64_t b = (int64_t)tile * (kThreads * kNvBlocksPerThread) + j * kThreads + threadIdx.x;
                    if (b >= nb) break;
                    const T* src = static_cast<const T*>(d.w) + b * 16;
                    T* dq = d.nv_deq ? static_cast<T*>(d.nv_deq) + b * 16 : nullptr;
                    float* ls = d.nv_loss ? d.nv_loss + b : nullptr;
                    if (d.importance)
                        nvfp4_block<T, -8, 16, true>(tb, c, src, d.importance + (b % bpr) * 16, d.nv_codes + b * 8,
                                                      d.nv_scales + b, dq, ls, z2, neg_zero);
                    else
                        nvfp4_block<T, -3, 11, false>(tb, c, src, nullptr, d.nv_codes + b * 8, d.nv_scales + b,
                                                       dq, ls, z2, neg_zero);
                }
            }
        }
        __syncthreads();        // s_item, s_gmax and the tables are reused by the next tile
    }
}

}  // namespace

// Scratch of fp4q_quantize_batch_static: the tile queue counter and the
// per-weight max and completion counters of one launch (kWsWords words).  It
// lives in the library's own device memory, so every GPU that loads the
// library holds it until the process exits; host code only ever sees a
// stand-in for it and gets its device address from cudaGetSymbolAddress.
static __device__ __align__(256) unsigned g_static_ws[kWsWords];

cudaError_t batch_static_workspace(unsigned** ws, size_t* bytes)
{
    static std::mutex mu;
    static unsigned* addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {                       // once per device, with that device current
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_ws);
        if (e != cudaSuccess) return e;
        addr[dev] = static_cast<unsigned*>(p);
    }
    *ws = addr[dev];
    *bytes = sizeof(g_static_ws);
    return cudaSuccess;
}

int64_t batch_mx_tiles(int64_t rows, int64_t cols)
{
    const int64_t per = (int64_t)kThreads * kMxBlocksPerThread;
    return (rows * (cols / 32) + per - 1) / per;
}

int64_t batch_nv_tiles(int64_t rows, int64_t cols)
{
    const int64_t per = (int64_t)kThreads * kNvBlocksPerThread;
    const int64_t n = (rows * (cols / 16) + per - 1) / per;
    return n < 1 ? 1 : n;           // an empty weight still gets a tile that writes max and S
}

void launch_batch(const BatchParams& p, bool bf16, unsigned* ws, int32_t* d_status, cudaStream_t s)
{
    cudaMemsetAsync(ws, 0, kWsWords * sizeof(unsigned), s);
    const int64_t items = p.seg_start[2 * p.n];
    // persistent: one generation of resident thread blocks (at most one per tile)
    auto grid_for = [&](const void* k) {
        const int64_t cap = (int64_t)resident_blocks_per_sm(k, kThreads, 0) * sm_count();
        return (unsigned)(items < cap ? (items < 1 ? 1 : items) : cap);
    };
    if (bf16) {
        const unsigned grid = grid_for(reinterpret_cast<const void*>(batch_kernel<__nv_bfloat16>));
        batch_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(p, ws, d_status, -0.0f);
    } else {
        const unsigned grid = grid_for(reinterpret_cast<const void*>(batch_kernel<float>));
        batch_kernel<float><<<grid, kThreads, 0, s>>>(p, ws, d_status, -0.0f);
    }
}

}  // namespace fp4q
