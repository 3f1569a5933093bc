// dynamic.cu -- NVFP4 ScaleSweep of a tensor that is quantized per call, in
// one launch.
//
// ScaleSweep summary, "Resultados Experimentais": the sweep is also applied to
// activations (the weights+activations configurations); an activation is
// quantized at every forward call, so the global max and the sweep both sit
// on the inference path, where small tensors make launch latency the cost.
// Here the global max (S = max|x|/(256*6), "Metodologia" sec. 2) and the
// per-block sweep are separated by a barrier inside one launch instead of
// by a second launch.
//
// Tensors of at most 16 x 256 blocks run as one thread-block cluster
// (nvfp4_cluster_kernel): one block per thread, the thread blocks' maxima
// exchanged through distributed shared memory between two hardware cluster
// barriers.  Larger tensors use a cooperative launch (every thread block
// resident at once, nvfp4_dynamic_kernel):
//
//   phase 1  every thread block reduces max|x| over a grid-stride share of
//            the tensor and merges it into the workspace with one atomicMax,
//            then counts itself in;
//   barrier  thread 0 of each thread block waits until every thread block
//            has counted in (bounded: after about two seconds it raises
//            FP4Q_FLAG_TIMEOUT and the thread block skips the sweep);
//   phase 2  the sweep of nvfp4_block.cuh over a grid-stride share of the
//            16-element blocks.
//
// The workspace holds three counters: the max bits, the arrivals and the
// departures; the last thread block to leave the barrier zeroes all three,
// so a zeroed workspace stays zeroed from call to call.  Both kernels use the
// per-block arithmetic of the two-launch path (fp4q_global_absmax +
// fp4q_nvfp4_sweep{mse,wmse}), so the bytes are the same.
#include <cooperative_groups.h>

#include "device.cuh"
#include "launch.h"
#include "nvfp4_block.cuh"
#include "wait.cuh"

namespace cg = cooperative_groups;

namespace fp4q {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ unsigned ld_volatile(const unsigned* p)
{
    return *reinterpret_cast<const volatile unsigned*>(p);
}

template <typename T, int LO, int NREAL, bool WMSE>
__global__ void __launch_bounds__(kThreads, WMSE ? 3 : 5)
nvfp4_dynamic_kernel(const T* __restrict__ w, int64_t nblocks, int64_t blocks_per_row,
                     const float* __restrict__ importance, float* __restrict__ d_amax,
                     uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, float* __restrict__ d_S,
                     T* __restrict__ deq, float* __restrict__ loss, unsigned* __restrict__ ws,
                     int32_t* __restrict__ d_status, float neg_zero)
{
    __shared__ NvTables tb;
    __shared__ uint32_t warp_max[kThreads / 32];
    __shared__ unsigned s_gmax, s_skip;

    // phase 1: max |x| (binary32 bits) over this thread block's share
    constexpr int kPerVec = sizeof(T) == 2 ? 8 : 4;
    const int64_t nvec = nblocks * (16 / kPerVec);
    const uint4* v = reinterpret_cast<const uint4*>(w);
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    uint32_t m = 0;
    for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < nvec; i += stride) {
        const uint4 u = ld_stream(v + i);
        if (sizeof(T) == 2) {
            m = __vmaxu2(m, __vmaxu2(u.x & 0x7FFF7FFFu, u.y & 0x7FFF7FFFu));
            m = __vmaxu2(m, __vmaxu2(u.z & 0x7FFF7FFFu, u.w & 0x7FFF7FFFu));
        } else {
            m = max(m, max(max(u.x & 0x7FFFFFFFu, u.y & 0x7FFFFFFFu), max(u.z & 0x7FFFFFFFu, u.w & 0x7FFFFFFFu)));
        }
    }
    if (sizeof(T) == 2) m = max(m & 0xFFFFu, m >> 16) << 16;     // bf16 pattern -> binary32 pattern
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = threadIdx.x < kThreads / 32 ? warp_max[threadIdx.x] : 0u;
        m = __reduce_max_sync(0xFFFFFFFFu, m);
        if (threadIdx.x == 0) {
            // barrier: count in, wait for every thread block, read the max
            if (m != 0u) atomicMax(ws, m);
            __threadfence();
            atomicAdd(ws + 1, 1u);
            unsigned skip = 0;
            if (!wait_geq(ws + 1, gridDim.x, kWaitLimit)) {
                atomicOr(d_status, kFlagTimeout);
                skip = 1;
            }
            __threadfence();
            s_gmax = ld_volatile(ws);
            s_skip = skip;
            __threadfence();                         // the max is read before counting out
            if (!skip && atomicAdd(ws + 2, 1u) == gridDim.x - 1) {
                ws[0] = 0u;                          // last one out: leave the workspace zeroed
                ws[1] = 0u;
                ws[2] = 0u;
            }
        }
    }
    __syncthreads();

    // phase 2: the sweep with the global scale of the whole tensor
    const float gmax = __uint_as_float(s_gmax);
    const int32_t flag = nvfp4_gmax_flag(gmax);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *d_amax = gmax;
        if (flag) atomicOr(d_status, flag);
    }
    if (s_skip || flag) return;                      // uniform across the thread block
    const NvScale c = nvfp4_scale(gmax);
    if (blockIdx.x == 0 && threadIdx.x == 0) *d_S = c.S;
    nvfp4_tables(tb, c.S);
    const uint64_t z2 = pk(neg_zero, neg_zero);
    for (int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x; b < nblocks; b += stride)
        nvfp4_block<T, LO, NREAL, WMSE>(tb, c, w + b * 16, WMSE ? importance + (b % blocks_per_row) * 16 : nullptr,
                                        codes + b * 8, scales + b, deq ? deq + b * 16 : nullptr,
                                        loss ? loss + b : nullptr, z2, neg_zero);
}

// Small tensors (at most kMaxCluster * kThreads blocks, one per thread): one
// thread-block cluster.  The thread blocks exchange their maxima through
// distributed shared memory between two hardware cluster barriers, so there
// is no workspace, no atomic and no polling; the hardware schedules the
// thread blocks of a cluster together, so the barriers always complete.
constexpr int kMaxCluster = 16;

template <typename T, int LO, int NREAL, bool WMSE>
__global__ void __launch_bounds__(kThreads)
nvfp4_cluster_kernel(const T* __restrict__ w, int64_t nblocks, int64_t blocks_per_row,
                     const float* __restrict__ importance, float* __restrict__ d_amax,
                     uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, float* __restrict__ d_S,
                     T* __restrict__ deq, float* __restrict__ loss, int32_t* __restrict__ d_status,
                     float neg_zero)
{
    __shared__ NvTables tb;
    __shared__ uint32_t warp_max[kThreads / 32];
    __shared__ uint32_t cta_max;
    cg::cluster_group cluster = cg::this_cluster();

    // phase 1: max |x| of this thread's block, then of the thread block
    const int64_t b = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    uint32_t m = 0;
    if (b < nblocks) {
        float x[16];
        load_block_amax<16>(w + b * 16, x, m);
    }
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = threadIdx.x < kThreads / 32 ? warp_max[threadIdx.x] : 0u;
        m = __reduce_max_sync(0xFFFFFFFFu, m);
        if (threadIdx.x == 0) cta_max = m;
    }
    cluster.sync();                                  // every thread block's maximum is in place
    uint32_t g = 0;
    for (unsigned r = 0; r < cluster.num_blocks(); ++r)
        g = max(g, *cluster.map_shared_rank(&cta_max, r));
    cluster.sync();                                  // no thread block leaves while its maximum is read

    // phase 2: the sweep with the global scale of the whole tensor
    const float gmax = __uint_as_float(g);
    const int32_t flag = nvfp4_gmax_flag(gmax);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *d_amax = gmax;
        if (flag) atomicOr(d_status, flag);
    }
    if (flag) return;                                // uniform across the cluster
    const NvScale c = nvfp4_scale(gmax);
    if (blockIdx.x == 0 && threadIdx.x == 0) *d_S = c.S;
    nvfp4_tables(tb, c.S);
    if (b < nblocks)
        nvfp4_block<T, LO, NREAL, WMSE>(tb, c, w + b * 16, WMSE ? importance + (b % blocks_per_row) * 16 : nullptr,
                                        codes + b * 8, scales + b, deq ? deq + b * 16 : nullptr,
                                        loss ? loss + b : nullptr, pk(neg_zero, neg_zero), neg_zero);
}

template <typename T, int LO, int NREAL, bool WMSE>
cudaError_t launch_cluster(const void* w, int64_t rows, int64_t cols, const float* importance, float* d_amax,
                           uint8_t* codes, uint8_t* scales, float* d_S, void* deq, float* loss, int32_t* d_status,
                           cudaStream_t s)
{
    auto kernel = nvfp4_cluster_kernel<T, LO, NREAL, WMSE>;
    static bool attr_set[64] = {};                   // per device; a race only repeats the call
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        cudaFuncSetAttribute(reinterpret_cast<const void*>(kernel), cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        if (dev >= 0 && dev < 64) attr_set[dev] = true;
    }
    const int64_t nblocks = rows * (cols / 16);
    const unsigned grid = (unsigned)((nblocks + kThreads - 1) / kThreads);
    const T* wp = static_cast<const T*>(w);
    int64_t bpr = cols / 16;
    T* dq = static_cast<T*>(deq);
    float nz = -0.0f;
    void* args[] = {&wp, (void*)&nblocks, &bpr, &importance, &d_amax, &codes, &scales, &d_S, &dq, &loss,
                    &d_status, &nz};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = grid;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(kernel), args);
}

template <typename T, int LO, int NREAL, bool WMSE>
cudaError_t launch_typed(const void* w, int64_t rows, int64_t cols, const float* importance, float* d_amax,
                         uint8_t* codes, uint8_t* scales, float* d_S, void* deq, float* loss, unsigned* ws,
                         int32_t* d_status, cudaStream_t s)
{
    auto kernel = nvfp4_dynamic_kernel<T, LO, NREAL, WMSE>;
    const int64_t nblocks = rows * (cols / 16);
    if (nblocks <= (int64_t)kMaxCluster * kThreads) {
        const cudaError_t e = launch_cluster<T, LO, NREAL, WMSE>(w, rows, cols, importance, d_amax, codes, scales,
                                                                 d_S, deq, loss, d_status, s);
        if (e == cudaSuccess) return e;
        (void)cudaGetLastError();                    // no such cluster here: use the grid barrier
    }
    // at most one thread block per resident slot: the barrier needs them all at once
    const int64_t cap = (int64_t)resident_blocks_per_sm(reinterpret_cast<const void*>(kernel), kThreads, 0) *
                        sm_count();
    int64_t grid = (nblocks + kThreads - 1) / kThreads;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;

    const T* wp = static_cast<const T*>(w);
    int64_t bpr = cols / 16;
    T* dq = static_cast<T*>(deq);
    float nz = -0.0f;
    void* args[] = {&wp, (void*)&nblocks, &bpr, &importance, &d_amax, &codes, &scales, &d_S, &dq, &loss, &ws,
                    &d_status, &nz};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, reinterpret_cast<const void*>(kernel), args);
}

}  // namespace

cudaError_t launch_nvfp4_dynamic(const void* w, bool bf16, int64_t rows, int64_t cols, const float* importance,
                                 float* d_amax, uint8_t* codes, uint8_t* scales, float* d_S, void* deq,
                                 float* loss, unsigned* ws, int32_t* d_status, cudaStream_t s)
{
    if (importance == nullptr) {
        if (bf16)
            return launch_typed<__nv_bfloat16, -3, 11, false>(w, rows, cols, nullptr, d_amax, codes, scales, d_S,
                                                               deq, loss, ws, d_status, s);
        return launch_typed<float, -3, 11, false>(w, rows, cols, nullptr, d_amax, codes, scales, d_S, deq, loss,
                                                  ws, d_status, s);
    }
    if (bf16)
        return launch_typed<__nv_bfloat16, -8, 16, true>(w, rows, cols, importance, d_amax, codes, scales, d_S,
                                                          deq, loss, ws, d_status, s);
    return launch_typed<float, -8, 16, true>(w, rows, cols, importance, d_amax, codes, scales, d_S, deq, loss,
                                             ws, d_status, s);
}

}  // namespace fp4q
