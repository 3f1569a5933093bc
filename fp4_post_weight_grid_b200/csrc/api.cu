// api.cu -- the C ABI declared in include/fp4q.h: argument checks, then one
// stream-ordered launch per call.  No allocation, no host synchronization.
#include <atomic>
#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

#include <cuda_runtime.h>

#include "batch.h"
#include "fp4q.h"
#include "launch.h"

namespace fp4q {

int sm_count()
{
    static std::atomic<int> cached[64];     // zero-initialized (static storage); any thread may fill a slot
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
    if (dev < 64) {
        const int c = cached[dev].load(std::memory_order_relaxed);
        if (c > 0) return c;
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    if (dev < 64) cached[dev].store(n, std::memory_order_relaxed);
    return n;
}

int resident_blocks_per_sm(const void* kernel, int threads, size_t dyn_smem)
{
    static std::mutex mu;
    static std::map<std::tuple<const void*, int, int, size_t>, int> cache;   // (kernel, device, threads, smem)
    static std::map<std::pair<const void*, int>, size_t> limit;              // (kernel, device) -> raised limit
    int dev = 0;
    cudaGetDevice(&dev);
    const auto key = std::make_tuple(kernel, dev, threads, dyn_smem);
    std::lock_guard<std::mutex> lock(mu);
    // A kernel's dynamic shared memory limit is raised, never lowered: the
    // default allows 48 KB, and setting a smaller limit for one size would make
    // a later launch of the same kernel with more (a cached size) fail.
    constexpr size_t kDefaultLimit = 48 * 1024;
    if (dyn_smem > kDefaultLimit) {
        size_t& cur = limit[std::make_pair(kernel, dev)];
        if (dyn_smem > cur) {
            if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn_smem) ==
                cudaSuccess)
                cur = dyn_smem;
            else
                (void)cudaGetLastError();    // the launch reports it; keep it out of later status checks
        }
    }
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, threads, dyn_smem) != cudaSuccess) {
        (void)cudaGetLastError();
        per_sm = 1;
    }
    if (per_sm <= 0) per_sm = 1;
    cache[key] = per_sm;
    return per_sm;
}

}  // namespace fp4q

namespace {

thread_local char g_last_cuda_error[256] = "no error";

// FP4Q_ERR_CUDA for a failed CUDA call, its message kept for fp4q_last_cuda_error.
fp4q_status cuda_failure(cudaError_t e)
{
    std::strncpy(g_last_cuda_error, cudaGetErrorString(e), sizeof(g_last_cuda_error) - 1);
    g_last_cuda_error[sizeof(g_last_cuda_error) - 1] = '\0';
    return FP4Q_ERR_CUDA;
}

fp4q_status after_launch()
{
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FP4Q_OK : cuda_failure(e);
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool valid_dtype(fp4q_dtype dt) { return dt == FP4Q_F32 || dt == FP4Q_BF16; }

// rows * cols without signed overflow
bool shape_ok(int64_t rows, int64_t cols, int64_t block)
{
    if (rows < 0 || cols < 0 || cols % block != 0) return false;
    if (cols != 0 && rows > INT64_MAX / 4 / cols) return false;
    return true;
}

// FP4Q_OK with *empty set when there is nothing to do (the data pointers of an
// empty tensor are not read and may be NULL).
fp4q_status check_quant_args(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols, int64_t block,
                             const void* codes, const void* scales, const int32_t* d_status,
                             const void* deq, const float* loss, uintptr_t codes_align, bool* empty)
{
    *empty = false;
    if (!valid_dtype(dt)) return FP4Q_ERR_DTYPE;
    if (!shape_ok(rows, cols, block)) return FP4Q_ERR_SHAPE;
    if (rows == 0 || cols == 0) { *empty = true; return FP4Q_OK; }
    if (!w || !codes || !scales || !d_status) return FP4Q_ERR_NULL;
    if (!aligned(w, 16) || !aligned(codes, codes_align) || (deq && !aligned(deq, 16)) ||
        (loss && !aligned(loss, 4)) || !aligned(d_status, 4))
        return FP4Q_ERR_ALIGN;
    return FP4Q_OK;
}

// A grouped call: every descriptor is checked before anything is enqueued;
// then the weights of each kind (kind(t): WMSE, or rotated) go out in
// launches of at most kGroupMax, in list order.  fill() sets a launch item's
// format-specific outputs.
template <typename Check, typename Kind, typename Fill, typename Launch>
fp4q_status group_call(const fp4q_batch_tensor* tensors, int32_t n, fp4q_dtype dt, int32_t* d_status,
                              Check check, Kind kind, Fill fill, Launch launch)
{
    if (!valid_dtype(dt)) return FP4Q_ERR_DTYPE;
    if (n < 0) return FP4Q_ERR_SHAPE;
    if (n == 0) return FP4Q_OK;
    if (!tensors || !d_status) return FP4Q_ERR_NULL;
    if (!aligned(d_status, 4)) return FP4Q_ERR_ALIGN;
    for (int32_t i = 0; i < n; ++i) {
        const fp4q_status st = check(tensors[i]);
        if (st != FP4Q_OK) return st;
    }
    for (int k = 0; k < 2; ++k) {
        fp4q::GroupItem items[fp4q::kGroupMax];
        int m = 0;
        for (int32_t i = 0; i < n; ++i) {
            const fp4q_batch_tensor& t = tensors[i];
            if (kind(t) != (k == 1)) continue;
            fp4q::GroupItem& it = items[m++];
            it = fp4q::GroupItem{};
            it.w = t.w;
            it.rows = t.rows;
            it.cols = t.cols;
            it.importance = t.importance;
            it.sign_masks = t.sign_masks;
            it.amax = t.amax;
            it.global_scale = t.global_scale;
            fill(it, t);
            if (m == fp4q::kGroupMax) {
                launch(items, m, k == 1);
                const fp4q_status st = after_launch();
                if (st != FP4Q_OK) return st;
                m = 0;
            }
        }
        if (m > 0) {
            launch(items, m, k == 1);
            const fp4q_status st = after_launch();
            if (st != FP4Q_OK) return st;
        }
    }
    return FP4Q_OK;
}

}  // namespace

extern "C" {

int fp4q_version(void) { return 10000; }

const char* fp4q_status_string(fp4q_status status)
{
    switch (status) {
    case FP4Q_OK: return "ok";
    case FP4Q_ERR_NULL: return "a required pointer is NULL";
    case FP4Q_ERR_SHAPE: return "invalid shape (negative size or cols not a multiple of the block size)";
    case FP4Q_ERR_DTYPE: return "unknown dtype or format";
    case FP4Q_ERR_ALIGN: return "pointer not aligned as required";
    case FP4Q_ERR_NONFINITE: return "non-finite input";
    case FP4Q_ERR_CUDA: return "CUDA launch error";
    case FP4Q_ERR_RANGE: return "max|x| outside the supported range";
    case FP4Q_ERR_ARG: return "invalid argument (workspace too small)";
    }
    return "unknown status";
}

const char* fp4q_last_cuda_error(void) { return g_last_cuda_error; }

fp4q_status fp4q_global_absmax(const void* x, fp4q_dtype dt, int64_t n, float* d_amax,
                               int32_t* d_status, fp4q_stream_t stream)
{
    if (!valid_dtype(dt)) return FP4Q_ERR_DTYPE;
    if (n < 0) return FP4Q_ERR_SHAPE;
    if (!d_amax || (n > 0 && !x)) return FP4Q_ERR_NULL;
    if ((x && !aligned(x, 16)) || !aligned(d_amax, 4) || (d_status && !aligned(d_status, 4)))
        return FP4Q_ERR_ALIGN;
    fp4q::launch_absmax(x, dt == FP4Q_BF16, n, d_amax, d_status, reinterpret_cast<cudaStream_t>(stream));
    return after_launch();
}

static fp4q_status nvfp4_common(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                                const float* d_amax, const float* importance, bool weighted,
                                uint8_t* codes, uint8_t* scales, float* d_S, void* deq,
                                float* loss, int32_t* d_status, fp4q_stream_t stream)
{
    bool empty = false;
    fp4q_status st = check_quant_args(w, dt, rows, cols, FP4Q_NVFP4_BLOCK, codes, scales, d_status,
                                      deq, loss, 8, &empty);
    if (st != FP4Q_OK || empty) return st;
    if (!d_amax || !d_S || (weighted && !importance)) return FP4Q_ERR_NULL;
    if (!aligned(d_amax, 4) || !aligned(d_S, 4) || (weighted && !aligned(importance, 16)))
        return FP4Q_ERR_ALIGN;
    fp4q::launch_nvfp4_sweep(w, dt == FP4Q_BF16, rows, cols, d_amax, weighted ? importance : nullptr,
                             codes, scales, d_S, deq, loss, d_status,
                             reinterpret_cast<cudaStream_t>(stream));
    return after_launch();
}

fp4q_status fp4q_nvfp4_sweepmse(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                                const float* d_amax, uint8_t* codes, uint8_t* scales_e4m3,
                                float* d_global_scale, void* deq, float* block_loss,
                                int32_t* d_status, fp4q_stream_t stream)
{
    return nvfp4_common(w, dt, rows, cols, d_amax, nullptr, false, codes, scales_e4m3,
                        d_global_scale, deq, block_loss, d_status, stream);
}

fp4q_status fp4q_nvfp4_sweepwmse(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                                 const float* d_amax, const float* importance, uint8_t* codes,
                                 uint8_t* scales_e4m3, float* d_global_scale, void* deq,
                                 float* block_loss, int32_t* d_status, fp4q_stream_t stream)
{
    return nvfp4_common(w, dt, rows, cols, d_amax, importance, true, codes, scales_e4m3,
                        d_global_scale, deq, block_loss, d_status, stream);
}

static fp4q_status mxfp4_common(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                                const uint32_t* masks, bool rotate, uint8_t* codes, uint8_t* scales,
                                void* deq, float* loss, int32_t* d_status, fp4q_stream_t stream)
{
    bool empty = false;
    fp4q_status st = check_quant_args(w, dt, rows, cols, FP4Q_MXFP4_BLOCK, codes, scales, d_status,
                                      deq, loss, 16, &empty);
    if (st != FP4Q_OK || empty) return st;
    if (rotate && !masks) return FP4Q_ERR_NULL;
    if (rotate && !aligned(masks, 4)) return FP4Q_ERR_ALIGN;
    fp4q::launch_mxfp4(w, dt == FP4Q_BF16, rows, cols, rotate ? masks : nullptr, codes, scales, deq,
                       loss, d_status, nullptr, reinterpret_cast<cudaStream_t>(stream));
    return after_launch();
}

fp4q_status fp4q_mxfp4_quant(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                             uint8_t* codes, uint8_t* scales_e8m0, void* deq, float* block_loss,
                             int32_t* d_status, fp4q_stream_t stream)
{
    return mxfp4_common(w, dt, rows, cols, nullptr, false, codes, scales_e8m0, deq, block_loss,
                        d_status, stream);
}

fp4q_status fp4q_mxfp4_quant_hadamard(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                                      const uint32_t* sign_masks, uint8_t* codes,
                                      uint8_t* scales_e8m0, void* deq, float* block_loss,
                                      int32_t* d_status, fp4q_stream_t stream)
{
    return mxfp4_common(w, dt, rows, cols, sign_masks, true, codes, scales_e8m0, deq, block_loss,
                        d_status, stream);
}

fp4q_status fp4q_mxfp4_quant_absmax(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                                    const uint32_t* sign_masks, uint8_t* codes, uint8_t* scales_e8m0,
                                    void* deq, float* block_loss, float* d_amax, int32_t* d_status,
                                    fp4q_stream_t stream)
{
    if (!valid_dtype(dt)) return FP4Q_ERR_DTYPE;
    if (!shape_ok(rows, cols, FP4Q_MXFP4_BLOCK)) return FP4Q_ERR_SHAPE;
    if (!d_amax) return FP4Q_ERR_NULL;
    if (!aligned(d_amax, 4)) return FP4Q_ERR_ALIGN;
    if (rows == 0 || cols == 0) {      // max over no elements: 0
        cudaMemsetAsync(d_amax, 0, sizeof(float), reinterpret_cast<cudaStream_t>(stream));
        return after_launch();
    }
    bool empty = false;
    fp4q_status st = check_quant_args(w, dt, rows, cols, FP4Q_MXFP4_BLOCK, codes, scales_e8m0, d_status,
                                      deq, block_loss, 16, &empty);
    if (st != FP4Q_OK) return st;
    if (sign_masks && !aligned(sign_masks, 4)) return FP4Q_ERR_ALIGN;
    fp4q::launch_mxfp4(w, dt == FP4Q_BF16, rows, cols, sign_masks, codes, scales_e8m0, deq, block_loss,
                       d_status, d_amax, reinterpret_cast<cudaStream_t>(stream));
    return after_launch();
}

fp4q_status fp4q_quantize_dual(const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                               const float* importance, const uint32_t* sign_masks, float* d_amax,
                               uint8_t* nv_codes, uint8_t* nv_scales, float* d_global_scale,
                               void* nv_deq, float* nv_loss, uint8_t* mx_codes, uint8_t* mx_scales,
                               void* mx_deq, float* mx_loss, int32_t* d_status, fp4q_stream_t stream)
{
    bool empty = false;
    fp4q_status st = check_quant_args(w, dt, rows, cols, FP4Q_MXFP4_BLOCK, nv_codes, nv_scales,
                                      d_status, nv_deq, nv_loss, 8, &empty);
    if (st != FP4Q_OK) return st;
    if (!d_amax || !d_global_scale) return FP4Q_ERR_NULL;
    if (!aligned(d_amax, 4) || !aligned(d_global_scale, 4) || (importance && !aligned(importance, 16)))
        return FP4Q_ERR_ALIGN;
    if (empty) return fp4q_mxfp4_quant_absmax(w, dt, rows, cols, sign_masks, mx_codes, mx_scales,
                                              mx_deq, mx_loss, d_amax, d_status, stream);
    st = fp4q_mxfp4_quant_absmax(w, dt, rows, cols, sign_masks, mx_codes, mx_scales, mx_deq, mx_loss,
                                 d_amax, d_status, stream);
    if (st != FP4Q_OK) return st;
    return nvfp4_common(w, dt, rows, cols, d_amax, importance, importance != nullptr, nv_codes, nv_scales,
                        d_global_scale, nv_deq, nv_loss, d_status, stream);
}

fp4q_status fp4q_focus_quant(fp4q_format fmt, const void* w, fp4q_dtype dt, int64_t rows, int64_t cols,
                             const uint8_t* scales, const float* d_global_scale, const void* coeffs_f16,
                             int32_t sub_block, uint8_t* codes, void* deq, float* block_loss, int32_t* d_status,
                             fp4q_stream_t stream)
{
    if (fmt != FP4Q_NVFP4 && fmt != FP4Q_MXFP4) return FP4Q_ERR_DTYPE;
    const bool mx = fmt == FP4Q_MXFP4;
    const int64_t bs = mx ? FP4Q_MXFP4_BLOCK : FP4Q_NVFP4_BLOCK;
    if (!(sub_block == 4 || sub_block == 8 || sub_block == 16 || (mx && sub_block == 32))) return FP4Q_ERR_ARG;
    bool empty = false;
    fp4q_status st = check_quant_args(w, dt, rows, cols, bs, codes, scales, d_status, deq, block_loss,
                                      mx ? 16 : 8, &empty);
    if (st != FP4Q_OK || empty) return st;
    if (!coeffs_f16 || (!mx && !d_global_scale)) return FP4Q_ERR_NULL;
    if (!aligned(coeffs_f16, 2) || (!mx && !aligned(d_global_scale, 4))) return FP4Q_ERR_ALIGN;
    if (!fp4q::launch_focus(mx, dt == FP4Q_BF16, sub_block, w, rows, cols, scales, d_global_scale, coeffs_f16,
                            codes, deq, block_loss, d_status, reinterpret_cast<cudaStream_t>(stream)))
        return FP4Q_ERR_ARG;
    return after_launch();
}

fp4q_status fp4q_mxfp4_unrotate(const void* y, fp4q_dtype dt, int64_t rows, int64_t cols,
                                const uint32_t* sign_masks, void* out, fp4q_stream_t stream)
{
    if (!valid_dtype(dt)) return FP4Q_ERR_DTYPE;
    if (!shape_ok(rows, cols, FP4Q_MXFP4_BLOCK)) return FP4Q_ERR_SHAPE;
    if (rows == 0 || cols == 0) return FP4Q_OK;
    if (!y || !sign_masks || !out) return FP4Q_ERR_NULL;
    if (!aligned(y, 16) || !aligned(out, 16) || !aligned(sign_masks, 4)) return FP4Q_ERR_ALIGN;
    fp4q::launch_unrotate(dt == FP4Q_BF16, y, rows, cols, sign_masks, out, reinterpret_cast<cudaStream_t>(stream));
    return after_launch();
}

size_t fp4q_gptq_workspace_bytes(int64_t rows)
{
    return rows > 0 ? fp4q::gptq_workspace_bytes(rows) : 0;
}

fp4q_status fp4q_nvfp4_gptq(float* w, int64_t rows, int64_t cols, const float* U, const float* d_amax,
                            uint8_t* codes, uint8_t* scales_e4m3, float* d_global_scale, float* deq,
                            void* workspace, size_t workspace_bytes, int32_t* d_status, fp4q_stream_t stream)
{
    bool empty = false;
    fp4q_status st = check_quant_args(w, FP4Q_F32, rows, cols, FP4Q_NVFP4_BLOCK, codes, scales_e4m3, d_status,
                                      deq, nullptr, 8, &empty);
    if (st != FP4Q_OK || empty) return st;
    if (cols > (int64_t)1 << 20) return FP4Q_ERR_SHAPE;        // U alone would be 4 TB
    if (!U || !d_amax || !d_global_scale || !workspace) return FP4Q_ERR_NULL;
    if (!aligned(U, 4) || !aligned(d_amax, 4) || !aligned(d_global_scale, 4) || !aligned(workspace, 16))
        return FP4Q_ERR_ALIGN;
    if (workspace_bytes < fp4q_gptq_workspace_bytes(rows)) return FP4Q_ERR_ARG;
    const cudaError_t e = fp4q::launch_nvfp4_gptq(w, rows, cols, U, d_amax, codes, scales_e4m3, d_global_scale, deq,
                                                  static_cast<float*>(workspace), d_status,
                                                  reinterpret_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FP4Q_OK : cuda_failure(e);
}

int64_t fp4q_mma_scale_bytes(int64_t rows, int64_t scale_cols)
{
    if (rows < 0 || scale_cols < 0 || (scale_cols != 0 && rows > INT64_MAX / 1024 / scale_cols)) return -1;
    return fp4q::mma_scale_bytes(rows, scale_cols);
}

fp4q_status fp4q_scales_to_mma_layout(const uint8_t* scales, int64_t rows, int64_t scale_cols, uint8_t* out,
                                      fp4q_stream_t stream)
{
    if (fp4q_mma_scale_bytes(rows, scale_cols) < 0) return FP4Q_ERR_SHAPE;
    if (rows == 0 || scale_cols == 0) return FP4Q_OK;
    if (!scales || !out) return FP4Q_ERR_NULL;
    if (!aligned(out, 16)) return FP4Q_ERR_ALIGN;
    fp4q::launch_mma_scale_layout(scales, rows, scale_cols, out, reinterpret_cast<cudaStream_t>(stream));
    return after_launch();
}

size_t fp4q_dynamic_workspace_bytes(void) { return 16; }

fp4q_status fp4q_nvfp4_sweep_dynamic(const void* x, fp4q_dtype dt, int64_t rows, int64_t cols,
                                     const float* importance, float* d_amax, uint8_t* codes,
                                     uint8_t* scales_e4m3, float* d_global_scale, void* deq,
                                     float* block_loss, void* workspace, size_t workspace_bytes,
                                     int32_t* d_status, fp4q_stream_t stream)
{
    if (!valid_dtype(dt)) return FP4Q_ERR_DTYPE;
    if (!shape_ok(rows, cols, FP4Q_NVFP4_BLOCK)) return FP4Q_ERR_SHAPE;
    if (!d_amax) return FP4Q_ERR_NULL;
    if (!aligned(d_amax, 4)) return FP4Q_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (rows == 0 || cols == 0) {      // max over no elements: 0
        cudaMemsetAsync(d_amax, 0, sizeof(float), s);
        return after_launch();
    }
    bool empty = false;
    fp4q_status st = check_quant_args(x, dt, rows, cols, FP4Q_NVFP4_BLOCK, codes, scales_e4m3, d_status,
                                      deq, block_loss, 8, &empty);
    if (st != FP4Q_OK) return st;
    if (!d_global_scale || !workspace) return FP4Q_ERR_NULL;
    if (!aligned(d_global_scale, 4) || !aligned(workspace, 16) || (importance && !aligned(importance, 16)))
        return FP4Q_ERR_ALIGN;
    if (workspace_bytes < fp4q_dynamic_workspace_bytes()) return FP4Q_ERR_ARG;
    const cudaError_t e = fp4q::launch_nvfp4_dynamic(x, dt == FP4Q_BF16, rows, cols, importance, d_amax, codes,
                                                     scales_e4m3, d_global_scale, deq, block_loss,
                                                     static_cast<unsigned*>(workspace), d_status, s);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();                    // a refused launch configuration is not sticky
        return cuda_failure(e);
    }
    return after_launch();
}

size_t fp4q_batch_workspace_bytes(void) { return (size_t)fp4q::kWsWords * sizeof(unsigned); }

fp4q_status fp4q_quantize_batch(const fp4q_batch_tensor* tensors, int32_t n, fp4q_dtype dt,
                                void* workspace, size_t workspace_bytes, int32_t* d_status,
                                fp4q_stream_t stream)
{
    if (!valid_dtype(dt)) return FP4Q_ERR_DTYPE;
    if (n < 0) return FP4Q_ERR_SHAPE;
    if (n == 0) return FP4Q_OK;
    if (!tensors || !workspace || !d_status) return FP4Q_ERR_NULL;
    if (!aligned(workspace, 16) || !aligned(d_status, 4)) return FP4Q_ERR_ALIGN;
    if (workspace_bytes < fp4q_batch_workspace_bytes()) return FP4Q_ERR_ARG;
    for (int32_t i = 0; i < n; ++i) {          // check every descriptor before enqueueing
        const fp4q_batch_tensor& t = tensors[i];
        bool empty = false;
        fp4q_status st = check_quant_args(t.w, dt, t.rows, t.cols, FP4Q_MXFP4_BLOCK, t.nv_codes, t.nv_scales,
                                          d_status, t.nv_deq, t.nv_loss, 8, &empty);
        if (st != FP4Q_OK) return st;
        if (!empty) {
            st = check_quant_args(t.w, dt, t.rows, t.cols, FP4Q_MXFP4_BLOCK, t.mx_codes, t.mx_scales,
                                  d_status, t.mx_deq, t.mx_loss, 16, &empty);
            if (st != FP4Q_OK) return st;
        }
        if (!t.amax || !t.global_scale) return FP4Q_ERR_NULL;
        if (!aligned(t.amax, 4) || !aligned(t.global_scale, 4) ||
            (t.importance && !aligned(t.importance, 16)) || (t.sign_masks && !aligned(t.sign_masks, 4)))
            return FP4Q_ERR_ALIGN;
    }
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    static thread_local fp4q::BatchParams p;     // ~19 KB: kept off the stack
    for (int32_t base = 0; base < n; base += fp4q::kMaxBatch) {
        const int32_t m = n - base < fp4q::kMaxBatch ? n - base : fp4q::kMaxBatch;
        std::memset(&p, 0, sizeof(p));
        p.n = m;
        int64_t item = 0;
        int seg = 0;
        auto add = [&](int t, bool nv) {
            const fp4q_batch_tensor& d = tensors[base + t];
            p.seg_start[seg] = (int32_t)item;
            p.seg_tensor[seg] = (int16_t)t;
            p.seg_nv[seg] = nv ? 1 : 0;
            item += nv ? fp4q::batch_nv_tiles(d.rows, d.cols) : fp4q::batch_mx_tiles(d.rows, d.cols);
            ++seg;
        };
        // MX(0) MX(1) NV(0) MX(2) NV(1) ... MX(m-1) NV(m-2) NV(m-1)
        add(0, false);
        for (int t = 1; t < m; ++t) {
            add(t, false);
            add(t - 1, true);
        }
        add(m - 1, true);
        if (item > INT32_MAX - 1) return FP4Q_ERR_SHAPE;
        p.seg_start[seg] = (int32_t)item;
        for (int t = 0; t < m; ++t) {
            p.t[t] = tensors[base + t];
            p.mx_tiles[t] = (int32_t)fp4q::batch_mx_tiles(p.t[t].rows, p.t[t].cols);
        }
        fp4q::launch_batch(p, dt == FP4Q_BF16, static_cast<unsigned*>(workspace), d_status, s);
        const fp4q_status st = after_launch();
        if (st != FP4Q_OK) return st;
    }
    return FP4Q_OK;
}

fp4q_status fp4q_quantize_batch_static(const fp4q_batch_tensor* tensors, int32_t n, fp4q_dtype dt,
                                       int32_t* d_status, fp4q_stream_t stream)
{
    if (n > FP4Q_BATCH_MAX) return FP4Q_ERR_ARG;    // the static scratch serves one launch
    if (n <= 0) return fp4q_quantize_batch(tensors, n, dt, nullptr, 0, d_status, stream);
    unsigned* ws = nullptr;
    size_t bytes = 0;
    const cudaError_t e = fp4q::batch_static_workspace(&ws, &bytes);
    if (e != cudaSuccess) {
        std::strncpy(g_last_cuda_error, cudaGetErrorString(e), sizeof(g_last_cuda_error) - 1);
        g_last_cuda_error[sizeof(g_last_cuda_error) - 1] = '\0';
        return FP4Q_ERR_CUDA;
    }
    return fp4q_quantize_batch(tensors, n, dt, ws, bytes, d_status, stream);
}

fp4q_status fp4q_mxfp4_quant_group(const fp4q_batch_tensor* tensors, int32_t n, fp4q_dtype dt,
                                   int32_t* d_status, fp4q_stream_t stream)
{
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    auto check = [&](const fp4q_batch_tensor& t) {
        if (!shape_ok(t.rows, t.cols, FP4Q_MXFP4_BLOCK)) return FP4Q_ERR_SHAPE;
        if (!t.amax) return FP4Q_ERR_NULL;
        if (!aligned(t.amax, 4)) return FP4Q_ERR_ALIGN;
        bool empty = false;
        const fp4q_status st = check_quant_args(t.w, dt, t.rows, t.cols, FP4Q_MXFP4_BLOCK, t.mx_codes, t.mx_scales,
                                                d_status, t.mx_deq, t.mx_loss, 16, &empty);
        if (st != FP4Q_OK) return st;
        if (!empty && t.sign_masks && !aligned(t.sign_masks, 4)) return FP4Q_ERR_ALIGN;
        return FP4Q_OK;
    };
    auto kind = [](const fp4q_batch_tensor& t) { return t.sign_masks != nullptr; };
    auto fill = [](fp4q::GroupItem& it, const fp4q_batch_tensor& t) {
        it.codes = t.mx_codes;
        it.scales = t.mx_scales;
        it.deq = t.mx_deq;
        it.loss = t.mx_loss;
    };
    auto launch = [&](const fp4q::GroupItem* items, int m, bool had) {
        fp4q::launch_mxfp4_group(items, m, dt == FP4Q_BF16, had, d_status, s);
    };
    return group_call(tensors, n, dt, d_status, check, kind, fill, launch);
}

fp4q_status fp4q_nvfp4_sweep_group(const fp4q_batch_tensor* tensors, int32_t n, fp4q_dtype dt,
                                   int32_t* d_status, fp4q_stream_t stream)
{
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    auto check = [&](const fp4q_batch_tensor& t) {
        bool empty = false;
        const fp4q_status st = check_quant_args(t.w, dt, t.rows, t.cols, FP4Q_NVFP4_BLOCK, t.nv_codes, t.nv_scales,
                                                d_status, t.nv_deq, t.nv_loss, 8, &empty);
        if (st != FP4Q_OK || empty) return st;
        if (!t.amax || !t.global_scale) return FP4Q_ERR_NULL;
        if (!aligned(t.amax, 4) || !aligned(t.global_scale, 4) || (t.importance && !aligned(t.importance, 16)))
            return FP4Q_ERR_ALIGN;
        return FP4Q_OK;
    };
    auto kind = [](const fp4q_batch_tensor& t) { return t.importance != nullptr; };
    auto fill = [](fp4q::GroupItem& it, const fp4q_batch_tensor& t) {
        it.codes = t.nv_codes;
        it.scales = t.nv_scales;
        it.deq = t.nv_deq;
        it.loss = t.nv_loss;
    };
    auto launch = [&](const fp4q::GroupItem* items, int m, bool wmse) {
        fp4q::launch_nvfp4_group(items, m, dt == FP4Q_BF16, wmse, d_status, s);
    };
    return group_call(tensors, n, dt, d_status, check, kind, fill, launch);
}

fp4q_status fp4q_dequant(fp4q_format format, const uint8_t* codes, const uint8_t* scales,
                         const float* d_global_scale, int64_t rows, int64_t cols, void* out,
                         fp4q_dtype out_dt, fp4q_stream_t stream)
{
    if (format != FP4Q_NVFP4 && format != FP4Q_MXFP4) return FP4Q_ERR_DTYPE;
    if (!valid_dtype(out_dt)) return FP4Q_ERR_DTYPE;
    const bool mx = format == FP4Q_MXFP4;
    if (!shape_ok(rows, cols, mx ? FP4Q_MXFP4_BLOCK : FP4Q_NVFP4_BLOCK)) return FP4Q_ERR_SHAPE;
    if (rows == 0 || cols == 0) return FP4Q_OK;
    if (!codes || !scales || !out || (!mx && !d_global_scale)) return FP4Q_ERR_NULL;
    if (!aligned(codes, mx ? 16 : 8) || !aligned(out, 16) || (!mx && !aligned(d_global_scale, 4)))
        return FP4Q_ERR_ALIGN;
    fp4q::launch_dequant(mx, codes, scales, d_global_scale, rows, cols, out, out_dt == FP4Q_BF16,
                         reinterpret_cast<cudaStream_t>(stream));
    return after_launch();
}

fp4q_status fp4q_probe_e2m1(const float* r, uint8_t* out, int64_t n, fp4q_stream_t stream)
{
    if (n < 0) return FP4Q_ERR_SHAPE;
    if (n == 0) return FP4Q_OK;
    if (!r || !out) return FP4Q_ERR_NULL;
    if (!aligned(r, 4)) return FP4Q_ERR_ALIGN;
    fp4q::launch_probe_e2m1(r, out, n, reinterpret_cast<cudaStream_t>(stream));
    return after_launch();
}

fp4q_status fp4q_probe_copy(const void* src, void* dst, int64_t bytes, fp4q_stream_t stream)
{
    if (bytes < 0 || bytes % 16) return FP4Q_ERR_SHAPE;
    if (bytes == 0) return FP4Q_OK;
    if (!src || !dst) return FP4Q_ERR_NULL;
    if (!aligned(src, 16) || !aligned(dst, 16)) return FP4Q_ERR_ALIGN;
    fp4q::launch_probe_copy(src, dst, bytes, reinterpret_cast<cudaStream_t>(stream));
    return after_launch();
}

fp4q_status fp4q_probe_wait(const uint32_t* flag, uint32_t target, uint32_t limit, int32_t* d_status,
                            fp4q_stream_t stream)
{
    if (!flag || !d_status) return FP4Q_ERR_NULL;
    if (!aligned(flag, 4) || !aligned(d_status, 4)) return FP4Q_ERR_ALIGN;
    if (limit > (1u << 24)) return FP4Q_ERR_ARG;
    fp4q::launch_probe_wait(flag, target, limit, d_status, reinterpret_cast<cudaStream_t>(stream));
    return after_launch();
}

fp4q_status fp4q_probe_e4m3(const float* v, uint8_t* out, int64_t n, fp4q_stream_t stream)
{
    if (n < 0) return FP4Q_ERR_SHAPE;
    if (n == 0) return FP4Q_OK;
    if (!v || !out) return FP4Q_ERR_NULL;
    if (!aligned(v, 4)) return FP4Q_ERR_ALIGN;
    fp4q::launch_probe_e4m3(v, out, n, reinterpret_cast<cudaStream_t>(stream));
    return after_launch();
}

}  // extern "C"
