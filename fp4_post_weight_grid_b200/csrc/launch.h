// launch.h -- internal launchers behind the C ABI (include/fp4q.h).
// Arguments are validated by api.cu before any of these is called.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "fp4q.h"

namespace fp4q {

// Number of SMs of the current device (cached per device).
int sm_count();

// Resident thread blocks per SM of `kernel` with `threads` threads and
// `dyn_smem` bytes of dynamic shared memory on the current device; raises the
// kernel's dynamic shared memory limit to dyn_smem when that is above the
// 48 KB default and above what was set before (never lowers it).  Cached per
// (kernel, device, threads, dyn_smem).
int resident_blocks_per_sm(const void* kernel, int threads, size_t dyn_smem);

// Grid for a grid-stride kernel: the work is split into equal shares for about
// two generations of resident thread blocks (a thread block that finishes early
// is replaced, which evens out the tail), never more blocks than the work needs.
template <typename Kernel>
inline int64_t grid_rounds(Kernel kernel, int threads, size_t dyn_smem, int64_t work_items)
{
    const int per_sm = resident_blocks_per_sm(reinterpret_cast<const void*>(kernel), threads, dyn_smem);
    const int64_t per_gen = (int64_t)per_sm * sm_count() * threads * 2;
    const int64_t rounds = (work_items + per_gen - 1) / per_gen;
    return rounds < 1 ? 1 : rounds;
}
template <typename Kernel>
inline int64_t resident_grid(Kernel kernel, int threads, size_t dyn_smem, int64_t work_items)
{
    const int64_t share = grid_rounds(kernel, threads, dyn_smem, work_items);
    const int64_t g = (work_items + threads * share - 1) / (threads * share);
    return g < 1 ? 1 : g;
}

// Global max|x| into *d_amax; with d_status != nullptr a one-warp kernel then
// flags a non-finite or out-of-range result.
void launch_absmax(const void* x, bool bf16, int64_t n, float* d_amax, int32_t* d_status, cudaStream_t s);

// One weight of a grouped launch (the fields the format's kernel reads;
// importance selects WMSE for NVFP4, sign_masks the rotation for MXFP4).
struct GroupItem {
    const void* w;
    int64_t rows, cols;
    const float* importance;
    const uint32_t* sign_masks;
    float* amax;                 // NVFP4: read; MXFP4: written (max|w|)
    float* global_scale;         // NVFP4: written
    uint8_t* codes;
    uint8_t* scales;
    void* deq;
    float* loss;
};
constexpr int kGroupMax = FP4Q_GROUP_MAX;    // weights per grouped launch

// Grouped launches over items[0..n), n <= kGroupMax, all of one dtype and one
// kind (NVFP4: all MSE or all WMSE; MXFP4: all plain or all rotated).
void launch_nvfp4_group(const GroupItem* items, int n, bool bf16, bool wmse, int32_t* d_status, cudaStream_t s);
void launch_mxfp4_group(const GroupItem* items, int n, bool bf16, bool had, int32_t* d_status, cudaStream_t s);

// NVFP4 ScaleSweep: importance == nullptr selects MSE (window -3..+7), otherwise
// WMSE (window -8..+7).
void launch_nvfp4_sweep(const void* w, bool bf16, int64_t rows, int64_t cols, const float* d_amax,
                        const float* importance, uint8_t* codes, uint8_t* scales, float* d_S,
                        void* deq, float* loss, int32_t* d_status, cudaStream_t s);

// MXFP4 with the E8M0 e0-1..e0+1 sweep; sign_masks != nullptr adds the block
// Hadamard; d_amax != nullptr also writes max|w| of the unrotated input there.
void launch_mxfp4(const void* w, bool bf16, int64_t rows, int64_t cols, const uint32_t* sign_masks,
                  uint8_t* codes, uint8_t* scales, void* deq, float* loss, int32_t* d_status,
                  float* d_amax, cudaStream_t s);

// NVFP4 global max + ScaleSweep in one cooperative launch; ws: 3 zeroed words.
cudaError_t launch_nvfp4_dynamic(const void* w, bool bf16, int64_t rows, int64_t cols, const float* importance,
                                 float* d_amax, uint8_t* codes, uint8_t* scales, float* d_S, void* deq,
                                 float* loss, unsigned* ws, int32_t* d_status, cudaStream_t s);

// FOCUS forward quantizer (mx: MXFP4 blocks of 32, else NVFP4 blocks of 16),
// sub in {4, 8, 16} (and 32 for MXFP4); false for an unsupported sub-block size.
bool launch_focus(bool mx, bool bf16, int sub, const void* w, int64_t rows, int64_t cols, const uint8_t* scales,
                  const float* d_S, const void* coeffs, uint8_t* codes, void* deq, float* loss,
                  int32_t* d_status, cudaStream_t s);

// Rotated-domain MXFP4 reconstruction back to the original domain.
void launch_unrotate(bool bf16, const void* y, int64_t rows, int64_t cols, const uint32_t* sign_masks, void* out,
                     cudaStream_t s);

// ScaleSweep inside GPTQ: w (fp32, rows x cols) is updated in place; E is the
// workspace of gptq_workspace_bytes(rows) bytes.
size_t gptq_workspace_bytes(int64_t rows);
cudaError_t launch_nvfp4_gptq(float* w, int64_t rows, int64_t cols, const float* U, const float* d_amax,
                              uint8_t* codes, uint8_t* scales, float* d_S, float* deq, float* E, int32_t* d_status,
                              cudaStream_t s);

// Block scales [rows][scols] -> the 128 x 4 tiled layout of block-scaled GEMMs.
int64_t mma_scale_bytes(int64_t rows, int64_t scols);
void launch_mma_scale_layout(const uint8_t* s, int64_t rows, int64_t scols, uint8_t* out, cudaStream_t st);

void launch_dequant(bool mx, const uint8_t* codes, const uint8_t* scales, const float* d_S,
                    int64_t rows, int64_t cols, void* out, bool out_bf16, cudaStream_t s);

void launch_probe_copy(const void* src, void* dst, int64_t bytes, cudaStream_t s);
void launch_probe_wait(const unsigned* flag, unsigned target, unsigned limit, int32_t* d_status, cudaStream_t s);
void launch_probe_e2m1(const float* r, uint8_t* out, int64_t n, cudaStream_t s);
void launch_probe_e4m3(const float* v, uint8_t* out, int64_t n, cudaStream_t s);

}  // namespace fp4q
