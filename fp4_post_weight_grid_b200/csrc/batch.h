// batch.h -- parameters of the batch kernel (batch.cu), built on the host.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "fp4q.h"

namespace fp4q {

using BatchTensor = fp4q_batch_tensor;

constexpr int kMaxBatch = FP4Q_BATCH_MAX;   // weights per launch (longer lists: several launches)
constexpr int kWsHeader = 4;                // words before the per-weight counters
constexpr int kWsWords = kWsHeader + 2 * kMaxBatch;

// Passed by value as a kernel parameter (about 19 KB).
struct BatchParams {
    int32_t n;                              // weights in this launch
    int32_t seg_start[2 * kMaxBatch + 1];   // first queue item of each segment; [2n] = total
    int16_t seg_tensor[2 * kMaxBatch];      // weight of each segment
    uint8_t seg_nv[2 * kMaxBatch];          // 0: MXFP4 tiles, 1: NVFP4 tiles
    int32_t mx_tiles[kMaxBatch];            // MXFP4 tiles per weight
    BatchTensor t[kMaxBatch];
};

int64_t batch_mx_tiles(int64_t rows, int64_t cols);
int64_t batch_nv_tiles(int64_t rows, int64_t cols);
void launch_batch(const BatchParams& p, bool bf16, unsigned* ws, int32_t* d_status, cudaStream_t s);

// Device address and size of the library's own batch scratch (batch.cu); the
// first call on a device looks the address up.
cudaError_t batch_static_workspace(unsigned** ws, size_t* bytes);

}  // namespace fp4q
