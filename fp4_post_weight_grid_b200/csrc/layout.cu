// layout.cu -- block scales in the tiled layout that Blackwell block-scaled
// FP4 GEMMs read.
//
// The MR-GPTQ summary ("Bridging the Gap Between Promise and Performance for
// Microscaling FP4 Quantization", technical summary sec. 3) runs the
// quantized weights through block-scaled FP4 GEMM kernels on Blackwell.  Those
// read an operand's block scales in tiles of 128 rows x 4 scale columns
// (zero-padded at the edges, the column tiles of one row tile stored
// together); a 512-byte tile is 32 lines of 16 bytes, line j holding the 4
// scale bytes of rows j, j+32, j+64 and j+96 of the tile.  One thread writes
// one line with a single 16-byte store.
#include "device.cuh"
#include "launch.h"

namespace fp4q {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
mma_scale_layout_kernel(const uint8_t* __restrict__ s, int64_t rows, int64_t scols, int64_t col_tiles,
                        int64_t lines, uint8_t* __restrict__ out)
{
    const bool words = (scols & 3) == 0 && (reinterpret_cast<uintptr_t>(s) & 3) == 0;
    for (int64_t L = (int64_t)blockIdx.x * kThreads + threadIdx.x; L < lines; L += (int64_t)gridDim.x * kThreads) {
        const int64_t tile = L >> 5;
        const int64_t j = L & 31;
        const int64_t r0 = (tile / col_tiles) * 128 + j;
        const int64_t c0 = (tile % col_tiles) * 4;
        uint32_t v[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int64_t r = r0 + 32 * i;
            uint32_t w = 0;
            if (r < rows) {
                const uint8_t* p = s + r * scols + c0;
                if (words) {
                    w = __ldg(reinterpret_cast<const uint32_t*>(p));        // c0 + 3 < scols
                } else {
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        if (c0 + k < scols) w |= (uint32_t)__ldg(p + k) << (8 * k);
                }
            }
            v[i] = w;
        }
        st_stream(out + L * 16, make_uint4(v[0], v[1], v[2], v[3]));
    }
}

}  // namespace

int64_t mma_scale_bytes(int64_t rows, int64_t scols)
{
    return ((rows + 127) / 128) * ((scols + 3) / 4) * 512;
}

void launch_mma_scale_layout(const uint8_t* s, int64_t rows, int64_t scols, uint8_t* out, cudaStream_t st)
{
    const int64_t col_tiles = (scols + 3) / 4;
    const int64_t lines = mma_scale_bytes(rows, scols) / 16;
    int64_t grid = (lines + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)sm_count() * 8;
    if (grid > cap) grid = cap;
    if (grid < 1) grid = 1;
    mma_scale_layout_kernel<<<(unsigned)grid, kThreads, 0, st>>>(s, rows, scols, col_tiles, lines, out);
}

}  // namespace fp4q
