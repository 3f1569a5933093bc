// layout.cu -- block scales in the tiled layout that Blackwell block-scaled
// FP4 GEMMs read.
//
// The MR-GPTQ summary ("Bridging the Gap Between Promise and Performance for
// Microscaling FP4 Quantization", technical summary sec. 3) runs the
// quantized weights through block-scaled FP4 GEMM kernels on Blackwell.  Those
// read an operand's block scales in tiles of 128 rows x 4 scale columns
// (zero-padded at the edges, the column tiles of one row tile stored
// together); a 512-byte tile is 32 lines of 16 bytes, line j holding the 4
// scale bytes of rows j, j+32, j+64 and j+96 of the tile.
#include "device.cuh"
#include "launch.h"

namespace fp4q {

namespace {

constexpr int kThreads = 256;
constexpr int kTileCols = 32;          // scale columns per thread block: 8 tiles of 4

// One thread block per 128 rows x 32 scale columns: the rows are read into
// shared memory with 16-byte loads (two threads per row), then every thread
// writes one 16-byte line of the 8 output tiles, so both the reads and the
// writes are contiguous.  Edges (rows past the end, columns past the end, a
// row length that is not a multiple of 16 bytes or a source that is not
// 16-byte aligned) take byte loads and are zero-filled.
__global__ void __launch_bounds__(kThreads)
mma_scale_layout_kernel(const uint8_t* __restrict__ s, int64_t rows, int64_t scols, int64_t col_tiles,
                        int64_t col_groups, uint8_t* __restrict__ out)
{
    __shared__ __align__(16) uint8_t t[128][kTileCols];
    const int64_t rt = blockIdx.x / col_groups;
    const int64_t cg = blockIdx.x % col_groups;
    const int64_t r0 = rt * 128, c0 = cg * kTileCols;
    {
        const int rr = threadIdx.x >> 1, half = threadIdx.x & 1;
        const int64_t r = r0 + rr, c = c0 + 16 * half;
        const uint8_t* p = s + r * scols + c;
        uint8_t* d = &t[rr][16 * half];
        if (r < rows && c + 16 <= scols && (reinterpret_cast<uintptr_t>(p) & 15) == 0) {
            *reinterpret_cast<uint4*>(d) = __ldg(reinterpret_cast<const uint4*>(p));
        } else {
            for (int k = 0; k < 16; ++k) d[k] = (r < rows && c + k < scols) ? __ldg(p + k) : (uint8_t)0;
        }
    }
    __syncthreads();
    const int ct = threadIdx.x >> 5, j = threadIdx.x & 31;      // output tile, line
    const int64_t tile_col = cg * (kTileCols / 4) + ct;
    if (tile_col < col_tiles) {
        uint4 v;
        v.x = *reinterpret_cast<const uint32_t*>(&t[j][4 * ct]);
        v.y = *reinterpret_cast<const uint32_t*>(&t[j + 32][4 * ct]);
        v.z = *reinterpret_cast<const uint32_t*>(&t[j + 64][4 * ct]);
        v.w = *reinterpret_cast<const uint32_t*>(&t[j + 96][4 * ct]);
        st_stream(out + ((rt * col_tiles + tile_col) * 32 + j) * 16, v);
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
    const int64_t col_groups = (scols + kTileCols - 1) / kTileCols;
    const int64_t grid = ((rows + 127) / 128) * col_groups;
    mma_scale_layout_kernel<<<(unsigned)grid, kThreads, 0, st>>>(s, rows, scols, col_tiles, col_groups, out);
}

}  // namespace fp4q
