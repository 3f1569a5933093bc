// gptq.cu -- ScaleSweep inside GPTQ.
//
// ScaleSweep summary, "Contribuicoes" 2: the sweep selects the block scales
// of GPTQ pipelines as well as of round-to-nearest ones.  GPTQ in its
// Cholesky form: U is the upper Cholesky factor of the inverse of the layer's
// dampened input Gram matrix (U^T U = H^-1, supplied by the caller).  Rows are
// independent; along a row, at the first column of every 16-column group the
// ScaleSweep (MSE window -3..+7) picks the group's pattern from the row's
// current, error-compensated values, and every column j is quantized with its
// group's step and spreads its scaled error over the later columns:
//   y_j = RN(E2M1(RN(w_j * inv)) * d);   e_j = RN((w_j - y_j) / U[j][j])
//   w_c = fma(-e_j, U[j][c], w_c)        for every c > j.
//
// Every element w_c receives the updates of the columns j < c one at a time,
// in ascending j, whether they are applied column by column or block by
// block; so the blocked algorithm below writes exactly the bytes of the plain
// sequential one.  Per block of 128 columns:
//   gptq_block_kernel   one thread per row (64 rows per thread block): the
//                       block's slice of each row and U's diagonal block in
//                       shared memory; the sweep at every group start, the
//                       column quantization, the error and the in-block
//                       updates; the scaled errors go to a workspace E;
//   gptq_update_kernel  the trailing update w[:, c] for the columns after the
//                       block, a 64 x 64 output tile per thread block, each
//                       output a chain of exact fused multiply-adds over the
//                       block's 128 columns in ascending order.
// The trailing update is a dense contraction, but it runs on the CUDA cores:
// its definition is a chain of single-rounding fused multiply-adds in a fixed
// order, which a tensor-core accumulation (another precision and order) would
// not reproduce.
#include "device.cuh"
#include "launch.h"
#include "nvfp4_block.cuh"

namespace fp4q {

namespace {

constexpr int kB = 128;           // columns per block
constexpr int kRowsA = 64;        // rows (threads) per thread block of the inner kernel
constexpr int kTile = 64;         // output tile of the update kernel (rows and columns)

__global__ void __launch_bounds__(kRowsA)
gptq_block_kernel(const float* __restrict__ w, int64_t rows, int64_t cols, int64_t j0, int bw,
                  const float* __restrict__ U, const float* __restrict__ d_amax, uint8_t* __restrict__ codes,
                  uint8_t* __restrict__ scales, float* __restrict__ d_S, float* __restrict__ deq,
                  float* __restrict__ E, int32_t* __restrict__ d_status, float neg_zero)
{
    extern __shared__ float sm[];
    __shared__ NvTables tb;
    const int ld = bw + 1;                           // padded row stride: no bank conflicts
    float* Ws = sm;                                  // [kRowsA][ld]
    float* Us = sm + kRowsA * ld;                    // [bw][bw]
    const float gmax = __ldg(d_amax);
    const int32_t flag = nvfp4_gmax_flag(gmax);
    if (flag) {
        if (blockIdx.x == 0 && threadIdx.x == 0 && j0 == 0) atomicOr(d_status, flag);
        return;
    }
    const NvScale c = nvfp4_scale(gmax);
    if (blockIdx.x == 0 && threadIdx.x == 0 && j0 == 0) *d_S = c.S;
    const int64_t r0 = (int64_t)blockIdx.x * kRowsA;
    for (int i = threadIdx.x; i < bw * bw; i += kRowsA)
        Us[i] = __ldg(U + (j0 + i / bw) * cols + j0 + i % bw);
    for (int i = threadIdx.x; i < kRowsA * bw; i += kRowsA) {
        const int rr = i / bw, k = i % bw;
        Ws[rr * ld + k] = r0 + rr < rows ? w[(r0 + rr) * cols + j0 + k] : 0.0f;
    }
    nvfp4_tables(tb, c.S);                           // synchronises: the slices are in place too

    const int64_t row = r0 + threadIdx.x;
    const bool active = row < rows;
    float* wr = Ws + threadIdx.x * ld;
    const uint64_t z2 = pk(neg_zero, neg_zero);
    float d = 1.0f, inv = 1.0f;
    uint64_t nib = 0;
#pragma unroll 1
    for (int j = 0; j < bw; ++j) {
        if ((j & 15) == 0) {                         // the ScaleSweep of the group's current values
            float x[16], wt[16];
            float amax = 0.0f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                x[i] = wr[j + i];
                amax = fmaxf(amax, fabsf(x[i]));
            }
            const float as = amax * c.invS;
            const float alpha2 = (16.0f * as * as) * (1.0f + 0x1p-16f);
            const int bp = nvfp4_select<-3, 11, false>(tb, c, x, amax, wt, alpha2, c.tau0, true, z2, neg_zero);
            const float4 st = tb.step[bp];
            d = st.x;
            inv = st.y;
            if (active) scales[row * (cols / 16) + (j0 + j) / 16] = (uint8_t)bp;
            nib = 0;
        }
        const float wj = wr[j];
        const uint32_t code = e2m1x2(__fmul_rn(wj, inv), 0.0f) & 0xFu;
        float q, unused;
        f16x2_to_f32(e2m1x2_to_f16x2(code), q, unused);
        const float y = __fmul_rn(q, d);
        const float e = __fdiv_rn(__fsub_rn(wj, y), Us[j * bw + j]);
        nib |= (uint64_t)code << (4 * (j & 15));
        if (active) {
            E[row * kB + j] = e;
            if (deq) deq[row * cols + j0 + j] = y;
            if ((j & 15) == 15) *reinterpret_cast<uint64_t*>(codes + (row * cols + j0 + j - 15) / 2) = nib;
        }
        const float* uj = Us + j * bw;
#pragma unroll 4
        for (int k = j + 1; k < bw; ++k) wr[k] = __fmaf_rn(-e, uj[k], wr[k]);
    }
}

__global__ void __launch_bounds__(256)
gptq_update_kernel(float* __restrict__ w, int64_t rows, int64_t cols, int64_t j0, int bw,
                   const float* __restrict__ U, const float* __restrict__ E)
{
    extern __shared__ float sm[];
    float* Es = sm;                                  // [bw][kTile]: E transposed, this tile's rows
    float* Ut = sm + bw * kTile;                     // [bw][kTile]: U rows of the block, this tile's columns
    const int64_t c_begin = j0 + bw;
    const int64_t r0 = (int64_t)blockIdx.x * kTile;
    const int64_t c0 = c_begin + (int64_t)blockIdx.y * kTile;
    for (int i = threadIdx.x; i < bw * kTile; i += 256) {
        const int k = i / kTile, t = i % kTile;      // coalesced along t for U, strided for E
        Ut[i] = c0 + t < cols ? __ldg(U + (j0 + k) * cols + c0 + t) : 0.0f;
    }
    for (int i = threadIdx.x; i < bw * kTile; i += 256) {
        const int t = i / bw, k = i % bw;            // coalesced along k for E
        Es[k * kTile + t] = r0 + t < rows ? __ldg(E + (r0 + t) * kB + k) : 0.0f;
    }
    __syncthreads();
    const int tr = (threadIdx.x >> 4) * 4, tc = (threadIdx.x & 15) * 4;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int64_t r = r0 + tr + i, cc = c0 + tc + jj;
            acc[i][jj] = (r < rows && cc < cols) ? w[r * cols + cc] : 0.0f;
        }
#pragma unroll 4
    for (int k = 0; k < bw; ++k) {
        const float4 a = *reinterpret_cast<const float4*>(Es + k * kTile + tr);
        const float4 b = *reinterpret_cast<const float4*>(Ut + k * kTile + tc);
        const float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) acc[i][jj] = __fmaf_rn(-av[i], bv[jj], acc[i][jj]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const int64_t r = r0 + tr + i, cc = c0 + tc + jj;
            if (r < rows && cc < cols) w[r * cols + cc] = acc[i][jj];
        }
}

}  // namespace

size_t gptq_workspace_bytes(int64_t rows) { return (size_t)rows * kB * sizeof(float); }

cudaError_t launch_nvfp4_gptq(float* w, int64_t rows, int64_t cols, const float* U, const float* d_amax,
                              uint8_t* codes, uint8_t* scales, float* d_S, float* deq, float* E, int32_t* d_status,
                              cudaStream_t s)
{
    const size_t smem_a_max = (size_t)(kRowsA * (kB + 1) + kB * kB) * sizeof(float);
    const size_t smem_b_max = (size_t)(2 * kB * kTile) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(gptq_block_kernel),
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a_max);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(reinterpret_cast<const void*>(gptq_update_kernel),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_b_max);
    if (e != cudaSuccess) return e;
    const unsigned grid_a = (unsigned)((rows + kRowsA - 1) / kRowsA);
    for (int64_t j0 = 0; j0 < cols; j0 += kB) {
        const int bw = (int)(cols - j0 < kB ? cols - j0 : kB);
        const size_t smem_a = (size_t)(kRowsA * (bw + 1) + bw * bw) * sizeof(float);
        gptq_block_kernel<<<grid_a, kRowsA, smem_a, s>>>(w, rows, cols, j0, bw, U, d_amax, codes, scales, d_S, deq, E,
                                                         d_status, -0.0f);
        const int64_t rem = cols - j0 - bw;
        if (rem > 0) {
            const dim3 grid_b((unsigned)((rows + kTile - 1) / kTile), (unsigned)((rem + kTile - 1) / kTile));
            const size_t smem_b = (size_t)(2 * bw * kTile) * sizeof(float);
            gptq_update_kernel<<<grid_b, 256, smem_b, s>>>(w, rows, cols, j0, bw, U, E);
        }
    }
    return cudaGetLastError();
}

}  // namespace fp4q
