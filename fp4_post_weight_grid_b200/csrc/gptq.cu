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
//   in-block GPTQ   4 threads per row, each holding two 16-column groups of
//                   the block in registers, U's diagonal block in shared
//                   memory: the sweep at every group start, the column
//                   quantization by the group's owner, the error broadcast by
//                   a warp shuffle, the in-block updates; the scaled errors go
//                   to a workspace E (two buffers, alternating per block);
//   trailing update the columns after a block, a 128 x 128 output tile per
//                   thread block (8 x 8 per thread), each output a chain of
//                   exact fused multiply-adds over the block's columns in
//                   ascending order.
// The in-block part has only the rows as parallelism (four threads per row
// along a sequential chain of columns), so on its own it leaves most of the
// GPU idle.  Block J's in-block part therefore runs in one launch with the
// bulk of block J-1's trailing update (the columns from block J+1 on), which
// fills the rest of the GPU; a small launch then applies block J's errors to
// block J+1's columns before block J+1's step.
// The trailing update is a dense contraction, but it runs on the CUDA cores:
// its definition is a chain of single-rounding fused multiply-adds in a fixed
// order, which a tensor-core accumulation (another precision and order) would
// not reproduce.
#include <type_traits>

#include "device.cuh"
#include "launch.h"
#include "nvfp4_block.cuh"

namespace fp4q {

namespace {

constexpr int kB = 128;           // columns per block
constexpr int kLanes = 4;         // threads per row in the in-block kernel: two 16-column groups each
constexpr int kThreadsA = 256;    // 64 rows per thread block
constexpr int kTB = 128;          // output tile of the update kernel (rows and columns)
constexpr int kBK = 32;           // block columns per shared-memory chunk of the update kernel
// U's diagonal block in shared memory: row j of 128 columns, with 4 floats of
// padding after every 32 columns, so that the four threads of a row (each
// reading its own 32 columns) hit different banks.
constexpr int kUs = kB + 16;
__device__ __forceinline__ int us_at(int j, int c) { return j * kUs + c + 4 * (c >> 5); }

// fma(-e, u, x) for the 16 values of one group, u from shared memory
__device__ __forceinline__ void gptq_update16(float (&x)[16], float e, const float* __restrict__ u)
{
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        const float4 t = *reinterpret_cast<const float4*>(u + 4 * v);
        x[4 * v + 0] = __fmaf_rn(-e, t.x, x[4 * v + 0]);
        x[4 * v + 1] = __fmaf_rn(-e, t.y, x[4 * v + 1]);
        x[4 * v + 2] = __fmaf_rn(-e, t.z, x[4 * v + 2]);
        x[4 * v + 3] = __fmaf_rn(-e, t.w, x[4 * v + 3]);
    }
}

// In-block GPTQ.  Thread `lane` of a row keeps the row's values of groups
// 2*lane and 2*lane+1 of the block in registers (x0, x1).  For every column j
// of group G, the owner (lane G/2) quantizes it (after the ScaleSweep of the
// group at its first column), computes e_j and broadcasts it to the row's
// other lanes with a warp shuffle; every lane then updates its own later
// columns with w_c = fma(-e_j, U[j][c], w_c), so each value sees the updates
// in ascending j.  Eight rows share a warp, so the owner's serial work runs
// on eight lanes at once.
__device__ __forceinline__ void gptq_block_body(int64_t cta, float* Us, NvTables& tb,
                                                const float* __restrict__ w, int64_t rows, int64_t cols,
                                                int64_t j0, int bw, const float* __restrict__ U,
                                                const float* __restrict__ d_amax, uint8_t* __restrict__ codes,
                                                uint8_t* __restrict__ scales, float* __restrict__ d_S,
                                                float* __restrict__ deq, float* __restrict__ Et, int64_t ldE,
                                                int32_t* __restrict__ d_status, float neg_zero)
{
    const float gmax = __ldg(d_amax);
    const int32_t flag = nvfp4_gmax_flag(gmax);
    if (flag) {
        if (cta == 0 && threadIdx.x == 0 && j0 == 0) atomicOr(d_status, flag);
        return;
    }
    const NvScale c = nvfp4_scale(gmax);
    if (cta == 0 && threadIdx.x == 0 && j0 == 0) *d_S = c.S;
    for (int i = threadIdx.x; i < bw * bw; i += kThreadsA)
        Us[us_at(i / bw, i % bw)] = __ldg(U + (j0 + i / bw) * cols + j0 + i % bw);
    nvfp4_tables(tb, c.S);                           // synchronises: U's block is in place too

    const int lane = threadIdx.x & (kLanes - 1);
    const int src0 = (threadIdx.x & 31) & ~(kLanes - 1);   // this row's first lane in the warp
    const int64_t row = cta * (kThreadsA / kLanes) + threadIdx.x / kLanes;
    const int ngroups = bw / 16;
    const bool active = row < rows;
    const bool has0 = 2 * lane < ngroups, has1 = 2 * lane + 1 < ngroups;
    float x0[16], x1[16];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        float (&xa)[16] = h == 0 ? x0 : x1;
        if (active && (h == 0 ? has0 : has1)) {
            const float4* p4 = reinterpret_cast<const float4*>(w + row * cols + j0 + 32 * lane + 16 * h);
#pragma unroll
            for (int v = 0; v < 4; ++v) {
                const float4 t = p4[v];
                xa[4 * v + 0] = t.x; xa[4 * v + 1] = t.y; xa[4 * v + 2] = t.z; xa[4 * v + 3] = t.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) xa[k] = 0.0f;
        }
    }
    const uint64_t z2 = pk(neg_zero, neg_zero);
    int p = 0;                                       // the owner lane of the group in flight
    auto run_group = [&](auto H) {
        constexpr int h = decltype(H)::value;
        const int G = 2 * p + h;
        if (G >= ngroups) return;                    // uniform across the warp
        float (&xa)[16] = h == 0 ? x0 : x1;
        float d = 1.0f, inv = 1.0f;
        if (lane == p) {                             // the ScaleSweep of the group's current values
            float wt[16];
            float amax = 0.0f;
#pragma unroll
            for (int k = 0; k < 16; ++k) amax = fmaxf(amax, fabsf(xa[k]));
            const float as = amax * c.invS;
            const float alpha2 = (16.0f * as * as) * (1.0f + 0x1p-16f);
            const int bp = nvfp4_select<-3, 11, false>(tb, c, xa, amax, wt, alpha2, c.tau0, true, z2, neg_zero);
            const float4 st = tb.step[bp];
            d = st.x;
            inv = st.y;
            if (active) scales[row * (cols / 16) + (j0 + 16 * G) / 16] = (uint8_t)bp;
        }
        uint64_t nib = 0;
        float y4[4];
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
            const int j = 16 * G + jj;
            float e = 0.0f;
            if (lane == p) {
                const float wj = xa[jj];
                const uint32_t code = e2m1x2(__fmul_rn(wj, inv), 0.0f) & 0xFu;
                float q, unused;
                f16x2_to_f32(e2m1x2_to_f16x2(code), q, unused);
                const float y = __fmul_rn(q, d);
                e = __fdiv_rn(__fsub_rn(wj, y), Us[us_at(j, j)]);
                nib |= (uint64_t)code << (4 * jj);
                y4[jj & 3] = y;
                if (active) {
                    Et[j * ldE + row] = e;
                    if (deq && (jj & 3) == 3)
                        *reinterpret_cast<float4*>(deq + row * cols + j0 + j - 3) = make_float4(y4[0], y4[1], y4[2], y4[3]);
                }
            }
            e = __shfl_sync(0xFFFFFFFFu, e, src0 + p);
            const float* uj = Us + us_at(j, 32 * lane);
            if (lane > p) {
                if (has0) gptq_update16(x0, e, uj);
                if (has1) gptq_update16(x1, e, uj + 16);
            } else if (lane == p) {
#pragma unroll
                for (int k = jj + 1; k < 16; ++k) xa[k] = __fmaf_rn(-e, uj[16 * h + k], xa[k]);
                if (h == 0 && has1) gptq_update16(x1, e, uj + 16);
            }
        }
        if (lane == p && active)
            *reinterpret_cast<uint64_t*>(codes + (row * cols + j0 + 16 * G) / 2) = nib;
    };
#pragma unroll 1
    for (p = 0; 2 * p < ngroups; ++p) {
        run_group(std::integral_constant<int, 0>{});
        run_group(std::integral_constant<int, 1>{});
    }
}

// Trailing update w[r][c] for the columns after the block: a 128 x 128 output
// tile per thread block, 8 x 8 outputs per thread (rows tr..tr+3, tr+64..tr+67
// and columns tc..tc+3, tc+64..tc+67).  The block's columns are taken in
// chunks of 32, in ascending order, through two shared-memory buffers filled
// by asynchronous copies (the next chunk loads while this one is used); each
// output is a chain of fused multiply-adds in ascending k.  Padding (rows or
// columns past the end, k past the block) is zero-filled, and fma(-0, 0, a)
// returns a unchanged.
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, bool valid)
{
    const unsigned dst = (unsigned)__cvta_generic_to_shared(smem);
    const int n = valid ? 16 : 0;                   // 0: no bytes read, 16 zero bytes written
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" :: "r"(dst), "l"(gmem), "r"(n) : "memory");
}

__device__ __forceinline__ void gptq_load_chunk(float* Es, float* Ut, const float* __restrict__ Et, int64_t ldE,
                                                const float* __restrict__ U, int64_t rows, int64_t cols, int64_t cend,
                                                int64_t j0, int bw, int kc, int64_t r0, int64_t c0)
{
    // 32 x 128 floats each, 16 bytes per copy: 4 copies of each per thread
#pragma unroll
    for (int s = 0; s < kBK * kTB / 4 / 256; ++s) {
        const int i = threadIdx.x + 256 * s;
        const int k = i / (kTB / 4), t = (i % (kTB / 4)) * 4;
        const bool kin = kc + k < bw;
        const bool ein = kin && r0 + t < rows;       // ldE is a multiple of 4: a 4-row group is all in or all out
        const bool uin = kin && c0 + t < cend;       // cend is a multiple of 16
        cp_async16(Es + k * kTB + t, ein ? Et + (int64_t)(kc + k) * ldE + r0 + t : Et, ein);
        cp_async16(Ut + k * kTB + t, uin ? U + (j0 + kc + k) * cols + c0 + t : U, uin);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void gptq_update_body(int64_t tile, int64_t row_tiles, float* sm, float* __restrict__ w,
                                                 int64_t rows, int64_t cols, int64_t j0, int bw,
                                                 int64_t cfrom, int64_t cto, const float* __restrict__ U,
                                                 const float* __restrict__ Et, int64_t ldE)
{
    // sm: 2 x {E chunk [k][row], U chunk [k][column]}
    const int64_t r0 = (tile % row_tiles) * kTB;
    const int64_t c0 = cfrom + (tile / row_tiles) * kTB;   // the tile's columns stop at cto (a multiple of 16)
    const int tr = (threadIdx.x >> 4) * 4, tc = (threadIdx.x & 15) * 4;
    const int nchunks = (bw + kBK - 1) / kBK;
    gptq_load_chunk(sm, sm + kBK * kTB, Et, ldE, U, rows, cols, cto, j0, bw, 0, r0, c0);
    // the tile's current values, four columns per 16-byte load (cols is a
    // multiple of 16, so a group of four is all in or all out)
    float acc[8][8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t r = r0 + tr + (i & 3) + (i >> 2) * 64;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t cc = c0 + tc + 64 * h;
            float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            if (r < rows && cc < cto) v = *reinterpret_cast<const float4*>(w + r * cols + cc);
            acc[i][4 * h + 0] = v.x; acc[i][4 * h + 1] = v.y; acc[i][4 * h + 2] = v.z; acc[i][4 * h + 3] = v.w;
        }
    }
    for (int ch = 0; ch < nchunks; ++ch) {
        float* Es = sm + (ch & 1) * 2 * kBK * kTB;
        float* Ut = Es + kBK * kTB;
        if (ch + 1 < nchunks) {
            float* En = sm + ((ch + 1) & 1) * 2 * kBK * kTB;
            gptq_load_chunk(En, En + kBK * kTB, Et, ldE, U, rows, cols, cto, j0, bw, (ch + 1) * kBK, r0, c0);
            asm volatile("cp.async.wait_group 1;" ::: "memory");
        } else {
            asm volatile("cp.async.wait_group 0;" ::: "memory");
        }
        __syncthreads();                             // chunk ch is in shared memory for every thread
#pragma unroll 2
        for (int k = 0; k < kBK; ++k) {
            const float4 a0 = *reinterpret_cast<const float4*>(Es + k * kTB + tr);
            const float4 a1 = *reinterpret_cast<const float4*>(Es + k * kTB + tr + 64);
            const float4 b0 = *reinterpret_cast<const float4*>(Ut + k * kTB + tc);
            const float4 b1 = *reinterpret_cast<const float4*>(Ut + k * kTB + tc + 64);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) acc[i][jj] = __fmaf_rn(-av[i], bv[jj], acc[i][jj]);
        }
        __syncthreads();                             // every thread is done with buffer ch & 1
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t r = r0 + tr + (i & 3) + (i >> 2) * 64;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t cc = c0 + tc + 64 * h;
            if (r < rows && cc < cto)
                *reinterpret_cast<float4*>(w + r * cols + cc) =
                    make_float4(acc[i][4 * h + 0], acc[i][4 * h + 1], acc[i][4 * h + 2], acc[i][4 * h + 3]);
        }
    }
}

// The trailing update of one block's errors on columns [cfrom, cto).
__global__ void __launch_bounds__(256, 2)
gptq_update_kernel(float* __restrict__ w, int64_t rows, int64_t cols, int64_t j0, int bw, int64_t cfrom,
                   int64_t cto, const float* __restrict__ U, const float* __restrict__ Et, int64_t ldE)
{
    extern __shared__ __align__(16) float sm[];
    const int64_t row_tiles = (rows + kTB - 1) / kTB;
    gptq_update_body(blockIdx.x, row_tiles, sm, w, rows, cols, j0, bw, cfrom, cto, U, Et, ldE);
}

// One step of the pipeline: thread blocks [0, nA) run the in-block GPTQ of the
// block at j0 (errors to Et); the others apply the previous block's errors
// (Ep, block jp of width bwp) to the columns from j0 + bw on.  The two halves
// touch disjoint columns of w: the in-block half only the block at j0 (whose
// update by the previous block the preceding launch already applied), the
// update half only the columns after it.  The in-block thread blocks come
// first so that they start first; the update tiles fill the rest of the GPU
// around them.
__global__ void __launch_bounds__(256, 2)
gptq_step_kernel(float* __restrict__ w, int64_t rows, int64_t cols, int64_t j0, int bw, int64_t nA,
                 const float* __restrict__ U, const float* __restrict__ d_amax, uint8_t* __restrict__ codes,
                 uint8_t* __restrict__ scales, float* __restrict__ d_S, float* __restrict__ deq,
                 float* __restrict__ Et, const float* __restrict__ Ep, int64_t jp, int bwp, int64_t ldE,
                 int32_t* __restrict__ d_status, float neg_zero)
{
    extern __shared__ __align__(16) float smem[];
    __shared__ NvTables tb;
    if ((int64_t)blockIdx.x < nA) {
        gptq_block_body(blockIdx.x, smem, tb, w, rows, cols, j0, bw, U, d_amax, codes, scales, d_S, deq, Et, ldE,
                        d_status, neg_zero);
    } else {
        const int64_t row_tiles = (rows + kTB - 1) / kTB;
        gptq_update_body((int64_t)blockIdx.x - nA, row_tiles, smem, w, rows, cols, jp, bwp, j0 + bw, cols, U, Ep,
                         ldE);
    }
}

}  // namespace

// Workspace: the scaled errors of two consecutive blocks, each transposed
// ([128][ldE] with ldE the row count rounded up to a multiple of 4, so every
// 16-byte copy is aligned): the in-block step of block J writes one buffer
// while the trailing update of block J-1 still reads the other.
static int64_t gptq_ld(int64_t rows) { return (rows + 3) / 4 * 4; }

size_t gptq_workspace_bytes(int64_t rows) { return (size_t)2 * gptq_ld(rows) * kB * sizeof(float); }

// Blocks J = 0, 1, ... of 128 columns.  Step J is one launch: the in-block
// GPTQ of block J beside the update of block J-1's errors on the columns
// from block J+1 on; then a small launch applies block J's errors to block
// J+1's columns, which step J+1 needs.  Every element receives the errors of
// the blocks before it in ascending order (the update of J-1 on block J+1's
// columns runs in step J, before the launch that applies J's), so the bytes
// are those of the column-by-column definition.
cudaError_t launch_nvfp4_gptq(float* w, int64_t rows, int64_t cols, const float* U, const float* d_amax,
                              uint8_t* codes, uint8_t* scales, float* d_S, float* deq, float* E, int32_t* d_status,
                              cudaStream_t s)
{
    // the two halves of the step kernel share one dynamic allocation
    const size_t smem = (size_t)(kB * kUs > 4 * kBK * kTB ? kB * kUs : 4 * kBK * kTB) * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(reinterpret_cast<const void*>(gptq_step_kernel),
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(reinterpret_cast<const void*>(gptq_update_kernel),
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int64_t ldE = gptq_ld(rows);
    float* Ebuf[2] = {E, E + kB * ldE};
    const int64_t nA = (rows + (kThreadsA / kLanes) - 1) / (kThreadsA / kLanes);
    const int64_t row_tiles = (rows + kTB - 1) / kTB;
    int bwp = 0;
    int parity = 0;
    for (int64_t j0 = 0; j0 < cols; j0 += kB, parity ^= 1) {
        const int bw = (int)(cols - j0 < kB ? cols - j0 : kB);
        // step: in-block j0, and block j0 - 128's errors on the columns from j0 + bw on
        const int64_t rem = j0 > 0 ? cols - j0 - bw : 0;
        const int64_t nB = rem > 0 ? row_tiles * ((rem + kTB - 1) / kTB) : 0;
        gptq_step_kernel<<<(unsigned)(nA + nB), kThreadsA, smem, s>>>(
            w, rows, cols, j0, bw, nA, U, d_amax, codes, scales, d_S, deq, Ebuf[parity], Ebuf[parity ^ 1],
            j0 - kB, bwp, ldE, d_status, -0.0f);
        // this block's errors on the next block's columns
        const int64_t c1 = j0 + bw, c2 = c1 + kB < cols ? c1 + kB : cols;
        if (c2 > c1)
            gptq_update_kernel<<<(unsigned)(row_tiles * ((c2 - c1 + kTB - 1) / kTB)), 256, smem, s>>>(
                w, rows, cols, j0, bw, c1, c2, U, Ebuf[parity], ldE);
        bwp = bw;
    }
    return cudaGetLastError();
}

}  // namespace fp4q
