// device.cuh -- sm_100a device primitives shared by the quantizer kernels.
//
// Number formats (ScaleSweep summary, "Declaracao do Problema"; MR-GPTQ
// summary, technical sec. 1): E2M1 elements, E4M3 block scales (NVFP4),
// E8M0 block scales (MXFP4).  The element rounding uses the hardware
// conversions of sm_100a (cvt.rn.satfinite.e2m1x2.f32: round to nearest,
// ties to even, saturating; the sign is kept), the pairs of binary32 use the
// packed f32x2 arithmetic of sm_100a (each lane an IEEE RN operation).
// Nothing here is fused into an FMA: the library is built with --fmad=false
// and every multiply/add below is an explicit RN operation.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace fp4q {

// ---------------------------------------------------------------- f32x2 pairs
// A pair of binary32 values in one 64-bit register: .x in the low half.
__device__ __forceinline__ uint64_t pk(float lo, float hi)
{
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void upk(uint64_t v, float& lo, float& hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b)
{
    uint64_t r;
    asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// Product a*b of a pair, for a product that feeds an add or a subtract.
// ptxas fuses a packed mul.rn.f32x2 followed by add/sub.rn.f32x2 into one
// fused multiply-add even when contraction is disabled, which changes the
// rounding.  Computing the product as fma(a, b, z) with z = (-0, -0) held in a
// register gives exactly RN(a*b) (adding -0 changes no value, zero signs
// included) and an fma result cannot be fused again.  `z` must come from a
// runtime value (a kernel argument) so that it is not folded back into a mul.
__device__ __forceinline__ uint64_t mul2_nofuse(uint64_t a, uint64_t b, uint64_t z)
{
    uint64_t r;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(z));
    return r;
}

// ---------------------------------------------------------------- E2M1
// Two binary32 values -> one byte holding two E2M1 nibbles, `lo` in bits 0..3
// and `hi` in bits 4..7 (the instruction stores its first source in the upper
// nibble).  Nibble = sign<<3 | magnitude code.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi)
{
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.u32.u8 %0, t;\n\t}"
        : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// One byte of two E2M1 nibbles -> f16x2 (low nibble -> low half).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte)
{
    uint32_t r;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.u8.u32 t, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(r) : "r"(byte));
    return r;
}

// Four pairs r[2j], r[2j+1] (j = 0..3) -> one word of four code bytes (pair j
// in byte j, r[2j] in its low nibble), and the four decoded pairs as f16x2.
// The code bytes stay in 8-bit PTX registers between the conversions.
__device__ __forceinline__ uint32_t e2m1x8_encode(const float (&r)[8], uint32_t (&h2)[4])
{
    uint32_t w;
    asm("{\n\t.reg .b8 t0, t1, t2, t3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t0, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t1, %8, %7;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t2, %10, %9;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t3, %12, %11;\n\t"
        "cvt.rn.f16x2.e2m1x2 %1, t0;\n\t"
        "cvt.rn.f16x2.e2m1x2 %2, t1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %3, t2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %4, t3;\n\t"
        "mov.b32 %0, {t0, t1, t2, t3};\n\t}"
        : "=r"(w), "=r"(h2[0]), "=r"(h2[1]), "=r"(h2[2]), "=r"(h2[3])
        : "f"(r[0]), "f"(r[1]), "f"(r[2]), "f"(r[3]), "f"(r[4]), "f"(r[5]), "f"(r[6]), "f"(r[7]));
    return w;
}

// f16x2 -> two binary32 (exact).
__device__ __forceinline__ void f16x2_to_f32(uint32_t h2, float& lo, float& hi)
{
    asm("{\n\t.reg .f16 a, b;\n\t"
        "mov.b32 {a, b}, %2;\n\t"
        "cvt.f32.f16 %0, a;\n\t"
        "cvt.f32.f16 %1, b;\n\t}"
        : "=f"(lo), "=f"(hi) : "r"(h2));
}

// f16x2 -> binary32 pair (exact).
__device__ __forceinline__ uint64_t f16x2_to_f2(uint32_t h2)
{
    float lo, hi;
    f16x2_to_f32(h2, lo, hi);
    return pk(lo, hi);
}

// Decoded E2M1 value pair of one code byte, as binary32.
__device__ __forceinline__ uint64_t e2m1x2_decode(uint32_t byte)
{
    float lo, hi;
    f16x2_to_f32(e2m1x2_to_f16x2(byte), lo, hi);
    return pk(lo, hi);
}

// Round a pair to E2M1 and return the rounded values as binary32, without
// materialising the code byte (the byte stays in an 8-bit PTX register between
// the two conversions).
__device__ __forceinline__ uint64_t e2m1x2_round(float lo, float hi)
{
    uint32_t h2;
    asm("{\n\t.reg .b8 t;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, t;\n\t}"
        : "=r"(h2) : "f"(hi), "f"(lo));
    float a, b;
    f16x2_to_f32(h2, a, b);
    return pk(a, b);
}

// ---------------------------------------------------------------- E4M3
// Pattern of v >= 0: round to nearest even, saturate at 448 (0x7E).
__device__ __forceinline__ uint32_t e4m3_rn_sat(float v)
{
    uint16_t r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(v));
    return r & 0xFFu;
}

// Value of a non-negative E4M3 pattern p in 0..126: subnormals p * 2^-9; normal
// patterns have exponent field p>>3 (bias 7) and mantissa p&7, i.e. binary32
// bits (p << 20) + ((127 - 7) << 23).
__device__ __forceinline__ float e4m3_value(uint32_t p)
{
    return p >= 8u ? __uint_as_float((p << 20) + (120u << 23)) : __fmul_rn((float)p, 0x1p-9f);
}

// ---------------------------------------------------------------- powers of two
// 2^e for e in [-127, 127], exact (2^-127 is the binary32 subnormal 0x00400000).
__device__ __forceinline__ float exp2i(int e)
{
    return e >= -126 ? __uint_as_float((uint32_t)(e + 127) << 23) : __uint_as_float(0x00400000u);
}

// ---------------------------------------------------------------- loads / stores
__device__ __forceinline__ uint4 ld_stream(const void* p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
    return r;
}

__device__ __forceinline__ void st_stream(void* p, uint4 v)
{
    asm volatile("st.global.cs.v4.u32 [%0], {%1, %2, %3, %4};"
                 :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

__device__ __forceinline__ void st_stream64(void* p, uint2 v)
{
    asm volatile("st.global.cs.v2.u32 [%0], {%1, %2};" :: "l"(p), "r"(v.x), "r"(v.y) : "memory");
}

// bf16 pair packed in a 32-bit word -> two binary32 (exact).
__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi)
{
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
}

// Two binary32 -> bf16 pair (round to nearest even), lo in the low half.
__device__ __forceinline__ uint32_t f32_to_bf16x2(float lo, float hi)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Load N consecutive elements (N multiple of 8 for bf16, of 4 for fp32) as binary32.
template <int N>
__device__ __forceinline__ void load_block(const __nv_bfloat16* p, float (&x)[N])
{
#pragma unroll
    for (int v = 0; v < N / 8; ++v) {
        uint4 u = ld_stream(p + 8 * v);
        bf16x2_to_f32(u.x, x[8 * v + 0], x[8 * v + 1]);
        bf16x2_to_f32(u.y, x[8 * v + 2], x[8 * v + 3]);
        bf16x2_to_f32(u.z, x[8 * v + 4], x[8 * v + 5]);
        bf16x2_to_f32(u.w, x[8 * v + 6], x[8 * v + 7]);
    }
}
template <int N>
__device__ __forceinline__ void load_block(const float* p, float (&x)[N])
{
#pragma unroll
    for (int v = 0; v < N / 4; ++v) {
        uint4 u = ld_stream(p + 4 * v);
        x[4 * v + 0] = __uint_as_float(u.x);
        x[4 * v + 1] = __uint_as_float(u.y);
        x[4 * v + 2] = __uint_as_float(u.z);
        x[4 * v + 3] = __uint_as_float(u.w);
    }
}

// load_block that also returns max |x| as binary32 bits (NaN above Inf above
// every finite value).  bf16: the maximum is taken on the raw 16-bit halves.
template <int N>
__device__ __forceinline__ void load_block_amax(const __nv_bfloat16* p, float (&x)[N], uint32_t& amax_bits)
{
    uint32_t m2 = 0;
#pragma unroll
    for (int v = 0; v < N / 8; ++v) {
        uint4 u = ld_stream(p + 8 * v);
        bf16x2_to_f32(u.x, x[8 * v + 0], x[8 * v + 1]);
        bf16x2_to_f32(u.y, x[8 * v + 2], x[8 * v + 3]);
        bf16x2_to_f32(u.z, x[8 * v + 4], x[8 * v + 5]);
        bf16x2_to_f32(u.w, x[8 * v + 6], x[8 * v + 7]);
        m2 = __vmaxu2(m2, __vmaxu2(u.x & 0x7FFF7FFFu, u.y & 0x7FFF7FFFu));
        m2 = __vmaxu2(m2, __vmaxu2(u.z & 0x7FFF7FFFu, u.w & 0x7FFF7FFFu));
    }
    amax_bits = max(m2 & 0xFFFFu, m2 >> 16) << 16;
}
template <int N>
__device__ __forceinline__ void load_block_amax(const float* p, float (&x)[N], uint32_t& amax_bits)
{
    uint32_t m = 0;
#pragma unroll
    for (int v = 0; v < N / 4; ++v) {
        uint4 u = ld_stream(p + 4 * v);
        x[4 * v + 0] = __uint_as_float(u.x);
        x[4 * v + 1] = __uint_as_float(u.y);
        x[4 * v + 2] = __uint_as_float(u.z);
        x[4 * v + 3] = __uint_as_float(u.w);
        m = max(m, max(max(u.x & 0x7FFFFFFFu, u.y & 0x7FFFFFFFu), max(u.z & 0x7FFFFFFFu, u.w & 0x7FFFFFFFu)));
    }
    amax_bits = m;
}

// Store N binary32 values rounded to the element type.
template <int N>
__device__ __forceinline__ void store_block(__nv_bfloat16* p, const float (&y)[N])
{
#pragma unroll
    for (int v = 0; v < N / 8; ++v) {
        uint4 u;
        u.x = f32_to_bf16x2(y[8 * v + 0], y[8 * v + 1]);
        u.y = f32_to_bf16x2(y[8 * v + 2], y[8 * v + 3]);
        u.z = f32_to_bf16x2(y[8 * v + 4], y[8 * v + 5]);
        u.w = f32_to_bf16x2(y[8 * v + 6], y[8 * v + 7]);
        st_stream(p + 8 * v, u);
    }
}
template <int N>
__device__ __forceinline__ void store_block(float* p, const float (&y)[N])
{
#pragma unroll
    for (int v = 0; v < N / 4; ++v) {
        uint4 u = make_uint4(__float_as_uint(y[4 * v + 0]), __float_as_uint(y[4 * v + 1]),
                             __float_as_uint(y[4 * v + 2]), __float_as_uint(y[4 * v + 3]));
        st_stream(p + 4 * v, u);
    }
}

constexpr int32_t kFlagNonfinite = 1;
constexpr int32_t kFlagRange = 2;
constexpr int32_t kFlagTimeout = 4;

}  // namespace fp4q
