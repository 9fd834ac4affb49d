// fp4q_device.cuh -- device-side format conversions shared by the quantizer,
// dequantizer and GEMM kernels of the fp4q library (sm_100a only).
//
// Formats (see the public header for the page citations):
//   E2M1 element  : sign<<3 | magnitude index, magnitudes {0,.5,1,1.5,2,3,4,6}
//   E4M3 scale    : OCP E4M3FN, largest finite 448
//   E3M3 scale    : 6-bit unsigned, bias 3, 2^-5 .. 30
//   E8M0 scale    : 2^(byte-127)
//
// All fp32 arithmetic that decides a code or produces an output goes through
// explicit round-to-nearest intrinsics (__fmul_rn, __fsub_rn, __fmaf_rn) and
// the library is compiled with -fmad=false, so no contraction changes a
// rounding behind our back.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

namespace fp4q {

constexpr float kFltMax = 3.402823466e+38f;

// ---------------------------------------------------------------- E2M1
// Encode 8 fp32 values to 8 E2M1 codes (RNE, saturating, sign kept), value i
// in nibble i of the result.
__device__ __forceinline__ uint32_t e2m1x8_encode(float y0, float y1, float y2, float y3,
                                                  float y4, float y5, float y6, float y7)
{
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
        "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
        : "=r"(out)
        : "f"(y0), "f"(y1), "f"(y2), "f"(y3), "f"(y4), "f"(y5), "f"(y6), "f"(y7));
    return out;
}

// Encode 4 values into the low 16 bits.
__device__ __forceinline__ uint32_t e2m1x4_encode(float y0, float y1, float y2, float y3)
{
    uint32_t out;
    asm("{\n\t.reg .b8 b0, b1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
        "mov.b32 %0, {b0, b1, b1, b1};\n\t}"
        : "=r"(out)
        : "f"(y0), "f"(y1), "f"(y2), "f"(y3));
    return out & 0xFFFFu;
}

// Decode the two E2M1 codes of one byte (low nibble first) to fp32; exact.
// The byte is handed to the conversion as the low half of a zero-extended
// 16-bit register, one conversion per byte.
__device__ __forceinline__ float2 e2m1x2_decode(uint32_t byte)
{
    uint32_t h2;
    const unsigned short b16 = (unsigned short)(byte & 0xFFu);
    asm("{\n\t.reg .b8 lo, hi;\n\t"
        "mov.b16 {lo, hi}, %1;\n\t"
        "cvt.rn.f16x2.e2m1x2 %0, lo;\n\t}"
        : "=r"(h2)
        : "h"(b16));
    return __half22float2(*reinterpret_cast<__half2*>(&h2));
}

// Decode 8 E2M1 codes (nibble i = value i) to fp32; exact.
__device__ __forceinline__ void e2m1x8_decode(uint32_t w, float (&v)[8])
{
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float2 f = e2m1x2_decode(w >> (8 * k));
        v[2 * k] = f.x;
        v[2 * k + 1] = f.y;
    }
}

// Decode the low 4 nibbles.
__device__ __forceinline__ void e2m1x4_decode(uint32_t w, float (&v)[4])
{
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float2 f = e2m1x2_decode(w >> (8 * k));
        v[2 * k] = f.x;
        v[2 * k + 1] = f.y;
    }
}

// ---------------------------------------------------------------- E4M3
// Non-negative r -> E4M3 code (RNE, saturating at 448).
__device__ __forceinline__ uint32_t e4m3_encode(float r)
{
    uint16_t out;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %2, %1;" : "=h"(out) : "f"(r), "f"(0.0f));
    return out & 0xFFu;
}

// E4M3 code (low 8 bits; sign bit honoured) -> fp32; exact.
__device__ __forceinline__ float e4m3_decode(uint32_t code)
{
    uint32_t h;
    uint16_t c = (uint16_t)(code & 0xFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(c));
    return __half2float(__ushort_as_half((unsigned short)(h & 0xFFFFu)));
}

// ---------------------------------------------------------------- E3M3
// Non-negative r -> E3M3 code, RNE, saturating at 30.  Below 2^-2 the format
// is a fixed-point grid of step 2^-5 (rint of r*32, ties to even = even code);
// from 2^-2 to 30 it has E4M3's 3-bit mantissa, so the E4M3 code shifted by
// 4 exponent steps is the answer, clamped at 30.
__device__ __forceinline__ uint32_t e3m3_encode(float r)
{
    if (r < 0.25f)
        return (uint32_t)rintf(__fmul_rn(r, 32.0f));
    uint32_t c4 = e4m3_encode(r);
    c4 = c4 > 0x5Fu ? 0x5Fu : c4;     // 0x5F = 30 in E4M3
    return c4 - 32u;
}

__device__ __forceinline__ float e3m3_decode(uint32_t code)
{
    code &= 0x3Fu;
    if (code < 8u)
        return __fmul_rn((float)code, 0.03125f);
    return e4m3_decode(code + 32u);
}

// UE5M3 ("Finer is Better" summary, findings: the wide-exponent block scale):
// unsigned, 5 exponent bits with bias 15 over 3 mantissa bits, subnormals at
// exponent 0, codes 0..254 finite (0xFF is not a number and never produced).
// Encode: nearest value, ties to the even code, saturating at 0xFE = 114688.
__device__ __forceinline__ uint32_t ue5m3_encode(float r)
{
    if (!(r < 114688.0f))
        return 0xFEu;
    if (r < 6.103515625e-05f) {   // below 2^-14: multiples of 2^-17, 8 -> the first normal
        return (uint32_t)rintf(__fmul_rn(r, 131072.0f));
    }
    const uint32_t bits = __float_as_uint(r);
    const uint32_t rounded = bits + 0x7FFFFu + ((bits >> 20) & 1u);   // to 3 mantissa bits, ties even
    const uint32_t code = (rounded >> 20) - (112u << 3);               // exponent bias 127 -> 15
    return code > 0xFEu ? 0xFEu : code;
}

__device__ __forceinline__ float ue5m3_decode(uint32_t code)
{
    const uint32_t e = (code >> 3) & 31u, m = code & 7u;
    if (e == 0u)
        return __fmul_rn((float)m, 7.62939453125e-06f);   // m * 2^-17
    return __uint_as_float(((e + 112u) << 23) | (m << 20));
}

// Block-scale format of the NVFP4-style quantizers: 0 = E4M3 (NVFP4), 1 = UE5M3.
template <int SFMT>
__device__ __forceinline__ uint32_t sf_encode(float r)
{
    if constexpr (SFMT == 1)
        return ue5m3_encode(r);
    else
        return e4m3_encode(r);
}

template <int SFMT>
__device__ __forceinline__ float sf_decode(uint32_t code)
{
    if constexpr (SFMT == 1)
        return ue5m3_decode(code);
    else
        return e4m3_decode(code);
}

// ---------------------------------------------------------------- loads
// Load N consecutive input elements starting at p (16-byte aligned when the
// byte count allows) into fp32 registers.
template <int N>
__device__ __forceinline__ void load_f32(const float* __restrict__ p, float (&x)[N])
{
    static_assert(N % 4 == 0, "fp32 loads come in float4");
#pragma unroll
    for (int i = 0; i < N; i += 4) {
        float4 v = __ldg(reinterpret_cast<const float4*>(p + i));
        x[i] = v.x; x[i + 1] = v.y; x[i + 2] = v.z; x[i + 3] = v.w;
    }
}

__device__ __forceinline__ void bf16x2_to_f32(uint32_t w, float& lo, float& hi)
{
    lo = __uint_as_float(w << 16);
    hi = __uint_as_float(w & 0xFFFF0000u);
}

template <int N>
__device__ __forceinline__ void load_bf16(const __nv_bfloat16* __restrict__ p, float (&x)[N])
{
    static_assert(N % 4 == 0, "bf16 loads come in groups of 4");
    if constexpr (N % 8 == 0) {
#pragma unroll
        for (int i = 0; i < N; i += 8) {
            uint4 v = __ldg(reinterpret_cast<const uint4*>(p + i));
            bf16x2_to_f32(v.x, x[i], x[i + 1]);
            bf16x2_to_f32(v.y, x[i + 2], x[i + 3]);
            bf16x2_to_f32(v.z, x[i + 4], x[i + 5]);
            bf16x2_to_f32(v.w, x[i + 6], x[i + 7]);
        }
    } else {
#pragma unroll
        for (int i = 0; i < N; i += 4) {
            uint2 v = __ldg(reinterpret_cast<const uint2*>(p + i));
            bf16x2_to_f32(v.x, x[i], x[i + 1]);
            bf16x2_to_f32(v.y, x[i + 2], x[i + 3]);
        }
    }
}

template <typename T, int N>
__device__ __forceinline__ void load_elems(const T* __restrict__ p, float (&x)[N])
{
    if constexpr (sizeof(T) == 4)
        load_f32<N>(reinterpret_cast<const float*>(p), x);
    else
        load_bf16<N>(reinterpret_cast<const __nv_bfloat16*>(p), x);
}

// ------------------------------------------------ warp-staged block loads
// 16-byte streaming load that does not allocate in L1.
__device__ __forceinline__ uint4 ldg_stream(const uint4* p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Shared-memory slot of 16-byte chunk p of block i when a block is CPB chunks
// (2, 4 or 8): XOR-swizzled so that a warp's row-wise stores (8 consecutive
// lanes = consecutive chunks) and its block-wise loads (8 consecutive lanes =
// the same chunk of consecutive blocks) both hit 8 distinct 16-byte bank
// groups per phase.
template <int CPB>
__device__ __forceinline__ int staged_slot(int i, int p)
{
    static_assert(CPB == 2 || CPB == 4 || CPB == 8, "2, 4 or 8 chunks per block");
    if constexpr (CPB == 8)
        return i * 8 + (p ^ (i & 7));
    else if constexpr (CPB == 4)
        return i * 4 + (p ^ ((i >> 1) & 3));
    else
        return i * 2 + (p ^ ((i >> 2) & 1));
}

// A warp loads its 32 consecutive blocks of B elements (block `base` + lane
// for each lane; blocks at or past nblk read as zero) as whole 512-byte rows
// and hands each lane its own block, via `buf` (this warp's 32 * B *
// sizeof(T) bytes of shared memory).  A lane reading its 64-128 contiguous
// bytes straight from global memory would touch 16-32 cache lines per warp
// instruction.
template <typename T, int B>
__device__ __forceinline__ void warp_load_blocks(const T* __restrict__ x, int64_t base, int64_t nblk,
                                                 uint4* buf, float (&xv)[B])
{
    constexpr int CPB = B * (int)sizeof(T) / 16;
    const int lane = threadIdx.x & 31;
    const int64_t left = nblk - base;
    const int nb = left < 32 ? (int)left : 32;
    const uint4* src = reinterpret_cast<const uint4*>(x + base * B);
    uint4 v[CPB];
#pragma unroll
    for (int k = 0; k < CPB; ++k) {
        const int c = lane + 32 * k;
        v[k] = c / CPB < nb ? ldg_stream(src + c) : make_uint4(0u, 0u, 0u, 0u);
    }
    __syncwarp();   // the previous blocks have been read back
#pragma unroll
    for (int k = 0; k < CPB; ++k) {
        const int c = lane + 32 * k;
        buf[staged_slot<CPB>(c / CPB, c % CPB)] = v[k];
    }
    __syncwarp();
#pragma unroll
    for (int p = 0; p < CPB; ++p) {
        const uint4 q = buf[staged_slot<CPB>(lane, p)];
        if constexpr (sizeof(T) == 4) {
            xv[4 * p] = __uint_as_float(q.x);
            xv[4 * p + 1] = __uint_as_float(q.y);
            xv[4 * p + 2] = __uint_as_float(q.z);
            xv[4 * p + 3] = __uint_as_float(q.w);
        } else {
            bf16x2_to_f32(q.x, xv[8 * p], xv[8 * p + 1]);
            bf16x2_to_f32(q.y, xv[8 * p + 2], xv[8 * p + 3]);
            bf16x2_to_f32(q.z, xv[8 * p + 4], xv[8 * p + 5]);
            bf16x2_to_f32(q.w, xv[8 * p + 6], xv[8 * p + 7]);
        }
    }
}

// The converse of warp_load_blocks for fp32 outputs of B elements per block
// (B = 8, 16 or 32): the warp's lanes put their blocks into `buf` (this warp's
// 32 * B * 4 bytes of shared memory) and the warp writes the 32 blocks as
// whole rows, 512 consecutive bytes per store instruction; blocks at or past
// nblk are not written.  A lane storing its own 32-128 contiguous bytes would
// touch 16-32 different 32-byte sectors per warp instruction.
template <int B>
__device__ __forceinline__ void warp_store_f32_blocks(float* __restrict__ out, int64_t base, int64_t nblk,
                                                      uint4* buf, const float (&v)[B])
{
    constexpr int CPB = B / 4;
    const int lane = threadIdx.x & 31;
    const int64_t left = nblk - base;
    const int nb = left < 32 ? (int)left : 32;
    __syncwarp();   // the buffer's previous contents have been read
#pragma unroll
    for (int p = 0; p < CPB; ++p)
        buf[staged_slot<CPB>(lane, p)] = make_uint4(__float_as_uint(v[4 * p]), __float_as_uint(v[4 * p + 1]),
                                                    __float_as_uint(v[4 * p + 2]), __float_as_uint(v[4 * p + 3]));
    __syncwarp();
    uint4* dst = reinterpret_cast<uint4*>(out + base * B);
#pragma unroll
    for (int k = 0; k < CPB; ++k) {
        const int c = lane + 32 * k;
        if (c / CPB < nb)
            dst[c] = buf[staged_slot<CPB>(c / CPB, c % CPB)];
    }
}

template <int N>
__device__ __forceinline__ void store_f32(float* __restrict__ p, const float (&x)[N])
{
#pragma unroll
    for (int i = 0; i < N; i += 4)
        *reinterpret_cast<float4*>(p + i) = make_float4(x[i], x[i + 1], x[i + 2], x[i + 3]);
}

// Store the packed codes of one block: N/2 bytes from the words w[].
template <int N>
__device__ __forceinline__ void store_codes(uint8_t* __restrict__ p, const uint32_t (&w)[(N + 7) / 8])
{
    if constexpr (N == 4)
        *reinterpret_cast<uint16_t*>(p) = (uint16_t)w[0];
    else if constexpr (N == 8)
        *reinterpret_cast<uint32_t*>(p) = w[0];
    else if constexpr (N == 16)
        *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
    else
        *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}

// Offset of scale (row r, scale column kb) in the tcgen05 block-scaled MMA
// scale-factor layout: 128-row x 4-column atoms of 512 bytes, atoms ordered
// with the scale-column index fastest; inside an atom, row r goes to
// 16*(r%32) + 4*((r/32)%4) and column kb to kb%4.
__device__ __forceinline__ int64_t mma_sf_offset(int64_t r, int64_t kb, int64_t kb_atoms)
{
    return ((r >> 7) * kb_atoms + (kb >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (kb & 3);
}

}  // namespace fp4q
