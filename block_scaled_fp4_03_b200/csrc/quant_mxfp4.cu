// quant_mxfp4.cu -- the MXFP4 path of MACaQ ("MACaQ: Fast, Model Agnostic
// Calibrated Quantization ..." review, section 1 Key Terms and section 3
// Method): per-channel online scale t, size-32 block-Hadamard rotation, OCP
// E8M0 shared exponent, Hessian-weighted exponent choice among the standard
// exponent plus {+1, 0, -1}, the 32x32 diagonal Hessian blocks it weights
// with, and the calibration of t from weight and activation statistics.
//
// Layout: row-major tensors, 32-element blocks along the last dimension.
// Every quantization decision is made by one thread per block in fp32 with
// explicit round-to-nearest operations, in the same order as the definition.
#include <cfloat>
#include <cstdint>

#include "fp4q_device.cuh"
#include "fp4q_internal.h"
#include "tc05_common.cuh"

namespace fp4q {

namespace {

constexpr int kThreads = 256;

// fp32 nearest to 1/sqrt(32) (the Hadamard normalisation), bit pattern 0x3E3504F3.
__device__ __forceinline__ float had_norm() { return __uint_as_float(0x3E3504F3u); }

// 2^e as fp32 for e in [-127, 127] (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float pow2f(int e)
{
    return e <= -127 ? __uint_as_float(0x00400000u) : __uint_as_float((uint32_t)(e + 127) << 23);
}

// u <- (u * t) then the in-register Sylvester butterflies for strides 1..16
// and the 1/sqrt(32) normalisation.
__device__ __forceinline__ void online_transform(float (&u)[32], const float* __restrict__ t,
                                                 bool had)
{
    if (t) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
            float4 tv = __ldg(reinterpret_cast<const float4*>(t + i));
            u[i] = __fmul_rn(u[i], tv.x);
            u[i + 1] = __fmul_rn(u[i + 1], tv.y);
            u[i + 2] = __fmul_rn(u[i + 2], tv.z);
            u[i + 3] = __fmul_rn(u[i + 3], tv.w);
        }
    }
    if (had) {
#pragma unroll
        for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                if ((i & h) == 0) {
                    const float p = u[i], q = u[i + h];
                    u[i] = __fadd_rn(p, q);
                    u[i + h] = __fsub_rn(p, q);
                }
            }
        }
        const float c = had_norm();
#pragma unroll
        for (int i = 0; i < 32; ++i)
            u[i] = __fmul_rn(u[i], c);
    }
}

// OCP MX shared exponent: floor(log2 a) - 2, clamped to [-127, 127]; a
// subnormal or zero block maximum gives -127.
__device__ __forceinline__ int mx_exponent(float a)
{
    const uint32_t E = __float_as_uint(a) >> 23;   // a >= 0
    if (E == 0u)
        return -127;
    const int e = (int)E - 129;
    return e < -127 ? -127 : e;
}

// Quantize one 32-block at exponent e: codes, deq, ordered squared error.
__device__ __forceinline__ float mx_eval(const float (&u)[32], int e, uint32_t (&cw)[4],
                                         float (&dq)[32])
{
    const float down = pow2f(-e);
    const float up = pow2f(e);
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int o = 8 * j;
        uint32_t w = e2m1x8_encode(__fmul_rn(u[o], down), __fmul_rn(u[o + 1], down),
                                   __fmul_rn(u[o + 2], down), __fmul_rn(u[o + 3], down),
                                   __fmul_rn(u[o + 4], down), __fmul_rn(u[o + 5], down),
                                   __fmul_rn(u[o + 6], down), __fmul_rn(u[o + 7], down));
        float v[8];
        e2m1x8_decode(w, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float d = __fmul_rn(v[i], up);
            const float er = __fsub_rn(u[o + i], d);
            acc = __fmaf_rn(er, er, acc);
            dq[o + i] = d;
        }
        cw[j] = w;
    }
    return acc;
}

template <typename T>
__device__ __forceinline__ void load32(const T* __restrict__ p, float (&u)[32])
{
    load_elems<T, 32>(p, u);
}

// ------------------------------------------------- OCP exponent (activations)
// One lane per 32-block, but the loads are cooperative: a warp reads its 32
// consecutive blocks (and their 32 channel-scale slices) as whole 512-byte
// rows, parks them in shared memory, and each lane reads its own block back.
// A lane reading 64-128 contiguous bytes straight from global memory would
// touch 16-32 cache lines per warp instruction; the L1 would then serve many
// times the wavefronts the bytes need and cap the kernel far below HBM rate.
// Shared-memory slots are XOR-swizzled so that both the row-wise stores and
// the block-wise loads are free of bank conflicts.
constexpr int kMxWarps = kThreads / 32;

// ERR: also produce the dequantized values / block errors (only when asked).
template <typename T, bool ERR>
__global__ void __launch_bounds__(kThreads, 2)
mx_quant_absmax_kernel(const T* __restrict__ x, uint32_t nblk, uint32_t kb,
                       const float* __restrict__ t, int had, uint8_t* __restrict__ codes,
                       uint8_t* __restrict__ scales, float* __restrict__ deq,
                       float* __restrict__ mse, int mma)
{
    // a GEMM launched after this kernel with programmatic stream serialization
    // may start its setup now; it waits for this grid's completion (and the
    // visibility of its writes) before reading A
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr int CPB = 32 * (int)sizeof(T) / 16;   // 16-byte chunks per block
    // one 4 KB buffer per warp: first the warp's blocks, then their t slices
    __shared__ uint4 buf[kMxWarps][32 * 8];
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    uint4* bw = buf[w];
    const uint64_t warp0 = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint64_t nwarps = ((uint64_t)gridDim.x * blockDim.x) >> 5;
    for (uint64_t base = warp0 * 32; base < nblk; base += nwarps * 32) {
        const uint32_t nb = (uint32_t)((nblk - base) < 32 ? (nblk - base) : 32);
        const uint4* src = reinterpret_cast<const uint4*>(x + base * 32);
        {
            uint4 v[CPB];
#pragma unroll
            for (int k = 0; k < CPB; ++k) {
                const int c = lane + 32 * k;
                v[k] = (uint32_t)(c / CPB) < nb ? ldg_stream(src + c) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int k = 0; k < CPB; ++k) {
                const int c = lane + 32 * k;
                bw[staged_slot<CPB>(c / CPB, c % CPB)] = v[k];
            }
        }
        __syncwarp();
        float u[32];
#pragma unroll
        for (int p = 0; p < CPB; ++p) {
            const uint4 q = bw[staged_slot<CPB>(lane, p)];
            if constexpr (CPB == 8) {
                u[4 * p] = __uint_as_float(q.x);
                u[4 * p + 1] = __uint_as_float(q.y);
                u[4 * p + 2] = __uint_as_float(q.z);
                u[4 * p + 3] = __uint_as_float(q.w);
            } else {
                bf16x2_to_f32(q.x, u[8 * p], u[8 * p + 1]);
                bf16x2_to_f32(q.y, u[8 * p + 2], u[8 * p + 3]);
                bf16x2_to_f32(q.z, u[8 * p + 4], u[8 * p + 5]);
                bf16x2_to_f32(q.w, u[8 * p + 6], u[8 * p + 7]);
            }
        }
        if (t) {
            const uint32_t kb0 = (uint32_t)(base % kb);
            uint4 tv[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int c = lane + 32 * k;
                const uint32_t kbi = (kb0 + (uint32_t)(c >> 3)) % kb;
                tv[k] = __ldg(reinterpret_cast<const uint4*>(t + (size_t)kbi * 32) + (c & 7));
            }
            __syncwarp();   // every lane has read its block
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int c = lane + 32 * k;
                bw[staged_slot<8>(c >> 3, c & 7)] = tv[k];
            }
            __syncwarp();
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const uint4 q = bw[staged_slot<8>(lane, p)];
                u[4 * p] = __fmul_rn(u[4 * p], __uint_as_float(q.x));
                u[4 * p + 1] = __fmul_rn(u[4 * p + 1], __uint_as_float(q.y));
                u[4 * p + 2] = __fmul_rn(u[4 * p + 2], __uint_as_float(q.z));
                u[4 * p + 3] = __fmul_rn(u[4 * p + 3], __uint_as_float(q.w));
            }
        }
        __syncwarp();   // the buffers are refilled next iteration
        online_transform(u, nullptr, had != 0);
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            a = fmaxf(a, fabsf(u[i]));
        const int e = mx_exponent(a);
        uint32_t cw[4];
        const uint64_t b = base + (uint64_t)lane;
        if constexpr (ERR) {
            float dq[32];
            const float sse = mx_eval(u, e, cw, dq);
            if ((uint32_t)lane < nb) {
                if (deq)
                    store_f32<32>(deq + b * 32, dq);
                if (mse)
                    mse[b] = __fmul_rn(sse, 1.0f / 32.0f);
            }
        } else {
            const float down = pow2f(-e);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int o = 8 * j;
                cw[j] = e2m1x8_encode(__fmul_rn(u[o], down), __fmul_rn(u[o + 1], down),
                                      __fmul_rn(u[o + 2], down), __fmul_rn(u[o + 3], down),
                                      __fmul_rn(u[o + 4], down), __fmul_rn(u[o + 5], down),
                                      __fmul_rn(u[o + 6], down), __fmul_rn(u[o + 7], down));
            }
        }
        if ((uint32_t)lane < nb) {
            *reinterpret_cast<uint4*>(codes + b * 16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            const uint64_t r = b / kb;
            scales[mma ? mma_sf_offset((int64_t)r, (int64_t)(b - r * kb), kb >> 2) : (int64_t)b] =
                (uint8_t)(e + 127);
        }
    }
}

// ------------------------------------- OCP exponent (activations), two lanes
// per block.  Lanes 2j and 2j+1 hold the two 16-element halves of a warp's
// block j (16 blocks per warp and step), which halves the registers a lane
// needs and lets four CTAs share an SM.  The rotation's strides 1-8 stay
// inside a half; stride 16 pairs element i of one half with element i of the
// other, exchanged with one shuffle, and each lane applies the same add or
// subtract (a + b on the first half, a - b on the second) as the one-lane
// form.  The maximum is the maximum of the two halves' maxima; the ordered
// squared error runs over the first half in one lane and continues over the
// second half in the other.  The channel scale t is kept whole in shared
// memory (16-byte chunks XOR-swizzled by column block, so a warp's reads are
// conflict-free); the warp's 16 blocks are read as whole rows, parked in
// shared memory and picked up by half, and the next group's loads are in
// flight while the current one is transformed.
constexpr int kMx2BlocksPerWarp = 16;
// largest cols/32 whose t table fits the shared-memory budget of this kernel
constexpr int kMx2MaxColBlocks = 512;

template <typename T, bool ERR>
__global__ void __launch_bounds__(kThreads, ERR ? 3 : 4)
mx_quant_absmax2_kernel(const T* __restrict__ x, uint32_t nblk, uint32_t kb,
                        const float* __restrict__ t, int had, uint8_t* __restrict__ codes,
                        uint8_t* __restrict__ scales, float* __restrict__ deq,
                        float* __restrict__ mse, int mma)
{
    // a GEMM launched after this kernel with programmatic stream serialization
    // may start its setup now; it waits for this grid's completion (and the
    // visibility of its writes) before reading A
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    constexpr int CPB = 32 * (int)sizeof(T) / 16;   // 16-byte chunks per block
    constexpr int CPL = CPB / 2;                      // chunks per lane (its half)
    constexpr int kStage = kMx2BlocksPerWarp * CPB;   // chunks per warp
    extern __shared__ uint4 mx2_smem[];
    uint4* ttab = mx2_smem;                                       // kb rows of 8 chunks
    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    uint4* stage = mx2_smem + (t ? (size_t)kb * 8 : 0) + (size_t)w * kStage;
    if (t) {
        const uint4* t4 = reinterpret_cast<const uint4*>(t);
        for (uint32_t i = threadIdx.x; i < kb * 8u; i += blockDim.x) {
            const uint32_t r = i >> 3, p = i & 7u;
            ttab[r * 8u + (p ^ (r & 7u))] = __ldg(t4 + i);
        }
        __syncthreads();
    }
    const int j = lane >> 1;          // this lane's block within the warp's group
    const int h = lane & 1;           // and its half
    const uint64_t warp0 = ((uint64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const uint64_t nwarps = ((uint64_t)gridDim.x * blockDim.x) >> 5;
    const uint64_t step = nwarps * kMx2BlocksPerWarp;
    uint4 v[CPL];
    auto fetch = [&](uint64_t gbase) {
        const uint64_t left = nblk - gbase;
        const uint32_t nb = (uint32_t)(left < kMx2BlocksPerWarp ? left : kMx2BlocksPerWarp);
        const uint4* src = reinterpret_cast<const uint4*>(x + gbase * 32);
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
            const int c = lane + 32 * k;
            v[k] = (uint32_t)(c / CPB) < nb ? ldg_stream(src + c) : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    uint64_t base = warp0 * kMx2BlocksPerWarp;
    if (base < nblk)
        fetch(base);
    for (; base < nblk; base += step) {
        const uint64_t left = nblk - base;
        const uint32_t nb = (uint32_t)(left < kMx2BlocksPerWarp ? left : kMx2BlocksPerWarp);
        __syncwarp();   // the previous group has been read back
#pragma unroll
        for (int k = 0; k < CPL; ++k) {
            const int c = lane + 32 * k;
            stage[staged_slot<CPB>(c / CPB, c % CPB)] = v[k];
        }
        __syncwarp();
        if (base + step < nblk)
            fetch(base + step);        // the next group's loads, in flight meanwhile
        float u[16];
#pragma unroll
        for (int p = 0; p < CPL; ++p) {
            const uint4 q = stage[staged_slot<CPB>(j, h * CPL + p)];
            if constexpr (sizeof(T) == 4) {
                u[4 * p] = __uint_as_float(q.x);
                u[4 * p + 1] = __uint_as_float(q.y);
                u[4 * p + 2] = __uint_as_float(q.z);
                u[4 * p + 3] = __uint_as_float(q.w);
            } else {
                bf16x2_to_f32(q.x, u[8 * p], u[8 * p + 1]);
                bf16x2_to_f32(q.y, u[8 * p + 2], u[8 * p + 3]);
                bf16x2_to_f32(q.z, u[8 * p + 4], u[8 * p + 5]);
                bf16x2_to_f32(q.w, u[8 * p + 6], u[8 * p + 7]);
            }
        }
        const uint64_t b = base + (uint64_t)j;
        const uint32_t kbi = (uint32_t)(b % kb);
        if (t) {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const uint4 q = ttab[kbi * 8u + ((uint32_t)(4 * h + p) ^ (kbi & 7u))];
                u[4 * p] = __fmul_rn(u[4 * p], __uint_as_float(q.x));
                u[4 * p + 1] = __fmul_rn(u[4 * p + 1], __uint_as_float(q.y));
                u[4 * p + 2] = __fmul_rn(u[4 * p + 2], __uint_as_float(q.z));
                u[4 * p + 3] = __fmul_rn(u[4 * p + 3], __uint_as_float(q.w));
            }
        }
        if (had) {
#pragma unroll
            for (int s = 1; s < 16; s <<= 1) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if ((i & s) == 0) {
                        const float p = u[i], q = u[i + s];
                        u[i] = __fadd_rn(p, q);
                        u[i + s] = __fsub_rn(p, q);
                    }
                }
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float o = __shfl_xor_sync(0xffffffffu, u[i], 1);
                u[i] = h == 0 ? __fadd_rn(u[i], o) : __fsub_rn(o, u[i]);
            }
            const float c = had_norm();
#pragma unroll
            for (int i = 0; i < 16; ++i)
                u[i] = __fmul_rn(u[i], c);
        }
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 16; ++i)
            a = fmaxf(a, fabsf(u[i]));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
        const int e = mx_exponent(a);
        const float down = pow2f(-e);
        uint32_t cw[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int o = 8 * q;
            cw[q] = e2m1x8_encode(__fmul_rn(u[o], down), __fmul_rn(u[o + 1], down),
                                  __fmul_rn(u[o + 2], down), __fmul_rn(u[o + 3], down),
                                  __fmul_rn(u[o + 4], down), __fmul_rn(u[o + 5], down),
                                  __fmul_rn(u[o + 6], down), __fmul_rn(u[o + 7], down));
        }
        const bool valid = (uint32_t)j < nb;
        if constexpr (ERR) {
            const float up = pow2f(e);
            float dq[16];
            float acc0 = 0.0f;     // the first half's error chain ...
            float acc = 0.0f;
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                float vv[8];
                e2m1x8_decode(cw[q], vv);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    dq[8 * q + i] = __fmul_rn(vv[i], up);
            }
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float er = __fsub_rn(u[i], dq[i]);
                acc0 = __fmaf_rn(er, er, acc0);
            }
            // ... continued over the second half from where the first ended
            acc = __shfl_xor_sync(0xffffffffu, acc0, 1);
            if (h == 1) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float er = __fsub_rn(u[i], dq[i]);
                    acc = __fmaf_rn(er, er, acc);
                }
            }
            if (valid) {
                if (deq)
                    store_f32<16>(deq + b * 32 + 16 * h, dq);
                if (mse && h == 1)
                    mse[b] = __fmul_rn(acc, 1.0f / 32.0f);
            }
        }
        if (valid) {
            *reinterpret_cast<uint2*>(codes + b * 16 + 8 * h) = make_uint2(cw[0], cw[1]);
            if (h == 0) {
                const uint64_t r = b / kb;
                scales[mma ? mma_sf_offset((int64_t)r, (int64_t)(b - r * kb), kb >> 2) : (int64_t)b] =
                    (uint8_t)(e + 127);
            }
        }
    }
}

// Block error d = u - deq(u, e) at exponent e.
__device__ __forceinline__ void mx_err(const float (&u)[32], int e, float (&d)[32])
{
    const float down = pow2f(-e);
    const float up = pow2f(e);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int o = 8 * j;
        uint32_t w = e2m1x8_encode(__fmul_rn(u[o], down), __fmul_rn(u[o + 1], down),
                                   __fmul_rn(u[o + 2], down), __fmul_rn(u[o + 3], down),
                                   __fmul_rn(u[o + 4], down), __fmul_rn(u[o + 5], down),
                                   __fmul_rn(u[o + 6], down), __fmul_rn(u[o + 7], down));
        float v[8];
        e2m1x8_decode(w, v);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            d[o + i] = __fsub_rn(u[o + i], __fmul_rn(v[i], up));
    }
}

// Hessian-weighted exponent (weights): among e0, e0 + 1, e0 - 1 (in that
// order, strict improvement only) the exponent with the least d^T H'_k d.
// For each candidate, v_i = sum_j H_ij d_j is an fma chain over j in order and
// the cost an fma chain of d_i v_i over i in order.  The three candidates'
// errors stay in registers and every row of H'_k (one broadcast 128-byte
// shared-memory read) feeds all three chains, so the kernel runs on the FMA
// pipe rather than on shared-memory bandwidth.
constexpr int kHessThreads = 128;

template <typename T>
__global__ void __launch_bounds__(kHessThreads, 3)
mx_quant_hessian_kernel(const T* __restrict__ x, int64_t rows, int64_t kb,
                        const float* __restrict__ t, int had, const float* __restrict__ hess,
                        uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                        float* __restrict__ deq, float* __restrict__ mse, int mma)
{
    __shared__ __align__(16) float Hs[32 * 32];   // H'_k, row-major
    const int64_t k = blockIdx.y;
    for (int i = threadIdx.x; i < 32 * 32; i += blockDim.x)
        Hs[i] = __ldg(hess + k * 1024 + i);
    __syncthreads();
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= rows)
        return;
    const int64_t b = r * kb + k;
    float u[32];
    load32<T>(x + b * 32, u);
    online_transform(u, t ? t + k * 32 : nullptr, had != 0);
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i)
        a = fmaxf(a, fabsf(u[i]));
    const int e0 = mx_exponent(a);
    // an exponent outside [-127, 127] is not a candidate; its chain runs on
    // the e0 error and is ignored
    const int eu = e0 + 1 <= 127 ? e0 + 1 : e0;
    const int ed = e0 - 1 >= -127 ? e0 - 1 : e0;
    float d0[32], d1[32], d2[32];
    mx_err(u, e0, d0);
    mx_err(u, eu, d1);
    mx_err(u, ed, d2);
    float c0 = 0.0f, c1 = 0.0f, c2 = 0.0f;
    const float4* H4 = reinterpret_cast<const float4*>(Hs);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        float v0 = 0.0f, v1 = 0.0f, v2 = 0.0f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const float4 h = H4[i * 8 + q];
            v0 = __fmaf_rn(h.x, d0[4 * q], v0);
            v1 = __fmaf_rn(h.x, d1[4 * q], v1);
            v2 = __fmaf_rn(h.x, d2[4 * q], v2);
            v0 = __fmaf_rn(h.y, d0[4 * q + 1], v0);
            v1 = __fmaf_rn(h.y, d1[4 * q + 1], v1);
            v2 = __fmaf_rn(h.y, d2[4 * q + 1], v2);
            v0 = __fmaf_rn(h.z, d0[4 * q + 2], v0);
            v1 = __fmaf_rn(h.z, d1[4 * q + 2], v1);
            v2 = __fmaf_rn(h.z, d2[4 * q + 2], v2);
            v0 = __fmaf_rn(h.w, d0[4 * q + 3], v0);
            v1 = __fmaf_rn(h.w, d1[4 * q + 3], v1);
            v2 = __fmaf_rn(h.w, d2[4 * q + 3], v2);
        }
        c0 = __fmaf_rn(d0[i], v0, c0);
        c1 = __fmaf_rn(d1[i], v1, c1);
        c2 = __fmaf_rn(d2[i], v2, c2);
    }
    int best_e = e0;
    float best = c0;
    if (eu != e0 && c1 < best) {
        best = c1;
        best_e = eu;
    }
    if (ed != e0 && c2 < best) {
        best = c2;
        best_e = ed;
    }
    uint32_t cw[4];
    float dq[32];
    const float sse = mx_eval(u, best_e, cw, dq);
    *reinterpret_cast<uint4*>(codes + b * 16) = make_uint4(cw[0], cw[1], cw[2], cw[3]);
    scales[mma ? mma_sf_offset(r, k, kb >> 2) : b] = (uint8_t)(best_e + 127);
    if (deq)
        store_f32<32>(deq + b * 32, dq);
    if (mse)
        mse[b] = __fmul_rn(sse, 1.0f / 32.0f);
}

// ------------------------------------------------------- Hessian blocks
// H'_k partial sums are taken over chunks of kTok tokens (hessian_partial_tc_kernel
// below) and summed in chunk order by hessian_reduce_kernel.
constexpr int kTok = 256;

__global__ void __launch_bounds__(kThreads)
hessian_reduce_kernel(const float* __restrict__ part, int64_t nchunk, int64_t total,
                      float* __restrict__ hess)
{
    const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (idx >= total)
        return;
    float s = 0.0f;
    for (int64_t c = 0; c < nchunk; ++c)
        s = __fadd_rn(s, __ldg(part + c * total + idx));
    hess[idx] = s;
}

// ------------------------------------------------------- channel scale
// Column statistics in fp64 over a chunk of kStatRows rows: sum and sum of
// squares.  A tile is one chunk x 256 columns: lane l of every warp owns the 8
// consecutive columns 8 l .. 8 l + 7 of the tile (one 16-byte bf16 vector or
// two fp32 vectors per row), and warp w adds rows w, w + 8, w + 16, ... of the
// chunk in that order, loading them in batches with the next batch in flight
// while the current one is added.  The 8 warps' partial sums are then added in
// warp order through shared memory.
constexpr int kStatRows = 256;
constexpr int kStatCols = 256;
constexpr int kStatWarps = kThreads / 32;
// 16-byte words a lane loads per batch: 4 rows of bf16 or 2 of fp32 (a deeper
// batch raises the double-buffered registers past two CTAs per SM)
constexpr int kStatBatchWords = 4;

template <typename T>
__device__ __forceinline__ void column_stats_tile(const T* __restrict__ x, int64_t rows, int64_t cols,
                                                  double* __restrict__ sum, double* __restrict__ sumsq,
                                                  int64_t tx, int64_t ty,
                                                  double (&red)[2][kStatWarps][kStatCols])
{
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int64_t c0 = tx * kStatCols + 8 * lane;
    const bool own = c0 < cols;
    const int64_t r0 = ty * kStatRows;
    const int64_t r1 = (r0 + kStatRows) < rows ? (r0 + kStatRows) : rows;
    double s[8], q[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        s[i] = 0.0;
        q[i] = 0.0;
    }
    // whole batches of kB rows are double-buffered, the rest go row by row
    constexpr int kWd = (int)sizeof(T) / 2;        // 16-byte words per row slice
    constexpr int kB = kStatBatchWords / kWd;      // rows per batch
    auto load_batch = [&](int64_t rb, uint4 (&wv)[kB][kWd]) {
#pragma unroll
        for (int k = 0; k < kB; ++k)
#pragma unroll
            for (int h = 0; h < kWd; ++h)
                wv[k][h] = __ldg(reinterpret_cast<const uint4*>(x + (rb + k * kStatWarps) * cols + c0) + h);
    };
    auto add_batch = [&](const uint4 (&wv)[kB][kWd]) {
#pragma unroll
        for (int k = 0; k < kB; ++k) {
#pragma unroll
            for (int h = 0; h < kWd; ++h) {
                const uint32_t u[4] = {wv[k][h].x, wv[k][h].y, wv[k][h].z, wv[k][h].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    if constexpr (sizeof(T) == 4) {
                        const double d = (double)__uint_as_float(u[e]);
                        s[4 * h + e] += d;
                        q[4 * h + e] = fma(d, d, q[4 * h + e]);
                    } else {
                        const double d0 = (double)__uint_as_float(u[e] << 16);
                        const double d1 = (double)__uint_as_float(u[e] & 0xFFFF0000u);
                        s[2 * e] += d0;
                        q[2 * e] = fma(d0, d0, q[2 * e]);
                        s[2 * e + 1] += d1;
                        q[2 * e + 1] = fma(d1, d1, q[2 * e + 1]);
                    }
                }
            }
        }
    };
    constexpr int64_t kSpan = (int64_t)(kB - 1) * kStatWarps;   // a batch's last row offset
    constexpr int64_t kStep = (int64_t)kB * kStatWarps;
    int64_t r = r0 + warp;
    if (own) {
        if (r + kSpan < r1) {
            uint4 wa[kB][kWd], wb[kB][kWd];
            load_batch(r, wa);
            for (;;) {
                const int64_t ra = r + kStep;
                const bool more_a = ra + kSpan < r1;
                if (more_a)
                    load_batch(ra, wb);
                add_batch(wa);
                r = ra;
                if (!more_a)
                    break;
                const int64_t rb = r + kStep;
                const bool more_b = rb + kSpan < r1;
                if (more_b)
                    load_batch(rb, wa);
                add_batch(wb);
                r = rb;
                if (!more_b)
                    break;
            }
        }
        for (; r < r1; r += kStatWarps) {
            float v[8];
            load_elems<T, 8>(x + r * cols + c0, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const double d = (double)v[i];
                s[i] += d;
                q[i] = fma(d, d, q[i]);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        red[0][warp][8 * lane + i] = s[i];
        red[1][warp][8 * lane + i] = q[i];
    }
    __syncthreads();
    // thread t finishes column t of the tile
    const int64_t c = tx * kStatCols + threadIdx.x;
    if (c < cols) {
        double ts = red[0][0][threadIdx.x], tq = red[1][0][threadIdx.x];
#pragma unroll
        for (int w = 1; w < kStatWarps; ++w) {
            ts += red[0][w][threadIdx.x];
            tq += red[1][w][threadIdx.x];
        }
        const int64_t o = ty * cols + c;
        if (sum)
            sum[o] = ts;
        sumsq[o] = tq;
    }
}

// Both tensors' statistics in one persistent launch: the weight tiles (sum and
// sum of squares, wch row chunks) come first, then the activation tiles (sum of
// squares, xch row chunks), and CTA b takes tiles b, b + gridDim.x, ...  A
// tile's partial sums do not depend on which CTA computes it or when.
template <typename TW, typename TX>
__global__ void __launch_bounds__(kThreads)
column_stats_kernel(const TW* __restrict__ w, int64_t n_out, double* __restrict__ wsum,
                    double* __restrict__ wsq, int64_t wch, const TX* __restrict__ x, int64_t tokens,
                    double* __restrict__ xsq, int64_t xch, int64_t cols)
{
    __shared__ double red[2][kStatWarps][kStatCols];
    const int64_t gx = (cols + kStatCols - 1) / kStatCols;
    const int64_t nw = gx * wch;
    const int64_t total = nw + gx * xch;
    for (int64_t t = blockIdx.x; t < total; t += gridDim.x) {
        if (t < nw) {
            column_stats_tile<TW>(w, n_out, cols, wsum, wsq, t % gx, t / gx, red);
        } else {
            const int64_t u = t - nw;
            column_stats_tile<TX>(x, tokens, cols, nullptr, xsq, u % gx, u / gx, red);
        }
        __syncthreads();   // the next tile reuses red
    }
}

// t_j = (sigma_j^W / rms_j^X)^alpha, t = 1 where a factor is zero; fp64, then
// rounded to fp32; t_inv = 1/t in fp32.  A CTA owns 32 columns; its 8 warps
// split the chunk partials (warp w sums chunks w, w + 8, ...), then one warp
// adds the 8 slices in a fixed order.
constexpr int kScaleSlices = kThreads / 32;

__global__ void __launch_bounds__(kThreads)
channel_scale_kernel(const double* __restrict__ wsum, const double* __restrict__ wsq,
                     int64_t wchunks, int64_t n_out, const double* __restrict__ xsq,
                     int64_t xchunks, int64_t tokens, int64_t cols, double alpha,
                     float* __restrict__ t, float* __restrict__ t_inv)
{
    __shared__ double red[3][kScaleSlices][32];
    const int lane = threadIdx.x & 31;
    const int slice = threadIdx.x >> 5;
    const int64_t j = (int64_t)blockIdx.x * 32 + lane;
    double s = 0.0, q = 0.0, h = 0.0;
    if (j < cols) {
        for (int64_t c = slice; c < wchunks; c += kScaleSlices) {
            s += __ldg(wsum + c * cols + j);
            q += __ldg(wsq + c * cols + j);
        }
        for (int64_t c = slice; c < xchunks; c += kScaleSlices)
            h += __ldg(xsq + c * cols + j);
    }
    red[0][slice][lane] = s;
    red[1][slice][lane] = q;
    red[2][slice][lane] = h;
    __syncthreads();
    if (slice != 0 || j >= cols)
        return;
    s = red[0][0][lane];
    q = red[1][0][lane];
    h = red[2][0][lane];
#pragma unroll
    for (int k = 1; k < kScaleSlices; ++k) {
        s += red[0][k][lane];
        q += red[1][k][lane];
        h += red[2][k][lane];
    }
    const double n = (double)n_out;
    const double mean = s / n;
    double var = q / n - mean * mean;
    var = var > 0.0 ? var : 0.0;
    const double sigma = sqrt(var);
    const double rms = sqrt(h / (double)tokens);
    double tj = 1.0;
    if (sigma > 0.0 && rms > 0.0)
        tj = pow(sigma / rms, alpha);
    const float t32 = (float)tj;
    t[j] = t32;
    if (t_inv)
        t_inv[j] = __frcp_rn(t32);
}

int grid_for(int64_t work, const void* kernel)
{
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0);
    if (per_sm < 1)
        per_sm = 1;
    int64_t want = (work + kThreads - 1) / kThreads;
    const int64_t cap = (int64_t)num_sms() * per_sm;
    want = want > cap ? cap : want;
    return (int)(want < 1 ? 1 : want);
}

// ------------------------------------------- Hessian blocks on tensor cores
// The same partial sums H'_k over a chunk of kTok tokens, as tcgen05 MMAs.
// Four column blocks k0..k0+3 of the transformed chunk X' (tokens x 128
// columns) are staged transposed, X'^T (128 rows = columns, K = tokens), in
// the K-major 128B-swizzled layout; the same tile is both MMA operands, so
// D = X'^T X' (128 x 128) holds the four wanted 32 x 32 blocks H'_k on its
// diagonal.  tf32 operands carry 11 significant bits, so every value is split
// x = hi + lo (hi = x rounded to tf32, lo = the remainder rounded to tf32) and
//   D = hi^T hi + hi^T lo + lo^T hi
// (lo^T lo, about 2^-22 relative, is dropped): three MMAs per k-step into one
// 128-column TMEM accumulator, so three CTAs share an SM.  Warps 0-3 stage
// (one token per lane, one column block per warp; the next K block's loads are
// in flight while the current one is transformed and stored) and then read
// back the diagonal block of their TMEM lane quarter; warp 4 owns the TMEM and
// issues the MMAs.  Waits are bounded (main-loop waits by `wait_limit` cycles);
// a CTA that gives up writes NaN into its partial blocks, which the reduction
// carries into H', and sets the caller's error word *err to 1.
constexpr int kHxKB = 32;                       // tokens per K block (128 B of tf32 per tile row)
constexpr int kHxTile = 128 * 128;              // bytes of one operand tile
constexpr int kHxThreads = 160;
// dynamic shared memory: 2 stages x (hi, lo) tiles, barriers, alignment slack;
// at most three CTAs fit an SM (each holds 128 of its 512 TMEM columns)
constexpr int kHxSmem = 4 * kHxTile + 2048;
constexpr int kHxCols = 128;
// kind::tf32, fp32 accumulate, K-major A and B, N = 128, M = 128
constexpr uint32_t kHxIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);




__device__ __forceinline__ void hx_mma(uint32_t tacc, uint64_t da, uint64_t db, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(tacc),
                 "l"(da), "l"(db), "r"(kHxIdesc), "r"(accumulate)
                 : "memory");
}



__device__ __forceinline__ float hx_tf32(float a)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(a));
    return __uint_as_float(r);
}

template <typename T>
__global__ void __launch_bounds__(kHxThreads, 1)
hessian_partial_tc_kernel(const T* __restrict__ x, int64_t rows, int64_t cols, const float* __restrict__ t,
                          int had, float* __restrict__ part, long long wait_limit, int* err)
{
    extern __shared__ uint8_t hx_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(hx_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + 4 * kHxTile);
    // bars: full[0], full[1] (128 stagers), empty[0], empty[1] (MMA commit),
    // acc_full, drain
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 6);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
    const uint32_t bar0 = smem_u32(bars);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t kb = cols / 32;
    const int64_t chunk = blockIdx.x;
    const int64_t k0 = 4 * (int64_t)blockIdx.y;
    const int nblk = (int)((kb - k0) < 4 ? (kb - k0) : 4);
    const int64_t r0 = chunk * kTok;
    constexpr int kSteps = kTok / kHxKB;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(bar0 + 8u * i, 128);
            mbar_init(bar0 + 8u * (2 + i), 1);
        }
        mbar_init(bar0 + 32u, 1);
        mbar_init(bar0 + 40u, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 4) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                     "r"(kHxCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp < 4) {
        // ---------------- staging: lane = token of the K block, warp = column block
        const int b = warp;
        const int64_t col0 = (k0 + b) * 32;
        constexpr int kRaw = 32 * (int)sizeof(T) / 16;     // 16-byte vectors per token row
        uint4 raw[kRaw];
        auto fetch = [&](int s) {
            const int64_t r = r0 + (int64_t)s * kHxKB + lane;
            if (b < nblk && r < rows) {
                const uint4* p = reinterpret_cast<const uint4*>(x + r * cols + col0);
#pragma unroll
                for (int v = 0; v < kRaw; ++v)
                    raw[v] = __ldg(p + v);
            } else {
#pragma unroll
                for (int v = 0; v < kRaw; ++v)
                    raw[v] = make_uint4(0u, 0u, 0u, 0u);
            }
        };
        fetch(0);
        for (int s = 0; s < kSteps && !*abort_flag; ++s) {
            const int st = s & 1;
            const uint32_t use = (uint32_t)(s >> 1);
            float u[32];
#pragma unroll
            for (int v = 0; v < kRaw; ++v) {
                if constexpr (sizeof(T) == 4) {
                    u[4 * v] = __uint_as_float(raw[v].x);
                    u[4 * v + 1] = __uint_as_float(raw[v].y);
                    u[4 * v + 2] = __uint_as_float(raw[v].z);
                    u[4 * v + 3] = __uint_as_float(raw[v].w);
                } else {
                    bf16x2_to_f32(raw[v].x, u[8 * v], u[8 * v + 1]);
                    bf16x2_to_f32(raw[v].y, u[8 * v + 2], u[8 * v + 3]);
                    bf16x2_to_f32(raw[v].z, u[8 * v + 4], u[8 * v + 5]);
                    bf16x2_to_f32(raw[v].w, u[8 * v + 6], u[8 * v + 7]);
                }
            }
            if (s + 1 < kSteps)
                fetch(s + 1);          // in flight while this block is transformed
            if (use > 0 && !mbar_wait(bar0 + 8u * (2 + st), (use - 1u) & 1u, abort_flag, wait_limit)) {
                *abort_flag = 1;
                break;
            }
            uint8_t* hi = sm + st * 2 * kHxTile;
            uint8_t* lo = hi + kHxTile;
            online_transform(u, t ? t + col0 : nullptr, had != 0);
            // X'^T: row m = 32 b + i, K position = lane; 16-byte chunk (lane/4)
            // XOR (m % 8) of the 128-byte row
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int m = 32 * b + i;
                const uint32_t off = (uint32_t)m * 128u + ((((uint32_t)lane >> 2) ^ ((uint32_t)m & 7u)) << 4) +
                                     ((uint32_t)lane & 3u) * 4u;
                const float h = hx_tf32(u[i]);
                *reinterpret_cast<float*>(hi + off) = h;
                *reinterpret_cast<float*>(lo + off) = hx_tf32(__fsub_rn(u[i], h));
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(bar0 + 8u * st);
        }
        // ---------------- epilogue: the diagonal 32 x 32 block of this lane quarter
        const bool ok =
            __all_sync(0xffffffffu, !*abort_flag && mbar_wait(bar0 + 32u, 0u, abort_flag, wait_limit));
        tc_fence_after();
        if (b < nblk) {
            float h[32];
            if (ok) {
                uint32_t r[32];
                tmem_ld32(tmem + ((uint32_t)(32 * b) << 16) + (uint32_t)(32 * b), r);
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    h[j] = __uint_as_float(r[j]);
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    h[j] = __uint_as_float(0x7FC00000u);
            }
            float* o = part + (chunk * kb + k0 + b) * 1024 + lane * 32;
#pragma unroll
            for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4*>(o + j) = make_float4(h[j], h[j + 1], h[j + 2], h[j + 3]);
        }
    } else if (lane == 0) {
        // ---------------- MMA issuer: D += hi hi^T + hi lo^T + lo hi^T per k-step
        bool issued = false;
        for (int s = 0; s < kSteps; ++s) {
            const int st = s & 1;
            if (!mbar_wait(bar0 + 8u * st, (uint32_t)(s >> 1) & 1u, abort_flag, wait_limit)) {
                *abort_flag = 1;
                break;
            }
            tc_fence_after();
            const uint32_t hi = smem_u32(sm + st * 2 * kHxTile);
            const uint32_t lo = hi + kHxTile;
#pragma unroll
            for (int k = 0; k < kHxKB / 8; ++k) {
                const uint64_t dh = sdesc_sw128(hi + 32u * k);
                const uint64_t dl = sdesc_sw128(lo + 32u * k);
                hx_mma(tmem, dh, dh, (s | k) != 0);
                hx_mma(tmem, dh, dl, 1u);
                hx_mma(tmem, dl, dh, 1u);
            }
            issued = true;
            tc_commit(bar0 + 8u * (2 + st));
        }
        if (!*abort_flag)
            tc_commit(bar0 + 32u);
        if (issued) {
            // every MMA of this CTA has finished before the TMEM goes away
            tc_commit(bar0 + 40u);
            if (!mbar_wait(bar0 + 40u, 0u, nullptr))
                *abort_flag = 1;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (threadIdx.x == 0 && *abort_flag)
        atomicExch(err, 1);
    if (warp == 4)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kHxCols) : "memory");
}

}  // namespace

size_t hessian_ws_bytes(int64_t rows, int64_t cols)
{
    const int64_t nchunk = (rows + kTok - 1) / kTok;
    return (size_t)nchunk * (size_t)(cols / 32) * 1024 * sizeof(float);
}

size_t channel_scale_ws_bytes(int64_t tokens, int64_t n_out, int64_t cols)
{
    const int64_t wch = (n_out + kStatRows - 1) / kStatRows;
    const int64_t xch = (tokens + kStatRows - 1) / kStatRows;
    return (size_t)(2 * wch + xch) * (size_t)cols * sizeof(double);
}

cudaError_t launch_mxfp4_quant(const void* x, int dtype, int64_t rows, int64_t cols,
                               const float* chan_scale, int hadamard, int rule, const float* hess,
                               uint8_t* codes, uint8_t* scales, float* deq, float* mse,
                               cudaStream_t s, int mma_layout)
{
    const int64_t kb = cols / 32;
    const int64_t nblk = rows * kb;
    if (rule == 4) {
        dim3 grid((unsigned)((rows + kHessThreads - 1) / kHessThreads), (unsigned)kb);
        if (dtype == 1)
            mx_quant_hessian_kernel<__nv_bfloat16><<<grid, kHessThreads, 0, s>>>(
                reinterpret_cast<const __nv_bfloat16*>(x), rows, kb, chan_scale, hadamard, hess,
                codes, scales, deq, mse, mma_layout);
        else
            mx_quant_hessian_kernel<float><<<grid, kHessThreads, 0, s>>>(
                reinterpret_cast<const float*>(x), rows, kb, chan_scale, hadamard, hess, codes,
                scales, deq, mse, mma_layout);
        return cudaGetLastError();
    }
    if (nblk > (int64_t)0xFFFFFFFFu)
        return cudaErrorInvalidValue;
    const bool err = deq || mse;
    if (kb <= kMx2MaxColBlocks) {
        // two lanes per block; the t table and the warps' staging in dynamic shared memory
        const int esz = dtype == 1 ? 2 : 4;
        const int smem = (chan_scale ? (int)kb * 128 : 0) + kMxWarps * kMx2BlocksPerWarp * 32 * esz;
        const void* kp = dtype == 1 ? (err ? (const void*)mx_quant_absmax2_kernel<__nv_bfloat16, true>
                                           : (const void*)mx_quant_absmax2_kernel<__nv_bfloat16, false>)
                                    : (err ? (const void*)mx_quant_absmax2_kernel<float, true>
                                           : (const void*)mx_quant_absmax2_kernel<float, false>);
        const cudaError_t ae = smem_opt_in(kp, kMx2MaxColBlocks * 128 + kMxWarps * kMx2BlocksPerWarp * 32 * 4);
        if (ae != cudaSuccess)
            return ae;
        int per_sm = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kp, kThreads, smem);
        per_sm = per_sm < 1 ? 1 : per_sm;
        const int64_t groups = (nblk + kMx2BlocksPerWarp - 1) / kMx2BlocksPerWarp;
        int64_t grid = (groups + kMxWarps - 1) / kMxWarps;
        const int64_t cap = (int64_t)num_sms() * per_sm;
        grid = grid > cap ? cap : grid;
        grid = grid < 1 ? 1 : grid;
        if (dtype == 1) {
            auto k = err ? mx_quant_absmax2_kernel<__nv_bfloat16, true> : mx_quant_absmax2_kernel<__nv_bfloat16, false>;
            k<<<(unsigned)grid, kThreads, smem, s>>>(reinterpret_cast<const __nv_bfloat16*>(x), (uint32_t)nblk,
                                                     (uint32_t)kb, chan_scale, hadamard, codes, scales, deq, mse,
                                                     mma_layout);
        } else {
            auto k = err ? mx_quant_absmax2_kernel<float, true> : mx_quant_absmax2_kernel<float, false>;
            k<<<(unsigned)grid, kThreads, smem, s>>>(reinterpret_cast<const float*>(x), (uint32_t)nblk, (uint32_t)kb,
                                                     chan_scale, hadamard, codes, scales, deq, mse, mma_layout);
        }
        return cudaGetLastError();
    }
    if (dtype == 1) {
        auto k = err ? mx_quant_absmax_kernel<__nv_bfloat16, true> : mx_quant_absmax_kernel<__nv_bfloat16, false>;
        k<<<grid_for(nblk, (const void*)k), kThreads, 0, s>>>(
            reinterpret_cast<const __nv_bfloat16*>(x), (uint32_t)nblk, (uint32_t)kb, chan_scale, hadamard,
            codes, scales, deq, mse, mma_layout);
    } else {
        auto k = err ? mx_quant_absmax_kernel<float, true> : mx_quant_absmax_kernel<float, false>;
        k<<<grid_for(nblk, (const void*)k), kThreads, 0, s>>>(reinterpret_cast<const float*>(x),
                                                               (uint32_t)nblk, (uint32_t)kb, chan_scale,
                                                               hadamard, codes, scales, deq, mse,
                                                               mma_layout);
    }
    return cudaGetLastError();
}

cudaError_t launch_hessian_blocks(const void* x, int dtype, int64_t rows, int64_t cols,
                                  const float* chan_scale, int hadamard, float* hess, float* part,
                                  int* err, cudaStream_t s)
{
    const int64_t kb = cols / 32;
    const int64_t nchunk = (rows + kTok - 1) / kTok;
    const long long limit = wait_limit_cycles();
    const cudaError_t hx_attr =
        dtype == 1 ? smem_opt_in((const void*)hessian_partial_tc_kernel<__nv_bfloat16>, kHxSmem)
                   : smem_opt_in((const void*)hessian_partial_tc_kernel<float>, kHxSmem);
    if (hx_attr != cudaSuccess)
        return hx_attr;
    dim3 grid((unsigned)nchunk, (unsigned)((kb + 3) / 4));
    if (dtype == 1)
        hessian_partial_tc_kernel<__nv_bfloat16><<<grid, kHxThreads, kHxSmem, s>>>(
            reinterpret_cast<const __nv_bfloat16*>(x), rows, cols, chan_scale, hadamard, part, limit, err);
    else
        hessian_partial_tc_kernel<float><<<grid, kHxThreads, kHxSmem, s>>>(
            reinterpret_cast<const float*>(x), rows, cols, chan_scale, hadamard, part, limit, err);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    const int64_t total = kb * 1024;
    hessian_reduce_kernel<<<(unsigned)((total + kThreads - 1) / kThreads), kThreads, 0, s>>>(
        part, nchunk, total, hess);
    return cudaGetLastError();
}

cudaError_t launch_mx_channel_scale(const void* x, int xdt, int64_t tokens, const void* w, int wdt,
                                    int64_t n_out, int64_t cols, float alpha, float* t,
                                    float* t_inv, void* ws, cudaStream_t s)
{
    const int64_t wch = (n_out + kStatRows - 1) / kStatRows;
    const int64_t xch = (tokens + kStatRows - 1) / kStatRows;
    double* wsum = reinterpret_cast<double*>(ws);
    double* wsq = wsum + wch * cols;
    double* xsq = wsq + wch * cols;
    const int64_t tiles = (cols + kStatCols - 1) / kStatCols * (wch + xch);
    auto launch = [&](auto kernel, const auto* wp, const auto* xp) {
        int per_sm = 0;
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0);
        const int64_t cap = (int64_t)num_sms() * (per_sm < 1 ? 1 : per_sm);
        const unsigned grid = (unsigned)(tiles < cap ? tiles : cap);
        kernel<<<grid, kThreads, 0, s>>>(wp, n_out, wsum, wsq, wch, xp, tokens, xsq, xch, cols);
    };
    const auto* wb = reinterpret_cast<const __nv_bfloat16*>(w);
    const auto* wf = reinterpret_cast<const float*>(w);
    const auto* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    const auto* xf = reinterpret_cast<const float*>(x);
    if (wdt == 1 && xdt == 1)
        launch(column_stats_kernel<__nv_bfloat16, __nv_bfloat16>, wb, xb);
    else if (wdt == 1)
        launch(column_stats_kernel<__nv_bfloat16, float>, wb, xf);
    else if (xdt == 1)
        launch(column_stats_kernel<float, __nv_bfloat16>, wf, xb);
    else
        launch(column_stats_kernel<float, float>, wf, xf);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    channel_scale_kernel<<<(unsigned)((cols + 31) / 32), kThreads, 0, s>>>(
        wsum, wsq, wch, n_out, xsq, xch, tokens, cols, (double)alpha, t, t_inv);
    return cudaGetLastError();
}

}  // namespace fp4q
