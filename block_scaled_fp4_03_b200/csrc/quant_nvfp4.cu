// quant_nvfp4.cu -- tensor amax, NVFP4 block quantization under the four
// scale rules, RaZeR remapping, and dequantization with per-block MSE.
//
// Method sources (web pages, by title and section):
//   NVFP4 format: "Why Gated DeltaNet Survives 4-Bit Quantization" review, s.1
//   scale rules : "Finer is Better (with the Right Scaling)", Methodology 2
//                 (abs-max, prevent-zero, 4-over-6, brute force, hierarchical)
//   RaZeR       : "RaZeR - Redundant Zero Remapping" summary, s.2.1-2.2
//
// Design: one thread owns one block of B contiguous elements (B <= 32), so
// the per-block decision -- the fp32 squared error accumulated with fma in
// element order -- is a single thread's register chain, bit-identical to the
// definition.  Warps walk the tensor in a grid-stride loop whose trip count
// is warp-uniform (lanes past the end are masked), so warp votes are legal.
// Inputs are read with 128-bit loads straight into registers; codes are
// packed in registers by the hardware e2m1x2 conversion and written with one
// vector store per block.
#include <cfloat>
#include <cmath>
#include <cstdint>
#include <mutex>
#include <utility>

#include "fp4q_device.cuh"
#include "fp4q_internal.h"

namespace fp4q {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float warp_max(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1)
        v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

// max |x| over the 16-byte vectors [v0, v1) of x, this CTA's threads
// striding by the block size with eight loads in flight per thread (the
// quantizer grids hold only 2-5 CTAs per SM).
template <typename T>
__device__ float cta_amax_part(const T* __restrict__ x, int64_t v0, int64_t v1)
{
    const uint4* xv = reinterpret_cast<const uint4*>(x);
    float m = 0.0f;
    auto fold = [&](const uint4& w) {
        if constexpr (sizeof(T) == 4) {
            m = fmaxf(m, fmaxf(fmaxf(fabsf(__uint_as_float(w.x)), fabsf(__uint_as_float(w.y))),
                               fmaxf(fabsf(__uint_as_float(w.z)), fabsf(__uint_as_float(w.w)))));
        } else {
            const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                float lo, hi;
                bf16x2_to_f32(ww[q], lo, hi);
                m = fmaxf(m, fmaxf(fabsf(lo), fabsf(hi)));
            }
        }
    };
    const int64_t st = blockDim.x;
    int64_t i = v0 + threadIdx.x;
    for (; i + 7 * st < v1; i += 8 * st) {
        uint4 w[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
            w[u] = __ldg(xv + i + u * st);
#pragma unroll
        for (int u = 0; u < 8; ++u)
            fold(w[u]);
    }
    for (; i < v1; i += st)
        fold(__ldg(xv + i));
    return m;
}

// max |x| of the elements past the last whole 16-byte vector.
template <typename T>
__device__ float amax_tail(const T* __restrict__ x, int64_t n)
{
    constexpr int V = 16 / sizeof(T);
    float m = 0.0f;
    for (int64_t i = n / V * V + threadIdx.x; i < n; i += blockDim.x) {
        float f;
        if constexpr (sizeof(T) == 4)
            f = reinterpret_cast<const float*>(x)[i];
        else
            f = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(x)[i] << 16);
        m = fmaxf(m, fabsf(f));
    }
    return m;
}

// Maximum over the CTA (every thread gets it).
__device__ __forceinline__ float cta_max(float m)
{
    __shared__ float red[kThreads / 32];
    __shared__ float s_m;
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = threadIdx.x < (int)(blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
        m = warp_max(m);
        if (threadIdx.x == 0)
            s_m = m;
    }
    __syncthreads();
    return s_m;
}

// Fused global maximum (GsArgs mode 3): every CTA takes the maximum of its own
// contiguous slice of x, publishes it and meets the others at a grid barrier
// (the launch is cooperative, so all CTAs are resident); then each reduces all
// partials.  The maximum is exact and order-free, so g is the same as from a
// separate pass.  The barrier wait is bounded: a CTA that gives up computes
// the maximum of the whole tensor itself (slower, same result).
template <typename T>
__device__ float fused_global_amax(const GsArgs& gs)
{
    __shared__ int s_alone;
    const T* x = reinterpret_cast<const T*>(gs.x);
    constexpr int V = 16 / sizeof(T);
    const int64_t nvec = gs.n / V;
    const int64_t per = (nvec + gridDim.x - 1) / gridDim.x;
    const int64_t v0 = (int64_t)blockIdx.x * per < nvec ? (int64_t)blockIdx.x * per : nvec;
    const int64_t v1 = v0 + per < nvec ? v0 + per : nvec;
    float m = cta_amax_part<T>(x, v0, v1);
    if (blockIdx.x == 0)
        m = fmaxf(m, amax_tail<T>(x, gs.n));
    m = cta_max(m);
    if (threadIdx.x == 0) {
        gs.fused_partials[blockIdx.x] = m;
        __threadfence();
        atomicAdd(gs.counter, 1u);
        int alone = 0;
        const long long t0 = clock64();
        for (;;) {
            unsigned int c;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(c) : "l"(gs.counter) : "memory");
            if (c >= gridDim.x)
                break;
            if (clock64() - t0 > gs.wait_limit) {
                alone = 1;
                break;
            }
        }
        s_alone = alone;
    }
    __syncthreads();
    if (s_alone) {
        m = cta_amax_part<T>(x, 0, nvec);
        m = fmaxf(m, amax_tail<T>(x, gs.n));
    } else {
        m = 0.0f;
        for (int i = threadIdx.x; i < (int)gridDim.x; i += blockDim.x)
            m = fmaxf(m, __ldcg(gs.fused_partials + i));
    }
    return cta_max(m);
}

// The per-tensor global scale for this launch (all threads of the CTA get it).
template <typename T>
__device__ float resolve_global_scale(const GsArgs& gs)
{
    __shared__ float s_g;
    if (gs.mode == 0)
        return 1.0f;
    if (gs.mode == 2)
        return __ldg(gs.given);
    if (gs.mode == 3) {
        const float m = fused_global_amax<T>(gs);
        if (threadIdx.x == 0) {
            float g = __fdiv_rn(m, gs.denom);
            if (!(g > 0.0f))
                g = 1.0f;
            s_g = g;
            if (blockIdx.x == 0 && gs.out)
                *gs.out = g;
        }
        __syncthreads();
        return s_g;
    }
    if (threadIdx.x < 32) {
        float m = 0.0f;
        for (int i = threadIdx.x; i < gs.n_partials; i += 32)
            m = fmaxf(m, __ldcg(gs.partials + i));
        m = warp_max(m);
        if (threadIdx.x == 0) {
            float g = __fdiv_rn(m, gs.denom);
            if (!(g > 0.0f))
                g = 1.0f;
            s_g = g;
            if (blockIdx.x == 0 && gs.out)
                *gs.out = g;
        }
    }
    __syncthreads();
    return s_g;
}

// ------------------------------------------------------------------ amax
template <typename T>
__global__ void __launch_bounds__(kThreads) amax_kernel(const T* __restrict__ x, int64_t n,
                                                        float* __restrict__ partials)
{
    constexpr int V = 16 / sizeof(T);            // elements per 16-byte vector
    const int64_t nvec = n / V;
    float m = 0.0f;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    const int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    // four independent 16-byte loads in flight per thread
    int64_t i = i0;
    for (; i + 3 * stride < nvec; i += 4 * stride) {
        uint4 w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u)
            w[u] = __ldg(reinterpret_cast<const uint4*>(x) + i + u * stride);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if constexpr (sizeof(T) == 4) {
                m = fmaxf(m, fmaxf(fmaxf(fabsf(__uint_as_float(w[u].x)), fabsf(__uint_as_float(w[u].y))),
                                   fmaxf(fabsf(__uint_as_float(w[u].z)), fabsf(__uint_as_float(w[u].w)))));
            } else {
                const uint32_t ww[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float lo, hi;
                    bf16x2_to_f32(ww[q], lo, hi);
                    m = fmaxf(m, fmaxf(fabsf(lo), fabsf(hi)));
                }
            }
        }
    }
    for (; i < nvec; i += stride) {
        uint4 v = __ldg(reinterpret_cast<const uint4*>(x) + i);
        if constexpr (sizeof(T) == 4) {
            m = fmaxf(m, fmaxf(fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))),
                               fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w)))));
        } else {
            uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float lo, hi;
                bf16x2_to_f32(w[k], lo, hi);
                m = fmaxf(m, fmaxf(fabsf(lo), fabsf(hi)));
            }
        }
    }
    // ragged tail (n not a multiple of the vector width)
    for (int64_t i = nvec * V + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        float f;
        if constexpr (sizeof(T) == 4)
            f = reinterpret_cast<const float*>(x)[i];
        else
            f = __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(x)[i] << 16);
        m = fmaxf(m, fabsf(f));
    }
    __shared__ float red[kThreads / 32];
    m = warp_max(m);
    if ((threadIdx.x & 31) == 0)
        red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
        m = threadIdx.x < kThreads / 32 ? red[threadIdx.x] : 0.0f;
        m = warp_max(m);
        if (threadIdx.x == 0)
            partials[blockIdx.x] = m;
    }
}

// ------------------------------------------------------- block evaluation
// Quantize one block with decoded scale sc and global scale g: packed codes
// (cw), dequantized values (dq) and the in-order fma squared error.
// The candidate as t = (S, inv): S = sc * g and inv = min(1/S, FLT_MAX) (0 for
// S = 0), both rounded to nearest, as quant_eval computes them.
__device__ __forceinline__ float2 scale_pair(float sc, float g)
{
    const float S = __fmul_rn(sc, g);
    return make_float2(S, (S == 0.0f) ? 0.0f : fminf(__frcp_rn(S), kFltMax));
}

template <int B>
__device__ __forceinline__ float quant_eval_t(const float (&x)[B], float2 t, uint32_t (&cw)[(B + 7) / 8],
                                              float (&dq)[B])
{
    const float S = t.x;
    const float inv = t.y;
    float acc = 0.0f;
    if constexpr (B == 4) {
        uint32_t w = e2m1x4_encode(__fmul_rn(x[0], inv), __fmul_rn(x[1], inv),
                                   __fmul_rn(x[2], inv), __fmul_rn(x[3], inv));
        float v[4];
        e2m1x4_decode(w, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float d = __fmul_rn(v[i], S);
            float e = __fsub_rn(x[i], d);
            acc = __fmaf_rn(e, e, acc);
            dq[i] = d;
        }
        cw[0] = w;
    } else {
#pragma unroll
        for (int j = 0; j < B / 8; ++j) {
            const int o = 8 * j;
            uint32_t w = e2m1x8_encode(__fmul_rn(x[o], inv), __fmul_rn(x[o + 1], inv),
                                       __fmul_rn(x[o + 2], inv), __fmul_rn(x[o + 3], inv),
                                       __fmul_rn(x[o + 4], inv), __fmul_rn(x[o + 5], inv),
                                       __fmul_rn(x[o + 6], inv), __fmul_rn(x[o + 7], inv));
            float v[8];
            e2m1x8_decode(w, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float d = __fmul_rn(v[i], S);
                float e = __fsub_rn(x[o + i], d);
                acc = __fmaf_rn(e, e, acc);
                dq[o + i] = d;
            }
            cw[j] = w;
        }
    }
    return acc;
}

template <int B>
__device__ __forceinline__ float quant_eval(const float (&x)[B], float sc, float g,
                                            uint32_t (&cw)[(B + 7) / 8], float (&dq)[B])
{
    return quant_eval_t<B>(x, scale_pair(sc, g), cw, dq);
}

// Squared error only (brute-force search); t = (S, inv) of the candidate,
// precomputed exactly as quant_eval computes them.
template <int B>
__device__ __forceinline__ float quant_sse(const float (&x)[B], float, float, float2 t)
{
    const float S = t.x;
    const float inv = t.y;
    float acc = 0.0f;
    if constexpr (B == 4) {
        uint32_t w = e2m1x4_encode(__fmul_rn(x[0], inv), __fmul_rn(x[1], inv),
                                   __fmul_rn(x[2], inv), __fmul_rn(x[3], inv));
        float v[4];
        e2m1x4_decode(w, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float e = __fsub_rn(x[i], __fmul_rn(v[i], S));
            acc = __fmaf_rn(e, e, acc);
        }
    } else {
#pragma unroll
        for (int j = 0; j < B / 8; ++j) {
            const int o = 8 * j;
            uint32_t w = e2m1x8_encode(__fmul_rn(x[o], inv), __fmul_rn(x[o + 1], inv),
                                       __fmul_rn(x[o + 2], inv), __fmul_rn(x[o + 3], inv),
                                       __fmul_rn(x[o + 4], inv), __fmul_rn(x[o + 5], inv),
                                       __fmul_rn(x[o + 6], inv), __fmul_rn(x[o + 7], inv));
            float v[8];
            e2m1x8_decode(w, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float e = __fsub_rn(x[o + i], __fmul_rn(v[i], S));
                acc = __fmaf_rn(e, e, acc);
            }
        }
    }
    return acc;
}

// Codes and in-order squared error of a block at the candidate t = (S, inv).
template <int B>
__device__ __forceinline__ float quant_codes_sse(const float (&x)[B], float2 t, uint32_t (&cw)[(B + 7) / 8])
{
    const float S = t.x;
    const float inv = t.y;
    float acc = 0.0f;
    if constexpr (B == 4) {
        const uint32_t w = e2m1x4_encode(__fmul_rn(x[0], inv), __fmul_rn(x[1], inv),
                                         __fmul_rn(x[2], inv), __fmul_rn(x[3], inv));
        float v[4];
        e2m1x4_decode(w, v);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float e = __fsub_rn(x[i], __fmul_rn(v[i], S));
            acc = __fmaf_rn(e, e, acc);
        }
        cw[0] = w;
    } else {
#pragma unroll
        for (int j = 0; j < B / 8; ++j) {
            const int o = 8 * j;
            const uint32_t w = e2m1x8_encode(__fmul_rn(x[o], inv), __fmul_rn(x[o + 1], inv),
                                             __fmul_rn(x[o + 2], inv), __fmul_rn(x[o + 3], inv),
                                             __fmul_rn(x[o + 4], inv), __fmul_rn(x[o + 5], inv),
                                             __fmul_rn(x[o + 6], inv), __fmul_rn(x[o + 7], inv));
            float v[8];
            e2m1x8_decode(w, v);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float e = __fsub_rn(x[o + i], __fmul_rn(v[i], S));
                acc = __fmaf_rn(e, e, acc);
            }
            cw[j] = w;
        }
    }
    return acc;
}

// Error of one element of magnitude a under scale S / reciprocal inv.
__device__ __forceinline__ float elem_err(float a, float S, float inv)
{
    uint32_t w = e2m1x4_encode(__fmul_rn(a, inv), 0.0f, 0.0f, 0.0f);
    float v[4];
    e2m1x4_decode(w, v);
    return __fsub_rn(a, __fmul_rn(v[0], S));
}

enum { R_ABSMAX = 0, R_PZ = 1, R_46 = 2, R_BF = 3 };

// Abs-max, prevent-zero and 4-over-6 (brute force has its own kernel below).
// SFMT: the block-scale format, 0 = E4M3 (NVFP4), 1 = UE5M3.
template <int B, typename T, int RULE, int SFMT, bool DEQ>
__global__ void __launch_bounds__(kThreads)
nvfp4_quant_kernel(const T* __restrict__ x, int64_t nblk, int64_t bpr, GsArgs gs,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int mma_layout,
                   float* __restrict__ deq, float* __restrict__ mse)
{
    const float g = resolve_global_scale<T>(gs);
    const float g6 = __fmul_rn(6.0f, g);
    const float g4 = __fmul_rn(4.0f, g);
    // (S, inv) of every scale code, computed once per CTA (the encoders return
    // at most 0xFE for UE5M3 and, for an all-NaN block, 0x7F for E4M3)
    constexpr int kCodes = SFMT == 1 ? 256 : 128;
    __shared__ float2 qtab[kCodes];
    for (int c = threadIdx.x; c < kCodes; c += blockDim.x)
        qtab[c] = scale_pair(sf_decode<SFMT>((uint32_t)c), g);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t kb_atoms = (bpr + 3) >> 2;
    // blocks of 128 bytes or more are loaded warp-cooperatively through shared
    // memory; dequantized blocks of 32 bytes or more are stored that way too
    // (the same buffer, sized for the larger of the two)
    constexpr bool kStaged = B * sizeof(T) >= 128;
    constexpr bool kStoreStaged = B >= 8;
    constexpr int kBufChunks = (kStaged ? 2 * B * (int)sizeof(T) : 1) > (kStoreStaged ? 8 * B : 1)
                                   ? (kStaged ? 2 * B * (int)sizeof(T) : 1)
                                   : (kStoreStaged ? 8 * B : 1);
    __shared__ uint4 stage_buf[kThreads / 32][kBufChunks];
    // small blocks (up to four 16-byte loads per lane): keep the next block's
    // load in flight while this one is quantized
    constexpr bool kPrefetch = !kStaged && B * sizeof(T) <= 64;
    float xn[B];
    if constexpr (kPrefetch) {
        const int64_t b0 = warp0 * 32 + lane;
        if (b0 < nblk) {
            load_elems<T, B>(x + b0 * B, xn);
        } else {
#pragma unroll
            for (int i = 0; i < B; ++i)
                xn[i] = 0.0f;
        }
    }
    // MMA-layout scale position: (row, k-block) of this lane's block, advanced
    // by the grid stride without a per-block 64-bit division
    int64_t r_cur = 0, kb_cur = 0, step_r = 0, step_kb = 0;
    if (mma_layout) {
        const int64_t b0 = warp0 * 32 + lane;
        const int64_t step = nwarps * 32;
        r_cur = b0 / bpr;
        kb_cur = b0 % bpr;
        step_r = step / bpr;
        step_kb = step % bpr;
    }

    for (int64_t base = warp0 * 32; base < nblk; base += nwarps * 32) {
        const int64_t b = base + lane;
        const bool valid = b < nblk;
        float xv[B];
        if constexpr (kStaged) {
            warp_load_blocks<T, B>(x, base, nblk, stage_buf[threadIdx.x >> 5], xv);
        } else if constexpr (kPrefetch) {
            // this iteration's block was loaded last iteration; start the next one
#pragma unroll
            for (int i = 0; i < B; ++i)
                xv[i] = xn[i];
            const int64_t bn = b + nwarps * 32;
            if (bn < nblk) {
                load_elems<T, B>(x + bn * B, xn);
            }
        } else if (valid) {
            load_elems<T, B>(x + b * B, xv);
        } else {
#pragma unroll
            for (int i = 0; i < B; ++i)
                xv[i] = 0.0f;
        }
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < B; ++i)
            a = fmaxf(a, fabsf(xv[i]));

        uint32_t cw[(B + 7) / 8];
        float dq[B];
        float sse;
        uint32_t sc;
        if constexpr (RULE == R_ABSMAX || RULE == R_PZ) {
            sc = sf_encode<SFMT>(__fdiv_rn(a, g6));
            if (RULE == R_PZ && sc == 0u)
                sc = 1u;
            sse = quant_eval_t<B>(xv, qtab[sc], cw, dq);
        } else if constexpr (RULE == R_46) {
            const uint32_t c6 = sf_encode<SFMT>(__fdiv_rn(a, g6));
            const uint32_t c4 = sf_encode<SFMT>(__fdiv_rn(a, g4));
            // codes and errors of both candidates; the dequantized values only
            // for the chosen one, and only when they are wanted
            sse = quant_codes_sse<B>(xv, qtab[c6], cw);
            sc = c6;
            // equal codes give equal errors, and a tie keeps the 6-mapping
            if (c4 != c6) {
                uint32_t cw4[(B + 7) / 8];
                const float s4 = quant_codes_sse<B>(xv, qtab[c4], cw4);
                if (s4 < sse) {
                    sc = c4;
                    sse = s4;
#pragma unroll
                    for (int j = 0; j < (B + 7) / 8; ++j)
                        cw[j] = cw4[j];
                }
            }
            if constexpr (DEQ) {
                uint32_t cwd[(B + 7) / 8];
                quant_eval_t<B>(xv, qtab[sc], cwd, dq);
            }
        }

        if (valid) {
            store_codes<B>(codes + b * (B / 2), cw);
            const int64_t so = mma_layout ? mma_sf_offset(r_cur, kb_cur, kb_atoms) : b;
            scales[so] = (uint8_t)sc;
            if (!kStoreStaged && DEQ)
                store_f32<B>(deq + b * B, dq);
            if (mse)
                mse[b] = __fmul_rn(sse, 1.0f / (float)B);
        }
        if constexpr (kStoreStaged) {
            if constexpr (DEQ)
                warp_store_f32_blocks<B>(deq, base, nblk, stage_buf[threadIdx.x >> 5], dq);
        }
        if (mma_layout) {
            kb_cur += step_kb;
            r_cur += step_r;
            if (kb_cur >= bpr) {
                kb_cur -= bpr;
                ++r_cur;
            }
        }
    }
}

// ------------------------------------------------------------------ RaZeR
struct SpecialArgs {
    float v[4];        // table in order
    int n;
    float mag[4];      // distinct magnitudes |v|
    int nmag;
    int mag_of[4];     // magnitude index of each table entry
    int neg[4];        // 1 if the table entry is negative
};

// SF = 0: E4M3 scale, selector in bit 7 (activations); SF = 1: E3M3 scale,
// selector in bits 7..6 (weights).  Block size 16.
//
// Per block: the plain E2M1 error e_i of every element is computed once.  For
// each distinct special magnitude a 16-bit mask marks the elements that are
// not zero-coded and for which that magnitude is strictly nearer than their
// grid neighbour; a signed table entry takes the elements of its magnitude
// mask whose sign matches.  Its in-order fma error chain then uses
// RN(|x| - RN(|v| S)) at the masked positions (the square equals that of
// x - RN(v S) for a same-signed v) and e_i elsewhere.
template <typename T, int SF>
__global__ void __launch_bounds__(kThreads, 3)
razer_quant_kernel(const T* __restrict__ x, int64_t nblk, GsArgs gs, SpecialArgs sp,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ meta,
                   float* __restrict__ deq, float* __restrict__ mse)
{
    constexpr int B = 16;
    const float g = resolve_global_scale<T>(gs);
    const float g6 = __fmul_rn(6.0f, g);
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;

    for (int64_t base = warp0 * 32; base < nblk; base += nwarps * 32) {
        const int64_t b = base + lane;
        const bool valid = b < nblk;
        float xv[B];
        if (valid) {
            load_elems<T, B>(x + b * B, xv);
        } else {
#pragma unroll
            for (int i = 0; i < B; ++i)
                xv[i] = 0.0f;
        }
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < B; ++i)
            a = fmaxf(a, fabsf(xv[i]));
        const float r = __fdiv_rn(a, g6);
        const uint32_t scc = SF == 1 ? e3m3_encode(r) : e4m3_encode(r);
        const float scv = SF == 1 ? e3m3_decode(scc) : e4m3_decode(scc);
        const float S = __fmul_rn(scv, g);
        const float inv = (S == 0.0f) ? 0.0f : fminf(__frcp_rn(S), kFltMax);

        // plain E2M1 quantization, its errors and the per-magnitude masks
        float e[B];
        uint32_t cw[2];
        uint32_t negm = 0u, zerom = 0u;
        uint32_t magm[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float y[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                y[i] = __fmul_rn(xv[8 * j + i], inv);
            cw[j] = e2m1x8_encode(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
            float v[8];
            e2m1x8_decode(cw[j], v);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int idx = 8 * j + i;
                e[idx] = __fsub_rn(xv[idx], __fmul_rn(v[i], S));
                const float ay = fabsf(y[i]);
                const float dg = fabsf(__fsub_rn(ay, fabsf(v[i])));
                const bool nz = v[i] != 0.0f;
                negm |= (uint32_t)signbit(y[i]) << idx;
                zerom |= (uint32_t)(!nz) << idx;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    if (k < sp.nmag) {
                        const bool near = nz && (fabsf(__fsub_rn(ay, sp.mag[k])) < dg);
                        magm[k] |= (uint32_t)near << idx;
                    }
                }
            }
        }
        // score each table entry in order; strict < keeps the earliest minimum
        float best = 0.0f;
        int sel = 0;
        uint32_t best_mask = 0u;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (k >= sp.n)
                break;
            const int mi = sp.mag_of[k];
            const uint32_t mm = mi == 0 ? magm[0] : mi == 1 ? magm[1] : mi == 2 ? magm[2] : magm[3];
            const uint32_t use = mm & (sp.neg[k] ? negm : ~negm);
            const float D = __fmul_rn(sp.mag[mi == 0 ? 0 : mi == 1 ? 1 : mi == 2 ? 2 : 3], S);
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < B; ++i) {
                const float es = __fsub_rn(fabsf(xv[i]), D);
                const float ei = ((use >> i) & 1u) ? es : e[i];
                acc = __fmaf_rn(ei, ei, acc);
            }
            if (k == 0 || acc < best) {
                best = acc;
                sel = k;
                best_mask = use;
            }
        }
        if (valid) {
            // codes: zero-coded elements take +0, the chosen elements the -0 code
            uint32_t ow[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                uint32_t w = cw[j];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const int idx = 8 * j + i;
                    const uint32_t clr = ((zerom >> idx) & 1u) | ((best_mask >> idx) & 1u);
                    w &= ~(clr * (0xFu << (4 * i)));
                    w |= ((best_mask >> idx) & 1u) << (4 * i + 3);
                }
                ow[j] = w;
            }
            *reinterpret_cast<uint2*>(codes + b * 8) = make_uint2(ow[0], ow[1]);
            meta[b] = (uint8_t)(SF == 1 ? ((uint32_t)sel << 6) | scc : ((uint32_t)sel << 7) | scc);
            if (deq) {
                // dequantized values from the final codes: the chosen special at
                // its positions, v * S (+0 for zero codes) elsewhere
                const float spv = sel == 0 ? sp.v[0] : sel == 1 ? sp.v[1] : sel == 2 ? sp.v[2] : sp.v[3];
                const float dsp = __fmul_rn(spv, S);
                float dq[B];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float vv[8];
                    e2m1x8_decode(ow[j], vv);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int idx = 8 * j + i;
                        dq[idx] = ((best_mask >> idx) & 1u) ? dsp : __fmul_rn(vv[i], S);
                    }
                }
                store_f32<B>(deq + b * B, dq);
            }
            if (mse)
                mse[b] = __fmul_rn(best, 1.0f / 16.0f);
        }
    }
}

// Paired tables (+v0, -v0, +v1, -v1, ...), NPAIR pairs, v > 0.  An element
// can only take the table entry whose sign matches its own (its grid value v
// is then nonzero with that sign), so with d = |y - v|:
//   +m candidate: special iff v > 0 and |y - m| < d
//   -m candidate: special iff v < 0 and |y + m| < d
// A nonzero v has the sign of y, so both distances are ||y| - m| (RN(-a) =
// -RN(a)): one subtraction per magnitude serves the pair.
// Each candidate's in-order fma chain takes either the grid error e or the
// special error es; the choice is a predicated fma pair on the FMA pipe
// rather than a select on the integer pipe, and the element's bit enters
// that candidate's mask under the same predicate.
// One pair's two candidates; operands: %0/%1 the +/- chains, %2/%3 their
// masks, e the grid error, m, es, the element's bit; ay = |y|, d, pp, pn shared.
#define FP4Q_RAZER_PAIR_PTX(A0, A1, M0, M1, E, MAG, ES, BIT)           \
    "sub.rn.f32 t, ay, " MAG ";\n\t"                                 \
    "abs.f32 t, t;\n\t"                                              \
    "setp.lt.and.f32 q, t, d, pp;\n\t"                               \
    "setp.lt.and.f32 r, t, d, pn;\n\t"                               \
    "@!q fma.rn.f32 " A0 ", " E ", " E ", " A0 ";\n\t"                 \
    "@q fma.rn.f32 " A0 ", " ES ", " ES ", " A0 ";\n\t"                \
    "@q or.b32 " M0 ", " M0 ", " BIT ";\n\t"                           \
    "@!r fma.rn.f32 " A1 ", " E ", " E ", " A1 ";\n\t"                 \
    "@r fma.rn.f32 " A1 ", " ES ", " ES ", " A1 ";\n\t"                \
    "@r or.b32 " M1 ", " M1 ", " BIT ";\n\t"

template <int NPAIR>
__device__ __forceinline__ void razer_pair_step(float y, float v, float e, const float (&mag)[NPAIR],
                                                const float (&es)[NPAIR], uint32_t bit,
                                                float (&acc)[2 * NPAIR], uint32_t (&mask)[2 * NPAIR])
{
    static_assert(NPAIR == 1 || NPAIR == 2, "one or two pairs");
    if constexpr (NPAIR == 1) {
        asm("{\n\t"
            ".reg .pred pp, pn, q, r;\n\t"
            ".reg .f32 d, t, ay;\n\t"
            "setp.gt.f32 pp, %5, 0f00000000;\n\t"
            "setp.lt.f32 pn, %5, 0f00000000;\n\t"
            "sub.rn.f32 d, %4, %5;\n\t"
            "abs.f32 d, d;\n\t"
            "abs.f32 ay, %4;\n\t"
            FP4Q_RAZER_PAIR_PTX("%0", "%1", "%2", "%3", "%6", "%7", "%8", "%9")
            "}"
            : "+f"(acc[0]), "+f"(acc[1]), "+r"(mask[0]), "+r"(mask[1])
            : "f"(y), "f"(v), "f"(e), "f"(mag[0]), "f"(es[0]), "r"(bit));
    } else {
        asm("{\n\t"
            ".reg .pred pp, pn, q, r;\n\t"
            ".reg .f32 d, t, ay;\n\t"
            "setp.gt.f32 pp, %9, 0f00000000;\n\t"
            "setp.lt.f32 pn, %9, 0f00000000;\n\t"
            "sub.rn.f32 d, %8, %9;\n\t"
            "abs.f32 d, d;\n\t"
            "abs.f32 ay, %8;\n\t"
            FP4Q_RAZER_PAIR_PTX("%0", "%1", "%4", "%5", "%10", "%11", "%13", "%15")
            FP4Q_RAZER_PAIR_PTX("%2", "%3", "%6", "%7", "%10", "%12", "%14", "%15")
            "}"
            : "+f"(acc[0]), "+f"(acc[1]), "+f"(acc[2]), "+f"(acc[3]), "+r"(mask[0]), "+r"(mask[1]),
              "+r"(mask[2]), "+r"(mask[3])
            : "f"(y), "f"(v), "f"(e), "f"(mag[0]), "f"(mag[1]), "f"(es[0]), "f"(es[1]), "r"(bit));
    }
}
#undef FP4Q_RAZER_PAIR_PTX

// Spread the 8 bits of b to bit 0 of the 8 nibbles of a word.
__device__ __forceinline__ uint32_t spread_bits_to_nibbles(uint32_t b)
{
    b = (b | (b << 12)) & 0x000F000Fu;
    b = (b | (b << 6)) & 0x03030303u;
    b = (b | (b << 3)) & 0x11111111u;
    return b;
}

// A block's elements as raw 16-byte words (read-only path) and their fp32
// values: bf16 is the high half of an fp32 (element 2i in the low half-word).
template <typename T, int B>
__device__ __forceinline__ void load_raw(const T* __restrict__ p, uint4 (&w)[B * sizeof(T) / 16])
{
#pragma unroll
    for (int k = 0; k < (int)(B * sizeof(T) / 16); ++k)
        w[k] = __ldg(reinterpret_cast<const uint4*>(p) + k);
}

template <typename T, int B>
__device__ __forceinline__ void raw_to_f32(const uint4 (&w)[B * sizeof(T) / 16], float (&x)[B])
{
#pragma unroll
    for (int k = 0; k < (int)(B * sizeof(T) / 16); ++k) {
        const uint32_t v[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if constexpr (sizeof(T) == 4) {
                x[4 * k + q] = __uint_as_float(v[q]);
            } else {
                x[8 * k + 2 * q] = __uint_as_float(v[q] << 16);
                x[8 * k + 2 * q + 1] = __uint_as_float(v[q] & 0xFFFF0000u);
            }
        }
    }
}

template <typename T, int SF, int NPAIR>
__global__ void __launch_bounds__(kThreads, 3)
razer_paired_kernel(const T* __restrict__ x, int64_t nblk, GsArgs gs, SpecialArgs sp,
                    uint8_t* __restrict__ codes, uint8_t* __restrict__ meta,
                    float* __restrict__ deq, float* __restrict__ mse)
{
    constexpr int B = 16;
    static_assert(NPAIR >= 1 && NPAIR <= 2, "the scale table holds two special magnitudes");
    const float g = resolve_global_scale<T>(gs);
    const float g6 = __fmul_rn(6.0f, g);
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    float mag[NPAIR];
#pragma unroll
    for (int m = 0; m < NPAIR; ++m)
        mag[m] = sp.v[2 * m];
    // per scale code, computed once per CTA: S = sc * g, inv = min(1/S, FLT_MAX)
    // (0 for S = 0) and each special magnitude times S (E3M3 encodes to 0..63,
    // E4M3 to 0..127)
    constexpr int kCodes = SF == 1 ? 64 : 128;
    __shared__ float4 rtab[kCodes];
    for (int c = threadIdx.x; c < kCodes; c += blockDim.x) {
        const float S = __fmul_rn(SF == 1 ? e3m3_decode((uint32_t)c) : e4m3_decode((uint32_t)c), g);
        const float inv = (S == 0.0f) ? 0.0f : fminf(__frcp_rn(S), kFltMax);
        rtab[c] = make_float4(S, inv, __fmul_rn(mag[0], S), NPAIR > 1 ? __fmul_rn(mag[NPAIR - 1], S) : 0.0f);
    }
    __syncthreads();

    // the next block's raw words are in flight while this one is quantized
    constexpr int kWords = B * (int)sizeof(T) / 16;
    uint4 wn[kWords];
#pragma unroll
    for (int k = 0; k < kWords; ++k)
        wn[k] = make_uint4(0u, 0u, 0u, 0u);
    if (warp0 * 32 + lane < nblk)
        load_raw<T, B>(x + (warp0 * 32 + lane) * B, wn);

    for (int64_t base = warp0 * 32; base < nblk; base += nwarps * 32) {
        const int64_t b = base + lane;
        const bool valid = b < nblk;
        float xv[B];
        raw_to_f32<T, B>(wn, xv);
        {
            const int64_t bn = b + nwarps * 32;
#pragma unroll
            for (int k = 0; k < kWords; ++k)
                wn[k] = make_uint4(0u, 0u, 0u, 0u);
            if (bn < nblk)
                load_raw<T, B>(x + bn * B, wn);
        }
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < B; ++i)
            a = fmaxf(a, fabsf(xv[i]));
        const float r = __fdiv_rn(a, g6);
        const uint32_t scc = SF == 1 ? e3m3_encode(r) : e4m3_encode(r);
        const float4 st = rtab[scc];
        const float S = st.x;
        const float inv = st.y;
        float D[NPAIR];
        D[0] = st.z;
        if constexpr (NPAIR > 1)
            D[NPAIR - 1] = st.w;

        float acc[2 * NPAIR];
        uint32_t mask[2 * NPAIR];
#pragma unroll
        for (int k = 0; k < 2 * NPAIR; ++k) {
            acc[k] = 0.0f;
            mask[k] = 0u;
        }
        uint32_t cw[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float y[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
                y[i] = __fmul_rn(xv[8 * j + i], inv);
            cw[j] = e2m1x8_encode(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
            float v[8];
            e2m1x8_decode(cw[j], v);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int idx = 8 * j + i;
                const float e = __fsub_rn(xv[idx], __fmul_rn(v[i], S));
                const float ax = fabsf(xv[idx]);
                float es[NPAIR];
#pragma unroll
                for (int m = 0; m < NPAIR; ++m)
                    es[m] = __fsub_rn(ax, D[m]);
                razer_pair_step<NPAIR>(y[i], v[i], e, mag, es, 1u << idx, acc, mask);
            }
        }
        float best = acc[0];
        int sel = 0;
#pragma unroll
        for (int k = 1; k < 2 * NPAIR; ++k) {
            if (acc[k] < best) {
                best = acc[k];
                sel = k;
            }
        }
        if (valid) {
            uint32_t chosen = mask[0];
#pragma unroll
            for (int k = 1; k < 2 * NPAIR; ++k)
                if (sel == k)
                    chosen = mask[k];
            uint32_t ow[2];
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                uint32_t w = cw[j];
                // -0 (0x8) is the special code: grid zeros take +0
                const uint32_t t = w ^ 0x88888888u;
                const uint32_t not8 = (((t & 0x77777777u) + 0x77777777u) | t) & 0x88888888u;
                w &= ~(~not8 & 0x88888888u);
                // chosen elements take -0
                const uint32_t ones = spread_bits_to_nibbles((chosen >> (8 * j)) & 0xFFu);
                w = (w & ~(ones * 0xFu)) | (ones << 3);
                ow[j] = w;
            }
            *reinterpret_cast<uint2*>(codes + b * 8) = make_uint2(ow[0], ow[1]);
            meta[b] = (uint8_t)(SF == 1 ? ((uint32_t)sel << 6) | scc : ((uint32_t)sel << 7) | scc);
            if (deq) {
                float spv = 0.0f;
#pragma unroll
                for (int k = 0; k < 2 * NPAIR; ++k)
                    if (sel == k)
                        spv = (k & 1) ? -mag[k >> 1] : mag[k >> 1];
                const float dsp = __fmul_rn(spv, S);
                float dq[B];
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    float vv[8];
                    e2m1x8_decode(ow[j], vv);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const int idx = 8 * j + i;
                        dq[idx] = ((chosen >> idx) & 1u) ? dsp : __fmul_rn(vv[i], S);
                    }
                }
                store_f32<B>(deq + b * B, dq);
            }
            if (mse)
                mse[b] = __fmul_rn(best, 1.0f / 16.0f);
        }
    }
}

// ------------------------------------------------------- brute-force scale
// Brute force over the scale format's codes (E4M3 1..126, UE5M3 1..254): the
// least in-order squared error, ties to the lowest code.  Exact shortcuts
// (each provably skips only codes that cannot win):
//  * from the first code at which the largest element rounds to zero
//    (|y| <= 0.25; |y| falls as the code grows) every element does, so that
//    code gives the all-zero error (the in-order sum of x^2) and every higher
//    code ties it with a higher code;
//  * below the abs-max code c6 the largest element clips to 6, its error
//    a - 6S grows as the code falls, and its square alone bounds the in-order
//    fma chain from below (the chain only adds non-negative terms and
//    rounding is monotone): the downward scan from c6 stops at the first
//    code whose bound already loses against c6 or the all-zero code;
//  * codes above c6 that no element can prefer: when g and the scale S_r of
//    c6 are powers of two (so x / S_r is exact and c6's encode picks, for every
//    element, the nearest point of its grid S_r G, G = {0, .5, 1, 1.5, 2, 3,
//    4, 6}) and no element clips at c6 (a <= 6 S_r), a code c with grid S_c G
//    can bring an element nearer only through a point p of S_c G in
//    (0, 6 S_r) that S_r G lacks, and only for elements strictly inside the
//    window between the midpoints of p and its two neighbours in S_r G (past
//    6 S_r every point is farther than 6 S_r itself).  If no element of the
//    block lies in any window of c, every |x_i - q_c(x_i)| >= |x_i -
//    q_r(x_i)|; the rounded errors and their in-order fma chain keep that
//    order, and a tie goes to the lower code c6, so c cannot win.  With
//    k = S_c / S_r the windows depend on k alone, and k depends only on the
//    offset of c from c6 and on whether c6 is a normal power of two or the
//    subnormal code 1, 2 or 4 (the same in E4M3 and UE5M3, both with three
//    mantissa bits).  BfWindows holds, per reference type and per 1/8-wide
//    bin of |x| / S_r in [0, 6], the mask of code offsets whose windows meet
//    the bin; a block ORs the masks of its elements' bins.  Codes with
//    k in {2, 4, 6, 8, 12} or k >= 13 add no point below 6 S_r and never
//    appear in a mask.
// Every other code of [clo, all-zero code) is evaluated in full.  A block
// with none left (most blocks) is stored at once; the seed c6 is evaluated
// with its codes kept, so a block that keeps c6 needs no second encode.  The
// others wait in a per-warp queue; once 32 are queued the warp takes them
// together: each lane reloads one, the (block, code) pairs still to evaluate
// are laid end to end and every lane takes every 32nd pair, reading the block
// from shared memory.  A block's best (error, code) is one 64-bit key --
// error bits (non-negative floats order like their bits) above the code --
// lowered with a shared-memory atomic minimum, so the lowest code wins ties
// exactly as in a sequential scan.
constexpr int kWarps = kThreads / 32;

// True when a fp32 value is a normal power of two in [2^-100, 2^100].
__device__ __forceinline__ bool pow2_in_range(float v)
{
    const uint32_t u = __float_as_uint(v);
    const uint32_t e = u >> 23;                  // sign bit included: negatives fail
    return (u & 0x007FFFFFu) == 0u && e >= 127u - 100u && e <= 127u + 100u;
}

// Per reference type (0 a normal power of two, 1-3 the subnormal codes 1, 2,
// 4) and per bin b of |x| / S_r (width 1/8, b = 0..48): bit j set when code
// c6 + 1 + j has a window meeting the bin.
struct BfWindows {
    unsigned long long m[4][49];
};

// Reference type of a scale code (3 mantissa bits): 1 + type, 0 when its
// scale is not a power of two.
__device__ __forceinline__ uint32_t ref_type(uint32_t c)
{
    if (c >= 8u)
        return (c & 7u) == 0u ? 1u : 0u;
    if (c == 0u || (c & (c - 1u)) != 0u)
        return 0u;
    return 33u - (uint32_t)__clz((int)c);   // subnormal 1, 2, 4 -> 2, 3, 4
}

// A block's search after the exact shortcuts: the better of c6 and the
// all-zero code so far, and the codes still to evaluate (clo .. c6 - 1, then
// the bits of um: code c6 + 1 + j; `over`: codes past c6 + 64 as well).
struct BfPlan {
    float best;
    uint32_t bc, c6, clo;
    int chi;
    unsigned long long um;
    bool over;
};

template <int B, int SFMT>
__device__ __forceinline__ BfPlan bf_plan(const float (&xv)[B], bool valid, const float2* tab,
                                          const unsigned long long* wmask, float g6, float four_over_g,
                                          bool g_pow2, uint32_t (&cw)[(B + 7) / 8], uint32_t& n_eval)
{
    constexpr uint32_t kLast = SFMT == 1 ? 254u : 126u;
    constexpr uint32_t kNone = kLast + 1u;
    BfPlan pl;
    float a = 0.0f;
    float sse0 = 0.0f;
#pragma unroll
    for (int i = 0; i < B; ++i) {
        a = fmaxf(a, fabsf(xv[i]));
        sse0 = __fmaf_rn(xv[i], xv[i], sse0);
    }
    uint32_t c6 = sf_encode<SFMT>(__fdiv_rn(a, g6));
    c6 = c6 == 0u ? 1u : c6;
    const float2 t6 = tab[c6];
    float best = quant_codes_sse<B>(xv, t6, cw);
    uint32_t bc = c6;
    n_eval += valid ? 1u : 0u;
    // first all-zero code (kNone = none): step from a nearby code to the
    // boundary (|y| is monotone in the code)
    uint32_t cz = sf_encode<SFMT>(__fmul_rn(a, four_over_g));
    cz = cz == 0u ? 1u : cz;
    {
        // usually the boundary is cz or cz + 1: test both without a loop
        const bool f0 = cz > 1u && __fmul_rn(a, tab[cz - 1u].y) <= 0.25f;
        const bool f1 = __fmul_rn(a, tab[cz].y) <= 0.25f;
        const bool f2 = cz + 1u >= kNone || __fmul_rn(a, tab[cz + 1u].y) <= 0.25f;
        if (f1 && !f0) {
        } else if (!f1 && f2) {
            ++cz;
        } else if (f1) {
            --cz;
            while (cz > 1u && __fmul_rn(a, tab[cz - 1u].y) <= 0.25f)
                --cz;
        } else {
            ++cz;
            do {
                ++cz;
            } while (cz < kNone && __fmul_rn(a, tab[cz].y) > 0.25f);
        }
    }
    n_eval += (valid && cz < kNone) ? 1u : 0u;
    if (cz < kNone && (sse0 < best || (sse0 == best && cz < bc))) {
        best = sse0;
        bc = cz;
    }
    // downward: codes below c6 while the clipped bound can still win
    uint32_t clo = c6;
    while (clo > 1u) {
        const float2 t = tab[clo - 1u];
        const float em = elem_err(a, t.x, t.y);
        if (__fmul_rn(em, em) > best)
            break;
        --clo;
    }
    const int chi = (int)(cz < kNone ? cz : kNone) - 1;   // last code to evaluate
    const int nup = valid ? chi - (int)c6 : 0;
    unsigned long long um = nup <= 0 ? 0ull : nup >= 64 ? ~0ull : ((1ull << nup) - 1ull);
    // c6 is a usable reference: a power-of-two scale with an exact
    // reciprocal at which no element clips; then only the codes whose
    // windows hold an element stay
    const uint32_t ty = ref_type(c6);
    const bool use_ref = g_pow2 && ty != 0u && __fmul_rn(t6.x, t6.y) == 1.0f && __fmul_rn(a, t6.y) <= 6.0f;
    if (use_ref) {
        unsigned long long allow = 0ull;
#pragma unroll
        for (int i = 0; i < B; ++i) {
            // |x| / S_r <= 6 exactly, so the bin is 0 .. 48
            const int bin = __float2int_rz(__fmul_rn(__fmul_rn(fabsf(xv[i]), t6.y), 8.0f));
            allow |= wmask[(ty - 1u) * 49u + (uint32_t)bin];
        }
        um &= allow;
    }
    pl.best = best;
    pl.bc = bc;
    pl.c6 = c6;
    pl.clo = valid ? clo : c6;
    pl.chi = chi;
    pl.um = um;
    // codes past c6 + 64 (all with k >= 13, so never in a window, for a usable
    // reference): in practice no block has any, its range above c6 being at
    // most about 40 codes in either format
    pl.over = valid && !use_ref && chi > (int)c6 + 64;
    return pl;
}

// Capacity of a warp's queue of blocks whose search continues after the
// shortcuts (a flush takes 32 of them; one step adds at most 32).
constexpr int kBfQueue = 64;

// Resident CTAs per SM the brute-force kernel is compiled for (its register cap).
template <int B>
constexpr int bf_min_ctas() { return B <= 4 ? 4 : B <= 16 ? 3 : 2; }

template <int B, typename T, int SFMT, bool DEQ>
__global__ void __launch_bounds__(kThreads, bf_min_ctas<B>())
nvfp4_bf_kernel(const T* __restrict__ x, int64_t nblk, int64_t bpr, GsArgs gs,
                uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int mma_layout,
                float* __restrict__ deq, float* __restrict__ mse, unsigned long long* evals,
                const __grid_constant__ BfWindows win)
{
    uint32_t n_eval = 0;   // this lane's error evaluations (seeds, all-zero codes, searches)
    constexpr uint32_t kLast = SFMT == 1 ? 254u : 126u;
    constexpr uint32_t kNone = kLast + 1u;
    // (S, inv) of every code: S = sc * g, inv = min(1/S, FLT_MAX), 0 for S = 0
    __shared__ float2 tab[kNone + 1];
    // the window masks, in shared memory: lanes index them by their own bins,
    // which constant-space reads would serialize
    __shared__ unsigned long long wmask[4 * 49];
    // each warp's 32 blocks being searched (dynamic: kWarps * 32 * B floats)
    extern __shared__ __align__(16) float blk_xs[];
    __shared__ unsigned long long key[kWarps][32];
    __shared__ int pre[kWarps][32];
    __shared__ uint32_t lowm[kWarps][32];            // next lower code | lower count << 8 | c6 << 16
    __shared__ unsigned long long upm[kWarps][32];   // upper codes left: bit j = code c6 + 1 + j
    // the warp's queue of blocks whose search continues: block index, the
    // best error so far with `over` in its sign bit (errors are non-negative),
    // codes (best | c6 << 8 | clo << 16 | chi << 24), the upper-code mask
    __shared__ unsigned long long q_idx[kWarps][kBfQueue];
    __shared__ unsigned long long q_um[kWarps][kBfQueue];
    __shared__ uint32_t q_best[kWarps][kBfQueue];
    __shared__ uint32_t q_codes[kWarps][kBfQueue];

    const float g = resolve_global_scale<T>(gs);
    const float g6 = __fmul_rn(6.0f, g);
    // only a starting point for the exact all-zero search
    const float four_over_g = __fmul_rn(4.0f, __frcp_rn(g));
    // every S = sc * g and every v * S is exact when g is a moderate power of two
    const bool g_pow2 = pow2_in_range(g);
    for (int c = threadIdx.x; c <= (int)kNone; c += blockDim.x) {
        const float S = __fmul_rn(sf_decode<SFMT>((uint32_t)c < kNone ? (uint32_t)c : kLast), g);
        tab[c] = make_float2(S, (S == 0.0f) ? 0.0f : fminf(__frcp_rn(S), kFltMax));
    }
    for (int i = threadIdx.x; i < 4 * 49; i += blockDim.x)
        wmask[i] = win.m[i / 49][i % 49];
    __syncthreads();

    const int lane = threadIdx.x & 31;
    const int w = threadIdx.x >> 5;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t kb_atoms = (bpr + 3) >> 2;
    int64_t r_cur = 0, kb_cur = 0, step_r = 0, step_kb = 0;
    if (mma_layout) {
        const int64_t b0 = warp0 * 32 + lane;
        const int64_t step = nwarps * 32;
        r_cur = b0 / bpr;
        kb_cur = b0 % bpr;
        step_r = step / bpr;
        step_kb = step % bpr;
    }
    float* xw = blk_xs + w * 32 * B;

    // Store block b's result at code bc (its codes at c6 are cw and its error
    // `best` when bc == c6 and no dequantized output is wanted).
    auto store_block = [&](int64_t b, const float (&xv)[B], uint32_t bc, uint32_t c6, uint32_t (&cw)[(B + 7) / 8],
                           float best, int64_t so) {
        float sse = best;
        float dq[B];
        if (bc != c6 || DEQ)
            sse = quant_eval_t<B>(xv, tab[bc], cw, dq);
        store_codes<B>(codes + b * (B / 2), cw);
        scales[so] = (uint8_t)bc;
        if constexpr (DEQ)
            store_f32<B>(deq + b * B, dq);
        if (mse)
            mse[b] = __fmul_rn(sse, 1.0f / (float)B);
    };

    // Finish the first n queued blocks: every lane takes one (reloading its
    // elements), the warp lays the blocks' remaining (block, code) pairs end to
    // end and every lane takes every 32nd pair, reading the block from shared
    // memory; a block's best (error, code) is a 64-bit key lowered with an
    // atomic minimum (error bits above the code: the lowest code wins ties).
    auto flush = [&](int n) {
        const bool act = lane < n;
        int64_t b = 0;
        float best = 0.0f;
        uint32_t bc = 0u, c6 = 1u, clo = 1u;
        int chi = 0;
        unsigned long long um = 0ull;
        bool over = false;
        float xv[B];
        if (act) {
            b = (int64_t)q_idx[w][lane];
            const uint32_t qb = q_best[w][lane];
            best = __uint_as_float(qb & 0x7FFFFFFFu);
            over = (qb >> 31) != 0u;
            const uint32_t qc = q_codes[w][lane];
            bc = qc & 0xFFu;
            c6 = (qc >> 8) & 0xFFu;
            clo = (qc >> 16) & 0xFFu;
            chi = (int)(qc >> 24);
            um = q_um[w][lane];
            load_elems<T, B>(x + b * B, xv);
        } else {
#pragma unroll
            for (int i = 0; i < B; ++i)
                xv[i] = 0.0f;
        }
        for (int c = (int)c6 + 65; c <= chi && over; ++c) {
            const float sc_ = quant_sse<B>(xv, 0.0f, 0.0f, tab[c]);
            n_eval += 1u;
            if (sc_ < best || (sc_ == best && (uint32_t)c < bc)) {
                best = sc_;
                bc = (uint32_t)c;
            }
        }
        const int nlow = act ? (int)(c6 - clo) : 0;
        const int span = nlow + __popcll(um);
        int incl = span;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, d);
            if (lane >= d)
                incl += v;
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        if (total > 0) {
#pragma unroll
            for (int i = 0; i < B; i += 4)
                *reinterpret_cast<float4*>(&xw[lane * B + i]) = make_float4(xv[i], xv[i + 1], xv[i + 2], xv[i + 3]);
            key[w][lane] = ((unsigned long long)__float_as_uint(best) << 32) | bc;
            pre[w][lane] = incl - span;
            lowm[w][lane] = clo | ((uint32_t)nlow << 8) | (c6 << 16);
            upm[w][lane] = um;
            __syncwarp();
            for (int t = lane; t < total; t += 32) {
                // owner: the last block whose range starts at or before t
                int j = 0;
#pragma unroll
                for (int st = 16; st > 0; st >>= 1)
                    if (pre[w][j + st] <= t)
                        j += st;
                const uint32_t lm = lowm[w][j];
                const int k = t - pre[w][j];
                const int nl = (int)((lm >> 8) & 0xFFu);
                uint32_t c;
                if (k < nl) {
                    c = (lm & 0xFFu) + (uint32_t)k;
                } else {
                    // the (k - nl)-th set bit (from 0) of the upper-code mask
                    const unsigned long long m = upm[w][j];
                    const uint32_t lo = (uint32_t)m, hi = (uint32_t)(m >> 32);
                    const int r = k - nl;
                    const int nlo = __popc(lo);
                    const uint32_t pos = r < nlo ? __fns(lo, 0u, r + 1) : 32u + __fns(hi, 0u, r - nlo + 1);
                    c = ((lm >> 16) & 0xFFu) + pos + 1u;
                }
                float xj[B];
#pragma unroll
                for (int i = 0; i < B; i += 4) {
                    const float4 q = *reinterpret_cast<const float4*>(&xw[j * B + i]);
                    xj[i] = q.x;
                    xj[i + 1] = q.y;
                    xj[i + 2] = q.z;
                    xj[i + 3] = q.w;
                }
                const float sc_ = quant_sse<B>(xj, 0.0f, 0.0f, tab[c]);
                atomicMin(&key[w][j], ((unsigned long long)__float_as_uint(sc_) << 32) | c);
                ++n_eval;
            }
            __syncwarp();
            bc = (uint32_t)key[w][lane];
            __syncwarp();
        }
        if (act) {
            uint32_t cw[(B + 7) / 8];
            const int64_t so = mma_layout ? mma_sf_offset(b / bpr, b % bpr, kb_atoms) : b;
            store_block(b, xv, bc, 0xFFFFu, cw, best, so);   // never c6: codes from bc
        }
    };

    // blocks of up to 32 bytes: the next block's load is in flight while this
    // one is searched (one load round trip per block otherwise stalls the warp)
    constexpr bool kPrefetch = B * sizeof(T) <= 32;
    float xn[kPrefetch ? B : 1];
    if constexpr (kPrefetch) {
        const int64_t b0 = warp0 * 32 + lane;
        if (b0 < nblk) {
            load_elems<T, B>(x + b0 * B, xn);
        } else {
#pragma unroll
            for (int i = 0; i < B; ++i)
                xn[i] = 0.0f;
        }
    }
    int pcount = 0;   // queued blocks of this warp (the same in every lane)

    for (int64_t base = warp0 * 32; base < nblk; base += nwarps * 32) {
        const int64_t b = base + lane;
        const bool valid = b < nblk;
        float xv[B];
        if constexpr (kPrefetch) {
#pragma unroll
            for (int i = 0; i < B; ++i)
                xv[i] = xn[i];
            const int64_t bn = b + nwarps * 32;
            if (bn < nblk)
                load_elems<T, B>(x + bn * B, xn);
        } else if (valid) {
            load_elems<T, B>(x + b * B, xv);
        } else {
#pragma unroll
            for (int i = 0; i < B; ++i)
                xv[i] = 0.0f;
        }
        uint32_t cw[(B + 7) / 8];
        const BfPlan pl = bf_plan<B, SFMT>(xv, valid, tab, wmask, g6, four_over_g, g_pow2, cw, n_eval);
        const bool pending = valid && (pl.clo < pl.c6 || pl.um != 0ull || pl.over);
        const int64_t so = mma_layout ? mma_sf_offset(r_cur, kb_cur, kb_atoms) : b;
        if (valid && !pending)
            store_block(b, xv, pl.bc, pl.c6, cw, pl.best, so);
        // queue the blocks whose search continues
        const uint32_t bal = __ballot_sync(0xffffffffu, pending);
        if (pending) {
            const int slot = pcount + __popc(bal & ((1u << lane) - 1u));
            q_idx[w][slot] = (unsigned long long)b;
            q_best[w][slot] = __float_as_uint(pl.best) | (pl.over ? 0x80000000u : 0u);
            q_codes[w][slot] = pl.bc | (pl.c6 << 8) | (pl.clo << 16) | ((uint32_t)pl.chi << 24);
            q_um[w][slot] = pl.um;
        }
        pcount += __popc(bal);
        __syncwarp();
        if (pcount >= 32) {
            flush(32);
            // move the rest of the queue to its front
            pcount -= 32;
            uint32_t t_best = 0, t_codes = 0;
            unsigned long long t_idx = 0, t_um = 0;
            if (lane < pcount) {
                t_idx = q_idx[w][32 + lane];
                t_um = q_um[w][32 + lane];
                t_best = q_best[w][32 + lane];
                t_codes = q_codes[w][32 + lane];
            }
            __syncwarp();
            if (lane < pcount) {
                q_idx[w][lane] = t_idx;
                q_um[w][lane] = t_um;
                q_best[w][lane] = t_best;
                q_codes[w][lane] = t_codes;
            }
            __syncwarp();
        }
        if (mma_layout) {
            kb_cur += step_kb;
            r_cur += step_r;
            if (kb_cur >= bpr) {
                kb_cur -= bpr;
                ++r_cur;
            }
        }
    }
    if (pcount > 0)
        flush(pcount);
    if (evals) {
        const uint32_t wsum = __reduce_add_sync(0xffffffffu, n_eval);
        if (lane == 0 && wsum)
            atomicAdd(evals, (unsigned long long)wsum);
    }
}

// ------------------------------------------------------ dequant + MSE
// SF: 0 E4M3, 1 E3M3, 2 E8M0, 3 UE5M3.  RAZ: the -0 code decodes to the block's
// special value (selector in the scale byte's top bits).
template <int B, int SF, bool RAZ, typename TR>
__global__ void __launch_bounds__(kThreads)
dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
               int64_t nblk, SpecialArgs sp, const float* __restrict__ gs_dev,
               const TR* __restrict__ ref, float* __restrict__ deq, float* __restrict__ mse)
{
    // warps walk 32 consecutive blocks at a time (a warp-uniform trip count),
    // so blocks of 32 bytes or more of the reference are read, and the
    // dequantized blocks written, as whole rows through shared memory
    constexpr bool kRefStaged = B * sizeof(TR) >= 32;
    constexpr bool kStoreStaged = B >= 8;
    __shared__ uint4 buf[kThreads / 32][(kRefStaged || kStoreStaged) ? 8 * B : 1];
    const float g = gs_dev ? __ldg(gs_dev) : 1.0f;
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t base = warp0 * 32; base < nblk; base += nwarps * 32) {
        const int64_t b = base + lane;
        const bool valid = b < nblk;
        const uint32_t sb = valid ? __ldg(scales + b) : 0u;
        uint32_t cw[(B + 7) / 8];
        if (!valid) {
#pragma unroll
            for (int j = 0; j < (B + 7) / 8; ++j)
                cw[j] = 0u;
        } else if constexpr (B == 4) {
            cw[0] = __ldg(reinterpret_cast<const uint16_t*>(codes + b * 2));
        } else if constexpr (B == 8) {
            cw[0] = __ldg(reinterpret_cast<const uint32_t*>(codes + b * 4));
        } else if constexpr (B == 16) {
            uint2 v = __ldg(reinterpret_cast<const uint2*>(codes + b * 8));
            cw[0] = v.x; cw[1] = v.y;
        } else {
            uint4 v = __ldg(reinterpret_cast<const uint4*>(codes + b * 16));
            cw[0] = v.x; cw[1] = v.y; cw[2] = v.z; cw[3] = v.w;
        }
        float v[B];
        if constexpr (B == 4) {
            float t[4];
            e2m1x4_decode(cw[0], t);
#pragma unroll
            for (int i = 0; i < 4; ++i)
                v[i] = t[i];
        } else {
#pragma unroll
            for (int j = 0; j < B / 8; ++j) {
                float t[8];
                e2m1x8_decode(cw[j], t);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    v[8 * j + i] = t[i];
            }
        }
        float dq[B];
        if constexpr (SF == 2) {
            // 2^(byte-127) as an fp32 bit pattern (byte 0 is the subnormal 2^-127)
            const float p2 = sb == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(sb << 23);
#pragma unroll
            for (int i = 0; i < B; ++i)
                dq[i] = __fmul_rn(v[i], p2);
        } else {
            uint32_t scc = sb;
            float spv = 0.0f;
            if constexpr (RAZ) {
                const uint32_t sel = SF == 1 ? (sb >> 6) : (sb >> 7);
                scc = SF == 1 ? (sb & 0x3Fu) : (sb & 0x7Fu);
                const uint32_t k = (int)sel < sp.n ? sel : 0u;
                spv = k == 0u ? sp.v[0] : k == 1u ? sp.v[1] : k == 2u ? sp.v[2] : sp.v[3];
            }
            const float scv = SF == 1 ? e3m3_decode(scc) : SF == 3 ? ue5m3_decode(scc) : e4m3_decode(scc);
            const float S = __fmul_rn(scv, g);
#pragma unroll
            for (int i = 0; i < B; ++i) {
                float vi = v[i];
                if constexpr (RAZ) {
                    const uint32_t code = (cw[i >> 3] >> (4 * (i & 7))) & 0xFu;
                    vi = code == 8u ? spv : vi;
                }
                dq[i] = __fmul_rn(vi, S);
            }
        }
        if (mse) {
            float xr[B];
            if constexpr (kRefStaged) {
                warp_load_blocks<TR, B>(ref, base, nblk, buf[threadIdx.x >> 5], xr);
            } else if (valid) {
                load_elems<TR, B>(ref + b * B, xr);
            } else {
#pragma unroll
                for (int i = 0; i < B; ++i)
                    xr[i] = 0.0f;
            }
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < B; ++i) {
                float e = __fsub_rn(xr[i], dq[i]);
                acc = __fmaf_rn(e, e, acc);
            }
            if (valid)
                mse[b] = __fmul_rn(acc, 1.0f / (float)B);
        }
        if (deq) {
            if constexpr (kStoreStaged)
                warp_store_f32_blocks<B>(deq, base, nblk, buf[threadIdx.x >> 5], dq);
            else if (valid)
                store_f32<B>(deq + b * B, dq);
        }
    }
}

// Launch a quantizer kernel over nblk blocks (one thread each) on a grid sized
// by grid_for; a fused global amax (gs.mode 3) needs every CTA resident at
// once, so that launch is cooperative and its grid at most kFusedMaxCtas.
template <typename... KArgs, typename... Args>
cudaError_t launch_quant_kernel(void (*kernel)(KArgs...), int64_t nblk, const GsArgs& gs, cudaStream_t s,
                                Args&&... args);
template <typename... KArgs, typename... Args>
cudaError_t launch_quant_kernel_smem(void (*kernel)(KArgs...), int64_t nblk, const GsArgs& gs, cudaStream_t s,
                                     int dyn_smem, Args&&... args);

int grid_for(int64_t work_threads, const void* kernel, size_t dyn_smem = 0)
{
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, dyn_smem);
    if (per_sm < 1)
        per_sm = 1;
    int64_t want = (work_threads + kThreads - 1) / kThreads;
    int64_t cap = (int64_t)num_sms() * per_sm;
    if (want > cap)
        want = cap;
    return (int)(want < 1 ? 1 : want);
}

// The brute-force window masks (see BfWindows), computed once in exact
// (dyadic, so exact in double) arithmetic.  Scale values in units of the
// subnormal step s of a 3-mantissa-bit format: code c < 8 is c s, code
// 8 + 8 d + m is 2^d (8 + m) s; a normal power-of-two reference behaves like
// code 8 (its offsets repeat the same ratios).
const BfWindows& bf_windows()
{
    static BfWindows w;
    static std::once_flag once;
    std::call_once(once, [] {
        const double G[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
        auto value = [](int c) { return c < 8 ? (double)c : std::ldexp((double)(8 + ((c - 8) & 7)), (c - 8) >> 3); };
        const int ref_code[4] = {8, 1, 2, 4};
        for (int t = 0; t < 4; ++t) {
            for (int b = 0; b < 49; ++b)
                w.m[t][b] = 0ull;
            const int r = ref_code[t];
            for (int j = 0; j < 64; ++j) {
                const double k = value(r + 1 + j) / value(r);
                for (int i = 1; i < 8; ++i) {
                    const double p = k * G[i];
                    bool on_grid = false;
                    for (int q = 0; q < 8; ++q)
                        on_grid = on_grid || G[q] == p;
                    if (p >= 6.0 || on_grid)
                        continue;
                    double q1 = 0.0, q2 = 6.0;
                    for (int q = 0; q < 8; ++q) {
                        if (G[q] < p && G[q] > q1)
                            q1 = G[q];
                        if (G[q] > p && G[q] < q2)
                            q2 = G[q];
                    }
                    const double lo = 0.5 * (q1 + p), hi = 0.5 * (p + q2);   // open window
                    for (int b = 0; b < 49; ++b)
                        if (b / 8.0 < hi && (b + 1) / 8.0 > lo)
                            w.m[t][b] |= 1ull << j;
                }
            }
        }
    });
    return w;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_quant_kernel(void (*kernel)(KArgs...), int64_t nblk, const GsArgs& gs, cudaStream_t s,
                                Args&&... args)
{
    return launch_quant_kernel_smem(kernel, nblk, gs, s, 0, std::forward<Args>(args)...);
}

// The same with `dyn_smem` bytes of dynamic shared memory per CTA.
template <typename... KArgs, typename... Args>
cudaError_t launch_quant_kernel_smem(void (*kernel)(KArgs...), int64_t nblk, const GsArgs& gs, cudaStream_t s,
                                     int dyn_smem, Args&&... args)
{
    if (dyn_smem > 0) {
        const cudaError_t e = smem_opt_in((const void*)kernel, dyn_smem);
        if (e != cudaSuccess)
            return e;
    }
    int grid = grid_for(nblk, (const void*)kernel, (size_t)dyn_smem);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    if (gs.mode == 3) {
        grid = grid < kFusedMaxCtas ? grid : kFusedMaxCtas;
        attr[0].id = cudaLaunchAttributeCooperative;
        attr[0].val.cooperative = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = (size_t)dyn_smem;
    cfg.stream = s;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int B, typename T, int RULE, int SFMT>
cudaError_t nvfp4_launch_t(const void* x, int64_t rows, int64_t cols, const GsArgs& gs,
                           uint8_t* codes, uint8_t* scales, int mma, float* deq, float* mse,
                           unsigned long long* evals, cudaStream_t s)
{
    const int64_t nblk = rows * (cols / B);
    if constexpr (RULE == R_BF) {
        const int dyn = kWarps * 32 * B * (int)sizeof(float);
        if (deq)
            return launch_quant_kernel_smem(nvfp4_bf_kernel<B, T, SFMT, true>, nblk, gs, s, dyn,
                                            reinterpret_cast<const T*>(x), nblk, cols / B, gs, codes, scales, mma, deq,
                                            mse, evals, bf_windows());
        return launch_quant_kernel_smem(nvfp4_bf_kernel<B, T, SFMT, false>, nblk, gs, s, dyn,
                                        reinterpret_cast<const T*>(x), nblk, cols / B, gs, codes, scales, mma, deq, mse,
                                        evals, bf_windows());
    } else {
        // dequantized values are a compile-time option: without them the
        // candidates' values need not stay live
        if (deq)
            return launch_quant_kernel(nvfp4_quant_kernel<B, T, RULE, SFMT, true>, nblk, gs, s,
                                       reinterpret_cast<const T*>(x), nblk, cols / B, gs, codes, scales, mma, deq, mse);
        return launch_quant_kernel(nvfp4_quant_kernel<B, T, RULE, SFMT, false>, nblk, gs, s,
                                   reinterpret_cast<const T*>(x), nblk, cols / B, gs, codes, scales, mma, deq, mse);
    }
}

template <int B, typename T, int SFMT>
cudaError_t nvfp4_launch_rule(int rule, const void* x, int64_t rows, int64_t cols,
                              const GsArgs& gs, uint8_t* codes, uint8_t* scales, int mma,
                              float* deq, float* mse, unsigned long long* evals, cudaStream_t s)
{
    switch (rule) {
    case R_ABSMAX: return nvfp4_launch_t<B, T, R_ABSMAX, SFMT>(x, rows, cols, gs, codes, scales, mma, deq, mse, evals, s);
    case R_PZ: return nvfp4_launch_t<B, T, R_PZ, SFMT>(x, rows, cols, gs, codes, scales, mma, deq, mse, evals, s);
    case R_46: return nvfp4_launch_t<B, T, R_46, SFMT>(x, rows, cols, gs, codes, scales, mma, deq, mse, evals, s);
    case R_BF: return nvfp4_launch_t<B, T, R_BF, SFMT>(x, rows, cols, gs, codes, scales, mma, deq, mse, evals, s);
    default: return cudaErrorInvalidValue;
    }
}

template <typename T, int SFMT>
cudaError_t nvfp4_launch_b(int block, int rule, const void* x, int64_t rows, int64_t cols,
                           const GsArgs& gs, uint8_t* codes, uint8_t* scales, int mma, float* deq,
                           float* mse, unsigned long long* evals, cudaStream_t s)
{
    switch (block) {
    case 4: return nvfp4_launch_rule<4, T, SFMT>(rule, x, rows, cols, gs, codes, scales, mma, deq, mse, evals, s);
    case 8: return nvfp4_launch_rule<8, T, SFMT>(rule, x, rows, cols, gs, codes, scales, mma, deq, mse, evals, s);
    case 16: return nvfp4_launch_rule<16, T, SFMT>(rule, x, rows, cols, gs, codes, scales, mma, deq, mse, evals, s);
    case 32: return nvfp4_launch_rule<32, T, SFMT>(rule, x, rows, cols, gs, codes, scales, mma, deq, mse, evals, s);
    default: return cudaErrorInvalidValue;
    }
}

template <int B, int SF, bool RAZ>
cudaError_t dequant_launch_t(const uint8_t* codes, const uint8_t* scales, int64_t nblk,
                             const SpecialArgs& sp, const float* gs_dev, const void* ref,
                             int ref_dt, float* deq, float* mse, cudaStream_t s)
{
    if (ref_dt == 1) {
        auto k = dequant_kernel<B, SF, RAZ, __nv_bfloat16>;
        k<<<grid_for(nblk, (const void*)k), kThreads, 0, s>>>(
            codes, scales, nblk, sp, gs_dev, reinterpret_cast<const __nv_bfloat16*>(ref), deq, mse);
    } else {
        auto k = dequant_kernel<B, SF, RAZ, float>;
        k<<<grid_for(nblk, (const void*)k), kThreads, 0, s>>>(
            codes, scales, nblk, sp, gs_dev, reinterpret_cast<const float*>(ref), deq, mse);
    }
    return cudaGetLastError();
}

template <int SF, bool RAZ>
cudaError_t dequant_launch_b(int block, const uint8_t* codes, const uint8_t* scales, int64_t nblk,
                             const SpecialArgs& sp, const float* gs_dev, const void* ref,
                             int ref_dt, float* deq, float* mse, cudaStream_t s)
{
    switch (block) {
    case 4: return dequant_launch_t<4, SF, RAZ>(codes, scales, nblk, sp, gs_dev, ref, ref_dt, deq, mse, s);
    case 8: return dequant_launch_t<8, SF, RAZ>(codes, scales, nblk, sp, gs_dev, ref, ref_dt, deq, mse, s);
    case 16: return dequant_launch_t<16, SF, RAZ>(codes, scales, nblk, sp, gs_dev, ref, ref_dt, deq, mse, s);
    case 32: return dequant_launch_t<32, SF, RAZ>(codes, scales, nblk, sp, gs_dev, ref, ref_dt, deq, mse, s);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_amax(const void* x, int dtype, int64_t n, float* partials, cudaStream_t s)
{
    if (dtype == 1)
        amax_kernel<__nv_bfloat16><<<kAmaxPartials, kThreads, 0, s>>>(
            reinterpret_cast<const __nv_bfloat16*>(x), n, partials);
    else
        amax_kernel<float><<<kAmaxPartials, kThreads, 0, s>>>(reinterpret_cast<const float*>(x), n,
                                                               partials);
    return cudaGetLastError();
}

cudaError_t launch_nvfp4_quant(const void* x, int dtype, int64_t rows, int64_t cols, int block,
                               int rule, const GsArgs& gs, uint8_t* codes, uint8_t* scales,
                               int mma_layout, float* deq, float* mse, unsigned long long* evals,
                               cudaStream_t s, int ue5m3)
{
    if (ue5m3) {
        if (dtype == 1)
            return nvfp4_launch_b<__nv_bfloat16, 1>(block, rule, x, rows, cols, gs, codes, scales,
                                                    mma_layout, deq, mse, evals, s);
        return nvfp4_launch_b<float, 1>(block, rule, x, rows, cols, gs, codes, scales, mma_layout,
                                        deq, mse, evals, s);
    }
    if (dtype == 1)
        return nvfp4_launch_b<__nv_bfloat16, 0>(block, rule, x, rows, cols, gs, codes, scales,
                                                mma_layout, deq, mse, evals, s);
    return nvfp4_launch_b<float, 0>(block, rule, x, rows, cols, gs, codes, scales, mma_layout, deq,
                                    mse, evals, s);
}

cudaError_t launch_razer_quant(const void* x, int dtype, int64_t rows, int64_t cols, int sf,
                               const float* specials_host, int n_special, const GsArgs& gs,
                               uint8_t* codes, uint8_t* meta, float* deq, float* mse,
                               cudaStream_t s)
{
    SpecialArgs sp{};
    for (int i = 0; i < n_special && i < 4; ++i) {
        const float v = specials_host[i];
        const float m = v < 0.0f ? -v : v;
        sp.v[i] = v;
        sp.neg[i] = v < 0.0f;
        int mi = 0;
        while (mi < sp.nmag && sp.mag[mi] != m)
            ++mi;
        if (mi == sp.nmag)
            sp.mag[sp.nmag++] = m;
        sp.mag_of[i] = mi;
    }
    sp.n = n_special;
    const int64_t nblk = rows * (cols / 16);
    // (+v, -v) pairs in table order take the single-pass kernel
    bool paired = n_special % 2 == 0;
    for (int i = 0; paired && i < n_special; i += 2)
        paired = specials_host[i] > 0.0f && specials_host[i + 1] == -specials_host[i];
    if (paired) {
        const int np = n_special / 2;
#define FP4Q_RAZER_PAIRED(TT, SFV, NP)                                                                  \
    return launch_quant_kernel(razer_paired_kernel<TT, SFV, NP>, nblk, gs, s, reinterpret_cast<const TT*>(x), \
                               nblk, gs, sp, codes, meta, deq, mse);
        if (dtype == 1) {
            if (sf == 1) {
                if (np == 1) FP4Q_RAZER_PAIRED(__nv_bfloat16, 1, 1) else FP4Q_RAZER_PAIRED(__nv_bfloat16, 1, 2)
            } else {
                FP4Q_RAZER_PAIRED(__nv_bfloat16, 0, 1)
            }
        } else {
            if (sf == 1) {
                if (np == 1) FP4Q_RAZER_PAIRED(float, 1, 1) else FP4Q_RAZER_PAIRED(float, 1, 2)
            } else {
                FP4Q_RAZER_PAIRED(float, 0, 1)
            }
        }
#undef FP4Q_RAZER_PAIRED
    }
    if (dtype == 1) {
        if (sf == 1)
            return launch_quant_kernel(razer_quant_kernel<__nv_bfloat16, 1>, nblk, gs, s,
                                       reinterpret_cast<const __nv_bfloat16*>(x), nblk, gs, sp, codes, meta, deq, mse);
        return launch_quant_kernel(razer_quant_kernel<__nv_bfloat16, 0>, nblk, gs, s,
                                   reinterpret_cast<const __nv_bfloat16*>(x), nblk, gs, sp, codes, meta, deq, mse);
    }
    if (sf == 1)
        return launch_quant_kernel(razer_quant_kernel<float, 1>, nblk, gs, s, reinterpret_cast<const float*>(x),
                                   nblk, gs, sp, codes, meta, deq, mse);
    return launch_quant_kernel(razer_quant_kernel<float, 0>, nblk, gs, s, reinterpret_cast<const float*>(x), nblk,
                               gs, sp, codes, meta, deq, mse);
}

cudaError_t launch_dequant_mse(const uint8_t* codes, const uint8_t* scales, int64_t rows,
                               int64_t cols, int block, int sf, const float* specials_host,
                               int n_special, const float* gs_dev, const void* ref, int ref_dt,
                               float* deq, float* mse, cudaStream_t s)
{
    SpecialArgs sp{};
    for (int i = 0; i < n_special && i < 4; ++i)
        sp.v[i] = specials_host[i];
    sp.n = n_special;
    const int64_t nblk = rows * (cols / block);
    const bool raz = specials_host != nullptr && n_special > 0;
    if (sf == 2)
        return dequant_launch_b<2, false>(block, codes, scales, nblk, sp, nullptr, ref, ref_dt, deq, mse, s);
    if (sf == 3)
        return dequant_launch_b<3, false>(block, codes, scales, nblk, sp, gs_dev, ref, ref_dt, deq, mse, s);
    if (sf == 1)
        return raz ? dequant_launch_b<1, true>(block, codes, scales, nblk, sp, gs_dev, ref, ref_dt, deq, mse, s)
                   : dequant_launch_b<1, false>(block, codes, scales, nblk, sp, gs_dev, ref, ref_dt, deq, mse, s);
    return raz ? dequant_launch_b<0, true>(block, codes, scales, nblk, sp, gs_dev, ref, ref_dt, deq, mse, s)
               : dequant_launch_b<0, false>(block, codes, scales, nblk, sp, gs_dev, ref, ref_dt, deq, mse, s);
}

}  // namespace fp4q
