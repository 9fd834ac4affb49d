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
#include <cstdint>

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

// The per-tensor global scale for this launch (all threads of the CTA get it).
__device__ float resolve_global_scale(const GsArgs& gs)
{
    __shared__ float s_g;
    if (gs.mode == 0)
        return 1.0f;
    if (gs.mode == 2)
        return __ldg(gs.given);
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
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += stride) {
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
template <int B>
__device__ __forceinline__ float quant_eval(const float (&x)[B], float sc, float g,
                                            uint32_t (&cw)[(B + 7) / 8], float (&dq)[B])
{
    const float S = __fmul_rn(sc, g);
    const float inv = (S == 0.0f) ? 0.0f : fminf(__frcp_rn(S), kFltMax);
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

// Squared error only (brute-force search).
template <int B>
__device__ __forceinline__ float quant_sse(const float (&x)[B], float sc, float g)
{
    uint32_t cw[(B + 7) / 8];
    float dq[B];
    return quant_eval<B>(x, sc, g, cw, dq);
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

template <int B, typename T, int RULE>
__global__ void __launch_bounds__(kThreads)
nvfp4_quant_kernel(const T* __restrict__ x, int64_t nblk, int64_t bpr, GsArgs gs,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int mma_layout,
                   float* __restrict__ deq, float* __restrict__ mse)
{
    const float g = resolve_global_scale(gs);
    const float g6 = __fmul_rn(6.0f, g);
    const float g4 = __fmul_rn(4.0f, g);
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t kb_atoms = (bpr + 3) >> 2;

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

        uint32_t cw[(B + 7) / 8];
        float dq[B];
        float sse;
        uint32_t sc;
        if constexpr (RULE == R_ABSMAX || RULE == R_PZ) {
            sc = e4m3_encode(__fdiv_rn(a, g6));
            if (RULE == R_PZ && sc == 0u)
                sc = 1u;
            sse = quant_eval<B>(xv, e4m3_decode(sc), g, cw, dq);
        } else if constexpr (RULE == R_46) {
            const uint32_t c6 = e4m3_encode(__fdiv_rn(a, g6));
            const uint32_t c4 = e4m3_encode(__fdiv_rn(a, g4));
            uint32_t cw4[(B + 7) / 8];
            float dq4[B];
            const float s6 = quant_eval<B>(xv, e4m3_decode(c6), g, cw, dq);
            const float s4 = quant_eval<B>(xv, e4m3_decode(c4), g, cw4, dq4);
            const bool take4 = s4 < s6;
            sc = take4 ? c4 : c6;
            sse = take4 ? s4 : s6;
#pragma unroll
            for (int j = 0; j < (B + 7) / 8; ++j)
                cw[j] = take4 ? cw4[j] : cw[j];
#pragma unroll
            for (int i = 0; i < B; ++i)
                dq[i] = take4 ? dq4[i] : dq[i];
        } else {
            // Brute force over E4M3 codes 1..126 in ascending order, keeping the
            // lowest code among equal errors.  Exact shortcuts:
            //  * once the largest element rounds to zero (|y| <= 0.25) every
            //    element does, and every larger scale gives the same error, so
            //    the scan stops there;
            //  * the squared error of the largest element alone is a lower bound
            //    of the in-order fma sum, so a candidate whose bound already
            //    loses is skipped.
            float sse0 = 0.0f;
#pragma unroll
            for (int i = 0; i < B; ++i)
                sse0 = __fmaf_rn(xv[i], xv[i], sse0);
            uint32_t c0 = e4m3_encode(__fdiv_rn(a, g6));
            c0 = c0 == 0u ? 1u : c0;
            float best = quant_sse<B>(xv, e4m3_decode(c0), g);
            uint32_t bc = c0;
            bool done = !valid;
            for (uint32_t c = 1; c <= 0x7Eu; ++c) {
                if (!done) {
                    const float scv = e4m3_decode(c);
                    const float S = __fmul_rn(scv, g);
                    const float inv = (S == 0.0f) ? 0.0f : fminf(__frcp_rn(S), kFltMax);
                    const float ym = __fmul_rn(a, inv);
                    if (ym <= 0.25f) {
                        done = true;
                        if (c != c0 && (sse0 < best || (sse0 == best && c < bc))) {
                            best = sse0;
                            bc = c;
                        }
                    } else if (c != c0) {
                        const float em = elem_err(a, S, inv);
                        const float lb = __fmul_rn(em, em);
                        if (lb < best || (lb == best && c < bc)) {
                            const float s = quant_sse<B>(xv, scv, g);
                            if (s < best || (s == best && c < bc)) {
                                best = s;
                                bc = c;
                            }
                        }
                    }
                }
                if (__all_sync(0xffffffffu, done))
                    break;
            }
            sc = bc;
            sse = quant_eval<B>(xv, e4m3_decode(bc), g, cw, dq);
        }

        if (valid) {
            store_codes<B>(codes + b * (B / 2), cw);
            const int64_t so = mma_layout ? mma_sf_offset(b / bpr, b % bpr, kb_atoms) : b;
            scales[so] = (uint8_t)sc;
            if (deq)
                store_f32<B>(deq + b * B, dq);
            if (mse)
                mse[b] = __fmul_rn(sse, 1.0f / (float)B);
        }
    }
}

// ------------------------------------------------------------------ RaZeR
struct SpecialArgs {
    float v[4];
    int n;
};

// SF = 0: E4M3 scale, selector in bit 7 (activations); SF = 1: E3M3 scale,
// selector in bits 7..6 (weights).  Block size 16.
template <typename T, int SF>
__global__ void __launch_bounds__(kThreads)
razer_quant_kernel(const T* __restrict__ x, int64_t nblk, GsArgs gs, SpecialArgs sp,
                   uint8_t* __restrict__ codes, uint8_t* __restrict__ meta,
                   float* __restrict__ deq, float* __restrict__ mse)
{
    constexpr int B = 16;
    const float g = resolve_global_scale(gs);
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

        // plain E2M1 quantization of every element
        float ay[B], vs[B], dstd[B];
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
                ay[8 * j + i] = fabsf(y[i]);
                vs[8 * j + i] = v[i];
                dstd[8 * j + i] = __fmul_rn(v[i], S);
            }
        }
        // score each special value in table order
        float best = 0.0f;
        int sel = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            if (k >= sp.n)
                break;
            const float spv = sp.v[k];
            const float spa = fabsf(spv);
            const bool spneg = signbit(spv);
            const float dsp = __fmul_rn(spv, S);
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < B; ++i) {
                const uint32_t code = (cw[i >> 3] >> (4 * (i & 7))) & 0xFu;
                const bool nz = (code & 7u) != 0u;
                const bool neg = (code & 8u) != 0u;
                const float dg = fabsf(__fsub_rn(ay[i], fabsf(vs[i])));
                const float ds = fabsf(__fsub_rn(ay[i], spa));
                const bool use = nz && (neg == spneg) && (ds < dg);
                const float e = __fsub_rn(xv[i], use ? dsp : dstd[i]);
                acc = __fmaf_rn(e, e, acc);
            }
            if (k == 0 || acc < best) {
                best = acc;
                sel = k;
            }
        }
        // outputs for the chosen special
        const float spv = sel == 0 ? sp.v[0] : sel == 1 ? sp.v[1] : sel == 2 ? sp.v[2] : sp.v[3];
        const float spa = fabsf(spv);
        const bool spneg = signbit(spv);
        const float dsp = __fmul_rn(spv, S);
        float dq[B];
        uint32_t ow[2] = {0u, 0u};
#pragma unroll
        for (int i = 0; i < B; ++i) {
            const uint32_t code = (cw[i >> 3] >> (4 * (i & 7))) & 0xFu;
            const bool nz = (code & 7u) != 0u;
            const bool neg = (code & 8u) != 0u;
            const float dg = fabsf(__fsub_rn(ay[i], fabsf(vs[i])));
            const float ds = fabsf(__fsub_rn(ay[i], spa));
            const bool use = nz && (neg == spneg) && (ds < dg);
            const uint32_t oc = !nz ? 0u : (use ? 8u : code);
            dq[i] = !nz ? 0.0f : (use ? dsp : dstd[i]);
            ow[i >> 3] |= oc << (4 * (i & 7));
        }
        if (valid) {
            *reinterpret_cast<uint2*>(codes + b * 8) = make_uint2(ow[0], ow[1]);
            meta[b] = (uint8_t)(SF == 1 ? ((uint32_t)sel << 6) | scc : ((uint32_t)sel << 7) | scc);
            if (deq)
                store_f32<B>(deq + b * B, dq);
            if (mse)
                mse[b] = __fmul_rn(best, 1.0f / 16.0f);
        }
    }
}

// ------------------------------------------------------ dequant + MSE
// SF: 0 E4M3, 1 E3M3, 2 E8M0.  RAZ: the -0 code decodes to the block's
// special value (selector in the scale byte's top bits).
template <int B, int SF, bool RAZ, typename TR>
__global__ void __launch_bounds__(kThreads)
dequant_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
               int64_t nblk, SpecialArgs sp, const float* __restrict__ gs_dev,
               const TR* __restrict__ ref, float* __restrict__ deq, float* __restrict__ mse)
{
    const float g = gs_dev ? __ldg(gs_dev) : 1.0f;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += stride) {
        const uint32_t sb = __ldg(scales + b);
        uint32_t cw[(B + 7) / 8];
        if constexpr (B == 4) {
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
            const float scv = SF == 1 ? e3m3_decode(scc) : e4m3_decode(scc);
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
        if (deq)
            store_f32<B>(deq + b * B, dq);
        if (mse) {
            float xr[B];
            load_elems<TR, B>(ref + b * B, xr);
            float acc = 0.0f;
#pragma unroll
            for (int i = 0; i < B; ++i) {
                float e = __fsub_rn(xr[i], dq[i]);
                acc = __fmaf_rn(e, e, acc);
            }
            mse[b] = __fmul_rn(acc, 1.0f / (float)B);
        }
    }
}

int grid_for(int64_t work_threads, const void* kernel)
{
    int per_sm = 0;
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, 0);
    if (per_sm < 1)
        per_sm = 1;
    int64_t want = (work_threads + kThreads - 1) / kThreads;
    int64_t cap = (int64_t)num_sms() * per_sm;
    if (want > cap)
        want = cap;
    return (int)(want < 1 ? 1 : want);
}

template <int B, typename T, int RULE>
cudaError_t nvfp4_launch_t(const void* x, int64_t rows, int64_t cols, const GsArgs& gs,
                           uint8_t* codes, uint8_t* scales, int mma, float* deq, float* mse,
                           cudaStream_t s)
{
    const int64_t nblk = rows * (cols / B);
    auto k = nvfp4_quant_kernel<B, T, RULE>;
    const int grid = grid_for(nblk, (const void*)k);
    k<<<grid, kThreads, 0, s>>>(reinterpret_cast<const T*>(x), nblk, cols / B, gs, codes, scales,
                                 mma, deq, mse);
    return cudaGetLastError();
}

template <int B, typename T>
cudaError_t nvfp4_launch_rule(int rule, const void* x, int64_t rows, int64_t cols,
                              const GsArgs& gs, uint8_t* codes, uint8_t* scales, int mma,
                              float* deq, float* mse, cudaStream_t s)
{
    switch (rule) {
    case R_ABSMAX: return nvfp4_launch_t<B, T, R_ABSMAX>(x, rows, cols, gs, codes, scales, mma, deq, mse, s);
    case R_PZ: return nvfp4_launch_t<B, T, R_PZ>(x, rows, cols, gs, codes, scales, mma, deq, mse, s);
    case R_46: return nvfp4_launch_t<B, T, R_46>(x, rows, cols, gs, codes, scales, mma, deq, mse, s);
    case R_BF: return nvfp4_launch_t<B, T, R_BF>(x, rows, cols, gs, codes, scales, mma, deq, mse, s);
    default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t nvfp4_launch_b(int block, int rule, const void* x, int64_t rows, int64_t cols,
                           const GsArgs& gs, uint8_t* codes, uint8_t* scales, int mma, float* deq,
                           float* mse, cudaStream_t s)
{
    switch (block) {
    case 4: return nvfp4_launch_rule<4, T>(rule, x, rows, cols, gs, codes, scales, mma, deq, mse, s);
    case 8: return nvfp4_launch_rule<8, T>(rule, x, rows, cols, gs, codes, scales, mma, deq, mse, s);
    case 16: return nvfp4_launch_rule<16, T>(rule, x, rows, cols, gs, codes, scales, mma, deq, mse, s);
    case 32: return nvfp4_launch_rule<32, T>(rule, x, rows, cols, gs, codes, scales, mma, deq, mse, s);
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

int num_sms()
{
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0)
            n = 148;
    }
    return n;
}

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
                               int mma_layout, float* deq, float* mse, cudaStream_t s)
{
    if (dtype == 1)
        return nvfp4_launch_b<__nv_bfloat16>(block, rule, x, rows, cols, gs, codes, scales,
                                             mma_layout, deq, mse, s);
    return nvfp4_launch_b<float>(block, rule, x, rows, cols, gs, codes, scales, mma_layout, deq,
                                 mse, s);
}

cudaError_t launch_razer_quant(const void* x, int dtype, int64_t rows, int64_t cols, int sf,
                               const float* specials_host, int n_special, const GsArgs& gs,
                               uint8_t* codes, uint8_t* meta, float* deq, float* mse,
                               cudaStream_t s)
{
    SpecialArgs sp{};
    for (int i = 0; i < n_special && i < 4; ++i)
        sp.v[i] = specials_host[i];
    sp.n = n_special;
    const int64_t nblk = rows * (cols / 16);
    if (dtype == 1) {
        if (sf == 1) {
            auto k = razer_quant_kernel<__nv_bfloat16, 1>;
            k<<<grid_for(nblk, (const void*)k), kThreads, 0, s>>>(
                reinterpret_cast<const __nv_bfloat16*>(x), nblk, gs, sp, codes, meta, deq, mse);
        } else {
            auto k = razer_quant_kernel<__nv_bfloat16, 0>;
            k<<<grid_for(nblk, (const void*)k), kThreads, 0, s>>>(
                reinterpret_cast<const __nv_bfloat16*>(x), nblk, gs, sp, codes, meta, deq, mse);
        }
    } else {
        if (sf == 1) {
            auto k = razer_quant_kernel<float, 1>;
            k<<<grid_for(nblk, (const void*)k), kThreads, 0, s>>>(
                reinterpret_cast<const float*>(x), nblk, gs, sp, codes, meta, deq, mse);
        } else {
            auto k = razer_quant_kernel<float, 0>;
            k<<<grid_for(nblk, (const void*)k), kThreads, 0, s>>>(
                reinterpret_cast<const float*>(x), nblk, gs, sp, codes, meta, deq, mse);
        }
    }
    return cudaGetLastError();
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
    if (sf == 1)
        return raz ? dequant_launch_b<1, true>(block, codes, scales, nblk, sp, gs_dev, ref, ref_dt, deq, mse, s)
                   : dequant_launch_b<1, false>(block, codes, scales, nblk, sp, gs_dev, ref, ref_dt, deq, mse, s);
    return raz ? dequant_launch_b<0, true>(block, codes, scales, nblk, sp, gs_dev, ref, ref_dt, deq, mse, s)
               : dequant_launch_b<0, false>(block, codes, scales, nblk, sp, gs_dev, ref, ref_dt, deq, mse, s);
}

}  // namespace fp4q
