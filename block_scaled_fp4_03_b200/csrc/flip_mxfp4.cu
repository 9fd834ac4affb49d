// flip_mxfp4.cu -- Flip-Refinement of MXFP4 weight codes ("MACaQ: Fast, Model
// Agnostic Calibrated Quantization ..." review, section 1 Key Terms and
// section 3 Method): starting from the round-to-nearest codes at the chosen
// block exponents, each output row repeatedly takes the single move of one
// code to a neighbouring E2M1 level with the largest closed-form decrease of
// sum_k d_k^T H'_k d_k (d = u - deq), updating the block gradient g = H'd
// incrementally, until no move gains or the row's move budget is spent.
//
// One warp owns one row; lane j holds element j of whichever 32-block is in
// hand.  Per-row state lives in shared memory: the gradient g and the codes
// of the whole row, and for every block the best move it offers (gain and
// element), so a step only re-scores the block it changed.  The rows of a CTA
// start together: their gradients need every H'_k once, which the CTA stages
// in shared memory (transposed, padded) one block at a time.
//
// Arithmetic follows the definition step by step in fp32 with explicit
// rounding: g_i = fma chain over j of H_ij d_j in j order; for a move of
// element i by D = (v' - v) 2^e, gain = 2 (D g_i) - (D D) H_ii; the row's
// best is the largest positive gain, ties to the lowest element and, within
// an element, to the downward move; after a move g_j <- fma(-D, H_ji, g_j).
#include <cstdint>

#include "fp4q_device.cuh"
#include "fp4q_internal.h"

namespace fp4q {

namespace {

constexpr int kFlipWarps = 4;
constexpr int kFlipThreads = 32 * kFlipWarps;

__device__ __forceinline__ float flip_pow2(int e)
{
    return e <= -127 ? __uint_as_float(0x00400000u) : __uint_as_float((uint32_t)(e + 127) << 23);
}

// E2M1 value of a code (sign bit 3, magnitude index in bits 2:0).
__device__ __forceinline__ float flip_value(uint32_t code)
{
    const uint32_t m = code & 7u;
    // bits of 0.5 * 2^(m/2) * (1 + (m&1)/2) for m >= 2; 0.5 for m == 1; 0 for m == 0
    float mag = m >= 2u ? __uint_as_float(((m << 22) + (126u << 23))) : (m == 1u ? 0.5f : 0.0f);
    return (code & 8u) ? -mag : mag;
}

// Ladder index of a code's value among the 15 distinct E2M1 values (-6 .. 6),
// and the code of a ladder index (+0 for the zero level).
__device__ __forceinline__ int flip_level(uint32_t code)
{
    const int m = (int)(code & 7u);
    return (code & 8u) ? 7 - m : 7 + m;
}

__device__ __forceinline__ uint32_t flip_code_of_level(int level)
{
    return level >= 7 ? (uint32_t)(level - 7) : (8u | (uint32_t)(7 - level));
}

struct Move {
    float gain;     // > 0 for a real move
    int idx;        // element index in the row * 2 + (1 for the upward move)
};

__device__ __forceinline__ bool better(float ga, int ia, float gb, int ib)
{
    return ga > gb || (ga == gb && ia < ib);
}

// The best move of this lane's element: the downward move first, the upward
// one only if strictly better; no move (gain 0, idx INT_MAX) if neither gains.
__device__ __forceinline__ Move element_best(uint32_t code, float g, float Hii, float scale2e, int elem)
{
    Move best{0.0f, 0x7FFFFFFF};
    const int level = flip_level(code);
    const float v = flip_value(code);
#pragma unroll
    for (int dir = 0; dir < 2; ++dir) {
        const int nl = level + (dir ? 1 : -1);
        if (nl < 0 || nl > 14)
            continue;
        const float D = __fmul_rn(__fsub_rn(flip_value(flip_code_of_level(nl)), v), scale2e);
        const float gain = __fsub_rn(__fmul_rn(2.0f, __fmul_rn(D, g)), __fmul_rn(__fmul_rn(D, D), Hii));
        if (gain > best.gain) {
            best.gain = gain;
            best.idx = elem * 2 + dir;
        }
    }
    return best;
}

__device__ __forceinline__ Move warp_best(Move m)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        const float og = __shfl_xor_sync(0xffffffffu, m.gain, off);
        const int oi = __shfl_xor_sync(0xffffffffu, m.idx, off);
        if (better(og, oi, m.gain, m.idx)) {
            m.gain = og;
            m.idx = oi;
        }
    }
    return m;
}

template <typename T>
__global__ void __launch_bounds__(kFlipThreads)
flip_refine_kernel(const T* __restrict__ w, int64_t rows, int64_t cols, const float* __restrict__ tinv,
                   int had, const float* __restrict__ hess, int max_moves, uint8_t* __restrict__ codes,
                   const uint8_t* __restrict__ scales, int32_t* __restrict__ moves)
{
    extern __shared__ __align__(16) uint8_t flip_smem[];
    const int64_t kb = cols / 32;
    // CTA: H'_k transposed with a padded row (conflict-free column reads), the
    // diagonal of every block; per warp: g, codes, per-block best move
    float* HsT = reinterpret_cast<float*>(flip_smem);                  // 32 x 33
    float* diag = HsT + 32 * 33;                                       // cols
    uint8_t* per_warp = reinterpret_cast<uint8_t*>(diag + cols);
    const size_t warp_bytes = (size_t)cols * 5 + (size_t)kb * 8;
    const int lane = threadIdx.x & 31;
    const int wid = threadIdx.x >> 5;
    float* g = reinterpret_cast<float*>(per_warp + wid * warp_bytes);
    float* bgain = g + cols;
    int* bidx = reinterpret_cast<int*>(bgain + kb);
    uint8_t* cs = reinterpret_cast<uint8_t*>(bidx + kb);

    for (int64_t i = threadIdx.x; i < cols; i += blockDim.x)
        diag[i] = __ldg(hess + (i >> 5) * 1024 + (i & 31) * 33);
    const float c_had = __uint_as_float(0x3E3504F3u);

    for (int64_t r0 = (int64_t)blockIdx.x * kFlipWarps; r0 < rows; r0 += (int64_t)gridDim.x * kFlipWarps) {
        const int64_t r = r0 + wid;
        const bool active = r < rows;
        // ---- gradients and per-block best moves of the CTA's rows
        for (int64_t k = 0; k < kb; ++k) {
            __syncthreads();   // the previous block's H'_k is no longer read
            for (int q = threadIdx.x; q < 1024; q += blockDim.x)
                HsT[(q & 31) * 33 + (q >> 5)] = __ldg(hess + k * 1024 + q);
            __syncthreads();
            if (!active)
                continue;
            const int64_t col = k * 32 + lane;
            float u = (sizeof(T) == 4)
                          ? reinterpret_cast<const float*>(w)[r * cols + col]
                          : __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(w)[r * cols + col] << 16);
            if (tinv)
                u = __fmul_rn(u, __ldg(tinv + col));
            if (had) {
#pragma unroll
                for (int h = 1; h < 32; h <<= 1) {
                    const float o = __shfl_xor_sync(0xffffffffu, u, h);
                    u = (lane & h) ? __fsub_rn(o, u) : __fadd_rn(u, o);
                }
                u = __fmul_rn(u, c_had);
            }
            const uint8_t byte = codes[(r * cols + col) >> 1];
            const uint32_t code = (col & 1) ? (uint32_t)(byte >> 4) : (uint32_t)(byte & 15u);
            const int e = (int)scales[r * kb + k] - 127;
            const float s2e = flip_pow2(e);
            const float d = __fsub_rn(u, __fmul_rn(flip_value(code), s2e));
            float v = 0.0f;
#pragma unroll
            for (int j = 0; j < 32; ++j)
                v = __fmaf_rn(HsT[j * 33 + lane], __shfl_sync(0xffffffffu, d, j), v);
            g[col] = v;
            cs[col] = (uint8_t)code;
            const Move m = warp_best(element_best(code, v, HsT[lane * 33 + lane], s2e, (int)col));
            if (lane == 0) {
                bgain[k] = m.gain;
                bidx[k] = m.idx;
            }
        }
        if (!active)
            continue;
        __syncwarp();
        // ---- greedy moves
        int n = 0;
        for (; n < max_moves; ++n) {
            Move m{0.0f, 0x7FFFFFFF};
            for (int64_t k = lane; k < kb; k += 32)
                if (better(bgain[k], bidx[k], m.gain, m.idx)) {
                    m.gain = bgain[k];
                    m.idx = bidx[k];
                }
            m = warp_best(m);
            if (!(m.gain > 0.0f))
                break;
            const int elem = m.idx >> 1;
            const int k = elem >> 5;
            const int i = elem & 31;
            const int e = (int)scales[r * kb + k] - 127;
            const float s2e = flip_pow2(e);
            const uint32_t old = cs[elem];
            const uint32_t nc = flip_code_of_level(flip_level(old) + ((m.idx & 1) ? 1 : -1));
            const float D = __fmul_rn(__fsub_rn(flip_value(nc), flip_value(old)), s2e);
            __syncwarp();   // every lane has read the old code and the cached moves
            if (lane == i)
                cs[elem] = (uint8_t)nc;
            const int64_t col = (int64_t)k * 32 + lane;
            const float gj = __fmaf_rn(-D, __ldg(hess + (int64_t)k * 1024 + lane * 32 + i), g[col]);
            g[col] = gj;
            const uint32_t cj = lane == i ? nc : (uint32_t)cs[col];
            const Move b = warp_best(element_best(cj, gj, diag[col], s2e, (int)col));
            if (lane == 0) {
                bgain[k] = b.gain;
                bidx[k] = b.idx;
            }
            __syncwarp();
        }
        // ---- codes back, two per byte
        for (int64_t j = lane; j < cols / 2; j += 32)
            codes[r * (cols / 2) + j] = (uint8_t)(cs[2 * j] | (cs[2 * j + 1] << 4));
        if (moves && lane == 0)
            moves[r] = n;
        __syncwarp();
    }
}

}  // namespace

size_t flip_refine_smem_bytes(int64_t cols)
{
    const int64_t kb = cols / 32;
    return (size_t)(32 * 33 + cols) * sizeof(float) + (size_t)kFlipWarps * ((size_t)cols * 5 + (size_t)kb * 8);
}

cudaError_t launch_mxfp4_flip_refine(const void* w, int dtype, int64_t rows, int64_t cols,
                                     const float* tinv, int hadamard, const float* hess, int max_moves,
                                     uint8_t* codes, const uint8_t* scales, int32_t* moves, cudaStream_t s)
{
    const size_t smem = flip_refine_smem_bytes(cols);
    int64_t ctas = (rows + kFlipWarps - 1) / kFlipWarps;
    const int64_t cap = (int64_t)num_sms() * 2;
    ctas = ctas < cap ? ctas : cap;
    if (dtype == 1) {
        auto k = flip_refine_kernel<__nv_bfloat16>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        k<<<(unsigned)ctas, kFlipThreads, smem, s>>>(reinterpret_cast<const __nv_bfloat16*>(w), rows, cols, tinv,
                                                      hadamard, hess, max_moves, codes, scales, moves);
    } else {
        auto k = flip_refine_kernel<float>;
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess)
            return e;
        k<<<(unsigned)ctas, kFlipThreads, smem, s>>>(reinterpret_cast<const float*>(w), rows, cols, tinv, hadamard,
                                                      hess, max_moves, codes, scales, moves);
    }
    return cudaGetLastError();
}

}  // namespace fp4q
