// flip_mxfp4.cu -- Flip-Refinement of MXFP4 weight codes ("MACaQ: Fast, Model
// Agnostic Calibrated Quantization ..." review, section 1 Key Terms and
// section 3 Method): starting from the round-to-nearest codes at the chosen
// block exponents, each output row repeatedly takes the single move of one
// code to a neighbouring E2M1 level with the largest closed-form decrease of
// sum_k d_k^T H'_k d_k (d = u - deq), updating the block gradient g = H'd
// incrementally, until no move gains or the row's move budget is spent.
//
// H' is block-diagonal, so a move changes only its own block's gradient and
// candidates: every block, on its own, produces a fixed sequence of "best
// move after t of its moves", and the row's greedy is the merge of its
// blocks' sequences that always takes the largest head.  Three launches:
//  1. flip_blocks_kernel: per (row, block), one warp runs the block's own
//     greedy for up to kSeq moves (H'_k staged once per CTA in shared memory)
//     and stores the heads -- the block's best move after 0..kSeq moves;
//  2. flip_merge_kernel: per row, one warp merges its blocks' heads (lane l
//     owns blocks l, l+32, ...), takes at most max_moves of them, and applies
//     the taken prefixes to the codes.  A row that would take a block's move
//     beyond the stored heads is put on a list instead;
//  3. flip_refine_kernel: rows on the list run the direct greedy: one warp
//     per row, the row's gradient and codes in shared memory, per-block best
//     moves cached so a step re-scores only the block it changed.
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

// Lane j's element of block k of row r: its current code, the block's 2^e,
// and the gradient g_j = sum_i H_ji d_i of the block (an fma chain over i in
// order).  HsT holds H'_k transposed with padded rows: HsT[c * 33 + r] = H[r][c].
template <typename T>
__device__ __forceinline__ void block_state(const T* __restrict__ w, int64_t r, int64_t cols, int64_t k,
                                            const float* __restrict__ tinv, int had,
                                            const uint8_t* __restrict__ codes,
                                            const uint8_t* __restrict__ scales, const float* HsT, int lane,
                                            uint32_t& code, float& g, float& s2e)
{
    const int64_t kb = cols / 32;
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
        u = __fmul_rn(u, __uint_as_float(0x3E3504F3u));
    }
    const uint8_t byte = codes[(r * cols + col) >> 1];
    code = (col & 1) ? (uint32_t)(byte >> 4) : (uint32_t)(byte & 15u);
    s2e = flip_pow2((int)scales[r * kb + k] - 127);
    const float d = __fsub_rn(u, __fmul_rn(flip_value(code), s2e));
    float v = 0.0f;
#pragma unroll
    for (int j = 0; j < 32; ++j)
        v = __fmaf_rn(HsT[j * 33 + lane], __shfl_sync(0xffffffffu, d, j), v);
    g = v;
}

__device__ __forceinline__ void stage_hess_block(const float* __restrict__ hess, int64_t k, float* HsT)
{
    for (int q = threadIdx.x; q < 1024; q += blockDim.x)
        HsT[(q & 31) * 33 + (q >> 5)] = __ldg(hess + k * 1024 + q);
}

// ------------------------------------------------------ 1: block sequences
constexpr int kSeq = 15;            // moves precomputed per block; heads 0..kSeq stored
constexpr int kBlocksWarps = 8;

__device__ __forceinline__ uint2 pack_move(const Move& m)
{
    return m.gain > 0.0f ? make_uint2(__float_as_uint(m.gain), (uint32_t)m.idx) : make_uint2(0u, 0xFFFFFFFFu);
}

template <typename T>
__global__ void __launch_bounds__(32 * kBlocksWarps)
flip_blocks_kernel(const T* __restrict__ w, int64_t rows, int64_t cols, const float* __restrict__ tinv, int had,
                   const float* __restrict__ hess, const uint8_t* __restrict__ codes,
                   const uint8_t* __restrict__ scales, uint2* __restrict__ heads, int32_t* __restrict__ fb_count)
{
    __shared__ float HsT[32 * 33];
    const int64_t kb = cols / 32;
    const int64_t k = blockIdx.x;
    if (k == 0 && blockIdx.y == 0 && threadIdx.x == 0)
        *fb_count = 0;
    stage_hess_block(hess, k, HsT);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int wid = threadIdx.x >> 5;
    const float Hjj = HsT[lane * 33 + lane];
    const int elem = (int)k * 32 + lane;
    for (int64_t r = (int64_t)blockIdx.y * kBlocksWarps + wid; r < rows; r += (int64_t)gridDim.y * kBlocksWarps) {
        uint32_t code;
        float g, s2e;
        block_state<T>(w, r, cols, k, tinv, had, codes, scales, HsT, lane, code, g, s2e);
        uint2* out = heads + (r * kb + k) * (kSeq + 1);
        for (int t = 0; t <= kSeq; ++t) {
            const Move m = warp_best(element_best(code, g, Hjj, s2e, elem));
            if (lane == 0)
                out[t] = pack_move(m);
            if (!(m.gain > 0.0f) || t == kSeq)
                break;
            // apply the block's own best move
            const int i = (m.idx >> 1) & 31;
            const uint32_t oldc = __shfl_sync(0xffffffffu, code, i);
            const uint32_t nc = flip_code_of_level(flip_level(oldc) + ((m.idx & 1) ? 1 : -1));
            const float D = __fmul_rn(__fsub_rn(flip_value(nc), flip_value(oldc)), s2e);
            if (lane == i)
                code = nc;
            g = __fmaf_rn(-D, HsT[i * 33 + lane], g);
        }
    }
}

// ------------------------------------------------------------- 2: merge
// LB = blocks per lane (ceil(kb / 32)).
template <int LB>
__global__ void __launch_bounds__(128)
flip_merge_kernel(int64_t rows, int64_t kb, int max_moves, const uint2* __restrict__ heads,
                  uint8_t* __restrict__ codes, int32_t* __restrict__ moves, int32_t* __restrict__ fb_list,
                  int32_t* __restrict__ fb_count)
{
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t r = warp0; r < rows; r += nwarps) {
        uint2 cur[LB], nxt[LB];
        int p[LB];
#pragma unroll
        for (int q = 0; q < LB; ++q) {
            const int64_t k = lane + 32 * q;
            p[q] = 0;
            cur[q] = make_uint2(0u, 0xFFFFFFFFu);
            nxt[q] = make_uint2(0u, 0xFFFFFFFFu);
            if (k < kb) {
                const uint2* hb = heads + (r * kb + k) * (kSeq + 1);
                cur[q] = hb[0];
                if (cur[q].y != 0xFFFFFFFFu)
                    nxt[q] = hb[1];
            }
        }
        int n = 0;
        bool overflow = false;
        for (; n < max_moves; ++n) {
            Move m{0.0f, 0x7FFFFFFF};
#pragma unroll
            for (int q = 0; q < LB; ++q) {
                const float gq = __uint_as_float(cur[q].x);
                const int iq = (int)cur[q].y;
                if (cur[q].y != 0xFFFFFFFFu && better(gq, iq, m.gain, m.idx)) {
                    m.gain = gq;
                    m.idx = iq;
                }
            }
            m = warp_best(m);
            if (!(m.gain > 0.0f))
                break;
            const int kw = (m.idx >> 1) >> 5;
            bool ovf = false;
            if ((kw & 31) == lane) {
#pragma unroll
                for (int q = 0; q < LB; ++q) {
                    if (q == (kw >> 5)) {
                        ++p[q];
                        if (p[q] > kSeq) {
                            ovf = true;   // the next head was not precomputed
                        } else {
                            cur[q] = nxt[q];
                            nxt[q] = make_uint2(0u, 0xFFFFFFFFu);
                            if (cur[q].y != 0xFFFFFFFFu && p[q] + 1 <= kSeq)
                                nxt[q] = heads[(r * kb + kw) * (kSeq + 1) + p[q] + 1];
                        }
                    }
                }
            }
            if (__any_sync(0xffffffffu, ovf)) {
                overflow = true;
                break;
            }
        }
        if (overflow) {
            if (lane == 0)
                fb_list[atomicAdd(fb_count, 1)] = (int32_t)r;
            continue;
        }
        // apply each block's taken prefix of moves
#pragma unroll
        for (int q = 0; q < LB; ++q) {
            const int64_t k = lane + 32 * q;
            if (k >= kb || p[q] == 0)
                continue;
            uint4* cp = reinterpret_cast<uint4*>(codes + (r * kb + k) * 16);
            uint4 v = *cp;
            const uint2* hb = heads + (r * kb + k) * (kSeq + 1);
            for (int t = 0; t < p[q]; ++t) {
                const uint32_t idx = hb[t].y;
                const uint32_t i = (idx >> 1) & 31u;
                const uint32_t sh = 4u * (i & 7u);
                const uint32_t word = i >> 3;
                const uint32_t cur_w = word == 0u ? v.x : word == 1u ? v.y : word == 2u ? v.z : v.w;
                const uint32_t oldc = (cur_w >> sh) & 15u;
                const uint32_t nc = flip_code_of_level(flip_level(oldc) + ((idx & 1u) ? 1 : -1));
                const uint32_t upd = (cur_w & ~(15u << sh)) | (nc << sh);
                v.x = word == 0u ? upd : v.x;
                v.y = word == 1u ? upd : v.y;
                v.z = word == 2u ? upd : v.z;
                v.w = word == 3u ? upd : v.w;
            }
            *cp = v;
        }
        if (moves && lane == 0)
            moves[r] = n;
    }
}

// -------------------------------------------- 3: direct greedy (list rows)
template <typename T>
__global__ void __launch_bounds__(kFlipThreads)
flip_refine_kernel(const T* __restrict__ w, int64_t cols, const float* __restrict__ tinv, int had,
                   const float* __restrict__ hess, int max_moves, uint8_t* __restrict__ codes,
                   const uint8_t* __restrict__ scales, int32_t* __restrict__ moves,
                   const int32_t* __restrict__ row_list, const int32_t* __restrict__ row_count)
{
    const int64_t nlist = *row_count;
    if ((int64_t)blockIdx.x * kFlipWarps >= nlist)
        return;
    extern __shared__ __align__(16) uint8_t flip_smem[];
    const int64_t kb = cols / 32;
    // CTA: H'_k transposed with padded rows, the diagonal of every block;
    // per warp: g, codes, per-block best move
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

    for (int64_t l0 = (int64_t)blockIdx.x * kFlipWarps; l0 < nlist; l0 += (int64_t)gridDim.x * kFlipWarps) {
        const bool active = l0 + wid < nlist;
        const int64_t r = active ? (int64_t)row_list[l0 + wid] : 0;
        // ---- gradients and per-block best moves of the CTA's rows
        for (int64_t k = 0; k < kb; ++k) {
            __syncthreads();   // the previous block's H'_k is no longer read
            stage_hess_block(hess, k, HsT);
            __syncthreads();
            if (!active)
                continue;
            uint32_t code;
            float v, s2e;
            block_state<T>(w, r, cols, k, tinv, had, codes, scales, HsT, lane, code, v, s2e);
            const int64_t col = k * 32 + lane;
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
            const float s2e = flip_pow2((int)scales[r * kb + k] - 127);
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

// Opt the direct-greedy kernel into its largest shared-memory footprint
// (8192 columns) once per device.
cudaError_t flip_refine_opt_in()
{
    const int smem = (int)flip_refine_smem_bytes(8192);
    cudaError_t e = smem_opt_in((const void*)flip_refine_kernel<__nv_bfloat16>, smem);
    if (e == cudaSuccess)
        e = smem_opt_in((const void*)flip_refine_kernel<float>, smem);
    return e;
}

size_t flip_refine_ws_bytes(int64_t rows, int64_t cols)
{
    const int64_t kb = cols / 32;
    const size_t list = ((size_t)rows * sizeof(int32_t) + 15) / 16 * 16;
    return 16 + list + (size_t)rows * (size_t)kb * (kSeq + 1) * sizeof(uint2);
}

cudaError_t launch_mxfp4_flip_refine(const void* w, int dtype, int64_t rows, int64_t cols,
                                     const float* tinv, int hadamard, const float* hess, int max_moves,
                                     uint8_t* codes, const uint8_t* scales, int32_t* moves, void* ws,
                                     cudaStream_t s)
{
    const int64_t kb = cols / 32;
    uint8_t* wsb = static_cast<uint8_t*>(ws);
    int32_t* fb_count = reinterpret_cast<int32_t*>(wsb);
    int32_t* fb_list = reinterpret_cast<int32_t*>(wsb + 16);
    uint2* heads = reinterpret_cast<uint2*>(wsb + 16 + ((size_t)rows * sizeof(int32_t) + 15) / 16 * 16);
    // 1: block sequences
    const int64_t ychunks = (rows + 8 * kBlocksWarps - 1) / (8 * kBlocksWarps);
    dim3 g1((unsigned)kb, (unsigned)(ychunks < 65535 ? ychunks : 65535));
    if (dtype == 1)
        flip_blocks_kernel<__nv_bfloat16><<<g1, 32 * kBlocksWarps, 0, s>>>(
            reinterpret_cast<const __nv_bfloat16*>(w), rows, cols, tinv, hadamard, hess, codes, scales, heads,
            fb_count);
    else
        flip_blocks_kernel<float><<<g1, 32 * kBlocksWarps, 0, s>>>(reinterpret_cast<const float*>(w), rows, cols,
                                                                    tinv, hadamard, hess, codes, scales, heads,
                                                                    fb_count);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    // 2: merge
    const unsigned g2 = (unsigned)((rows + 3) / 4);
    const int lb = (int)((kb + 31) / 32);
#define FP4Q_FLIP_MERGE(LBV)                                                                              \
    flip_merge_kernel<LBV><<<g2, 128, 0, s>>>(rows, kb, max_moves, heads, codes, moves, fb_list, fb_count)
    switch (lb) {
    case 1: FP4Q_FLIP_MERGE(1); break;
    case 2: FP4Q_FLIP_MERGE(2); break;
    case 3: FP4Q_FLIP_MERGE(3); break;
    case 4: FP4Q_FLIP_MERGE(4); break;
    case 5: FP4Q_FLIP_MERGE(5); break;
    case 6: FP4Q_FLIP_MERGE(6); break;
    case 7: FP4Q_FLIP_MERGE(7); break;
    case 8: FP4Q_FLIP_MERGE(8); break;
    default: return cudaErrorInvalidValue;
    }
#undef FP4Q_FLIP_MERGE
    e = cudaGetLastError();
    if (e != cudaSuccess)
        return e;
    // 3: rows whose merge ran past a block's precomputed moves
    const size_t smem = flip_refine_smem_bytes(cols);
    int64_t ctas = (rows + kFlipWarps - 1) / kFlipWarps;
    const int64_t cap = (int64_t)num_sms() * 2;
    ctas = ctas < cap ? ctas : cap;
    // the shared-memory opt-in is set once per device for the largest width
    e = flip_refine_opt_in();
    if (e != cudaSuccess)
        return e;
    if (dtype == 1)
        flip_refine_kernel<__nv_bfloat16><<<(unsigned)ctas, kFlipThreads, smem, s>>>(
            reinterpret_cast<const __nv_bfloat16*>(w), cols, tinv, hadamard, hess, max_moves, codes, scales, moves,
            fb_list, fb_count);
    else
        flip_refine_kernel<float><<<(unsigned)ctas, kFlipThreads, smem, s>>>(
            reinterpret_cast<const float*>(w), cols, tinv, hadamard, hess, max_moves, codes, scales, moves, fb_list,
            fb_count);
    return cudaGetLastError();
}

}  // namespace fp4q
