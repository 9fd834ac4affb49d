// gemm_operands.cu -- operand preparation for the tensor-core GEMM.
//
// (1) Scale bytes from the row-major layout to the tcgen05 scale layout
// (for operands quantized row-major, e.g. MXFP4 weights after
// Flip-Refinement, which reads its exponents row-major).
//
// (2) RaZeR operands.  A RaZeR block ("RaZeR: Redundant Zero Remapping" summary, section 2.2)
// decodes its -0 code to the block's special value sv (a multiple of 0.5,
// section 2.2 value constraint) times the block scale; the tensor core decodes
// -0 as zero.  The summary's Blackwell kernels handle the remapping in two
// passes on the existing tensor cores (section 2.3).  Here the two passes are
// two E2M1 tensors with the same block scales: every special value the
// quantizer offers is a sum p + q of two E2M1 values (+-5 = +-(4 + 1),
// +-3.5 = +-(3 + 0.5)), so
//   main  = the codes with every -0 replaced by p of the block's selector,
//   extra = q at the -0 positions and +0 elsewhere,
// and main + extra reproduces the RaZeR values exactly.  The GEMM multiplies
// both tensors into one accumulator.  The block scale moves to an E4M3 byte
// (every E3M3 value is an E4M3 value) in the tcgen05 scale layout.
#include <cstdint>

#include "fp4q_device.cuh"
#include "fp4q_internal.h"

namespace fp4q {

namespace {

constexpr int kPrepThreads = 256;

struct PqTable {
    uint32_t p[4], q[4];
};

// One thread per 16-element block.
template <int SF>
__global__ void __launch_bounds__(kPrepThreads)
razer_prepare_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ meta, int64_t nblk,
                     int64_t bpr, PqTable pq, uint8_t* __restrict__ main_codes,
                     uint8_t* __restrict__ extra_codes, uint8_t* __restrict__ scales_mma)
{
    const int64_t kb_atoms = bpr >> 2;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += stride) {
        const uint2 w = __ldg(reinterpret_cast<const uint2*>(codes + b * 8));
        const uint32_t m = __ldg(meta + b);
        const uint32_t sel = SF == 1 ? m >> 6 : m >> 7;
        const uint32_t sc = SF == 1 ? m & 0x3Fu : m & 0x7Fu;
        // E3M3 -> E4M3: normal codes shift by 32 exponent steps; the eight
        // subnormals k * 2^-5 are E4M3 normals (exact, so the encode is too)
        const uint32_t e4 = SF == 1 ? (sc < 8u ? e4m3_encode(__fmul_rn((float)sc, 0.03125f)) : sc + 32u) : sc;
        const uint32_t p = sel == 0u ? pq.p[0] : sel == 1u ? pq.p[1] : sel == 2u ? pq.p[2] : pq.p[3];
        const uint32_t q = sel == 0u ? pq.q[0] : sel == 1u ? pq.q[1] : sel == 2u ? pq.q[2] : pq.q[3];
        uint32_t mo[2], eo[2];
        const uint32_t ww[2] = {w.x, w.y};
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            // nibbles equal to 8 (-0): t has a zero nibble exactly there
            const uint32_t t = ww[j] ^ 0x88888888u;
            const uint32_t nonzero = (((t & 0x77777777u) + 0x77777777u) | t) & 0x88888888u;
            const uint32_t ones = (~nonzero & 0x88888888u) >> 3;   // 1 in each -0 nibble
            mo[j] = (ww[j] & ~(ones * 0xFu)) | (ones * p);
            eo[j] = ones * q;
        }
        *reinterpret_cast<uint2*>(main_codes + b * 8) = make_uint2(mo[0], mo[1]);
        *reinterpret_cast<uint2*>(extra_codes + b * 8) = make_uint2(eo[0], eo[1]);
        const int64_t r = b / bpr;
        scales_mma[mma_sf_offset(r, b - r * bpr, kb_atoms)] = (uint8_t)e4;
    }
}

// One thread per 4 scale bytes of a row (one 32-bit word of an atom row).
__global__ void __launch_bounds__(kPrepThreads)
scales_to_mma_kernel(const uint8_t* __restrict__ scales, int64_t rows, int64_t nscales,
                     uint8_t* __restrict__ out)
{
    const int64_t words = nscales >> 2;
    const int64_t n = rows * words;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
        const int64_t r = i / words;
        const int64_t c = (i - r * words) * 4;
        const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(scales + r * nscales + c));
        *reinterpret_cast<uint32_t*>(out + mma_sf_offset(r, c, words)) = v;
    }
}

}  // namespace

cudaError_t launch_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t nscales, uint8_t* out,
                                 cudaStream_t s)
{
    const int64_t n = rows * (nscales / 4);
    int64_t want = (n + kPrepThreads - 1) / kPrepThreads;
    const int64_t cap = (int64_t)num_sms() * 8;
    const int grid = (int)(want < 1 ? 1 : (want > cap ? cap : want));
    scales_to_mma_kernel<<<grid, kPrepThreads, 0, s>>>(scales, rows, nscales, out);
    return cudaGetLastError();
}

cudaError_t launch_razer_gemm_prepare(const uint8_t* codes, const uint8_t* meta, int64_t rows,
                                      int64_t cols, int sf, const uint8_t* p_code,
                                      const uint8_t* q_code, uint8_t* main_codes,
                                      uint8_t* extra_codes, uint8_t* scales_mma, cudaStream_t s)
{
    PqTable pq;
    for (int i = 0; i < 4; ++i) {
        pq.p[i] = p_code[i] & 0xFu;
        pq.q[i] = q_code[i] & 0xFu;
    }
    const int64_t bpr = cols / 16;
    const int64_t nblk = rows * bpr;
    int64_t want = (nblk + kPrepThreads - 1) / kPrepThreads;
    const int64_t cap = (int64_t)num_sms() * 8;
    const int grid = (int)(want < 1 ? 1 : (want > cap ? cap : want));
    if (sf == 1)
        razer_prepare_kernel<1><<<grid, kPrepThreads, 0, s>>>(codes, meta, nblk, bpr, pq, main_codes,
                                                             extra_codes, scales_mma);
    else
        razer_prepare_kernel<0><<<grid, kPrepThreads, 0, s>>>(codes, meta, nblk, bpr, pq, main_codes,
                                                             extra_codes, scales_mma);
    return cudaGetLastError();
}

}  // namespace fp4q
