// gemm_w4a4.cu -- NVFP4 W4A4 GEMM on the 5th-generation tensor cores.
//
// out[m][n] = bf16( g_a * g_w * sum_k (v_a[m][k] * sc_a[m][k/16]) * (v_w[n][k] * sc_w[n][k/16]) )
// i.e. A . W^T with both operands NVFP4 (E2M1 codes, one E4M3 scale per 16
// elements along K, an FP32 global scale each): the W4A4 inference of the
// "Why Gated DeltaNet Survives 4-Bit Quantization" review, section 1.
//
// Kernel shape (one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0     TMA producer: FP4 code tiles (128B-swizzled, K-major) by
//              cp.async.bulk.tensor, scale-factor atoms (512 contiguous bytes
//              each, already in the MMA layout) by cp.async.bulk
//   warp 1     TMEM owner + MMA issuer: tcgen05.cp moves the scale atoms into
//              TMEM, tcgen05.mma.kind::mxf4nvf4.block_scale.block16 (M=128,
//              N=256, K=64) accumulates in TMEM, tcgen05.commit frees stages
//   warps 2-5  epilogue: tcgen05.ld of the fp32 accumulator, x g_a g_w,
//              round to bf16, 64-byte row stores
// Stages: 4 x (A 16 KiB + B 32 KiB + SFA 2 KiB + SFB 4 KiB).  TMEM: 256
// accumulator columns + 48 scale columns per stage.
//
// Every mbarrier wait is bounded in time.  A wait that gives up sets the
// error word in the workspace and a shared abort flag; all roles leave their
// loops, wait (bounded) for their own copies and MMAs, and the TMEM is
// released before the CTA exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cstdint>
#include <mutex>

#include "fp4q_device.cuh"
#include "fp4q_internal.h"

namespace fp4q {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 256;                       // K elements per stage (128 bytes per row)
constexpr int kStages = 4;
constexpr int kAStage = kBM * kBK / 2;         // 16 KiB
constexpr int kBStage = kBN * kBK / 2;         // 32 KiB
constexpr int kSfaStage = kBM * kBK / 16;      // 2 KiB (4 atoms of 512 B)
constexpr int kSfbStage = kBN * kBK / 16;      // 4 KiB (2 row atoms x 4)
constexpr int kStageBytes = kAStage + kBStage + kSfaStage + kSfbStage;
constexpr int kBarBytes = 256;
constexpr int kSmemBytes = kStages * kStageBytes + 1024 + kBarBytes;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol0 = 256;              // accumulator uses columns [0, 256)
constexpr uint32_t kSfColsPerStage = 48;       // SFA 4 k-steps x 4 + SFB 4 k-steps x 8
constexpr long long kWaitCycles = 4000000000LL;   // about 2 s at the boost clock

static_assert(kStageBytes % 1024 == 0, "stage bases must keep the 1024-byte swizzle alignment");
static_assert(kSfCol0 + kStages * kSfColsPerStage <= kTmemCols, "TMEM budget");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Block-scaled instruction descriptor: A and B E2M1 (format 1 of the
// mxf4nvf4 kind), K-major, UE4M3 scales, N = 256, M = 128, dense K = 64.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(kBN >> 3) << 17) |
                            ((uint32_t)(kBM >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok)
                 : "r"(bar), "r"(parity)
                 : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity; false if it did not complete in time.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const long long t0 = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - t0 > kWaitCycles)
            return false;
    }
    return true;
}

// ---------------------------------------------------------------- copies
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y,
                                            uint32_t bar)
{
    asm volatile("cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
                 " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
                 : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// Copy one 512-byte scale atom (32 rows x 16 bytes in shared memory) into 4
// TMEM columns, replicated into the four 32-lane quarters.
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t tacc, uint64_t da, uint64_t db, uint32_t idesc,
                                       uint32_t accumulate, uint32_t tsfa, uint32_t tsfb)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(tacc),
                 "l"(da), "l"(db), "r"(idesc), "r"(accumulate), "r"(tsfa), "r"(tsfb)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                 "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                 "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
                   "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
                   "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
                   "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
                   "=r"(r[31])
                 : "r"(taddr)
                 : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, K-major, 128-byte swizzle: 8-row groups
// 1024 bytes apart (leading offset unused, encoded 1), sm100 version 1.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Descriptor of a scale atom for tcgen05.cp: 32 rows of 16 bytes, no
// swizzle, 8-row core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t sdesc_sf(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

struct GemmParams {
    const uint8_t* sfa;       // A scales, MMA layout
    const uint8_t* sfb;       // W scales, MMA layout
    const float* ga;          // A global scale (device)
    const float* gw;          // W global scale (device)
    __nv_bfloat16* out;       // M x N row-major
    int* err;                 // error word (workspace)
    int tiles_m, tiles_n, kblocks, kb_atoms, N;
};

__global__ void __launch_bounds__(kThreads, 1)
w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const GemmParams p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
    // bars[0, S) full, [S, 2S) empty, 2S acc_full, 2S+1 acc_empty, 2S+2 drain
    uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 3);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t bar0 = smem_u32(bars);
    auto full_bar = [&](int s) { return bar0 + 8u * (uint32_t)s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (uint32_t)(kStages + s); };
    const uint32_t acc_full = bar0 + 8u * (2 * kStages);
    const uint32_t acc_empty = bar0 + 8u * (2 * kStages + 1);
    const uint32_t drain = bar0 + 8u * (2 * kStages + 2);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 128);
        mbar_init(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    const int num_tiles = p.tiles_m * p.tiles_n;

    auto give_up = [&]() {
        *abort_flag = 1;
        atomicExch(p.err, 1);
    };

    if (warp == 0) {
        if (lane == 0) {
            // ------------------------------------------------ producer
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0, issued_parity = 0;   // per-stage bit sets
            for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x) {
                const int mt = tile % p.tiles_m;
                const int nt = tile / p.tiles_m;
                for (int kb = 0; kb < p.kblocks; ++kb) {
                    if (!mbar_wait(empty_bar(stage), phase ^ 1u) || *abort_flag) {
                        give_up();
                        break;
                    }
                    const uint32_t fb = full_bar(stage);
                    mbar_expect_tx(fb, kStageBytes);
                    uint8_t* st = smem + stage * kStageBytes;
                    tma_load_2d(smem_u32(st), &tmA, kb * (kBK / 2), mt * kBM, fb);
                    tma_load_2d(smem_u32(st + kAStage), &tmB, kb * (kBK / 2), nt * kBN, fb);
                    const uint8_t* sa = p.sfa + ((int64_t)mt * p.kb_atoms + (int64_t)kb * 4) * 512;
                    const uint8_t* sb0 = p.sfb + ((int64_t)(2 * nt) * p.kb_atoms + (int64_t)kb * 4) * 512;
                    const uint8_t* sb1 = p.sfb + ((int64_t)(2 * nt + 1) * p.kb_atoms + (int64_t)kb * 4) * 512;
                    bulk_load(smem_u32(st + kAStage + kBStage), sa, kSfaStage, fb);
                    bulk_load(smem_u32(st + kAStage + kBStage + kSfaStage), sb0, kSfbStage / 2, fb);
                    bulk_load(smem_u32(st + kAStage + kBStage + kSfaStage + kSfbStage / 2), sb1,
                              kSfbStage / 2, fb);
                    issued |= 1u << stage;
                    issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (*abort_flag) {
                // let the copies this thread started land before the CTA exits
                for (int s = 0; s < kStages; ++s)
                    if (issued & (1u << s))
                        mbar_wait(full_bar(s), (issued_parity >> s) & 1u);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------ MMA issuer
            int stage = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool issued_any = false;
            for (int tile = blockIdx.x; tile < num_tiles && !*abort_flag; tile += gridDim.x) {
                if (!mbar_wait(acc_empty, acc_phase ^ 1u) || *abort_flag) {
                    give_up();
                    break;
                }
                tc_fence_after();
                bool ok = true;
                for (int kb = 0; kb < p.kblocks; ++kb) {
                    if (!mbar_wait(full_bar(stage), phase) || *abort_flag) {
                        give_up();
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    uint8_t* st = smem + stage * kStageBytes;
                    const uint32_t sa_s = smem_u32(st + kAStage + kBStage);
                    const uint32_t sb_s = sa_s + kSfaStage;
                    const uint32_t tsfa = tmem + kSfCol0 + (uint32_t)stage * kSfColsPerStage;
                    const uint32_t tsfb = tsfa + 16;
#pragma unroll
                    for (int s = 0; s < 4; ++s) {
                        tc_cp_sf(tsfa + 4 * s, sdesc_sf(sa_s + 512 * s));
                        tc_cp_sf(tsfb + 8 * s, sdesc_sf(sb_s + 512 * s));
                        tc_cp_sf(tsfb + 8 * s + 4, sdesc_sf(sb_s + kSfbStage / 2 + 512 * s));
                    }
                    const uint32_t a_s = smem_u32(st);
                    const uint32_t b_s = a_s + kAStage;
#pragma unroll
                    for (int s = 0; s < 4; ++s)
                        tc_mma(tmem, sdesc_sw128(a_s + 32 * s), sdesc_sw128(b_s + 32 * s), kIdesc,
                               (kb | s) != 0, tsfa + 4 * s, tsfb + 8 * s);
                    issued_any = true;
                    tc_commit(empty_bar(stage));
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok)
                    break;
                tc_commit(acc_full);
                acc_phase ^= 1u;
            }
            if (issued_any) {
                // every MMA and copy this thread issued has finished once this arrives
                tc_commit(drain);
                if (!mbar_wait(drain, 0))
                    give_up();
            }
        }
    } else {
        // ---------------------------------------------------- epilogue
        const int q = warp & 3;                      // TMEM lane quarter of this warp
        uint32_t acc_phase = 0;
        const float scale = __fmul_rn(__ldg(p.ga), __ldg(p.gw));
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
            bool ok = !*abort_flag && mbar_wait(acc_full, acc_phase);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) {
                if (lane == 0)
                    give_up();
                break;
            }
            tc_fence_after();
            const int mt = tile % p.tiles_m;
            const int nt = tile / p.tiles_m;
            const int64_t row = (int64_t)mt * kBM + q * 32 + lane;
            __nv_bfloat16* orow = p.out + row * p.N + (int64_t)nt * kBN;
            const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
#pragma unroll 1
            for (int c = 0; c < kBN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tq + 32 * c, r);
                uint32_t pk[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    __nv_bfloat162 h = __floats2bfloat162_rn(__fmul_rn(__uint_as_float(r[2 * j]), scale),
                                                             __fmul_rn(__uint_as_float(r[2 * j + 1]), scale));
                    pk[j] = *reinterpret_cast<uint32_t*>(&h);
                }
                uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    dst[j] = make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
            }
            tc_fence_before();
            mbar_arrive(acc_empty);
            acc_phase ^= 1u;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
}

// ------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// 2-D map over packed codes: rows x (K/2) bytes, box box_rows x 128 bytes, 128B swizzle.
bool make_code_map(CUtensorMap* m, const void* base, int64_t rows, int64_t kbytes, int box_rows)
{
    auto fn = encode_fn();
    if (!fn)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)kbytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)kbytes};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool gemm_shape_supported(int64_t M, int64_t N, int64_t K)
{
    return M > 0 && N > 0 && K > 0 && M % kBM == 0 && N % kBN == 0 && K % kBK == 0 && M / kBM < (1 << 30) &&
           N / kBN < (1 << 20);
}

cudaError_t launch_w4a4_gemm(const uint8_t* a_codes, const uint8_t* a_sf, const float* ga,
                             const uint8_t* w_codes, const uint8_t* w_sf, const float* gw, int64_t M,
                             int64_t N, int64_t K, void* out, int* err, cudaStream_t s)
{
    CUtensorMap ta, tb;
    if (!make_code_map(&ta, a_codes, M, K / 2, kBM) || !make_code_map(&tb, w_codes, N, K / 2, kBN))
        return cudaErrorInvalidValue;
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(w4a4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        kSmemBytes);
    });
    if (attr_err != cudaSuccess)
        return attr_err;
    GemmParams p;
    p.sfa = a_sf;
    p.sfb = w_sf;
    p.ga = ga;
    p.gw = gw;
    p.out = reinterpret_cast<__nv_bfloat16*>(out);
    p.err = err;
    p.tiles_m = (int)(M / kBM);
    p.tiles_n = (int)(N / kBN);
    p.kblocks = (int)(K / kBK);
    p.kb_atoms = (int)(K / 64);
    p.N = (int)N;
    const int tiles = p.tiles_m * p.tiles_n;
    const int grid = tiles < num_sms() ? tiles : num_sms();
    w4a4_gemm_kernel<<<grid, kThreads, kSmemBytes, s>>>(ta, tb, p);
    return cudaGetLastError();
}

}  // namespace fp4q
