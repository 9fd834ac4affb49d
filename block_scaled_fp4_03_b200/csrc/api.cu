// api.cu -- the C ABI declared in include/fp4q.h: argument checking on the
// host, then launches on the caller's stream.  No allocation, no state.
#include <cmath>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/fp4q.h"
#include "fp4q_internal.h"

using namespace fp4q;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned_or_null(const void* p) { return p == nullptr || aligned16(p); }
bool valid_block(int b) { return b == 4 || b == 8 || b == 16 || b == 32; }
bool valid_dtype(int d) { return d == FP4Q_F32 || d == FP4Q_BF16; }
cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

int from_cuda(cudaError_t e) { return e == cudaSuccess ? FP4Q_OK : FP4Q_ERR_CUDA; }

// Quantize workspace: [0, 4096) the partial maxima of a separate amax pass,
// FP4Q_WS_BF_EVALS the brute-force evaluation counter, kQuantCounter the
// fused amax's grid-barrier counter, [kQuantFused, +4 * kFusedMaxCtas) the
// fused amax's per-CTA maxima.
constexpr size_t kQuantWs = 8192;
constexpr size_t kQuantCounter = 3584;
constexpr size_t kQuantFused = 4096;
// Flip-Refinement: a row's state lives in shared memory (5 bytes per column
// per row, 4 rows per CTA), and a row's move budget is bounded
constexpr int64_t kFlipMaxCols = 8192;
constexpr int kFlipMaxMoves = 1 << 20;
// GEMM workspace: [0, 4096) amax partials, 4096 g_a, 4160 error word, then the
// quantized A (codes, then MMA-layout scales) from 8192 on.
constexpr size_t kGemmHeader = 8192;
constexpr size_t kGemmGa = 4096;
constexpr size_t kGemmErr = 4160;
constexpr size_t kGemmCounter = 4168;   // fused amax of the dense A: barrier counter
constexpr size_t kGemmFused = 4224;     // and per-CTA maxima
// Hessian workspace: [0, 256) header (error word at 0), then the partial sums.
constexpr size_t kHessHeader = 256;
bool valid_out_dtype(int d) { return d == FP4Q_BF16 || d == FP4Q_F32; }
size_t gemm_ws_bytes(int64_t M, int64_t K) { return kGemmHeader + (size_t)M * (size_t)K / 2 + (size_t)M * (size_t)K / 16; }
size_t mx_gemm_ws_bytes(int64_t M, int64_t K) { return kGemmHeader + (size_t)M * (size_t)K / 2 + (size_t)M * (size_t)K / 32; }
static_assert(kAmaxPartials * sizeof(float) <= FP4Q_WS_BF_EVALS && FP4Q_WS_BF_EVALS + 8 <= kQuantCounter &&
                  kQuantCounter + 4 <= kQuantFused && kQuantFused + 4 * kFusedMaxCtas <= kQuantWs,
              "quantize workspace regions must not overlap");
static_assert(kGemmErr + 4 <= kGemmCounter && kGemmCounter + 4 <= kGemmFused &&
                  kGemmFused + 4 * kFusedMaxCtas <= kGemmHeader,
              "GEMM workspace header regions must not overlap");

// A fused global amax (GsArgs mode 3) whose partials and barrier counter live
// in the workspace at the given offsets; the counter is cleared on `s`.
cudaError_t fused_gs(GsArgs& gs, const void* x, int64_t n, uint8_t* ws, size_t fused_off, size_t counter_off,
                     cudaStream_t s)
{
    gs.mode = 3;
    gs.x = x;
    gs.n = n;
    gs.fused_partials = reinterpret_cast<float*>(ws + fused_off);
    gs.counter = reinterpret_cast<unsigned int*>(ws + counter_off);
    gs.wait_limit = wait_limit_cycles();
    return cudaMemsetAsync(gs.counter, 0, sizeof(unsigned int), s);
}

// Run a quantizer launch; if its fused amax cannot be launched cooperatively
// here (the device holds fewer resident CTAs than its grid, e.g. when shared
// under MPS), or fp4q_debug_force_amax_pass asks for it, fall back to a
// separate amax pass whose partials go to ws[0, 4 * kAmaxPartials).
template <typename F>
cudaError_t launch_with_gs(GsArgs& gs, const void* x, int dtype, int64_t n, void* ws, cudaStream_t s, F&& launch)
{
    const bool forced = gs.mode == 3 && force_amax_pass();
    cudaError_t e = forced ? cudaErrorCooperativeLaunchTooLarge : launch(gs);
    if (e == cudaErrorCooperativeLaunchTooLarge && gs.mode == 3) {
        if (!forced)
            (void)cudaGetLastError();
        gs.mode = 1;
        gs.partials = reinterpret_cast<const float*>(ws);
        gs.n_partials = kAmaxPartials;
        e = launch_amax(x, dtype, n, reinterpret_cast<float*>(ws), s);
        if (e == cudaSuccess)
            e = launch(gs);
    }
    return e;
}

// Resolve a global-scale request into launch arguments (running the amax
// pre-pass for AMAX).  Returns FP4Q_OK or an error.
int prepare_gs(int gs_mode, float denom, const void* x, int dtype, int64_t n, float* global_scale,
               void* ws, size_t ws_bytes, cudaStream_t s, GsArgs& gs)
{
    gs = GsArgs{};
    gs.mode = gs_mode;
    gs.denom = denom;
    if (gs_mode == FP4Q_GS_NONE)
        return FP4Q_OK;
    if (gs_mode == FP4Q_GS_GIVEN) {
        if (!global_scale)
            return FP4Q_ERR_ARG;
        gs.given = global_scale;
        return FP4Q_OK;
    }
    if (gs_mode != FP4Q_GS_AMAX)
        return FP4Q_ERR_ARG;
    if (!ws || ws_bytes < kQuantWs)
        return FP4Q_ERR_WORKSPACE;
    if (!aligned16(ws))
        return FP4Q_ERR_ALIGN;
    gs.out = global_scale;
    return from_cuda(fused_gs(gs, x, n, static_cast<uint8_t*>(ws), kQuantFused, kQuantCounter, s));
}

}  // namespace

extern "C" {

size_t fp4q_workspace_size(int op, int64_t rows, int64_t cols, int64_t n)
{
    if (rows < 0 || cols < 0 || n < 0)
        return 0;
    switch (op) {
    case FP4Q_OP_QUANTIZE: return kQuantWs;
    case FP4Q_OP_FLIP: return (rows <= 0 || cols <= 0 || cols % 32) ? 0 : flip_refine_ws_bytes(rows, cols);
    case FP4Q_OP_HESSIAN: return cols % 32 ? 0 : kHessHeader + hessian_ws_bytes(rows, cols);
    case FP4Q_OP_CHANNEL_SCALE: return channel_scale_ws_bytes(rows, n, cols);
    case FP4Q_OP_GEMM: return gemm_ws_bytes(rows, cols);
    case FP4Q_OP_MX_GEMM: return mx_gemm_ws_bytes(rows, cols);
    default: return 0;
    }
}

const char* fp4q_status_str(int status)
{
    switch (status) {
    case FP4Q_OK: return "ok";
    case FP4Q_ERR_ARG: return "invalid argument";
    case FP4Q_ERR_ALIGN: return "misaligned pointer";
    case FP4Q_ERR_UNSUPPORTED: return "unsupported";
    case FP4Q_ERR_CUDA: return "CUDA error";
    case FP4Q_ERR_TIMEOUT: return "device wait timed out";
    case FP4Q_ERR_WORKSPACE: return "workspace missing or too small";
    case FP4Q_ERR_TOO_LARGE: return "problem exceeds the library's built-in scratch";
    default: return "unknown status";
    }
}

const char* fp4q_version(void) { return "fp4q 0.1.0 sm_100a"; }

int fp4_block_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int block, int rule,
                       int scale_fmt, int gs_mode, float* global_scale, uint8_t* codes,
                       uint8_t* scales, int sf_layout, float* dequant, float* block_mse,
                       void* workspace, size_t workspace_bytes, void* stream)
{
    if (scale_fmt != FP4Q_SF_E4M3 && scale_fmt != FP4Q_SF_UE5M3)
        return FP4Q_ERR_ARG;
    const bool ue5m3 = scale_fmt == FP4Q_SF_UE5M3;
    const bool empty = rows == 0 || cols == 0;   // empty tensors may come with NULL buffers
    if ((!empty && (!x || !codes || !scales)) || !valid_dtype(dtype) || rows < 0 || cols < 0)
        return FP4Q_ERR_ARG;
    if (!valid_block(block) || cols % block != 0)
        return FP4Q_ERR_ARG;
    if (rule < FP4Q_ABSMAX || rule > FP4Q_BRUTE_FORCE)
        return FP4Q_ERR_ARG;
    if (gs_mode < FP4Q_GS_NONE || gs_mode > FP4Q_GS_GIVEN)
        return FP4Q_ERR_ARG;
    if (sf_layout == FP4Q_SFLAYOUT_MMA) {
        if (ue5m3 || block != 16 || rows % 128 != 0 || (cols / 16) % 4 != 0)
            return FP4Q_ERR_ARG;
    } else if (sf_layout != FP4Q_SFLAYOUT_ROWMAJOR) {
        return FP4Q_ERR_ARG;
    }
    if (!aligned16(x) || !aligned16(codes) || !aligned_or_null(dequant) ||
        !aligned_or_null(global_scale) || !aligned_or_null(block_mse))
        return FP4Q_ERR_ALIGN;
    cudaStream_t s = as_stream(stream);
    GsArgs gs;
    int st = prepare_gs(gs_mode, ue5m3 ? 6.0f * 114688.0f : 2688.0f, x, dtype, rows * cols, global_scale, workspace,
                        workspace_bytes, s, gs);
    if (st != FP4Q_OK)
        return st;
    unsigned long long* evals =
        (workspace && workspace_bytes >= kQuantWs)
            ? reinterpret_cast<unsigned long long*>(static_cast<uint8_t*>(workspace) + FP4Q_WS_BF_EVALS)
            : nullptr;
    return from_cuda(launch_with_gs(gs, x, dtype, rows * cols, workspace, s, [&](const GsArgs& g) {
        return launch_nvfp4_quant(x, dtype, rows, cols, block, rule, g, codes, scales,
                                  sf_layout == FP4Q_SFLAYOUT_MMA, dequant, block_mse, evals, s, ue5m3 ? 1 : 0);
    }));
}

int nvfp4_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int block, int rule,
                   int gs_mode, float* global_scale, uint8_t* codes, uint8_t* scales,
                   int sf_layout, float* dequant, float* block_mse, void* workspace,
                   size_t workspace_bytes, void* stream)
{
    return fp4_block_quantize(x, dtype, rows, cols, block, rule, FP4Q_SF_E4M3, gs_mode,
                              global_scale, codes, scales, sf_layout, dequant, block_mse, workspace,
                              workspace_bytes, stream);
}

int razer_quantize(const void* x, int dtype, int64_t rows, int64_t cols, int scale_fmt,
                   const float* specials, int n_special, int gs_mode, float* global_scale,
                   uint8_t* codes, uint8_t* meta, float* dequant, float* block_mse,
                   void* workspace, size_t workspace_bytes, void* stream)
{
    const bool empty = rows == 0 || cols == 0;
    if ((!empty && (!x || !codes || !meta)) || !specials || !valid_dtype(dtype) || rows < 0 ||
        cols < 0)
        return FP4Q_ERR_ARG;
    if (cols % 16 != 0)
        return FP4Q_ERR_ARG;
    if (scale_fmt == FP4Q_SF_E3M3) {
        if (n_special < 1 || n_special > 4)
            return FP4Q_ERR_ARG;
    } else if (scale_fmt == FP4Q_SF_E4M3) {
        if (n_special < 1 || n_special > 2)
            return FP4Q_ERR_ARG;
    } else {
        return FP4Q_ERR_ARG;
    }
    for (int i = 0; i < n_special; ++i) {
        const float v = specials[i];
        const float twice = v * 2.0f;
        if (!(std::fabs(v) <= 32.0f) || v == 0.0f || twice != std::nearbyint(twice))
            return FP4Q_ERR_ARG;
    }
    if (gs_mode < FP4Q_GS_NONE || gs_mode > FP4Q_GS_GIVEN)
        return FP4Q_ERR_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned_or_null(dequant) ||
        !aligned_or_null(global_scale) || !aligned_or_null(block_mse))
        return FP4Q_ERR_ALIGN;
    cudaStream_t s = as_stream(stream);
    GsArgs gs;
    const float denom = scale_fmt == FP4Q_SF_E3M3 ? 180.0f : 2688.0f;
    int st = prepare_gs(gs_mode, denom, x, dtype, rows * cols, global_scale, workspace,
                        workspace_bytes, s, gs);
    if (st != FP4Q_OK)
        return st;
    return from_cuda(launch_with_gs(gs, x, dtype, rows * cols, workspace, s, [&](const GsArgs& g) {
        return launch_razer_quant(x, dtype, rows, cols, scale_fmt, specials, n_special, g, codes, meta, dequant,
                                  block_mse, s);
    }));
}

int mxfp4_quantize(const void* x, int dtype, int64_t rows, int64_t cols,
                   const float* chan_scale, int hadamard32, int rule, const float* hess_blocks,
                   uint8_t* codes, uint8_t* scales, float* dequant, float* block_mse,
                   void* stream)
{
    const bool empty = rows == 0 || cols == 0;
    if ((!empty && (!x || !codes || !scales)) || !valid_dtype(dtype) || rows < 0 || cols < 0 ||
        cols % 32 != 0)
        return FP4Q_ERR_ARG;
    if (rule != FP4Q_ABSMAX && rule != FP4Q_HESSIAN_EXP)
        return FP4Q_ERR_ARG;
    if (rule == FP4Q_HESSIAN_EXP && !hess_blocks)
        return FP4Q_ERR_ARG;
    if (!aligned16(x) || !aligned16(codes) || !aligned_or_null(chan_scale) ||
        !aligned_or_null(hess_blocks) || !aligned_or_null(dequant) || !aligned_or_null(block_mse))
        return FP4Q_ERR_ALIGN;
    if (rows == 0 || cols == 0)
        return FP4Q_OK;
    return from_cuda(launch_mxfp4_quant(x, dtype, rows, cols, chan_scale, hadamard32 != 0, rule,
                                        hess_blocks, codes, scales, dequant, block_mse,
                                        as_stream(stream)));
}

int mxfp4_flip_refine(const void* w, int dtype, int64_t rows, int64_t cols, const float* chan_scale,
                      int hadamard32, const float* hess_blocks, int max_moves, uint8_t* codes,
                      const uint8_t* scales, int32_t* moves, void* workspace, size_t workspace_bytes,
                      void* stream)
{
    const bool empty = rows == 0 || cols == 0;
    if ((!empty && (!w || !codes || !scales || !hess_blocks)) || !valid_dtype(dtype) || rows < 0 ||
        cols < 0 || cols % 32 != 0 || max_moves < 0 || max_moves > kFlipMaxMoves)
        return FP4Q_ERR_ARG;
    if (!aligned16(w) || !aligned16(codes) || !aligned_or_null(chan_scale) ||
        !aligned_or_null(hess_blocks) || !aligned_or_null(moves))
        return FP4Q_ERR_ALIGN;
    if (cols > kFlipMaxCols)
        return FP4Q_ERR_UNSUPPORTED;
    if (empty)
        return FP4Q_OK;
    if (!workspace || workspace_bytes < flip_refine_ws_bytes(rows, cols))
        return FP4Q_ERR_WORKSPACE;
    if (!aligned16(workspace))
        return FP4Q_ERR_ALIGN;
    return from_cuda(launch_mxfp4_flip_refine(w, dtype, rows, cols, chan_scale, hadamard32 != 0,
                                              hess_blocks, max_moves, codes, scales, moves, workspace,
                                              as_stream(stream)));
}

int fp4_hessian_blocks(const void* x, int dtype, int64_t rows, int64_t cols,
                       const float* chan_scale, int hadamard32, float* hess_blocks,
                       void* workspace, size_t workspace_bytes, void* stream)
{
    if (!x || !hess_blocks || !valid_dtype(dtype) || rows < 0 || cols < 0 || cols % 32 != 0)
        return FP4Q_ERR_ARG;
    if (!aligned16(x) || !aligned16(hess_blocks) || !aligned_or_null(chan_scale))
        return FP4Q_ERR_ALIGN;
    if (cols == 0)
        return FP4Q_OK;
    const size_t need = kHessHeader + hessian_ws_bytes(rows, cols);
    if (!workspace || workspace_bytes < need)
        return FP4Q_ERR_WORKSPACE;
    if (!aligned16(workspace))
        return FP4Q_ERR_ALIGN;
    cudaStream_t s = as_stream(stream);
    int* err = static_cast<int*>(workspace);
    if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess)
        return FP4Q_ERR_CUDA;
    if (rows == 0)
        return from_cuda(cudaMemsetAsync(hess_blocks, 0, (size_t)(cols / 32) * 1024 * sizeof(float), s));
    float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kHessHeader);
    return from_cuda(launch_hessian_blocks(x, dtype, rows, cols, chan_scale, hadamard32 != 0,
                                           hess_blocks, part, err, s));
}

int mxfp4_channel_scale(const void* x, int x_dtype, int64_t tokens, const void* w,
                        int w_dtype, int64_t n_out, int64_t cols, float alpha, float* t,
                        float* t_inv, void* workspace, size_t workspace_bytes, void* stream)
{
    if (!x || !w || !t || !valid_dtype(x_dtype) || !valid_dtype(w_dtype))
        return FP4Q_ERR_ARG;
    if (tokens <= 0 || n_out <= 0 || cols <= 0 || cols % 8 != 0 || !(std::isfinite(alpha)))
        return FP4Q_ERR_ARG;
    if (!aligned16(x) || !aligned16(w) || !aligned16(t) || !aligned_or_null(t_inv))
        return FP4Q_ERR_ALIGN;
    const size_t need = channel_scale_ws_bytes(tokens, n_out, cols);
    if (!workspace || workspace_bytes < need)
        return FP4Q_ERR_WORKSPACE;
    if (!aligned16(workspace))
        return FP4Q_ERR_ALIGN;
    return from_cuda(launch_mx_channel_scale(x, x_dtype, tokens, w, w_dtype, n_out, cols, alpha, t,
                                             t_inv, workspace, as_stream(stream)));
}

int fp4_dequant_mse(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                    int block, int scale_fmt, const float* specials, int n_special,
                    const float* global_scale, const void* ref, int ref_dtype, float* dequant,
                    float* block_mse, void* stream)
{
    const bool empty = rows == 0 || cols == 0;
    if ((!empty && (!codes || !scales)) || rows < 0 || cols < 0 || !valid_block(block) ||
        cols % block != 0)
        return FP4Q_ERR_ARG;
    if (scale_fmt < FP4Q_SF_E4M3 || scale_fmt > FP4Q_SF_UE5M3)
        return FP4Q_ERR_ARG;
    if (scale_fmt == FP4Q_SF_UE5M3 && specials)
        return FP4Q_ERR_ARG;
    if (scale_fmt == FP4Q_SF_E8M0 && (block != 32 || specials))
        return FP4Q_ERR_ARG;
    if (specials) {
        if (block != 16 || n_special < 1 || n_special > (scale_fmt == FP4Q_SF_E3M3 ? 4 : 2))
            return FP4Q_ERR_ARG;
    }
    if (block_mse && !ref && !empty)
        return FP4Q_ERR_ARG;
    if (ref && !valid_dtype(ref_dtype))
        return FP4Q_ERR_ARG;
    if (!aligned16(codes) || !aligned_or_null(ref) || !aligned_or_null(dequant) ||
        !aligned_or_null(block_mse) || !aligned_or_null(global_scale))
        return FP4Q_ERR_ALIGN;
    if (rows == 0 || cols == 0)
        return FP4Q_OK;
    return from_cuda(launch_dequant_mse(codes, scales, rows, cols, block, scale_fmt, specials,
                                        specials ? n_special : 0, global_scale, ref, ref_dtype,
                                        dequant, block_mse, as_stream(stream)));
}

int w4a4_gemm(const void* a, int a_format, int a_rule, const uint8_t* a_scales,
              const float* a_global_scale, const uint8_t* w_codes, const uint8_t* w_scales,
              const float* w_global_scale, int64_t M, int64_t N, int64_t K, void* out,
              int out_dtype, void* workspace, size_t workspace_bytes, void* stream)
{
    if (!a || !w_codes || !w_scales || !w_global_scale || !out || !workspace || !valid_out_dtype(out_dtype))
        return FP4Q_ERR_ARG;
    if (a_format != FP4Q_F32 && a_format != FP4Q_BF16 && a_format != FP4Q_NVFP4_PACKED)
        return FP4Q_ERR_ARG;
    if (a_format == FP4Q_NVFP4_PACKED && (!a_scales || !a_global_scale))
        return FP4Q_ERR_ARG;
    if (a_format != FP4Q_NVFP4_PACKED && (a_rule < FP4Q_ABSMAX || a_rule > FP4Q_BRUTE_FORCE))
        return FP4Q_ERR_ARG;
    if (M <= 0 || N <= 0 || K <= 0)
        return FP4Q_ERR_ARG;
    if (!gemm_shape_supported(M, N, K))
        return FP4Q_ERR_UNSUPPORTED;
    if (!aligned16(a) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(out) ||
        !aligned16(workspace) || !aligned_or_null(a_scales) || !aligned16(w_global_scale) ||
        !aligned_or_null(a_global_scale))
        return FP4Q_ERR_ALIGN;
    const size_t need = a_format == FP4Q_NVFP4_PACKED ? kGemmHeader : gemm_ws_bytes(M, K);
    if (workspace_bytes < need)
        return FP4Q_ERR_WORKSPACE;
    cudaStream_t s = as_stream(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int* err = reinterpret_cast<int*>(ws + kGemmErr);
    if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess)
        return FP4Q_ERR_CUDA;
    const uint8_t* a_codes = static_cast<const uint8_t*>(a);
    const uint8_t* a_sf = a_scales;
    const float* ga = a_global_scale;
    if (a_format != FP4Q_NVFP4_PACKED) {
        uint8_t* qcodes = ws + kGemmHeader;
        uint8_t* qsf = qcodes + (size_t)M * (size_t)K / 2;
        float* g = reinterpret_cast<float*>(ws + kGemmGa);
        GsArgs gs{};
        gs.denom = 2688.0f;
        gs.out = g;
        cudaError_t e = fused_gs(gs, a, M * K, ws, kGemmFused, kGemmCounter, s);
        if (e == cudaSuccess)
            e = launch_with_gs(gs, a, a_format, M * K, ws, s, [&](const GsArgs& gg) {
                return launch_nvfp4_quant(a, a_format, M, K, 16, a_rule, gg, qcodes, qsf, 1, nullptr, nullptr,
                                          nullptr, s);
            });
        if (e != cudaSuccess)
            return FP4Q_ERR_CUDA;
        a_codes = qcodes;
        a_sf = qsf;
        ga = g;
    }
    return from_cuda(launch_w4a4_gemm(a_codes, a_sf, ga, w_codes, w_scales, w_global_scale, M, N, K,
                                      out, out_dtype == FP4Q_F32, err, s));
}

int fp4q_gemm_status(const void* workspace, void* stream)
{
    if (!workspace)
        return FP4Q_ERR_ARG;
    int flag = 0;
    cudaStream_t s = as_stream(stream);
    if (cudaMemcpyAsync(&flag, static_cast<const uint8_t*>(workspace) + kGemmErr, sizeof(int),
                        cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return FP4Q_ERR_CUDA;
    return flag ? FP4Q_ERR_TIMEOUT : FP4Q_OK;
}

int fp4q_mma_ceiling(int mx, int iters, int* err, void* stream)
{
    if (!err || iters < 1 || iters > (1 << 20) || (mx != 0 && mx != 1))
        return FP4Q_ERR_ARG;
    if ((reinterpret_cast<uintptr_t>(err) & 3u) != 0)
        return FP4Q_ERR_ALIGN;
    return from_cuda(launch_mma_ceiling(mx, iters, err, as_stream(stream)));
}

double fp4q_mma_ceiling_flops(int iters)
{
    return iters < 1 ? 0.0 : (double)mma_ceiling_pairs() * (double)iters * 4.0 * 2.0 * 256.0 * 256.0 * 64.0;
}

int fp4q_hessian_status(const void* workspace, void* stream)
{
    // NULL: the error word of fp4_hessian_blocks_noalloc on the current device
    const void* word = workspace ? workspace : noalloc_hessian_error_word();
    if (!word)
        return FP4Q_ERR_CUDA;
    int flag = 0;
    cudaStream_t s = as_stream(stream);
    if (cudaMemcpyAsync(&flag, word, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return FP4Q_ERR_CUDA;
    return flag ? FP4Q_ERR_TIMEOUT : FP4Q_OK;
}

// E2M1 codes (p, q) with value(p) + value(q) == v exactly: p the largest
// magnitude of the special's sign that leaves an E2M1 remainder.  False when
// no such pair exists.
static bool split_special(float v, uint8_t* p, uint8_t* q)
{
    static const float kMag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};
    const uint8_t sign = v < 0.0f ? 8u : 0u;
    const float m = std::fabs(v);
    for (int i = 7; i >= 1; --i) {
        if (kMag[i] > m)
            continue;
        const float r = m - kMag[i];
        for (int j = 0; j < 8; ++j) {
            if (kMag[j] == r) {
                *p = (uint8_t)(sign | i);
                *q = (uint8_t)(j == 0 ? 0 : (sign | j));
                return true;
            }
        }
    }
    return false;
}

int razer_gemm_prepare(const uint8_t* codes, const uint8_t* meta, int64_t rows, int64_t cols,
                       int scale_fmt, const float* specials, int n_special, uint8_t* main_codes,
                       uint8_t* extra_codes, uint8_t* scales_mma, void* stream)
{
    const bool empty = rows == 0 || cols == 0;
    if (rows < 0 || cols < 0 || !specials)
        return FP4Q_ERR_ARG;
    if (!empty && (!codes || !meta || !main_codes || !extra_codes || !scales_mma))
        return FP4Q_ERR_ARG;
    if (scale_fmt == FP4Q_SF_E3M3) {
        if (n_special < 1 || n_special > 4)
            return FP4Q_ERR_ARG;
    } else if (scale_fmt == FP4Q_SF_E4M3) {
        if (n_special < 1 || n_special > 2)
            return FP4Q_ERR_ARG;
    } else {
        return FP4Q_ERR_ARG;
    }
    uint8_t pc[4] = {0, 0, 0, 0}, qc[4] = {0, 0, 0, 0};
    for (int i = 0; i < n_special; ++i) {
        const float v = specials[i];
        const float twice = v * 2.0f;
        if (!(std::fabs(v) <= 32.0f) || v == 0.0f || twice != std::nearbyint(twice))
            return FP4Q_ERR_ARG;
        if (!split_special(v, &pc[i], &qc[i]))
            return FP4Q_ERR_UNSUPPORTED;
    }
    if (rows % 128 != 0 || cols % 64 != 0)
        return FP4Q_ERR_ARG;
    if (!aligned_or_null(codes) || !aligned_or_null(main_codes) || !aligned_or_null(extra_codes))
        return FP4Q_ERR_ALIGN;
    if (empty)
        return FP4Q_OK;
    return from_cuda(launch_razer_gemm_prepare(codes, meta, rows, cols, scale_fmt, pc, qc, main_codes,
                                               extra_codes, scales_mma, as_stream(stream)));
}

int razer_w4a4_gemm(const uint8_t* a_codes, const uint8_t* a_extra, const uint8_t* a_scales,
                    const float* a_global_scale, const uint8_t* w_codes, const uint8_t* w_extra,
                    const uint8_t* w_scales, const float* w_global_scale, int64_t M, int64_t N,
                    int64_t K, void* out, int out_dtype, void* workspace, size_t workspace_bytes, void* stream)
{
    if (!a_codes || !a_scales || !a_global_scale || !w_codes || !w_scales || !w_global_scale || !out ||
        !workspace || !valid_out_dtype(out_dtype))
        return FP4Q_ERR_ARG;
    if (M <= 0 || N <= 0 || K <= 0)
        return FP4Q_ERR_ARG;
    if (!gemm_shape_supported(M, N, K))
        return FP4Q_ERR_UNSUPPORTED;
    if (!aligned16(a_codes) || !aligned_or_null(a_extra) || !aligned16(a_scales) || !aligned16(w_codes) ||
        !aligned_or_null(w_extra) || !aligned16(w_scales) || !aligned16(out) || !aligned16(workspace) ||
        !aligned16(a_global_scale) || !aligned16(w_global_scale))
        return FP4Q_ERR_ALIGN;
    if (workspace_bytes < kGemmHeader)
        return FP4Q_ERR_WORKSPACE;
    cudaStream_t s = as_stream(stream);
    int* err = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) + kGemmErr);
    if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess)
        return FP4Q_ERR_CUDA;
    return from_cuda(launch_w4a4_gemm(a_codes, a_scales, a_global_scale, w_codes, w_scales, w_global_scale,
                                      M, N, K, out, out_dtype == FP4Q_F32, err, s, a_extra, w_extra));
}

int fp4_scales_to_mma(const uint8_t* scales, int64_t rows, int64_t nscales, uint8_t* out, void* stream)
{
    if (rows < 0 || nscales < 0 || rows % 128 != 0 || nscales % 4 != 0)
        return FP4Q_ERR_ARG;
    if (rows == 0 || nscales == 0)
        return FP4Q_OK;
    if (!scales || !out)
        return FP4Q_ERR_ARG;
    if (!aligned16(scales) || !aligned16(out))
        return FP4Q_ERR_ALIGN;
    return from_cuda(launch_scales_to_mma(scales, rows, nscales, out, as_stream(stream)));
}

int mxfp4_gemm(const void* a, int a_format, const uint8_t* a_scales, const float* chan_scale,
               int hadamard32, const uint8_t* w_codes, const uint8_t* w_scales, int64_t M, int64_t N,
               int64_t K, void* out, int out_dtype, void* workspace, size_t workspace_bytes, void* stream)
{
    if (!a || !w_codes || !w_scales || !out || !workspace || !valid_out_dtype(out_dtype))
        return FP4Q_ERR_ARG;
    if (a_format != FP4Q_F32 && a_format != FP4Q_BF16 && a_format != FP4Q_MXFP4_PACKED)
        return FP4Q_ERR_ARG;
    if (a_format == FP4Q_MXFP4_PACKED && (!a_scales || chan_scale))
        return FP4Q_ERR_ARG;
    if (M <= 0 || N <= 0 || K <= 0)
        return FP4Q_ERR_ARG;
    if (!gemm_shape_supported(M, N, K))
        return FP4Q_ERR_UNSUPPORTED;
    if (!aligned16(a) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(out) ||
        !aligned16(workspace) || !aligned_or_null(a_scales) || !aligned_or_null(chan_scale))
        return FP4Q_ERR_ALIGN;
    const size_t need = a_format == FP4Q_MXFP4_PACKED ? kGemmHeader : mx_gemm_ws_bytes(M, K);
    if (workspace_bytes < need)
        return FP4Q_ERR_WORKSPACE;
    cudaStream_t s = as_stream(stream);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int* err = reinterpret_cast<int*>(ws + kGemmErr);
    if (cudaMemsetAsync(err, 0, sizeof(int), s) != cudaSuccess)
        return FP4Q_ERR_CUDA;
    const uint8_t* a_codes = static_cast<const uint8_t*>(a);
    const uint8_t* a_sf = a_scales;
    if (a_format != FP4Q_MXFP4_PACKED) {
        // the prologue: u = a * t, block rotation, E8M0 quantization, scales
        // written straight into the GEMM's layout
        uint8_t* qcodes = ws + kGemmHeader;
        uint8_t* qsf = qcodes + (size_t)M * (size_t)K / 2;
        if (launch_mxfp4_quant(a, a_format, M, K, chan_scale, hadamard32 != 0, FP4Q_ABSMAX, nullptr, qcodes,
                               qsf, nullptr, nullptr, s, 1) != cudaSuccess)
            return FP4Q_ERR_CUDA;
        a_codes = qcodes;
        a_sf = qsf;
    }
    return from_cuda(launch_w4a4_gemm(a_codes, a_sf, nullptr, w_codes, w_scales, nullptr, M, N, K, out,
                                      out_dtype == FP4Q_F32, err, s, nullptr, nullptr, 1,
                                      a_format != FP4Q_MXFP4_PACKED));
}

}  // extern "C"
